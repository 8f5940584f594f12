"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before touching the GPU (runs without a GPU)."""
import ctypes
import os
import re

import pytest

from mla_decode_attention_12_b200 import _lib, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "mla_decode.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MLA_API\s+[\w\s\*]*?\b(mla_\w+)\s*\(", text)))


def test_header_declares_the_api():
    names = declared_functions()
    for must in ("mla_get_metadata", "mla_decode_with_kvcache", "mla_decode_workspace_bytes"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(7):
        assert _lib.status_string(code)
    assert _lib.status_string(99) == "unknown status"


def test_sizes(lib):
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.mla_metadata_sizes(64, 128, 1, 74, ctypes.byref(a), ctypes.byref(b)) == 0
    assert (a.value, b.value) == (74 * 8, 64 + 1)
    assert lib.mla_metadata_sizes(32, 256, 1, 74, ctypes.byref(a), ctypes.byref(b)) == 0
    assert b.value == 32 * 2 + 1
    assert lib.mla_metadata_sizes(-1, 128, 1, 74, ctypes.byref(a), ctypes.byref(b)) == 1
    # workspace: a control block of fixed size (status word + 2 int32 counters for each of
    # up to 16384 virtual batches), then (NV + parts) * 128 * (2 + 512) floats
    nv, parts = 64, 74
    control = 256 + 2 * 4 * 16384
    # split LSEs and split maxima (one float per slot row each), then the split partial outputs
    want = control + 2 * (((nv + parts) * 128 * 4 + 255) // 256 * 256) + (nv + parts) * 128 * 512 * 4
    assert lib.mla_decode_workspace_bytes(64, 1, 128, 1, 74) == want
    # the same control block for every problem size, so calls of different sizes can share
    # one workspace without one call's partials landing on another's counters
    for sizes in ((64, 1, 128, 1), (4, 1, 128, 1), (1, 1, 16, 1), (8192, 2, 128, 1)):
        assert lib.mla_decode_workspace_zero_bytes(*sizes) == control
    assert lib.mla_decode_workspace_bytes(64, 0, 128, 1, 74) == 0
    # more virtual batches (requests x row groups of 128 query rows) than the control block holds
    assert lib.mla_decode_workspace_bytes(16384, 1, 128, 1, 74) > 0
    assert lib.mla_decode_workspace_bytes(16385, 1, 128, 1, 74) == 0
    assert lib.mla_decode_workspace_bytes(8193, 2, 128, 1, 74) == 0


def _decode(lib, **over):
    fake = 1 << 20  # aligned non-null "device" pointers: validation must reject before any use
    args = dict(q=fake, batch=2, s_q=1, h_q=16, d_qk=576, kvcache=fake, num_blocks=8, page_size=64, h_kv=1,
                block_table=fake, max_blocks=4, seqlens=fake, dv=512, dtype=0, md=fake, num_parts=74,
                num_splits=fake, causal=0, scale=0.0, active_heads=0, o=fake, lse=fake, ws=fake,
                ws_bytes=1 << 40, stream=None)
    args.update(over)
    return lib.mla_decode_with_kvcache(*args.values())


@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(ws=None), 1), (dict(block_table=None), 1),
    (dict(batch=-1), 1), (dict(s_q=0), 1), (dict(h_q=0), 1), (dict(num_blocks=0), 1),
    (dict(causal=2), 1), (dict(dtype=7), 1), (dict(q=(1 << 20) + 2), 1), (dict(ws=(1 << 20) + 16), 1),
    (dict(page_size=32), 2), (dict(h_kv=2), 2), (dict(d_qk=192), 2), (dict(dv=256), 2),
    (dict(ws_bytes=1000), 3), (dict(batch=16385, h_q=128), 2),
    # the "FP8 with scale" cache (dtype 2) carries 64 RoPE values: d_qk must be 576
    (dict(dtype=2, d_qk=512), 2), (dict(dtype=2, kvcache=(1 << 20) + 8), 1), (dict(dtype=3), 1),
])
def test_decode_rejects_bad_arguments(lib, over, code):
    assert _decode(lib, **over) == code


def test_decode_empty_batch_is_a_no_op(lib):
    assert _decode(lib, batch=0, q=None, o=None) == 0
    assert _decode(lib, batch=0, q=None, o=None, dtype=2) == 0


def test_combine_accepts_the_fp8_cache_dtype(lib):
    # mla_decode_combine of an FP8-cache call writes bfloat16 o: dtype 2 is valid there too
    # (checked with an empty batch, which enqueues nothing).
    fake = 1 << 20
    assert lib.mla_decode_combine(0, 1, 16, 1, 512, 2, fake, 74, 0, fake, fake, fake, 1 << 30, None) == 0
    assert lib.mla_decode_combine(0, 1, 16, 1, 512, 3, fake, 74, 0, fake, fake, fake, 1 << 30, None) == 1


def test_status_reads_reject_null_outputs(lib):
    assert lib.mla_read_noalloc_status(0, None, None) == 1
    assert lib.mla_read_device_status(None, 0, None, None) == 1


def test_metadata_rejects_bad_arguments(lib):
    fake = 1 << 20
    assert lib.mla_get_metadata(fake, 4, 0, 1, 74, 0, fake, fake, None) == 1
    assert lib.mla_get_metadata(fake, 4, 128, 2, 74, 0, fake, fake, None) == 2
    assert lib.mla_get_metadata(fake, 4, 128, 1, 0, 1, fake, fake, None) == 1
    assert lib.mla_get_metadata(None, 4, 128, 1, 74, 0, fake, fake, None) == 1


def test_host_metadata_rejects_negative_lengths(lib):
    import numpy as np

    sl = np.array([5, -1], np.int32)
    md = np.zeros(74 * 8, np.int32)
    ns = np.zeros(3, np.int32)
    assert lib.mla_get_metadata_host(sl.ctypes.data, 2, 16, 1, 74, 0, md.ctypes.data, ns.ctypes.data) == 1


@pytest.mark.parametrize("case", ["fp16_q", "bf16_cache", "row_bytes", "d_qk_512", "mixed_16bit"])
def test_binding_rejects_mismatched_cache_formats(case):
    # The Python binding checks dtypes and row widths before it touches the library or a GPU.
    import torch

    from mla_decode_attention_12_b200 import api

    q = torch.zeros(1, 1, 16, 576, dtype=torch.bfloat16)
    kv = torch.zeros(2, 64, 1, 656, dtype=torch.uint8)
    fp8 = True
    if case == "fp16_q":
        q = q.half()
    elif case == "bf16_cache":
        kv = torch.zeros(2, 64, 1, 576, dtype=torch.bfloat16)
    elif case == "row_bytes":
        kv = torch.zeros(2, 64, 1, 576, dtype=torch.uint8)
    elif case == "d_qk_512":
        q = torch.zeros(1, 1, 16, 512, dtype=torch.bfloat16)
    else:  # a 16-bit call whose cache has another dtype
        kv = torch.zeros(2, 64, 1, 576, dtype=torch.float16)
        fp8 = False
    bt = torch.zeros(1, 2, dtype=torch.int32)
    sl = torch.ones(1, dtype=torch.int32)
    md = torch.zeros(74, 8, dtype=torch.int32)
    ns = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError):
        api.DecodeCall(q, kv, bt, sl, 512, md, ns, is_fp8_kvcache=fp8)


def _sparse(lib, **over):
    fake = 1 << 20
    args = dict(q=fake, batch=2, s_q=1, h_q=16, d_qk=576, kvcache=fake, num_blocks=8, page_size=64, h_kv=1,
                indices=fake, topk=128, dv=512, dtype=2, md=fake, num_parts=74, num_splits=fake, scale=0.0,
                active_heads=0, o=fake, lse=fake, ws=fake, ws_bytes=1 << 40, stream=None)
    args.update(over)
    return lib.mla_decode_sparse(*args.values())


@pytest.mark.parametrize("over,code", [
    (dict(indices=None), 1), (dict(topk=-1), 1), (dict(s_q=0), 1), (dict(batch=-1), 1),
    (dict(dtype=7), 1), (dict(d_qk=512), 2), (dict(page_size=32), 2), (dict(h_kv=2), 2),
    (dict(ws_bytes=1000), 3), (dict(kvcache=(1 << 20) + 8), 1),
])
def test_sparse_decode_rejects_bad_arguments(lib, over, code):
    # Bad lists, sizes or formats are rejected on the host before a launch.
    assert _sparse(lib, **over) == code


def test_sparse_metadata_rejects_bad_arguments(lib):
    fake = 1 << 20
    assert lib.mla_get_metadata_sparse(4, -1, 128, 1, 74, fake, fake, None) == 1
    assert lib.mla_get_metadata_sparse(4, 64, 0, 1, 74, fake, fake, None) == 1
    assert lib.mla_get_metadata_sparse(4, 64, 128, 2, 74, fake, fake, None) == 2
    assert lib.mla_get_metadata_sparse(4, 64, 128, 1, 0, fake, fake, None) == 1


def test_sparse_prefill_rejects_bad_arguments(lib):
    fake = 1 << 20
    base = dict(q=fake, s_q=4, h_q=128, d_qk=576, kv=fake, s_kv=1000, h_kv=1, indices=fake, topk=64, dv=512, dtype=0,
                sm_scale=0.0, md=fake, num_parts=74, ns=fake, out=fake, max_logits=fake, lse=fake, ws=fake,
                ws_bytes=1 << 40, stream=None)

    def call(**over):
        a = dict(base)
        a.update(over)
        return lib.mla_sparse_prefill(*a.values())

    assert call(dtype=2) == 2           # an FP8 cache is the sparse decode's, not the prefill's
    assert call(dtype=5) == 1
    assert call(indices=None) == 1 and call(max_logits=None) == 1
    assert call(s_kv=0) == 1 and call(topk=-1) == 1 and call(s_q=-1) == 1
    assert call(d_qk=512) == 2 and call(h_kv=2) == 2 and call(dv=256) == 2
    assert call(ws_bytes=100) == 3
    assert call(s_q=0, q=None, out=None) == 0


def test_python_calls_take_the_documented_positional_order():
    # upstream FlashMLA documentation, "Usage / MLA Decoding":
    #   get_mla_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv, h_q, is_fp8, topk)
    #   flash_mla_with_kvcache(q, kvcache, block_table, cache_seqlens, dv, tile_scheduler_metadata,
    #                          num_splits, is_causal, is_fp8_kvcache, indices)
    import inspect

    import mla_decode_attention_12_b200 as mla

    def positional(fn):
        return [p.name for p in inspect.signature(fn).parameters.values()
                if p.kind in (p.POSITIONAL_ONLY, p.POSITIONAL_OR_KEYWORD)]

    assert positional(mla.get_mla_metadata) == ["cache_seqlens", "heads_per_kv", "h_kv", "h_q", "is_fp8_kvcache",
                                                "topk"]
    assert positional(mla.flash_mla_with_kvcache) == ["q", "kvcache", "block_table", "cache_seqlens", "dv",
                                                      "tile_scheduler_metadata", "num_splits", "causal",
                                                      "is_fp8_kvcache", "indices"]
    assert positional(mla.flash_mla_sparse_fwd)[:4] == ["q", "kv", "indices", "sm_scale"]
