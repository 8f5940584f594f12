"""The allocation-free decode entry point gives the same results as the regular one.

mla_decode_with_kvcache_noalloc is for callers that cannot allocate device
memory at decode time (pre-planned runtimes, plugins that only receive tensor
pointers, allocation-free latency paths): it keeps its split-KV scratch in a
fixed array inside the library instead of a caller-provided workspace.  This
test calls it through the C ABI several times in a row, on different problems
whose sequences are split across partitions (so the scratch holds partial
results), and checks that each output is bit-identical to
mla_decode_with_kvcache run on a torch-allocated workspace (both run the same
kernels on the same inputs with the same workspace layout), and that the
scratch's device status reads MLA_OK after each call.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import mla_decode_attention_12_b200 as mla
from mla_decode_attention_12_b200 import _lib
from mla_decode_attention_12_b200 import workloads as W

pytestmark = pytest.mark.gpu

@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_decode_attention_12_b200 import build

    build.build()
    return _lib.load()


def _device_problem(p):
    dt = torch.bfloat16 if p.dtype == W.BF16 else torch.float16
    q = torch.from_numpy(p.q.view(np.int16)).view(dt).cuda()
    kv = (torch.from_numpy(p.kvcache) if p.fp8_kv else torch.from_numpy(p.kvcache.view(np.int16)).view(dt)).cuda()
    bt = torch.from_numpy(p.block_table).cuda()
    sl = torch.from_numpy(p.cache_seqlens).cuda()
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1)
    return q, kv, bt, sl, md, ns


def _args(p, q, kv, bt, sl, md, ns, o, lse):
    return (q.data_ptr(), p.batch, p.s_q, p.h_q, p.d_qk, kv.data_ptr(), p.num_blocks, 64, 1, bt.data_ptr(),
            bt.shape[1], sl.data_ptr(), 512, 2 if p.fp8_kv else p.dtype, md.data_ptr(), md.shape[0], ns.data_ptr(),
            int(p.causal),
            p.scale, 0, o.data_ptr(), lse.data_ptr())


def _regular(lib, p, t):
    q, kv, bt, sl, md, ns = t
    o = torch.empty(p.batch, p.s_q, p.h_q, 512, dtype=q.dtype, device="cuda")
    lse = torch.empty(p.batch, p.s_q, p.h_q, dtype=torch.float32, device="cuda")
    nbytes = mla.workspace_bytes(p.batch, p.s_q, p.h_q, 1, md.shape[0])
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert lib.mla_decode_with_kvcache(*_args(p, q, kv, bt, sl, md, ns, o, lse), ws.data_ptr(), nbytes, st) == 0
    torch.cuda.synchronize()
    return o, lse


def _noalloc(lib, p, t):
    q, kv, bt, sl, md, ns = t
    o = torch.full((p.batch, p.s_q, p.h_q, 512), float("nan"), dtype=q.dtype, device="cuda")
    lse = torch.full((p.batch, p.s_q, p.h_q), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert lib.mla_decode_with_kvcache_noalloc(*_args(p, q, kv, bt, sl, md, ns, o, lse), st) == 0
    status = ctypes.c_int(-1)
    assert lib.mla_read_noalloc_status(0, ctypes.byref(status), st) == 0  # synchronises the stream
    assert status.value == 0, f"device status {status.value} after an allocation-free call"
    return o, lse


def test_noalloc_matches_regular_on_two_calls(lib):
    problems = [
        W.make_problem([20000, 7000, 3000, 100], s_q=1, h_q=128, seed=901),
        W.make_problem([2500, 64, 700, 1, 4100], s_q=2, h_q=64, causal=True, seed=902),
        W.make_problem([20000, 3000, 100], s_q=1, h_q=128, seed=903, fp8_kv=True),  # "FP8 with scale" cache
    ]
    # a larger problem after a smaller one, then the first again: the scratch is shared
    for p in problems + problems[:1]:
        t = _device_problem(p)
        assert int(t[5][-1]) > p.batch * ((p.s_q * p.h_q + 127) // 128), "no sequence was split"
        o_ref, lse_ref = _regular(lib, p, t)
        o, lse = _noalloc(lib, p, t)
        assert torch.isfinite(o).all()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    # 4096 requests of 128 rows need far more than the fixed scratch: rejected on the
    # host with MLA_ERR_WORKSPACE before anything is enqueued.
    fake = 1 << 20
    rc = lib.mla_decode_with_kvcache_noalloc(fake, 4096, 1, 128, 576, fake, 4096, 64, 1, fake, 1, fake, 512, 0,
                                             fake, 74, fake, 0, 0.0, 0, fake, fake, None)
    assert rc == 3
