"""GPU parity of decoding over the "FP8 with scale" KV cache.

The cache format is the upstream FlashMLA documentation's ("FP8 KV Cache"):
656-byte token rows of 512 float8_e4m3 latent values, 4 float32 scales (one per
128 values) and 64 bfloat16 RoPE values; the kernel dequantizes to bfloat16 and
computes as for a bfloat16 cache.  Each case runs through the C ABI and is
compared element by element with the FP64 oracle (which dequantizes the same
bytes itself) under the tolerances of the 16-bit path.  The cases span ragged
page tails with NaN in every never-visible byte, causal masks that leave rows
empty, one to three row groups, split sequences (combine), padding heads, few
partitions, and rows fewer than one TMA box.
"""
import numpy as np
import pytest
import torch

import mla_decode_attention_12_b200 as mla
from mla_decode_attention_12_b200 import workloads as W
from tests.gpu_helpers import compare, oracle_full, run_gpu, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_decode_attention_12_b200 import build
    build.build()


def fp8(seqlens, **kw):
    return W.make_problem(seqlens, fp8_kv=True, **kw)


CASES = {
    "tiny": lambda: fp8([256, 193], s_q=1, h_q=16, seed=201),
    "compute_like": lambda: fp8([1000, 3000, 64, 65, 1], s_q=1, h_q=128, seed=202),
    "ragged_poison": lambda: fp8([700, 65, 3, 129, 0, 64], s_q=2, h_q=32, causal=True, seed=203, poison=True,
                                 extra_pages=5),
    "long_split_like": lambda: fp8([20000, 7000, 3000, 100], s_q=1, h_q=128, seed=204, poison=True),
    "rows256_two_groups": lambda: fp8([1500, 640], s_q=2, h_q=128, causal=True, seed=205),
    "rows384_three_groups": lambda: fp8([400, 90], s_q=3, h_q=128, seed=206),
    "one_head": lambda: fp8([5000, 17], s_q=1, h_q=1, seed=207),
    "empty_and_short": lambda: fp8([0, 1, 2, 0, 63, 64], s_q=4, h_q=16, causal=True, seed=208),
    "large_logits": lambda: fp8([2000, 700], s_q=1, h_q=128, seed=209, scale=0.3),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_parity(oracle_mod, name):
    p = CASES[name]()
    o, lse, md, ns = run_gpu(p)
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, f"fp8 {name}"))


@pytest.mark.parametrize("parts", [1, 3])
def test_fp8_few_partitions(oracle_mod, parts):
    p = fp8([2500, 64, 0, 700, 1, 130], s_q=2, h_q=64, causal=True, seed=210 + parts, poison=True)
    o, lse, md, ns = run_gpu(p, num_parts=parts)
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, f"fp8 parts={parts}"))


def test_fp8_active_heads(oracle_mod):
    p = fp8([300, 420, 511, 129, 64, 2], s_q=2, h_q=64, causal=True, active_heads=16, seed=212)
    q, kv, bt, sl = to_device(p)
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1, is_fp8_kvcache=True)
    o = torch.full((p.batch, p.s_q, p.h_q, 512), 7.0, dtype=q.dtype, device="cuda")
    lse = torch.full((p.batch, p.s_q, p.h_q), 7.0, dtype=torch.float32, device="cuda")
    mla.flash_mla_with_kvcache(q, kv, bt, sl, p.dv, md, ns, causal=True, softmax_scale=p.scale, out=o, lse=lse,
                               active_heads=16, is_fp8_kvcache=True)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o[:, :, :16].contiguous(), lse[:, :, :16].contiguous(), o_ref[:, :, :16], lse_ref[:, :, :16],
                  p.dtype, "fp8 active heads"))
    assert bool((o[:, :, 16:] == 7.0).all()) and bool((lse[:, :, 16:] == 7.0).all())


def test_fp8_matches_bf16_cache_of_dequantized_rows(oracle_mod):
    # The FP8 kernel on a cache and the bfloat16 kernel on the oracle's dequantization of
    # the same cache compute the same thing; their outputs agree to the bfloat16 path's own
    # accuracy (not bit for bit: the two kernels order their work differently).
    p = fp8([900, 2000, 65], s_q=2, h_q=64, causal=True, seed=213)
    o8, l8, _, _ = run_gpu(p)
    pb = W.Problem(name="dequantized", q=p.q, kvcache=oracle_mod.dequant_fp8(p.kvcache), block_table=p.block_table,
                   cache_seqlens=p.cache_seqlens, dtype=W.BF16, causal=True, scale=p.scale)
    o16, l16, _, _ = run_gpu(pb)
    assert (o8.float() - o16.float()).abs().max().item() <= 2e-2
    assert (l8 - l16).abs().max().item() <= 1e-2


def test_fp8_two_stage_calls_match_single_call():
    p = CASES["long_split_like"]()
    o1, lse1, md, ns = run_gpu(p)
    q, kv, bt, sl = to_device(p)
    call = mla.DecodeCall(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale, is_fp8_kvcache=True)
    call.splitkv()
    call.combine()
    torch.cuda.synchronize()
    assert int(ns[-1].item()) > ns.numel() - 1, "the case must split some sequence"
    assert torch.equal(call.out, o1) and torch.equal(call.lse, lse1)


def test_fp8_repeat_calls_are_deterministic():
    p = CASES["compute_like"]()
    o1, l1, _, _ = run_gpu(p)
    o2, l2, _, _ = run_gpu(p)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fp8_host_buffers_end_to_end(oracle_mod):
    # pinned host tensors through the public call: copied in, decoded, copied back
    p = fp8([700, 64], s_q=2, h_q=16, causal=True, seed=214)
    q, kv, bt, sl = (t.cpu().pin_memory() for t in to_device(p))
    md, ns = mla.get_mla_metadata(sl.cuda(), p.s_q * p.h_q, 1, is_fp8_kvcache=True)
    o, lse = mla.flash_mla_with_kvcache(q, kv, bt, sl, 512, md.cpu(), ns.cpu(), causal=True, softmax_scale=p.scale,
                                        is_fp8_kvcache=True)
    assert not o.is_cuda and kv.dtype == torch.uint8
    o_ref, lse_ref = oracle_full(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, "fp8 host buffers"))
