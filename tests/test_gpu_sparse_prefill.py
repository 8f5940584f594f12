"""GPU parity of the sparse MLA prefill (upstream FlashMLA documentation, "Sparse MLA Prefill":
out, base-2 max_logits and base-2 lse) against the oracle's ``sparse_prefill``, and of the
token-level sparse decode over a 16-bit paged cache against ``decode_sparse``, element by
element on seeded problems: topk below, at and above a page, not a multiple of 64, invalid
entries (-1 and rows past the end, s_kv not a multiple of 64), tokens with no valid entry,
16 to 128 heads, one to three partitions, and the full-size prefill workload (sampled tokens).
"""
import math

import numpy as np
import pytest
import torch

import mla_decode_attention_12_b200 as mla
from mla_decode_attention_12_b200 import workloads as W
from tests.gpu_helpers import compare

pytestmark = pytest.mark.gpu

LN2 = math.log(2.0)
MAX_LOGITS_ABS = 1e-2  # the largest base-2 scaled logit: fp32 accumulation of 576 bf16 products


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_decode_attention_12_b200 import build
    build.build()


def _dev(bits, dtype=torch.bfloat16):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dtype).cuda()


def _prefill(p, num_parts=None):
    dt = torch.bfloat16 if p.dtype == W.BF16 else torch.float16
    out, mx, lse = mla.flash_mla_sparse_fwd(_dev(p.q, dt), _dev(p.kv, dt), torch.from_numpy(p.indices).cuda(),
                                            p.sm_scale, num_parts=num_parts)
    torch.cuda.synchronize()
    return out, mx, lse


def _check_prefill(p, out, mx, lse, o_ref, mx_ref, lse_ref, what):
    # LSE compared in natural-log units under the decode's tolerance
    print(compare(out, lse.double() * LN2, o_ref, lse_ref * LN2, p.dtype, what))
    m = mx.double().cpu().numpy()
    fin = np.isfinite(mx_ref)
    assert np.array_equal(np.isfinite(m), fin), f"{what}: max_logits finiteness differs"
    assert np.all(m[~fin] == mx_ref[~fin])
    if fin.any():
        assert np.abs(m[fin] - mx_ref[fin]).max() <= MAX_LOGITS_ABS, what


PREFILL = {
    "topk256": lambda: W.make_prefill_problem(60, 128, 1000, 256, seed=501),
    "topk100_invalid": lambda: W.make_prefill_problem(40, 64, 777, 100, invalid_frac=0.25, seed=502),
    "topk64_h16": lambda: W.make_prefill_problem(30, 16, 200, 64, seed=503),
    "topk2048_few_kv": lambda: W.make_prefill_problem(20, 128, 1500, 2048, seed=504),  # lists longer than kv
    "fp16": lambda: W.make_prefill_problem(25, 32, 300, 130, dtype=W.FP16, seed=505),
}


@pytest.mark.parametrize("name", sorted(PREFILL))
def test_prefill_parity(oracle_mod, name):
    p = PREFILL[name]()
    out, mx, lse = _prefill(p)
    o_ref, mx_ref, lse_ref = oracle_mod.sparse_prefill(p.q, p.kv, p.indices, p.sm_scale, dtype=p.dtype)
    _check_prefill(p, out, mx, lse, o_ref, mx_ref, lse_ref, name)


@pytest.mark.parametrize("parts", [1, 3])
def test_prefill_few_partitions_and_empty_lists(oracle_mod, parts):
    # tokens split over partitions (the combine merges maxima and base-2 LSEs) and tokens whose
    # lists hold no valid entry (out 0, max_logits = lse = -inf)
    p = W.make_prefill_problem(12, 64, 500, 300, invalid_frac=0.1, seed=510 + parts)
    p.indices[3, 0, :] = -1
    p.indices[7, 0, :] = 500 + 17
    out, mx, lse = _prefill(p, num_parts=parts)
    o_ref, mx_ref, lse_ref = oracle_mod.sparse_prefill(p.q, p.kv, p.indices, p.sm_scale)
    assert np.isneginf(lse_ref[3]).all() and np.isneginf(mx_ref[7]).all()
    _check_prefill(p, out, mx, lse, o_ref, mx_ref, lse_ref, f"parts={parts}")
    assert bool((out[3] == 0).all()) and bool((out[7] == 0).all())


def test_sparse_decode_over_a_16_bit_cache(oracle_mod):
    # the same kernel path as the prefill, through the paged decode interface
    p = W.make_sparse_problem([2000, 700, 90], 300, s_q=2, h_q=64, invalid_frac=0.2, seed=520)
    q, kv = _dev(p.q), _dev(p.kvcache)
    ind, sl = torch.from_numpy(p.indices).cuda(), torch.from_numpy(p.cache_seqlens).cuda()
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1, h_q=p.h_q, topk=300)
    o, lse = mla.flash_mla_with_kvcache(q, kv, None, sl, 512, md, ns, softmax_scale=p.scale, indices=ind,
                                        is_fp8_kvcache=False)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_mod.decode_sparse(p.q, p.kvcache, p.indices, scale=p.scale)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, "sparse decode, bf16 cache"))


def test_prefill_full_size_sampled(oracle_mod):
    # the benchmark's prefill workload as timed: sampled tokens against the oracle, all finite
    p = W.make_prefill_workload("sparse_prefill")
    out, mx, lse = _prefill(p)
    toks = np.unique(np.concatenate([np.random.default_rng(96).choice(p.s_q, 6, replace=False), [0, p.s_q - 1]]))
    o_ref, mx_ref, lse_ref = oracle_mod.sparse_prefill(p.q[toks], p.kv, p.indices[toks], p.sm_scale)
    idx = torch.from_numpy(toks).cuda()
    _check_prefill(p, out[idx], mx[idx], lse[idx], o_ref, mx_ref, lse_ref, "sparse_prefill sampled")
    assert torch.isfinite(out).all() and torch.isfinite(lse).all() and torch.isfinite(mx).all()


def test_prefill_several_row_groups(oracle_mod):
    # 256 heads per token: two row groups per query token over the same list
    p = W.make_prefill_problem(10, 256, 600, 200, invalid_frac=0.1, seed=530)
    out, mx, lse = _prefill(p)
    o_ref, mx_ref, lse_ref = oracle_mod.sparse_prefill(p.q, p.kv, p.indices, p.sm_scale)
    _check_prefill(p, out, mx, lse, o_ref, mx_ref, lse_ref, "h_q=256")


def test_sparse_decode_16bit_several_row_groups(oracle_mod):
    p = W.make_sparse_problem([1500, 400], 250, s_q=2, h_q=256, invalid_frac=0.2, seed=531)
    q, kv = _dev(p.q), _dev(p.kvcache)
    ind, sl = torch.from_numpy(p.indices).cuda(), torch.from_numpy(p.cache_seqlens).cuda()
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1, h_q=p.h_q, topk=250)
    o, lse = mla.flash_mla_with_kvcache(q, kv, None, sl, 512, md, ns, softmax_scale=p.scale, indices=ind)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle_mod.decode_sparse(p.q, p.kvcache, p.indices, scale=p.scale)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, "sparse decode, bf16 cache, h_q=256"))
