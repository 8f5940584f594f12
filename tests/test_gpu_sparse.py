"""GPU parity of the token-level sparse decode over an "FP8 with scale" cache (upstream
FlashMLA documentation, "Sparse Attention (indices tensor)") against the FP64 oracle's
``decode_sparse_fp8``, element by element, on seeded problems: lists shorter and longer
than a page, topk not a multiple of 64, invalid entries (-1, other negatives, rows past the
cache), rows listed several times, tokens with no valid entry, several partitions per token
(split and combined), 16 to 128 heads, and the full-size benchmark workload (sampled rows).
"""
import numpy as np
import pytest
import torch

import mla_decode_attention_12_b200 as mla
from mla_decode_attention_12_b200 import workloads as W
from tests.gpu_helpers import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mla_decode_attention_12_b200 import build
    build.build()


def _run(p, num_parts=None, active_heads=None, sentinel=None):
    q = torch.from_numpy(p.q.view(np.int16)).view(torch.bfloat16).cuda()
    kv = torch.from_numpy(p.kvcache).cuda()
    ind = torch.from_numpy(p.indices).cuda()
    sl = torch.from_numpy(p.cache_seqlens).cuda()
    topk = p.indices.shape[2]
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q, 1, num_parts=num_parts, h_q=p.h_q, topk=topk)
    ws = torch.zeros(mla.workspace_bytes(p.batch * p.s_q, 1, p.h_q, 1, md.shape[0]), dtype=torch.uint8, device="cuda")
    o = lse = None
    if sentinel is not None:
        o = torch.full((p.batch, p.s_q, p.h_q, 512), sentinel, dtype=torch.bfloat16, device="cuda")
        lse = torch.full((p.batch, p.s_q, p.h_q), sentinel, dtype=torch.float32, device="cuda")
    o, lse = mla.flash_mla_with_kvcache(q, kv, None, sl, 512, md, ns, softmax_scale=p.scale, workspace=ws, out=o,
                                        lse=lse, active_heads=active_heads, is_fp8_kvcache=True, indices=ind)
    torch.cuda.synchronize()
    assert mla.read_device_status(ws) == 0
    return o, lse, md, ns


def _oracle(oracle_mod, p):
    return oracle_mod.decode_sparse_fp8(p.q, p.kvcache, p.indices, scale=p.scale)


SMALL = {
    "topk256_h128": lambda: W.make_sparse_problem([3000, 700, 64, 5], 256, s_q=1, h_q=128, fp8_kv=True, seed=401),
    "topk200_sq2_h64_invalid": lambda: W.make_sparse_problem([900, 2500, 130], 200, s_q=2, h_q=64, fp8_kv=True,
                                                             invalid_frac=0.3, seed=402),
    "topk64_h16": lambda: W.make_sparse_problem([500, 63, 1], 64, s_q=3, h_q=16, fp8_kv=True, seed=403),
    "topk1000_long": lambda: W.make_sparse_problem([20000, 9000], 1000, s_q=1, h_q=128, fp8_kv=True,
                                                   invalid_frac=0.05, seed=404),
    "topk33_h40": lambda: W.make_sparse_problem([77, 300], 33, s_q=2, h_q=40, fp8_kv=True, seed=405),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_sparse_parity_small(oracle_mod, name):
    p = SMALL[name]()
    o, lse, md, ns = _run(p)
    o_ref, lse_ref = _oracle(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, name))


@pytest.mark.parametrize("parts", [1, 3])
def test_sparse_few_partitions(oracle_mod, parts):
    # many chunks per partition and tokens split over partitions (the combine runs)
    p = W.make_sparse_problem([4000, 1500, 300], 700, s_q=2, h_q=64, fp8_kv=True, invalid_frac=0.1, seed=410 + parts)
    o, lse, md, ns = _run(p, num_parts=parts)
    o_ref, lse_ref = _oracle(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, f"parts={parts}"))


def test_sparse_edge_entries(oracle_mod):
    # Entries that are not valid (-1, other negatives, rows at and past the end of the cache)
    # anywhere in a list, a row listed many times, and tokens whose lists hold no valid entry
    # (O = 0, LSE = -inf); the cache's never-visible rows hold NaN codes.
    p = W.make_sparse_problem([700, 300, 90], 150, s_q=2, h_q=32, fp8_kv=True, seed=420, poison=True)
    rows = p.num_blocks * 64
    ind = p.indices
    ind[0, 0, 5] = -7
    ind[0, 0, 70] = rows          # the first row past the cache
    ind[0, 1, 3] = rows + 12345
    ind[0, 1, 100] = 2 ** 31 - 1
    ind[1, 0, :] = ind[1, 0, 17]  # one row listed 150 times
    ind[1, 1, :] = -1             # nothing valid
    ind[2, 0, :] = rows + 1       # nothing valid either
    ind[2, 1, 64:] = -1           # only the first "page" of the list
    o, lse, md, ns = _run(p)
    o_ref, lse_ref = _oracle(oracle_mod, p)
    assert np.isneginf(lse_ref[1, 1]).all() and np.isneginf(lse_ref[2, 0]).all()
    print(compare(o, lse, o_ref, lse_ref, p.dtype, "edge entries"))
    assert bool((o[1, 1] == 0).all()) and bool((o[2, 0] == 0).all())


def test_sparse_active_heads(oracle_mod):
    # padding heads (zero queries, a tensor-parallel rank's) are neither written nor combined
    p = W.make_sparse_problem([3000, 800], 500, s_q=2, h_q=64, fp8_kv=True, active_heads=16, seed=430)
    o, lse, md, ns = _run(p, active_heads=16, sentinel=7.0)
    o_ref, lse_ref = _oracle(oracle_mod, p)
    print(compare(o[:, :, :16].contiguous(), lse[:, :, :16].contiguous(), o_ref[:, :, :16], lse_ref[:, :, :16],
                  p.dtype, "sparse, 16 active heads"))
    assert bool((o[:, :, 16:] == 7.0).all()) and bool((lse[:, :, 16:] == 7.0).all())


def test_sparse_metadata_kernel_matches_host_schedule():
    # the device schedule of the sparse decode is the dense algorithm over tokens of topk entries
    # (at the sparse calls' per-chunk cost)
    for tokens, topk, h_q in ((7, 2048, 128), (300, 100, 64), (3, 64, 256)):
        sl = torch.zeros(1, dtype=torch.int32, device="cuda")
        md, ns = mla.get_mla_metadata(sl.expand(tokens).contiguous(), h_q, 1, h_q=h_q, topk=topk)
        md_h, ns_h = mla.get_mla_metadata_sparse_host(tokens, topk, h_q, 1, md.shape[0])
        assert np.array_equal(md.cpu().numpy(), md_h) and np.array_equal(ns.cpu().numpy(), ns_h)


def test_sparse_full_size_sampled(oracle_mod):
    # The benchmark's sparse workload as timed: sampled rows against the oracle, every row
    # finite.  The oracle runs on the sampled tokens over a compact copy of the rows they list
    # (the same bytes, renumbered), not on the whole 0.5 GB cache.
    p = W.make_workload("sparse_fp8")
    o, lse, md, ns = _run(p)
    assert int(ns[-1].item()) > ns.numel() - 1, "the workload must split some token over partitions"
    rows_total = p.batch * p.s_q * p.h_q
    topk = p.indices.shape[2]
    rng = np.random.default_rng(97)
    sample = np.unique(np.concatenate([rng.choice(rows_total, 40, replace=False), [0, rows_total - 1]]))
    tok = sample // p.h_q
    toks = np.unique(tok)
    ind = p.indices.reshape(-1, topk)[toks]
    valid = (ind >= 0) & (ind < p.num_blocks * 64)
    uniq = np.unique(ind[valid])
    kv_rows = p.kvcache.reshape(-1, 656)[uniq]
    kv_small = np.concatenate([kv_rows, np.zeros(((-len(uniq)) % 64, 656), np.uint8)]).reshape(-1, 64, 1, 656)
    ind_small = np.where(valid, np.searchsorted(uniq, np.where(valid, ind, 0)), -1).astype(np.int32)
    q_small = p.q.reshape(-1, 1, p.h_q, p.d_qk)[toks]
    o_ref, lse_ref = oracle_mod.decode_sparse_fp8(q_small, kv_small, ind_small.reshape(len(toks), 1, topk),
                                                  scale=p.scale)
    pos = {t: i for i, t in enumerate(toks)}
    sel = np.array([pos[t] for t in tok])
    heads = sample % p.h_q
    o_r = o_ref.reshape(len(toks), p.h_q, 512)[sel, heads]
    l_r = lse_ref.reshape(len(toks), p.h_q)[sel, heads]
    idx = torch.from_numpy(sample).cuda()
    print(compare(o.reshape(rows_total, 512)[idx], lse.reshape(rows_total)[idx], o_r, l_r, p.dtype,
                  "sparse_fp8 sampled"))
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("h_q,s_q", [(256, 1), (192, 2)])
def test_sparse_several_row_groups(oracle_mod, h_q, s_q):
    # more than 128 heads per token: each token's rows form two row groups (virtual batches
    # numbered group-major), both reading the token's own entry list
    p = W.make_sparse_problem([2500, 900, 300], 400, s_q=s_q, h_q=h_q, fp8_kv=True, invalid_frac=0.1, seed=440 + h_q)
    o, lse, md, ns = _run(p)
    o_ref, lse_ref = _oracle(oracle_mod, p)
    print(compare(o, lse, o_ref, lse_ref, p.dtype, f"sparse h_q={h_q} s_q={s_q}"))
