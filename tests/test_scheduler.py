"""Properties of the tile scheduler (host build of the same code the metadata kernel runs).

Several schedules are correct; what must hold for any of them: every page of
every (request, row group) is processed by exactly one partition, empty
sequences still get one (empty) chunk, the split counts in num_splits match the
chunks, split indices count up from 0 in partition order, and the work is
balanced.
"""
import os
import re

import numpy as np
import pytest

import mla_decode_attention_12_b200 as mla

_SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "mla_decode_attention_12_b200", "csrc",
                    "scheduler.cuh")
FIXED = int(re.search(r"constexpr int kFixedCost = (\d+);", open(_SRC).read()).group(1))
FIXED_SPARSE = int(re.search(r"constexpr int kFixedCostSparse = (\d+);", open(_SRC).read()).group(1))
FIXED_FP8 = int(re.search(r"constexpr int kFixedCostFp8 = (\d+);", open(_SRC).read()).group(1))


def pages(L):
    return (int(L) + 63) // 64


def chunks_of(md, seqlens, groups):
    """Replays the kernel's chunk iteration: yields (part, vb, lo, hi, split_idx)."""
    out = []
    for p, (bv, bb, ev, eb, bs, *_rest) in enumerate(md):
        vb, blk = bv, bb
        while vb < ev or (vb == ev and blk < eb):
            n = pages(seqlens[vb % len(seqlens)])  # group-major: vb = g * batch + b
            hi = eb if vb == ev else n
            out.append((p, vb, blk, hi, bs if vb == bv else 0))
            vb, blk = vb + 1, 0
    return out


def check_schedule(seqlens, heads_per_kv, num_parts, sparse_topk=None, fp8=False):
    """The properties of the paged decode's schedule (over an FP8 cache with fp8), or, with
    sparse_topk, of the sparse decode's: len(seqlens) query tokens of sparse_topk entries."""
    seqlens = np.asarray(seqlens, np.int32)
    if sparse_topk is None:
        md, ns = mla.get_mla_metadata_host(seqlens, heads_per_kv, 1, num_parts, is_fp8_kvcache=fp8)
        F = FIXED_FP8 if fp8 else FIXED
    else:
        assert np.all(seqlens == sparse_topk)
        md, ns = mla.get_mla_metadata_sparse_host(seqlens.size, sparse_topk, heads_per_kv, 1, num_parts)
        F = FIXED_SPARSE
    groups = (heads_per_kv + 127) // 128
    nv = seqlens.size * groups
    assert md.shape == (num_parts, 8) and ns.shape == (nv + 1,)
    assert ns[0] == 0 and np.all(np.diff(ns) >= 1)
    ch = chunks_of(md, seqlens, groups)
    covered = {}
    per_vb = {}
    for p, vb, lo, hi, sidx in ch:
        assert 0 <= vb < nv
        n = pages(seqlens[vb % seqlens.size])
        assert 0 <= lo <= hi <= n
        assert hi > lo or n == 0, "non-empty sequences never get empty chunks"
        for blk in range(lo, hi):
            assert (vb, blk) not in covered, "page processed twice"
            covered[(vb, blk)] = p
        per_vb.setdefault(vb, []).append((p, lo, sidx))
    for vb in range(nv):
        n = pages(seqlens[vb % seqlens.size])
        for blk in range(n):
            assert (vb, blk) in covered, f"page {blk} of vb {vb} never processed"
        lst = per_vb.get(vb, [])
        assert len(lst) == ns[vb + 1] - ns[vb] >= 1
        assert [s for _, _, s in lst] == list(range(len(lst)))
        assert [lo for _, lo, _ in lst] == sorted(lo for _, lo, _ in lst)
    # balance: every partition's cost, pages plus the fixed cost of each of its
    # chunks, stays within the budget F + max(ceil((W - F) / num_parts), F) (a partition
    # is never given less than one chunk's overhead of pages)
    W = sum((pages(L) + F) * groups for L in seqlens)
    T = max(-(-(W - F) // num_parts), F) + F
    cost = np.zeros(num_parts, np.int64)
    for p, vb, lo, hi, _ in ch:
        cost[p] += (hi - lo) + F
    assert cost.max(initial=0) <= T
    return md, ns, cost, T


@pytest.mark.parametrize("seqlens,hpk", [
    ([256, 193], 16),
    ([65536, 49152, 32768, 8192], 128),
    ([0, 0, 5], 16),
    ([0], 128),
    ([1], 512),
    ([64, 128, 65], 200),
    (list(range(0, 4000, 37)), 128),
])
def test_schedule_fixed_cases(seqlens, hpk):
    check_schedule(seqlens, hpk, 74)


@pytest.mark.parametrize("seed", range(40))
def test_schedule_random(seed):
    rng = np.random.default_rng(seed)
    b = int(rng.integers(1, 300))
    kind = seed % 4
    if kind == 0:
        L = rng.integers(0, 20000, b)
    elif kind == 1:
        L = np.floor(np.exp(rng.uniform(0, np.log(70000), b)))
    elif kind == 2:
        L = rng.integers(0, 70, b)
    else:
        L = np.where(rng.random(b) < 0.1, rng.integers(30000, 100000, b), rng.integers(1, 300, b))
    hpk = int(rng.choice([1, 16, 64, 128, 129, 256, 300]))
    parts = int(rng.choice([1, 2, 7, 74, 148]))
    check_schedule(L.astype(np.int32), hpk, parts)


def test_last_partition_absorbs_remainder():
    # Many tiny sequences: per-partition budgets leave scraps; nothing may be dropped.
    md, ns, cost, T = check_schedule([1] * 1000, 16, 74)
    assert cost.sum() == 1000 * (1 + FIXED)


def test_long_sequences_are_split_evenly():
    md, ns, cost, T = check_schedule([65536, 49152, 32768, 8192], 128, 74)
    assert ns[-1] > 4  # at least one sequence is split, so the combine kernel runs
    assert cost.max() <= T


@pytest.mark.parametrize("tokens,topk,h_q,parts", [(128, 2048, 128, 74), (7, 2048, 128, 74), (300, 100, 64, 74),
                                                   (3, 64, 256, 74), (2048, 2048, 128, 74), (5, 0, 128, 3)])
def test_sparse_schedule(tokens, topk, h_q, parts):
    # the sparse calls' schedule: the same algorithm at their own per-chunk cost
    check_schedule([topk] * tokens, h_q, parts, sparse_topk=topk)


def test_sparse_schedule_uses_its_own_chunk_cost():
    md_s, _ = mla.get_mla_metadata_sparse_host(64, 2048, 128, 1, 74)
    md_d, _ = mla.get_mla_metadata_host(np.full(64, 2048, np.int32), 128, 1, 74)
    assert FIXED_SPARSE != FIXED and not np.array_equal(md_s, md_d)


@pytest.mark.parametrize("seed", range(8))
def test_fp8_cache_schedule(seed):
    # the paged decode over an FP8 cache: the same algorithm at that cache's per-chunk cost
    rng = np.random.default_rng(100 + seed)
    L = rng.integers(0, 20000, int(rng.integers(1, 200))).astype(np.int32)
    check_schedule(L, int(rng.choice([16, 64, 128, 256])), int(rng.choice([1, 7, 74])), fp8=True)
