"""Pins for the oracle's token-level sparse decoding.

Upstream FlashMLA documentation, "Sparse Attention (indices tensor)": each query
token (b, s) attends the cache rows listed in indices[b, s, :topk], an entry being
the flat row page * page_size + offset (no block table), -1 marking an invalid
entry.  The oracle reads every entry outside the cache as invalid, counts each
valid entry once per listing (a gather, as the sparse prefill's equivalent code
gathers kv[indices]) and applies no causal mask.  Pinned against:

* brute force through torch fp64 on a flat view of the cache (16-bit and FP8);
* the dense oracle: the full token list of each sequence, in order, gives the
  dense result bit for bit;
* invalid entries (-1 and rows past the cache) inserted anywhere change nothing;
* closed forms: no valid entry (O = 0, LSE = -inf), one row listed n times
  (O = v, LSE = x + ln n);
* the order of the entries does not matter.
"""
import math

import numpy as np
import pytest
import torch

from mla_decode_attention_12_b200 import workloads as W


def _f64(bits, dtype=W.BF16):
    tdt = torch.bfloat16 if dtype == W.BF16 else torch.float16
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(tdt).double()


def _brute(q_bits, kv_rows, indices, scale, dtype=W.BF16, dv=512):
    """kv_rows: torch f64 [n_rows, h_kv, d_qk] (flat view of the pages)."""
    q = _f64(q_bits, dtype)
    B, S, H, D = q.shape
    h_kv = kv_rows.shape[1]
    o = torch.zeros(B, S, H, dv, dtype=torch.float64)
    lse = torch.full((B, S, H), -math.inf, dtype=torch.float64)
    grp = H // h_kv
    for b in range(B):
        for s in range(S):
            ix = [int(i) for i in indices[b, s] if 0 <= int(i) < kv_rows.shape[0]]
            if not ix:
                continue
            for g in range(h_kv):
                K = kv_rows[torch.tensor(ix), g]                         # [n, D]
                logits = (q[b, s, g * grp:(g + 1) * grp] @ K.T) * scale  # [grp, n]
                lse[b, s, g * grp:(g + 1) * grp] = torch.logsumexp(logits, -1)
                o[b, s, g * grp:(g + 1) * grp] = torch.softmax(logits, -1) @ K[:, :dv]
    return o.numpy(), lse.numpy()


SPARSE_CASES = [
    dict(seqlens=[300, 77, 0], topk=128, s_q=2, h_q=8, invalid_frac=0.1),
    dict(seqlens=[500, 64], topk=64, s_q=1, h_q=16),
    dict(seqlens=[200, 130], topk=96, s_q=1, h_q=8, h_kv=2),
]


@pytest.mark.parametrize("kw", SPARSE_CASES, ids=lambda k: str(k["seqlens"]))
def test_sparse_brute_force_torch(oracle_mod, kw):
    p = W.make_sparse_problem(seed=61, **kw)
    o, lse = oracle_mod.decode_sparse(p.q, p.kvcache, p.indices, scale=p.scale)
    kv_rows = _f64(p.kvcache).reshape(-1, p.h_kv, p.d_qk)
    ob, lb = _brute(p.q, kv_rows, p.indices, p.scale)
    np.testing.assert_allclose(o, ob, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12)


def test_sparse_fp8_brute_force_torch(oracle_mod):
    from tests.test_oracle_fp8_pins import _torch_dequant

    p = W.make_sparse_problem([300, 150], topk=128, s_q=2, h_q=8, seed=62, fp8_kv=True, invalid_frac=0.05)
    o, lse = oracle_mod.decode_sparse_fp8(p.q, p.kvcache, p.indices, scale=p.scale)
    kv_rows = _torch_dequant(p.kvcache).double().view(-1, p.h_kv, 576)
    ob, lb = _brute(p.q, kv_rows, p.indices, p.scale)
    np.testing.assert_allclose(o, ob, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12)


def _dense_list(p, topk):
    ix = np.full((p.batch, p.s_q, topk), -1, np.int32)
    for b, L in enumerate(p.cache_seqlens):
        j = np.arange(int(L))
        ix[b, :, :L] = p.block_table[b, j // 64] * 64 + j % 64
    return ix


def test_full_token_list_equals_dense_decode(oracle_mod):
    p = W.make_problem([300, 77, 1, 0], s_q=2, h_q=8, seed=63)
    o, lse = oracle_mod.decode_sparse(p.q, p.kvcache, _dense_list(p, 320), scale=p.scale)
    od, ld = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, scale=p.scale)
    assert np.array_equal(o, od) and np.array_equal(lse, ld)


def test_invalid_entries_change_nothing(oracle_mod):
    # the original 64 entries keep their order at random positions of a 96-entry list; the
    # other 32 are invalid (-1, negative, or rows past the cache): bit-identical results
    p = W.make_sparse_problem([400, 90], topk=64, s_q=2, h_q=8, seed=64)
    o, lse = oracle_mod.decode_sparse(p.q, p.kvcache, p.indices, scale=p.scale)
    rng = np.random.default_rng(0)
    n_rows = p.num_blocks * 64
    junk = np.array([-1, -5, n_rows, n_rows + 7], np.int32)
    bad = np.empty((p.batch, p.s_q, 96), np.int32)
    for b in range(p.batch):
        for s in range(p.s_q):
            keep = np.sort(rng.choice(96, size=64, replace=False))
            bad[b, s] = junk[rng.integers(0, 4, size=96)]
            bad[b, s, keep] = p.indices[b, s]
    o2, l2 = oracle_mod.decode_sparse(p.q, p.kvcache, bad, scale=p.scale)
    assert np.array_equal(o, o2) and np.array_equal(lse, l2)


def test_no_valid_entry_is_empty(oracle_mod):
    p = W.make_sparse_problem([100], topk=32, h_q=4, seed=65)
    ix = np.full_like(p.indices, -1)
    ix[0, 0, 3] = p.num_blocks * 64  # past the cache: invalid too
    o, lse = oracle_mod.decode_sparse(p.q, p.kvcache, ix, scale=p.scale)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_one_row_listed_n_times(oracle_mod):
    # every entry the same row r: O = v_r exactly, LSE = x_r + ln n (each listing is a term)
    p = W.make_sparse_problem([100], topk=24, h_q=4, seed=66)
    r = int(p.indices[0, 0, 5])
    ix = np.full_like(p.indices, r)
    o, lse = oracle_mod.decode_sparse(p.q, p.kvcache, ix, scale=p.scale)
    k = _f64(p.kvcache).reshape(-1, 1, p.d_qk)[r, 0].numpy()
    q = _f64(p.q)[0, 0].numpy()
    for h in range(4):
        np.testing.assert_allclose(o[0, 0, h], k[:512], rtol=1e-13, atol=1e-15)
        assert lse[0, 0, h] == pytest.approx(p.scale * float(q[h] @ k) + math.log(24), rel=1e-13, abs=1e-13)


def test_entry_order_does_not_matter(oracle_mod):
    p = W.make_sparse_problem([700, 300], topk=256, s_q=1, h_q=16, seed=67, invalid_frac=0.2)
    o, lse = oracle_mod.decode_sparse(p.q, p.kvcache, p.indices, scale=p.scale)
    perm = np.random.default_rng(1).permutation(256)
    o2, l2 = oracle_mod.decode_sparse(p.q, p.kvcache, p.indices[:, :, perm], scale=p.scale)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, l2, rtol=1e-13, atol=1e-13)
