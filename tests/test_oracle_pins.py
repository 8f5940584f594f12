"""Pins for the FP64 oracle: closed forms, hand cases, brute force and invariants.

The oracle is the plain definition of MLA decoding over a paged cache (the
"FlashMLA" usage page, flash_mla_with_kvcache; upstream FlashMLA documentation,
"Usage / MLA Decoding" return values and "MLA Mode" footnote).  Nothing on the
pages prints numeric outputs, so these tests fix it against mathematics that is
independent of its code:

* hand-worked closed forms (``tests/golden/hand_cases.txt``);
* special cases with closed forms (one visible token, zero queries, equal keys,
  empty sequences);
* brute force through an independent library path (torch fp64 on a contiguous
  K built by a separate gather, torch's softmax / logsumexp);
* invariants: split-then-combine equals unsplit, any page permutation with a
  matching block table gives bit-identical output, LSE equals the logsumexp of
  the scaled logits, NaN in never-visible cache rows changes nothing.

Each is chosen so that a plausible mistake (dropped scale, V taken from the
wrong columns, wrong causal offset, wrong kv-head mapping, transposed page
index, wrong LSE base) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

from mla_decode_attention_12_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.txt")


# ---------------------------------------------------------------------------
# bit decoding
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,tdt", [(W.BF16, torch.bfloat16), (W.FP16, torch.float16)])
def test_half_decoding_matches_torch(oracle_mod, dtype, tdt):
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 1 << 16, size=4000, dtype=np.uint32).astype(np.uint16)
    # edge patterns: zeros, subnormals, max finite, infinities
    bits[:8] = [0x0000, 0x8000, 0x0001, 0x03FF, 0x7BFF, 0x7C00, 0xFC00, 0x7F7F]
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(tdt).double().numpy()
    got = oracle_mod.half_bits_to_float64(bits, dtype)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------------------
# hand cases from the golden file
# ---------------------------------------------------------------------------

def _parse_golden():
    cases, cur = [], None
    for raw in open(GOLDEN):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        key, _, val = (p.strip() for p in line.partition("="))
        if key == "case":
            cur = {"name": val, "keys": {}, "o": {}, "lse": {}}
            cases.append(cur)
        elif key.startswith("k") and key[1:].isdigit():
            cur["keys"][int(key[1:])] = val
        elif key.startswith("o["):
            s, d = (int(t) for t in key[2:-1].split("]["))
            cur["o"][(s, d)] = float(val)
        elif key.startswith("lse["):
            cur["lse"][int(key[4:-1])] = float(val)
        else:
            cur[key] = val
    return cases


def _sparse_vec(spec, n):
    v = np.zeros(n, np.float32)
    for item in spec.split():
        i, x = item.split(":")
        v[int(i)] = float(x)
    return v


@pytest.mark.parametrize("case", _parse_golden(), ids=lambda c: c["name"])
def test_hand_cases(oracle_mod, case):
    d_qk, dv, s_q = int(case["d_qk"]), int(case["dv"]), int(case["s_q"])
    L = int(case["seqlen"])
    qv = _sparse_vec(case["q"], d_qk)
    q = np.broadcast_to(W.to_bits(qv, W.BF16), (1, s_q, 1, d_qk)).copy()
    kv = np.zeros((1, 64, 1, d_qk), np.uint16)
    for j, spec in case["keys"].items():
        kv[0, j, 0] = W.to_bits(_sparse_vec(spec, d_qk), W.BF16)
    table = np.zeros((1, 1), np.int32)
    o, lse = oracle_mod.decode(q, kv, table, np.array([L], np.int32), dv=dv,
                               causal=bool(int(case["causal"])), scale=float(case["scale"]))
    expect_o = np.zeros((s_q, dv))
    for (s, d), x in case["o"].items():
        expect_o[s, d] = x
    np.testing.assert_allclose(o[0, :, 0, :], expect_o, rtol=1e-14, atol=1e-15)
    for s, x in case["lse"].items():
        assert lse[0, s, 0] == pytest.approx(x, rel=1e-14)


# ---------------------------------------------------------------------------
# closed-form special cases
# ---------------------------------------------------------------------------

def _f64(bits, dtype=W.BF16):
    tdt = torch.bfloat16 if dtype == W.BF16 else torch.float16
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(tdt).double().numpy()


def _token_rows(p, b):
    """[L_b, d_qk] f64 rows of request b, gathered through the block table."""
    L = int(p.cache_seqlens[b])
    kv = _f64(p.kvcache, p.dtype)
    rows = [kv[p.block_table[b, j // 64], j % 64, 0] for j in range(L)]
    return np.array(rows).reshape(L, p.d_qk)


def test_single_visible_token(oracle_mod):
    # causal, s_q = 3, L = 3: query 0 sees exactly one token -> O = v_0, LSE = x_0
    p = W.make_problem([3], s_q=3, h_q=4, d_qk=576, causal=True, seed=11)
    o, lse = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens,
                               causal=True, scale=p.scale)
    K = _token_rows(p, 0)
    q = _f64(p.q)[0, 0]  # [h, d]
    for h in range(4):
        assert np.array_equal(o[0, 0, h], K[0, :512])
        assert lse[0, 0, h] == pytest.approx(p.scale * float(q[h] @ K[0]), rel=1e-13)


def test_zero_query_is_mean_of_values(oracle_mod):
    # q = 0 -> all logits 0 -> O = mean_j v_j, LSE = ln n  (pins padded heads)
    p = W.make_problem([150, 64, 1], s_q=2, h_q=8, causal=True, active_heads=0, seed=12)
    o, lse = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens,
                               causal=True, scale=p.scale)
    vis = p.visible()
    for b in range(3):
        K = _token_rows(p, b)
        for s in range(2):
            n = vis[b, s]
            if n == 0:
                assert np.all(o[b, s] == 0) and np.all(np.isneginf(lse[b, s]))
                continue
            np.testing.assert_allclose(o[b, s], np.broadcast_to(K[:n, :512].mean(0), (8, 512)),
                                       rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(lse[b, s], math.log(n), rtol=1e-14)


def test_identical_keys_give_uniform_weights(oracle_mod):
    p = W.make_problem([200], h_q=4, seed=13)
    row = p.kvcache[p.block_table[0, 0], 0].copy()
    p.kvcache[:] = row  # every cached row identical
    o, lse = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, scale=p.scale)
    k = _f64(row)[0]
    q = _f64(p.q)[0, 0]
    for h in range(4):
        np.testing.assert_allclose(o[0, 0, h], k[:512], rtol=1e-12, atol=1e-13)
        x = p.scale * float(q[h] @ k)
        assert lse[0, 0, h] == pytest.approx(x + math.log(200), rel=1e-12, abs=1e-12)


def test_empty_sequence(oracle_mod):
    p = W.make_problem([0, 70], h_q=4, seed=14)
    o, lse = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, scale=p.scale)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(o[1])) and np.all(np.isfinite(lse[1]))


# ---------------------------------------------------------------------------
# brute force through torch fp64 (unpaged, contiguous K)
# ---------------------------------------------------------------------------

def _brute(p):
    q = torch.from_numpy(_f64(p.q, p.dtype))
    kvf = _f64(p.kvcache, p.dtype)
    B, S, H, D = q.shape
    o = torch.zeros(B, S, H, p.dv, dtype=torch.float64)
    lse = torch.full((B, S, H), -math.inf, dtype=torch.float64)
    group = H // p.h_kv
    vis = p.visible()
    for b in range(B):
        L = int(p.cache_seqlens[b])
        idx = [(int(p.block_table[b, j // 64]), j % 64) for j in range(L)]
        for g in range(p.h_kv):
            K = torch.tensor(np.array([kvf[pg, t, g] for pg, t in idx]).reshape(L, D))
            for s in range(S):
                n = int(vis[b, s])
                if n == 0:
                    continue
                qs = q[b, s, g * group:(g + 1) * group]          # [group, D]
                logits = (qs @ K[:n].T) * p.scale                # [group, n]
                lse[b, s, g * group:(g + 1) * group] = torch.logsumexp(logits, -1)
                o[b, s, g * group:(g + 1) * group] = torch.softmax(logits, -1) @ K[:n, :p.dv]
    return o.numpy(), lse.numpy()


BRUTE_CASES = [
    dict(seqlens=[256, 193], s_q=1, h_q=16, d_qk=576),
    dict(seqlens=[65, 1, 130], s_q=2, h_q=8, d_qk=576, causal=True),
    dict(seqlens=[100, 37], s_q=4, h_q=4, d_qk=512, causal=True, dtype=W.FP16, std=0.5),
    dict(seqlens=[77, 129], s_q=1, h_q=8, h_kv=2, d_qk=576),
    dict(seqlens=[3, 2], s_q=3, h_q=2, d_qk=576, causal=True),
]


@pytest.mark.parametrize("kw", BRUTE_CASES, ids=lambda k: str(k["seqlens"]))
def test_brute_force_torch(oracle_mod, kw):
    p = W.make_problem(seed=21, **kw)
    o, lse = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, dtype=p.dtype,
                               causal=p.causal, scale=p.scale)
    ob, lb = _brute(p)
    np.testing.assert_allclose(o, ob, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12)


def test_lse_is_logsumexp_of_scaled_logits(oracle_mod):
    from scipy.special import logsumexp

    p = W.make_problem([300], h_q=8, seed=31, scale=0.07)
    _, lse = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, scale=0.07)
    K = _token_rows(p, 0)
    x = 0.07 * (_f64(p.q)[0, 0] @ K.T)  # [h, L]
    np.testing.assert_allclose(lse[0, 0], logsumexp(x, axis=-1), rtol=1e-13)


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
def test_split_then_combine_equals_unsplit(oracle_mod, causal):
    p = W.make_problem([500, 129, 64], s_q=2, h_q=8, causal=causal, seed=41)
    kw = dict(causal=causal, scale=p.scale)
    o, lse = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, **kw)
    cuts = [0, 64, 128, 499, 1 << 20]
    parts = [oracle_mod.decode_range(p.q, p.kvcache, p.block_table, p.cache_seqlens, lo, hi, **kw)
             for lo, hi in zip(cuts[:-1], cuts[1:])]
    oc, lc = oracle_mod.combine(np.stack([x[0] for x in parts]), np.stack([x[1] for x in parts]))
    np.testing.assert_allclose(oc, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lc, lse, rtol=1e-12, atol=1e-13)


def test_page_permutation_is_bit_identical(oracle_mod):
    p = W.make_problem([300, 64, 5], s_q=2, h_q=4, causal=True, seed=51, extra_pages=3)
    o, lse = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, causal=True,
                               scale=p.scale)
    perm = np.random.default_rng(3).permutation(p.num_blocks)
    kv2 = np.empty_like(p.kvcache)
    kv2[perm] = p.kvcache  # page x moves to perm[x]
    t2 = np.where(p.block_table >= 0, perm[np.maximum(p.block_table, 0)], -1).astype(np.int32)
    o2, lse2 = oracle_mod.decode(p.q, kv2, t2, p.cache_seqlens, causal=True, scale=p.scale)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_nan_in_unused_cache_rows_changes_nothing(oracle_mod):
    kw = dict(s_q=2, h_q=4, causal=True, seed=61, extra_pages=4)
    clean = W.make_problem([100, 64, 1], **kw)
    dirty = W.make_problem([100, 64, 1], poison=True, **kw)
    assert np.isnan(_f64(dirty.kvcache)).any()
    a = oracle_mod.decode(clean.q, clean.kvcache, clean.block_table, clean.cache_seqlens,
                          causal=True, scale=clean.scale)
    b = oracle_mod.decode(dirty.q, dirty.kvcache, dirty.block_table, dirty.cache_seqlens,
                          causal=True, scale=dirty.scale)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert np.isfinite(b[0]).all()


def test_decode_rows_matches_decode(oracle_mod):
    p = W.make_problem([90, 200], s_q=2, h_q=8, causal=True, seed=71)
    o, lse = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, causal=True,
                               scale=p.scale)
    rows = np.array([0, 5, 17, 31], np.int64)
    o2, l2 = oracle_mod.decode_rows(p.q, p.kvcache, p.block_table, p.cache_seqlens, rows,
                                    causal=True, scale=p.scale)
    assert np.array_equal(o2, o.reshape(-1, 512)[rows])
    assert np.array_equal(l2, lse.reshape(-1)[rows])


def test_weights_sum_to_one(oracle_mod):
    # V = all-ones columns -> O must be exactly the sum of weights = 1
    p = W.make_problem([333], h_q=4, seed=81)
    p.kvcache[..., :512] = W.to_bits(np.ones(1, np.float32), W.BF16)[0]
    o, _ = oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, scale=p.scale)
    np.testing.assert_allclose(o, 1.0, rtol=1e-13)
