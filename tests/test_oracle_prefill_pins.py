"""Pins of the oracle's sparse MLA prefill (upstream FlashMLA documentation, "Sparse MLA
Prefill / Return Values and Equivalent PyTorch Code"), checked against things other than
itself: torch fp64 brute force following the documentation's steps, a hand-worked two-entry
case, closed forms (one entry, no valid entry, one row listed n times), the base-2 relation to
the separately pinned sparse decode oracle, and invariance under inserted invalid entries."""
import math

import numpy as np
import pytest
import torch

from mla_decode_attention_12_b200 import workloads as W

BF16 = W.BF16


def _bits(x: np.ndarray, dtype=torch.bfloat16) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dtype).view(torch.int16).numpy().view(np.uint16)


def _values(bits: np.ndarray, dtype=torch.bfloat16) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dtype).double()


def _problem(s_q, h_q, s_kv, topk, seed, d_qk=576, invalid=0.0, h_kv=1):
    rng = np.random.default_rng(seed)
    q = _bits(rng.standard_normal((s_q, h_q, d_qk)))
    kv = _bits(rng.standard_normal((s_kv, h_kv, d_qk)))
    ind = np.stack([np.stack([rng.choice(s_kv, size=topk, replace=topk > s_kv) for _ in range(h_kv)])
                    for _ in range(s_q)]).astype(np.int32)
    if invalid:
        bad = rng.random(ind.shape) < invalid
        ind[bad] = np.where(rng.random(ind.shape) < 0.5, -1, s_kv + rng.integers(0, 100, ind.shape))[bad]
    return q, kv, ind


def _torch_reference(q_bits, kv_bits, ind, sm_scale, dv=512):
    """The documentation's equivalent code, written with torch in fp64, valid entries only."""
    q, kv = _values(q_bits), _values(kv_bits)
    s_q, h_q, _ = q.shape
    s_kv, h_kv, _ = kv.shape
    out = torch.zeros(s_q, h_q, dv, dtype=torch.float64)
    mx = torch.full((s_q, h_q), -math.inf, dtype=torch.float64)
    lse = torch.full((s_q, h_q), -math.inf, dtype=torch.float64)
    for i in range(s_q):
        for g in range(h_kv):
            sel = ind[i, g]
            sel = torch.from_numpy(sel[(sel >= 0) & (sel < s_kv)].astype(np.int64))
            if sel.numel() == 0:
                continue
            focused = kv[sel, g]                                   # [n, d_qk]
            heads = slice(g * (h_q // h_kv), (g + 1) * (h_q // h_kv))
            P = (q[i, heads] @ focused.T) * sm_scale * math.log2(math.e)
            m = P.max(dim=-1).values
            l2 = torch.log2(torch.exp2(P - m[:, None]).sum(dim=-1)) + m
            S = torch.exp2(P - l2[:, None])
            out[i, heads] = S @ focused[:, :dv]
            mx[i, heads], lse[i, heads] = m, l2
    return out.numpy(), mx.numpy(), lse.numpy()


PREFILL_CASES = [
    dict(s_q=3, h_q=8, s_kv=300, topk=50, seed=1),
    dict(s_q=2, h_q=16, s_kv=130, topk=200, seed=2, invalid=0.3),
    dict(s_q=4, h_q=4, s_kv=64, topk=7, seed=3, d_qk=512),
    dict(s_q=2, h_q=8, s_kv=90, topk=33, seed=4, h_kv=2, invalid=0.2),
]


@pytest.mark.parametrize("kw", PREFILL_CASES)
def test_prefill_brute_force_torch(oracle_mod, kw):
    q, kv, ind = _problem(**kw)
    scale = 1.0 / math.sqrt(q.shape[-1])
    out, mx, lse = oracle_mod.sparse_prefill(q, kv, ind, scale)
    r_out, r_mx, r_lse = _torch_reference(q, kv, ind, scale)
    fin = np.isfinite(r_lse)
    assert np.array_equal(np.isfinite(lse), fin) and np.array_equal(np.isfinite(mx), fin)
    assert np.allclose(out, r_out, atol=1e-12, rtol=1e-10)
    assert np.allclose(mx[fin], r_mx[fin], atol=1e-12, rtol=1e-12)
    assert np.allclose(lse[fin], r_lse[fin], atol=1e-12, rtol=1e-12)


def test_prefill_hand_two_entries(oracle_mod):
    # q = e0, rows e0 and 0, sm_scale = ln 2: P = (1, 0) in base-2 units, so max_logits = 1,
    # lse = log2(2^1 + 2^0) = log2 3, out[0] = 2^(1 - log2 3) = 2/3, every other column 0.
    q = np.zeros((1, 1, 576), np.float32)
    q[0, 0, 0] = 1.0
    kv = np.zeros((2, 1, 576), np.float32)
    kv[0, 0, 0] = 1.0
    out, mx, lse = oracle_mod.sparse_prefill(_bits(q), _bits(kv), np.array([[[0, 1]]], np.int32), math.log(2.0))
    assert abs(mx[0, 0] - 1.0) < 1e-15
    assert abs(lse[0, 0] - math.log2(3.0)) < 1e-15
    assert abs(out[0, 0, 0] - 2.0 / 3.0) < 1e-15
    assert np.all(out[0, 0, 1:] == 0.0)


def test_prefill_single_entry_and_no_entry(oracle_mod):
    q, kv, ind = _problem(2, 4, 40, 5, seed=7)
    ind[0, 0, :] = -1
    ind[0, 0, 3] = 17          # exactly one valid entry
    ind[1, 0, :] = [-1, 40, 41, -5, 10 ** 6]  # nothing valid
    out, mx, lse = oracle_mod.sparse_prefill(q, kv, ind, 0.05)
    v = _values(kv)[17, 0, :512].numpy()
    assert np.array_equal(out[0], np.broadcast_to(v, (4, 512)))  # weight 2^0 = 1, exactly
    assert np.array_equal(mx[0], lse[0])
    p = (_values(q)[0] @ _values(kv)[17, 0]).numpy() * 0.05 * math.log2(math.e)
    assert np.allclose(mx[0], p, rtol=1e-13, atol=1e-13)
    assert np.all(out[1] == 0.0) and np.all(np.isneginf(mx[1])) and np.all(np.isneginf(lse[1]))


def test_prefill_row_listed_n_times(oracle_mod):
    q, kv, ind = _problem(1, 4, 20, 9, seed=8)
    ind[:] = 5
    out, mx, lse = oracle_mod.sparse_prefill(q, kv, ind, 0.1)
    assert np.allclose(lse, mx + math.log2(9.0), rtol=0, atol=1e-13)
    assert np.allclose(out[0], np.broadcast_to(_values(kv)[5, 0, :512].numpy(), (4, 512)), rtol=0, atol=1e-14)


def test_prefill_is_the_sparse_decode_in_base_2(oracle_mod):
    # The same attention as the (separately pinned) sparse decode oracle over a paged view of
    # the flat kv: out equal, lse_prefill = lse_decode / ln 2, and max_logits the largest
    # scaled logit times log2(e).
    q, kv, ind = _problem(3, 8, 256, 70, seed=9, invalid=0.2)
    scale = 0.07
    out, mx, lse = oracle_mod.sparse_prefill(q, kv, ind, scale)
    o_d, l_d = oracle_mod.decode_sparse(q[:, None], kv.reshape(4, 64, 1, 576), ind, scale=scale)
    assert np.allclose(out, o_d[:, 0], atol=1e-12, rtol=1e-10)
    fin = np.isfinite(l_d[:, 0])
    assert np.allclose(lse[fin], l_d[:, 0][fin] / math.log(2.0), atol=1e-12, rtol=1e-12)
    logits = np.einsum("shd,sgkd->shk", _values(q).numpy(),
                       _values(kv).numpy()[np.clip(ind, 0, 255)].reshape(3, 1, 70, 576))
    valid = (ind[:, 0] >= 0) & (ind[:, 0] < 256)
    best = np.where(valid[:, None, :], logits, -np.inf).max(axis=2) * scale * math.log2(math.e)
    assert np.allclose(mx, best, atol=1e-12, rtol=1e-12)


def test_prefill_invalid_entries_change_nothing(oracle_mod):
    q, kv, ind = _problem(2, 8, 100, 40, seed=10)
    base = oracle_mod.sparse_prefill(q, kv, ind, 0.05)
    rng = np.random.default_rng(11)
    wide = np.full((2, 1, 64), -1, np.int32)
    for i in range(2):
        pos = np.sort(rng.choice(64, 40, replace=False))
        wide[i, 0, pos] = ind[i, 0]
        others = np.setdiff1d(np.arange(64), pos)
        wide[i, 0, others[::2]] = 100 + rng.integers(0, 50, others[::2].size)  # past the end
    again = oracle_mod.sparse_prefill(q, kv, wide, 0.05)
    for a, b in zip(base, again):
        assert np.array_equal(a, b)
