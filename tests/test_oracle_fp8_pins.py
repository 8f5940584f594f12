"""Pins for the oracle's "FP8 with scale" KV cache path.

The format is fixed by the upstream FlashMLA documentation ("FP8 KV Cache"
section, reproduced on the "FlashMLA vLLM Optimization" page): a token row is
656 bytes, 512 float8_e4m3 latent values, 4 float32 scales (the k-th for latent
values [128k, 128k + 128)), then 64 bfloat16 RoPE values that are not quantized;
the kernel dequantizes the cache to bfloat16 and computes in bfloat16.  These
tests pin the oracle against things its code does not share:

* every one of the 256 e4m3 codes against torch's ``float8_e4m3fn`` decoding,
  plus landmarks of the encoding written out by hand;
* a hand-worked row (byte positions, scale blocks, RoPE offset, a tie that
  round-to-nearest-even breaks downwards);
* dequantization of random rows against an independent library path (torch's
  e4m3 decoding, float32 product, float32 -> bfloat16 rounding);
* attention over the cache against torch fp64 on that library-dequantized K;
* NaN in never-visible rows changes nothing.
"""
import math
import struct

import numpy as np
import pytest
import torch

from mla_decode_attention_12_b200 import workloads as W

# ---------------------------------------------------------------------------
# e4m3 decoding
# ---------------------------------------------------------------------------


def test_e4m3_all_codes_match_torch(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    got = oracle_mod.e4m3_to_float64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert nan.sum() == 2  # S.1111.111 only
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9),   # subnormals (m/8) * 2^-6
    (0x08, 2.0 ** -6),                                        # smallest normal
    (0x38, 1.0), (0x3C, 1.5), (0x40, 2.0), (0x3A, 1.25),      # bias 7
    (0x7E, 448.0), (0xFE, -448.0), (0xB8, -1.0),              # largest finite, sign bit
])
def test_e4m3_landmarks(oracle_mod, code, value):
    assert oracle_mod.e4m3_to_float64(np.array([code], np.uint8))[0] == value


def test_e4m3_negative_zero_and_nan(oracle_mod):
    v = oracle_mod.e4m3_to_float64(np.array([0x80, 0x7F, 0xFF], np.uint8))
    assert v[0] == 0.0 and math.copysign(1.0, v[0]) == -1.0
    assert np.isnan(v[1]) and np.isnan(v[2])


# ---------------------------------------------------------------------------
# a hand-worked row
# ---------------------------------------------------------------------------


def _row(latent: dict, scales, rope: dict) -> np.ndarray:
    r = np.zeros(656, np.uint8)
    for i, c in latent.items():
        r[i] = c
    r[512:528] = np.frombuffer(struct.pack("<4f", *scales), np.uint8)
    for i, bits in rope.items():
        r[528 + 2 * i:530 + 2 * i] = np.frombuffer(struct.pack("<H", bits), np.uint8)
    return r


def test_dequant_hand_row(oracle_mod):
    # scales: 0.5 for latent [0,128), 3.0 for [128,256), 2^-7 for [256,384), -2.0 for [384,512);
    # 0.828125 = 53/64 and 1.2109375 = 155/128 only appear in the rounding rows below.
    row = _row({0: 0x38, 127: 0x40, 128: 0x3C, 255: 0xB8, 256: 0x7E, 384: 0x01, 511: 0x3A},
               (0.5, 3.0, 2.0 ** -7, -2.0), {0: 0x3FC0, 63: 0xC2F6})
    out = oracle_mod.dequant_fp8(row[None])[0]
    expect = np.zeros(576, np.uint16)
    expect[0] = 0x3F00      # 1.0 * 0.5 = 0.5
    expect[127] = 0x3F80    # 2.0 * 0.5 = 1.0   (still the first scale)
    expect[128] = 0x4090    # 1.5 * 3.0 = 4.5   (second scale starts at 128)
    expect[255] = 0xC040    # -1.0 * 3.0 = -3.0
    expect[256] = 0x4060    # 448 * 2^-7 = 3.5
    expect[384] = 0xBB80    # 2^-9 * -2 = -2^-8
    expect[511] = 0xC020    # 1.25 * -2 = -2.5
    expect[512] = 0x3FC0    # RoPE value 0 = 1.5, copied
    expect[575] = 0xC2F6    # RoPE value 63, copied
    # zero codes times a negative scale give -0.0 (0x8000)
    expect[385:511] = 0x8000
    assert np.array_equal(out, expect), np.nonzero(out != expect)


@pytest.mark.parametrize("code,scale,bits", [
    (0x3A, 0.828125, 0x3F84),   # 1.25 * 53/64 = 1.03515625 = 132.5 ulps: tie, even -> down (0x3F84)
    (0x3D, 1.2109375, 0x3FFC),  # 1.625 * 155/128 = 1.9677734375 = 251.875 ulps -> up to 1.96875
    (0x3F, 1.0703125, 0x4000),  # 1.875 * 137/128 = 2.0068359375 = 0.4375 ulp above 2 -> 2.0
    (0x3C, 1.0078125, 0x3FC2),  # 1.5 * 129/128 = 1.51171875 = 193.5 ulps: tie, odd -> up (1.515625)
])
def test_dequant_rounds_to_nearest_even(oracle_mod, code, scale, bits):
    row = _row({0: code}, (scale, 1.0, 1.0, 1.0), {})
    assert oracle_mod.dequant_fp8(row[None])[0, 0] == bits


# ---------------------------------------------------------------------------
# random rows against torch's decoding and rounding
# ---------------------------------------------------------------------------


def _torch_dequant(rows: np.ndarray) -> torch.Tensor:
    """Library path: e4m3 -> float32 (torch), float32 product, -> bfloat16 (torch RNE)."""
    r = torch.from_numpy(np.ascontiguousarray(rows).reshape(-1, 656))
    lat = r[:, :512].contiguous().view(torch.float8_e4m3fn).to(torch.float32)
    sc = r[:, 512:528].contiguous().view(torch.float32)                 # [n, 4]
    deq = (lat.view(-1, 4, 128) * sc[:, :, None]).view(-1, 512).to(torch.bfloat16)
    rope = r[:, 528:].contiguous().view(torch.bfloat16)
    return torch.cat([deq, rope], 1)


def test_dequant_random_rows_match_torch(oracle_mod):
    rng = np.random.default_rng(31)
    rows = W._fp8_rows(rng, 300)
    # wider scales too: fp32 scales with full 24-bit significands, tiny and large
    sc = (rng.standard_normal((300, 4)) * np.exp2(rng.integers(-20, 6, (300, 4)))).astype("<f4")
    rows[150:, 512:528] = sc[150:].view(np.uint8)
    got = oracle_mod.dequant_fp8(rows)
    ref = _torch_dequant(rows).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------------------
# attention over the FP8 cache
# ---------------------------------------------------------------------------

FP8_BRUTE_CASES = [
    dict(seqlens=[256, 193], s_q=1, h_q=16),
    dict(seqlens=[65, 1, 130], s_q=2, h_q=8, causal=True),
    dict(seqlens=[77, 129], s_q=1, h_q=8, h_kv=2),
]


def _brute_fp8(p):
    q = torch.from_numpy(p.q.view(np.int16)).view(torch.bfloat16).double()
    kv = _torch_dequant(p.kvcache).double().view(p.num_blocks, 64, p.h_kv, 576)
    B, S, H, D = q.shape
    o = torch.zeros(B, S, H, 512, dtype=torch.float64)
    lse = torch.full((B, S, H), -math.inf, dtype=torch.float64)
    group = H // p.h_kv
    vis = p.visible()
    for b in range(B):
        L = int(p.cache_seqlens[b])
        pages = torch.as_tensor(p.block_table[b, [j // 64 for j in range(L)]].astype(np.int64))
        offs = torch.arange(L) % 64
        for g in range(p.h_kv):
            K = kv[pages, offs, g]                                  # [L, 576]
            for s in range(S):
                n = int(vis[b, s])
                if n == 0:
                    continue
                logits = (q[b, s, g * group:(g + 1) * group] @ K[:n].T) * p.scale
                lse[b, s, g * group:(g + 1) * group] = torch.logsumexp(logits, -1)
                o[b, s, g * group:(g + 1) * group] = torch.softmax(logits, -1) @ K[:n, :512]
    return o.numpy(), lse.numpy()


@pytest.mark.parametrize("kw", FP8_BRUTE_CASES, ids=lambda k: str(k["seqlens"]))
def test_fp8_decode_brute_force_torch(oracle_mod, kw):
    p = W.make_problem(seed=41, fp8_kv=True, **kw)
    o, lse = oracle_mod.decode_fp8(p.q, p.kvcache, p.block_table, p.cache_seqlens,
                                   causal=p.causal, scale=p.scale)
    ob, lb = _brute_fp8(p)
    np.testing.assert_allclose(o, ob, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=1e-12, atol=1e-12)


def test_fp8_nan_in_unused_rows_changes_nothing(oracle_mod):
    kw = dict(s_q=2, h_q=8, causal=True, seed=42, fp8_kv=True, extra_pages=3)
    clean = W.make_problem([100, 63, 1], **kw)
    dirty = W.make_problem([100, 63, 1], poison=True, **kw)
    assert (dirty.kvcache == 0xFF).any()
    a = oracle_mod.decode_fp8(clean.q, clean.kvcache, clean.block_table, clean.cache_seqlens,
                              causal=True, scale=clean.scale)
    b = oracle_mod.decode_fp8(dirty.q, dirty.kvcache, dirty.block_table, dirty.cache_seqlens,
                              causal=True, scale=dirty.scale)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_fp8_decode_rows_matches_decode(oracle_mod):
    p = W.make_problem([90, 200], s_q=1, h_q=16, seed=43, fp8_kv=True)
    o, lse = oracle_mod.decode_fp8(p.q, p.kvcache, p.block_table, p.cache_seqlens, scale=p.scale)
    ids = np.array([0, 5, 17, 31])
    ro, rl = oracle_mod.decode_rows_fp8(p.q, p.kvcache, p.block_table, p.cache_seqlens, ids,
                                        scale=p.scale)
    assert np.array_equal(ro, o.reshape(-1, 512)[ids]) and np.array_equal(rl, lse.reshape(-1)[ids])


# ---------------------------------------------------------------------------
# the seeded FP8 cache generator (shared input module): recipe and poisoning
# ---------------------------------------------------------------------------


def test_fp8_generator_recipe():
    rng = np.random.default_rng(7)
    rows = W._fp8_rows(rng, 4000)
    lat = rows[:, :512]
    assert not np.any((lat & 0x7F) == 0x7F), "no e4m3 NaN codes in drawn rows"
    sc = rows[:, 512:528].copy().view("<f4")
    assert np.all((sc >= 2.0 ** -8) & (sc < 2.0 ** -7))
    vals = torch.from_numpy(np.ascontiguousarray(lat)).view(torch.float8_e4m3fn).float().numpy()
    deq = np.abs(vals.reshape(-1, 4, 128) * sc[:, :, None])
    assert deq.max() <= 3.5 and 0.5 < deq.mean() < 1.1
    rope = torch.from_numpy(rows[:, 528:].copy().view(np.int16)).view(torch.bfloat16).float().numpy()
    assert abs(rope.std() - 1.0) < 0.05


def test_fp8_problem_poison_marks_only_never_visible_rows():
    p = W.make_problem([100, 64, 1], s_q=1, h_q=8, fp8_kv=True, poison=True, extra_pages=2, seed=9)
    assert p.kvcache.shape[-1] == 656 and p.kvcache.dtype == np.uint8
    for b, L in enumerate(p.cache_seqlens):
        for j in range(int(L)):
            row = p.kvcache[p.block_table[b, j // 64], j % 64, 0]
            assert not np.all(row == 0xFF)
        if L % 64:
            tail = p.kvcache[p.block_table[b, (L - 1) // 64], L % 64:, 0]
            assert np.all(tail == 0xFF)
    assert p.kv_row_bytes() == 656 and p.kv_bytes() == 165 * 656
