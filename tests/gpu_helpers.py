"""Shared helpers for the GPU parity tests: move a seeded problem to the device,
run it through the C ABI, and compare with the FP64 oracle under the stated
tolerances."""
from __future__ import annotations

import numpy as np
import torch

import mla_decode_attention_12_b200 as mla
from mla_decode_attention_12_b200 import workloads as W

# Tolerances: max |dO| <= 2e-2, max |dLSE| <= 1e-2 for 16-bit inputs, and the
# mean absolute error of O no worse than 2x that of the FP64 result rounded to
# the output dtype (the "not worse than production" MAE rule of the
# "FlashMLA vLLM Optimization" page, validation section).
O_MAX_ABS = 2e-2
LSE_MAX_ABS = 1e-2
MAE_FACTOR = 2.0


def tdtype(dtype: int):
    return torch.bfloat16 if dtype == W.BF16 else torch.float16


def to_device(p: W.Problem, device="cuda"):
    dt = tdtype(p.dtype)
    q = torch.from_numpy(p.q.view(np.int16)).view(dt).to(device)
    if p.fp8_kv:  # "FP8 with scale" rows stay bytes
        kv = torch.from_numpy(p.kvcache).to(device)
    else:
        kv = torch.from_numpy(p.kvcache.view(np.int16)).view(dt).to(device)
    bt = torch.from_numpy(p.block_table).to(device)
    sl = torch.from_numpy(p.cache_seqlens).to(device)
    return q, kv, bt, sl


def run_gpu(p: W.Problem, device="cuda", num_parts=None, check_status=True):
    q, kv, bt, sl = to_device(p, device)
    md, ns = mla.get_mla_metadata(sl, p.s_q * p.h_q // p.h_kv, p.h_kv, is_fp8_kvcache=p.fp8_kv, num_parts=num_parts)
    ws = torch.zeros(mla.workspace_bytes(p.batch, p.s_q, p.h_q, p.h_kv, md.shape[0]), dtype=torch.uint8,
                     device=device)
    o, lse = mla.flash_mla_with_kvcache(q, kv, bt, sl, p.dv, md, ns, causal=p.causal, softmax_scale=p.scale,
                                        workspace=ws, is_fp8_kvcache=p.fp8_kv)
    torch.cuda.synchronize()
    if check_status:
        st = mla.read_device_status(ws)
        assert st == 0, f"device status {st}"
    return o, lse, md, ns


def round_to(x: np.ndarray, dtype: int) -> np.ndarray:
    return torch.from_numpy(x).to(tdtype(dtype)).double().numpy()


def compare(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what=""):
    """Element-by-element check of GPU (torch) against oracle (numpy f64) results."""
    o = o_gpu.double().cpu().numpy().reshape(o_ref.shape)
    l = lse_gpu.double().cpu().numpy().reshape(lse_ref.shape)
    assert np.isfinite(o).all(), f"{what}: non-finite O"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(l), fin), f"{what}: LSE finiteness differs"
    assert np.all(l[~fin] == lse_ref[~fin]), f"{what}: empty rows must have LSE = -inf"
    d_o = np.abs(o - o_ref)
    d_l = np.abs(l[fin] - lse_ref[fin]) if fin.any() else np.zeros(1)
    mae = d_o.mean()
    mae_round = np.abs(round_to(o_ref, dtype) - o_ref).mean()
    info = (f"{what}: max|dO|={d_o.max():.3e} max|dLSE|={d_l.max():.3e} MAE={mae:.3e} "
            f"MAE(rounded oracle)={mae_round:.3e}")
    assert d_o.max() <= O_MAX_ABS, info
    assert d_l.max() <= LSE_MAX_ABS, info
    assert mae <= MAE_FACTOR * mae_round + 1e-7, info
    return info


def oracle_full(oracle_mod, p: W.Problem):
    """FP64 oracle result of a whole problem (16-bit or FP8 cache)."""
    if p.fp8_kv:
        return oracle_mod.decode_fp8(p.q, p.kvcache, p.block_table, p.cache_seqlens, dv=p.dv, causal=p.causal,
                                     scale=p.scale)
    return oracle_mod.decode(p.q, p.kvcache, p.block_table, p.cache_seqlens, dv=p.dv, dtype=p.dtype,
                             causal=p.causal, scale=p.scale)


def oracle_rows(oracle_mod, p: W.Problem, rows):
    """FP64 oracle result of selected flat rows (b * s_q + s) * h_q + h."""
    if p.fp8_kv:
        return oracle_mod.decode_rows_fp8(p.q, p.kvcache, p.block_table, p.cache_seqlens, rows, dv=p.dv,
                                          causal=p.causal, scale=p.scale)
    return oracle_mod.decode_rows(p.q, p.kvcache, p.block_table, p.cache_seqlens, rows, dv=p.dv, dtype=p.dtype,
                                  causal=p.causal, scale=p.scale)
