"""FP64 CPU oracle for MLA decoding over a paged latent KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``mla_decode_attention_12_b200``) never imports it and shares no code with it.

The arithmetic lives in ``mla_oracle.c`` (plain C, fp64, OpenMP over rows); this
module compiles it with gcc on first use and wraps it with numpy.

Functions and the passages they follow (page title, section):

* :func:`decode` -- the plain definition of ``flash_mla_with_kvcache``: the
  "FlashMLA" usage page (deepep.org) call and its three stages, the upstream
  FlashMLA documentation "Usage / MLA Decoding" return values (out, lse), its
  "MLA Mode" footnote (d_qk = 576, d_v = 512) and its FP8-format section (a
  token row is the 512 latent columns followed by the 64 RoPE columns, so V is
  the leading d_v columns).
* :func:`decode_range` -- the same over a token sub-range; the partial results
  that split-KV produces ("FlashMLA vLLM Optimization", background section:
  the split-KV and combine kernels).
* :func:`combine` -- the log-sum-exp merge of such partials.
* :func:`decode_rows` -- :func:`decode` for selected rows of a large problem.
* :func:`half_bits_to_float64` -- exact decoding of bfloat16 / float16 bits.
* :func:`e4m3_to_float64`, :func:`dequant_fp8` -- the "FP8 with scale" KV cache
  of the upstream FlashMLA documentation ("FP8 KV Cache" section, reproduced on
  the "FlashMLA vLLM Optimization" page): 656-byte token rows of 512
  float8_e4m3 latent values, 4 float32 scales and 64 bfloat16 RoPE values,
  dequantized to bfloat16.
* :func:`sparse_prefill` -- the sparse MLA prefill (upstream FlashMLA documentation,
  "Sparse MLA Prefill"): out, base-2 max_logits and base-2 lse over per-query index lists
  into a flat kv.
* :func:`decode_sparse`, :func:`decode_sparse_fp8` -- token-level sparse decoding (the
  upstream FlashMLA documentation's "Sparse Attention (indices tensor)"): each query
  token attends the flat cache rows (page * page_size + offset) listed in
  ``indices[b, s, :topk]``; -1 (or any row past the cache) is an invalid entry.
* :func:`decode_fp8`, :func:`decode_rows_fp8` -- attention over such a cache:
  the page says the kernel dequantizes the cache to bfloat16 and computes in
  bfloat16, so this is :func:`decode` of the dequantized rows.

Every function here is pinned by tests in ``tests/test_oracle_pins.py`` against
closed forms, brute force through an independent library path, invariants and
hand-worked cases.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB = os.path.join(_HERE, "_mla_oracle.so")
_lock = threading.Lock()
_lib = None

BF16 = 0
FP16 = 1


class _Shape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("s_q", ctypes.c_int),
        ("h_q", ctypes.c_int),
        ("h_kv", ctypes.c_int),
        ("d_qk", ctypes.c_int),
        ("dv", ctypes.c_int),
        ("page_size", ctypes.c_int),
        ("max_blocks_per_seq", ctypes.c_int),
        ("num_blocks", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("causal", ctypes.c_int),
        ("scale", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile ``mla_oracle.c`` into ``_mla_oracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            lib.mla_oracle_decode.argtypes = [ctypes.POINTER(_Shape), P, P, P, P, P, P]
            lib.mla_oracle_decode.restype = ctypes.c_int
            lib.mla_oracle_decode_range.argtypes = [
                ctypes.POINTER(_Shape), P, P, P, P, ctypes.c_long, ctypes.c_long, P, P]
            lib.mla_oracle_decode_range.restype = ctypes.c_int
            lib.mla_oracle_decode_rows.argtypes = [
                ctypes.POINTER(_Shape), P, P, P, P, P, ctypes.c_long, P, P]
            lib.mla_oracle_decode_rows.restype = ctypes.c_int
            lib.mla_oracle_combine.argtypes = [
                ctypes.c_int, ctypes.c_long, ctypes.c_int, P, P, P, P]
            lib.mla_oracle_combine.restype = None
            lib.mla_oracle_half_to_double.argtypes = [ctypes.c_uint16, ctypes.c_int]
            lib.mla_oracle_half_to_double.restype = ctypes.c_double
            lib.mla_oracle_decode_sparse.argtypes = [ctypes.POINTER(_Shape), P, P, P, ctypes.c_int, P, P]
            lib.mla_oracle_decode_sparse.restype = ctypes.c_int
            I = ctypes.c_int
            lib.mla_oracle_sparse_prefill.argtypes = [I, I, I, I, I, ctypes.c_long, I, I, ctypes.c_double,
                                                      P, P, P, P, P, P]
            lib.mla_oracle_sparse_prefill.restype = ctypes.c_int
            lib.mla_oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.mla_oracle_e4m3_to_double.restype = ctypes.c_double
            lib.mla_oracle_dequant_fp8_rows.argtypes = [P, ctypes.c_long, P]
            lib.mla_oracle_dequant_fp8_rows.restype = None
            lib.mla_oracle_num_threads.argtypes = []
            lib.mla_oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


class use_library:
    """Context manager: route this module's calls through another build of the
    oracle source (the mutation tests compile deliberately broken copies)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        _load()
        self._saved = _lib
        lib = ctypes.CDLL(self.path)
        for name in ("mla_oracle_decode", "mla_oracle_decode_range", "mla_oracle_decode_rows",
                     "mla_oracle_combine", "mla_oracle_half_to_double", "mla_oracle_num_threads",
                     "mla_oracle_e4m3_to_double", "mla_oracle_dequant_fp8_rows", "mla_oracle_decode_sparse",
                     "mla_oracle_sparse_prefill"):
            src = getattr(self._saved, name)
            dst = getattr(lib, name)
            dst.argtypes, dst.restype = src.argtypes, src.restype
        _lib = lib
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def num_threads() -> int:
    """OpenMP threads the oracle uses (``OMP_NUM_THREADS`` or all cores)."""
    return int(_load().mla_oracle_num_threads())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _prep(q_bits, kv_bits, block_table, seqlens, dv, dtype, causal, scale, page_size):
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kv_bits = np.ascontiguousarray(kv_bits, dtype=np.uint16)
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    if q_bits.ndim != 4 or kv_bits.ndim != 4:
        raise ValueError("q must be [b, s_q, h_q, d_qk] and kvcache [blocks, page, h_kv, d_qk]")
    b, s_q, h_q, d_qk = q_bits.shape
    nb, ps, h_kv, d_k2 = kv_bits.shape
    if d_k2 != d_qk or ps != page_size:
        raise ValueError("kvcache shape does not match q / page_size")
    if block_table.shape[0] != b or seqlens.shape != (b,):
        raise ValueError("block_table / cache_seqlens batch mismatch")
    if h_q % h_kv:
        raise ValueError("h_q must be a multiple of h_kv")
    if scale is None:
        scale = 1.0 / np.sqrt(d_qk)
    sh = _Shape(b, s_q, h_q, h_kv, d_qk, dv, page_size, block_table.shape[1], nb,
                dtype, int(bool(causal)), float(scale))
    return sh, q_bits, kv_bits, block_table, seqlens


def decode(q_bits, kv_bits, block_table, seqlens, dv=512, dtype=BF16, causal=False,
           scale=None, page_size=64):
    """Full attention.  Returns (O [b,s_q,h_q,dv] f64, LSE [b,s_q,h_q] f64, natural log)."""
    sh, q_bits, kv_bits, block_table, seqlens = _prep(
        q_bits, kv_bits, block_table, seqlens, dv, dtype, causal, scale, page_size)
    o = np.empty((sh.batch, sh.s_q, sh.h_q, dv), np.float64)
    lse = np.empty((sh.batch, sh.s_q, sh.h_q), np.float64)
    rc = _load().mla_oracle_decode(ctypes.byref(sh), _ptr(q_bits), _ptr(kv_bits),
                                   _ptr(block_table), _ptr(seqlens), _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle rejected its arguments")
    return o, lse


def decode_range(q_bits, kv_bits, block_table, seqlens, lo, hi, dv=512, dtype=BF16,
                 causal=False, scale=None, page_size=64):
    """Attention restricted to cached tokens lo <= j < hi (clipped to what each row sees)."""
    sh, q_bits, kv_bits, block_table, seqlens = _prep(
        q_bits, kv_bits, block_table, seqlens, dv, dtype, causal, scale, page_size)
    o = np.empty((sh.batch, sh.s_q, sh.h_q, dv), np.float64)
    lse = np.empty((sh.batch, sh.s_q, sh.h_q), np.float64)
    rc = _load().mla_oracle_decode_range(ctypes.byref(sh), _ptr(q_bits), _ptr(kv_bits),
                                         _ptr(block_table), _ptr(seqlens), int(lo), int(hi),
                                         _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle rejected its arguments")
    return o, lse


def decode_rows(q_bits, kv_bits, block_table, seqlens, row_ids, dv=512, dtype=BF16,
                causal=False, scale=None, page_size=64):
    """Attention for flat rows r = (b*s_q + s)*h_q + h only.  Returns (O [n,dv], LSE [n])."""
    sh, q_bits, kv_bits, block_table, seqlens = _prep(
        q_bits, kv_bits, block_table, seqlens, dv, dtype, causal, scale, page_size)
    row_ids = np.ascontiguousarray(row_ids, dtype=np.int64)
    o = np.empty((row_ids.size, dv), np.float64)
    lse = np.empty((row_ids.size,), np.float64)
    rc = _load().mla_oracle_decode_rows(ctypes.byref(sh), _ptr(q_bits), _ptr(kv_bits),
                                        _ptr(block_table), _ptr(seqlens), _ptr(row_ids),
                                        row_ids.size, _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle rejected its arguments")
    return o, lse


def combine(o_parts, lse_parts):
    """Merge partials over disjoint token ranges: o_parts [k, ..., dv], lse_parts [k, ...]."""
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    k = o_parts.shape[0]
    dv = o_parts.shape[-1]
    lead = lse_parts.shape[1:]
    rows = int(np.prod(lead)) if lead else 1
    o = np.empty(lead + (dv,), np.float64)
    lse = np.empty(lead, np.float64)
    _load().mla_oracle_combine(k, rows, dv, _ptr(o_parts), _ptr(lse_parts), _ptr(o), _ptr(lse))
    return o, lse


def half_bits_to_float64(bits, dtype=BF16) -> np.ndarray:
    """Decode bfloat16 (dtype 0) or float16 (dtype 1) bit patterns exactly."""
    bits = np.asarray(bits, dtype=np.uint16)
    f = _load().mla_oracle_half_to_double
    flat = [f(int(x), dtype) for x in bits.ravel()]
    return np.array(flat, dtype=np.float64).reshape(bits.shape)


FP8_ROW_BYTES = 656  # bytes per token of the "FP8 with scale" cache


def e4m3_to_float64(codes) -> np.ndarray:
    """Decode float8_e4m3 bytes exactly (NaN for S.1111.111)."""
    codes = np.asarray(codes, dtype=np.uint8)
    f = _load().mla_oracle_e4m3_to_double
    return np.array([f(int(x)) for x in codes.ravel()], dtype=np.float64).reshape(codes.shape)


def dequant_fp8(kv_u8) -> np.ndarray:
    """Dequantize an "FP8 with scale" cache [..., 656] uint8 into bfloat16 bits [..., 576]."""
    kv_u8 = np.ascontiguousarray(kv_u8, dtype=np.uint8)
    if kv_u8.shape[-1] != FP8_ROW_BYTES:
        raise ValueError("an FP8 cache row is 656 bytes")
    n = kv_u8.size // FP8_ROW_BYTES
    out = np.empty(kv_u8.shape[:-1] + (576,), np.uint16)
    _load().mla_oracle_dequant_fp8_rows(_ptr(kv_u8), n, _ptr(out))
    return out


def decode_fp8(q_bits, kv_u8, block_table, seqlens, dv=512, causal=False, scale=None, page_size=64):
    """Attention over an "FP8 with scale" cache: bfloat16 q, out; d_qk = 576."""
    return decode(q_bits, dequant_fp8(kv_u8), block_table, seqlens, dv, BF16, causal, scale, page_size)


def decode_rows_fp8(q_bits, kv_u8, block_table, seqlens, row_ids, dv=512, causal=False, scale=None,
                    page_size=64):
    """:func:`decode_rows` over an "FP8 with scale" cache."""
    return decode_rows(q_bits, dequant_fp8(kv_u8), block_table, seqlens, row_ids, dv, BF16, causal,
                       scale, page_size)


def decode_sparse(q_bits, kv_bits, indices, dv=512, dtype=BF16, scale=None, page_size=64):
    """Sparse attention over listed cache rows.  Returns (O [b,s_q,h_q,dv] f64, LSE [b,s_q,h_q] f64).

    ``indices`` [b, s_q, topk] int32 flat row indices (page * page_size + offset); entries
    outside the cache (-1 included) are invalid.  Each valid entry is one term (repeats count).
    """
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kv_bits = np.ascontiguousarray(kv_bits, dtype=np.uint16)
    indices = np.ascontiguousarray(indices, dtype=np.int32)
    if q_bits.ndim != 4 or kv_bits.ndim != 4 or indices.ndim != 3:
        raise ValueError("q [b,s_q,h_q,d_qk], kvcache [blocks,page,h_kv,d_qk], indices [b,s_q,topk]")
    b, s_q, h_q, d_qk = q_bits.shape
    nb, ps, h_kv, d2 = kv_bits.shape
    if d2 != d_qk or ps != page_size or indices.shape[:2] != (b, s_q) or h_q % h_kv:
        raise ValueError("shape mismatch")
    if scale is None:
        scale = 1.0 / np.sqrt(d_qk)
    sh = _Shape(b, s_q, h_q, h_kv, d_qk, dv, page_size, 1, nb, dtype, 0, float(scale))
    o = np.empty((b, s_q, h_q, dv), np.float64)
    lse = np.empty((b, s_q, h_q), np.float64)
    rc = _load().mla_oracle_decode_sparse(ctypes.byref(sh), _ptr(q_bits), _ptr(kv_bits), _ptr(indices),
                                          int(indices.shape[2]), _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle rejected its arguments")
    return o, lse


def decode_sparse_fp8(q_bits, kv_u8, indices, dv=512, scale=None, page_size=64):
    """:func:`decode_sparse` over an "FP8 with scale" cache (dequantized first)."""
    return decode_sparse(q_bits, dequant_fp8(kv_u8), indices, dv, BF16, scale, page_size)


def sparse_prefill(q_bits, kv_bits, indices, sm_scale, dv=512, dtype=BF16):
    """Sparse MLA prefill (upstream FlashMLA documentation, "Sparse MLA Prefill").

    ``q_bits`` [s_q, h_q, d_qk], ``kv_bits`` [s_kv, h_kv, d_qk] (16-bit bit patterns),
    ``indices`` [s_q, h_kv, topk] int32 (-1 or any index >= s_kv is invalid).  Returns
    ``(out [s_q, h_q, dv], max_logits [s_q, h_q], lse [s_q, h_q])`` in float64, with
    max_logits and lse in base 2 of the logits scaled by sm_scale * log2(e).
    """
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kv_bits = np.ascontiguousarray(kv_bits, dtype=np.uint16)
    indices = np.ascontiguousarray(indices, dtype=np.int32)
    if q_bits.ndim != 3 or kv_bits.ndim != 3 or indices.ndim != 3:
        raise ValueError("q [s_q,h_q,d_qk], kv [s_kv,h_kv,d_qk], indices [s_q,h_kv,topk]")
    s_q, h_q, d_qk = q_bits.shape
    s_kv, h_kv, d2 = kv_bits.shape
    if d2 != d_qk or indices.shape[:2] != (s_q, h_kv):
        raise ValueError("shape mismatch")
    out = np.empty((s_q, h_q, dv), np.float64)
    mx = np.empty((s_q, h_q), np.float64)
    lse = np.empty((s_q, h_q), np.float64)
    rc = _load().mla_oracle_sparse_prefill(s_q, h_q, h_kv, d_qk, dv, s_kv, int(indices.shape[2]), dtype,
                                           float(sm_scale), _ptr(q_bits), _ptr(kv_bits), _ptr(indices),
                                           _ptr(out), _ptr(mx), _ptr(lse))
    if rc:
        raise ValueError("oracle rejected its arguments")
    return out, mx, lse
