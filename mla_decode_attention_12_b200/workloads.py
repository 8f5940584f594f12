"""Seeded synthetic inputs for MLA decoding: the decode workloads and generic problems.

This module draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the CUDA path and the FP64 oracle can take their
inputs from it.  All arrays are numpy; 16-bit floats are returned as their raw
bit patterns (``uint16``) so that both sides see identical bytes.

Layouts (the ones the library's C ABI takes):

* ``q``            ``[batch, s_q, h_q, d_qk]`` 16-bit, row-major.
* ``kvcache``      ``[num_blocks, page_size, h_kv, d_qk]`` 16-bit; a token row is the
                   latent part (first 512 columns, also V) then the RoPE part.
* ``block_table``  ``[batch, max_blocks_per_seq]`` int32 physical page ids, a seeded
                   Fisher-Yates permutation of the pages; unused slots are -1.
* ``cache_seqlens`` ``[batch]`` int32.
* FP8 cache (``Problem.fp8_kv``): ``kvcache`` is ``[num_blocks, page_size, h_kv, 656]``
  uint8 in the "FP8 with scale" layout of the upstream FlashMLA documentation
  ("FP8 KV Cache"): 512 float8_e4m3 latent bytes, 4 little-endian float32 scales
  (one per 128 latent values), 64 bfloat16 RoPE values.  The generator draws the
  e4m3 bit fields and the scales directly (it does not quantize anything).

The workloads follow the decode configurations the pages benchmark (paged
cache with 64-token pages, MQA mode d_qk = 576 / d_v = 512, variable sequence
lengths; "FlashMLA" usage page and the upstream FlashMLA documentation,
"Performance" and "Usage / MLA Decoding").
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

PAGE = 64
BF16 = 0
FP16 = 1
FP8_ROW_BYTES = 656


@dataclasses.dataclass
class Problem:
    """One decode call's inputs (host arrays) plus its shape parameters."""

    name: str
    q: np.ndarray            # uint16 [b, s_q, h_q, d_qk]
    kvcache: np.ndarray      # uint16 [num_blocks, page, h_kv, d_qk]
    block_table: np.ndarray  # int32 [b, max_blocks]
    cache_seqlens: np.ndarray  # int32 [b]
    dtype: int               # 0 = bfloat16, 1 = float16
    causal: bool
    scale: float
    dv: int = 512
    page_size: int = PAGE
    active_heads: int | None = None  # heads >= this are zero-filled (padded heads)
    seed: int = 0
    fp8_kv: bool = False     # kvcache holds 656-byte "FP8 with scale" rows (uint8)
    indices: np.ndarray | None = None  # int32 [b, s_q, topk] flat cache rows (sparse decode), -1 invalid

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def s_q(self) -> int:
        return self.q.shape[1]

    @property
    def h_q(self) -> int:
        return self.q.shape[2]

    @property
    def d_qk(self) -> int:
        return self.q.shape[3]

    @property
    def h_kv(self) -> int:
        return self.kvcache.shape[2]

    @property
    def num_blocks(self) -> int:
        return self.kvcache.shape[0]

    def valid_entries(self) -> np.ndarray:
        """Sparse problems: [b, s_q, topk] bool, the entries inside the cache."""
        rows = self.num_blocks * self.page_size
        return (self.indices >= 0) & (self.indices < rows)

    def visible(self) -> np.ndarray:
        """[b, s_q] number of cached tokens each query token attends (causal: bottom-right;
        sparse: its valid entries)."""
        if self.indices is not None:
            return self.valid_entries().sum(axis=2).astype(np.int64)
        L = self.cache_seqlens.astype(np.int64)[:, None]
        if not self.causal:
            return np.broadcast_to(L, (self.batch, self.s_q)).copy()
        s = np.arange(self.s_q, dtype=np.int64)[None, :]
        return np.clip(L - self.s_q + 1 + s, 0, L)

    def flops(self) -> float:
        """2 * (d_qk + d_v) per visible (query row, key) pair, all heads."""
        return 2.0 * (self.d_qk + self.dv) * float(self.visible().sum()) * self.h_q

    def kv_row_bytes(self) -> int:
        """Bytes of one cached token row: d_qk 16-bit values, or 656 for the FP8 cache."""
        return FP8_ROW_BYTES if self.fp8_kv else self.d_qk * 2

    def kv_bytes(self) -> int:
        """Cached rows read once: sum_b L_b * h_kv * row bytes (sparse: every query token's
        valid entries, each read once for that token)."""
        if self.indices is not None:
            return int(self.valid_entries().sum()) * self.h_kv * self.kv_row_bytes()
        return int(self.cache_seqlens.astype(np.int64).sum()) * self.h_kv * self.kv_row_bytes()

    def io_bytes(self) -> int:
        """Algorithmic bytes: KV once + Q + O (16-bit) + LSE (fp32) (+ the entry lists)."""
        rows = self.batch * self.s_q * self.h_q
        extra = 0 if self.indices is None else self.indices.size * 4
        return self.kv_bytes() + rows * (self.d_qk * 2 + self.dv * 2 + 4) + extra


def _round_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """float32 -> 16-bit bit patterns (bfloat16 RNE or IEEE float16 RNE)."""
    if dtype == BF16:
        return _round_bf16_bits(x)
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def _normal_bits(rng: np.random.Generator, shape, std: float, dtype: int) -> np.ndarray:
    out = np.empty(shape, np.uint16)
    flat = out.reshape(-1)
    chunk = 1 << 24
    for i in range(0, flat.size, chunk):
        n = min(chunk, flat.size - i)
        x = rng.standard_normal(n, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        flat[i:i + n] = to_bits(x, dtype)
    return out


def _fp8_rows(rng: np.random.Generator, n: int) -> np.ndarray:
    """n random "FP8 with scale" token rows, uint8 [n, 656].

    Latent bytes: random sign, exponent field ~ round(N(13, 1.5)) clipped to
    [0, 15], uniform 3-bit fraction (the NaN pattern S.1111.111 is replaced by
    S.1111.110).  Scales (1 + U[0, 1)) * 2^-8, the range amax / 448 takes for a
    block of 128 N(0, 1) values, so the values are at most 3.5 in magnitude and
    mostly below 1, like a per-128-block quantized N(0, 1) latent.  RoPE: bfloat16
    N(0, 1).
    """
    rows = np.empty((n, FP8_ROW_BYTES), np.uint8)
    chunk = 1 << 16
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        sign = rng.integers(0, 2, size=(m, 512), dtype=np.uint8) << np.uint8(7)
        e = np.clip(np.rint(rng.normal(13.0, 1.5, size=(m, 512))), 0, 15).astype(np.uint8)
        f = rng.integers(0, 8, size=(m, 512), dtype=np.uint8)
        f[(e == 15) & (f == 7)] = 6
        rows[i:i + m, :512] = sign | (e << np.uint8(3)) | f
        scales = ((1.0 + rng.random((m, 4), dtype=np.float32)) * np.float32(2.0 ** -8)).astype("<f4")
        rows[i:i + m, 512:528] = scales.view(np.uint8)
        rope = _normal_bits(rng, (m, 64), 1.0, BF16).astype("<u2")
        rows[i:i + m, 528:] = rope.view(np.uint8)
    return rows


def make_problem(
    seqlens,
    *,
    s_q: int = 1,
    h_q: int = 16,
    d_qk: int = 576,
    h_kv: int = 1,
    dtype: int = BF16,
    causal: bool = False,
    std: float = 1.0,
    scale: float | None = None,
    seed: int = 0,
    active_heads: int | None = None,
    poison: bool = False,
    extra_pages: int = 0,
    extra_table_cols: int = 0,
    name: str = "problem",
    fp8_kv: bool = False,
) -> Problem:
    """Seeded problem with the given sequence lengths.

    ``poison`` fills what a correct kernel must never use with NaN: the tail
    rows of each sequence's last page and every page no sequence owns
    (``extra_pages`` of them).  Unused block-table slots are always -1.
    ``fp8_kv`` draws an "FP8 with scale" cache (bfloat16 q, d_qk = 576); its
    poison is all-ones bytes (NaN latent values, scales and RoPE values).
    """
    if fp8_kv and (dtype != BF16 or d_qk != 576):
        raise ValueError("the FP8 cache goes with bfloat16 queries and d_qk = 576")
    rng = np.random.Generator(np.random.PCG64(seed))
    seqlens = np.asarray(seqlens, dtype=np.int32)
    b = seqlens.size
    nblk = [(int(L) + PAGE - 1) // PAGE for L in seqlens]
    used = int(sum(nblk))
    num_blocks = max(1, used + extra_pages)
    max_blocks = max(1, max(nblk) if nblk else 1) + extra_table_cols

    q = _normal_bits(rng, (b, s_q, h_q, d_qk), std, dtype)
    if active_heads is not None and active_heads < h_q:
        q[:, :, active_heads:, :] = 0
    if fp8_kv:
        kv = _fp8_rows(rng, num_blocks * PAGE * h_kv).reshape(num_blocks, PAGE, h_kv, FP8_ROW_BYTES)
    else:
        kv = _normal_bits(rng, (num_blocks, PAGE, h_kv, d_qk), std, dtype)

    perm = rng.permutation(num_blocks).astype(np.int32)
    table = np.full((b, max_blocks), -1, np.int32)
    pos = 0
    for i, n in enumerate(nblk):
        table[i, :n] = perm[pos:pos + n]
        pos += n

    if poison:
        nan_bits = np.uint8(0xFF) if fp8_kv else np.uint16(0x7FC0) if dtype == BF16 else np.uint16(0x7E00)
        for i, L in enumerate(seqlens):
            n = nblk[i]
            if n and int(L) % PAGE:
                kv[table[i, n - 1], int(L) % PAGE:, :, :] = nan_bits
        for p in perm[pos:]:
            kv[p] = nan_bits

    if scale is None:
        scale = 1.0 / math.sqrt(d_qk)
    return Problem(name=name, q=q, kvcache=kv, block_table=table, cache_seqlens=seqlens,
                   dtype=dtype, causal=causal, scale=float(scale), active_heads=active_heads,
                   seed=seed, fp8_kv=fp8_kv)


def make_sparse_problem(seqlens, topk: int, *, s_q: int = 1, invalid_frac: float = 0.0, **kw) -> Problem:
    """A paged-cache problem plus, per query token, `topk` attended rows of its own sequence.

    Each query token's entries are distinct positions of its request's cached tokens drawn
    uniformly (all of them, in random order, when the sequence is shorter than topk), mapped to
    flat rows page * 64 + offset through the block table; the remaining slots and a random
    `invalid_frac` of the drawn ones are -1.  Everything else is as in :func:`make_problem`
    (causal stays off: the list is what each query sees).
    """
    p = make_problem(seqlens, s_q=s_q, **kw)
    rng = np.random.Generator(np.random.PCG64(p.seed + 7877))
    idx = np.full((p.batch, s_q, topk), -1, np.int32)
    for b, L in enumerate(p.cache_seqlens):
        L = int(L)
        for s in range(s_q):
            n = min(L, topk)
            if n == 0:
                continue
            j = rng.choice(L, size=n, replace=False)
            rows = p.block_table[b, j // PAGE].astype(np.int64) * PAGE + j % PAGE
            if invalid_frac > 0:
                rows[rng.random(n) < invalid_frac] = -1
            idx[b, s, :n] = rows
    p.indices = idx
    return p


@dataclasses.dataclass
class PrefillProblem:
    """Sparse MLA prefill inputs: q [s_q, h_q, d_qk], kv [s_kv, 1, d_qk] (16-bit bit patterns),
    indices int32 [s_q, 1, topk] (-1 or >= s_kv invalid)."""

    name: str
    q: np.ndarray
    kv: np.ndarray
    indices: np.ndarray
    sm_scale: float
    dtype: int = BF16
    dv: int = 512
    seed: int = 0

    @property
    def s_q(self) -> int:
        return self.q.shape[0]

    @property
    def h_q(self) -> int:
        return self.q.shape[1]

    @property
    def d_qk(self) -> int:
        return self.q.shape[2]

    @property
    def s_kv(self) -> int:
        return self.kv.shape[0]

    def valid_entries(self) -> np.ndarray:
        return (self.indices >= 0) & (self.indices < self.s_kv)

    def flops(self) -> float:
        """2 * (d_qk + d_v) per (query row, valid entry) pair."""
        return 2.0 * (self.d_qk + self.dv) * float(self.valid_entries().sum()) * self.h_q

    active_heads = None
    fp8_kv = False

    def kv_bytes(self) -> int:
        """The kv rows, once: every token's entries are rows of the same (L2-sized) kv."""
        return self.s_kv * self.d_qk * 2

    def gathered_bytes(self) -> int:
        """The rows the query tokens' valid entries name, one read per entry."""
        return int(self.valid_entries().sum()) * self.d_qk * 2

    def io_bytes(self) -> int:
        """Algorithmic bytes: q, the kv once, out (16-bit), lse and max_logits, the lists."""
        rows = self.s_q * self.h_q
        return self.kv_bytes() + rows * (self.d_qk * 2 + self.dv * 2 + 8) + self.indices.size * 4


def make_prefill_problem(s_q: int, h_q: int, s_kv: int, topk: int, *, d_qk: int = 576, dtype: int = BF16,
                         invalid_frac: float = 0.0, seed: int = 0, name: str = "prefill") -> PrefillProblem:
    """Seeded sparse-prefill inputs: N(0, 1) q and kv, and for every query token `topk` distinct
    kv rows drawn uniformly (all of them, shuffled, when s_kv < topk; the rest -1), a random
    `invalid_frac` of which become -1 or a row past the end."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _normal_bits(rng, (s_q, h_q, d_qk), 1.0, dtype)
    kv = _normal_bits(rng, (s_kv, 1, d_qk), 1.0, dtype)
    ind = np.full((s_q, 1, topk), -1, np.int32)
    n = min(s_kv, topk)
    for i in range(s_q):
        ind[i, 0, :n] = rng.choice(s_kv, size=n, replace=False)
    if invalid_frac > 0:
        bad = rng.random(ind.shape) < invalid_frac
        past = s_kv + rng.integers(0, 1000, ind.shape)
        ind[bad] = np.where(rng.random(ind.shape) < 0.5, -1, past)[bad]
    return PrefillProblem(name=name, q=q, kv=kv, indices=ind, sm_scale=1.0 / math.sqrt(d_qk), dtype=dtype, seed=seed)


PREFILL_WORKLOADS = ("sparse_prefill",)


def make_prefill_workload(name: str) -> PrefillProblem:
    """The sparse-prefill workload: 2048 query tokens of 128 heads, each attending 2048 of 16384
    kv rows (bf16 N(0, 1), sm_scale 1 / sqrt(576))."""
    if name != "sparse_prefill":
        raise KeyError(name)
    k = len(WORKLOADS) + len(SPARSE_WORKLOADS) + 1
    return make_prefill_problem(2048, 128, 16384, 2048, seed=1000 + k, name=name)


# ----------------------------------------------------------------------------
# The decode workloads: the five decode configurations, and the compute one over an
# FP8 cache.  Workload k (1-based position in WORKLOADS) draws from seed 1000 + k.
# ----------------------------------------------------------------------------

WORKLOADS = ("tiny", "compute", "spec_padded", "long_split", "fp16_norope", "fp8_compute")
# Token-level sparse decode over an FP8 cache (its own path: indices instead of a block table).
SPARSE_WORKLOADS = ("sparse_fp8",)


def workload_seqlens(name: str, rng: np.random.Generator) -> np.ndarray:
    if name == "tiny":
        return np.array([256, 193], np.int32)
    if name in ("compute", "fp8_compute"):
        return rng.integers(1024, 8192, size=64, endpoint=True).astype(np.int32)
    if name == "sparse_fp8":
        return rng.integers(8192, 16384, size=64, endpoint=True).astype(np.int32)
    if name == "spec_padded":
        return rng.integers(4096 - 512, 4096 + 512, size=128, endpoint=True).astype(np.int32)
    if name == "long_split":
        return np.array([65536, 49152, 32768, 8192], np.int32)
    if name == "fp16_norope":
        u = rng.uniform(math.log(512), math.log(16384), size=32)
        return np.floor(np.exp(u)).astype(np.int32)
    raise KeyError(name)


def make_workload(name: str, *, poison: bool = False, seqlens=None) -> Problem:
    """One of the decode workloads (synthetic data, fixed seed 1000 + index).

    ``seqlens`` overrides the sequence lengths (for scaled-down parity cases with
    the same head / dtype / mask structure).
    """
    k = (WORKLOADS + SPARSE_WORKLOADS).index(name) + 1
    seed = 1000 + k
    rng = np.random.Generator(np.random.PCG64(seed + 7919))
    L = workload_seqlens(name, rng) if seqlens is None else np.asarray(seqlens, np.int32)
    common = dict(seed=seed, poison=poison, name=name)
    if name == "tiny":
        return make_problem(L, s_q=1, h_q=16, d_qk=576, **common)
    if name == "compute":
        return make_problem(L, s_q=1, h_q=128, d_qk=576, **common)
    if name == "spec_padded":
        return make_problem(L, s_q=2, h_q=64, d_qk=576, causal=True, active_heads=16, **common)
    if name == "long_split":
        return make_problem(L, s_q=1, h_q=128, d_qk=576, **common)
    if name == "fp16_norope":
        return make_problem(L, s_q=4, h_q=64, d_qk=512, causal=True, dtype=FP16, std=0.5,
                            **common)
    if name == "fp8_compute":
        return make_problem(L, s_q=1, h_q=128, d_qk=576, fp8_kv=True, **common)
    if name == "sparse_fp8":
        return make_sparse_problem(L, 2048, s_q=2, h_q=128, fp8_kv=True, **common)
    raise KeyError(name)
