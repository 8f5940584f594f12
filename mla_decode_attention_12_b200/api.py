"""PyTorch-facing calls with the names of the pages' API.

``get_mla_metadata`` and ``flash_mla_with_kvcache`` follow the call sequence of
the "FlashMLA" usage page (deepep.org): metadata once per decoding step, then
one decode call per layer returning ``(o, lse)``.  Torch provides device memory
and the current stream; the arithmetic is done by the C library's kernels.

Inputs on the CPU are accepted too: they are copied to the current CUDA device
(non-blocking from pinned memory), the kernels run there, and the outputs are
copied back.  This is the end-to-end path with host buffers.
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _lib

_DTYPES = {torch.bfloat16: 0, torch.float16: 1}
MLA_BF16_FP8KV = 2   # bfloat16 q / o over an "FP8 with scale" cache (656-byte rows)
FP8_ROW_BYTES = 656
_workspaces: dict = {}


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def num_sm_parts(device=None) -> int:
    """Scheduler partitions of a device (one per pair of SMs)."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else torch.device(device).index or 0)
    out = ctypes.c_int(0)
    _lib.check(_lib.load().mla_num_sm_parts(dev.index, ctypes.byref(out)), "mla_num_sm_parts")
    return out.value


def metadata_sizes(batch: int, heads_per_kv: int, h_kv: int, num_parts: int):
    a, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _lib.check(_lib.load().mla_metadata_sizes(batch, heads_per_kv, h_kv, num_parts, ctypes.byref(a),
                                              ctypes.byref(b)), "mla_metadata_sizes")
    return a.value, b.value


def get_mla_metadata(cache_seqlens: torch.Tensor, heads_per_kv: int, h_kv: int = 1, h_q: int | None = None,
                     is_fp8_kvcache: bool = False, topk: int | None = None, *, num_parts: int | None = None,
                     out=None):
    """Tile-scheduler metadata for one decoding step.

    The arguments follow the upstream FlashMLA documentation's call ("Usage / MLA
    Decoding": ``get_mla_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv, h_q, is_fp8,
    topk)``).  ``cache_seqlens``: int32 [batch] on a CUDA device.  ``heads_per_kv`` is
    ``s_q * h_q // h_kv``.  ``is_fp8_kvcache``: the decode calls read an "FP8 with scale"
    cache (a schedule tuned for its slower pages; any schedule is valid for either cache).
    Returns ``(tile_scheduler_metadata [num_parts, 8] int32, num_splits [batch *
    ceil(heads_per_kv / 128) + 1] int32)`` on the same device; ``out`` = (md, ns) writes
    into existing tensors instead.

    With ``topk`` (and ``h_q``): the schedule of the token-level sparse decode, whose
    batch * s_q query tokens each attend ``topk`` listed entries (upstream FlashMLA
    documentation, "Sparse Attention (indices tensor)"); num_splits then has
    ``batch * s_q * ceil(h_q / h_kv / 128) + 1`` entries.
    """
    if not cache_seqlens.is_cuda or cache_seqlens.dtype != torch.int32 or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous int32 CUDA tensor")
    dev = cache_seqlens.device
    if out is not None and num_parts is None:
        num_parts = out[0].shape[0]
    if num_parts is None:
        num_parts = num_sm_parts(dev)
    batch = cache_seqlens.numel()
    if topk is not None:
        if h_q is None or (heads_per_kv * h_kv) % h_q:
            raise ValueError("the sparse schedule needs h_q, a divisor of heads_per_kv * h_kv")
        tokens = batch * (heads_per_kv * h_kv // h_q)
        n_md, n_ns = metadata_sizes(tokens, h_q // h_kv, h_kv, num_parts)
        if out is not None:
            md, ns = out
            if md.numel() != n_md or ns.numel() != n_ns or md.dtype != torch.int32 or ns.dtype != torch.int32:
                raise ValueError("metadata output tensors have the wrong size or dtype")
        else:
            md = torch.empty(n_md, dtype=torch.int32, device=dev).view(num_parts, 8)
            ns = torch.empty(n_ns, dtype=torch.int32, device=dev)
        with torch.cuda.device(dev):
            _lib.check(_lib.load().mla_get_metadata_sparse(tokens, int(topk), h_q, h_kv, num_parts, _ptr(md),
                                                           _ptr(ns), _stream(dev)), "mla_get_metadata_sparse")
        return md, ns
    n_md, n_ns = metadata_sizes(batch, heads_per_kv, h_kv, num_parts)
    if out is not None:
        md, ns = out
        if md.numel() != n_md or ns.numel() != n_ns or md.dtype != torch.int32 or ns.dtype != torch.int32:
            raise ValueError("metadata output tensors have the wrong size or dtype")
    else:
        md = torch.empty(n_md, dtype=torch.int32, device=dev).view(num_parts, 8)
        ns = torch.empty(n_ns, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _lib.check(_lib.load().mla_get_metadata(_ptr(cache_seqlens), batch, heads_per_kv, h_kv, num_parts,
                                                int(bool(is_fp8_kvcache)), _ptr(md), _ptr(ns), _stream(dev)),
                   "mla_get_metadata")
    return md, ns


def get_mla_metadata_host(cache_seqlens, heads_per_kv: int, h_kv: int = 1, num_parts: int = 74,
                          is_fp8_kvcache: bool = False):
    """The same schedule computed on the host (numpy in, numpy out)."""
    import numpy as np

    sl = np.ascontiguousarray(cache_seqlens, dtype=np.int32)
    n_md, n_ns = metadata_sizes(sl.size, heads_per_kv, h_kv, num_parts)
    md = np.zeros(n_md, np.int32)
    ns = np.zeros(n_ns, np.int32)
    _lib.check(_lib.load().mla_get_metadata_host(sl.ctypes.data, sl.size, heads_per_kv, h_kv, num_parts,
                                                 int(bool(is_fp8_kvcache)), md.ctypes.data, ns.ctypes.data),
               "mla_get_metadata_host")
    return md.reshape(num_parts, 8), ns


def get_mla_metadata_sparse_host(num_tokens: int, topk: int, h_q: int, h_kv: int = 1, num_parts: int = 74):
    """The sparse decode's schedule (num_tokens query tokens of topk entries) computed on the host."""
    import numpy as np

    n_md, n_ns = metadata_sizes(num_tokens, h_q // h_kv, h_kv, num_parts)
    md = np.zeros(n_md, np.int32)
    ns = np.zeros(n_ns, np.int32)
    _lib.check(_lib.load().mla_get_metadata_sparse_host(num_tokens, topk, h_q, h_kv, num_parts, md.ctypes.data,
                                                        ns.ctypes.data), "mla_get_metadata_sparse_host")
    return md.reshape(num_parts, 8), ns


def workspace_bytes(batch: int, s_q: int, h_q: int, h_kv: int, num_parts: int) -> int:
    n = _lib.load().mla_decode_workspace_bytes(batch, s_q, h_q, h_kv, num_parts)
    if n == 0:
        raise ValueError("invalid sizes for the decode workspace")
    return n


def workspace_zero_bytes(batch: int, s_q: int, h_q: int, h_kv: int) -> int:
    """Leading workspace bytes (status word and counters) that must be zero before first use."""
    return _lib.load().mla_decode_workspace_zero_bytes(batch, s_q, h_q, h_kv)


def get_workspace(nbytes: int, device: torch.device, zero_bytes: int) -> torch.Tensor:
    """A cached, grow-only workspace per (device, stream) whose control block is zero.

    ``zero_bytes`` is the control block's size (the same for every problem): it is
    zeroed when the workspace is allocated, and every call that meets no device error
    leaves it zero for the next call of any size.  ``read_device_status(ws, clear=True)``
    zeroes it again after a device error.
    """
    key = (device.index, _stream(device))
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < max(nbytes, zero_bytes):
        ws = torch.empty(max(nbytes, zero_bytes), dtype=torch.uint8, device=device)
        ws[:zero_bytes].zero_()
        _workspaces[key] = ws
    return ws


class DecodeCall:
    """Marshalled arguments of one decode call (device tensors), reusable across stages."""

    def __init__(self, q, kvcache, block_table, cache_seqlens, dv, tile_scheduler_metadata, num_splits,
                 causal=False, softmax_scale=None, workspace=None, out=None, lse=None, active_heads=None,
                 is_fp8_kvcache=False, indices=None):
        dev = q.device
        self.sparse = indices is not None
        if self.sparse:
            if indices.dtype != torch.int32 or indices.dim() != 3 or indices.shape[:2] != q.shape[:2]:
                raise ValueError("indices must be int32 [batch, s_q, topk]")
            if not indices.is_contiguous() or indices.device != dev:
                raise ValueError(f"indices must be contiguous and on {dev}")
        if is_fp8_kvcache:
            if q.dtype != torch.bfloat16 or kvcache.dtype != torch.uint8 or kvcache.shape[-1] != FP8_ROW_BYTES:
                raise ValueError("an FP8 cache takes bfloat16 q and a uint8 kvcache of 656-byte rows")
            if q.shape[-1] != 576:
                raise ValueError("an FP8 cache has d_qk = 576")
        elif q.dtype not in _DTYPES or kvcache.dtype != q.dtype:
            raise ValueError("q and kvcache must both be bfloat16 or both float16")
        tensors = [("q", q), ("kvcache", kvcache), ("tile_scheduler_metadata", tile_scheduler_metadata),
                   ("num_splits", num_splits)]
        if not self.sparse:  # the sparse decode reads no block table and no lengths
            tensors += [("block_table", block_table), ("cache_seqlens", cache_seqlens)]
        for name, t in tensors:
            if not t.is_contiguous() or t.device != dev:
                raise ValueError(f"{name} must be contiguous and on {dev}")
        b, s_q, h_q, d_qk = q.shape
        num_blocks, page, h_kv, d2 = kvcache.shape
        if not is_fp8_kvcache and d2 != d_qk:
            raise ValueError("q and kvcache rows must have the same width")
        if not self.sparse:
            if block_table.dtype != torch.int32 or cache_seqlens.dtype != torch.int32:
                raise ValueError("block_table and cache_seqlens must be int32")
            if ((not is_fp8_kvcache and d2 != d_qk) or block_table.dim() != 2 or block_table.shape[0] != b
                    or cache_seqlens.numel() != b):
                raise ValueError("inconsistent shapes")
        num_parts = tile_scheduler_metadata.shape[0]
        if out is None:
            out = torch.empty(b, s_q, h_q, dv, dtype=q.dtype, device=dev)
        if lse is None:
            lse = torch.empty(b, s_q, h_q, dtype=torch.float32, device=dev)
        ws_b, ws_s = (b * s_q, 1) if self.sparse else (b, s_q)  # sparse: every token is a request
        if workspace is None:
            workspace = get_workspace(workspace_bytes(ws_b, ws_s, h_q, h_kv, num_parts), dev,
                                      workspace_zero_bytes(ws_b, ws_s, h_q, h_kv))
        scale = float(softmax_scale) if softmax_scale is not None else 1.0 / math.sqrt(d_qk)
        self.device = dev
        self.out, self.lse, self.workspace = out, lse, workspace
        self._keep = (q, kvcache, block_table, cache_seqlens, tile_scheduler_metadata, num_splits, indices)
        active = 0 if active_heads is None else int(active_heads)  # 0: every head is real
        dtype = MLA_BF16_FP8KV if is_fp8_kvcache else _DTYPES[q.dtype]
        if self.sparse:
            self.args = (_ptr(q), b, s_q, h_q, d_qk, _ptr(kvcache), num_blocks, page, h_kv, _ptr(indices),
                         indices.shape[2], dv, dtype, _ptr(tile_scheduler_metadata), num_parts, _ptr(num_splits),
                         scale, active, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel())
        else:
            self.args = (_ptr(q), b, s_q, h_q, d_qk, _ptr(kvcache), num_blocks, page, h_kv, _ptr(block_table),
                         block_table.shape[1], _ptr(cache_seqlens), dv, dtype,
                         _ptr(tile_scheduler_metadata), num_parts, _ptr(num_splits), int(bool(causal)), scale,
                         active, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel())
        self.combine_args = (ws_b, ws_s, h_q, h_kv, dv, dtype, _ptr(num_splits), num_parts, active,
                             _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel())

    def run(self):
        """Split-KV kernel then combine kernel (mla_decode_with_kvcache / mla_decode_sparse)."""
        fn = "mla_decode_sparse" if self.sparse else "mla_decode_with_kvcache"
        with torch.cuda.device(self.device):
            _lib.check(getattr(_lib.load(), fn)(*self.args, _stream(self.device)), fn)
        return self.out, self.lse

    def splitkv(self):
        fn = "mla_decode_sparse_splitkv" if self.sparse else "mla_decode_splitkv"
        with torch.cuda.device(self.device):
            _lib.check(getattr(_lib.load(), fn)(*self.args, _stream(self.device)), fn)

    def combine(self):
        with torch.cuda.device(self.device):
            _lib.check(_lib.load().mla_decode_combine(*self.combine_args, _stream(self.device)),
                       "mla_decode_combine")


def flash_mla_with_kvcache(q: torch.Tensor, kvcache: torch.Tensor, block_table: torch.Tensor,
                           cache_seqlens: torch.Tensor, dv: int, tile_scheduler_metadata: torch.Tensor,
                           num_splits: torch.Tensor, causal: bool = False, is_fp8_kvcache: bool = False,
                           indices: torch.Tensor | None = None, *, softmax_scale: float | None = None,
                           workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                           lse: torch.Tensor | None = None, active_heads: int | None = None):
    """MLA decode over a paged cache; returns ``(o [b, s_q, h_q, dv], lse [b, s_q, h_q] float32)``.

    ``is_fp8_kvcache``: ``kvcache`` is uint8 [num_blocks, 64, h_kv, 656] in the "FP8
    with scale" format of the upstream FlashMLA documentation ("FP8 KV Cache": 512
    float8_e4m3 latent values, 4 float32 scales, 64 bfloat16 RoPE values per token),
    ``q`` bfloat16 with d_qk = 576; the cache is dequantized to bfloat16 in the kernel.

    ``active_heads``: heads ``[active_heads, h_q)`` are padding whose outputs are not
    written (a multiple of 8 no larger than ``h_q``; anything else means all heads).

    ``indices`` int32 [b, s_q, topk]: token-level sparse decoding (upstream FlashMLA
    documentation, "Sparse Attention (indices tensor)"): query token (i, j) attends the
    cache rows ``indices[i, j, k]`` (page * 64 + offset; -1 or any row outside the cache is
    invalid) instead of a block-table prefix; ``block_table``, ``cache_seqlens`` and
    ``causal`` are not used, the cache must be FP8 with scale, and the metadata comes from
    ``get_mla_metadata(..., h_q=h_q, topk=topk)``.

    ``q`` [b, s_q, h_q, d_qk] and ``kvcache`` [num_blocks, 64, h_kv, d_qk] are bf16 or
    fp16; ``block_table`` [b, max_blocks] and ``cache_seqlens`` [b] are int32.  With
    ``q`` on the CPU the inputs are copied to the current CUDA device (non-blocking
    when pinned) and the results copied back (host-buffer path).
    """
    host = not q.is_cuda
    if host:
        dev = torch.device("cuda", torch.cuda.current_device())
        nb = q.is_pinned()
        q, kvcache, block_table, cache_seqlens, tile_scheduler_metadata, num_splits, indices = (
            None if t is None else t.to(dev, non_blocking=nb) for t in
            (q, kvcache, block_table, cache_seqlens, tile_scheduler_metadata, num_splits, indices))
    call = DecodeCall(q, kvcache, block_table, cache_seqlens, dv, tile_scheduler_metadata, num_splits,
                      causal=causal, softmax_scale=softmax_scale, workspace=workspace, out=out, lse=lse,
                      active_heads=active_heads, is_fp8_kvcache=is_fp8_kvcache, indices=indices)
    out, lse = call.run()
    if host:
        return out.cpu(), lse.cpu()
    return out, lse


def flash_mla_sparse_fwd(q: torch.Tensor, kv: torch.Tensor, indices: torch.Tensor, sm_scale: float, d_v: int = 512,
                         num_parts: int | None = None, workspace: torch.Tensor | None = None):
    """Sparse MLA prefill (upstream FlashMLA documentation, "Sparse MLA Prefill").

    ``q`` [s_q, h_q, 576] and ``kv`` [s_kv, 1, 576] bf16 (or fp16), ``indices`` int32
    [s_q, 1, topk] (-1 or any index >= s_kv is invalid).  Returns ``(out [s_q, h_q, d_v],
    max_logits [s_q, h_q] float32, lse [s_q, h_q] float32)``, max_logits and lse in base 2 of
    the logits scaled by ``sm_scale * log2(e)``.  The tile schedule is computed on the device
    as part of the call.
    """
    if q.dtype not in _DTYPES or kv.dtype != q.dtype:
        raise ValueError("q and kv must both be bfloat16 or both float16")
    if q.dim() != 3 or kv.dim() != 3 or indices.dim() != 3 or indices.dtype != torch.int32:
        raise ValueError("q [s_q, h_q, d_qk], kv [s_kv, h_kv, d_qk], indices int32 [s_q, h_kv, topk]")
    s_q, h_q, d_qk = q.shape
    s_kv, h_kv, d2 = kv.shape
    if d2 != d_qk or indices.shape[:2] != (s_q, h_kv):
        raise ValueError("inconsistent shapes")
    dev = q.device
    for name, t in (("q", q), ("kv", kv), ("indices", indices)):
        if not t.is_contiguous() or t.device != dev:
            raise ValueError(f"{name} must be contiguous and on {dev}")
    topk = indices.shape[2]
    if num_parts is None:
        num_parts = num_sm_parts(dev)
    n_md, n_ns = metadata_sizes(s_q, h_q // h_kv, h_kv, num_parts)
    md = torch.empty(n_md, dtype=torch.int32, device=dev).view(num_parts, 8)
    ns = torch.empty(n_ns, dtype=torch.int32, device=dev)
    out = torch.empty(s_q, h_q, d_v, dtype=q.dtype, device=dev)
    max_logits = torch.empty(s_q, h_q, dtype=torch.float32, device=dev)
    lse = torch.empty(s_q, h_q, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = get_workspace(workspace_bytes(s_q, 1, h_q, h_kv, num_parts), dev,
                                  workspace_zero_bytes(s_q, 1, h_q, h_kv))
    lib = _lib.load()
    with torch.cuda.device(dev):
        st = _stream(dev)
        _lib.check(lib.mla_get_metadata_sparse(s_q, topk, h_q, h_kv, num_parts, _ptr(md), _ptr(ns), st),
                   "mla_get_metadata_sparse")
        _lib.check(lib.mla_sparse_prefill(_ptr(q), s_q, h_q, d_qk, _ptr(kv), s_kv, h_kv, _ptr(indices), topk, d_v,
                                          _DTYPES[q.dtype], float(sm_scale), _ptr(md), num_parts, _ptr(ns),
                                          _ptr(out), _ptr(max_logits), _ptr(lse), _ptr(workspace), workspace.numel(),
                                          st), "mla_sparse_prefill")
    return out, max_logits, lse


def read_device_status(workspace: torch.Tensor, clear: bool = True) -> int:
    """Device-side status recorded in a workspace (synchronises the current stream).

    ``clear`` zeroes the workspace's whole control block afterwards (status word and the
    split / combine counters), so that it can be used again after a device error."""
    v = ctypes.c_int(0)
    dev = workspace.device
    with torch.cuda.device(dev):
        _lib.check(_lib.load().mla_read_device_status(_ptr(workspace), int(clear), ctypes.byref(v), _stream(dev)),
                   "mla_read_device_status")
    return v.value
