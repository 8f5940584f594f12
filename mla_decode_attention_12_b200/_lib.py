"""ctypes binding of the C ABI in ``include/mla_decode.h`` (library ``_mla_decode.so``).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  Loading fails loudly when the library has not been built; there
is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "_mla_decode.so")

MLA_OK = 0
STATUS_NAMES = {
    0: "MLA_OK",
    1: "MLA_ERR_INVALID_ARG",
    2: "MLA_ERR_UNSUPPORTED",
    3: "MLA_ERR_WORKSPACE",
    4: "MLA_ERR_CUDA",
    5: "MLA_ERR_TIMEOUT",
    6: "MLA_ERR_DEVICE_CHECK",
}

# Every entry point the header declares, with its ctypes signature.
_I, _P, _SZ, _F = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
SIGNATURES = {
    "mla_status_string": ([_I], ctypes.c_char_p),
    "mla_num_sm_parts": ([_I, ctypes.POINTER(_I)], _I),
    "mla_metadata_sizes": ([_I, _I, _I, _I, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)], _I),
    "mla_get_metadata": ([_P, _I, _I, _I, _I, _I, _P, _P, _P], _I),
    "mla_get_metadata_host": ([_P, _I, _I, _I, _I, _I, _P, _P], _I),
    "mla_decode_workspace_bytes": ([_I, _I, _I, _I, _I], _SZ),
    "mla_decode_workspace_zero_bytes": ([_I, _I, _I, _I], _SZ),
    "mla_decode_with_kvcache": ([_P, _I, _I, _I, _I,          # q, batch, s_q, h_q, d_qk
                                 _P, _I, _I, _I,              # kvcache, num_blocks, page_size, h_kv
                                 _P, _I, _P, _I, _I,          # block_table, max_blocks, seqlens, dv, dtype
                                 _P, _I, _P, _I, _F,          # tile_md, num_parts, num_splits, causal, scale
                                 _I,                          # active_heads
                                 _P, _P, _P, _SZ, _P], _I),   # o, lse, workspace, ws_bytes, stream
    "mla_decode_splitkv": ([_P, _I, _I, _I, _I, _P, _I, _I, _I, _P, _I, _P, _I, _I,
                            _P, _I, _P, _I, _F, _I, _P, _P, _P, _SZ, _P], _I),
    "mla_decode_combine": ([_I, _I, _I, _I, _I, _I, _P, _I, _I, _P, _P, _P, _SZ, _P], _I),
    "mla_read_device_status": ([_P, _I, ctypes.POINTER(_I), _P], _I),
    "mla_decode_with_kvcache_noalloc": ([_P, _I, _I, _I, _I, _P, _I, _I, _I, _P, _I, _P, _I, _I,
                                         _P, _I, _P, _I, _F, _I, _P, _P, _P], _I),
    "mla_read_noalloc_status": ([_I, ctypes.POINTER(_I), _P], _I),
    "mla_get_metadata_sparse": ([_I, _I, _I, _I, _I, _P, _P, _P], _I),
    "mla_get_metadata_sparse_host": ([_I, _I, _I, _I, _I, _P, _P], _I),
    "mla_decode_sparse": ([_P, _I, _I, _I, _I,          # q, batch, s_q, h_q, d_qk
                           _P, _I, _I, _I,              # kvcache, num_blocks, page_size, h_kv
                           _P, _I, _I, _I,              # indices, topk, dv, dtype
                           _P, _I, _P, _F, _I,          # tile_md, num_parts, num_splits, scale, active_heads
                           _P, _P, _P, _SZ, _P], _I),   # o, lse, workspace, ws_bytes, stream
    "mla_decode_sparse_splitkv": ([_P, _I, _I, _I, _I, _P, _I, _I, _I, _P, _I, _I, _I,
                                   _P, _I, _P, _F, _I, _P, _P, _P, _SZ, _P], _I),
    "mla_sparse_prefill": ([_P, _I, _I, _I, _P, _I, _I,      # q, s_q, h_q, d_qk, kv, s_kv, h_kv
                            _P, _I, _I, _I, _F,              # indices, topk, dv, dtype, sm_scale
                            _P, _I, _P,                      # tile_md, num_parts, num_splits
                            _P, _P, _P, _P, _SZ, _P], _I),   # out, max_logits, lse, workspace, bytes, stream
}

_lock = threading.Lock()
_lib = None


class MLAError(RuntimeError):
    """A library call returned a status other than MLA_OK."""

    def __init__(self, status: int, where: str):
        self.status = status
        msg = status_string(status) if _lib is not None else STATUS_NAMES.get(status, "?")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({msg})")


def load() -> ctypes.CDLL:
    """Load ``_mla_decode.so``; raises if it is missing (build it with ``build.py``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m mla_decode_attention_12_b200.build` (nvcc, sm_100a)")
            _lib = bind(LIB_PATH)
    return _lib


def bind(path: str) -> ctypes.CDLL:
    """Open a build of the library at `path` with every entry point's signature set."""
    lib = ctypes.CDLL(path)
    for name, (argtypes, restype) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = argtypes
        fn.restype = restype
    return lib


def status_string(status: int) -> str:
    return load().mla_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != MLA_OK:
        raise MLAError(status, where)
