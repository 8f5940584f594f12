"""Blackwell-native (sm_100a) MLA decoding over a paged latent KV cache.

Public calls (the names of the pages' API; "FlashMLA" usage page, deepep.org):

* :func:`get_mla_metadata` -- tile-scheduler metadata, once per decoding step;
* :func:`flash_mla_with_kvcache` -- one decode call per layer, returns ``(o, lse)``
  (``indices=``: the token-level sparse decode);
* :func:`flash_mla_sparse_fwd` -- the sparse MLA prefill, returns ``(out, max_logits, lse)``.

Both are thin wrappers over the C ABI in ``include/mla_decode.h``; the kernels
live in ``csrc/``.  ``workloads`` generates seeded synthetic inputs.
"""
from .api import (DecodeCall, flash_mla_sparse_fwd, flash_mla_with_kvcache, get_mla_metadata, get_mla_metadata_host,
                  get_mla_metadata_sparse_host, metadata_sizes, num_sm_parts, read_device_status, workspace_bytes,
                  workspace_zero_bytes)
from ._lib import MLAError

__all__ = ["DecodeCall", "flash_mla_sparse_fwd", "flash_mla_with_kvcache", "get_mla_metadata", "get_mla_metadata_host",
           "get_mla_metadata_sparse_host", "metadata_sizes", "num_sm_parts", "read_device_status", "workspace_bytes",
           "workspace_zero_bytes", "MLAError"]
