"""NVFP4 KV-cache append and block-causal chunk attention for B200 (sm_100a).

The product is the C-ABI library ``libnvkv.so`` (include/nvkv.h).  This
package is its thin Python binding (``_lib``: ctypes marshalling, same names
as the C entry points) plus ``KVCache``, which allocates the caller-owned
device planes with PyTorch.  Importing fails loudly if the library is absent.
"""
from . import _lib
from ._lib import (NVKV_KV_BF16, NVKV_KV_NVFP4, NvkvError, bf16_kv_append, bf16_kv_overwrite,
                   chunk_attention_bf16kv, chunk_attention_nvfp4kv, kv_ring_begin_shot,
                   kv_ring_evict, nvfp4_kv_append, nvkv_attention_workspace_bytes,
                   nvfp4_kv_overwrite, nvkv_desc_init, nvkv_desc_set_shard,
                   nvkv_encode_block_scale, nvkv_encode_e2m1, nvkv_lse_merge, nvkv_plane_bytes,
                   nvkv_ring_init, nvkv_ring_push_chunk, nvkv_ring_visible,
                   nvkv_status_string)
from .cache import KVCache, lse_merge, lse_merge_ptrs
from .pipeline import HostPipeline

__all__ = ["KVCache", "HostPipeline", "lse_merge", "lse_merge_ptrs", "NvkvError", "NVKV_KV_NVFP4", "NVKV_KV_BF16",
           "nvkv_desc_init", "nvkv_desc_set_shard", "nvkv_lse_merge",
           "nvkv_plane_bytes", "nvkv_ring_init", "kv_ring_evict", "kv_ring_begin_shot",
           "nvkv_ring_visible", "nvkv_ring_push_chunk", "nvfp4_kv_append", "bf16_kv_append",
           "nvfp4_kv_overwrite", "bf16_kv_overwrite",
           "nvkv_attention_workspace_bytes", "chunk_attention_nvfp4kv", "chunk_attention_bf16kv",
           "nvkv_encode_e2m1", "nvkv_encode_block_scale", "nvkv_status_string"]
