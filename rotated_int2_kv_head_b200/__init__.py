"""libkvq: rotated INT2 KV cache for B200 (sm_100a).

rotate -> quantize -> append, and decode attention over the packed cache, as
hand-written CUDA kernels behind a C ABI (include/kvq.h).  This package holds
the CUDA sources (csrc/), the in-tree build (build.py) and a thin ctypes
binding (kvq.py) with the same function names as the C ABI.
"""
from .kvq import (HostStep, KVQ_DECODE_OUT_ROTATED, KVQ_DEV_BAD_LEN, KVQ_DEV_CAPACITY, KVQ_DEV_TIMEOUT,
                  KVQ_DEV_BAD_TABLE, KVQ_ROT_DENSE, KVQ_ROT_PERM_FWHT, KVCache, KvqError, PagedKVCache,
                  decode_workspace,
                  kvq_cache_bytes, kvq_clear_status, kvq_debug_quantize_f32, kvq_debug_rotate_f32,
                  kvq_decode_attention, kvq_decode_attention_ex, kvq_decode_attention_noalloc,
                  kvq_decode_attention_adapter,
                  kvq_decode_attention_timed,
                  kvq_decode_workspace_size, kvq_get_status, kvq_identify_sinks,
                  kvq_rotate_quantize_append, lib, kvq_prerope_append, kvq_prerope_decode,
                  kvq_append_decode, kvq_append_decode_host, kvq_step_workspace_size,
                  step_workspace,
                  kvq_prerope_workspace_size, prerope_workspace, kvq_debug_rotate_group_f32,
                  kvq_debug_wait_timeout)

__all__ = [
    "HostStep", "KVCache", "PagedKVCache", "KvqError", "KVQ_DEV_BAD_TABLE", "KVQ_DECODE_OUT_ROTATED", "KVQ_ROT_DENSE", "KVQ_ROT_PERM_FWHT",
    "KVQ_DEV_CAPACITY",
    "KVQ_DEV_BAD_LEN", "KVQ_DEV_TIMEOUT", "decode_workspace", "kvq_cache_bytes",
    "kvq_clear_status", "kvq_debug_quantize_f32", "kvq_debug_rotate_f32",
    "kvq_decode_attention", "kvq_decode_attention_ex", "kvq_decode_attention_noalloc",
    "kvq_decode_attention_adapter",
    "kvq_decode_attention_timed",
    "kvq_decode_workspace_size", "kvq_get_status", "kvq_identify_sinks",
    "kvq_rotate_quantize_append", "lib", "kvq_prerope_append", "kvq_prerope_decode",
    "kvq_append_decode", "kvq_append_decode_host", "kvq_step_workspace_size", "step_workspace",
    "kvq_prerope_workspace_size", "prerope_workspace", "kvq_debug_rotate_group_f32",
    "kvq_debug_wait_timeout",
]
