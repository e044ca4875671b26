"""Chunk attention over a segmented KV cache, native on B200 (sm_100a).

The compute lives in ``libvkv.so`` (C ABI, declared in ``include/vkv.h``);
``kv_cache_attention_chunk_b200.vkv`` is a thin ctypes binding with the same
entry-point names.  ``workloads`` builds seeded synthetic inputs.
"""
__all__ = ["vkv", "workloads"]
