"""CSA2 compressed sparse attention over a shared FP4 global KV cache, on B200 (sm_100a).

The compute lives in libcsa2.so (hand-written CUDA, C ABI in include/csa2.h);
this package is its ctypes binding.  The library is loaded on first use of any
binding name; without the built library that raises ImportError -- there is no
CPU fallback.  (`python -m compressed_sparse_attention_score_b200.build` builds it.)
"""
_NAMES = ("EXPORTED", "MODE", "GlobalKVCache", "csa2_cache", "csa2_check", "csa2_index_score", "csa2_merge",
          "csa2_pack_kv", "csa2_pack_swa", "csa2_sparse_attn", "csa2_sparse_attn_noalloc", "csa2_swa_attn",
          "csa2_topk", "csa2_version", "csa2_workspace_size", "raw", "LIB_PATH", "csa2_append_kv", "csa2_plan_v41",
          "csa2_pack_kv_gated", "csa2_index_topk", "DecodeStep", "LAYER_SWA")


def __getattr__(name):
    if name in _NAMES:
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)


__all__ = list(_NAMES)
