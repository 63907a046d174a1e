"""CSA2 compressed sparse attention over a shared FP4 global KV cache, on B200 (sm_100a).

The compute lives in libcsa2.so (hand-written CUDA, C ABI in include/csa2.h);
this package is its ctypes binding.  Importing it without the built library
raises ImportError -- there is no CPU fallback.
"""
from ._lib import (EXPORTED, MODE, GlobalKVCache, csa2_cache, csa2_check, csa2_index_score,  # noqa: F401
                   csa2_merge, csa2_pack_kv, csa2_pack_swa, csa2_sparse_attn, csa2_swa_attn, csa2_topk,
                   csa2_version, csa2_workspace_size, raw, LIB_PATH)
