"""B200-native (sm_100a) Qwen Sparse Attention: a C-ABI CUDA library
(libqsa.so, include/qsa.h) with a thin Python binding."""
from .api import (QSAConfig, append, cp_attend, cp_global_topk, cp_merge, cp_pool_build, cp_select,
                  decode, decode_attend, decode_fp8, decode_noalloc, decode_paged,
                  decode_workspace_size,
                  pool_build, pool_build_paged, prefill, prefill_workspace_size, select,
                  select_decode, set_keys_visited)
from ._lib import QsaError, LIB_PATH

__all__ = ["QSAConfig", "append", "set_keys_visited", "prefill", "select", "decode", "decode_noalloc", "decode_paged", "decode_fp8",
           "decode_attend",
           "select_decode", "pool_build", "pool_build_paged", "prefill_workspace_size",
           "decode_workspace_size", "cp_pool_build", "cp_select", "cp_global_topk", "cp_attend",
           "cp_merge", "QsaError", "LIB_PATH"]
