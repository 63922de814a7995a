"""ctypes view of libqsa.so (the C ABI declared in include/qsa.h).

Loading fails loudly when the library has not been built: there is no
fallback implementation of any step.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqsa.so")

QSA_OK = 0
QSA_ERR_INVALID_ARG = 1
QSA_ERR_UNSUPPORTED = 2
QSA_ERR_WORKSPACE = 3
QSA_ERR_CUDA = 4

QSA_F32 = 0
QSA_BF16 = 1

# every symbol include/qsa.h declares
EXPORTED = [
    "qsa_status_string", "qsa_last_error", "qsa_version", "qsa_kernel_launch_count",
    "qsa_set_stage_events", "qsa_set_keys_visited",
    "qsa_prefill_workspace_size", "qsa_prefill", "qsa_select",
    "qsa_decode_workspace_size", "qsa_decode", "qsa_select_decode",
    "qsa_pool_build", "qsa_decode_noalloc", "qsa_decode_paged", "qsa_pool_build_paged",
    "qsa_decode_fp8", "qsa_decode_attend",
    "qsa_cp_select", "qsa_cp_global_topk", "qsa_cp_attend", "qsa_cp_merge",
    "qsa_cp_pool_build", "qsa_append",
]


class QsaConfigC(ctypes.Structure):
    _fields_ = [
        ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("idx_heads", ctypes.c_int),
        ("idx_dim", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("budget", ctypes.c_int),
        ("softmax_scale", ctypes.c_float),
        ("index_scale", ctypes.c_float),
        ("gate_headwise", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("rope_dim", ctypes.c_int),
        ("rope_theta", ctypes.c_float),
    ]


class QsaError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {status_name(status)}: {msg}")
        self.status = status


_lib = None

P = ctypes.c_void_p
I = ctypes.c_int
SZ = ctypes.c_size_t
CFG = ctypes.POINTER(QsaConfigC)


def _declare(lib):
    sig = {
        "qsa_status_string": (ctypes.c_char_p, [I]),
        "qsa_last_error": (ctypes.c_char_p, []),
        "qsa_version": (I, []),
        "qsa_kernel_launch_count": (ctypes.c_ulonglong, []),
        "qsa_set_stage_events": (I, [ctypes.POINTER(ctypes.c_void_p), I]),
        "qsa_set_keys_visited": (None, [P]),
        "qsa_prefill_workspace_size": (SZ, [CFG, I, I, I]),
        "qsa_prefill": (I, [CFG, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]),
        "qsa_select": (I, [CFG, I, I, I, P, P, P, P, P, P, P, P, P, SZ, P]),
        "qsa_decode_workspace_size": (SZ, [CFG, I, I, I]),
        "qsa_decode": (I, [CFG, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]),
        "qsa_select_decode": (I, [CFG, I, I, I, P, P, P, P, P, P, P, P, P, P, SZ, P]),
        "qsa_pool_build": (I, [CFG, I, I, P, P, P, P, P]),
        "qsa_decode_noalloc": (I, [CFG, I, I, I] + [P] * 15),
        # cfg, batch, n_q, max_blocks, block_table, num_pages, kv_len, q, k, v, iq, ik, iw,
        # gate, pooled, out, lse, sel, nsel, dev_err, ws, ws_bytes, stream (15 pointers)
        "qsa_decode_paged": (I, [CFG, I, I, I, P, I] + [P] * 15 + [SZ, P]),
        # cfg, batch, max_blocks, block_table, num_pages, kv_len, ik, pooled, dev_err, stream
        "qsa_pool_build_paged": (I, [CFG, I, I, P, I, P, P, P, P, P]),
        # cfg, batch, n_q, cap, kv_len, q, k, k_scale, v, v_scale, rotated, iq, ik, iw, gate,
        # pooled, out, lse, sel, nsel, dev_err, ws, ws_bytes, stream
        "qsa_decode_fp8": (I, [CFG, I, I, I, P, P, P, P, P, P, I] + [P] * 11 + [SZ, P]),
        "qsa_decode_attend": (I, [CFG, I, I, I] + [P] * 11 + [SZ, P]),
        # cfg, batch, n_q, cap, block_lo, kv_len, iq, ik, iw, pooled, cand_score, cand_id,
        # dev_err, ws, ws_bytes, stream
        "qsa_cp_select": (I, [CFG, I, I, I, I] + [P] * 9 + [SZ, P]),
        # cfg, batch, cap, block_lo, kv_len, ik_shard, pooled_shard, dev_err, stream
        "qsa_cp_pool_build": (I, [CFG, I, I, I, P, P, P, P, P]),
        # cfg, batch, n_q, cap, kv_len, k_new, v_new, ik_new, k_cache, v_cache, ik_cache,
        # pooled_cache, block_table, num_pages, dev_err, stream
        "qsa_append": (I, [CFG, I, I, I] + [P] * 9 + [I, P, P]),
        # cfg, batch, n_q, world, kv_len, cand_score, cand_id, sel, nsel, stream
        "qsa_cp_global_topk": (I, [CFG, I, I, I] + [P] * 6),
        # cfg, batch, n_q, cap, block_lo, kv_len, q, k, v, gate, sel, nsel, part_out,
        # part_lse, dev_err, ws, ws_bytes, stream
        "qsa_cp_attend": (I, [CFG, I, I, I, I] + [P] * 11 + [SZ, P]),
        # cfg, batch, n_q, world, part_out, part_lse, out, lse, stream
        "qsa_cp_merge": (I, [CFG, I, I, I] + [P] * 5),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args


def lib():
    """The loaded library; raises if libqsa.so is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m block_sparse_attention_17_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        _declare(l)
        _lib = l
    return _lib


def status_name(s: int) -> str:
    return lib().qsa_status_string(int(s)).decode()


def check(status: int, where: str):
    if status != QSA_OK:
        raise QsaError(status, where, lib().qsa_last_error().decode())
