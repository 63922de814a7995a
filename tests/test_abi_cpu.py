"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/qsa.h declares, and rejects bad arguments with a status
code before anything is launched.

The rejection tests pass made-up device addresses that no kernel may read.
They run only where no CUDA device is visible: should a validation check
regress, the call then fails to launch instead of sending a kernel to those
addresses on a real GPU."""
import ctypes
import os
import re

import pytest

from block_sparse_attention_17_b200 import _lib

try:
    import torch
    _GPU_VISIBLE = torch.cuda.is_available()
except Exception:  # pragma: no cover
    _GPU_VISIBLE = False

# tests that hand the library made-up device addresses
fake_pointers = pytest.mark.skipif(_GPU_VISIBLE, reason="made-up device addresses: run only "
                                   "where no CUDA device is visible")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    txt = open(os.path.join(ROOT, "include", "qsa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    lib = _lib.lib()
    syms = header_symbols()
    assert "qsa_prefill" in syms and "qsa_decode" in syms and "qsa_select" in syms
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(_lib.EXPORTED)
    assert lib.qsa_version() == 101


def test_status_strings():
    for code, name in [(0, "QSA_OK"), (1, "QSA_ERR_INVALID_ARG"), (2, "QSA_ERR_UNSUPPORTED"),
                       (3, "QSA_ERR_WORKSPACE"), (4, "QSA_ERR_CUDA")]:
        assert _lib.status_name(code) == name


def cfg(**kw):
    base = dict(num_q_heads=16, num_kv_heads=2, head_dim=128, idx_heads=4, idx_dim=64,
                block_size=64, budget=2048, softmax_scale=0.0, index_scale=0.0,
                gate_headwise=0, dtype=_lib.QSA_BF16)
    base.update(kw)
    return _lib.QsaConfigC(**base)


FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced
MISALIGNED = ctypes.c_void_p(0x10008)


def call_prefill(c, T=8192, ws_bytes=None, ptrs=None, batch=1, max_seqlen=8192):
    lib = _lib.lib()
    ws = lib.qsa_prefill_workspace_size(ctypes.byref(c), batch, T, max_seqlen)
    if ws_bytes is None:
        ws_bytes = ws
    p = dict(cu=FAKE, q=FAKE, k=FAKE, v=FAKE, iq=FAKE, ik=FAKE, iw=FAKE, gate=FAKE, out=FAKE)
    p.update(ptrs or {})
    return lib.qsa_prefill(ctypes.byref(c), batch, T, max_seqlen, p["cu"], p["q"], p["k"],
                           p["v"], p["iq"], p["ik"], p["iw"], p["gate"], p["out"], None, None,
                           None, None, ctypes.c_void_p(0x20000), ws_bytes, None)


@fake_pointers
@pytest.mark.parametrize("kw,code", [
    (dict(num_kv_heads=3), _lib.QSA_ERR_INVALID_ARG),        # Hq % Hkv != 0
    (dict(budget=2000), _lib.QSA_ERR_INVALID_ARG),            # budget % B != 0
    (dict(num_q_heads=0), _lib.QSA_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.QSA_ERR_INVALID_ARG),
    (dict(softmax_scale=-1.0), _lib.QSA_ERR_INVALID_ARG),
    (dict(head_dim=96), _lib.QSA_ERR_UNSUPPORTED),
    (dict(block_size=32, budget=2048), _lib.QSA_ERR_UNSUPPORTED),
    (dict(idx_dim=48), _lib.QSA_ERR_UNSUPPORTED),
    (dict(budget=64 * 65), _lib.QSA_ERR_UNSUPPORTED),         # k > 64
    (dict(num_q_heads=34, num_kv_heads=2), _lib.QSA_ERR_UNSUPPORTED),   # G > 16
    (dict(rope_dim=6, rope_theta=1e4), _lib.QSA_ERR_INVALID_ARG),         # not a multiple of 4
    (dict(rope_dim=128, rope_theta=1e4), _lib.QSA_ERR_INVALID_ARG),       # > idx_dim
    (dict(rope_dim=-4, rope_theta=1e4), _lib.QSA_ERR_INVALID_ARG),
    (dict(rope_dim=32, rope_theta=0.0), _lib.QSA_ERR_INVALID_ARG),
    (dict(rope_dim=32, rope_theta=float("nan")), _lib.QSA_ERR_INVALID_ARG),
])
def test_prefill_rejects_bad_config(kw, code):
    assert call_prefill(cfg(**kw)) == code
    assert _lib.lib().qsa_last_error()


@fake_pointers
def test_prefill_rejects_null_and_misaligned_pointers():
    assert call_prefill(cfg(), ptrs={"q": None}) == _lib.QSA_ERR_INVALID_ARG
    assert b"q is NULL" in _lib.lib().qsa_last_error()
    assert call_prefill(cfg(), ptrs={"k": MISALIGNED}) == _lib.QSA_ERR_INVALID_ARG
    assert b"aligned" in _lib.lib().qsa_last_error()


@fake_pointers
def test_prefill_rejects_small_workspace():
    c = cfg()
    need = _lib.lib().qsa_prefill_workspace_size(ctypes.byref(c), 1, 8192, 8192)
    assert need > 0
    assert call_prefill(c, ws_bytes=need - 1) == _lib.QSA_ERR_WORKSPACE


@fake_pointers
def test_prefill_rejects_bad_lengths():
    assert call_prefill(cfg(), T=-1) == _lib.QSA_ERR_INVALID_ARG
    assert call_prefill(cfg(), batch=0, T=10) == _lib.QSA_ERR_INVALID_ARG
    assert call_prefill(cfg(), T=100, max_seqlen=200) == _lib.QSA_ERR_INVALID_ARG
    # more than 4096 blocks per sequence
    assert call_prefill(cfg(), T=64 * 4097, max_seqlen=64 * 4097) == _lib.QSA_ERR_UNSUPPORTED


def test_empty_prefill_is_ok_without_gpu():
    # nothing to do: returns before touching any pointer or the device
    lib = _lib.lib()
    c = cfg()
    st = lib.qsa_prefill(ctypes.byref(c), 0, 0, 0, *([None] * 13), None, 0, None)
    assert st == _lib.QSA_OK


@fake_pointers
def test_decode_rejects_bad_geometry():
    lib = _lib.lib()
    c = cfg()
    ws = lib.qsa_decode_workspace_size(ctypes.byref(c), 32, 1, 32768)
    assert ws > 0

    def call(n_q=1, cap=32768, ws_bytes=ws, c=c):
        return lib.qsa_decode(ctypes.byref(c), 32, n_q, cap, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                              FAKE, FAKE, FAKE, FAKE, None, None, None, None,
                              ctypes.c_void_p(0x20000), ws_bytes, None)
    assert call(cap=32768 + 1) == _lib.QSA_ERR_INVALID_ARG          # cap % B
    assert call(n_q=0) == _lib.QSA_ERR_INVALID_ARG
    assert call(n_q=5) == _lib.QSA_ERR_UNSUPPORTED
    g16 = cfg(num_kv_heads=1)                                          # group size 16
    assert call(n_q=3, c=g16) == _lib.QSA_ERR_UNSUPPORTED              # 3 * 16 rows > 32
    assert call(ws_bytes=ws - 256) == _lib.QSA_ERR_WORKSPACE
    assert call(c=cfg(idx_heads=6)) == _lib.QSA_ERR_UNSUPPORTED        # heads summed by lane groups


def test_workspace_sizes_grow_with_the_problem():
    lib = _lib.lib()
    c = cfg()
    a = lib.qsa_prefill_workspace_size(ctypes.byref(c), 1, 4096, 4096)
    b = lib.qsa_prefill_workspace_size(ctypes.byref(c), 1, 8192, 8192)
    assert 0 < a < b
    assert lib.qsa_decode_workspace_size(ctypes.byref(c), 4, 1, 4096) < \
        lib.qsa_decode_workspace_size(ctypes.byref(c), 8, 1, 4096)


@fake_pointers
def test_paged_decode_rejects_bad_arguments():
    lib = _lib.lib()
    c = cfg()
    max_blocks = 512
    ws = lib.qsa_decode_workspace_size(ctypes.byref(c), 32, 1, max_blocks * c.block_size)
    assert ws > 0

    def call(n_q=1, max_blocks=max_blocks, table=FAKE, num_pages=32 * 512, ws_bytes=ws, c=c):
        return lib.qsa_decode_paged(ctypes.byref(c), 32, n_q, max_blocks, table, num_pages, FAKE,
                                    FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                    None, None, None, ctypes.c_void_p(0x20000), ws_bytes, None)
    assert call(table=None) == _lib.QSA_ERR_INVALID_ARG
    assert call(table=MISALIGNED) == _lib.QSA_ERR_INVALID_ARG
    assert call(max_blocks=0) == _lib.QSA_ERR_INVALID_ARG
    assert call(num_pages=0) == _lib.QSA_ERR_INVALID_ARG
    assert call(n_q=0) == _lib.QSA_ERR_INVALID_ARG
    assert call(n_q=5) == _lib.QSA_ERR_UNSUPPORTED                    # n_q > 4
    assert call(n_q=3, c=cfg(num_kv_heads=1)) == _lib.QSA_ERR_UNSUPPORTED   # 3 * 16 rows > 32
    assert call(c=cfg(dtype=_lib.QSA_F32)) == _lib.QSA_ERR_UNSUPPORTED  # tensor-map gather: bf16
    assert call(ws_bytes=ws - 256) == _lib.QSA_ERR_WORKSPACE
    st = lib.qsa_pool_build_paged(ctypes.byref(c), 32, max_blocks, None, 16, FAKE, FAKE, FAKE,
                                  None, None)
    assert st == _lib.QSA_ERR_INVALID_ARG


@fake_pointers
def test_decode_attend_rejects_bad_arguments():
    # attention over caller-given selections: every check happens before a launch
    lib = _lib.lib()
    c = cfg()
    ws = lib.qsa_decode_workspace_size(ctypes.byref(c), 32, 1, 32768)

    def call(n_q=1, cap=32768, sel=FAKE, nsel=FAKE, q=FAKE, ws_bytes=ws, c=c):
        return lib.qsa_decode_attend(ctypes.byref(c), 32, n_q, cap, FAKE, q, FAKE, FAKE, FAKE,
                                     sel, nsel, FAKE, None, None, ctypes.c_void_p(0x20000),
                                     ws_bytes, None)
    assert call(sel=None) == _lib.QSA_ERR_INVALID_ARG
    assert call(nsel=None) == _lib.QSA_ERR_INVALID_ARG
    assert call(q=MISALIGNED) == _lib.QSA_ERR_INVALID_ARG
    assert call(cap=32768 + 1) == _lib.QSA_ERR_INVALID_ARG
    assert call(n_q=5) == _lib.QSA_ERR_UNSUPPORTED
    assert call(ws_bytes=ws - 256) == _lib.QSA_ERR_WORKSPACE
    assert lib.qsa_decode_attend(ctypes.byref(c), 0, 1, 32768, *([None] * 11), 0,
                                 None) == _lib.QSA_OK             # empty batch: nothing to do


def test_binding_refuses_tensors_on_another_device():
    # the binding launches on one GPU with raw pointers: a tensor elsewhere must
    # raise before any call into the library
    import torch
    from block_sparse_attention_17_b200 import api
    cuda0 = torch.device("cuda", 0)
    with pytest.raises(ValueError, match="same GPU"):
        api._one_device(cuda0, None, q=torch.zeros(1))
    api._one_device(torch.device("cpu"), None, q=torch.zeros(1), k=None)


@fake_pointers
def test_append_rejects_bad_arguments():
    lib = _lib.lib()
    c = cfg()
    P = FAKE
    # K / V given without their caches
    assert lib.qsa_append(ctypes.byref(c), 2, 1, 4096, P, P, P, P, None, None, P, P, None, 0,
                          None, None) == _lib.QSA_ERR_INVALID_ARG
    # no indexer rows
    assert lib.qsa_append(ctypes.byref(c), 2, 1, 4096, P, None, None, None, None, None, P, P, None,
                          0, None, None) == _lib.QSA_ERR_INVALID_ARG
    # misaligned pooled cache, cap not a multiple of B, n_q past the limit
    assert lib.qsa_append(ctypes.byref(c), 2, 1, 4096, P, None, None, P, None, None, P, MISALIGNED,
                          None, 0, None, None) == _lib.QSA_ERR_INVALID_ARG
    assert lib.qsa_append(ctypes.byref(c), 2, 1, 4000, P, None, None, P, None, None, P, P, None, 0,
                          None, None) == _lib.QSA_ERR_INVALID_ARG
    assert lib.qsa_append(ctypes.byref(c), 2, 5, 4096, P, None, None, P, None, None, P, P, None, 0,
                          None, None) == _lib.QSA_ERR_UNSUPPORTED
    # a block table with no pages
    assert lib.qsa_append(ctypes.byref(c), 2, 1, 4096, P, None, None, P, None, None, P, P, P, 0,
                          None, None) == _lib.QSA_ERR_INVALID_ARG
    # an empty batch launches nothing
    assert lib.qsa_append(ctypes.byref(c), 0, 1, 4096, None, None, None, None, None, None, None,
                          None, None, 0, None, None) == _lib.QSA_OK


def test_keys_visited_binding_refuses_bad_counters():
    import block_sparse_attention_17_b200 as qsa
    for bad in (torch.zeros(1, dtype=torch.int64), torch.zeros(2, dtype=torch.int64),
                torch.zeros(1, dtype=torch.float32), 7):
        with pytest.raises(ValueError):
            qsa.set_keys_visited(bad)
    qsa.set_keys_visited(None)   # off: no device needed
