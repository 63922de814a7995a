"""Python binding of the QSA C ABI (argument marshalling only).

Every function takes CUDA torch tensors, allocates any output the caller did
not pass (torch is used for device memory and streams only), and calls the
matching entry point of libqsa.so on the current stream. Each step of the
computation runs in the library's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import threading
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib

_DT = {torch.float32: _lib.QSA_F32, torch.bfloat16: _lib.QSA_BF16}


@dataclass(frozen=True)
class QSAConfig:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    idx_heads: int
    idx_dim: int
    block_size: int
    budget: int
    softmax_scale: float = 0.0     # 0 => head_dim ** -0.5
    index_scale: float = 0.0       # 0 => idx_dim ** -0.5
    gate_headwise: bool = False
    dtype: torch.dtype = torch.bfloat16
    rope_dim: int = 0              # indexer rotary embedding (0 = off)
    rope_theta: float = 10000.0

    @property
    def topk(self) -> int:
        return self.budget // self.block_size

    @classmethod
    def from_workload(cls, w) -> "QSAConfig":
        return cls(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                   head_dim=w.head_dim, idx_heads=w.idx_heads, idx_dim=w.idx_dim,
                   block_size=w.block_size, budget=w.budget,
                   gate_headwise=bool(w.gate_headwise),
                   dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                   rope_dim=int(w.rope_dim), rope_theta=float(w.rope_theta))

    def c(self) -> _lib.QsaConfigC:
        if self.dtype not in _DT:
            raise TypeError(f"unsupported dtype {self.dtype}")
        return _lib.QsaConfigC(self.num_q_heads, self.num_kv_heads, self.head_dim,
                               self.idx_heads, self.idx_dim, self.block_size, self.budget,
                               float(self.softmax_scale), float(self.index_scale),
                               int(bool(self.gate_headwise)), _DT[self.dtype],
                               int(self.rope_dim), float(self.rope_theta))


_thread = threading.local()   # this host thread's visited-keys counter (its device)


def set_keys_visited(counter: Optional[torch.Tensor]) -> None:
    """Debug counter of visited keys for this host thread (qsa_set_keys_visited):
    counter is a one-element int64 CUDA tensor the caller zeroes; the attention
    kernels of later calls add the (query, head, key) triples they attend over.
    Calls on another GPU than the counter's are refused while it is set. None
    turns it off."""
    if counter is not None:
        if not (isinstance(counter, torch.Tensor) and counter.is_cuda and
                counter.dtype == torch.int64 and counter.numel() == 1):
            raise ValueError("counter must be a one-element int64 CUDA tensor")
    _lib.lib().qsa_set_keys_visited(None if counter is None else ctypes.c_void_p(counter.data_ptr()))
    _thread.keys_visited_device = None if counter is None else counter.device


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _one_device(dev, stream=None, **tensors):
    """Every tensor argument must live on ``dev``, the GPU the call runs on (the
    library launches on the current device and takes device pointers as they
    are); a mismatch raises instead of launching."""
    for name, t in tensors.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}: every tensor of one "
                             "call must be on the same GPU")
    if stream is not None and stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, expected {dev}")
    kvd = getattr(_thread, "keys_visited_device", None)
    if kvd is not None and kvd != dev:
        raise ValueError(f"the visited-keys counter is on {kvd}, the call on {dev}")


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]):
    if workspace is not None:
        if workspace.device != device:
            raise ValueError(f"workspace is on {workspace.device}, expected {device}")
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace smaller than {nbytes} bytes")
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def prefill_workspace_size(cfg: QSAConfig, batch: int, total_tokens: int, max_seqlen: int) -> int:
    c = cfg.c()
    n = _lib.lib().qsa_prefill_workspace_size(ctypes.byref(c), batch, total_tokens, max_seqlen)
    if n == 0 and total_tokens > 0:
        _lib.check(_lib.QSA_ERR_INVALID_ARG, "qsa_prefill_workspace_size")
    return int(n)


def decode_workspace_size(cfg: QSAConfig, batch: int, n_q: int, cap: int) -> int:
    c = cfg.c()
    n = _lib.lib().qsa_decode_workspace_size(ctypes.byref(c), batch, n_q, cap)
    if n == 0 and batch > 0:
        _lib.check(_lib.QSA_ERR_INVALID_ARG, "qsa_decode_workspace_size")
    return int(n)


def _check_prefill(cfg, q, k, v, iq, ik, iw, gate, cu_seqlens):
    T = q.shape[0]
    dt = cfg.dtype
    _need(q, "q", dt, (T, cfg.num_q_heads, cfg.head_dim))
    _need(k, "k", dt, (T, cfg.num_kv_heads, cfg.head_dim))
    _need(v, "v", dt, (T, cfg.num_kv_heads, cfg.head_dim))
    _need(iq, "iq", dt, (T, cfg.idx_heads, cfg.idx_dim))
    _need(ik, "ik", dt, (T, cfg.idx_dim))
    _need(iw, "iw", torch.float32, (T, cfg.idx_heads))
    if gate is not None:
        _need(gate, "gate", dt, (T, cfg.num_q_heads) if cfg.gate_headwise
              else (T, cfg.num_q_heads, cfg.head_dim))
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    return T, cu_seqlens.shape[0] - 1


def prefill(cfg: QSAConfig, q, k, v, iq, ik, iw, gate, cu_seqlens, max_seqlen: int, *,
            out=None, lse=None, sel=None, nsel=None, pooled=None, workspace=None,
            want_lse=False, want_sel=False, want_pooled=False, stream=None) -> dict:
    """QSA prefill over packed sequences (qsa_prefill). Returns a dict with
    "out" and, when requested or passed in, "lse", "sel", "nsel", "pooled"."""
    T, batch = _check_prefill(cfg, q, k, v, iq, ik, iw, gate, cu_seqlens)
    dev = q.device
    K1 = cfg.topk + 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(T, cfg.num_q_heads, dtype=torch.float32, device=dev)
    if sel is None and want_sel:
        sel = torch.empty(T, K1, dtype=torch.int32, device=dev)
    if nsel is None and want_sel:
        nsel = torch.empty(T, dtype=torch.int32, device=dev)
    if pooled is None and want_pooled:
        nb = -(-max_seqlen // cfg.block_size)
        pooled = torch.zeros(batch, nb, cfg.idx_dim, dtype=torch.float32, device=dev)
    ws_bytes = prefill_workspace_size(cfg, batch, T, max_seqlen)
    ws = _workspace(ws_bytes, dev, workspace)
    _one_device(dev, stream, q=q, k=k, v=v, iq=iq, ik=ik, iw=iw, gate=gate, cu_seqlens=cu_seqlens,
                out=out, lse=lse, sel=sel, nsel=nsel, pooled=pooled)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_prefill(ctypes.byref(c), batch, T, int(max_seqlen), _ptr(cu_seqlens),
                                    _ptr(q), _ptr(k), _ptr(v), _ptr(iq), _ptr(ik), _ptr(iw),
                                    _ptr(gate), _ptr(out), _ptr(lse), _ptr(sel), _ptr(nsel),
                                    _ptr(pooled), _ptr(ws), ws.numel(), _stream(stream))
        _lib.check(st, "qsa_prefill")
    # int32 error word at the start of the workspace: non-zero once the call
    # has run if a kernel gave up on a bounded wait
    return {"out": out, "lse": lse, "sel": sel, "nsel": nsel, "pooled": pooled,
            "error_word": ws[:4].view(torch.int32)}


def select(cfg: QSAConfig, iq, ik, iw, cu_seqlens, max_seqlen: int, *, want_scores=False,
           want_pooled=False, workspace=None, stream=None) -> dict:
    """Selection only (qsa_select): sel [T, k+1], nsel [T], optional scores
    [T, max_seqlen // B] and pooled keys."""
    T = iq.shape[0]
    dt = cfg.dtype
    _need(iq, "iq", dt, (T, cfg.idx_heads, cfg.idx_dim))
    _need(ik, "ik", dt, (T, cfg.idx_dim))
    _need(iw, "iw", torch.float32, (T, cfg.idx_heads))
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    batch = cu_seqlens.shape[0] - 1
    dev = iq.device
    sel = torch.empty(T, cfg.topk + 1, dtype=torch.int32, device=dev)
    nsel = torch.empty(T, dtype=torch.int32, device=dev)
    scores = (torch.empty(T, max(1, max_seqlen // cfg.block_size), dtype=torch.float32,
                          device=dev) if want_scores else None)
    pooled = None
    if want_pooled:
        nb = -(-max_seqlen // cfg.block_size)
        pooled = torch.zeros(batch, nb, cfg.idx_dim, dtype=torch.float32, device=dev)
    ws = _workspace(prefill_workspace_size(cfg, batch, T, max_seqlen), dev, workspace)
    _one_device(dev, stream, ik=ik, iw=iw, cu_seqlens=cu_seqlens)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_select(ctypes.byref(c), batch, T, int(max_seqlen), _ptr(cu_seqlens),
                                   _ptr(iq), _ptr(ik), _ptr(iw), _ptr(sel), _ptr(nsel),
                                   _ptr(scores), _ptr(pooled), _ptr(ws), ws.numel(),
                                   _stream(stream))
        _lib.check(st, "qsa_select")
    return {"sel": sel, "nsel": nsel, "scores": scores, "pooled": pooled}


def _check_decode(cfg, q, k_cache, v_cache, iq, ik_cache, iw, gate, pooled_cache, kv_len):
    dt = cfg.dtype
    batch, n_q = q.shape[0], q.shape[1]
    cap = k_cache.shape[1]
    _need(q, "q", dt, (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    if k_cache is not None:
        _need(k_cache, "k_cache", dt, (batch, cap, cfg.num_kv_heads, cfg.head_dim))
        _need(v_cache, "v_cache", dt, (batch, cap, cfg.num_kv_heads, cfg.head_dim))
    _need(iq, "iq", dt, (batch, n_q, cfg.idx_heads, cfg.idx_dim))
    _need(ik_cache, "ik_cache", dt, (batch, cap, cfg.idx_dim))
    _need(iw, "iw", torch.float32, (batch, n_q, cfg.idx_heads))
    if gate is not None:
        _need(gate, "gate", dt, (batch, n_q, cfg.num_q_heads) if cfg.gate_headwise
              else (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(pooled_cache, "pooled_cache", torch.float32,
          (batch, cap // cfg.block_size, cfg.idx_dim))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    return batch, n_q, cap


def decode(cfg: QSAConfig, q, k_cache, v_cache, iq, ik_cache, iw, gate, pooled_cache, kv_len,
           *, out=None, lse=None, sel=None, nsel=None, dev_err=None, workspace=None,
           want_lse=False, want_sel=False, stream=None) -> dict:
    """One QSA decode step (qsa_decode). pooled_cache is updated in place for
    the blocks this step completes."""
    batch, n_q, cap = _check_decode(cfg, q, k_cache, v_cache, iq, ik_cache, iw, gate,
                                    pooled_cache, kv_len)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(batch, n_q, cfg.num_q_heads, dtype=torch.float32, device=dev)
    if sel is None and want_sel:
        sel = torch.empty(batch, n_q, cfg.topk + 1, dtype=torch.int32, device=dev)
    if nsel is None and want_sel:
        nsel = torch.empty(batch, n_q, dtype=torch.int32, device=dev)
    ws = _workspace(decode_workspace_size(cfg, batch, n_q, cap), dev, workspace)
    _one_device(dev, stream, k_cache=k_cache, v_cache=v_cache, iq=iq, ik_cache=ik_cache, iw=iw,
                gate=gate, pooled_cache=pooled_cache, kv_len=kv_len, out=out, lse=lse, sel=sel,
                nsel=nsel, dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_decode(ctypes.byref(c), batch, n_q, cap, _ptr(kv_len), _ptr(q),
                                   _ptr(k_cache), _ptr(v_cache), _ptr(iq), _ptr(ik_cache), _ptr(iw),
                                   _ptr(gate), _ptr(pooled_cache), _ptr(out), _ptr(lse), _ptr(sel),
                                   _ptr(nsel), _ptr(dev_err), _ptr(ws), ws.numel(), _stream(stream))
        _lib.check(st, "qsa_decode")
    return {"out": out, "lse": lse, "sel": sel, "nsel": nsel}


def decode_noalloc(cfg: QSAConfig, q, k_cache, v_cache, iq, ik_cache, iw, gate, pooled_cache,
                   kv_len, *, out=None, lse=None, sel=None, nsel=None, dev_err=None,
                   want_lse=False, want_sel=False, stream=None) -> dict:
    """qsa_decode_noalloc: the decode step with the library's static 4 MiB
    device scratch instead of a workspace, for callers that cannot allocate
    scratch memory. Calls that overlap on the GPU share that scratch and race.
    (Outputs the caller does not pass are still allocated here, by torch.)"""
    batch, n_q, cap = _check_decode(cfg, q, k_cache, v_cache, iq, ik_cache, iw, gate,
                                    pooled_cache, kv_len)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(batch, n_q, cfg.num_q_heads, dtype=torch.float32, device=dev)
    if sel is None and want_sel:
        sel = torch.empty(batch, n_q, cfg.topk + 1, dtype=torch.int32, device=dev)
    if nsel is None and want_sel:
        nsel = torch.empty(batch, n_q, dtype=torch.int32, device=dev)
    _one_device(dev, stream, k_cache=k_cache, v_cache=v_cache, iq=iq, ik_cache=ik_cache, iw=iw,
                gate=gate, pooled_cache=pooled_cache, kv_len=kv_len, out=out, lse=lse, sel=sel,
                nsel=nsel, dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_decode_noalloc(ctypes.byref(c), batch, n_q, cap, _ptr(kv_len), _ptr(q),
                                           _ptr(k_cache), _ptr(v_cache), _ptr(iq), _ptr(ik_cache),
                                           _ptr(iw), _ptr(gate), _ptr(pooled_cache), _ptr(out),
                                           _ptr(lse), _ptr(sel), _ptr(nsel), _ptr(dev_err),
                                           _stream(stream))
        _lib.check(st, "qsa_decode_noalloc")
    return {"out": out, "lse": lse, "sel": sel, "nsel": nsel}


def decode_attend(cfg: QSAConfig, q, k_cache, v_cache, gate, kv_len, sel, nsel, *, out=None,
                  lse=None, want_lse=False, dev_err=None, workspace=None, stream=None) -> dict:
    """Decode attention over caller-given selections (qsa_decode_attend):
    sel [batch, n_q, k + 1] int32 block ids (ascending, nsel[b, i] used),
    nsel [batch, n_q] int32; returns {"out", "lse"}."""
    dt = cfg.dtype
    batch, n_q = q.shape[0], q.shape[1]
    cap = k_cache.shape[1]
    _need(q, "q", dt, (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(k_cache, "k_cache", dt, (batch, cap, cfg.num_kv_heads, cfg.head_dim))
    _need(v_cache, "v_cache", dt, (batch, cap, cfg.num_kv_heads, cfg.head_dim))
    gshape = ((batch, n_q, cfg.num_q_heads) if cfg.gate_headwise
              else (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(gate, "gate", dt, gshape)
    _need(kv_len, "kv_len", torch.int32, (batch,))
    _need(sel, "sel", torch.int32, (batch, n_q, cfg.topk + 1))
    _need(nsel, "nsel", torch.int32, (batch, n_q))
    dev = q.device
    out = out if out is not None else torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty(batch, n_q, cfg.num_q_heads, dtype=torch.float32, device=dev)
    ws = _workspace(decode_workspace_size(cfg, batch, n_q, cap), dev, workspace)
    _one_device(dev, stream, k_cache=k_cache, v_cache=v_cache, gate=gate, kv_len=kv_len, sel=sel,
                nsel=nsel, out=out, lse=lse, dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_decode_attend(ctypes.byref(c), batch, n_q, cap, _ptr(kv_len), _ptr(q),
                                          _ptr(k_cache), _ptr(v_cache), _ptr(gate), _ptr(sel),
                                          _ptr(nsel), _ptr(out), _ptr(lse), _ptr(dev_err), _ptr(ws),
                                          ws.numel(), _stream(stream))
        _lib.check(st, "qsa_decode_attend")
    return {"out": out, "lse": lse}


def select_decode(cfg: QSAConfig, iq, ik_cache, iw, pooled_cache, kv_len, *, want_scores=False,
                  dev_err=None, workspace=None, stream=None) -> dict:
    """Decode selection only (qsa_select_decode); also finalises the pooled
    rows completed by this step."""
    dt = cfg.dtype
    batch, n_q = iq.shape[0], iq.shape[1]
    cap = ik_cache.shape[1]
    _need(iq, "iq", dt, (batch, n_q, cfg.idx_heads, cfg.idx_dim))
    _need(ik_cache, "ik_cache", dt, (batch, cap, cfg.idx_dim))
    _need(iw, "iw", torch.float32, (batch, n_q, cfg.idx_heads))
    _need(pooled_cache, "pooled_cache", torch.float32, (batch, cap // cfg.block_size, cfg.idx_dim))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    dev = iq.device
    sel = torch.empty(batch, n_q, cfg.topk + 1, dtype=torch.int32, device=dev)
    nsel = torch.empty(batch, n_q, dtype=torch.int32, device=dev)
    scores = (torch.empty(batch, n_q, cap // cfg.block_size, dtype=torch.float32, device=dev)
              if want_scores else None)
    ws = _workspace(decode_workspace_size(cfg, batch, n_q, cap), dev, workspace)
    _one_device(dev, stream, ik_cache=ik_cache, iw=iw, pooled_cache=pooled_cache, kv_len=kv_len,
                dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_select_decode(ctypes.byref(c), batch, n_q, cap, _ptr(kv_len), _ptr(iq),
                                          _ptr(ik_cache), _ptr(iw), _ptr(pooled_cache), _ptr(sel),
                                          _ptr(nsel), _ptr(scores), _ptr(dev_err), _ptr(ws),
                                          ws.numel(), _stream(stream))
        _lib.check(st, "qsa_select_decode")
    return {"sel": sel, "nsel": nsel, "scores": scores}


def pool_build(cfg: QSAConfig, ik_cache, kv_len, pooled_cache=None, *, dev_err=None,
               stream=None):
    """Rebuild the pooled-key cache from the indexer-key cache (qsa_pool_build)."""
    batch, cap = ik_cache.shape[0], ik_cache.shape[1]
    _need(ik_cache, "ik_cache", cfg.dtype, (batch, cap, cfg.idx_dim))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    if pooled_cache is None:
        pooled_cache = torch.zeros(batch, cap // cfg.block_size, cfg.idx_dim,
                                   dtype=torch.float32, device=ik_cache.device)
    dev = ik_cache.device
    _one_device(dev, stream, kv_len=kv_len, pooled_cache=pooled_cache, dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_pool_build(ctypes.byref(c), batch, cap, _ptr(kv_len), _ptr(ik_cache),
                                       _ptr(pooled_cache), _ptr(dev_err), _stream(stream))
        _lib.check(st, "qsa_pool_build")
    return pooled_cache


def append(cfg: QSAConfig, ik_new, ik_cache, pooled_cache, kv_len, *, k_new=None, v_new=None,
           k_cache=None, v_cache=None, block_table=None, dev_err=None, stream=None) -> None:
    """Indexer front end of a decode step (qsa_append): writes the step's new
    rows (ik_new [batch, n_q, di]; k_new / v_new [batch, n_q, Hkv, D], optional)
    at positions kv_len - n_q .. kv_len - 1 of the caches and pools the blocks
    they complete into pooled_cache, in one launch. block_table [batch,
    max_blocks] int32 selects paged caches ([num_pages, B, ...])."""
    dt = cfg.dtype
    batch, n_q = ik_new.shape[0], ik_new.shape[1]
    _need(ik_new, "ik_new", dt, (batch, n_q, cfg.idx_dim))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    B = cfg.block_size
    if block_table is not None:
        _need(block_table, "block_table", torch.int32, (batch, block_table.shape[1]))
        cap, num_pages = block_table.shape[1] * B, ik_cache.shape[0]
        _need(ik_cache, "ik_cache", dt, (num_pages, B, cfg.idx_dim))
        kv_shape = (num_pages, B, cfg.num_kv_heads, cfg.head_dim)
    else:
        cap, num_pages = ik_cache.shape[1], 0
        _need(ik_cache, "ik_cache", dt, (batch, cap, cfg.idx_dim))
        kv_shape = (batch, cap, cfg.num_kv_heads, cfg.head_dim)
    _need(pooled_cache, "pooled_cache", torch.float32, (batch, cap // B, cfg.idx_dim))
    if k_new is not None:
        _need(k_new, "k_new", dt, (batch, n_q, cfg.num_kv_heads, cfg.head_dim))
        _need(v_new, "v_new", dt, (batch, n_q, cfg.num_kv_heads, cfg.head_dim))
        _need(k_cache, "k_cache", dt, kv_shape)
        _need(v_cache, "v_cache", dt, kv_shape)
    dev = ik_new.device
    _one_device(dev, stream, ik_cache=ik_cache, pooled_cache=pooled_cache, kv_len=kv_len,
                k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache,
                block_table=block_table, dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_append(ctypes.byref(c), batch, n_q, cap, _ptr(kv_len), _ptr(k_new),
                                   _ptr(v_new), _ptr(ik_new), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(ik_cache), _ptr(pooled_cache), _ptr(block_table),
                                   num_pages, _ptr(dev_err), _stream(stream))
        _lib.check(st, "qsa_append")


def decode_paged(cfg: QSAConfig, q, k_pages, v_pages, iq, ik_pages, iw, gate, pooled_cache,
                 kv_len, block_table, *, out=None, lse=None, sel=None, nsel=None, dev_err=None,
                 workspace=None, want_lse=False, want_sel=False, stream=None) -> dict:
    """One QSA decode step over a paged cache (qsa_decode_paged): page p holds
    B rows, k_pages/v_pages [num_pages, B, Hkv, D], ik_pages [num_pages, B, di];
    block_table [batch, max_blocks] int32 maps a sequence's block to its page."""
    dt = cfg.dtype
    batch, n_q = q.shape[0], q.shape[1]
    num_pages, B = k_pages.shape[0], cfg.block_size
    max_blocks = block_table.shape[1]
    _need(q, "q", dt, (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(k_pages, "k_pages", dt, (num_pages, B, cfg.num_kv_heads, cfg.head_dim))
    _need(v_pages, "v_pages", dt, (num_pages, B, cfg.num_kv_heads, cfg.head_dim))
    _need(iq, "iq", dt, (batch, n_q, cfg.idx_heads, cfg.idx_dim))
    _need(ik_pages, "ik_pages", dt, (num_pages, B, cfg.idx_dim))
    _need(iw, "iw", torch.float32, (batch, n_q, cfg.idx_heads))
    gshape = ((batch, n_q, cfg.num_q_heads) if cfg.gate_headwise
              else (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(gate, "gate", dt, gshape)
    _need(pooled_cache, "pooled_cache", torch.float32, (batch, max_blocks, cfg.idx_dim))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    _need(block_table, "block_table", torch.int32, (batch, max_blocks))
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(batch, n_q, cfg.num_q_heads, dtype=torch.float32, device=dev)
    if sel is None and want_sel:
        sel = torch.empty(batch, n_q, cfg.topk + 1, dtype=torch.int32, device=dev)
    if nsel is None and want_sel:
        nsel = torch.empty(batch, n_q, dtype=torch.int32, device=dev)
    ws = _workspace(decode_workspace_size(cfg, batch, n_q, max_blocks * B), dev, workspace)
    _one_device(dev, stream, k_pages=k_pages, v_pages=v_pages, iq=iq, ik_pages=ik_pages, iw=iw,
                gate=gate, pooled_cache=pooled_cache, kv_len=kv_len, block_table=block_table,
                out=out, lse=lse, sel=sel, nsel=nsel, dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_decode_paged(ctypes.byref(c), batch, n_q, max_blocks, _ptr(block_table),
                                         num_pages, _ptr(kv_len), _ptr(q), _ptr(k_pages),
                                         _ptr(v_pages), _ptr(iq), _ptr(ik_pages), _ptr(iw),
                                         _ptr(gate), _ptr(pooled_cache), _ptr(out), _ptr(lse),
                                         _ptr(sel), _ptr(nsel), _ptr(dev_err), _ptr(ws), ws.numel(),
                                         _stream(stream))
        _lib.check(st, "qsa_decode_paged")
    return {"out": out, "lse": lse, "sel": sel, "nsel": nsel}


def pool_build_paged(cfg: QSAConfig, ik_pages, kv_len, block_table, pooled_cache=None, *,
                     dev_err=None, stream=None):
    """qsa_pool_build over a paged indexer-key cache (qsa_pool_build_paged)."""
    num_pages = ik_pages.shape[0]
    batch, max_blocks = block_table.shape
    _need(ik_pages, "ik_pages", cfg.dtype, (num_pages, cfg.block_size, cfg.idx_dim))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    _need(block_table, "block_table", torch.int32, (batch, max_blocks))
    if pooled_cache is None:
        pooled_cache = torch.zeros(batch, max_blocks, cfg.idx_dim, dtype=torch.float32,
                                   device=ik_pages.device)
    dev = ik_pages.device
    _one_device(dev, stream, kv_len=kv_len, block_table=block_table, pooled_cache=pooled_cache,
                dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_pool_build_paged(ctypes.byref(c), batch, max_blocks, _ptr(block_table),
                                             num_pages, _ptr(kv_len), _ptr(ik_pages),
                                             _ptr(pooled_cache), _ptr(dev_err), _stream(stream))
        _lib.check(st, "qsa_pool_build_paged")
    return pooled_cache


def decode_fp8(cfg: QSAConfig, q, k_cache, k_scale, v_cache, v_scale, iq, ik_cache, iw, gate,
               pooled_cache, kv_len, *, rotated=False, out=None, lse=None, sel=None, nsel=None,
               dev_err=None, workspace=None, want_lse=False, want_sel=False, stream=None) -> dict:
    """One QSA decode step over fp8 (e4m3) K/V caches (qsa_decode_fp8):
    k_cache/v_cache [batch, cap, Hkv, D] uint8 codes (or torch.float8_e4m3fn),
    k_scale/v_scale [batch, cap, Hkv] fp32 row scales; rotated: the caches hold
    the Walsh-Hadamard-rotated rows."""
    batch, n_q = q.shape[0], q.shape[1]
    cap = k_cache.shape[1]
    if k_cache.dtype != torch.uint8:
        k_cache, v_cache = k_cache.view(torch.uint8), v_cache.view(torch.uint8)
    shp = (batch, cap, cfg.num_kv_heads, cfg.head_dim)
    _need(q, "q", cfg.dtype, (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(k_cache, "k_cache", torch.uint8, shp)
    _need(v_cache, "v_cache", torch.uint8, shp)
    _need(k_scale, "k_scale", torch.float32, shp[:3])
    _need(v_scale, "v_scale", torch.float32, shp[:3])
    _need(iq, "iq", cfg.dtype, (batch, n_q, cfg.idx_heads, cfg.idx_dim))
    _need(ik_cache, "ik_cache", cfg.dtype, (batch, cap, cfg.idx_dim))
    _need(iw, "iw", torch.float32, (batch, n_q, cfg.idx_heads))
    gshape = ((batch, n_q, cfg.num_q_heads) if cfg.gate_headwise
              else (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(gate, "gate", cfg.dtype, gshape)
    _need(pooled_cache, "pooled_cache", torch.float32, (batch, cap // cfg.block_size, cfg.idx_dim))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(batch, n_q, cfg.num_q_heads, dtype=torch.float32, device=dev)
    if sel is None and want_sel:
        sel = torch.empty(batch, n_q, cfg.topk + 1, dtype=torch.int32, device=dev)
    if nsel is None and want_sel:
        nsel = torch.empty(batch, n_q, dtype=torch.int32, device=dev)
    ws = _workspace(decode_workspace_size(cfg, batch, n_q, cap), dev, workspace)
    _one_device(dev, stream, k_cache=k_cache, k_scale=k_scale, v_cache=v_cache, v_scale=v_scale,
                iq=iq, ik_cache=ik_cache, iw=iw, gate=gate, pooled_cache=pooled_cache,
                kv_len=kv_len, out=out, lse=lse, sel=sel, nsel=nsel, dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_decode_fp8(ctypes.byref(c), batch, n_q, cap, _ptr(kv_len), _ptr(q),
                                       _ptr(k_cache), _ptr(k_scale), _ptr(v_cache), _ptr(v_scale),
                                       1 if rotated else 0, _ptr(iq), _ptr(ik_cache), _ptr(iw),
                                       _ptr(gate), _ptr(pooled_cache), _ptr(out), _ptr(lse),
                                       _ptr(sel), _ptr(nsel), _ptr(dev_err), _ptr(ws), ws.numel(),
                                       _stream(stream))
        _lib.check(st, "qsa_decode_fp8")
    return {"out": out, "lse": lse, "sel": sel, "nsel": nsel}


# ------------------------------------------------- context-parallel decode
def cp_pool_build(cfg: QSAConfig, ik_shard, kv_len, block_lo: int, *, dev_err=None,
                  stream=None) -> torch.Tensor:
    """Pooled rows of a context-parallel shard (qsa_cp_pool_build): ik_shard
    [batch, cap, di] holds blocks [block_lo, block_lo + cap / B); kv_len are the
    full lengths. Returns pooled_shard [batch, cap / B, di] fp32 (rows of
    incomplete blocks are zero)."""
    dt = cfg.dtype
    batch, cap = ik_shard.shape[0], ik_shard.shape[1]
    _need(ik_shard, "ik_shard", dt, (batch, cap, cfg.idx_dim))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    dev = ik_shard.device
    pooled = torch.zeros(batch, cap // cfg.block_size, cfg.idx_dim, dtype=torch.float32,
                         device=dev)
    _one_device(dev, stream, kv_len=kv_len, dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_cp_pool_build(ctypes.byref(c), batch, cap, int(block_lo),
                                          _ptr(kv_len), _ptr(ik_shard), _ptr(pooled),
                                          _ptr(dev_err), _stream(stream))
        _lib.check(st, "qsa_cp_pool_build")
    return pooled


def cp_select(cfg: QSAConfig, iq, ik_shard, iw, pooled_shard, kv_len, block_lo: int, *,
              dev_err=None, workspace=None, stream=None) -> dict:
    """Shard selection of a context-parallel decode step (qsa_cp_select):
    this process holds blocks [block_lo, block_lo + cap / B) of every sequence
    (ik_shard [batch, cap, di], pooled_shard [batch, cap / B, di]); kv_len are
    the full lengths. Returns the shard's candidates {"score" [batch, n_q, k]
    fp32, "id" [batch, n_q, k] int32 global block ids}."""
    dt = cfg.dtype
    batch, n_q = iq.shape[0], iq.shape[1]
    cap = ik_shard.shape[1]
    _need(iq, "iq", dt, (batch, n_q, cfg.idx_heads, cfg.idx_dim))
    _need(ik_shard, "ik_shard", dt, (batch, cap, cfg.idx_dim))
    _need(iw, "iw", torch.float32, (batch, n_q, cfg.idx_heads))
    _need(pooled_shard, "pooled_shard", torch.float32, (batch, cap // cfg.block_size, cfg.idx_dim))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    dev = iq.device
    score = torch.empty(batch, n_q, cfg.topk, dtype=torch.float32, device=dev)
    ids = torch.empty(batch, n_q, cfg.topk, dtype=torch.int32, device=dev)
    ws = _workspace(decode_workspace_size(cfg, batch, n_q, cap), dev, workspace)
    _one_device(dev, stream, ik_shard=ik_shard, iw=iw, pooled_shard=pooled_shard, kv_len=kv_len,
                dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_cp_select(ctypes.byref(c), batch, n_q, cap, int(block_lo),
                                      _ptr(kv_len), _ptr(iq), _ptr(ik_shard), _ptr(iw),
                                      _ptr(pooled_shard), _ptr(score), _ptr(ids), _ptr(dev_err),
                                      _ptr(ws), ws.numel(), _stream(stream))
        _lib.check(st, "qsa_cp_select")
    return {"score": score, "id": ids}


def cp_global_topk(cfg: QSAConfig, cand_score, cand_id, kv_len, *, stream=None) -> dict:
    """Global selection from every process's candidates (qsa_cp_global_topk):
    cand_score / cand_id [world, batch, n_q, k]. Returns {"sel" [batch, n_q,
    k + 1], "nsel" [batch, n_q]} as qsa_decode writes them (global ids)."""
    world, batch, n_q, k = cand_score.shape
    _need(cand_score, "cand_score", torch.float32, (world, batch, n_q, cfg.topk))
    _need(cand_id, "cand_id", torch.int32, (world, batch, n_q, cfg.topk))
    _need(kv_len, "kv_len", torch.int32, (batch,))
    dev = cand_score.device
    sel = torch.empty(batch, n_q, cfg.topk + 1, dtype=torch.int32, device=dev)
    nsel = torch.empty(batch, n_q, dtype=torch.int32, device=dev)
    _one_device(dev, stream, cand_id=cand_id, kv_len=kv_len)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_cp_global_topk(ctypes.byref(c), batch, n_q, world, _ptr(kv_len),
                                           _ptr(cand_score), _ptr(cand_id), _ptr(sel),
                                           _ptr(nsel), _stream(stream))
        _lib.check(st, "qsa_cp_global_topk")
    return {"sel": sel, "nsel": nsel}


def cp_attend(cfg: QSAConfig, q, k_shard, v_shard, gate, kv_len, sel, nsel, block_lo: int, *,
              dev_err=None, workspace=None, stream=None) -> dict:
    """Attention over the shard's share of the global selection
    (qsa_cp_attend). Returns {"out" [batch, n_q, Hq, D] fp32 gated partials,
    "lse" [batch, n_q, Hq]}."""
    dt = cfg.dtype
    batch, n_q = q.shape[0], q.shape[1]
    cap = k_shard.shape[1]
    _need(q, "q", dt, (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(k_shard, "k_shard", dt, (batch, cap, cfg.num_kv_heads, cfg.head_dim))
    _need(v_shard, "v_shard", dt, (batch, cap, cfg.num_kv_heads, cfg.head_dim))
    gshape = ((batch, n_q, cfg.num_q_heads) if cfg.gate_headwise
              else (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(gate, "gate", dt, gshape)
    _need(kv_len, "kv_len", torch.int32, (batch,))
    _need(sel, "sel", torch.int32, (batch, n_q, cfg.topk + 1))
    _need(nsel, "nsel", torch.int32, (batch, n_q))
    dev = q.device
    out = torch.empty(batch, n_q, cfg.num_q_heads, cfg.head_dim, dtype=torch.float32, device=dev)
    lse = torch.empty(batch, n_q, cfg.num_q_heads, dtype=torch.float32, device=dev)
    ws = _workspace(decode_workspace_size(cfg, batch, n_q, cap), dev, workspace)
    _one_device(dev, stream, k_shard=k_shard, v_shard=v_shard, gate=gate, kv_len=kv_len, sel=sel,
                nsel=nsel, dev_err=dev_err)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_cp_attend(ctypes.byref(c), batch, n_q, cap, int(block_lo),
                                      _ptr(kv_len), _ptr(q), _ptr(k_shard), _ptr(v_shard),
                                      _ptr(gate), _ptr(sel), _ptr(nsel), _ptr(out), _ptr(lse),
                                      _ptr(dev_err), _ptr(ws), ws.numel(), _stream(stream))
        _lib.check(st, "qsa_cp_attend")
    return {"out": out, "lse": lse}


def cp_merge(cfg: QSAConfig, part_out, part_lse, *, out=None, stream=None) -> dict:
    """Log-sum-exp merge of every process's gated partials (qsa_cp_merge):
    part_out [world, batch, n_q, Hq, D] fp32, part_lse [world, batch, n_q, Hq].
    Returns {"out" (cfg.dtype), "lse"}."""
    world, batch, n_q = part_out.shape[0], part_out.shape[1], part_out.shape[2]
    _need(part_out, "part_out", torch.float32,
          (world, batch, n_q, cfg.num_q_heads, cfg.head_dim))
    _need(part_lse, "part_lse", torch.float32, (world, batch, n_q, cfg.num_q_heads))
    dev = part_out.device
    if out is None:
        out = torch.empty(batch, n_q, cfg.num_q_heads, cfg.head_dim, dtype=cfg.dtype, device=dev)
    _need(out, "out", cfg.dtype, (batch, n_q, cfg.num_q_heads, cfg.head_dim))
    lse = torch.empty(batch, n_q, cfg.num_q_heads, dtype=torch.float32, device=dev)
    _one_device(dev, stream, part_lse=part_lse, out=out)
    c = cfg.c()
    with torch.cuda.device(dev):
        st = _lib.lib().qsa_cp_merge(ctypes.byref(c), batch, n_q, world, _ptr(part_out),
                                     _ptr(part_lse), _ptr(out), _ptr(lse), _stream(stream))
        _lib.check(st, "qsa_cp_merge")
    return {"out": out, "lse": lse}
