"""Seeded synthetic workloads for Qwen Sparse Attention (QSA).

This module only defines shapes and draws random numbers. It holds none of the
method's arithmetic, so both the CUDA path (through the binding) and the
CPU oracle read their inputs from here.

Recipe (one ``numpy.random.default_rng(seed)`` PCG64 stream per workload):

* ragged prefill only: the sequence lengths are drawn first,
  ``rng.integers(lo, hi, endpoint=True, size=batch)``;
* then, in this order: q, k, v, iq, ik, iw, gate;
* q, k, v, iq, ik ~ N(0, 1) / sqrt(last dim); iw ~ U(0, 1); gate ~ N(0, 1);
* bf16 workloads round every fp32 draw to the nearest bf16 (ties to even),
  so both sides see exactly the same values.

Prefill tensors are packed over tokens (``cu_seqlens``):
  q [T, Hq, D], k/v [T, Hkv, D], iq [T, Hi, di], ik [T, di], iw [T, Hi],
  gate [T, Hq, D].
Decode tensors are per sequence:
  q [batch, n_q, Hq, D], k_cache/v_cache [batch, cap, Hkv, D],
  iq [batch, n_q, Hi, di], ik_cache [batch, cap, di], iw [batch, n_q, Hi],
  gate [batch, n_q, Hq, D]; kv_len [batch] counts the tokens present after
  this step's n_q tokens were appended.

The shapes follow the workloads the Qwen4-Exp pages describe: a 48-layer hybrid
model whose QSA layers see contexts up to 262,144 tokens (dev.to article
"Qwen4-Exp: How Per-Layer N-gram Embeddings and Sparse Attention...",
section "What This Means for Practitioners") and MTP draft verification with
one draft token (llama.cpp PR #27739 page, the MTP draft-head commit texts).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Optional

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                    # "prefill" or "decode"
    dtype: str                   # "f32" or "bf16"
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    budget: int
    idx_heads: int
    idx_dim: int
    seed: int
    # prefill
    seqlens: tuple = ()
    ragged_range: Optional[tuple] = None   # (lo, hi): lengths drawn from the seed
    # decode
    batch: int = 0
    kv_len: int = 0
    n_q: int = 0
    cap: int = 0                 # cache rows per sequence (0 => kv_len rounded up to B)
    gate_headwise: bool = False
    rope_dim: int = 0            # indexer rotary embedding (0 = off)
    rope_theta: float = 10000.0
    description: str = ""

    @property
    def topk(self) -> int:
        return self.budget // self.block_size

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def cache_rows(self) -> int:
        if self.cap:
            return self.cap
        b = self.block_size
        return (self.kv_len + b - 1) // b * b


WORKLOADS = {
    "prefill_f32_t1024": Workload(
        name="prefill_f32_t1024", kind="prefill", dtype="f32",
        num_q_heads=4, num_kv_heads=1, head_dim=64, block_size=64, budget=256,
        idx_heads=2, idx_dim=32, seed=0, seqlens=(1024,),
        description="tiny fp32 prefill, 1 sequence of 1024 tokens"),
    "prefill_bf16_t8192": Workload(
        name="prefill_bf16_t8192", kind="prefill", dtype="bf16",
        num_q_heads=16, num_kv_heads=2, head_dim=128, block_size=64, budget=2048,
        idx_heads=4, idx_dim=64, seed=1, seqlens=(8192,),
        description="bf16 prefill, 1 sequence of 8192 tokens"),
    "decode_bf16_b32_kv32768": Workload(
        name="decode_bf16_b32_kv32768", kind="decode", dtype="bf16",
        num_q_heads=16, num_kv_heads=2, head_dim=128, block_size=64, budget=2048,
        idx_heads=4, idx_dim=64, seed=2, batch=32, kv_len=32768, n_q=1,
        description="bf16 decode, 32 sequences x 32768 cached tokens, 1 new token"),
    "mtp_verify_bf16_b4_kv262144": Workload(
        name="mtp_verify_bf16_b4_kv262144", kind="decode", dtype="bf16",
        num_q_heads=16, num_kv_heads=2, head_dim=128, block_size=128, budget=4096,
        idx_heads=4, idx_dim=64, seed=3, batch=4, kv_len=262144, n_q=2,
        description="bf16 MTP-verify decode, 4 sequences x 262144 cached tokens, 2 new tokens"),
    "ragged_prefill_bf16_4seq": Workload(
        name="ragged_prefill_bf16_4seq", kind="prefill", dtype="bf16",
        num_q_heads=32, num_kv_heads=4, head_dim=128, block_size=128, budget=4096,
        idx_heads=8, idx_dim=64, seed=4, ragged_range=(8192, 32768), seqlens=(),
        batch=4,
        description="bf16 ragged prefill, 4 sequences with lengths in [8192, 32768]"),
}

# the order in which the five workloads are listed by the project statement
WORKLOAD_ORDER = [
    "prefill_f32_t1024",
    "prefill_bf16_t8192",
    "decode_bf16_b32_kv32768",
    "mtp_verify_bf16_b4_kv262144",
    "ragged_prefill_bf16_4seq",
]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even), returned
    as a new float32 array. Inputs are finite draws, so NaN handling is not
    needed."""
    return _round_bf16_inplace(np.array(x, dtype=np.float32, order="C"))


def _round_bf16_inplace(x: np.ndarray) -> np.ndarray:
    """round_to_bf16 on a C-contiguous float32 array that the caller owns,
    in place, one slice at a time (no array-sized temporaries)."""
    u = x.reshape(-1).view(np.uint32)
    step = 1 << 20
    buf = np.empty(min(step, u.size), dtype=np.uint32)
    for s0 in range(0, u.size, step):
        seg = u[s0:s0 + step]
        lsb = buf[:seg.size]
        np.right_shift(seg, np.uint32(16), out=lsb)
        lsb &= np.uint32(1)
        lsb += np.uint32(0x7FFF)
        seg += lsb
        seg &= np.uint32(0xFFFF0000)
    return x


def _normal(rng, shape, scale, dtype):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return _round_bf16_inplace(x) if dtype == "bf16" else x


def _uniform(rng, shape, dtype_unused=None):
    return rng.random(size=shape, dtype=np.float32)


def resolve_seqlens(w: Workload, rng: Optional[np.random.Generator] = None):
    """Return (seqlens, rng): for ragged workloads the lengths are the first draw."""
    if rng is None:
        rng = np.random.default_rng(w.seed)
    if w.ragged_range is not None and not w.seqlens:
        lo, hi = w.ragged_range
        lens = rng.integers(lo, hi, endpoint=True, size=w.batch)
        return tuple(int(x) for x in lens), rng
    return tuple(int(x) for x in w.seqlens), rng


def make_prefill_inputs(w: Workload) -> dict:
    assert w.kind == "prefill"
    seqlens, rng = resolve_seqlens(w)
    T = int(sum(seqlens))
    D, Hq, Hkv, Hi, di = w.head_dim, w.num_q_heads, w.num_kv_heads, w.idx_heads, w.idx_dim
    inv = lambda d: 1.0 / np.sqrt(d)
    out = {}
    out["q"] = _normal(rng, (T, Hq, D), inv(D), w.dtype)
    out["k"] = _normal(rng, (T, Hkv, D), inv(D), w.dtype)
    out["v"] = _normal(rng, (T, Hkv, D), inv(D), w.dtype)
    out["iq"] = _normal(rng, (T, Hi, di), inv(di), w.dtype)
    out["ik"] = _normal(rng, (T, di), inv(di), w.dtype)
    out["iw"] = _uniform(rng, (T, Hi))
    gshape = (T, Hq) if w.gate_headwise else (T, Hq, D)
    out["gate"] = _normal(rng, gshape, 1.0, w.dtype)
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    out["cu_seqlens"] = cu
    out["seqlens"] = np.asarray(seqlens, dtype=np.int64)
    out["max_seqlen"] = int(max(seqlens)) if seqlens else 0
    return out


def make_decode_inputs(w: Workload, kv_lens: Optional[np.ndarray] = None) -> dict:
    """kv_lens (optional) overrides the per-sequence post-append lengths; they
    must not exceed the cache rows."""
    assert w.kind == "decode"
    rng = np.random.default_rng(w.seed)
    b, nq, cap = w.batch, w.n_q, w.cache_rows()
    D, Hq, Hkv, Hi, di = w.head_dim, w.num_q_heads, w.num_kv_heads, w.idx_heads, w.idx_dim
    inv = lambda d: 1.0 / np.sqrt(d)
    out = {}
    out["q"] = _normal(rng, (b, nq, Hq, D), inv(D), w.dtype)
    out["k_cache"] = _normal(rng, (b, cap, Hkv, D), inv(D), w.dtype)
    out["v_cache"] = _normal(rng, (b, cap, Hkv, D), inv(D), w.dtype)
    out["iq"] = _normal(rng, (b, nq, Hi, di), inv(di), w.dtype)
    out["ik_cache"] = _normal(rng, (b, cap, di), inv(di), w.dtype)
    out["iw"] = _uniform(rng, (b, nq, Hi))
    gshape = (b, nq, Hq) if w.gate_headwise else (b, nq, Hq, D)
    out["gate"] = _normal(rng, gshape, 1.0, w.dtype)
    if kv_lens is None:
        kv_lens = np.full(b, w.kv_len, dtype=np.int32)
    kv_lens = np.asarray(kv_lens, dtype=np.int32)
    assert kv_lens.shape == (b,) and int(kv_lens.max(initial=0)) <= cap
    out["kv_len"] = kv_lens
    out["cap"] = cap
    return out


def make_inputs(w: Workload, **kw) -> dict:
    return make_prefill_inputs(w) if w.kind == "prefill" else make_decode_inputs(w, **kw)
