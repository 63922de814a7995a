"""Plain fp64 CPU oracle for Qwen Sparse Attention (QSA).

TEST INFRASTRUCTURE ONLY. Nothing in the library imports this module: only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` use
it. It shares no code with the CUDA path; the only common module is the seeded
input generator (``block_sparse_attention_17_b200.workloads``), which holds no
arithmetic of the method.

What QSA computes, as the pages state it:

* instagit "Native Backend Components for the Qwen4-Generation Preview Family
  in MTPLX", section "Qwen Sparse Attention (QSA)": standard gated GQA whose
  causal mask is intersected with a per-query-token selection; the selection
  comes from a DeepSeek-V3.2-style indexer that relu-scores mean-pooled key
  blocks and keeps the top-(budget/ratio) blocks plus the incomplete tail block.
* dev.to "Qwen4-Exp: How Per-Layer N-gram Embeddings and Sparse Attention ...",
  section "Qwen Sparse Attention: Block-Level Selection ...": keys are compressed
  into blocks, blocks are scored, the best ones get full attention, and the
  trailing incomplete block is always kept uncompressed.
* llama.cpp PR #27739 page, the QSA block-composition commit text ("The value
  gate ..."): the indexer settings -- weights per head, n_head_scale = 1,
  softmax_scale = index_head_dim ** -0.5, candidate window end = kv_len / ratio
  (complete blocks only) -- and the sigmoid gate on the output; worked example at
  kv_len 3002, budget 2048, ratio 4.
* ramgpt "Porting Qwen4 to llama.cpp", sections "QSA Should First Be
  Implemented as Selection Semantics" (visible width bound
  w = min(n_kv, budget + ratio - 1), dense equality below it) and
  "Above the Budget, Correctness Becomes Set Selection" (Jaccard overlap).

Readings where the pages leave a step open (each one is also listed in the
design notes of the repository):

* R1 tail: the tail is the n mod B newest visible tokens; when n is a multiple
  of B the tail is empty and the query's own block is complete and competes in
  the top-k like any other block.
* R2 candidates: only complete visible blocks j < floor(n / B) are scored.
* R3 one indexer key row per token, shared by every indexer head.
* R4 one selection per query token, shared by all query and KV heads.
* R5 w[t, h] is an input per query token per indexer head.
* R6 score scale c = index_scale (default idx_dim ** -0.5).
* R7 ties: lower block index wins; -0 is the same score as +0.
* R8 GQA: query head h reads KV head h // (Hq / Hkv).
* R9 gate: elementwise over [Hq, D] (headwise [Hq] optional), out = sigmoid(g) * o.
* R10 attention scale: softmax_scale (default head_dim ** -0.5).
* R11 decode: kv_len counts tokens after this step's n_q tokens were appended;
  new query i sees n = kv_len - n_q + 1 + i tokens.
* R12 indexer rotary embedding, optional (rope_dim = 0 turns it off and is the
  default): the query of the indexer is rotated at its own position (the token
  index within the sequence, n - 1 for a query that sees n tokens); the pooled
  key of block j is the mean of the block's raw indexer keys rotated at the
  block's first position j * B; both with one angle table. The rotation is the
  ordinary partial rotary embedding: pairs (f, f + rope_dim / 2) of the first
  rope_dim dims, frequency f has inverse wavelength theta ** (-2 f / rope_dim)
  rounded to fp32, and the angle is the fp32 product of the position and that
  value (cos and sin of the fp32 angle are then taken in fp64).

Every pin of these functions lives in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Iterable, Optional, Sequence

import numpy as np


# --------------------------------------------------------------------------
# step 1: block mean-pooling of indexer keys
# (instagit MTPLX page, "Qwen Sparse Attention (QSA)": mean-pooled key blocks;
#  dev.to page, "Qwen Sparse Attention": the key sequence is compressed into blocks)
# --------------------------------------------------------------------------
def pool_blocks(ik_rows: np.ndarray, block_size: int) -> np.ndarray:
    """kbar[j] = (1/B) * sum_{i<B} ik[j*B + i] for every complete block j.

    ik_rows: [n, di] indexer keys of one sequence. Returns [floor(n/B), di] fp64.
    """
    ik_rows = np.asarray(ik_rows, dtype=np.float64)
    n, di = ik_rows.shape
    nblk = n // block_size
    out = np.empty((nblk, di), dtype=np.float64)
    for j in range(nblk):
        out[j] = ik_rows[j * block_size:(j + 1) * block_size].sum(axis=0) / block_size
    return out


# --------------------------------------------------------------------------
# optional: rotary embedding of the indexer (R12)
# (llama.cpp PR #27739 page, QSA block-composition commit text: the indexer is
#  fed the roped query and the raw keys, and the pooled indexer keys take the
#  same rope angles as the query; instagit MTPLX page, "Multidimensional Rotary
#  Embeddings (M-RoPE)": for text the rotary embedding is the ordinary partial
#  rotary embedding)
# --------------------------------------------------------------------------
def rope_params(cfg) -> tuple:
    """(rope_dim, theta as an fp32 value) of a config; rope_dim 0 = no rotation."""
    r = int(getattr(cfg, "rope_dim", 0) or 0)
    theta = float(np.float32(getattr(cfg, "rope_theta", 10000.0) or 10000.0))
    return r, theta


def rope_inv_freq(rope_dim: int, theta: float) -> np.ndarray:
    """theta ** (-2 f / rope_dim) for f < rope_dim / 2, each rounded to fp32."""
    th = float(np.float32(theta))
    return np.array([np.float32(th ** (-2.0 * f / rope_dim)) for f in range(rope_dim // 2)],
                    dtype=np.float32)


def rope_angles(pos: int, rope_dim: int, theta: float) -> np.ndarray:
    """The fp32 products pos * inv_freq[f] (round to nearest even), as fp64."""
    return (np.float32(pos) * rope_inv_freq(rope_dim, theta)).astype(np.float64)


def rope_rotate(x, pos: int, rope_dim: int, theta: float) -> np.ndarray:
    """Rotates the pairs (x[f], x[f + h]), h = rope_dim / 2, of the last axis
    by angle[f] (counter-clockwise: (1, 0) goes to (cos, sin)); the dims from
    rope_dim on are unchanged."""
    x = np.array(x, dtype=np.float64)
    if rope_dim == 0:
        return x
    h = rope_dim // 2
    a = rope_angles(pos, rope_dim, theta)
    c, s = np.cos(a), np.sin(a)
    x1 = x[..., :h].copy()
    x2 = x[..., h:rope_dim].copy()
    x[..., :h] = x1 * c - x2 * s
    x[..., h:rope_dim] = x2 * c + x1 * s
    return x


def pooled_keys(cfg, ik_rows) -> np.ndarray:
    """Step 1 with R12: block means, row j rotated at position j * B."""
    B = cfg.block_size
    kbar = pool_blocks(ik_rows, B)
    r, theta = rope_params(cfg)
    if r:
        for j in range(kbar.shape[0]):
            kbar[j] = rope_rotate(kbar[j], j * B, r, theta)
    return kbar


# --------------------------------------------------------------------------
# step 2: relu-weighted indexer score of every candidate block
# (PR #27739 page, QSA composition commit: weights, n_head_scale = 1,
#  softmax_scale = index_head_dim ** -0.5, window end = kv_len / ratio)
# --------------------------------------------------------------------------
def index_scores(iq_t: np.ndarray, iw_t: np.ndarray, kbar: np.ndarray,
                 index_scale: float) -> np.ndarray:
    """s[j] = c * sum_h w[h] * max(0, iq[h] . kbar[j]) for the given candidates.

    iq_t: [Hi, di]; iw_t: [Hi]; kbar: [nc, di]. Returns [nc] fp64.
    """
    iq_t = np.asarray(iq_t, dtype=np.float64)
    iw_t = np.asarray(iw_t, dtype=np.float64)
    kbar = np.asarray(kbar, dtype=np.float64)
    dots = kbar @ iq_t.T                      # [nc, Hi]
    return index_scale * (np.maximum(dots, 0.0) @ iw_t)


# --------------------------------------------------------------------------
# step 3: top-(budget/B) candidates under (score desc, index asc)
# (instagit MTPLX page: top-(budget/ratio) blocks; R7 for ties)
# --------------------------------------------------------------------------
def select_topk(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the min(k, nc) best candidates, returned in ascending order.

    The order is a stable sort by descending score; equal scores (and +0/-0)
    keep ascending block index, so the lower index wins a tie.
    """
    scores = np.asarray(scores, dtype=np.float64)
    nc = scores.shape[0]
    keyed = sorted(range(nc), key=lambda j: (-(scores[j] + 0.0), j))
    return np.array(sorted(keyed[:min(k, nc)]), dtype=np.int64)


# --------------------------------------------------------------------------
# step 4: the visible token set of one query
# --------------------------------------------------------------------------
def visible_positions(n: int, block_size: int, selected: Sequence[int]) -> np.ndarray:
    """Positions of the selected complete blocks followed by the tail
    [floor(n/B)*B, n). (instagit + dev.to pages: the incomplete tail block is
    always kept; R1 for n a multiple of B.)"""
    nc = n // block_size
    parts = [np.arange(j * block_size, (j + 1) * block_size) for j in selected]
    parts.append(np.arange(nc * block_size, n))
    return np.concatenate(parts).astype(np.int64) if parts else np.zeros(0, np.int64)


# --------------------------------------------------------------------------
# step 5: gated GQA attention over a token set
# (instagit MTPLX page: standard gated GQA; PR #27739 page: the sigmoid gate on the output)
# --------------------------------------------------------------------------
def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def gated_attention(q_t: np.ndarray, K: np.ndarray, V: np.ndarray,
                    positions: np.ndarray, gate_t: np.ndarray,
                    softmax_scale: float):
    """One query token over the keys at ``positions``.

    q_t [Hq, D]; K, V [n, Hkv, D]; gate_t [Hq, D] or [Hq].
    Returns out [Hq, D] = sigmoid(gate) * softmax(scale * q K^T) V and the
    natural-log LSE [Hq] of the scaled logits.
    """
    q_t = np.asarray(q_t, dtype=np.float64)
    Hq, D = q_t.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    o = np.zeros((Hq, D), dtype=np.float64)
    lse = np.full(Hq, -np.inf, dtype=np.float64)
    if len(positions) == 0:
        return o, lse
    for kvh in range(Hkv):
        Ks = np.asarray(K[positions, kvh, :], dtype=np.float64)    # [n, D]
        Vs = np.asarray(V[positions, kvh, :], dtype=np.float64)
        for h in range(kvh * G, (kvh + 1) * G):                     # heads reading this KV head
            logits = softmax_scale * (Ks @ q_t[h])
            m = logits.max()
            p = np.exp(logits - m)
            l = p.sum()
            o[h] = (p @ Vs) / l
            lse[h] = m + math.log(l)
    g = sigmoid(gate_t)
    if g.ndim == 1:
        g = g[:, None]
    return g * o, lse


# --------------------------------------------------------------------------
# composition: one query of QSA
# --------------------------------------------------------------------------
@dataclass
class QueryResult:
    n: int
    nc: int
    scores: np.ndarray     # [nc] fp64
    selected: np.ndarray   # ascending block ids
    tail: int              # tail length in tokens
    block_size: int
    out: Optional[np.ndarray] = None   # [Hq, D]
    lse: Optional[np.ndarray] = None   # [Hq]

    @property
    def nsel(self) -> int:
        """Selected blocks, counting the tail block when it is non-empty."""
        return len(self.selected) + (1 if self.tail > 0 else 0)

    @property
    def tokens(self) -> int:
        """Visible tokens: B per selected complete block plus the tail."""
        return len(self.selected) * self.block_size + self.tail


def _scales(cfg):
    sm = getattr(cfg, "softmax_scale", None) or cfg.head_dim ** -0.5
    isc = getattr(cfg, "index_scale", None) or cfg.idx_dim ** -0.5
    return float(sm), float(isc)


def qsa_query(cfg, n: int, kbar: np.ndarray, iq_t, iw_t, q_t=None, K=None, V=None,
              gate_t=None, attend: bool = True) -> QueryResult:
    """QSA for one query that sees n tokens of its sequence.

    kbar: pooled keys of the sequence (at least floor(n/B) rows; rotated by
    pooled_keys when the config has a rotary embedding).
    """
    B = cfg.block_size
    k = cfg.budget // B
    sm_scale, idx_scale = _scales(cfg)
    nc = n // B
    r, theta = rope_params(cfg)
    if r and nc > 0:
        iq_t = rope_rotate(iq_t, n - 1, r, theta)     # R12: the query's own position
    s = index_scores(iq_t, iw_t, kbar[:nc], idx_scale) if nc > 0 else np.zeros(0)
    sel = select_topk(s, k)
    tail = n - nc * B
    res = QueryResult(n=n, nc=nc, scores=s, selected=sel, tail=tail, block_size=B)
    if attend:
        pos = visible_positions(n, B, sel)
        res.out, res.lse = gated_attention(q_t, K, V, pos, gate_t, sm_scale)
    return res


def qsa_prefill(cfg, inp: dict, queries: Optional[Iterable[int]] = None,
                attend: bool = True) -> dict:
    """QSA prefill over packed sequences. ``queries`` are global token indices
    (default: every token). Returns {token: QueryResult} plus the pooled keys
    of every sequence under key "pooled" (list of [floor(L/B), di])."""
    cu = np.asarray(inp["cu_seqlens"], dtype=np.int64)
    nseq = len(cu) - 1
    pooled = [pooled_keys(cfg, inp["ik"][cu[b]:cu[b + 1]]) for b in range(nseq)]
    T = int(cu[-1])
    qs = range(T) if queries is None else queries
    res = {}
    for t in qs:
        t = int(t)
        b = int(np.searchsorted(cu, t, side="right") - 1)
        s0 = int(cu[b])
        n = t - s0 + 1
        r = qsa_query(cfg, n, pooled[b], inp["iq"][t], inp["iw"][t],
                      q_t=inp["q"][t] if attend else None,
                      K=inp["k"][s0:int(cu[b + 1])] if attend else None,
                      V=inp["v"][s0:int(cu[b + 1])] if attend else None,
                      gate_t=inp["gate"][t] if attend else None, attend=attend)
        res[t] = r
    return {"queries": res, "pooled": pooled}


def decode_visible(kv_len: int, n_q: int, i: int) -> int:
    """R11: tokens visible to new query i of a step that appended n_q tokens."""
    return kv_len - n_q + 1 + i


def qsa_decode(cfg, inp: dict, pairs: Optional[Iterable[tuple]] = None,
               attend: bool = True) -> dict:
    """QSA decode. ``pairs`` are (sequence, new-query index) pairs, default all.
    The pooled keys are recomputed here from the raw indexer-key cache rows."""
    kv = np.asarray(inp["kv_len"], dtype=np.int64)
    batch, n_q = inp["q"].shape[0], inp["q"].shape[1]
    if pairs is None:
        pairs = [(b, i) for b in range(batch) for i in range(n_q)]
    pooled_cache = {}
    res = {}
    for b, i in pairs:
        L = int(kv[b])
        if b not in pooled_cache:
            pooled_cache[b] = pooled_keys(cfg, inp["ik_cache"][b, :L])
        n = decode_visible(L, n_q, i)
        r = qsa_query(cfg, n, pooled_cache[b], inp["iq"][b, i], inp["iw"][b, i],
                      q_t=inp["q"][b, i] if attend else None,
                      K=inp["k_cache"][b, :L] if attend else None,
                      V=inp["v_cache"][b, :L] if attend else None,
                      gate_t=inp["gate"][b, i] if attend else None, attend=attend)
        res[(b, i)] = r
    return {"queries": res, "pooled": pooled_cache}


# --------------------------------------------------------------------------
# independent dense reference: causal gated GQA with no selection
# (ramgpt page, "QSA Should First Be Implemented as Selection Semantics":
#  below the budget nothing can be pruned and QSA equals dense attention)
# --------------------------------------------------------------------------
def dense_gated_gqa(q, k, v, gate, softmax_scale: float):
    """Dense causal attention of one sequence, written as full matrices.

    q [L, Hq, D], k/v [L, Hkv, D], gate [L, Hq, D] or [L, Hq].
    Returns out [L, Hq, D], lse [L, Hq].
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    L, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    causal = np.tril(np.ones((L, L), dtype=bool))
    out = np.empty((L, Hq, D))
    lse = np.empty((L, Hq))
    for h in range(Hq):
        S = softmax_scale * (q[:, h, :] @ k[:, h // G, :].T)
        S = np.where(causal, S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        l = P.sum(axis=1, keepdims=True)
        out[:, h, :] = (P @ v[:, h // G, :]) / l
        lse[:, h] = (m + np.log(l))[:, 0]
    g = sigmoid(gate)
    if g.ndim == 2:
        g = g[:, :, None]
    return g * out, lse


# --------------------------------------------------------------------------
# measurements named by the pages
# --------------------------------------------------------------------------
def jaccard(a: Iterable[int], b: Iterable[int]) -> float:
    """J(A, B) = |A n B| / |A u B| (ramgpt page, "Above the Budget ...")."""
    a, b = set(int(x) for x in a), set(int(x) for x in b)
    u = a | b
    return 1.0 if not u else len(a & b) / len(u)


def visible_width_bound(n_kv: int, budget: int, block_size: int) -> int:
    """w = min(n_kv, budget + ratio - 1) (ramgpt page, "QSA Should First ...")."""
    return min(n_kv, budget + block_size - 1)


def near_tie_excused(oracle_scores: np.ndarray, sel_a: Iterable[int], sel_b: Iterable[int],
                     k: int, rel: float = 1e-5) -> bool:
    """True when two selections differ only by blocks whose oracle scores lie
    within rel * max|s| of the k-th best oracle score (a near-tie at the
    selection boundary). Identical selections are trivially excused."""
    a, b = set(int(x) for x in sel_a), set(int(x) for x in sel_b)
    if a == b:
        return True
    s = np.asarray(oracle_scores, dtype=np.float64)
    if len(a) != len(b):
        return False
    kk = min(k, len(s))
    kth = np.sort(s)[::-1][kk - 1]
    tol = rel * max(float(np.abs(s).max()), 1e-300)
    return all(abs(s[j] - kth) <= tol for j in (a ^ b))
