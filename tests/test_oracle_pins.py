"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

Each test checks an oracle step against something other than the oracle itself:
closed forms, brute force on tiny inputs, a worked example printed on the
pages, an invariant, or a library routine for a special case. The mutation
tests at the end plant plausible mistakes in the oracle (on the CPU) and check
that some pin turns red.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import qsa_oracle as O
from block_sparse_attention_17_b200.workloads import WORKLOADS, make_prefill_inputs, make_decode_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


class Cfg:
    def __init__(self, **kw):
        self.num_q_heads = 4
        self.num_kv_heads = 2
        self.head_dim = 16
        self.block_size = 4
        self.budget = 8
        self.idx_heads = 2
        self.idx_dim = 8
        self.softmax_scale = None
        self.index_scale = None
        self.__dict__.update(kw)


# ---------------------------------------------------------------- pooling
def pin_pool_closed_form(pool=None):
    pool = pool or O.pool_blocks
    B, di = 8, 5
    consts = np.array([[1.5, -2.0, 0.25, 3.0, 0.0],
                       [-7.0, 4.5, 1.0, -0.5, 2.0],
                       [0.125, 0.0, -1.0, 9.0, -3.5]])
    # three complete blocks of constant rows plus a 5-token incomplete block
    rows = np.concatenate([np.repeat(consts, B, axis=0),
                           np.full((5, di), 1e6)])
    kbar = pool(rows, B)
    assert kbar.shape == (3, di)
    np.testing.assert_array_equal(kbar, consts)
    # an arithmetic ramp inside each block: the mean is the midpoint
    ramp = np.arange(4 * B, dtype=np.float64)[:, None] * np.ones((1, di))
    kb = pool(ramp, B)
    expect = np.array([(j * B + (B - 1) / 2.0) for j in range(4)])[:, None] * np.ones((1, di))
    np.testing.assert_array_equal(kb, expect)


def test_pool_closed_form():
    pin_pool_closed_form()


def test_pool_matches_long_double_sum():
    rng = np.random.default_rng(11)
    B = 64
    ik = rng.standard_normal((7 * B + 13, 32))
    kbar = O.pool_blocks(ik, B)
    ld = ik[: 7 * B].astype(np.longdouble).reshape(7, B, 32).sum(axis=1) / np.longdouble(B)
    np.testing.assert_allclose(kbar, ld.astype(np.float64), rtol=0, atol=1e-15)


# ---------------------------------------------------------------- scores
def pin_scores_hand_example(score=None):
    score = score or O.index_scores
    iq = np.array([[1.0, 0.0], [0.0, 1.0]])
    w = np.array([2.0, 3.0])
    kbar = np.array([[1.0, -1.0], [-2.0, 5.0], [-1.0, -1.0], [4.0, 2.0]])
    c = 0.5
    # by hand: row0 relu(1)*2 + relu(-1)*3 = 2; row1 0*2 + 5*3 = 15;
    #          row2 0; row3 4*2 + 2*3 = 14; times c
    expect = np.array([1.0, 7.5, 0.0, 7.0])
    np.testing.assert_array_equal(score(iq, w, kbar, c), expect)
    # the per-head weight multiplies that head's relu term only
    iq2 = np.array([[1.0, 1.0], [-1.0, 0.0]])
    w2 = np.array([0.25, 4.0])
    kb2 = np.array([[2.0, 1.0], [-3.0, 0.0]])
    # row0: h0 relu(3)*0.25 = 0.75, h1 relu(-2) = 0 -> 0.75 ; row1: h0 relu(-3)=0, h1 relu(3)*4 = 12
    np.testing.assert_array_equal(score(iq2, w2, kb2, 1.0), np.array([0.75, 12.0]))


def test_scores_hand_example():
    pin_scores_hand_example()


def test_scores_default_scale_is_inverse_sqrt_idx_dim():
    # the pages fix softmax_scale = index_head_dim ** -0.5 and n_head_scale = 1
    cfg = Cfg(idx_dim=16, idx_heads=1, block_size=2, budget=2)
    iq = np.zeros((1, 16)); iq[0, 0] = 1.0
    kbar = np.zeros((1, 16)); kbar[0, 0] = 8.0
    r = O.qsa_query(cfg, 3, kbar, iq, np.array([1.0]), attend=False)
    assert r.scores[0] == pytest.approx(8.0 / 4.0, rel=0, abs=0)


# ---------------------------------------------------------------- top-k
def brute_force_topk(scores, k):
    """The unique k-subset A with: every member beats every non-member under
    (higher score, then lower index). Enumerates all subsets."""
    nc = len(scores)
    kk = min(k, nc)
    winners = []
    for A in itertools.combinations(range(nc), kk):
        Aset = set(A)
        ok = all((scores[a] > scores[b]) or (scores[a] == scores[b] and a < b)
                 for a in Aset for b in range(nc) if b not in Aset)
        if ok:
            winners.append(A)
    assert len(winners) == 1
    return list(winners[0])


def pin_topk_brute_force(select=None):
    select = select or O.select_topk
    rng = np.random.default_rng(5)
    cases = []
    for nc in range(0, 11):
        for k in (1, 2, 3, 4, 7):
            cases.append((rng.integers(-2, 3, size=nc).astype(np.float64), k))   # heavy ties
            cases.append((rng.standard_normal(nc), k))
            z = np.maximum(rng.standard_normal(nc), 0.0)                          # relu zeros
            if nc:
                z[rng.integers(0, nc)] = -0.0
            cases.append((z, k))
    for s, k in cases:
        got = list(select(s, k))
        assert got == brute_force_topk(s, k), (s, k, got)


def test_topk_brute_force():
    pin_topk_brute_force()


def test_topk_negative_zero_ties_with_zero():
    # -0 and +0 are the same score; the lower index wins
    s = np.array([0.0, 0.0, -0.0, 1.0, -0.0])
    assert list(O.select_topk(s, 3)) == [0, 1, 3]
    s2 = np.array([-0.0, 0.0])
    assert list(O.select_topk(s2, 1)) == [0]


# ---------------------------------------------------------------- worked example
def test_worked_example_kv3002():
    g = json.load(open(os.path.join(GOLDEN, "qsa_worked_example_kv3002.json")))
    n, budget, B = g["kv_len"], g["budget"], g["compress_ratio"]
    cfg = Cfg(block_size=B, budget=budget, idx_heads=2, idx_dim=8, num_q_heads=8, num_kv_heads=2)
    rng = np.random.default_rng(0)
    ik = rng.standard_normal((n, 8))
    kbar = O.pool_blocks(ik, B)
    r = O.qsa_query(cfg, n, kbar, rng.standard_normal((2, 8)), rng.random(2), attend=False)
    assert r.nc == g["candidate_blocks"]
    assert len(r.selected) == g["selected_blocks"]
    heads = 8
    assert heads * r.tokens == g["keys_visited_sparse"]
    assert heads * n == g["keys_visited_dense"]
    # the visible set is bounded by the pages' width formula
    assert r.tokens <= O.visible_width_bound(n, budget, B)


# ---------------------------------------------------------------- invariants
def test_count_tail_invariant_and_bound():
    cfg = Cfg(block_size=4, budget=12, idx_heads=2, idx_dim=8)
    rng = np.random.default_rng(3)
    L = 61
    ik = rng.standard_normal((L, 8))
    kbar = O.pool_blocks(ik, 4)
    k = cfg.budget // cfg.block_size
    for n in range(1, L + 1):
        r = O.qsa_query(cfg, n, kbar, rng.standard_normal((2, 8)), rng.random(2), attend=False)
        nc = n // 4
        assert r.nc == nc and r.tail == n % 4
        assert len(r.selected) == min(k, nc)
        assert r.nsel == min(k, nc) + (1 if n % 4 else 0)
        pos = O.visible_positions(n, 4, r.selected)
        assert len(pos) == r.tokens == min(k, nc) * 4 + n % 4
        assert len(set(pos.tolist())) == len(pos)
        assert pos.max() == n - 1 if (n % 4) else True   # the tail holds the newest token
        assert len(pos) <= O.visible_width_bound(n, cfg.budget, 4)
        assert all(p < n for p in pos)
        # the tail block is never a candidate
        assert all(j < nc for j in r.selected)


def test_visible_positions_explicit():
    # B = 4, n = 11: blocks 0, 1 complete; tail = {8, 9, 10}
    assert O.visible_positions(11, 4, [1]).tolist() == [4, 5, 6, 7, 8, 9, 10]
    assert O.visible_positions(11, 4, [0, 1]).tolist() == list(range(11))
    # n a multiple of B: empty tail
    assert O.visible_positions(8, 4, [1]).tolist() == [4, 5, 6, 7]
    assert O.visible_positions(3, 4, []).tolist() == [0, 1, 2]


# ---------------------------------------------------------------- dense equivalence
def _rand_seq(rng, L, Hq, Hkv, D, Hi, di, headwise=False):
    q = rng.standard_normal((L, Hq, D)) / math.sqrt(D)
    k = rng.standard_normal((L, Hkv, D)) / math.sqrt(D)
    v = rng.standard_normal((L, Hkv, D)) / math.sqrt(D)
    iq = rng.standard_normal((L, Hi, di))
    ik = rng.standard_normal((L, di))
    iw = rng.random((L, Hi))
    gate = rng.standard_normal((L, Hq) if headwise else (L, Hq, D))
    return dict(q=q, k=k, v=v, iq=iq, ik=ik, iw=iw, gate=gate,
                cu_seqlens=np.array([0, L], dtype=np.int32))


def torch_sdpa_gated(q, k, v, gate, scale):
    """Library cross-check: torch's fp64 CPU SDPA (causal, GQA) times sigmoid(gate)."""
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                                         scale=scale, enable_gqa=True)
    o = o[0].permute(1, 0, 2).numpy()
    g = torch.sigmoid(torch.from_numpy(gate)).numpy()
    if g.ndim == 2:
        g = g[:, :, None]
    return g * o


@pytest.mark.parametrize("headwise", [False, True])
def test_dense_equivalence_when_budget_covers_context(headwise):
    L, Hq, Hkv, D = 37, 6, 2, 16
    cfg = Cfg(num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=4, budget=40,
              idx_heads=3, idx_dim=8)
    inp = _rand_seq(np.random.default_rng(7), L, Hq, Hkv, D, 3, 8, headwise)
    res = O.qsa_prefill(cfg, inp)
    got = np.stack([res["queries"][t].out for t in range(L)])
    lse = np.stack([res["queries"][t].lse for t in range(L)])
    dense, dlse = O.dense_gated_gqa(inp["q"], inp["k"], inp["v"], inp["gate"], D ** -0.5)
    np.testing.assert_allclose(got, dense, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, dlse, rtol=0, atol=1e-12)
    lib = torch_sdpa_gated(inp["q"], inp["k"], inp["v"], inp["gate"], D ** -0.5)
    np.testing.assert_allclose(dense, lib, rtol=0, atol=1e-12)


def test_dense_equivalence_at_the_width_bound():
    # below n = budget + B - 1 nothing can be pruned (ramgpt page): equal to dense
    B, budget = 4, 12
    L = budget + B - 1
    cfg = Cfg(num_q_heads=4, num_kv_heads=1, head_dim=8, block_size=B, budget=budget,
              idx_heads=2, idx_dim=8)
    inp = _rand_seq(np.random.default_rng(9), L, 4, 1, 8, 2, 8)
    res = O.qsa_prefill(cfg, inp)
    got = np.stack([res["queries"][t].out for t in range(L)])
    dense, _ = O.dense_gated_gqa(inp["q"], inp["k"], inp["v"], inp["gate"], 8 ** -0.5)
    np.testing.assert_allclose(got, dense, rtol=0, atol=1e-13)
    # one more token and a block can be dropped: the visible set shrinks
    inp2 = _rand_seq(np.random.default_rng(10), L + 2, 4, 1, 8, 2, 8)
    r = O.qsa_prefill(cfg, inp2, queries=[L + 1])["queries"][L + 1]
    assert r.tokens < L + 2


def test_sparse_attention_matches_masked_sdpa():
    # the attention over a selection equals library SDPA with the selection as mask
    L, Hq, Hkv, D, B = 50, 4, 2, 8, 4
    cfg = Cfg(num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=B, budget=12,
              idx_heads=2, idx_dim=8)
    inp = _rand_seq(np.random.default_rng(12), L, Hq, Hkv, D, 2, 8)
    res = O.qsa_prefill(cfg, inp)
    mask = np.zeros((L, L), dtype=bool)
    for t in range(L):
        r = res["queries"][t]
        mask[t, O.visible_positions(t + 1, B, r.selected)] = True
    qt = torch.from_numpy(inp["q"]).permute(1, 0, 2)[None]
    kt = torch.from_numpy(inp["k"]).permute(1, 0, 2)[None]
    vt = torch.from_numpy(inp["v"]).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=D ** -0.5, enable_gqa=True)
    lib = torch.sigmoid(torch.from_numpy(inp["gate"])).numpy() * o[0].permute(1, 0, 2).numpy()
    got = np.stack([res["queries"][t].out for t in range(L)])
    np.testing.assert_allclose(got, lib, rtol=0, atol=1e-12)


def test_single_block_closed_form():
    # k = 1; K = 0 makes the softmax uniform, so out = sigmoid(g) * mean(V over S(t)).
    # V[s] = s identifies which tokens were attended.
    B, L, D = 4, 23, 4
    cfg = Cfg(num_q_heads=2, num_kv_heads=1, head_dim=D, block_size=B, budget=B,
              idx_heads=1, idx_dim=2)
    q = np.random.default_rng(1).standard_normal((L, 2, D))
    k = np.zeros((L, 1, D))
    v = np.repeat(np.arange(L, dtype=np.float64)[:, None, None], D, axis=2)
    ik = np.zeros((L, 2)); ik[8:12, 0] = 3.0      # block 2 dominates
    iq = np.zeros((L, 1, 2)); iq[:, 0, 0] = 1.0
    gate = np.zeros((L, 2, D))                    # sigmoid(0) = 1/2
    inp = dict(q=q, k=k, v=v, iq=iq, ik=ik, iw=np.ones((L, 1)), gate=gate,
               cu_seqlens=np.array([0, L], np.int32))
    t = L - 1                                     # n = 23: blocks 0..4 complete, tail {20, 21, 22}
    r = O.qsa_prefill(cfg, inp, queries=[t])["queries"][t]
    assert list(r.selected) == [2]
    expect = 0.5 * np.mean([8, 9, 10, 11, 20, 21, 22])
    np.testing.assert_allclose(r.out, expect, rtol=0, atol=1e-14)
    # lse of all-zero logits over 7 tokens is log(7)
    np.testing.assert_allclose(r.lse, math.log(7.0), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- decode
def test_decode_equals_prefill_at_the_same_positions():
    # R11: a decode step with n_q new tokens at kv_len is the prefill of those
    # positions over the same cache rows
    w = WORKLOADS["mtp_verify_bf16_b4_kv262144"].with_(
        batch=2, kv_len=300, n_q=2, block_size=16, budget=64, num_q_heads=4,
        num_kv_heads=2, head_dim=16, idx_heads=2, idx_dim=8)
    inp = make_decode_inputs(w, kv_lens=np.array([300, 257], np.int32))
    dec = O.qsa_decode(w, inp)
    for b in range(2):
        L = int(inp["kv_len"][b])
        pre = dict(q=np.zeros((L, 4, 16)), k=inp["k_cache"][b, :L], v=inp["v_cache"][b, :L],
                   iq=np.zeros((L, 2, 8)), ik=inp["ik_cache"][b, :L], iw=np.zeros((L, 2)),
                   gate=np.zeros((L, 4, 16)), cu_seqlens=np.array([0, L], np.int32))
        for i in range(2):
            t = L - 2 + i
            pre["q"][t] = inp["q"][b, i]; pre["iq"][t] = inp["iq"][b, i]
            pre["iw"][t] = inp["iw"][b, i]; pre["gate"][t] = inp["gate"][b, i]
            pr = O.qsa_prefill(w, pre, queries=[t])["queries"][t]
            dr = dec["queries"][(b, i)]
            assert pr.n == dr.n == t + 1
            assert list(pr.selected) == list(dr.selected)
            np.testing.assert_array_equal(pr.out, dr.out)


# ---------------------------------------------------------------- metrics
def test_jaccard_and_near_tie():
    assert O.jaccard([1, 2, 3], [2, 3, 4]) == 0.5
    assert O.jaccard([], []) == 1.0
    s = np.array([5.0, 4.0, 3.0, 3.0 - 1e-7, 1.0])
    assert O.near_tie_excused(s, [0, 1, 2], [0, 1, 3], k=3)
    assert not O.near_tie_excused(s, [0, 1, 2], [0, 1, 4], k=3)
    assert not O.near_tie_excused(s, [0, 1, 2], [0, 1], k=3)


def test_workload_recipe_shapes():
    # the ragged prefill lengths are the seed's first draw
    from block_sparse_attention_17_b200.workloads import resolve_seqlens
    lens, _ = resolve_seqlens(WORKLOADS["ragged_prefill_bf16_4seq"])
    assert lens == (26045, 31369, 29854, 20758)
    assert all(L % 128 for L in lens)
    w = WORKLOADS["prefill_f32_t1024"].with_(seqlens=(100, 0, 37))
    inp = make_prefill_inputs(w)
    assert inp["q"].shape == (137, 4, 64) and inp["cu_seqlens"].tolist() == [0, 100, 100, 137]


# ---------------------------------------------------------------- indexer rotary embedding (R12)
COS1, SIN1 = 0.5403023058681398, 0.8414709848078965     # cos(1), sin(1)


def pin_rope_closed_form(rotate=None, inv_freq=None):
    rotate = rotate or O.rope_rotate
    inv_freq = inv_freq or O.rope_inv_freq
    # frequencies: theta ** (-2 f / r); 10000 ** (-1/2) = 0.01, 10000 ** 0 = 1
    np.testing.assert_array_equal(inv_freq(4, 10000.0), np.float32([1.0, 0.01]))
    np.testing.assert_array_equal(inv_freq(8, 256.0), np.float32([1.0, 0.25, 0.0625, 0.015625]))
    # rope_dim 2: one pair rotated by pos radians; (1, 0) goes to (cos, sin)
    np.testing.assert_allclose(rotate([1.0, 0.0], 1, 2, 10000.0), [COS1, SIN1], rtol=0, atol=1e-15)
    np.testing.assert_allclose(rotate([0.0, 1.0], 1, 2, 10000.0), [-SIN1, COS1], rtol=0, atol=1e-15)
    # position 0 is the identity
    x = np.array([0.3, -1.25, 2.0, 0.5, 7.0, -3.0])
    np.testing.assert_array_equal(rotate(x, 0, 4, 10000.0), x)
    # rope_dim 4 of 6 dims at position 100: frequency 1 turns by fp32(100 * fp32(0.01)) = 1 rad;
    # the pair of dim 1 is dim 3 (half split), and dims 4, 5 are untouched
    e1 = np.array([0.0, 1.0, 0.0, 0.0, 7.0, -3.0])
    np.testing.assert_allclose(rotate(e1, 100, 4, 10000.0), [0.0, COS1, 0.0, SIN1, 7.0, -3.0],
                               rtol=0, atol=1e-15)
    # frequency 0 turns by 100 rad: e0 -> (cos 100, 0, sin 100, 0)
    e0 = np.array([1.0, 0.0, 0.0, 0.0])
    np.testing.assert_allclose(rotate(e0, 100, 4, 10000.0),
                               [0.8623188722876839, 0.0, -0.5063656411097588, 0.0], rtol=0, atol=1e-15)


def test_rope_closed_form():
    pin_rope_closed_form()


def pin_rope_complex_and_norm(rotate=None):
    """Against complex multiplication z_f * exp(i a_f) with z_f = x_f + i x_{f+h},
    and the norm of every pair is kept."""
    rotate = rotate or O.rope_rotate
    rng = np.random.default_rng(12)
    for r, di, pos, theta in [(8, 8, 37, 10000.0), (16, 32, 1000, 500000.0), (4, 8, 262143, 10000.0)]:
        x = rng.standard_normal(di)
        y = rotate(x, pos, r, theta)
        h = r // 2
        a = O.rope_angles(pos, r, theta)
        z = (x[:h] + 1j * x[h:r]) * np.exp(1j * a)
        np.testing.assert_allclose(y[:h], z.real, rtol=0, atol=1e-13)
        np.testing.assert_allclose(y[h:r], z.imag, rtol=0, atol=1e-13)
        np.testing.assert_array_equal(y[r:], x[r:])
        np.testing.assert_allclose(y[:h] ** 2 + y[h:r] ** 2, x[:h] ** 2 + x[h:r] ** 2, rtol=1e-13)


def test_rope_complex_and_norm():
    pin_rope_complex_and_norm()


def pin_rope_relative(rotate=None):
    """rot(q, m) . rot(k, n) depends on m - n only (same frequencies and turning
    direction on both sides); fp32 angles keep it to rounding at small positions."""
    rotate = rotate or O.rope_rotate
    rng = np.random.default_rng(13)
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    for m, n, d in [(9, 3, 5), (40, 40, 17), (3, 30, 64)]:
        a = rotate(q, m, 16, 10000.0) @ rotate(k, n, 16, 10000.0)
        b = rotate(q, m + d, 16, 10000.0) @ rotate(k, n + d, 16, 10000.0)
        c = rotate(q, m - n, 16, 10000.0) @ k if m >= n else q @ rotate(k, n - m, 16, 10000.0)
        assert abs(a - b) < 2e-5 * (np.abs(q) @ np.abs(k)), (m, n, d)
        assert abs(a - c) < 2e-5 * (np.abs(q) @ np.abs(k)), (m, n)


def test_rope_relative_position():
    pin_rope_relative()


def pin_rope_positions_in_scores(query=None):
    """With R12 the score of block j is the unrotated score of the query turned by
    its offset (n - 1) - j * B from the block's first token: the query sits at
    its own position and every pooled key at its block's first position."""
    query = query or O.qsa_query
    rng = np.random.default_rng(14)
    B, di, Hi, r = 8, 16, 3, 12
    cfg = Cfg(block_size=B, budget=4 * B, idx_dim=di, idx_heads=Hi, rope_dim=r, rope_theta=10000.0)
    plain = Cfg(block_size=B, budget=4 * B, idx_dim=di, idx_heads=Hi)
    n = 83
    ik = rng.standard_normal((n, di))
    iq, iw = rng.standard_normal((Hi, di)), rng.random(Hi)
    res = query(cfg, n, O.pooled_keys(cfg, ik), iq, iw, attend=False)
    raw = O.pool_blocks(ik, B)
    c = di ** -0.5
    for j in range(n // B):
        qj = np.stack([O.rope_rotate(iq[h], (n - 1) - j * B, r, 10000.0) for h in range(Hi)])
        expect = c * (np.maximum(qj @ raw[j], 0.0) @ iw)
        assert abs(res.scores[j] - expect) <= 1e-5 * (1.0 + abs(expect)), j
    # rope_dim 0 is the plain score
    res0 = query(plain, n, O.pooled_keys(plain, ik), iq, iw, attend=False)
    np.testing.assert_allclose(res0.scores, c * (np.maximum(raw[:n // B] @ iq.T, 0.0) @ iw), rtol=1e-14)


def test_rope_positions_in_scores():
    pin_rope_positions_in_scores()


# ---------------------------------------------------------------- mutation battery
def _mut_pool_divide_by_n(ik_rows, B):
    ik_rows = np.asarray(ik_rows, np.float64)
    nblk = ik_rows.shape[0] // B
    return np.stack([ik_rows[j * B:(j + 1) * B].sum(0) / (B + 1) for j in range(nblk)]) \
        if nblk else np.zeros((0, ik_rows.shape[1]))


def _mut_pool_includes_partial(ik_rows, B):
    ik_rows = np.asarray(ik_rows, np.float64)
    nblk = -(-ik_rows.shape[0] // B)
    return np.stack([ik_rows[j * B:(j + 1) * B].mean(0) for j in range(nblk)])


def _mut_score_no_relu(iq, w, kbar, c):
    return c * ((np.asarray(kbar) @ np.asarray(iq).T) @ np.asarray(w))


def _mut_score_weights_outside_relu(iq, w, kbar, c):
    return c * np.maximum((np.asarray(kbar) @ np.asarray(iq).T) @ np.asarray(w), 0.0)


def _mut_score_transposed(iq, w, kbar, c):
    d = np.asarray(kbar) @ np.asarray(iq).T
    return c * (np.maximum(d, 0.0) @ np.asarray(w)[::-1])


def _mut_topk_high_index_wins(scores, k):
    nc = len(scores)
    keyed = sorted(range(nc), key=lambda j: (-(scores[j] + 0.0), -j))
    return np.array(sorted(keyed[:min(k, nc)]), dtype=np.int64)


def _mut_topk_unstable_negzero(scores, k):
    nc = len(scores)
    keyed = sorted(range(nc), key=lambda j: (-np.copysign(1.0, scores[j]) * (scores[j] == 0) - scores[j], j))
    return np.array(sorted(keyed[:min(k, nc)]), dtype=np.int64)


def _mut_rope_clockwise(x, pos, r, theta):
    return O.rope_rotate(x, -pos, r, theta)


def _mut_rope_interleaved(x, pos, r, theta):
    x = np.array(x, dtype=np.float64)
    a = O.rope_angles(pos, r, theta)
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[0:r:2].copy(), x[1:r:2].copy()
    x[0:r:2], x[1:r:2] = x1 * c - x2 * s, x2 * c + x1 * s
    return x


def _mut_rope_freq(r, theta):
    return np.array([np.float32(float(theta) ** (-1.0 * f / r)) for f in range(r // 2)], np.float32)


_rope_calls = [0]


def _mut_rope_sign_by_parity(x, pos, r, theta):
    # the second operand of every dot turned the other way
    _rope_calls[0] += 1
    return O.rope_rotate(x, pos if _rope_calls[0] % 2 else -pos, r, theta)


@pytest.mark.parametrize("name,target,mut,pin", [
    ("pool/B+1", "pool_blocks", _mut_pool_divide_by_n, pin_pool_closed_form),
    ("pool/partial", "pool_blocks", _mut_pool_includes_partial, pin_pool_closed_form),
    ("score/no-relu", "index_scores", _mut_score_no_relu, pin_scores_hand_example),
    ("score/weights-outside", "index_scores", _mut_score_weights_outside_relu, pin_scores_hand_example),
    ("score/weights-reversed", "index_scores", _mut_score_transposed, pin_scores_hand_example),
    ("topk/tie-high", "select_topk", _mut_topk_high_index_wins, pin_topk_brute_force),
    ("topk/negzero", "select_topk", _mut_topk_unstable_negzero, pin_topk_brute_force),
    ("rope/clockwise", "rope_rotate", _mut_rope_clockwise, pin_rope_closed_form),
    ("rope/interleaved", "rope_rotate", _mut_rope_interleaved, pin_rope_closed_form),
    ("rope/interleaved-c", "rope_rotate", _mut_rope_interleaved, pin_rope_complex_and_norm),
    ("rope/freq-f-over-r", "rope_inv_freq", _mut_rope_freq,
     lambda m: pin_rope_closed_form(inv_freq=m)),
    ("rope/k-other-way", "rope_rotate", _mut_rope_sign_by_parity, pin_rope_relative),
])
def test_mutation_turns_a_pin_red(name, target, mut, pin):
    with pytest.raises(AssertionError):
        pin(mut)


def test_mutations_of_attention_turn_dense_pin_red(monkeypatch):
    # wrong GQA map (h % Hkv instead of h // G) must break dense equality
    orig = O.gated_attention

    def bad(q_t, K, V, positions, gate_t, scale):
        Hq, Hkv = q_t.shape[0], K.shape[1]
        Kp = K[:, [h % Hkv for h in range(Hkv)], :][:, ::-1, :]
        return orig(q_t, Kp, V, positions, gate_t, scale)

    monkeypatch.setattr(O, "gated_attention", bad)
    with pytest.raises(AssertionError):
        test_dense_equivalence_when_budget_covers_context(False)
    monkeypatch.setattr(O, "gated_attention", orig)

    # dropping the tail must break the count invariant
    orig_vis = O.visible_positions
    monkeypatch.setattr(O, "visible_positions",
                        lambda n, B, sel: orig_vis((n // B) * B, B, sel))
    with pytest.raises(AssertionError):
        test_single_block_closed_form()


def test_mutations_of_rope_positions_turn_score_pin_red(monkeypatch):
    # the query rotated at n (the count) instead of its position n - 1
    def query_at_n(cfg, n, kbar, iq_t, iw_t, **kw):
        r, th = O.rope_params(cfg)
        return O.qsa_query(cfg, n, kbar, O.rope_rotate(iq_t, 1, r, th), iw_t, **kw)
    with pytest.raises(AssertionError):
        pin_rope_positions_in_scores(query_at_n)

    # pooled keys rotated at the block's last token instead of its first
    orig_rot = O.rope_rotate

    def pooled_at_last(cfg, ik_rows):
        B = cfg.block_size
        kbar = O.pool_blocks(ik_rows, B)
        r, th = O.rope_params(cfg)
        for j in range(kbar.shape[0]):
            kbar[j] = orig_rot(kbar[j], j * B + B - 1, r, th) if r else kbar[j]
        return kbar
    monkeypatch.setattr(O, "pooled_keys", pooled_at_last)
    with pytest.raises(AssertionError):
        pin_rope_positions_in_scores()
