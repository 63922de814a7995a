"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small cases compare every query; the full-size workloads compare sampled
queries, in the launch configuration bench.py times. Selections must be
identical except for near-ties (|s - s_k| <= 1e-5 * max|s| in the oracle's
scores), which are reported; outputs must be within 1e-4 (fp32 inputs) or
2e-2 (bf16 inputs) max abs error.
"""
import functools

import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200.workloads import (WORKLOADS, make_decode_inputs,
                                                      make_prefill_inputs, resolve_seqlens)
from oracle import qsa_oracle as O
from tests import qsa_testlib as TL

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=4)
def _prefill_case(name, seqlens=None):
    w = WORKLOADS[name]
    if seqlens is not None:
        w = w.with_(seqlens=tuple(seqlens), ragged_range=None)
    inp = make_prefill_inputs(w)
    return w, inp


@functools.lru_cache(maxsize=3)
def _decode_case(name, batch=None, kv_lens=None, cap=None):
    w = WORKLOADS[name]
    if batch is not None:
        w = w.with_(batch=batch, cap=cap or 0, kv_len=max(kv_lens))
    inp = make_decode_inputs(w, kv_lens=None if kv_lens is None else np.array(kv_lens, np.int32))
    return w, inp


def run_prefill(w, inp):
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    r = qsa.prefill(cfg, d["q"], d["k"], d["v"], d["iq"], d["ik"], d["iw"], d["gate"],
                    d["cu_seqlens"], inp["max_seqlen"], want_lse=True, want_sel=True,
                    want_pooled=True)
    torch.cuda.synchronize()
    assert int(r["error_word"].item()) == 0, "a prefill kernel gave up on a bounded wait"
    return r


def prefill_parity(w, inp, queries):
    gpu = run_prefill(w, inp)
    orc = O.qsa_prefill(w, inp, queries=queries)
    rep = TL.check_queries(orc["queries"], gpu, lambda t: t, w)
    # pooled keys of every complete block
    pooled = gpu["pooled"].cpu().numpy()
    for b, pb in enumerate(orc["pooled"]):
        if len(pb):
            np.testing.assert_allclose(pooled[b, :len(pb)], pb, rtol=TL.TOL_POOLED_REL, atol=1e-7)
    return rep


def test_prefill_f32_t1024_all_queries():
    w, inp = _prefill_case("prefill_f32_t1024")
    rep = prefill_parity(w, inp, None)
    assert rep["n"] == 1024
    assert len(rep["excused_near_ties"]) <= 2, rep


def test_prefill_bf16_reduced_all_queries():
    # the 8192-token workload's geometry at 2600 tokens: past the budget
    # (2048 + 64 - 1), with a ragged tail (2600 % 64 = 40)
    w, inp = _prefill_case("prefill_bf16_t8192", (2600,))
    rep = prefill_parity(w, inp, None)
    assert len(rep["excused_near_ties"]) <= 3, rep


def test_prefill_ragged_reduced_edge_lengths():
    # empty, 1-token, exactly-one-block and ragged sequences in one packed batch
    lens = (1000, 4500, 0, 3001, 129, 1, 128)
    w, inp = _prefill_case("ragged_prefill_bf16_4seq", lens)
    cu = inp["cu_seqlens"]
    rng = np.random.default_rng(0)
    qs = []
    for b, L in enumerate(lens):
        pos = range(L) if L <= 200 else TL.sample_positions(L, w.block_size, 80, rng)
        qs += [int(cu[b]) + p for p in pos]
    rep = prefill_parity(w, inp, qs)
    assert len(rep["excused_near_ties"]) <= 2, rep


# The tensor-core prefill gives each CTA 2 x 128 / G consecutive query tokens
# (32 at G = 8): the full-size tests take one random query from every such span
# (8192-token workload) or from every eighth span (ragged workload, 3376 spans),
# so every CTA row of the launch bench.py times is compared at full size.
CTA_SPAN = 32


@pytest.mark.parametrize("name,stride", [("prefill_bf16_t8192", 1),
                                         ("ragged_prefill_bf16_4seq", 8)])
def test_prefill_full_size_sampled(name, stride):
    w, inp = _prefill_case(name)
    cu = inp["cu_seqlens"]
    rng = np.random.default_rng(1)
    qs = set()
    for b in range(len(cu) - 1):
        L = int(cu[b + 1] - cu[b])
        qs.update(int(cu[b]) + p for p in TL.sample_positions(L, w.block_size, 24, rng))
        for s0 in range(0, L, CTA_SPAN * stride):
            qs.add(int(cu[b]) + s0 + int(rng.integers(0, min(CTA_SPAN, L - s0))))
    rep = prefill_parity(w, inp, sorted(qs))
    print(f"{name}: {rep['n']} queries, excused near-ties {rep['excused_near_ties']}, "
          f"max abs err {rep['max_abs_err']:.3g}")
    assert len(rep["excused_near_ties"]) <= 3, rep


def test_prefill_select_scores_value_gate():
    # scores are compared by value: a scale error is invisible to a selection
    # (llama.cpp PR #27739 page, the "value gate" of the QSA composition)
    w, inp = _prefill_case("prefill_bf16_t8192", (2600,))
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    r = qsa.select(cfg, d["iq"], d["ik"], d["iw"], d["cu_seqlens"], inp["max_seqlen"],
                   want_scores=True)
    sc = r["scores"].cpu().numpy()
    qs = [0, 63, 64, 1000, 2047, 2111, 2112, 2599]
    orc = O.qsa_prefill(w, inp, queries=qs, attend=False)["queries"]
    for t, q in orc.items():
        if q.nc:
            np.testing.assert_allclose(sc[t, :q.nc], q.scores, rtol=TL.TOL_SCORE_REL,
                                       atol=TL.TOL_SCORE_REL * np.abs(q.scores).max())
        assert np.all(np.isneginf(sc[t, q.nc:]))


def test_prefill_dense_equivalence_on_gpu():
    # budget >= context: nothing can be pruned and QSA equals dense causal
    # gated GQA (ramgpt page, "QSA Should First Be Implemented as Selection Semantics")
    w = WORKLOADS["prefill_f32_t1024"].with_(seqlens=(300, 77), budget=320)
    inp = make_prefill_inputs(w)
    gpu = run_prefill(w, inp)
    out = gpu["out"].cpu().numpy()
    cu = inp["cu_seqlens"]
    for b in range(2):
        s, e = int(cu[b]), int(cu[b + 1])
        dense, _ = O.dense_gated_gqa(inp["q"][s:e], inp["k"][s:e], inp["v"][s:e],
                                     inp["gate"][s:e], w.head_dim ** -0.5)
        assert np.max(np.abs(out[s:e] - dense)) <= TL.TOL_OUT["f32"]


def test_prefill_deterministic():
    w, inp = _prefill_case("prefill_bf16_t8192", (2600,))
    a = run_prefill(w, inp)
    b = run_prefill(w, inp)
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["sel"], b["sel"])


# ------------------------------------------------------------------- decode
def run_decode(w, inp, d=None):
    cfg = qsa.QSAConfig.from_workload(w)
    d = d or TL.upload(inp, w)
    kv = d["kv_len"]
    # the pooled cache holds every block completed before this step
    pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = qsa.decode(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"], d["ik_cache"], d["iw"],
                   d["gate"], pooled, kv, want_lse=True, want_sel=True, dev_err=err)
    torch.cuda.synchronize()
    r["pooled"] = pooled
    r["err"] = int(err.item())
    return r


def decode_parity(w, inp, pairs=None, d=None):
    gpu = run_decode(w, inp, d)
    assert gpu["err"] == 0
    orc = O.qsa_decode(w, inp, pairs=pairs)
    rep = TL.check_queries(orc["queries"], gpu, lambda bi: bi, w)
    pooled = gpu["pooled"].cpu().numpy()
    for b, pb in orc["pooled"].items():
        np.testing.assert_allclose(pooled[b, :len(pb)], pb, rtol=TL.TOL_POOLED_REL, atol=1e-7)
    return rep


def test_decode_reduced_mixed_lengths():
    # lengths below the budget (dense-equivalent), at block multiples, and ragged
    w, inp = _decode_case("decode_bf16_b32_kv32768", 6, (4097, 64, 2112, 2113, 130, 1), 4160)
    rep = decode_parity(w, inp)
    assert len(rep["excused_near_ties"]) <= 1, rep


def test_mtp_verify_reduced():
    w, inp = _decode_case("mtp_verify_bf16_b4_kv262144", 3, (9000, 4225, 2), 9088)
    rep = decode_parity(w, inp)
    assert len(rep["excused_near_ties"]) <= 1, rep


@pytest.mark.parametrize("name", ["decode_bf16_b32_kv32768", "mtp_verify_bf16_b4_kv262144"])
def test_decode_full_size(name):
    w, inp = _decode_case(name)
    rep = decode_parity(w, inp)
    print(f"{name}: {rep['n']} queries, excused near-ties {rep['excused_near_ties']}, "
          f"max abs err {rep['max_abs_err']:.3g}")
    assert len(rep["excused_near_ties"]) <= 1, rep


def test_decode_nan_poison_of_unselected_rows():
    # poison every K/V row the oracle did not select: a gather consumer never
    # reads them (llama.cpp PR #27739 page: NaN-poison probe of the consumer)
    w, inp = _decode_case("decode_bf16_b32_kv32768", 6, (4097, 64, 2112, 2113, 130, 1), 4160)
    orc = O.qsa_decode(w, inp, attend=False)["queries"]
    clean = run_decode(w, inp)
    pois = {k: v.copy() for k, v in inp.items() if isinstance(v, np.ndarray)}
    for (b, i), r in orc.items():
        keep = np.zeros(pois["k_cache"].shape[1], dtype=bool)
        keep[O.visible_positions(r.n, w.block_size, r.selected)] = True
        pois["k_cache"][b, ~keep] = np.nan
        pois["v_cache"][b, ~keep] = np.nan
    dirty = run_decode(w, {**inp, **pois})
    assert torch.isfinite(dirty["out"].float()).all()
    assert torch.equal(clean["out"], dirty["out"])


def test_decode_pooled_cache_rebuild_is_bit_identical():
    # incremental decode finalisation, rebuild and prefill pooling write the same bits
    w, inp = _decode_case("decode_bf16_b32_kv32768", 6, (4097, 64, 2112, 2113, 130, 1), 4160)
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    inc = run_decode(w, inp, d)["pooled"]
    full = qsa.pool_build(cfg, d["ik_cache"], d["kv_len"])
    torch.cuda.synchronize()
    assert torch.equal(inc, full)
    # prefill of the same rows (sequence 0) pools identically
    L = int(inp["kv_len"][0])
    ik = d["ik_cache"][0, :L].contiguous()
    z = lambda *s: torch.zeros(*s, dtype=TL.tdtype(w), device="cuda")
    cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
    r = qsa.select(cfg, z(L, w.idx_heads, w.idx_dim), ik,
                   torch.zeros(L, w.idx_heads, device="cuda"), cu, L, want_pooled=True)
    nb = L // w.block_size
    assert torch.equal(r["pooled"][0, :nb], full[0, :nb])


def test_decode_out_of_range_kv_len_sets_device_error():
    w, inp = _decode_case("decode_bf16_b32_kv32768", 6, (4097, 64, 2112, 2113, 130, 1), 4160)
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    kv = d["kv_len"].clone()
    kv[2] = 5000   # > cap
    pooled = qsa.pool_build(cfg, d["ik_cache"], (d["kv_len"] - 1).to(torch.int32))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = qsa.decode(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"], d["ik_cache"], d["iw"],
                   d["gate"], pooled, kv, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) != 0
    assert torch.all(r["out"][2] == 0)
    assert torch.isfinite(r["out"].float()).all()


def test_empty_batch_is_a_no_op():
    w = WORKLOADS["prefill_bf16_t8192"]
    cfg = qsa.QSAConfig.from_workload(w)
    e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = qsa.prefill(cfg, e(0, 16, 128), e(0, 2, 128), e(0, 2, 128), e(0, 4, 64), e(0, 64),
                    torch.empty(0, 4, device="cuda"), e(0, 16, 128), cu, 0)
    assert r["out"].shape == (0, 16, 128)
