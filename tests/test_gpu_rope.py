"""The indexer rotary embedding on the GPU: the indexer query turned at its
own position and the pooled key of block j at j * B, fused into the kernels
that pool and score (prefill pooling and selection, the one-launch decode, the
selection kernel of the two-kernel decode, the cache rebuild, paged caches).
Every query is compared with the fp64 oracle, the scores by value, and the
pooled rows both with the oracle and bit for bit between the paths that write
them. Positions up to 262,143 exercise the fp32 angles far from zero."""
import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200.workloads import (WORKLOADS, make_decode_inputs,
                                                      make_prefill_inputs)
from oracle import qsa_oracle as O
from tests import qsa_testlib as TL
from tests.test_gpu_parity import decode_parity, prefill_parity
from tests.test_gpu_paths import _decode_launches, _two_kernel_parity

pytestmark = pytest.mark.gpu


def _prefill(name, seqlens, **rope):
    w = WORKLOADS[name].with_(ragged_range=None, seqlens=seqlens, **rope)
    return w, make_prefill_inputs(w)


def _decode(name, kv_lens=None, **kw):
    w = WORKLOADS[name]
    if kv_lens is None:
        w = w.with_(**kw)
        return w, make_decode_inputs(w)
    w = w.with_(kv_len=max(kv_lens), **kw)
    return w, make_decode_inputs(w, kv_lens=np.array(kv_lens, np.int32))


@pytest.mark.parametrize("name,seqlens,rope_dim,theta", [
    ("prefill_f32_t1024", (1024,), 32, 1e6),             # CUDA-core prefill, every dim turned
    ("prefill_bf16_t8192", (2600,), 32, 1e4),             # tensor-core prefill, half the dims
])
def test_prefill_rope_all_queries(name, seqlens, rope_dim, theta):
    w, inp = _prefill(name, seqlens, rope_dim=rope_dim, rope_theta=theta)
    rep = prefill_parity(w, inp, None)
    print(f"{name} rope {rope_dim}: excused near-ties {rep['excused_near_ties']}")
    assert len(rep["excused_near_ties"]) <= 3, rep


def test_prefill_rope_ragged_sampled():
    # ragged sequences with tails, the 32 / 4-head tensor-core geometry, B = 128
    lens = (3000, 257, 4100, 1)
    w, inp = _prefill("ragged_prefill_bf16_4seq", lens, rope_dim=64, rope_theta=5e5)
    cu = inp["cu_seqlens"]
    rng = np.random.default_rng(5)
    qs = []
    for b, L in enumerate(lens):
        pos = range(L) if L <= 200 else TL.sample_positions(L, w.block_size, 80, rng)
        qs += [int(cu[b]) + p for p in pos]
    rep = prefill_parity(w, inp, qs)
    assert len(rep["excused_near_ties"]) <= 2, rep


def test_prefill_rope_scores_value_gate():
    w, inp = _prefill("prefill_bf16_t8192", (2600,), rope_dim=64, rope_theta=1e4)
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


@pytest.mark.parametrize("n_q", [1, 2, 4])
def test_decode_rope_one_launch_and_two_kernel(n_q):
    w, inp = _decode("decode_bf16_b32_kv32768", kv_lens=(3000, 500, 64, n_q), n_q=n_q, batch=4,
                     cap=3008, rope_dim=64, rope_theta=1e4)
    d = TL.upload(inp, w)
    assert _decode_launches(w, d) == 1
    rep = decode_parity(w, inp, d=d)
    assert len(rep["excused_near_ties"]) <= 1, rep
    rep = _two_kernel_parity(w, inp, d)
    assert len(rep["excused_near_ties"]) <= 1, rep


def test_decode_rope_fp32_cuda_core_path():
    w, inp = _decode("decode_bf16_b32_kv32768", kv_lens=(2049, 64, 1000, 1), dtype="f32",
                     batch=4, cap=2112, rope_dim=32, rope_theta=1e4)
    rep = decode_parity(w, inp)
    assert len(rep["excused_near_ties"]) <= 1, rep


@pytest.mark.parametrize("name", ["decode_bf16_b32_kv32768", "mtp_verify_bf16_b4_kv262144"])
def test_decode_rope_full_size(name):
    # positions up to 262,143: fp32 angles up to 2.6e5 rad
    w, inp = _decode(name, rope_dim=64, rope_theta=1e6)
    rep = decode_parity(w, inp)
    print(f"{name} rope: excused near-ties {rep['excused_near_ties']}")
    assert len(rep["excused_near_ties"]) <= 2, rep


def test_decode_rope_pooled_rows_agree_across_paths():
    # the step's incremental pooling (one launch), the rebuild and the prefill's
    # pooled_out write the same bits for the turned means
    w, inp = _decode("mtp_verify_bf16_b4_kv262144", kv_lens=(9000, 4225, 2), batch=3, cap=9088,
                     rope_dim=64, rope_theta=1e6)
    d = TL.upload(inp, w)
    cfg = qsa.QSAConfig.from_workload(w)
    kv = d["kv_len"]
    pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
    qsa.decode(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"], d["ik_cache"], d["iw"], d["gate"],
               pooled, kv)
    rebuilt = qsa.pool_build(cfg, d["ik_cache"], kv)
    torch.cuda.synchronize()
    assert torch.equal(pooled, rebuilt)
    orc = O.qsa_decode(w, inp, attend=False)["pooled"]
    got = pooled.cpu().numpy()
    for b, pb in orc.items():
        np.testing.assert_allclose(got[b, :len(pb)], pb, rtol=TL.TOL_POOLED_REL, atol=1e-7)


def test_paged_decode_rope_is_bit_identical_to_contiguous():
    from tests.test_gpu_paged import _contiguous, _paged, _run_paged
    w, inp = _decode("decode_bf16_b32_kv32768", kv_lens=(4097, 64, 2112, 2113, 130, 1), batch=6,
                     cap=4160, rope_dim=32, rope_theta=1e4)
    d = TL.upload(inp, w)
    ref = _contiguous(w, d)
    table, kp, vp, ikp = _paged(w, d)
    got = _run_paged(w, d, table, kp, vp, ikp)
    assert ref["err"] == 0 and got["err"] == 0
    assert torch.equal(got["pooled"], ref["pooled"])
    for key in ("out", "lse", "sel", "nsel"):
        assert torch.equal(got[key], ref[key]), key
    rep = TL.check_queries(O.qsa_decode(w, inp)["queries"], got, lambda bi: bi, w)
    assert len(rep["excused_near_ties"]) <= 1, rep
