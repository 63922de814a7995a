"""Paged KV cache for decode (qsa_decode_paged, qsa_pool_build_paged).

The page is the QSA block: block j of sequence b lives in page
block_table[b, j] of a pool shared by all sequences. The math is qsa_decode's,
so the paged call must give bit-identical results to qsa_decode on the same
rows laid out contiguously, and the same parity with the fp64 oracle. Pages
that no block maps to hold NaN, so a wrong gather shows up in the output.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200.workloads import WORKLOADS, make_decode_inputs
from oracle import qsa_oracle as O
from tests import qsa_testlib as TL

pytestmark = pytest.mark.gpu


def _case(name, batch, kv_lens, cap):
    w = WORKLOADS[name].with_(batch=batch, cap=cap, kv_len=max(kv_lens))
    inp = make_decode_inputs(w, kv_lens=np.array(kv_lens, np.int32))
    return w, inp


def _paged(w, d, n_spare=5, seed=11):
    """Scatter the contiguous caches into a page pool under a random block table."""
    batch, cap = d["k_cache"].shape[0], d["k_cache"].shape[1]
    B = w.block_size
    max_blocks = cap // B
    num_pages = batch * max_blocks + n_spare
    perm = np.random.default_rng(seed).permutation(num_pages)[: batch * max_blocks]
    table = torch.from_numpy(perm.reshape(batch, max_blocks).astype(np.int32)).cuda()
    idx = table.reshape(-1).long()

    def scatter(cache):
        rows = cache.reshape(batch * max_blocks, B, *cache.shape[2:])
        pool = torch.full((num_pages, B, *cache.shape[2:]), float("nan"), dtype=cache.dtype,
                          device=cache.device)
        pool[idx] = rows
        return pool

    return table, scatter(d["k_cache"]), scatter(d["v_cache"]), scatter(d["ik_cache"])


def _contiguous(w, d):
    cfg = qsa.QSAConfig.from_workload(w)
    kv = d["kv_len"]
    pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = qsa.decode(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"], d["ik_cache"], d["iw"],
                   d["gate"], pooled, kv, want_lse=True, want_sel=True, dev_err=err)
    r["pooled"], r["err"] = pooled, int(err.item())
    return r


def _run_paged(w, d, table, kp, vp, ikp):
    cfg = qsa.QSAConfig.from_workload(w)
    kv = d["kv_len"]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pooled = qsa.pool_build_paged(cfg, ikp, (kv - w.n_q).to(torch.int32), table, dev_err=err)
    pooled_before = pooled.clone()
    r = qsa.decode_paged(cfg, d["q"], kp, vp, d["iq"], ikp, d["iw"], d["gate"], pooled, kv, table,
                         want_lse=True, want_sel=True, dev_err=err)
    torch.cuda.synchronize()
    r["pooled_before"], r["pooled"], r["err"] = pooled_before, pooled, int(err.item())
    return r


@pytest.mark.parametrize("name,batch,kv_lens,cap", [
    ("decode_bf16_b32_kv32768", 6, (4097, 64, 2112, 2113, 130, 1), 4160),
    ("mtp_verify_bf16_b4_kv262144", 3, (9000, 4225, 2), 9088),
])
def test_paged_decode_is_bit_identical_to_contiguous(name, batch, kv_lens, cap):
    w, inp = _case(name, batch, kv_lens, cap)
    d = TL.upload(inp, w)
    ref = _contiguous(w, d)
    table, kp, vp, ikp = _paged(w, d)
    got = _run_paged(w, d, table, kp, vp, ikp)
    assert ref["err"] == 0 and got["err"] == 0
    cfg = qsa.QSAConfig.from_workload(w)
    pooled_ref = qsa.pool_build(cfg, d["ik_cache"], (d["kv_len"] - w.n_q).to(torch.int32))
    assert torch.equal(got["pooled_before"], pooled_ref)
    assert torch.equal(got["pooled"], ref["pooled"])
    for key in ("out", "lse", "sel", "nsel"):
        assert torch.equal(got[key], ref[key]), key
    assert torch.isfinite(got["out"].float()).all()
    # and the oracle agrees with the paged call directly
    orc = O.qsa_decode(w, inp)["queries"]
    rep = TL.check_queries(orc, got, lambda bi: bi, w)
    assert len(rep["excused_near_ties"]) <= 1, rep


def test_paged_decode_reports_a_bad_page_id():
    w, inp = _case("decode_bf16_b32_kv32768", 2, (300, 200), 320)
    d = TL.upload(inp, w)
    table, kp, vp, ikp = _paged(w, d)
    cfg = qsa.QSAConfig.from_workload(w)
    kv = d["kv_len"]
    pooled = qsa.pool_build_paged(cfg, ikp, (kv - w.n_q).to(torch.int32), table)
    bad = table.clone()
    bad[1, 0] = kp.shape[0] + 3          # a used block of sequence 1 names no page of the pool
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    r = qsa.decode_paged(cfg, d["q"], kp, vp, d["iq"], ikp, d["iw"], d["gate"], pooled, kv, bad,
                         dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 3
    # sequence 0 is untouched by the bad entry
    ref = _contiguous(w, d)
    assert torch.equal(r["out"][0], ref["out"][0])
