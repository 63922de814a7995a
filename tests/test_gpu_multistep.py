"""Several decode steps in a row after a prefill: the pooled-key side cache.

A decode step pools only the blocks its new tokens complete, so a wrong row
(the indexer rows of the wrong cache position, or a pooled row written for the
wrong block) shows up only after steps that complete blocks, and the port on
the llama.cpp PR #27739 page recomputes the pooled keys over the whole cache at
every step, which would hide such a fault (its mutation battery plants "the
indexer key at cache row 0 instead of row past_len"). Here a prefill of L
tokens gives the pooled rows, then decode steps append tokens one step at a
time (n_q = 1 with B = 64, n_q = 2 with B = 128) until at least two blocks
are completed; every step is compared with the oracle, and the pooled cache at
the end is compared bit for bit with a rebuild from the indexer-key cache and
with a prefill of all L + n tokens.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200.workloads import WORKLOADS, make_decode_inputs
from oracle import qsa_oracle as O
from tests import qsa_testlib as TL

pytestmark = pytest.mark.gpu


def _prefill_pooled(cfg, w, d, b_lens, rng):
    """qsa_prefill over the first b_lens[b] cache rows of every sequence; the
    queries, indexer queries, weights and gates are fresh draws (only the pooled
    keys are used). Returns pooled_out [batch, ceil(max/B), di]."""
    batch = len(b_lens)
    dt = TL.tdtype(w)
    ks, vs, iks = [], [], []
    for b, L in enumerate(b_lens):
        ks.append(d["k_cache"][b, :L])
        vs.append(d["v_cache"][b, :L])
        iks.append(d["ik_cache"][b, :L])
    k = torch.cat(ks).contiguous()
    v = torch.cat(vs).contiguous()
    ik = torch.cat(iks).contiguous()
    T = k.shape[0]
    g = lambda *s: torch.from_numpy(rng.standard_normal(s).astype(np.float32) * 0.1).to("cuda", dt)
    q, iq, gate = g(T, w.num_q_heads, w.head_dim), g(T, w.idx_heads, w.idx_dim), \
        g(T, w.num_q_heads, w.head_dim)
    iw = torch.from_numpy(rng.random((T, w.idx_heads)).astype(np.float32)).to("cuda")
    cu = torch.tensor(np.concatenate([[0], np.cumsum(b_lens)]), dtype=torch.int32, device="cuda")
    r = qsa.prefill(cfg, q, k, v, iq, ik, iw, gate, cu, max(b_lens), want_pooled=True)
    torch.cuda.synchronize()
    assert int(r["error_word"].item()) == 0
    return r["pooled"]


@pytest.mark.parametrize("name,L,steps,rope_dim", [
    # n_q = 1, B = 64: from 1277 and 700 tokens: blocks 19 and 20, blocks 10 and 11
    ("decode_bf16_b32_kv32768", (1277, 700), 70, 0),
    # n_q = 2, B = 128: from 2301 and 1020 tokens, 2 tokens a step: blocks 17
    # and 18, blocks 7 and 8
    ("mtp_verify_bf16_b4_kv262144", (2301, 1020), 70, 0),
    # with the indexer rotary embedding (pooled rows turned at their blocks'
    # positions by the prefill, the steps and the rebuild alike)
    ("decode_bf16_b32_kv32768", (1277, 700), 70, 64),
])
def test_prefill_then_decode_steps_keep_the_side_cache(name, L, steps, rope_dim):
    w0 = WORKLOADS[name].with_(rope_dim=rope_dim, rope_theta=1e4)
    n_q = w0.n_q
    cap = ((max(L) + steps * n_q) // w0.block_size + 1) * w0.block_size
    w = w0.with_(batch=len(L), kv_len=cap, cap=cap)
    inp = make_decode_inputs(w, kv_lens=np.full(len(L), cap, np.int32))
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    rng = np.random.default_rng(7)
    B = w.block_size
    nblk = cap // B
    pf = _prefill_pooled(cfg, w, d, L, rng)
    # the decode side cache: the prefill's pooled rows, NaN everywhere else
    pooled = torch.full((w.batch, nblk, w.idx_dim), float("nan"), device="cuda")
    for b, Lb in enumerate(L):
        pooled[b, :Lb // B] = pf[b, :Lb // B]
    dt = TL.tdtype(w)
    excused = []
    for s in range(1, steps + 1):
        kv_np = np.array([Lb + s * n_q for Lb in L], np.int32)
        step_in = {k: v for k, v in inp.items()}
        for nm, shape in (("q", (w.batch, n_q, w.num_q_heads, w.head_dim)),
                          ("iq", (w.batch, n_q, w.idx_heads, w.idx_dim)),
                          ("gate", (w.batch, n_q, w.num_q_heads, w.head_dim))):
            x = rng.standard_normal(shape).astype(np.float32) * np.float32(0.1)
            step_in[nm] = TL.round_like(x, w)
        step_in["iw"] = rng.random((w.batch, n_q, w.idx_heads)).astype(np.float32)
        step_in["kv_len"] = kv_np
        dd = {nm: torch.from_numpy(np.ascontiguousarray(step_in[nm])).to("cuda")
              for nm in ("q", "iq", "gate", "iw")}
        for nm in ("q", "iq", "gate"):
            dd[nm] = dd[nm].to(dt)
        kv = torch.from_numpy(kv_np).to("cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        r = qsa.decode(cfg, dd["q"], d["k_cache"], d["v_cache"], dd["iq"], d["ik_cache"],
                       dd["iw"], dd["gate"], pooled, kv, want_lse=True, want_sel=True,
                       dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        orc = O.qsa_decode(w, step_in)["queries"]
        rep = TL.check_queries(orc, r, lambda bi: bi, w)
        excused += [(s, k) for k in rep["excused_near_ties"]]
    print(f"{name}: {steps} steps, excused near-ties {excused}")
    assert len(excused) <= 2
    final = torch.from_numpy(np.array([Lb + steps * n_q for Lb in L], np.int32)).to("cuda")
    rebuilt = qsa.pool_build(cfg, d["ik_cache"], final)
    pf_all = _prefill_pooled(cfg, w, d, [int(x) for x in final.cpu()], rng)
    torch.cuda.synchronize()
    for b in range(w.batch):
        nb = int(final[b]) // B
        assert nb >= L[b] // B + 2, "the steps must complete at least two blocks"
        assert torch.equal(pooled[b, :nb], rebuilt[b, :nb]), b
        assert torch.equal(pooled[b, :nb], pf_all[b, :nb]), b
        assert torch.isnan(pooled[b, nb:]).all(), "a row past the complete blocks was written"
