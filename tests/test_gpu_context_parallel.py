"""Context-parallel decode on one GPU: the ranks' shards are processed one
after another through the library (qsa_cp_select on each shard, the global
top-k over the stacked candidates, qsa_cp_attend on each shard, the
log-sum-exp merge), with torch.stack standing in for the all-gathers. The
selection must be bit-identical to qsa_decode on the whole cache (lists and
counts, tail blocks included), and the outputs must match the oracle within
the dtype's tolerance (the partials are fp32, so the only rounding is the
merged output's); bf16 runs the tensor-map attention kernel, fp32 the
CUDA-core one."""
import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200 import context_parallel as cp
from block_sparse_attention_17_b200.workloads import WORKLOADS, make_decode_inputs
from oracle import qsa_oracle as O
from tests import qsa_testlib as TL

pytestmark = pytest.mark.gpu


def _emulated_cp(cfg, w, d, world):
    B = w.block_size
    nblk = d["k_cache"].shape[1] // B
    kv = d["kv_len"]
    shards = [cp.shard_blocks(nblk, world, r) for r in range(world)]
    rows = lambda t, b0, b1: t[:, b0 * B:b1 * B].contiguous()
    cands, fns = [], []
    for b0, b1 in shards:
        # the shard's pooled rows hold the blocks completed before this step
        ik = rows(d["ik_cache"], b0, b1)
        pooled = qsa.cp_pool_build(cfg, ik, (kv - w.n_q).to(torch.int32), b0)
        f = cp.library_fns(cfg, d["q"], rows(d["k_cache"], b0, b1), rows(d["v_cache"], b0, b1),
                           d["iq"], ik, d["iw"], d["gate"], pooled, b0)
        fns.append(f)
        cands.append(f.select(kv))
    glob = fns[0].global_topk(torch.stack([c["score"] for c in cands]),
                              torch.stack([c["id"] for c in cands]), kv)
    parts = [f.attend(kv, glob["sel"], glob["nsel"]) for f in fns]
    merged = fns[0].merge(torch.stack([p["out"] for p in parts]),
                          torch.stack([p["lse"] for p in parts]))
    return merged, glob


@pytest.mark.parametrize("world,n_q,dtype,rope_dim", [
    (2, 1, "bf16", 0), (3, 1, "bf16", 0), (4, 2, "bf16", 0), (3, 1, "f32", 0), (2, 3, "bf16", 0),
    (3, 1, "bf16", 64), (2, 2, "f32", 32)])
def test_context_parallel_decode_emulated_ranks(world, n_q, dtype, rope_dim):
    # rope_dim > 0: the indexer rotary embedding, where every shard must turn its
    # pooled rows at their global block positions
    w = WORKLOADS["decode_bf16_b32_kv32768"].with_(batch=4, cap=64 * 120, kv_len=64 * 120,
                                                   n_q=n_q, dtype=dtype, rope_dim=rope_dim,
                                                   rope_theta=10000.0)
    # full, ragged, ending inside an early shard, and a short one
    kv = np.array([64 * 120, 64 * 117 + 5, 64 * 37 + 63, 200], np.int32)
    inp = make_decode_inputs(w, kv_lens=kv)
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    pooled = qsa.pool_build(cfg, d["ik_cache"], (d["kv_len"] - n_q).to(torch.int32))
    # each shard's pool build gives the whole cache's rows, bit for bit
    B, nblk = w.block_size, w.cap // w.block_size
    for r in range(world):
        b0, b1 = cp.shard_blocks(nblk, world, r)
        ps = qsa.cp_pool_build(cfg, d["ik_cache"][:, b0 * B:b1 * B].contiguous(),
                               (d["kv_len"] - n_q).to(torch.int32), b0)
        assert torch.equal(ps, pooled[:, b0:b1]), r
    ref = qsa.decode(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"], d["ik_cache"], d["iw"],
                     d["gate"], pooled, d["kv_len"], want_lse=True, want_sel=True)
    merged, glob = _emulated_cp(cfg, w, d, world)
    torch.cuda.synchronize()
    assert torch.equal(glob["nsel"], ref["nsel"])
    for b in range(w.batch):
        for i in range(n_q):
            m = int(ref["nsel"][b, i])
            assert torch.equal(glob["sel"][b, i, :m], ref["sel"][b, i, :m]), (b, i)
    tol = TL.TOL_OUT[w.dtype]
    orc = O.qsa_decode(w, inp)["queries"]
    got = merged["out"].double().cpu().numpy()
    lse = merged["lse"].double().cpu().numpy()
    for (b, i), r in orc.items():
        assert np.max(np.abs(got[b, i] - r.out)) <= tol, (b, i)
        assert np.max(np.abs(lse[b, i] - r.lse)) <= max(tol, 1e-4), (b, i)
