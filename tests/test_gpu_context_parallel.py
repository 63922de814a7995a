"""Context-parallel decode on one GPU: the ranks' shards are processed one
after another through the library (qsa_select_decode on each shard, the
candidate exchange, qsa_decode_attend on each rank's share, the log-sum-exp
merge), with torch.stack standing in for the all-gathers. The result must
equal qsa_decode on the whole cache: the same selected blocks, the same gated
outputs within the bf16 tolerance (the partials are rounded to bf16 before the
merge), and the oracle's outputs."""
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
    B, k = w.block_size, w.topk
    nblk = d["k_cache"].shape[1] // B
    kv = d["kv_len"]
    shards = [cp.shard_blocks(nblk, world, r) for r in range(world)]
    loc = []
    for r, (b0, b1) in enumerate(shards):
        kvl = cp.local_kv(kv, b0, b1, B)
        ik = d["ik_cache"][:, b0 * B:b1 * B].contiguous()
        pooled = qsa.pool_build(cfg, ik, (kvl - 1).to(torch.int32))
        s = qsa.select_decode(cfg, d["iq"], ik, d["iw"], pooled, kvl, want_scores=True)
        loc.append((kvl, cp.local_candidates(s["sel"], s["nsel"], s["scores"], k, b0)))
    gids, count = cp.global_topk(torch.stack([c[0] for _, c in loc]),
                                 torch.stack([c[1] for _, c in loc]), k)
    outs, lses = [], []
    for r, (b0, b1) in enumerate(shards):
        kvl = loc[r][0]
        sel, nsel = cp.local_share(gids, b0, b1, kvl, B, k, r == world - 1)
        a = qsa.decode_attend(cfg, d["q"], d["k_cache"][:, b0 * B:b1 * B].contiguous(),
                              d["v_cache"][:, b0 * B:b1 * B].contiguous(), d["gate"], kvl,
                              sel, nsel, want_lse=True)
        outs.append(a["out"])
        lses.append(a["lse"])
    out, lse = cp.merge_partials(torch.stack(outs), torch.stack(lses))
    return out, lse, gids, count


@pytest.mark.parametrize("world", [2, 3, 4])
def test_context_parallel_decode_emulated_ranks(world):
    w = WORKLOADS["decode_bf16_b32_kv32768"].with_(batch=3, cap=64 * 120, kv_len=64 * 120)
    kv = np.array([64 * 120, 64 * 117 + 5, 64 * 100 + 63], np.int32)
    inp = make_decode_inputs(w, kv_lens=kv)
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    pooled = qsa.pool_build(cfg, d["ik_cache"], (d["kv_len"] - 1).to(torch.int32))
    ref = qsa.decode(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"], d["ik_cache"], d["iw"],
                     d["gate"], pooled, d["kv_len"], want_lse=True, want_sel=True)
    out, lse, gids, count = _emulated_cp(cfg, w, d, world)
    torch.cuda.synchronize()
    k = w.topk
    for b in range(w.batch):
        n = int(kv[b])
        ref_sel = [j for j in ref["sel"][b, 0].tolist()[:int(ref["nsel"][b, 0])] if j < n // 64]
        assert [j for j in gids[b].tolist() if j >= 0] == ref_sel
        assert int(count[b]) == min(k, n // 64)
    torch.testing.assert_close(out.to(torch.bfloat16).float(), ref["out"].float(), atol=2e-2, rtol=0)
    torch.testing.assert_close(lse, ref["lse"], atol=1e-3, rtol=0)
    orc = O.qsa_decode(w, inp)["queries"]
    got = out.double().cpu().numpy()
    for b in range(w.batch):
        np.testing.assert_allclose(got[b, 0], orc[(b, 0)].out, atol=2e-2, rtol=0)
