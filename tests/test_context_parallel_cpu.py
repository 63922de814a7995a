"""Context-parallel decode's host logic (block_sparse_attention_17_b200.
context_parallel) on CPU: world_size-2 and -3 gloo ranks, each rank's compute
steps (local pooling, scoring, top-k; attention over a given block list) done
by the fp64 oracle, the candidate exchange and the partial merge by the module
under test. The result must equal the oracle's single-process decode: the same
selected blocks and the same gated outputs."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from block_sparse_attention_17_b200 import context_parallel as cp  # noqa: E402
from block_sparse_attention_17_b200.workloads import WORKLOADS, make_decode_inputs  # noqa: E402
from oracle import qsa_oracle as O  # noqa: E402


def _case():
    # 3 sequences of a few hundred blocks, one new token each; B = 16 keeps it small
    w = WORKLOADS["decode_bf16_b32_kv32768"].with_(dtype="f32", batch=3, block_size=16,
                                                   budget=16 * 8, cap=16 * 60, kv_len=16 * 60)
    kv = np.array([16 * 60, 16 * 53 + 7, 16 * 45 + 1], np.int32)
    return w, make_decode_inputs(w, kv_lens=kv)


def _oracle_fns(w, inp, b0, b1):
    """This rank's compute steps on its shard, by the oracle (fp64)."""
    B, k = w.block_size, w.topk
    sm, isc = w.head_dim ** -0.5, w.idx_dim ** -0.5
    nloc = b1 - b0
    ik = inp["ik_cache"][:, b0 * B:b1 * B]
    K, V = inp["k_cache"][:, b0 * B:b1 * B], inp["v_cache"][:, b0 * B:b1 * B]

    def select_fn(kv_loc):
        batch = kv_loc.shape[0]
        sel = torch.full((batch, 1, k + 1), -1, dtype=torch.int32)
        nsel = torch.zeros(batch, 1, dtype=torch.int32)
        scores = torch.full((batch, 1, nloc), float("-inf"), dtype=torch.float64)
        for b in range(batch):
            n = int(kv_loc[b])
            kbar = O.pool_blocks(ik[b, :n], B)
            s = O.index_scores(inp["iq"][b, 0], inp["iw"][b, 0], kbar, isc)
            chosen = list(O.select_topk(s, k)) + ([n // B] if n % B else [])
            sel[b, 0, :len(chosen)] = torch.tensor(chosen, dtype=torch.int32)
            nsel[b, 0] = len(chosen)
            scores[b, 0, :len(s)] = torch.from_numpy(s)
        return {"sel": sel, "nsel": nsel, "scores": scores}

    def attend_fn(kv_loc, sel, nsel):
        batch = kv_loc.shape[0]
        out = torch.zeros(batch, 1, w.num_q_heads, w.head_dim, dtype=torch.float64)
        lse = torch.full((batch, 1, w.num_q_heads), float("-inf"), dtype=torch.float64)
        for b in range(batch):
            n = int(kv_loc[b])
            pos = [np.arange(j * B, min((j + 1) * B, n)) for j in sel[b, 0, :int(nsel[b, 0])].tolist()]
            pos = np.concatenate(pos) if pos else np.zeros(0, np.int64)
            o, l = O.gated_attention(inp["q"][b, 0], K[b], V[b], pos, inp["gate"][b, 0], sm)
            out[b, 0], lse[b, 0] = torch.from_numpy(o), torch.from_numpy(l)
        return {"out": out, "lse": lse}
    return select_fn, attend_fn


def _rank_main(rank, world, port, results):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, inp = _case()
        nblk = w.cap // w.block_size
        b0, b1 = cp.shard_blocks(nblk, world, rank)
        select_fn, attend_fn = _oracle_fns(w, inp, b0, b1)
        cfg = cp.qsa.QSAConfig.from_workload(w)
        q = torch.from_numpy(inp["q"]).double()
        r = cp.decode_step(cfg, q, None, None, None, None, None, None, None,
                           torch.from_numpy(inp["kv_len"]), b0=b0, b1=b1,
                           is_last=rank == world - 1, select_fn=select_fn, attend_fn=attend_fn)
        results[rank] = (r["out"].numpy(), r["lse"].numpy(), r["sel"].numpy(), r["count"].numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_decode_gloo_matches_single_process(world):
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                       join=True, start_method="spawn")
    assert sorted(results.keys()) == list(range(world))
    w, inp = _case()
    orc = O.qsa_decode(w, inp)["queries"]
    for rank in range(world):
        out, lse, sel, count = results[rank]
        for b in range(w.batch):
            ref = orc[(b, 0)]
            got = [j for j in sel[b].tolist() if j >= 0]
            assert got == list(ref.selected), (rank, b)
            assert int(count[b]) == len(ref.selected)
            np.testing.assert_allclose(out[b, 0], ref.out, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(lse[b, 0], ref.lse, rtol=1e-10, atol=1e-12)
        np.testing.assert_array_equal(out, results[0][0])   # every rank holds the same result


def test_global_topk_order_and_ties():
    # scores tie across ranks: the lower block id wins; -0 ties +0
    cs = torch.tensor([[[3.0, 1.0, -0.0]], [[1.0, 2.0, float("-inf")]]])
    cid = torch.tensor([[[10, 4, 7]], [[2, 30, 2 ** 62]]])
    ids, count = cp.global_topk(cs, cid, 3)
    assert ids.tolist() == [[2, 10, 30]] and count.tolist() == [3]
    cs = torch.tensor([[[0.0, 5.0]], [[-0.0, float("-inf")]]])
    cid = torch.tensor([[[9, 1]], [[3, 2 ** 62]]])
    ids, count = cp.global_topk(cs, cid, 2)
    assert ids.tolist() == [[1, 3]] and count.tolist() == [2]


def test_shard_blocks_cover_the_cache_once():
    for nblk in (1, 7, 64, 513):
        for world in (1, 2, 3, 8):
            ranges = [cp.shard_blocks(nblk, world, r) for r in range(world)]
            covered = [j for b0, b1 in ranges for j in range(b0, b1)]
            assert covered == list(range(nblk))


def test_local_candidates_skip_the_tail_and_unused_slots():
    # local selection: blocks 1, 5 (complete) and the tail block 7 (score -inf)
    sel = torch.tensor([[[1, 5, 7, -1]]], dtype=torch.int32)
    nsel = torch.tensor([[3]], dtype=torch.int32)
    scores = torch.tensor([[[0.1, 2.0, 0.3, 0.4, 0.5, 1.5, 0.0, float("-inf")]]])
    sc, gid = cp.local_candidates(sel, nsel, scores, 3, b0=100)
    assert gid.tolist() == [[101, 105, 2 ** 62]]
    assert sc[0, :2].tolist() == [2.0, 1.5] and sc[0, 2].item() == float("-inf")


def test_local_share_adds_the_tail_on_the_last_rank_only():
    gids = torch.tensor([[3, 10, 25, -1], [8, 9, -1, -1]])
    kv = torch.tensor([16 * 16 + 5, 16 * 16], dtype=torch.int32)   # rows in the shard
    sel, nsel = cp.local_share(gids, 8, 24, kv, 16, 4, is_last=True)
    assert sel[0, 0].tolist() == [2, 16, -1, -1, -1] and nsel[0, 0].item() == 2   # tail block 16
    assert sel[1, 0].tolist() == [0, 1, -1, -1, -1] and nsel[1, 0].item() == 2    # no tail
    sel, nsel = cp.local_share(gids, 8, 24, kv, 16, 4, is_last=False)
    assert sel[0, 0].tolist() == [2, -1, -1, -1, -1] and nsel[0, 0].item() == 1


def test_merge_partials_weights_and_empty_ranks():
    outs = torch.tensor([[[[1.0, 2.0]]], [[[3.0, 4.0]]], [[[9.0, 9.0]]]])     # [R, b, 1, 2]
    lses = torch.tensor([[[0.0]], [[float(np.log(3.0))]], [[float("-inf")]]])  # [R, b, 1]
    out, lse = cp.merge_partials(outs[..., None, :].squeeze(-2), lses)
    # weights 1/4 and 3/4; the rank with nothing attended weighs nothing
    assert torch.allclose(out, torch.tensor([[[2.5, 3.5]]]))
    assert torch.allclose(lse, torch.tensor([[float(np.log(4.0))]]))
    out, lse = cp.merge_partials(outs[:1] * 0, torch.full((1, 1, 1), float("-inf")))
    assert torch.equal(out, torch.zeros(1, 1, 2)) and lse.item() == float("-inf")
