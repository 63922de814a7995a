"""Context-parallel decode's host logic (block_sparse_attention_17_b200.
context_parallel) on CPU: world_size-2 and -3 gloo ranks. Each rank's four
compute steps, which the library runs as kernels on a GPU (shard selection,
global top-k, shard attention, log-sum-exp merge), are done here by fp64
stand-ins written from the pages' definitions with the oracle's functions;
the module under test drives them and moves the candidates and partials
between the ranks with all-gathers. The result must equal the oracle's
single-process decode: the same selected blocks and the same gated outputs,
for one and two new tokens per sequence and for sequences that end inside an
early shard."""
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


def _case(n_q):
    # 3 sequences of up to 60 blocks; B = 16 keeps it small; the third one
    # ends in the first half of the cache (inside an early shard)
    w = WORKLOADS["decode_bf16_b32_kv32768"].with_(dtype="f32", batch=3, block_size=16,
                                                   budget=16 * 8, cap=16 * 60, kv_len=16 * 60,
                                                   n_q=n_q)
    kv = np.array([16 * 60, 16 * 53 + 7, 16 * 21 + 1], np.int32)
    return w, make_decode_inputs(w, kv_lens=kv)


def _oracle_fns(w, inp, b0, b1):
    """This rank's four steps on shard [b0, b1), in fp64 with the oracle's
    functions (global block ids; the shard sees the full cache rows)."""
    B, k, n_q = w.block_size, w.topk, w.n_q
    sm, isc = w.head_dim ** -0.5, w.idx_dim ** -0.5

    def visible(kv, i):
        return int(kv) - n_q + 1 + i

    def select(kv_len):
        batch = kv_len.shape[0]
        score = torch.full((batch, n_q, k), float("-inf"), dtype=torch.float64)
        ids = torch.full((batch, n_q, k), -1, dtype=torch.int32)
        for b in range(batch):
            kbar = O.pool_blocks(inp["ik_cache"][b, :int(kv_len[b])], B)
            for i in range(n_q):
                nc = visible(kv_len[b], i) // B
                mine = list(range(b0, min(b1, nc)))
                if not mine:
                    continue
                s = O.index_scores(inp["iq"][b, i], inp["iw"][b, i], kbar[mine], isc)
                top = O.select_topk(s, k)
                score[b, i, :len(top)] = torch.from_numpy(s[top])
                ids[b, i, :len(top)] = torch.tensor([mine[t] for t in top], dtype=torch.int32)
        return {"score": score, "id": ids}

    def global_topk(cs, cid, kv_len):
        W, batch = cs.shape[0], cs.shape[1]
        sel = torch.full((batch, n_q, k + 1), -1, dtype=torch.int32)
        nsel = torch.zeros(batch, n_q, dtype=torch.int32)
        for b in range(batch):
            for i in range(n_q):
                cands = [(float(cs[r, b, i, j]), int(cid[r, b, i, j]))
                         for r in range(W) for j in range(k) if int(cid[r, b, i, j]) >= 0]
                cands.sort(key=lambda c: (-c[0], c[1]))
                chosen = sorted(c[1] for c in cands[:k])
                n = visible(kv_len[b], i)
                if n % B:
                    chosen.append(n // B)
                sel[b, i, :len(chosen)] = torch.tensor(chosen, dtype=torch.int32)
                nsel[b, i] = len(chosen)
        return {"sel": sel, "nsel": nsel}

    def attend(kv_len, sel, nsel):
        batch = kv_len.shape[0]
        out = torch.zeros(batch, n_q, w.num_q_heads, w.head_dim, dtype=torch.float64)
        lse = torch.full((batch, n_q, w.num_q_heads), float("-inf"), dtype=torch.float64)
        for b in range(batch):
            for i in range(n_q):
                n = visible(kv_len[b], i)
                blocks = [j for j in sel[b, i, :int(nsel[b, i])].tolist() if b0 <= j < b1]
                pos = [np.arange(j * B, min((j + 1) * B, n)) for j in blocks]
                pos = np.concatenate(pos) if pos else np.zeros(0, np.int64)
                if len(pos) == 0:
                    continue
                o, l = O.gated_attention(inp["q"][b, i], inp["k_cache"][b], inp["v_cache"][b],
                                         pos, inp["gate"][b, i], sm)
                out[b, i], lse[b, i] = torch.from_numpy(o), torch.from_numpy(l)
        return {"out": out, "lse": lse}

    def merge(po, pl):
        lse = torch.logsumexp(pl, dim=0)
        wgt = torch.nan_to_num(torch.exp(pl - lse[None]), nan=0.0)
        return {"out": (wgt[..., None] * po).sum(dim=0), "lse": lse}

    return cp.CpFns(select=select, global_topk=global_topk, attend=attend, merge=merge)


def _rank_main(rank, world, n_q, port, results):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, inp = _case(n_q)
        nblk = w.cap // w.block_size
        b0, b1 = cp.shard_blocks(nblk, world, rank)
        cfg = cp.qsa.QSAConfig.from_workload(w)
        r = cp.decode_step(cfg, None, None, None, None, None, None, None, None,
                           torch.from_numpy(inp["kv_len"]), b0=b0,
                           fns=_oracle_fns(w, inp, b0, b1))
        results[rank] = (r["out"].numpy(), r["lse"].numpy(), r["sel"].numpy(), r["nsel"].numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,n_q", [(2, 1), (3, 1), (3, 2)])
def test_context_parallel_decode_gloo_matches_single_process(world, n_q):
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, n_q, _free_port(), results), nprocs=world,
                       join=True, start_method="spawn")
    assert sorted(results.keys()) == list(range(world))
    w, inp = _case(n_q)
    orc = O.qsa_decode(w, inp)["queries"]
    for rank in range(world):
        out, lse, sel, nsel = results[rank]
        for b in range(w.batch):
            for i in range(n_q):
                ref = orc[(b, i)]
                exp = list(ref.selected) + ([ref.nc] if ref.tail else [])
                assert sel[b, i, :int(nsel[b, i])].tolist() == exp, (rank, b, i)
                np.testing.assert_allclose(out[b, i], ref.out, rtol=1e-10, atol=1e-12)
                np.testing.assert_allclose(lse[b, i], ref.lse, rtol=1e-10, atol=1e-12)
        np.testing.assert_array_equal(out, results[0][0])   # every rank holds the same result


def test_shard_blocks_cover_the_cache_once():
    for nblk in (1, 7, 64, 513):
        for world in (1, 2, 3, 8):
            ranges = [cp.shard_blocks(nblk, world, r) for r in range(world)]
            covered = [j for b0, b1 in ranges for j in range(b0, b1)]
            assert covered == list(range(nblk))


def test_decode_step_passes_each_rank_result_through_the_gather():
    # a world of 2 emulated by a gather that stacks this rank's tensor with a
    # second rank's (a fixed tensor): the global top-k and the merge must see
    # [world, ...] arrays in rank order
    seen = {}

    def gather(t):
        other = torch.full_like(t, 7)
        return torch.stack([t, other])

    fns = cp.CpFns(
        select=lambda kv: {"score": torch.ones(1, 1, 2), "id": torch.tensor([[[1, 2]]])},
        global_topk=lambda cs, cid, kv: seen.setdefault("g", (cs, cid)) and
        {"sel": torch.tensor([[[1, 2, -1]]]), "nsel": torch.tensor([[2]])},
        attend=lambda kv, sel, nsel: {"out": torch.zeros(1, 1, 1, 4), "lse": torch.zeros(1, 1, 1)},
        merge=lambda po, pl: seen.setdefault("m", (po, pl)) and
        {"out": po[0], "lse": pl[0]})
    cfg = cp.qsa.QSAConfig(num_q_heads=1, num_kv_heads=1, head_dim=4, idx_heads=1, idx_dim=4,
                           block_size=64, budget=128)
    r = cp.decode_step(cfg, None, None, None, None, None, None, None, None,
                       torch.tensor([300], dtype=torch.int32), b0=0, fns=fns, gather_fn=gather)
    cs, cid = seen["g"]
    assert cs.shape == (2, 1, 1, 2) and cid[0].tolist() == [[[1, 2]]] and cid[1].eq(7).all()
    po, pl = seen["m"]
    assert po.shape == (2, 1, 1, 1, 4) and pl.shape == (2, 1, 1, 1)
    assert r["nsel"].tolist() == [[2]]
