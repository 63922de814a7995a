"""Context-parallel QSA decode: the KV cache of long sequences sharded by
blocks over the processes of a group (one process per GPU).

Rank r holds cache blocks [b0, b1) of every sequence of the batch (K, V,
indexer keys and their pooled rows, at local block ids 0 .. b1 - b0). One
decode step (one new token per sequence) is:

1. local selection: the rank pools and scores its own complete blocks and
   keeps its top k (qsa_select_decode on the shard);
2. an all-gather of every rank's (score, global block id) candidates; the
   global top k under the order (score descending, block id ascending) is
   exactly the top k of the whole cache, because each of its blocks is in the
   top k of its own shard (the selection rule of the llama.cpp PR #27739 page
   and the instagit MTPLX page, unchanged);
3. local attention: the rank attends its share of the global selection (and,
   on the rank holding the sequence's last rows, the incomplete tail block)
   with qsa_decode_attend, giving a gated output and its log-sum-exp;
4. an all-gather of the (output, lse) pairs and their log-sum-exp merge: with
   w_r = exp(lse_r - logsumexp_r lse_r), out = sum_r w_r out_r, which is the
   gated attention over the union (the sigmoid gate is elementwise, so it
   commutes with the weighted sum).

The scores are computed per shard with the library's own arithmetic, so the
selection equals the single-GPU one. Requirements: one new token per sequence
(n_q = 1); every rank's shard holds at least one visible token of every
sequence, and the shards before the last are full (the sequence's tail lives
on the last rank).

The collectives are torch.distributed all-gathers (NCCL over NVLink on B200);
the compute steps and the gather can be replaced (select_fn, attend_fn,
gather_fn), which is how the host logic is tested on CPU ranks.
"""
from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import api as qsa

_BIG = 2 ** 62


def shard_blocks(nblk: int, world: int, rank: int) -> tuple:
    """Contiguous block range [b0, b1) of `rank` when nblk cache blocks are
    split over `world` ranks (ceil(nblk / world) blocks each, the last rank
    the rest)."""
    per = -(-nblk // world)
    b0 = min(nblk, rank * per)
    return b0, min(nblk, b0 + per)


def local_kv(kv_len: torch.Tensor, b0: int, b1: int, block_size: int) -> torch.Tensor:
    """Rows of each sequence inside the shard [b0, b1) (int32)."""
    return torch.clamp(kv_len.to(torch.int64) - b0 * block_size, 0,
                       (b1 - b0) * block_size).to(torch.int32)


def local_candidates(sel: torch.Tensor, nsel: torch.Tensor, scores: torch.Tensor, k: int,
                     b0: int) -> tuple:
    """The shard's top-k complete blocks as (score [batch, k], global id
    [batch, k]); unused slots hold (-inf, a large id). sel/nsel/scores are the
    local selection's outputs for one new token per sequence; the tail block,
    whose score is -inf, is not a candidate."""
    s = sel[:, 0, :].to(torch.int64)
    used = torch.arange(s.shape[1], device=s.device)[None, :] < nsel[:, 0:1].to(torch.int64)
    ids = torch.where(used, s, torch.zeros_like(s)).clamp(min=0)
    sc = torch.gather(scores[:, 0, :], 1, ids)
    valid = used & torch.isfinite(sc)
    order = torch.sort((~valid).to(torch.int8), dim=1, stable=True).indices[:, :k]
    valid = torch.gather(valid, 1, order)
    sc = torch.where(valid, torch.gather(sc, 1, order), torch.full_like(sc[:, :k], float("-inf")))
    gid = torch.where(valid, torch.gather(ids, 1, order) + b0,
                      torch.full_like(order, _BIG))
    return sc, gid


def global_topk(cand_score: torch.Tensor, cand_id: torch.Tensor, k: int) -> tuple:
    """Top k of the gathered candidates ([ranks, batch, k] each) under (score
    descending, block id ascending): (ids [batch, k] ascending, -1 padded;
    count [batch])."""
    R, batch, kk = cand_score.shape
    sc = cand_score.permute(1, 0, 2).reshape(batch, R * kk)
    gid = cand_id.permute(1, 0, 2).reshape(batch, R * kk)
    o1 = torch.sort(gid, dim=1, stable=True).indices            # id ascending
    sc, gid = torch.gather(sc, 1, o1), torch.gather(gid, 1, o1)
    o2 = torch.sort(sc, dim=1, descending=True, stable=True).indices[:, :k]
    top_sc, top_id = torch.gather(sc, 1, o2), torch.gather(gid, 1, o2)
    ok = torch.isfinite(top_sc)
    top_id = torch.where(ok, top_id, torch.full_like(top_id, _BIG))
    top_id = torch.sort(top_id, dim=1).values
    count = ok.sum(dim=1)
    return torch.where(top_id < _BIG, top_id, torch.full_like(top_id, -1)), count


def local_share(global_ids: torch.Tensor, b0: int, b1: int, kv_loc: torch.Tensor,
                block_size: int, k: int, is_last: bool) -> tuple:
    """The blocks of [b0, b1) in the global selection as local ids, ascending,
    plus (on the last rank) the incomplete tail block: (sel [batch, 1, k + 1]
    int32, -1 padded; nsel [batch, 1] int32)."""
    batch = global_ids.shape[0]
    mine = (global_ids >= b0) & (global_ids < b1)
    loc = torch.where(mine, global_ids - b0, torch.full_like(global_ids, _BIG))
    loc = torch.sort(loc, dim=1).values
    cnt = mine.sum(dim=1)
    sel = torch.full((batch, k + 1), -1, dtype=torch.int64, device=global_ids.device)
    sel[:, :k] = torch.where(loc < _BIG, loc, torch.full_like(loc, -1))
    if is_last:
        kv = kv_loc.to(torch.int64)
        has_tail = (kv % block_size) > 0
        tail_pos = torch.where(has_tail, cnt, torch.full_like(cnt, k))   # slot k: past nsel
        sel.scatter_(1, tail_pos[:, None], torch.where(has_tail, kv // block_size,
                                                       torch.full_like(kv, -1))[:, None])
        cnt = cnt + has_tail.to(cnt.dtype)
    return sel[:, None, :].to(torch.int32).contiguous(), cnt[:, None].to(torch.int32).contiguous()


def merge_partials(outs: torch.Tensor, lses: torch.Tensor) -> tuple:
    """Log-sum-exp merge of gated partial outputs [ranks, batch, 1, Hq, D]
    (or [.., Hq]) with their natural-log lse [ranks, batch, 1, Hq]: (out fp32,
    lse)."""
    lse = torch.logsumexp(lses, dim=0)
    w = torch.nan_to_num(torch.exp(lses - lse[None]), nan=0.0)
    shape = w.shape + (1,) * (outs.dim() - w.dim())
    out = (w.reshape(shape) * outs.to(torch.float64 if outs.dtype == torch.float64
                                       else torch.float32)).sum(dim=0)
    return out, lse


def _all_gather(group):
    def gather(t: torch.Tensor) -> torch.Tensor:
        parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)
    return gather


def decode_step(cfg: qsa.QSAConfig, q, k_shard, v_shard, iq, ik_shard, iw, gate, pooled_shard,
                kv_len, *, b0: int, b1: int, is_last: bool, group=None,
                select_fn: Optional[Callable] = None, attend_fn: Optional[Callable] = None,
                gather_fn: Optional[Callable] = None) -> dict:
    """One context-parallel decode step on this rank's shard [b0, b1) (see the
    module docstring). q, iq, iw, gate: the step's inputs for the batch
    ([batch, 1, ...], the same on every rank); k_shard, v_shard, ik_shard,
    pooled_shard: this rank's rows of the caches; kv_len [batch]: the
    sequences' full lengths. Returns {"out" (q's dtype), "lse", "sel" (global
    block ids of the selected complete blocks, ascending, -1 padded),
    "count"}; every rank returns the same values."""
    B, k = cfg.block_size, cfg.topk
    if q.shape[1] != 1:
        raise ValueError("context-parallel decode takes one new token per sequence")
    kv_loc = local_kv(kv_len, b0, b1, B)
    if select_fn is None:
        select_fn = lambda kvl: qsa.select_decode(cfg, iq, ik_shard, iw, pooled_shard, kvl,
                                                  want_scores=True)
    if attend_fn is None:
        attend_fn = lambda kvl, sel, nsel: qsa.decode_attend(cfg, q, k_shard, v_shard, gate, kvl,
                                                             sel, nsel, want_lse=True)
    if gather_fn is None:
        gather_fn = _all_gather(group)
    loc = select_fn(kv_loc)
    cs, cid = local_candidates(loc["sel"], loc["nsel"], loc["scores"], k, b0)
    gids, count = global_topk(gather_fn(cs), gather_fn(cid), k)
    sel, nsel = local_share(gids, b0, b1, kv_loc, B, k, is_last)
    part = attend_fn(kv_loc, sel, nsel)
    out, lse = merge_partials(gather_fn(part["out"]), gather_fn(part["lse"]))
    return {"out": out.to(q.dtype), "lse": lse, "sel": gids, "count": count}
