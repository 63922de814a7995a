"""Context-parallel QSA decode: the KV cache of long sequences sharded by
blocks over the processes of a group (one process per GPU).

Rank r holds cache blocks [b0, b1) of every sequence (K, V, indexer keys and
their pooled rows, at local block ids 0 .. b1 - b0). One decode step (n_q new
tokens per sequence, appended to the rank that holds those rows) is:

1. qsa_cp_select on every rank: the rank pools the blocks of its shard this
   step completes, scores its complete visible blocks and keeps each query's
   top k as candidates (score, global block id);
2. an all-gather of the candidates, then qsa_cp_global_topk: the top k under
   (score descending, block id ascending) plus each query's tail block, which
   is exactly the single-GPU selection (each globally selected block is in its
   own shard's top k, and every shard scores with the same arithmetic);
3. qsa_cp_attend on every rank: gated attention over the selected blocks that
   lie in its shard, as fp32 partials with their log-sum-exp;
4. an all-gather of the partials, then qsa_cp_merge: the log-sum-exp merge
   (the sigmoid gate is elementwise and commutes with the weighted sum).

Every step of the method runs in the library's kernels; this module only
picks the shard ranges and moves the candidates and partials between ranks
with torch.distributed all-gathers (NCCL over NVLink on B200). The pages
describe no multi-GPU QSA; the split (contiguous block ranges) follows the
step's data dependencies. The library calls and the gather can be replaced
(``fns``, ``gather_fn``), which is how the host logic is tested on CPU ranks.
"""
from dataclasses import dataclass
from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import api as qsa


def shard_blocks(nblk: int, world: int, rank: int) -> tuple:
    """Contiguous block range [b0, b1) of `rank` when nblk cache blocks are
    split over `world` ranks (ceil(nblk / world) blocks each, the last rank
    the rest)."""
    per = -(-nblk // world)
    b0 = min(nblk, rank * per)
    return b0, min(nblk, b0 + per)


@dataclass
class CpFns:
    """The four compute steps of a context-parallel decode step (defaults:
    the library's entry points)."""
    select: Callable
    global_topk: Callable
    attend: Callable
    merge: Callable


def library_fns(cfg: qsa.QSAConfig, q, k_shard, v_shard, iq, ik_shard, iw, gate, pooled_shard,
                b0: int, workspace=None) -> CpFns:
    return CpFns(
        select=lambda kv: qsa.cp_select(cfg, iq, ik_shard, iw, pooled_shard, kv, b0,
                                        workspace=workspace),
        global_topk=lambda cs, cid, kv: qsa.cp_global_topk(cfg, cs, cid, kv),
        attend=lambda kv, sel, nsel: qsa.cp_attend(cfg, q, k_shard, v_shard, gate, kv, sel, nsel,
                                                   b0, workspace=workspace),
        merge=lambda po, pl: qsa.cp_merge(cfg, po, pl))


def _all_gather(group):
    def gather(t: torch.Tensor) -> torch.Tensor:
        parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)
    return gather


def decode_step(cfg: qsa.QSAConfig, q, k_shard, v_shard, iq, ik_shard, iw, gate, pooled_shard,
                kv_len, *, b0: int, group=None, fns: Optional[CpFns] = None,
                gather_fn: Optional[Callable] = None, workspace=None) -> dict:
    """One context-parallel decode step on this rank's shard, which starts at
    block b0 (see the module docstring). q, iq, iw, gate: the step's inputs
    for the batch ([batch, n_q, ...], the same on every rank); k_shard, v_shard,
    ik_shard, pooled_shard: this rank's rows of the caches; kv_len [batch]
    int32: the sequences' full lengths. Returns {"out" (cfg.dtype), "lse",
    "sel" (global ids, as qsa_decode writes them), "nsel"}; every rank returns
    the same values."""
    if fns is None:
        fns = library_fns(cfg, q, k_shard, v_shard, iq, ik_shard, iw, gate, pooled_shard, b0,
                          workspace)
    if gather_fn is None:
        gather_fn = _all_gather(group)
    cand = fns.select(kv_len)
    glob = fns.global_topk(gather_fn(cand["score"]), gather_fn(cand["id"]), kv_len)
    part = fns.attend(kv_len, glob["sel"], glob["nsel"])
    merged = fns.merge(gather_fn(part["out"]), gather_fn(part["lse"]))
    return {"out": merged["out"], "lse": merged["lse"], "sel": glob["sel"], "nsel": glob["nsel"]}
