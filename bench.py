#!/usr/bin/env python
"""Throughput of Qwen Sparse Attention (QSA) on B200 through the C ABI.

One step = one full QSA call over one batch of synthetic input: pooling,
indexer scoring, top-k selection, sparse attention and the sigmoid gate
(qsa_prefill for prefill workloads, qsa_decode for decode workloads).
The metric counts selected-KV tokens: the sum over query tokens of the number
of keys each query attends, |S(t)| = min(k, floor(n/B)) * B + n mod B.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference]

Under torchrun every rank runs its own shard: the workload's shapes with its own
seed (independent problems, no collective on the data path: weak scaling); the
reported value is all ranks' tokens over the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_attention_17_b200.workloads import (WORKLOADS, make_decode_inputs,  # noqa: E402
                                                      make_prefill_inputs, resolve_seqlens)

METRIC = "QSA selected-KV tokens/s (prefill, decode) + µs/decode step; % HBM/TC roofline"
UNIT = "selected-KV tokens/s"
DEFAULT_WORKLOAD = "prefill_bf16_t8192"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ helpers
def selected_tokens(n: int, B: int, k: int) -> int:
    nc = n // B
    return min(k, nc) * B + n % B


def workload_units(w):
    """Selected-KV tokens per step and the list of visible lengths."""
    if w.kind == "prefill":
        seqlens, _ = resolve_seqlens(w)
        ns = [p + 1 for L in seqlens for p in range(L)]
    else:
        ns = [w.kv_len - w.n_q + 1 + i for _ in range(w.batch) for i in range(w.n_q)]
    return sum(selected_tokens(n, w.block_size, w.topk) for n in ns), ns


def code_sha(text: str) -> str:
    """sha256 of C/CUDA source with its comments, trailing spaces and blank
    lines removed: the code a counter capture describes (a comment edit does
    not void it)."""
    import hashlib
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the kernel code as it is now (code_sha prefix match); else None."""
    src = os.path.join(ROOT, "block_sparse_attention_17_b200", "csrc", kernel_file)
    table = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not (os.path.exists(src) and os.path.exists(table)):
        return None
    sha = code_sha(open(src).read())
    for line in open(table):
        parts = line.split()
        if len(parts) == 4 and not line.startswith("#") and parts[0] == kernel_file \
                and sha.startswith(parts[1]) and parts[2] == workload:
            return int(parts[3])
    return None


def rank_workload(w, rank: int):
    """The shard rank ``rank`` processes: the workload's shapes, its own seed.

    Rank 0 keeps the workload's seed, so a 1-GPU run and rank 0 of an N-GPU run
    draw the same inputs; ragged workloads draw their lengths per rank too.
    """
    return w if rank == 0 else w.with_(seed=w.seed + 7919 * rank)


def reduce_over_ranks(dist, units: float, ms: float, device):
    """(sum of ``units`` over ranks, max of ``ms`` over ranks).

    Two collectives, taken in the same order by every rank; ``device`` is the
    device the process group's backend reduces on (cuda for NCCL, cpu for gloo).
    """
    if dist is None:
        return units, ms
    import torch
    u = torch.tensor([float(units)], dtype=torch.float64, device=device)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(u.item()), float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def config_of(w, extra=None):
    c = {"workload": w.name, "kind": w.kind, "dtype": w.dtype, "Hq": w.num_q_heads,
         "Hkv": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
         "budget": w.budget, "idx_heads": w.idx_heads, "idx_dim": w.idx_dim, "seed": w.seed}
    if w.kind == "prefill":
        seqlens, _ = resolve_seqlens(w)
        c.update(seqlens=list(seqlens), global_batch=len(seqlens), seq_len=max(seqlens))
    else:
        c.update(batch=w.batch, kv_len=w.kv_len, n_q=w.n_q, global_batch=w.batch,
                 seq_len=w.kv_len)
    if extra:
        c.update(extra)
    return c


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during timing."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.device_id = device_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.device_id:
                cmd += ["-i", self.device_id]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ cpu baseline
def oracle_sample(w, inp, budget_s: float, max_queries=None, seed=0):
    """Time the fp64 oracle, as it stands, on an evenly spread sample of the
    workload's queries until about budget_s seconds of CPU work are done.
    Returns (selected tokens processed, seconds, queries, cores)."""
    from threadpoolctl import threadpool_limits
    from oracle import qsa_oracle as O
    rng = np.random.default_rng(seed)
    if w.kind == "prefill":
        T = int(inp["cu_seqlens"][-1])
        order = rng.permutation(T)
    else:
        pairs = [(b, i) for b in range(w.batch) for i in range(w.n_q)]
        order = [pairs[j] for j in rng.permutation(len(pairs))]
    done, toks = 0, 0
    chunk = 16
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        for c0 in range(0, len(order), chunk):
            items = order[c0:c0 + chunk]
            if w.kind == "prefill":
                res = O.qsa_prefill(w, inp, queries=[int(x) for x in items])["queries"]
            else:
                res = O.qsa_decode(w, inp, pairs=[tuple(x) for x in items])["queries"]
            toks += sum(r.tokens for r in res.values())
            done += len(items)
            el = time.perf_counter() - t0
            if el >= budget_s or (max_queries and done >= max_queries):
                break
        el = time.perf_counter() - t0
    return toks, el, done, 1


# ------------------------------------------------------------------ ours
def run_ours(args, w, rank, world, dist):
    import torch
    import block_sparse_attention_17_b200 as qsa
    from block_sparse_attention_17_b200 import _lib

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = _lib.lib()
    peaks, peak_kind = load_peaks()
    cfg = qsa.QSAConfig.from_workload(w)
    dt = cfg.dtype
    units, ns = workload_units(w)

    t_gen = time.perf_counter()
    inp = make_prefill_inputs(w) if w.kind == "prefill" else make_decode_inputs(w)
    t_gen = time.perf_counter() - t_gen
    host = {}
    for name, arr in inp.items():
        if not isinstance(arr, np.ndarray) or name == "seqlens":
            continue
        t = torch.from_numpy(np.ascontiguousarray(arr))
        if arr.dtype == np.float32 and name != "iw":
            t = t.to(dt)
        host[name] = t.pin_memory()
    d = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    torch.cuda.synchronize()

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ev_stage = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for e in ev_stage:          # torch creates the CUDA event on its first record
        e.record(stream)
    torch.cuda.synchronize()
    arr_t = ctypes_voidp_array([e.cuda_event for e in ev_stage])
    assert all(e.cuda_event for e in ev_stage)

    if w.kind == "prefill":
        T = host["q"].shape[0]
        out = torch.empty_like(d["q"])
        ws = torch.empty(qsa.prefill_workspace_size(cfg, len(inp["seqlens"]), T,
                                                    inp["max_seqlen"]), dtype=torch.uint8,
                         device=dev)

        def step(dd=d, o=out):
            qsa.prefill(cfg, dd["q"], dd["k"], dd["v"], dd["iq"], dd["ik"], dd["iw"], dd["gate"],
                        dd["cu_seqlens"], inp["max_seqlen"], out=o, workspace=ws)
        flops = 4.0 * w.head_dim * w.num_q_heads * units
        alg = {"bound": "tensor", "work": flops, "peak_key": "bf16_tflops", "unit": "TFLOP/s"}
        in_names = ["q", "k", "v", "iq", "ik", "iw", "gate", "cu_seqlens"]
    else:
        kv = d["kv_len"]
        pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
        out = torch.empty_like(d["q"])
        ws = torch.empty(qsa.decode_workspace_size(cfg, w.batch, w.n_q, inp["cap"]),
                         dtype=torch.uint8, device=dev)
        sel = torch.empty(w.batch, w.n_q, w.topk + 1, dtype=torch.int32, device=dev)
        nsel = torch.empty(w.batch, w.n_q, dtype=torch.int32, device=dev)

        if args.kv != "bf16":
            # the same rows as e4m3 with one fp32 scale per (token, KV head) row,
            # optionally stored in the Walsh-Hadamard-rotated basis
            rotated = args.kv == "fp8-rotated"
            Dh = w.head_dim
            Hm = torch.ones(1, 1, dtype=torch.float64)
            while Hm.shape[0] < Dh:
                Hm = torch.cat([torch.cat([Hm, Hm], 1), torch.cat([Hm, -Hm], 1)], 0)
            Hm = (Hm / Dh ** 0.5).to(dev, torch.float32)
            fp8 = {}
            for n in ("k_cache", "v_cache"):
                x = d[n].float()
                if rotated:
                    x = x @ Hm
                scale = (x.abs().amax(-1) / 448.0).clamp_min(1e-30)
                codes = (x / scale[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
                fp8[n] = (codes.contiguous(), scale.contiguous())
                del x

            def step(dd=d, o=out):
                qsa.decode_fp8(cfg, dd["q"], fp8["k_cache"][0], fp8["k_cache"][1],
                               fp8["v_cache"][0], fp8["v_cache"][1], dd["iq"], dd["ik_cache"],
                               dd["iw"], dd["gate"], pooled, dd["kv_len"], rotated=rotated, out=o,
                               sel=sel, nsel=nsel, workspace=ws)
        elif args.paged:
            # the same rows scattered into a page pool (page = one block) under a
            # seeded random block table
            B = w.block_size
            max_blocks = inp["cap"] // B
            perm = np.random.default_rng(w.seed + 1).permutation(w.batch * max_blocks)
            table = torch.from_numpy(perm.reshape(w.batch, max_blocks).astype(np.int32)).to(dev)
            idx = table.reshape(-1).long()

            def scatter(cache):
                pool = torch.empty((w.batch * max_blocks, B, *cache.shape[2:]), dtype=cache.dtype,
                                   device=dev)
                pool[idx] = cache.reshape(w.batch * max_blocks, B, *cache.shape[2:])
                return pool
            pages = {n: scatter(d[n]) for n in ("k_cache", "v_cache", "ik_cache")}
            pooled = qsa.pool_build_paged(cfg, pages["ik_cache"], (kv - w.n_q).to(torch.int32),
                                          table)

            def step(dd=d, o=out):
                qsa.decode_paged(cfg, dd["q"], pages["k_cache"], pages["v_cache"], dd["iq"],
                                 pages["ik_cache"], dd["iw"], dd["gate"], pooled, dd["kv_len"],
                                 table, out=o, sel=sel, nsel=nsel, workspace=ws)
        else:
            def step(dd=d, o=out):
                qsa.decode(cfg, dd["q"], dd["k_cache"], dd["v_cache"], dd["iq"], dd["ik_cache"],
                           dd["iw"], dd["gate"], pooled, dd["kv_len"], out=o, sel=sel, nsel=nsel,
                           workspace=ws)
        step()
        torch.cuda.synchronize()
        kv_bytes = decode_selected_kv_bytes(w, sel.cpu().numpy(), nsel.cpu().numpy(),
                                            inp["kv_len"], args.kv)
        esz = 2 if w.dtype == "bf16" else 4
        io = w.batch * w.n_q * (2 * w.num_q_heads * w.head_dim * esz)   # q + out
        io += w.batch * w.n_q * w.num_q_heads * w.head_dim * esz         # gate
        io += decode_selection_bytes(w, inp["kv_len"])
        alg = {"bound": "hbm", "work": kv_bytes + io, "peak_key": "hbm_gbs", "unit": "GB/s"}
        in_names = ["q", "iq", "iw", "gate", "kv_len"]   # one decode step's new inputs

    # warm-up (eager)
    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    def timed(run_once, stages):
        """Time K steps, each bracketed by CUDA events on the launching stream,
        with the L2 flush outside the events; returns per-step ms and, with
        stages, the attention-stage ms read from the library's stage events."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        attn = []
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            run_once()
            ends[i].record(stream)
            torch.cuda.synchronize()       # read this step's stage events before reuse
            if stages:
                # prefill: the attention kernel; decode: the whole step (the
                # selection runs inside the decode kernel)
                attn.append(ev_stage[0 if w.kind == "decode" else 1].elapsed_time(ev_stage[2]))
        return [starts[i].elapsed_time(ends[i]) for i in range(args.steps)], attn

    # one step captured as a CUDA graph (the library makes no host sync, reads
    # no device memory on the host and allocates nothing, so it captures whole);
    # captured without stage events, so the kernels chain by programmatic
    # dependent launch as in a user's graph
    graph = None
    if not args.eager:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize()
        for _ in range(2):
            flush.zero_()
            graph.replay()
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    dev_id = ""
    try:
        dev_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid).replace("GPU-", "")
    except Exception:
        dev_id = str(local)
    clocks = ClockSampler(dev_id)
    clocks.start()
    n0 = lib.qsa_kernel_launch_count()
    torch.cuda.synchronize()
    # eager steps with stage events: the attention kernel's own duration
    lib.qsa_set_stage_events(arr_t, 3)
    eager_ms, stage_attn = timed(step, True)
    lib.qsa_set_stage_events(None, 0)
    launches = lib.qsa_kernel_launch_count() - n0
    if graph is not None:
        step_ms, _ = timed(graph.replay, False)
    else:
        step_ms = eager_ms
    torch.cuda.synchronize()
    clk = clocks.stop()
    total_ms = float(sum(step_ms))
    job_units, total_ms = reduce_over_ranks(dist, units, total_ms, dev)
    if dist is not None:
        dist.barrier()
    value = job_units * args.steps / (total_ms / 1e3)

    # roofline of the dominant kernel: attention (+ combine for decode)
    attn_ms = float(np.mean(stage_attn))
    peak = float(peaks.get(alg["peak_key"], FALLBACK_PEAKS[alg["peak_key"]]))
    if alg["bound"] == "tensor":
        achieved = alg["work"] / (attn_ms / 1e3) / 1e12
    else:
        achieved = alg["work"] / (attn_ms / 1e3) / 1e9
    kfile = ("qsa_decode_attn.cu" if w.kind == "decode" else
             "qsa_attn_tc.cu" if (w.dtype == "bf16" and w.head_dim == 128) else "qsa_attn_simt.cu")
    roof = {"bound": alg["bound"], "achieved": round(achieved, 3), "peak": peak,
            "unit": alg["unit"], "frac": round(achieved / peak, 5),
            "traffic": recorded_traffic(kfile, w.name),
            "kernel": ("qsa decode step (selection + attention + merge, one kernel)"
                       if w.kind == "decode" else "qsa attention"),
            "kernel_ms": round(attn_ms, 5), "peak_source": f"{peak_kind} ({alg['peak_key']})",
            "algorithmic_per_launch": alg["work"]}

    # end to end: pinned host inputs -> device, the call, result -> host
    e2e = None
    if not args.no_e2e:
        out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h2d = sum(host[n].numel() * host[n].element_size() for n in in_names)
        d2h = out_host.numel() * out_host.element_size()
        e_st = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        e_en = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.steps + 1):
            flush.zero_()
            if i > 0:
                e_st[i - 1].record(stream)
            for n in in_names:
                d[n].copy_(host[n], non_blocking=True)
            step()
            out_host.copy_(out, non_blocking=True)
            if i > 0:
                e_en[i - 1].record(stream)
        torch.cuda.synchronize()
        e2e_ms = float(sum(e_st[i].elapsed_time(e_en[i]) for i in range(args.steps)))
        _, e2e_ms = reduce_over_ranks(dist, units, e2e_ms, dev)
        e2e = {"value": job_units * args.steps / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms / args.steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        toks, secs, nq, cores = oracle_sample(w, inp, args.cpu_seconds)
        cpu = {"value": toks / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{nq} query tokens drawn at random from this workload, fp64 numpy "
                         f"oracle, {secs:.1f} s"}

    extra = {"l2": "flushed before every timed step (256 MiB write, outside the events)",
             "timing": ("CUDA-graph replay of one library call per step" if graph is not None
                        else "eager library call per step"),
             "eager_ms_per_step": float(np.mean(eager_ms)),
             "median_ms_per_step": float(np.median(step_ms)),
             "eager_median_ms_per_step": float(np.median(eager_ms)),
             "kv_layout": "paged (one block per page)" if (args.paged and w.kind == "decode")
             else "contiguous",
             "kv_format": args.kv if w.kind == "decode" else "bf16",
             "selected_kv_tokens_per_step": units, "job_selected_kv_tokens_per_step": job_units,
             "shards": "one per rank: the workload's shapes, seed + 7919 * rank",
             "input_gen_s": round(t_gen, 2)}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded numpy draws, shapes of the workload)",
            "config": config_of(w, extra), "parallelism": f"dp{world}",
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(launches), "clocks": clk,
            "impl": "ours"}
    if w.kind == "decode":
        line["us_per_decode_step"] = total_ms / args.steps * 1e3
    return line


def ctypes_voidp_array(ptrs):
    import ctypes
    arr = (ctypes.c_void_p * len(ptrs))(*[ctypes.c_void_p(p) for p in ptrs])
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))


def decode_selection_bytes(w, kv_len):
    """Bytes the selection of one decode step must move: the pooled keys of every
    complete block (fp32, read once), the indexer rows of the blocks the step
    completes (read) and their pooled rows (written), the queries' indexer q and
    weights, and the selection lists written."""
    esz = 2 if w.dtype == "bf16" else 4
    total = 0
    for kv in np.asarray(kv_len).tolist():
        total += (kv // w.block_size) * w.idx_dim * 4
        new_blocks = kv // w.block_size - (kv - w.n_q) // w.block_size
        total += new_blocks * w.block_size * w.idx_dim * esz + new_blocks * w.idx_dim * 4
    total += w.batch * w.n_q * w.idx_heads * (w.idx_dim * esz + 4)
    total += w.batch * w.n_q * (w.topk + 2) * 4
    return total


def decode_selected_kv_bytes(w, sel, nsel, kv_len, kv_format="bf16"):
    """Distinct visible K/V bytes the step must read: per sequence, the union
    over its new queries of their selected tokens, times Hkv heads, K and V
    (fp8 caches: one byte per element plus a 4-byte scale per row)."""
    esz = 2 if w.dtype == "bf16" else 4
    B = w.block_size
    total = 0
    for b in range(w.batch):
        toks = set()
        for i in range(w.n_q):
            n = int(kv_len[b]) - w.n_q + 1 + i
            nc = n // B
            for e in range(int(nsel[b, i])):
                blk = int(sel[b, i, e])
                hi = min((blk + 1) * B, n) if blk == nc else (blk + 1) * B
                toks.update(range(blk * B, hi))
        total += len(toks)
    if kv_format != "bf16":
        return total * w.num_kv_heads * (w.head_dim + 4) * 2
    return total * w.num_kv_heads * w.head_dim * 2 * esz


# ------------------------------------------------------------- reference arm
def run_reference(args, w):
    """The fp64 oracle, as it stands, on the host cores: each step is a bounded
    random sample of the workload's queries."""
    inp = make_prefill_inputs(w) if w.kind == "prefill" else make_decode_inputs(w)
    per_step_s = args.ref_step_seconds
    tot_tok, tot_s, tot_q = 0, 0.0, 0
    for i in range(args.warmup + args.steps):
        toks, secs, nq, cores = oracle_sample(w, inp, per_step_s, seed=1000 + i)
        if i >= args.warmup:
            tot_tok += toks
            tot_s += secs
            tot_q += nq
    value = tot_tok / tot_s
    sample = (f"{tot_q} query tokens over {args.steps} steps (~{per_step_s:.1f} s each), drawn at "
              f"random from this workload, fp64 numpy oracle, 1 thread")
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy draws, shapes of the workload)",
            "config": config_of(w), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager calls only (no CUDA graph)")
    ap.add_argument("--paged", action="store_true",
                    help="decode workloads: run qsa_decode_paged over a page pool")
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8", "fp8-rotated"],
                    help="decode workloads: K/V cache format (fp8: qsa_decode_fp8)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=2.0)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    w = rank_workload(WORKLOADS[args.workload], rank)

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, w)))
        return 0

    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    try:
        line = run_ours(args, w, rank, world, dist)
        if rank == 0:
            print(json.dumps(line))
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
