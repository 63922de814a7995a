#!/usr/bin/env python
"""Throughput of Qwen Sparse Attention (QSA) on B200 through the C ABI.

One step = one full QSA call over one batch of synthetic input: pooling,
indexer scoring, top-k selection, sparse attention and the sigmoid gate
(qsa_prefill for prefill workloads, qsa_decode for decode workloads).
The metric counts selected-KV tokens: the sum over query tokens of the number
of keys each query attends, |S(t)| = min(k, floor(n/B)) * B + n mod B.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--decode NAME,NAME | none] [--impl ours|reference]

The JSON line's headline (value, e2e, roofline, cpu_baseline) is the prefill
workload (default: the ragged 4-sequence prefill, the largest one-GPU
workload); the same line carries a "decode" object per decode workload (default:
the 32-sequence decode and the 4-sequence MTP verification), each with its
microseconds per decode step, roofline, end-to-end figure, CPU baseline and
selection agreement with the fp64 oracle.

Under torchrun every rank runs its own shard: the workload's shapes with its own
seed (independent problems, no collective on the data path: weak scaling); the
reported value is all ranks' tokens over the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import json
import multiprocessing as mp
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
DEFAULT_WORKLOAD = "ragged_prefill_bf16_4seq"
DEFAULT_DECODE = "decode_bf16_b32_kv32768,mtp_verify_bf16_b4_kv262144"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
L2_NOTE = "GPU arm: L2 flushed before every timed step (256 MiB write, outside the events)"
TC_ROWS, TC_TILES, TC_KEYS = 128, 2, 128   # the tensor-core prefill kernel's tile shape


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
    if kernel_file is None:
        return None
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


def config_of(w, world=1):
    """The workload as the JSON line names it (identical in both arms)."""
    c = {"workload": w.name, "kind": w.kind, "dtype": w.dtype, "Hq": w.num_q_heads,
         "Hkv": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
         "budget": w.budget, "idx_heads": w.idx_heads, "idx_dim": w.idx_dim, "seed": w.seed}
    if w.kind == "prefill":
        seqlens, _ = resolve_seqlens(w)
        c.update(seqlens=list(seqlens), global_batch=len(seqlens), seq_len=max(seqlens))
    else:
        c.update(batch=w.batch, kv_len=w.kv_len, n_q=w.n_q, global_batch=w.batch,
                 seq_len=w.kv_len)
    c.update(l2=L2_NOTE, parallelism=f"dp{world}")
    return c


def host_cores() -> int:
    """CPU cores this process may use: its affinity mask, capped by a cgroup
    CPU quota when one is set."""
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 1
    try:
        with open("/sys/fs/cgroup/cpu.max") as f:
            quota, period = f.read().split()[:2]
        if quota != "max":
            n = min(n, max(1, int(int(quota) // int(period))))
    except Exception:
        pass
    return max(1, n)


def make_inputs(w):
    return make_prefill_inputs(w) if w.kind == "prefill" else make_decode_inputs(w)


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
# The fp64 oracle, as it stands, timed on the host cores. Worker processes are
# forked before this process makes its first CUDA call (a fork after it is not
# safe); they inherit the generated inputs through _CPU_INPUTS.
_CPU_INPUTS = {}


def _cpu_worker_init():
    from threadpoolctl import threadpool_limits
    global _TP_LIMIT
    _TP_LIMIT = threadpool_limits(limits=1)


def _oracle_items(args):
    """Oracle results for a list of items (query tokens or (sequence, query)
    pairs) of workload ``name``: (selected tokens, {item: (selected blocks,
    scores)})."""
    from oracle import qsa_oracle as O
    name, items = args
    w, inp = _CPU_INPUTS[name]
    if w.kind == "prefill":
        res = O.qsa_prefill(w, inp, queries=[int(x) for x in items])["queries"]
    else:
        res = O.qsa_decode(w, inp, pairs=[tuple(int(v) for v in x) for x in items])["queries"]
    toks = sum(r.tokens for r in res.values())
    return toks, {k: (r.selected.tolist(), r.scores) for k, r in res.items()}


def _all_items(w, inp, rng):
    if w.kind == "prefill":
        T = int(inp["cu_seqlens"][-1])
        return [int(x) for x in rng.permutation(T)]
    pairs = [(b, i) for b in range(w.batch) for i in range(w.n_q)]
    return [pairs[j] for j in rng.permutation(len(pairs))]


def cpu_leg(w, inp, seconds_all: float, seconds_one: float, cores: int, seed=0):
    """Times the oracle on one thread (about seconds_one) and on ``cores``
    processes (about seconds_all), each over a random sample of the workload's
    queries (decode: whole steps when they fit). Must run before the first
    CUDA call of this process. Returns the baseline dict and the oracle's
    selection and scores of every query it computed (for the agreement check)."""
    from threadpoolctl import threadpool_limits
    _CPU_INPUTS[w.name] = (w, inp)
    items = _all_items(w, inp, np.random.default_rng(seed))
    chunk = 8 if w.kind == "prefill" else 1
    oracle_sel = {}
    # one thread
    toks1, done1 = 0, 0
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        while True:
            for c0 in range(0, len(items), chunk):
                tk, sel = _oracle_items((w.name, items[c0:c0 + chunk]))
                toks1 += tk
                done1 += len(items[c0:c0 + chunk])
                oracle_sel.update(sel)
                if time.perf_counter() - t0 >= seconds_one:
                    break
            if time.perf_counter() - t0 >= seconds_one or w.kind == "prefill":
                break
        el1 = time.perf_counter() - t0
    rate1 = toks1 / el1
    # all cores: a sample sized from the one-thread rate
    per_item = el1 / max(1, done1)
    n_all = max(cores * chunk, int(seconds_all * cores / per_item))
    if w.kind == "prefill":
        sample = items[done1:done1 + n_all] if done1 + n_all <= len(items) else items[:n_all]
    else:
        reps = max(1, -(-n_all // len(items)))
        sample = items * reps
    tasks = [(w.name, sample[c0:c0 + chunk]) for c0 in range(0, len(sample), chunk)]
    ctx = mp.get_context("fork")
    with ctx.Pool(cores, initializer=_cpu_worker_init) as pool:
        pool.map(_oracle_items, tasks[:cores])          # warm the workers (imports)
        t0 = time.perf_counter()
        outs = pool.map(_oracle_items, tasks, chunksize=1)
        elA = time.perf_counter() - t0
    toksA = sum(o[0] for o in outs)
    for o in outs:
        oracle_sel.update(o[1])
    unit_q = "query tokens" if w.kind == "prefill" else "(sequence, new query) pairs"
    base = {"value": toksA / elA, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{len(sample)} {unit_q} drawn at random from this workload "
                      f"({'whole decode steps, ' if w.kind == 'decode' else ''}fp64 numpy oracle "
                      f"as it stands), {cores} processes of one thread each, {elA:.1f} s wall",
            "one_thread": {"value": rate1, "unit": UNIT, "cores": 1,
                           "sample": f"{done1} {unit_q}, {el1:.1f} s"}}
    if w.kind == "decode":
        steps_all = len(sample) / len(items)
        base["us_per_decode_step"] = elA / steps_all * 1e6
        base["one_thread"]["us_per_decode_step"] = el1 / (done1 / len(items)) * 1e6
    del _CPU_INPUTS[w.name]
    raw = {"tokens": toksA, "seconds": elA, "items": len(sample)}
    return base, oracle_sel, raw


def selection_agreement(w, oracle_sel, gpu_sel, gpu_nsel, index_of):
    """Selection of the GPU path against the oracle's on the queries the CPU
    leg computed: exact matches, near-ties (differences only among blocks whose
    oracle scores lie within 1e-5 * max|s| of the k-th score, the tolerance
    the selection contract allows), unexcused mismatches, and mean Jaccard."""
    k = w.topk
    exact = ties = bad = 0
    jac = []
    for key, (osel, scores) in oracle_sel.items():
        ix = index_of(key)
        m = len(osel)
        g = [int(x) for x in gpu_sel[ix][:m]] if int(gpu_nsel[ix]) >= m else []
        a, b = set(int(x) for x in osel), set(g)
        jac.append(len(a & b) / len(a | b) if (a | b) else 1.0)
        if a == b and len(g) == m:
            exact += 1
            continue
        s = np.asarray(scores, np.float64)
        diff = a ^ b
        if len(g) != m or len(b) != m or any(j < 0 or j >= len(s) for j in diff):
            bad += 1
            continue
        kth = np.sort(s)[::-1][min(k, len(s)) - 1]
        tol = 1e-5 * max(float(np.abs(s).max()), 1e-300)
        if all(abs(s[j] - kth) <= tol for j in diff):
            ties += 1
        else:
            bad += 1
    return {"queries": len(oracle_sel), "exact": exact, "near_ties_excused": ties,
            "mismatches": bad, "mean_jaccard": float(np.mean(jac)) if jac else None}


# ------------------------------------------------------------------ ours
def prefill_executed_flop(w, inp, sel, nsel):
    """MMA flop the tensor-core prefill kernel executes: per (CTA, KV head),
    the 128-key steps over the union of its 2 x (128 / G) queries' selected
    and tail blocks, times 128 rows per occupied tile, QK^T and PV."""
    G = w.num_q_heads // w.num_kv_heads
    Qt = TC_ROWS // G
    kNh = TC_KEYS // w.block_size
    cu = np.asarray(inp["cu_seqlens"], np.int64)
    total = 0
    for b in range(len(cu) - 1):
        s0, L = int(cu[b]), int(cu[b + 1] - cu[b])
        for q0 in range(0, L, TC_TILES * Qt):
            nq = min(TC_TILES * Qt, L - q0)
            rows = sel[s0 + q0:s0 + q0 + nq]
            cnt = nsel[s0 + q0:s0 + q0 + nq]
            mask = np.arange(rows.shape[1])[None, :] < cnt[:, None]
            n_union = len(np.unique(rows[mask]))
            n_iter = -(-n_union // kNh)
            nt = 2 if nq > Qt else 1
            total += nt * n_iter
    return float(total) * w.num_kv_heads * TC_ROWS * TC_KEYS * w.head_dim * 4


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


def ctypes_voidp_array(ptrs):
    import ctypes
    arr = (ctypes.c_void_p * len(ptrs))(*[ctypes.c_void_p(p) for p in ptrs])
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))


def gpu_leg(args, w, inp, steps, warmup, dist, dev, kv_format="bf16", paged=False):
    """Times one workload on this rank's GPU. Returns a dict of per-step times
    (graph replay and eager), the dominant kernel's event-timed duration, the
    algorithmic work, the end-to-end time, clocks, launches and the selection
    of one call (for the agreement check)."""
    import torch
    import block_sparse_attention_17_b200 as qsa
    from block_sparse_attention_17_b200 import _lib

    lib = _lib.lib()
    cfg = qsa.QSAConfig.from_workload(w)
    dt = cfg.dtype
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
    res = {}

    if w.kind == "prefill":
        T = host["q"].shape[0]
        out = torch.empty_like(d["q"])
        ws = torch.empty(qsa.prefill_workspace_size(cfg, len(inp["seqlens"]), T,
                                                    inp["max_seqlen"]), dtype=torch.uint8,
                         device=dev)

        def step(dd=d, o=out):
            qsa.prefill(cfg, dd["q"], dd["k"], dd["v"], dd["iq"], dd["ik"], dd["iw"], dd["gate"],
                        dd["cu_seqlens"], inp["max_seqlen"], out=o, workspace=ws)
        r = qsa.prefill(cfg, d["q"], d["k"], d["v"], d["iq"], d["ik"], d["iw"], d["gate"],
                        d["cu_seqlens"], inp["max_seqlen"], want_sel=True)
        torch.cuda.synchronize()
        res["sel"] = r["sel"].cpu().numpy()
        res["nsel"] = r["nsel"].cpu().numpy()
        del r
        res["alg"] = {"bound": "tensor", "peak_key": "bf16_tflops", "unit": "TFLOP/s",
                      "work": 4.0 * w.head_dim * w.num_q_heads * workload_units(w)[0]}
        in_names = ["q", "k", "v", "iq", "ik", "iw", "gate", "cu_seqlens"]
        append = None
    else:
        kv = d["kv_len"]
        pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
        out = torch.empty_like(d["q"])
        ws = torch.empty(qsa.decode_workspace_size(cfg, w.batch, w.n_q, inp["cap"]),
                         dtype=torch.uint8, device=dev)
        sel = torch.empty(w.batch, w.n_q, w.topk + 1, dtype=torch.int32, device=dev)
        nsel = torch.empty(w.batch, w.n_q, dtype=torch.int32, device=dev)
        if kv_format != "bf16":
            # the same rows as e4m3 with one fp32 scale per (token, KV head) row,
            # optionally stored in the Walsh-Hadamard-rotated basis
            rotated = kv_format == "fp8-rotated"
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
        elif paged:
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
        res["sel"] = sel.cpu().numpy()
        res["nsel"] = nsel.cpu().numpy()
        kv_bytes = decode_selected_kv_bytes(w, res["sel"], res["nsel"], inp["kv_len"], kv_format)
        esz = 2 if w.dtype == "bf16" else 4
        io = w.batch * w.n_q * (2 * w.num_q_heads * w.head_dim * esz)   # q + out
        io += w.batch * w.n_q * w.num_q_heads * w.head_dim * esz         # gate
        io += decode_selection_bytes(w, inp["kv_len"])
        res["alg"] = {"bound": "hbm", "peak_key": "hbm_gbs", "unit": "GB/s",
                      "work": kv_bytes + io, "selected_kv_bytes": kv_bytes}
        # one decode step's new inputs: the query-side tensors and the n_q new
        # rows of the K, V and indexer-key caches (appended at kv_len - n_q)
        in_names = ["q", "iq", "iw", "gate", "kv_len"]
        kv0 = int(inp["kv_len"][0])
        same_len = bool(np.all(np.asarray(inp["kv_len"]) == kv0)) and kv_format == "bf16" \
            and not paged
        append = None
        if same_len:
            rows = slice(kv0 - w.n_q, kv0)
            append = [(d[n], host[n][:, rows].contiguous().pin_memory(), rows)
                      for n in ("k_cache", "v_cache", "ik_cache")]

    # warm-up (eager)
    for _ in range(max(warmup, 0)):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    # the visited-keys debug counter over one more eager step, outside the timed
    # region: the (query, head, key) triples the attention kernels attended over
    ctr = torch.zeros(1, dtype=torch.int64, device=dev)
    qsa.set_keys_visited(ctr)
    try:
        step()
    finally:
        qsa.set_keys_visited(None)
    torch.cuda.synchronize()
    res["keys_visited"] = int(ctr.item())

    def timed(run_once, stages):
        """Time the steps, each bracketed by CUDA events on the launching
        stream, with the L2 flush outside the events; returns per-step ms and,
        with stages, the dominant kernel's ms read from the library's stage
        events (prefill: the attention kernel; decode: the whole step, which
        is one kernel)."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        attn = []
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            run_once()
            ends[i].record(stream)
            torch.cuda.synchronize()       # read this step's stage events before reuse
            if stages:
                attn.append(ev_stage[0 if w.kind == "decode" else 1].elapsed_time(ev_stage[2]))
        return [starts[i].elapsed_time(ends[i]) for i in range(steps)], attn

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
        dev_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid).replace("GPU-", "")
    except Exception:
        dev_id = str(dev.index or 0)
    clocks = ClockSampler(dev_id)
    clocks.start()
    n0 = lib.qsa_kernel_launch_count()
    torch.cuda.synchronize()
    lib.qsa_set_stage_events(arr_t, 3)
    eager_ms, stage_ms = timed(step, True)
    lib.qsa_set_stage_events(None, 0)
    launches = lib.qsa_kernel_launch_count() - n0
    if graph is not None:
        step_ms, _ = timed(graph.replay, False)
    else:
        step_ms = eager_ms
    torch.cuda.synchronize()
    res["clocks"] = clocks.stop()
    res.update(step_ms=step_ms, eager_ms=eager_ms, stage_ms=stage_ms, launches=int(launches),
               graph=graph is not None)

    # end to end through the public API: pinned host inputs -> device, the
    # call, result -> host, all inside the timed region. A decode step's inputs
    # (the query-side tensors and the new K, V and indexer-key rows) travel as
    # one packed pinned buffer, one copy; qsa_append writes the new rows into the
    # caches (and pools the block they complete) and qsa_decode runs the step.
    if not args.no_e2e and w.kind == "decode" and append is not None:
        out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        pieces = [(n, host[n]) for n in in_names] + \
                 [(n, hsrc) for n, (_, hsrc, _) in zip(("k_new", "v_new", "ik_new"), append)]
        offs, total = {}, 0
        for n, t in pieces:
            offs[n] = total
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        pack_host = torch.empty(total, dtype=torch.uint8, pin_memory=True)
        for n, t in pieces:
            nb = t.numel() * t.element_size()
            pack_host[offs[n]:offs[n] + nb].copy_(t.contiguous().view(-1).view(torch.uint8))
        pack_dev = torch.empty(total, dtype=torch.uint8, device=dev)
        dv = {n: pack_dev[offs[n]:offs[n] + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
              for n, t in pieces}
        kv_dev = dv["kv_len"]
        e_st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        e_en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps + 1):
            flush.zero_()
            if i > 0:
                e_st[i - 1].record(stream)
            pack_dev.copy_(pack_host, non_blocking=True)
            qsa.append(cfg, dv["ik_new"], d["ik_cache"], pooled, kv_dev, k_new=dv["k_new"],
                       v_new=dv["v_new"], k_cache=d["k_cache"], v_cache=d["v_cache"])
            qsa.decode(cfg, dv["q"], d["k_cache"], d["v_cache"], dv["iq"], d["ik_cache"], dv["iw"],
                       dv["gate"], pooled, kv_dev, out=out, sel=sel, nsel=nsel, workspace=ws)
            out_host.copy_(out, non_blocking=True)
            if i > 0:
                e_en[i - 1].record(stream)
        torch.cuda.synchronize()
        res["e2e_ms"] = float(sum(e_st[i].elapsed_time(e_en[i]) for i in range(steps)))
        res["h2d"], res["d2h"] = int(total), int(out_host.numel() * out_host.element_size())
        res["e2e_note"] = ("one packed pinned copy of the step's inputs, qsa_append of the new "
                           "K/V/indexer rows, qsa_decode, the output copied back")
    elif not args.no_e2e:
        out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h2d = sum(host[n].numel() * host[n].element_size() for n in in_names)
        if append:
            h2d += sum(hsrc.numel() * hsrc.element_size() for _, hsrc, _ in append)
        d2h = out_host.numel() * out_host.element_size()
        e_st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        e_en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps + 1):
            flush.zero_()
            if i > 0:
                e_st[i - 1].record(stream)
            for n in in_names:
                d[n].copy_(host[n], non_blocking=True)
            if append:
                for dcache, hsrc, rows in append:
                    dcache[:, rows].copy_(hsrc, non_blocking=True)
            step()
            out_host.copy_(out, non_blocking=True)
            if i > 0:
                e_en[i - 1].record(stream)
        torch.cuda.synchronize()
        res["e2e_ms"] = float(sum(e_st[i].elapsed_time(e_en[i]) for i in range(steps)))
        res["h2d"], res["d2h"] = int(h2d), int(d2h)
    if graph is not None:
        del graph
    del d, host, flush, ws
    torch.cuda.empty_cache()
    return res


def assemble(w, r, units, steps, dist, dev, peaks, peak_kind, kernel_file, kernel_name,
             cpu=None, agreement=None, extra_roof=None):
    """The per-workload JSON fields from a gpu_leg result."""
    total_ms = float(sum(r["step_ms"]))
    job_units, total_ms = reduce_over_ranks(dist, units, total_ms, dev)
    value = job_units * steps / (total_ms / 1e3)
    kern_ms = float(np.mean(r["stage_ms"]))
    alg = r["alg"]
    peak = float(peaks.get(alg["peak_key"], FALLBACK_PEAKS[alg["peak_key"]]))
    scale = 1e12 if alg["bound"] == "tensor" else 1e9
    achieved = alg["work"] / (kern_ms / 1e3) / scale
    roof = {"bound": alg["bound"], "achieved": round(achieved, 3), "peak": peak,
            "unit": alg["unit"], "frac": round(achieved / peak, 5),
            "traffic": recorded_traffic(kernel_file, w.name),
            "kernel": kernel_name, "kernel_ms": round(kern_ms, 5),
            "peak_source": f"{peak_kind} ({alg['peak_key']})",
            "algorithmic_per_launch": alg["work"]}
    if extra_roof:
        roof.update(extra_roof)
    e2e = None
    if "e2e_ms" in r:
        _, e2e_ms = reduce_over_ranks(dist, units, r["e2e_ms"], dev)
        e2e = {"value": job_units * steps / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
               "ms_per_step": e2e_ms / steps}
        if "e2e_note" in r:
            e2e["calls"] = r["e2e_note"]
    timing = {"timing": ("CUDA-graph replay of one library call per step" if r["graph"]
                         else "eager library call per step"),
              "eager_ms_per_step": float(np.mean(r["eager_ms"])),
              "median_ms_per_step": float(np.median(r["step_ms"])),
              "eager_median_ms_per_step": float(np.median(r["eager_ms"])),
              "selected_kv_tokens_per_step": units, "job_selected_kv_tokens_per_step": job_units}
    ns = workload_units(w)[1]
    visited = {"counted": r["keys_visited"], "expected": w.num_q_heads * units,
               "dense": w.num_q_heads * int(sum(ns)),
               "note": "one step with qsa_set_keys_visited on: (query, head, key) triples "
                       "attended; expected = Hq * sum(min(k, nc) * B + tail), dense = Hq * "
                       "sum(visible tokens)"}
    return {"value": value, "ms_per_step": total_ms / steps, "roofline": roof, "e2e": e2e,
            "clocks": r["clocks"], "gpu_launches": r["launches"], "cpu_baseline": cpu,
            "selection_vs_oracle": agreement, "keys_visited": visited, "timing": timing}


def index_fn(w):
    return (lambda t: t) if w.kind == "prefill" else (lambda bi: (bi[0], bi[1]))


def run_ours(args, rank, world, dist):
    import torch
    local = int(os.environ.get("LOCAL_RANK", "0"))
    peaks, peak_kind = load_peaks()
    head_w = WORKLOADS[args.workload]
    if args.seqlens:   # a smaller case of the prefill workload (profiling captures)
        head_w = head_w.with_(seqlens=tuple(int(x) for x in args.seqlens.split(",")),
                              ragged_range=None)
    head_w = rank_workload(head_w, rank)
    dec_names = [] if args.decode in ("", "none") else [x for x in args.decode.split(",") if x]
    dec_ws = [rank_workload(WORKLOADS[n], rank) for n in dec_names]
    all_ws = [head_w] + dec_ws

    # inputs on the host, then the CPU legs (before this process's first CUDA
    # call: their worker processes are forked)
    gen_s, inputs = {}, {}
    for w in all_ws:
        t0 = time.perf_counter()
        inputs[w.name] = make_inputs(w)
        gen_s[w.name] = round(time.perf_counter() - t0, 2)
    cpu, oracle_sel = {}, {}
    do_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    cores = args.cpu_cores or host_cores()
    if do_cpu:
        for w in all_ws:
            cpu[w.name], oracle_sel[w.name], _ = cpu_leg(w, inputs[w.name], args.cpu_seconds,
                                                         args.cpu_seconds_one, cores)

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    tk = lambda w: "qsa_attn_tc.cu" if (w.dtype == "bf16" and w.head_dim == 128) \
        else "qsa_attn_simt.cu"

    # headline workload
    w = head_w
    units, _ = workload_units(w)
    r = gpu_leg(args, w, inputs[w.name], args.steps, args.warmup, dist, dev, paged=False)
    extra_roof = None
    if w.kind == "prefill" and w.dtype == "bf16" and w.head_dim == 128:
        ex = prefill_executed_flop(w, inputs[w.name], r["sel"], r["nsel"])
        kern_ms = float(np.mean(r["stage_ms"]))
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        extra_roof = {"executed_flop_per_launch": ex,
                      "executed_achieved": round(ex / (kern_ms / 1e3) / 1e12, 3),
                      "executed_frac": round(ex / (kern_ms / 1e3) / 1e12 / peak, 5),
                      "executed_over_algorithmic": round(ex / r["alg"]["work"], 4)}
    agree = (selection_agreement(w, oracle_sel[w.name], r["sel"], r["nsel"], index_fn(w))
             if w.name in oracle_sel else None)
    head = assemble(w, r, units, args.steps, dist, dev, peaks, peak_kind,
                    "qsa_decode_attn.cu" if w.kind == "decode" else tk(w),
                    "qsa decode step (one kernel)" if w.kind == "decode" else "qsa attention",
                    cpu.get(w.name), agree, extra_roof)
    del r

    decode_objs = {}
    for wd in dec_ws:
        units_d, _ = workload_units(wd)
        rd = gpu_leg(args, wd, inputs[wd.name], args.decode_steps, max(args.warmup, 10), dist,
                     dev, kv_format=args.kv, paged=args.paged)
        agree_d = (selection_agreement(wd, oracle_sel[wd.name], rd["sel"], rd["nsel"],
                                       index_fn(wd)) if wd.name in oracle_sel else None)
        # (the recorded DRAM counters are those of the contiguous bf16 caches)
        obj = assemble(wd, rd, units_d, args.decode_steps, dist, dev, peaks, peak_kind,
                       "qsa_decode_attn.cu" if args.kv == "bf16" and not args.paged else None,
                       "qsa decode step (selection + attention + merge, one kernel)",
                       cpu.get(wd.name), agree_d,
                       {"selected_kv_bytes": rd["alg"]["selected_kv_bytes"]})
        obj["us_per_decode_step"] = obj["ms_per_step"] * 1e3
        obj["median_us_per_decode_step"] = obj["timing"]["median_ms_per_step"] * 1e3
        obj["steps"] = args.decode_steps
        obj["config"] = config_of(wd, world)
        obj["config"]["kv_layout"] = "paged (one block per page)" if args.paged else "contiguous"
        obj["config"]["kv_format"] = args.kv
        obj["input_gen_s"] = gen_s[wd.name]
        decode_objs[wd.name] = obj
        del rd

    cfg = config_of(w, world)
    line = {"metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded numpy draws, shapes of the workload)",
            "config": cfg, "roofline": head["roofline"], "cpu_baseline": head["cpu_baseline"],
            "e2e": head["e2e"], "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
            "selection_vs_oracle": head["selection_vs_oracle"],
            "keys_visited": head["keys_visited"], "timing": head["timing"],
            "shards": "one per rank: the workload's shapes, seed + 7919 * rank",
            "input_gen_s": gen_s[w.name], "impl": "ours"}
    if decode_objs:
        line["decode"] = decode_objs
    return line


# ------------------------------------------------------------- reference arm
def run_reference(args):
    """The fp64 oracle, as it stands, on the host cores: each step is a bounded
    random sample of the workload's queries, spread over all cores."""
    w = WORKLOADS[args.workload]
    inp = make_inputs(w)
    cores = args.cpu_cores or host_cores()
    tot_tok, tot_s, tot_q = 0.0, 0.0, 0
    one = None
    for i in range(args.warmup + args.steps):
        # the all-core part of the leg is the step; its one-thread part sizes it
        base, _, raw = cpu_leg(w, inp, args.ref_step_seconds, 0.5, cores, seed=1000 + i)
        if i >= args.warmup:
            tot_tok += raw["tokens"]
            tot_s += raw["seconds"]
            tot_q += raw["items"]
            one = base["one_thread"]
    value = tot_tok / tot_s
    sample = (f"{tot_q} query tokens over {args.steps} steps (~{args.ref_step_seconds:.1f} s "
              f"each), drawn at random from this workload, fp64 numpy oracle, {cores} processes")
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy draws, shapes of the workload)",
            "config": config_of(w), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample, "one_thread": one},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--decode", default=DEFAULT_DECODE,
                    help="comma-separated decode workloads timed in the same run ('none': skip)")
    ap.add_argument("--decode-steps", type=int, default=100)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager calls only (no CUDA graph)")
    ap.add_argument("--paged", action="store_true",
                    help="decode workloads: run qsa_decode_paged over a page pool")
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8", "fp8-rotated"],
                    help="decode workloads: K/V cache format (fp8: qsa_decode_fp8)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="wall seconds of the all-core oracle sample per workload")
    ap.add_argument("--cpu-seconds-one", type=float, default=4.0,
                    help="seconds of the one-thread oracle sample per workload")
    ap.add_argument("--cpu-cores", type=int, default=0, help="0: every host core")
    ap.add_argument("--ref-step-seconds", type=float, default=2.0)
    ap.add_argument("--seqlens", default="",
                    help="prefill workload: comma-separated sequence lengths replacing the "
                         "workload's (a smaller case for profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    for n in ([] if args.decode in ("", "none") else args.decode.split(",")):
        if n and (n not in WORKLOADS or WORKLOADS[n].kind != "decode"):
            ap.error(f"--decode: {n} is not a decode workload")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)))
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
        line = run_ours(args, rank, world, dist)
        if rank == 0:
            print(json.dumps(line))
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
