"""Shared helpers of the parity tests: device upload of seeded inputs and the
comparison of CUDA results with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_attention_17_b200.workloads import round_to_bf16
from oracle import qsa_oracle as O

# tolerances on outputs (max abs error), by input dtype
TOL_OUT = {"f32": 1e-4, "bf16": 2e-2}
# pooled keys and scores are fp32 sums of a few hundred terms
TOL_POOLED_REL = 1e-6
TOL_SCORE_REL = 1e-5
NEAR_TIE_REL = 1e-5


def tdtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def round_like(x: np.ndarray, w) -> np.ndarray:
    """fp32 draws as the workload's dtype sees them (bf16 values for bf16
    workloads), so that the oracle and the GPU get the same numbers."""
    return round_to_bf16(x) if w.dtype == "bf16" else np.asarray(x, np.float32)


def upload(inp: dict, w, device="cuda") -> dict:
    dt = tdtype(w)
    dev = {}
    for name, arr in inp.items():
        if not isinstance(arr, np.ndarray):
            continue
        t = torch.from_numpy(np.ascontiguousarray(arr))
        if arr.dtype == np.float32 and name not in ("iw",):
            t = t.to(dt)
        dev[name] = t.to(device)
    return dev


def compare_selection(orc, gpu_sel_row, gpu_nsel, n, w):
    """Returns (ok, excused) for one query. gpu_sel_row: k+1 ints."""
    B, k = w.block_size, w.topk
    nc = n // B
    tail = n % B
    row = [int(x) for x in gpu_sel_row]
    m = min(k, nc)
    exp_n = m + (1 if tail else 0)
    if int(gpu_nsel) != exp_n:
        return False, False
    blocks = row[:m]
    if tail and row[m] != nc:
        return False, False
    if any(x != -1 for x in row[exp_n:]):
        return False, False
    if blocks != sorted(blocks) or len(set(blocks)) != m or any(b < 0 or b >= nc for b in blocks):
        return False, False
    if blocks == [int(x) for x in orc.selected]:
        return True, False
    if O.near_tie_excused(orc.scores, orc.selected, blocks, k, NEAR_TIE_REL):
        return True, True
    return False, False


def check_queries(results: dict, gpu: dict, index_of, w, check_lse=True):
    """Compare oracle QueryResults with GPU outputs.

    results: {key: QueryResult}; index_of(key) -> index tuple into the GPU
    tensors (token for prefill, (b, i) for decode). Returns a report dict and
    raises AssertionError on any unexcused mismatch."""
    tol = TOL_OUT[w.dtype]
    out = gpu["out"].float().cpu().numpy()
    lse = gpu["lse"].cpu().numpy() if gpu.get("lse") is not None else None
    sel = gpu["sel"].cpu().numpy()
    nsel = gpu["nsel"].cpu().numpy()
    excused, worst, worst_lse = [], 0.0, 0.0
    for key, r in results.items():
        ix = index_of(key)
        ok, exc = compare_selection(r, sel[ix], nsel[ix], r.n, w)
        assert ok, f"selection mismatch at {key}: gpu {sel[ix].tolist()} nsel {nsel[ix]} " \
                   f"oracle {r.selected.tolist()} (n={r.n})"
        if exc:
            excused.append(key)
            continue
        err = float(np.max(np.abs(out[ix].astype(np.float64) - r.out))) if r.out.size else 0.0
        worst = max(worst, err)
        assert err <= tol, f"output error {err} > {tol} at {key}"
        if check_lse and lse is not None:
            finite = np.isfinite(r.lse)
            assert np.array_equal(finite, np.isfinite(lse[ix]))
            if finite.any():
                e2 = float(np.max(np.abs(lse[ix][finite] - r.lse[finite])))
                worst_lse = max(worst_lse, e2)
                assert e2 <= max(tol, 1e-4), f"lse error {e2} at {key}"
    return {"n": len(results), "excused_near_ties": excused, "max_abs_err": worst,
            "max_lse_err": worst_lse}


def sample_positions(L: int, B: int, count: int, rng) -> list:
    """Positions of one sequence for sampled checks: the first and last
    tokens, both sides of several block boundaries, and random ones."""
    if L == 0:
        return []
    pts = {0, L - 1, min(L - 1, B - 1), min(L - 1, B)}
    for j in (1, 2, 5, L // B // 2, L // B - 1, L // B):
        for off in (-1, 0, 1):
            p = j * B + off
            if 0 <= p < L:
                pts.add(p)
    extra = rng.choice(L, size=min(L, max(0, count - len(pts))), replace=False)
    pts.update(int(x) for x in extra)
    return sorted(pts)
