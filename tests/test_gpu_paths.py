"""Parity of the kernel variants the workloads above do not reach: the fp32
decode path (CUDA-core attention + split combine), bf16 decode with 24 and 32
query rows per KV head (the tensor-map decode with two 16-row tiles, in one
launch and after the selection kernel; MTP verification of 2 and 3 draft
tokens at full cache size), the selection kernel followed by the tensor-map
attention kernel, head-wise gates on the tensor-core prefill and the
tensor-map decode, and bf16 prefill with head_dim 64 (CUDA-core prefill).
Every query is compared with the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200 import _lib
from block_sparse_attention_17_b200.workloads import (WORKLOADS, make_decode_inputs,
                                                      make_prefill_inputs)
from oracle import qsa_oracle as O
from tests import qsa_testlib as TL
from tests.test_gpu_parity import decode_parity, prefill_parity, run_decode

pytestmark = pytest.mark.gpu


def _decode(name, **kw):
    kv_lens = kw.pop("kv_lens")
    w = WORKLOADS[name].with_(kv_len=max(kv_lens), **kw)
    return w, make_decode_inputs(w, kv_lens=np.array(kv_lens, np.int32))


def _prefill(name, **kw):
    w = WORKLOADS[name].with_(ragged_range=None, **kw)
    return w, make_prefill_inputs(w)


def test_decode_fp32_cuda_core_path():
    w, inp = _decode("decode_bf16_b32_kv32768", dtype="f32", batch=4, cap=2112,
                     kv_lens=(2049, 64, 1000, 1))
    rep = decode_parity(w, inp)
    assert len(rep["excused_near_ties"]) <= 1, rep


def _two_kernel_parity(w, inp, d):
    """The selection kernel (qsa_select_decode) followed by the attention
    kernel over its lists (qsa_decode_attend): the kernels qsa_decode runs
    when the in-cluster selection does not apply. Compared with the oracle."""
    cfg = qsa.QSAConfig.from_workload(w)
    kv = d["kv_len"]
    pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
    s = qsa.select_decode(cfg, d["iq"], d["ik_cache"], d["iw"], pooled, kv)
    a = qsa.decode_attend(cfg, d["q"], d["k_cache"], d["v_cache"], d["gate"], kv, s["sel"],
                          s["nsel"], want_lse=True)
    torch.cuda.synchronize()
    gpu = {"out": a["out"], "lse": a["lse"], "sel": s["sel"], "nsel": s["nsel"]}
    return TL.check_queries(O.qsa_decode(w, inp)["queries"], gpu, lambda bi: bi, w)


@pytest.mark.parametrize("n_q", [3, 4])
def test_decode_bf16_two_row_tiles(n_q):
    # n_q new tokens x 8 query heads per KV head = 24 or 32 rows: the tensor-map
    # decode holds two tiles of 16 rows, in one launch (selection inside the
    # clusters) and as the attention kernel after the selection kernel
    w, inp = _decode("decode_bf16_b32_kv32768", n_q=n_q, batch=3, cap=3008,
                     kv_lens=(3000, 500, n_q))
    d = TL.upload(inp, w)
    assert _decode_launches(w, d) == 1
    rep = decode_parity(w, inp, d=d)
    assert len(rep["excused_near_ties"]) <= 1, rep
    rep = _two_kernel_parity(w, inp, d)
    assert len(rep["excused_near_ties"]) <= 1, rep


@pytest.mark.parametrize("n_q", [3, 4])
def test_mtp_verify_more_drafts_full_size(n_q):
    # MTP verification of n_q - 1 draft tokens on the 4 x 262144-token caches
    # (the pages measure n = 2 drafts; 24 and 32 rows per KV head)
    w = WORKLOADS["mtp_verify_bf16_b4_kv262144"].with_(n_q=n_q)
    inp = make_decode_inputs(w)
    rep = decode_parity(w, inp)
    print(f"n_q {n_q}: excused near-ties {rep['excused_near_ties']}")
    assert len(rep["excused_near_ties"]) <= 1, rep


def test_prefill_headwise_gate_tensor_cores():
    w, inp = _prefill("prefill_bf16_t8192", seqlens=(1500, 700), gate_headwise=True)
    assert inp["gate"].shape == (2200, w.num_q_heads)
    rep = prefill_parity(w, inp, None)
    assert len(rep["excused_near_ties"]) <= 2, rep


def test_decode_headwise_gate():
    w, inp = _decode("decode_bf16_b32_kv32768", batch=3, cap=4160, gate_headwise=True,
                     kv_lens=(4100, 2048, 70))
    assert inp["gate"].shape == (3, 1, w.num_q_heads)
    rep = decode_parity(w, inp)
    assert len(rep["excused_near_ties"]) <= 1, rep


def test_prefill_bf16_head_dim_64_cuda_core_path():
    w, inp = _prefill("prefill_bf16_t8192", seqlens=(1200,), head_dim=64)
    rep = prefill_parity(w, inp, None)
    assert len(rep["excused_near_ties"]) <= 2, rep


def _decode_launches(w, d):
    """Kernel launches of one qsa.decode call on the uploaded inputs d (after a
    warm-up call)."""
    cfg = qsa.QSAConfig.from_workload(w)
    kv = d["kv_len"]
    pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))

    def call():
        qsa.decode(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"], d["ik_cache"], d["iw"],
                   d["gate"], pooled, kv)
    call()
    torch.cuda.synchronize()
    lib = _lib.lib()
    n0 = lib.qsa_kernel_launch_count()
    call()
    torch.cuda.synchronize()
    return lib.qsa_kernel_launch_count() - n0


@pytest.mark.parametrize("name,kv_lens,cap", [
    ("decode_bf16_b32_kv32768", (4100, 2048, 70), 4160),
    ("mtp_verify_bf16_b4_kv262144", (9000, 129, 2), 9088),
])
def test_decode_one_launch_and_two_kernel_paths(name, kv_lens, cap):
    # A cache of a few thousand blocks, and the same rows at the start of a
    # 12800-block cache: one launch each (the selection inside the decode
    # kernel's clusters keeps only candidates, so it fits either cache). The
    # selection kernel + attention kernel pair matches the oracle as well.
    w, inp = _decode(name, batch=len(kv_lens), cap=cap, kv_lens=kv_lens)
    d = TL.upload(inp, w)
    assert _decode_launches(w, d) == 1
    big = 12800 * w.block_size
    for key in ("k_cache", "v_cache", "ik_cache"):
        t = torch.zeros((t0 := d[key]).shape[0], big, *t0.shape[2:], dtype=t0.dtype, device="cuda")
        t[:, :cap] = t0
        d[key] = t
    assert _decode_launches(w, d) == 1
    rep = decode_parity(w, inp, d=d)
    assert len(rep["excused_near_ties"]) <= 1, rep
    rep = _two_kernel_parity(w, inp, d)
    assert len(rep["excused_near_ties"]) <= 1, rep


@pytest.mark.parametrize("name", ["decode_bf16_b32_kv32768", "mtp_verify_bf16_b4_kv262144"])
def test_decode_topk_concentrated_in_one_range(name):
    # The one-launch decode's clusters take each CTA's top k of its own range
    # of blocks as candidates; here one range holds most of the top k. The
    # indexer keys of the first 48 blocks are scaled by 8 (exact in bf16).
    B = WORKLOADS[name].block_size
    kv = 800 * B + 3
    w, inp = _decode(name, batch=2, cap=801 * B, kv_lens=(kv, kv - 70))
    ik = inp["ik_cache"].copy()
    ik[:, :48 * B] *= 8.0
    inp["ik_cache"] = ik
    d = TL.upload(inp, w)
    assert _decode_launches(w, d) == 1
    gpu = run_decode(w, inp, d)
    assert gpu["err"] == 0
    rep = TL.check_queries(O.qsa_decode(w, inp)["queries"], gpu, lambda bi: bi, w)
    assert len(rep["excused_near_ties"]) <= 1, rep
    sel = gpu["sel"].cpu().numpy()
    k = w.topk
    for b in range(w.batch):
        for i in range(w.n_q):
            assert (sel[b, i, :k] < 48).sum() >= 24, sel[b, i]
