"""The visited-keys debug counter (qsa_set_keys_visited; the keys_visited count
of the llama.cpp PR #27739 page's QSA commit text: 16400 sparse against 24016
dense at kv_len 3002). Each attention kernel counts, where it decides which
keys a row sees, the (query, head, key) triples it attends over; a correct
sparse consumer gives Hq * sum over queries of (min(k, nc) * B + tail), the
oracle's own count, whatever extra tile work it executes, and the dense count
when the budget covers the context. Checked on every attention path: the
tensor-core and CUDA-core prefill, the one-launch decode, the selection kernel
followed by the attention kernel, the fp32 decode, MTP verification, the
context-parallel shards and the fp8 caches."""
import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200 import context_parallel as cp
from block_sparse_attention_17_b200.workloads import (WORKLOADS, make_decode_inputs,
                                                      make_prefill_inputs)
from oracle import qsa_oracle as O
from tests import qsa_testlib as TL

pytestmark = pytest.mark.gpu


class Counter:
    def __enter__(self):
        self.t = torch.zeros(1, dtype=torch.int64, device="cuda")
        qsa.set_keys_visited(self.t)
        return self

    def __exit__(self, *exc):
        qsa.set_keys_visited(None)

    @property
    def value(self):
        torch.cuda.synchronize()
        return int(self.t.item())


def expected(w, results):
    return w.num_q_heads * sum(r.tokens for r in results.values())


@pytest.mark.parametrize("name,seqlens,budget", [
    ("prefill_f32_t1024", (1024,), None),               # CUDA-core prefill
    ("prefill_bf16_t8192", (2600,), None),              # tensor-core prefill, B = 64
    ("ragged_prefill_bf16_4seq", (3000, 257, 1, 4100), None),   # tensor-core prefill, B = 128
    ("prefill_bf16_t8192", (1500,), 2048),              # budget covers the context: dense
])
def test_prefill_counts_the_selected_keys(name, seqlens, budget):
    w = WORKLOADS[name].with_(ragged_range=None, seqlens=seqlens)
    if budget:
        w = w.with_(budget=budget)
    inp = make_prefill_inputs(w)
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    with Counter() as c:
        qsa.prefill(cfg, d["q"], d["k"], d["v"], d["iq"], d["ik"], d["iw"], d["gate"],
                    d["cu_seqlens"], inp["max_seqlen"])
        got = c.value
    orc = O.qsa_prefill(w, inp, attend=False)["queries"]
    assert got == expected(w, orc)
    if budget:   # every query sees all of its prefix
        assert got == w.num_q_heads * sum(L * (L + 1) // 2 for L in seqlens)
    # off again: nothing is added
    with Counter() as c2:
        pass
    qsa.prefill(cfg, d["q"], d["k"], d["v"], d["iq"], d["ik"], d["iw"], d["gate"],
                d["cu_seqlens"], inp["max_seqlen"])
    assert c2.value == 0


@pytest.mark.parametrize("name,kw", [
    ("decode_bf16_b32_kv32768", dict(batch=4, cap=3008, kv_lens=(3000, 500, 64, 1))),
    ("decode_bf16_b32_kv32768", dict(batch=3, cap=3008, kv_lens=(3000, 700, 4), n_q=4)),
    ("decode_bf16_b32_kv32768", dict(batch=4, cap=2112, kv_lens=(2049, 64, 1000, 1), dtype="f32")),
    ("mtp_verify_bf16_b4_kv262144", dict()),
])
def test_decode_counts_the_selected_keys(name, kw):
    kw = dict(kw)
    kv_lens = kw.pop("kv_lens", None)
    w = WORKLOADS[name].with_(**kw)
    if kv_lens is None:
        inp = make_decode_inputs(w)
    else:
        w = w.with_(kv_len=max(kv_lens))
        inp = make_decode_inputs(w, kv_lens=np.array(kv_lens, np.int32))
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    kv = d["kv_len"]
    want = expected(w, O.qsa_decode(w, inp, attend=False)["queries"])
    pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
    with Counter() as c:   # qsa_decode (one launch where the clusters fit)
        qsa.decode(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"], d["ik_cache"], d["iw"],
                   d["gate"], pooled, kv)
        assert c.value == want
    pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
    s = qsa.select_decode(cfg, d["iq"], d["ik_cache"], d["iw"], pooled, kv)
    with Counter() as c:   # the attention kernel over the selection kernel's lists
        qsa.decode_attend(cfg, d["q"], d["k_cache"], d["v_cache"], d["gate"], kv, s["sel"],
                          s["nsel"])
        assert c.value == want


def test_fp8_decode_counts_the_selected_keys():
    w = WORKLOADS["decode_bf16_b32_kv32768"].with_(batch=4, cap=3008, kv_len=3000)
    inp = make_decode_inputs(w, kv_lens=np.array([3000, 500, 64, 1], np.int32))
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    kv = d["kv_len"]
    codes = {}
    for n in ("k_cache", "v_cache"):
        x = d[n].float()
        sc = (x.abs().amax(-1) / 448.0).clamp_min(1e-30)
        codes[n] = ((x / sc[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).contiguous(),
                    sc.contiguous())
    pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
    with Counter() as c:
        qsa.decode_fp8(cfg, d["q"], codes["k_cache"][0], codes["k_cache"][1], codes["v_cache"][0],
                       codes["v_cache"][1], d["iq"], d["ik_cache"], d["iw"], d["gate"], pooled, kv)
        got = c.value
    assert got == expected(w, O.qsa_decode(w, inp, attend=False)["queries"])


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_shards_count_the_selected_keys(world):
    w = WORKLOADS["decode_bf16_b32_kv32768"].with_(batch=4, cap=64 * 120, kv_len=64 * 120)
    kvn = np.array([64 * 120, 64 * 117 + 5, 64 * 37 + 63, 200], np.int32)
    inp = make_decode_inputs(w, kv_lens=kvn)
    cfg = qsa.QSAConfig.from_workload(w)
    d = TL.upload(inp, w)
    kv = d["kv_len"]
    B, nblk = w.block_size, w.cap // w.block_size
    fns, cands = [], []
    for r in range(world):
        b0, b1 = cp.shard_blocks(nblk, world, r)
        sh = lambda t: t[:, b0 * B:b1 * B].contiguous()
        pooled = qsa.cp_pool_build(cfg, sh(d["ik_cache"]), (kv - w.n_q).to(torch.int32), b0)
        f = cp.library_fns(cfg, d["q"], sh(d["k_cache"]), sh(d["v_cache"]), d["iq"],
                           sh(d["ik_cache"]), d["iw"], d["gate"], pooled, b0)
        fns.append(f)
        cands.append(f.select(kv))
    glob = fns[0].global_topk(torch.stack([c["score"] for c in cands]),
                              torch.stack([c["id"] for c in cands]), kv)
    with Counter() as c:
        for f in fns:
            f.attend(kv, glob["sel"], glob["nsel"])
        got = c.value
    assert got == expected(w, O.qsa_decode(w, inp, attend=False)["queries"])
