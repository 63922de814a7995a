"""qsa_decode_noalloc against qsa_decode.

qsa_decode_noalloc serves callers that cannot allocate device memory for
scratch (their own allocator owns the GPU's memory, or their loop must never
call cudaMalloc): it takes its scratch from a static device array instead of a
caller workspace. This file sorts last so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200.workloads import WORKLOADS, make_decode_inputs
from tests import qsa_testlib as TL

pytestmark = pytest.mark.gpu


def _case(name, batch, kv_lens, cap, **kw):
    w = WORKLOADS[name].with_(batch=batch, kv_len=max(kv_lens), cap=cap, **kw)
    inp = make_decode_inputs(w, kv_lens=np.array(kv_lens, np.int32))
    return w, inp, TL.upload(inp, w)


# The first two cases take the one-launch decode (the static array then holds
# only the error word); the last two take the selection kernel + attention
# kernel path (fp32, and three new tokens with eight heads per KV head), which
# keeps its counters, score keys, selection lists and split partials in the
# array, so the second call of each case runs on the first call's leftovers.
@pytest.mark.parametrize("name,batch,kv_lens,cap,kw", [
    ("decode_bf16_b32_kv32768", 6, (4097, 64, 2112, 2113, 130, 1), 4160, {}),
    ("mtp_verify_bf16_b4_kv262144", 3, (9000, 4225, 2), 9088, {}),
    ("decode_bf16_b32_kv32768", 3, (2000, 65, 1), 2112, {"dtype": "f32"}),
    ("mtp_verify_bf16_b4_kv262144", 3, (9000, 4226, 3), 9088, {"n_q": 3}),
])
def test_noalloc_decode_matches_workspace_decode_twice(name, batch, kv_lens, cap, kw):
    w, inp, d = _case(name, batch, kv_lens, cap, **kw)
    cfg = qsa.QSAConfig.from_workload(w)
    prefix = (d["kv_len"] - w.n_q).to(torch.int32)
    for call in range(2):
        # reference: the workspace entry point; the same kernels run on the
        # same inputs, so every output is bit-identical
        pooled_ref = qsa.pool_build(cfg, d["ik_cache"], prefix)
        ref = qsa.decode(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"], d["ik_cache"],
                         d["iw"], d["gate"], pooled_ref, d["kv_len"], want_lse=True,
                         want_sel=True)
        pooled = qsa.pool_build(cfg, d["ik_cache"], prefix)
        got = qsa.decode_noalloc(cfg, d["q"], d["k_cache"], d["v_cache"], d["iq"],
                                 d["ik_cache"], d["iw"], d["gate"], pooled, d["kv_len"],
                                 want_lse=True, want_sel=True)
        torch.cuda.synchronize()
        assert torch.equal(got["out"], ref["out"]), call
        assert torch.equal(got["sel"], ref["sel"]) and torch.equal(got["nsel"], ref["nsel"])
        assert torch.equal(got["lse"], ref["lse"]), call
        assert torch.equal(pooled, pooled_ref)


def test_noalloc_rejects_geometry_beyond_the_static_scratch():
    # 64 sequences of 1M-token caches need far more than the 4 MiB scratch; the
    # size check comes first, and every pointer is NULL, so even a regression
    # of that check could not reach a kernel (the NULL checks come next)
    import ctypes
    from block_sparse_attention_17_b200 import _lib
    w = WORKLOADS["decode_bf16_b32_kv32768"]
    cfg = qsa.QSAConfig.from_workload(w)
    batch, cap = 64, 1 << 20
    assert qsa.decode_workspace_size(cfg, batch, 1, cap) > 4 << 20
    c = cfg.c()
    st = _lib.lib().qsa_decode_noalloc(ctypes.byref(c), batch, 1, cap, *([None] * 14), None)
    assert st == _lib.QSA_ERR_WORKSPACE
    assert b"static scratch" in _lib.lib().qsa_last_error()
