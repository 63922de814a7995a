"""fp8 (e4m3) K/V caches for decode (qsa_decode_fp8), plain and stored in a
Walsh-Hadamard-rotated basis (ramgpt "Porting Qwen4 to llama.cpp", section
"Quantized KV Is a Representation Contract").

The caches are quantized here, per (token, KV head) row: scale = max|x| / 448,
code = e4m3(x / scale). The oracle attends over what the codes stand for,
scale * decode(code) -- rotated back with H (symmetric and orthonormal) when the
rows were stored as H k, H v -- so the comparison isolates the kernel from the
quantization error. Rows past each sequence's last token hold NaN codes: a
gather must never let them reach the output.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200.workloads import WORKLOADS, make_decode_inputs
from oracle import qsa_oracle as O
from tests import qsa_testlib as TL

pytestmark = pytest.mark.gpu


def hadamard(n):
    """Sylvester-order Walsh-Hadamard matrix scaled to be orthonormal."""
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h / np.sqrt(n)


def quantize_rows(x):
    """x [..., D] float64 -> (e4m3 codes as uint8 tensor, fp32 scales [...], values)."""
    amax = np.abs(x).max(axis=-1)
    scale = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
    codes = torch.from_numpy((x / scale[..., None]).astype(np.float32)).to(torch.float8_e4m3fn)
    values = codes.to(torch.float64).numpy() * scale[..., None].astype(np.float64)
    return codes.view(torch.uint8), torch.from_numpy(scale), values


def _case(name, batch, kv_lens, cap):
    w = WORKLOADS[name].with_(batch=batch, cap=cap, kv_len=max(kv_lens))
    return w, make_decode_inputs(w, kv_lens=np.array(kv_lens, np.int32))


@pytest.mark.parametrize("rotated", [False, True])
@pytest.mark.parametrize("name,batch,kv_lens,cap", [
    ("decode_bf16_b32_kv32768", 5, (4097, 64, 2113, 130, 1), 4160),
    ("mtp_verify_bf16_b4_kv262144", 3, (9000, 4225, 2), 9088),
])
def test_fp8_decode_matches_the_oracle_on_the_dequantized_rows(name, batch, kv_lens, cap, rotated):
    w, inp = _case(name, batch, kv_lens, cap)
    H = hadamard(w.head_dim)
    stored = {}
    eff = {}
    for key in ("k_cache", "v_cache"):
        x = inp[key].astype(np.float64)
        if rotated:
            x = x @ H                      # each row r -> H r (H symmetric)
        codes, scale, values = quantize_rows(x)
        for b, n in enumerate(kv_lens):    # rows past the sequence: NaN codes
            codes[b, n:] = 0x7F
        stored[key] = (codes.cuda(), scale.cuda())
        eff[key] = values @ H if rotated else values   # what the rows stand for
    d = TL.upload(inp, w)
    cfg = qsa.QSAConfig.from_workload(w)
    kv = d["kv_len"]
    pooled = qsa.pool_build(cfg, d["ik_cache"], (kv - w.n_q).to(torch.int32))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    gpu = qsa.decode_fp8(cfg, d["q"], stored["k_cache"][0], stored["k_cache"][1],
                         stored["v_cache"][0], stored["v_cache"][1], d["iq"], d["ik_cache"],
                         d["iw"], d["gate"], pooled, kv, rotated=rotated, want_lse=True,
                         want_sel=True, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.isfinite(gpu["out"].float()).all()
    orc = O.qsa_decode(w, {**inp, "k_cache": eff["k_cache"], "v_cache": eff["v_cache"]})
    rep = TL.check_queries(orc["queries"], gpu, lambda bi: bi, w)
    assert len(rep["excused_near_ties"]) <= 1, rep


def test_fp8_decode_rejects_unsupported_geometry():
    w, inp = _case("decode_bf16_b32_kv32768", 2, (300, 200), 320)
    cfg = qsa.QSAConfig.from_workload(w.with_(dtype="f32"))
    d = TL.upload(inp, w)
    z8 = torch.zeros(2, 320, w.num_kv_heads, w.head_dim, dtype=torch.uint8, device="cuda")
    zs = torch.ones(2, 320, w.num_kv_heads, dtype=torch.float32, device="cuda")
    pooled = torch.zeros(2, 320 // w.block_size, w.idx_dim, device="cuda")
    with pytest.raises(qsa.QsaError):
        qsa.decode_fp8(cfg, d["q"].float(), z8, zs, z8, zs, d["iq"].float(), d["ik_cache"].float(),
                       d["iw"], d["gate"].float(), pooled, d["kv_len"])
