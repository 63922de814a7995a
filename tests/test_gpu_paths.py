"""Parity of the kernel variants the workloads above do not reach: the fp32
decode path (CUDA-core attention + split combine), bf16 decode with more than
16 query rows per KV head (the same CUDA-core path), head-wise gates on the
tensor-core prefill and the tensor-map decode, and bf16 prefill with
head_dim 64 (CUDA-core prefill). Every query is compared with the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_17_b200 as qsa
from block_sparse_attention_17_b200.workloads import (WORKLOADS, make_decode_inputs,
                                                      make_prefill_inputs)
from oracle import qsa_oracle as O
from tests import qsa_testlib as TL
from tests.test_gpu_parity import decode_parity, prefill_parity

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


def test_decode_bf16_24_rows_per_kv_head():
    # n_q = 3 new tokens x 8 query heads per KV head = 24 rows: past the
    # 16-row tensor-map path, served by the CUDA-core decode
    w, inp = _decode("decode_bf16_b32_kv32768", n_q=3, batch=3, cap=3008,
                     kv_lens=(3000, 500, 3))
    rep = decode_parity(w, inp)
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
