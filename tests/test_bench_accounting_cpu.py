"""bench.py's algorithmic units for the decode roofline, pinned to numbers
worked out by hand from the workload shapes (no GPU)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_sparse_attention_17_b200.workloads import WORKLOADS  # noqa: E402


def test_decode_step_bytes_of_the_32_sequence_workload():
    w = WORKLOADS["decode_bf16_b32_kv32768"]
    kv = np.full(32, 32768)
    # every query selects 32 complete blocks of 64 tokens (no tail at 32768)
    sel = np.tile(np.arange(32, dtype=np.int32) * 7, (32, 1, 1)).reshape(32, 1, 32)
    sel = np.concatenate([sel, np.full((32, 1, 1), -1, np.int32)], axis=2)
    nsel = np.full((32, 1), 32)
    kvb = bench.decode_selected_kv_bytes(w, sel, nsel, kv)
    assert kvb == 32 * 2048 * 2 * 128 * 2 * 2            # seqs x tokens x Hkv x D x (K, V) x bf16
    # selection: pooled rows of 512 blocks (fp32, di 64) per sequence; the block
    # this step completes (64 rows x 64 bf16 read, one fp32 row written); iq
    # (4 heads x 64 bf16) and iw (4 fp32); the lists (k + 2 int32 per query)
    per_seq = 512 * 64 * 4 + 64 * 64 * 2 + 64 * 4 + 4 * (64 * 2 + 4) + (32 + 2) * 4
    assert bench.decode_selection_bytes(w, kv) == 32 * per_seq
    # fp8 caches: one byte per element plus a 4-byte scale per (token, KV head) row
    assert bench.decode_selected_kv_bytes(w, sel, nsel, kv, "fp8") == 32 * 2048 * 2 * (128 + 4) * 2


def test_mtp_union_counts_shared_blocks_once():
    w = WORKLOADS["mtp_verify_bf16_b4_kv262144"].with_(batch=1)
    kv = np.array([262144])
    # query 0 sees 262143 tokens (2047 complete blocks + a 127-token tail block
    # 2047); query 1 sees 262144 (2048 complete blocks, no tail). Both pick
    # blocks 0..31; query 0 adds its tail, query 1 picks block 2047 instead of 31.
    s0 = list(range(32)) + [2047]
    s1 = list(range(31)) + [2047]
    sel = np.full((1, 2, 33), -1, np.int32)
    sel[0, 0, :33] = s0
    sel[0, 1, :32] = s1
    nsel = np.array([[33, 32]])
    toks = 32 * 128 + 128                # blocks 0..31, and block 2047 whole (query 1)
    assert bench.decode_selected_kv_bytes(w, sel, nsel, kv) == toks * 2 * 128 * 2 * 2
