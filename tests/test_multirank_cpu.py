"""Multi-rank host logic of bench.py on CPU: world_size-2 gloo ranks.

QSA's units (sequences of a packed prefill, sequences of a decode batch) are
independent problems, so ranks shard them with no collective on the data path;
the only collectives are the timing reductions checked here.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_sparse_attention_17_b200.workloads import (WORKLOADS,  # noqa: E402
                                                      make_decode_inputs, resolve_seqlens)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.rank_workload(WORKLOADS["ragged_prefill_bf16_4seq"], rank)
        units, _ = bench.workload_units(w)
        ms = 10.0 + 5.0 * rank                   # rank 1 is the slow one
        job_units, job_ms = bench.reduce_over_ranks(dist, units, ms, torch.device("cpu"))
        dist.barrier()
        results[rank] = (units, job_units, job_ms)
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world2():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world,
                       join=True, start_method="spawn")
    assert sorted(results.keys()) == [0, 1]
    u0, j0, t0 = results[0]
    u1, j1, t1 = results[1]
    # every rank sees the job totals: the units summed, the slowest rank's time
    assert j0 == j1 == u0 + u1
    assert t0 == t1 == 15.0
    # the shards differ (ragged lengths are drawn per rank)
    assert u0 != u1


def test_rank_shards_are_distinct_and_rank0_is_the_workload():
    for name, w in WORKLOADS.items():
        assert bench.rank_workload(w, 0) is w
        seeds = {bench.rank_workload(w, r).seed for r in range(8)}
        assert len(seeds) == 8, name
        for r in range(1, 4):
            wr = bench.rank_workload(w, r)
            # same shapes, only the draws change
            assert (wr.num_q_heads, wr.num_kv_heads, wr.head_dim, wr.block_size,
                    wr.budget) == (w.num_q_heads, w.num_kv_heads, w.head_dim,
                                   w.block_size, w.budget), name
    wr = bench.rank_workload(WORKLOADS["ragged_prefill_bf16_4seq"], 1)
    lens, _ = resolve_seqlens(wr)
    assert len(lens) == 4 and all(8192 <= n <= 32768 for n in lens)
    small = WORKLOADS["decode_bf16_b32_kv32768"].with_(batch=2, kv_len=256)
    a = make_decode_inputs(bench.rank_workload(small, 0))
    b = make_decode_inputs(bench.rank_workload(small, 1))
    assert not (a["q"] == b["q"]).all()


def test_single_process_reduction_is_identity():
    assert bench.reduce_over_ranks(None, 123.0, 4.5, None) == (123.0, 4.5)


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


@pytest.mark.timeout(300)
def test_reference_arm_rank0_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "prefill_f32_t1024", "--steps", "1", "--warmup", "0",
                        "--ref-step-seconds", "0.5"], env=env, capture_output=True,
                       text=True, timeout=280)
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
