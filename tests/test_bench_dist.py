"""The multi-process logic of bench.py on CPU (gloo, world size 2).

Under torchrun each rank is an independent replica of the workload (its own
sequences, no data-path collective); the only collectives are the barrier and
the element-wise MAX of the ranks' times, and the reported value is every
rank's KV tokens over the slowest rank's time. The reference arm runs on rank
0 only.
"""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from decode_attention_dq_b200 import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # Rank r takes (1 + r) ms per step and its decode 0.5 / (1 + r) ms.
        times = bench.max_over_ranks([1.0 + rank, 0.5 / (1.0 + rank)], dist, "cpu")
        value = bench.whole_job_rate(1000, world, times[0])
        w = bench.replica_workload(synth.WORKLOADS["serve_b128_t8k"], rank)
        dist.barrier()
        out[rank] = (times, value, w.seed, w.B, w.T)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    (t0, v0, s0, b0, T0), (t1, v1, s1, b1, T1) = res[0], res[1]
    assert t0 == t1 == [2.0, 0.5]  # the MAX over ranks, the same on every rank
    assert v0 == v1 == pytest.approx(2 * 1000 / 2.0e-3)
    assert (b0, T0) == (b1, T1) and s0 != s1  # replicas: same shapes, own sequences


def test_single_process_needs_no_group():
    assert bench.max_over_ranks([3.0, 4.0], None, "cpu") == [3.0, 4.0]
    assert bench.whole_job_rate(128 * 8192, 1, 2.0) == pytest.approx(128 * 8192 / 2.0e-3)
    w = synth.WORKLOADS["serve_b128_t8k"]
    assert bench.replica_workload(w, 0) is w


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"workload": "tiny_b1_t256", "steps": 1, "warmup": 0})()
    assert bench.run_reference(args) is None


def test_prefill_pair_count_and_traffic_gate():
    # Useful tensor work of a causal chunk: query token i at position
    # q_start + i sees q_start + i + 1 keys, for every sequence and head.
    import bench
    for B, Hq, q_start, n_q in [(1, 1, 0, 1), (2, 4, 10, 7), (16, 32, 7680, 512)]:
        brute = B * Hq * sum(q_start + i + 1 for i in range(n_q))
        assert bench.chunk_pairs(B, Hq, q_start, n_q) == brute
    # DRAM traffic is only reported for the captured workload and source
    assert bench.prefill_traffic("serve_b32_t8k", 128, 36, 36) is None
    assert bench.prefill_traffic("qwen3_8b_b16_t8k", 512, 31, 31) is None
    t = bench.prefill_traffic("qwen3_8b_b16_t8k", 512, 36, 36)
    assert t is None or t == bench.PREFILL_TRAFFIC["bytes"]
