"""The multi-GPU host logic of bench.py on CPU with two gloo ranks: each rank gets its
own seeded replica of the workload, the timing is the max over ranks, and the reported
throughput is the whole job's (weak scaling)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [1.5, 2.25][rank]
        out[rank] = bench.max_over_ranks(ms, dist, "cpu")
        w = synth.WORKLOADS["yolo20x20_b1_h4_d64"]
        x = synth.make_inputs(bench.rank_workload(w, rank))
        out[2 + rank] = float(synth.bf16_bits_to_f32(x["q"]).astype(np.float64).sum())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 2.25                  # both ranks see the slowest rank's time
    assert out[2] != out[3]                          # replicas draw different seeded data


def test_weak_scaling_value():
    w = synth.WORKLOADS["seq4096_b8_h32_d128"]
    one = bench.weak_scaling_tflops(w, 1, 2.0)
    assert one == pytest.approx(w.flops / 2e-3 / 1e12)
    assert bench.weak_scaling_tflops(w, 8, 2.0) == pytest.approx(8 * one)
    assert bench.max_over_ranks(3.0) == 3.0
