"""Multi-process plumbing of the benchmark on CPU (gloo, world size 2).

The forward pass partitions into independent (row, head) problems, so ranks
share nothing on the data path: each rank draws its own batch and the job's
throughput is ranks x tokens / max-over-ranks time. These tests run that
plumbing with real processes and the gloo backend, and check on the CPU
oracle that a rank's shard is computed exactly as if it ran alone.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from bayesian_filter_scan_b200.inputs import WORKLOADS, make_inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS[1].with_(B=1, H=2, T=96)
        inp = make_inputs(w, seed=bench.rank_seed(w, rank))
        r = oracle.forward_inputs(inp, w, num_threads=1)
        # every rank reports a different local time; the job takes the max
        local_ms = 10.0 * (rank + 1)
        ms, value = bench.aggregate(world, w.tokens, local_ms, steps=5, dist=dist, device="cpu")
        digest = float(np.abs(r["out"]).sum())
        q.put((rank, ms, value, digest, inp["q"].float().sum().item()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_aggregate():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = WORKLOADS[1].with_(B=1, H=2, T=96)
    for rank, ms, value, digest, qsum in res:
        assert ms == 20.0 / 5                       # max over ranks, per step
        assert abs(value - world * w.tokens / (ms * 1e-3)) < 1e-6
        alone = oracle.forward_inputs(make_inputs(w, seed=bench.rank_seed(w, rank)), w, num_threads=1)
        assert digest == float(np.abs(alone["out"]).sum())
    # ranks draw different batches
    assert res[0][4] != res[1][4]


def test_single_process_aggregate_without_dist():
    ms, value = bench.aggregate(1, 1000, 50.0, steps=10, dist=None, device="cpu")
    assert ms == 5.0 and abs(value - 1000 / 5e-3) < 1e-6
