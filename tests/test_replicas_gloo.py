"""The N > 1 path of bench.py (independent replicas, weak scaling) on two gloo
ranks on CPU: each rank draws its own token stream, and the whole-job
throughput divides all ranks' tokens by the slowest rank's time."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import moe_inputs as mi


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(10.0 + 5.0 * rank)
        w = mi.WORKLOADS["deepseek_v3"].with_(T=4, d_model=16)
        h = mi.normal_f32(w.seed, bench.h_stream_id(rank, 3), 0, w.T * w.d_model, 1.0)
        gathered = [torch.zeros(w.T * w.d_model) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(h))
        out[rank] = (t, [g.numpy().copy() for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_replicas_on_gloo():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        t, hs = res[r]
        assert t == 15.0                                   # the slowest rank's time
        assert not np.array_equal(hs[0], hs[1])            # distinct token streams
    assert bench.job_throughput(2, 4096, 20, 100.0) == 2 * 4096 * 20 / 0.1
