"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): each rank gets an independent problem (different
seeds, same shape), the job time is the max over ranks, and the whole-job value counts every rank's work."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from exact_io_aware_48_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = inputs.workloads()["tiny"]
        w.seed += rank  # what bench.Problem does per rank
        q = w.tensors()[0]
        digest = torch.tensor([float(q.float().sum())], dtype=torch.float64)
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, digest)
        pairs = bench.visible_pairs(w.B, w.H, w.N, w.causal)
        step_flops = 3.5 * bench.fwd_flops(w.d, pairs)
        local_ms = 10.0 * (rank + 1)  # rank 1 is the slow one
        value, total_ms = bench.aggregate(local_ms, step_flops, 5, world, "cpu")
        out[rank] = (value, total_ms, [float(g) for g in gathered], step_flops)
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_aggregate():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    (v0, t0, g0, f0), (v1, t1, g1, f1) = out[0], out[1]
    assert t0 == t1 == 20.0                      # max over ranks
    assert v0 == v1 == pytest.approx(2 * f0 * 5 / 0.020 / 1e12)
    assert g0 == g1 and g0[0] != g0[1]           # independent inputs per rank


def test_visible_pairs_counts():
    assert bench.visible_pairs(1, 1, 4, True) == 10
    assert bench.visible_pairs(2, 3, 5, False) == 2 * 3 * 25
    assert bench.visible_pairs(2, 1, 300, False, key_lens=[300, 7]) == 300 * 307
    # general path agrees with the closed forms
    assert bench.visible_pairs(1, 2, 300, True, block_mask=np.ones((3, 3), np.uint8)) == 2 * 300 * 301 // 2
    m = np.eye(3, dtype=np.uint8)
    assert bench.visible_pairs(1, 1, 300, False, block_mask=m) == 128 * 128 * 2 + 44 * 44
