"""The multi-GPU host logic of bench.py on CPU: two gloo ranks.

The decode path partitions into independent (sequence, KV head) units, so ranks share no
data; the only cross-rank steps are the barrier around the timed region and the MAX
reduction of the elapsed time. These run here over gloo with world size 2.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from tests import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]                      # rank 1 is the slow one
        dist.barrier()
        ms = bench.reduce_max(local_ms, world, "cpu")
        gbs = bench.weak_scaling_gbs(1e9, ms, world)
        # each rank draws its own sequences for the same batch slot
        cfg = synth.CONFIGS[1].with_(T_cap=64)
        src = bench.rank_sequence_offset(0, rank, cfg.B)
        k = synth.keys(cfg, src, 0, 4)
        out[rank] = (ms, gbs, float(np.abs(k).sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    (ms0, g0, k0), (ms1, g1, k1) = out[0], out[1]
    assert ms0 == ms1 == 5.0                             # every rank reports the slowest
    assert g0 == g1 == pytest.approx(2 * 1e9 / 5e-3 / 1e9)
    assert k0 != k1                                      # disjoint synthetic sequences


def test_single_rank_is_identity():
    assert bench.reduce_max(7.5, 1) == 7.5
    assert bench.weak_scaling_gbs(2e9, 1.0, 1) == pytest.approx(2000.0)
