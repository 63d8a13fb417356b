"""Multi-rank host logic of bench.py on CPU with the gloo backend (world size 2).

Each rank decodes its own batch (same shape, its own seed, no data exchange); the
timed region is reduced as the maximum over ranks and the whole-job rate counts
every rank's bytes over that maximum."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from mla_inputs import make_workload, preset


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = preset("tiny")
        seed = bench.shard_seed(spec.seed, rank)
        w = make_workload(spec.with_(seed=seed))
        local_ms = 10.0 + 5.0 * rank                    # rank 1 is the slow one
        out[rank] = (seed, float(w.q_nope.float().sum()), bench.reduce_max(local_ms))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_take_the_max():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    (s0, q0, m0), (s1, q1, m1) = res[0], res[1]
    assert s0 != s1 and q0 != q1          # different batches on the two ranks
    assert m0 == m1 == 15.0               # both see the slowest rank's time
    rate = bench.whole_job_rate(world, 1000, m0, steps=3)
    assert rate == pytest.approx(2 * 1000 * 3 / 15e-3 / 1e9)


def test_single_process_reduce_is_identity():
    assert bench.reduce_max(3.5) == 3.5
