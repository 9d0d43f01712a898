"""The multi-rank path of bench.py on CPU: two gloo ranks, each with its own
replica seed, reduce their step times by max and their work by sum (no data-path
collective exists; these reductions are timing plumbing only)."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank       # rank 1 is the slower one
        units = 100.0 * (rank + 1)
        t, u = bench.reduce_timing(ms, units, world)
        out[rank] = (t, u, bench.rank_seed(2, rank))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_seeds():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0          # max over ranks
    assert res[0][1] == res[1][1] == 300.0         # summed work
    assert res[0][2] == 1002 and res[1][2] != res[0][2]  # rank 0 keeps the workload seed


def test_single_rank_is_identity():
    assert bench.reduce_timing(3.5, 7.0, 1) == (3.5, 7.0)


def test_useful_flops_excludes_padding():
    from packgen import make_workload
    w = make_workload(2, with_arrays=False)
    real = [d for d in w.descs if not d.is_dummy]
    assert len(real) == len(w.descs) - 1
    n2 = sum((d.frames * d.grid_h * d.grid_w + d.n_text) ** 2 for d in real)
    assert bench.useful_flops(w) == 4.0 * 128 * 24 * n2
