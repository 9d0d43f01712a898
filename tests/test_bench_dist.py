"""The multi-rank path of bench.py on CPU: two gloo ranks, each with its own
replica seed, reduce their step times by max and their work by sum (no data-path
collective exists; these reductions are timing plumbing only). The replica
launcher (``--gpus N`` outside torchrun) is driven end to end with a CPU stand-in
for the GPU arm."""

import argparse
import json
import os
import socket
import sys

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


def _stub_arm(args, rank, world, local_rank):
    """Stands in for a GPU arm: each rank reports a step time and its work,
    reduced the way the arms reduce them; rank 0 writes the line."""
    ids = [None] * world
    dist.all_gather_object(ids, (rank, local_rank, int(os.environ["RANK"]),
                                 int(os.environ["WORLD_SIZE"])))
    t, u = bench.reduce_timing(10.0 + 5.0 * rank, 100.0 * (rank + 1), world)
    if rank == 0:
        with open(args.out, "w") as f:
            json.dump({"n_gpus": world, "ms_per_step": t, "units": u, "ids": ids}, f)


def test_launcher_runs_n_ranks_end_to_end(tmp_path):
    args = argparse.Namespace(out=str(tmp_path / "line.json"), op="block", gpus=2)
    bench.launch_replicas(args, 2, backend="gloo", arm=_stub_arm)
    line = json.load(open(args.out))
    assert line["n_gpus"] == 2
    assert line["ms_per_step"] == 15.0 and line["units"] == 300.0
    # rank r runs as local rank r (GPU r) and sees the rank variables torchrun would set
    assert sorted(map(tuple, line["ids"])) == [(0, 0, 0, 2), (1, 1, 1, 2)]


def test_main_spawns_replicas_without_a_launcher(monkeypatch):
    calls = []
    monkeypatch.setattr(bench, "launch_replicas", lambda args, n: calls.append((n, args.op)))
    for var in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(var, raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--steps", "2", "--warmup", "3"])
    bench.main()
    assert calls == [(4, "block")]


def test_main_under_torchrun_takes_the_world_size(monkeypatch):
    seen = []
    monkeypatch.setattr(bench, "run_rank",
                        lambda args, rank, world, local_rank: seen.append((args.gpus, rank, world)))
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "2", "--warmup", "3"])
    bench.main()
    assert seen == [(2, 1, 2)]
