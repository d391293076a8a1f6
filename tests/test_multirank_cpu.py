"""Host-side logic of the N > 1 benchmark path on CPU: two gloo ranks (127.0.0.1).

bench.py runs replicas, one process per GPU, and reports the slowest rank: these tests check
that max_over_ranks returns the maximum on every rank, that barrier() completes, that the
ranks read their identity from the environment the launcher sets, and that the reference
arm does its work on rank 0 only.
"""
import importlib.util
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    bench = _load_bench()
    w, r, local = bench.dist_info()
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(w)
        slowest = bench.max_over_ranks(1.25 + 3.0 * rank, w)
        bench.barrier(w)
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(f"{w} {r} {local} {slowest}\n")


def test_two_gloo_ranks_max_and_barrier(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        w, r, local, slowest = open(tmp_path / f"rank{rank}.txt").read().split()
        assert (int(w), int(r), int(local)) == (world, rank, rank)
        assert float(slowest) == pytest.approx(4.25)


def test_single_rank_helpers_are_identities(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    bench = _load_bench()
    assert bench.dist_info() == (1, 0, 0)
    assert bench.max_over_ranks(2.5, 1) == 2.5
    bench.barrier(1)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench = _load_bench()
    args = bench.parse(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"])
    assert bench.reference_arm(args) == 0
    assert capsys.readouterr().out == ""
