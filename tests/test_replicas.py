"""The multi-GPU path of bench.py on CPU processes (gloo, world size 2): the
layer exchanges no data across GPUs, so N GPUs run N independent replicas and
the only collective is the maximum of the timings (see bench.init_dist,
barrier, max_over_ranks, replica_value); the reference arm runs on rank 0
alone. No GPU is used."""

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    r, w, _ = bench.init_dist(backend="gloo")
    bench.barrier(w)
    # each rank's timed region: rank 1 is the slow one
    ms = 100.0 + 25.0 * r
    got = bench.max_over_ranks(ms, w)
    value = bench.replica_value(w, 1e12, 10, got)
    with open(os.path.join(outdir, f"rank{r}.txt"), "w") as f:
        f.write(f"{r} {w} {got} {value}\n")
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_replicas_take_the_slowest_time(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    rows = sorted(open(tmp_path / f"rank{i}.txt").read().split() for i in range(2))
    for r, (rank, world, got, value) in enumerate(rows):
        assert int(rank) == r and int(world) == 2
        assert float(got) == 125.0                       # the max over ranks, on every rank
        assert float(value) == pytest.approx(2 * 1e12 * 10 / 0.125 / 1e12)   # whole-job, weak scaling


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_value(1, 2e12, 4, 8.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"])
    args = bench.parse_args()
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""
