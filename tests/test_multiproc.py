"""The multi-process path of the bench on CPU: two ranks over gloo (one
process per rank, as torchrun launches them) reduce their step times to the
slowest rank's and rank 0 reports the whole job's rate; the reference arm does
its work on rank 0 only.  The path needs no exchange beyond this timing
reduction (independent replicas)."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slower one
        ms = bench.max_over_ranks(local_ms, torch.device("cpu"), world)
        rate = bench.whole_job_rate(1000.0, world, ms)
        dist.barrier()
        if rank == 0:
            with open(out_path, "w") as f:
                json.dump({"ms": ms, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_to_slowest_and_aggregate(tmp_path):
    out = tmp_path / "r.json"
    mp.start_processes(_rank_main, args=(2, _free_port(), str(out)), nprocs=2, join=True,
                       start_method="spawn")
    r = json.loads(out.read_text())
    assert r["ms"] == pytest.approx(15.0)
    assert r["rate"] == pytest.approx(1000.0 * 2 / 0.015)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5
    assert bench.whole_job_rate(64.0, 1, 2.0) == pytest.approx(32000.0)


def test_reference_arm_idles_on_nonzero_ranks(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    args = bench.argparse.Namespace(gpus=2, steps=1, warmup=0, seed=0)
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""
