"""The benchmark's multi-rank logic on CPU with gloo at world size 2: the barrier, the max over
ranks of the timed duration, rank-0-only output and the reference arm's rank gating.  (On GPUs the
same functions run over NCCL, one replica per GPU; the GEMV itself exchanges nothing.)"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    w, r, local = bench.dist_setup(world)
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    # each rank "measured" a different duration; every rank must see the slowest
    out[rank] = bench.max_over_ranks(1.5 + rank, w)
    bench.barrier(w)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_max_over_ranks_and_barrier_world2():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn")
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)


def test_reference_arm_runs_on_rank_zero_only():
    class Args:
        steps, warmup = 1, 0
    # a non-zero rank leaves without building the workload or touching the oracle
    assert bench.run_reference(Args(), 2, 1) is None


def test_reference_arm_line_at_rank_zero(monkeypatch):
    # the reference arm's JSON line on the 256 x 512 workload: the oracle timed on host cores,
    # with the keys the benchmark contract asks of that arm
    monkeypatch.setattr(bench, "WORKLOAD", "tiny")

    class Args:
        steps, warmup = 2, 1
    line = bench.run_reference(Args(), 1, 0)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert (line["steps"], line["warmup"], line["n_gpus"]) == (2, 1, 1)
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["higher_is_better"] is True
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1
    assert cpu["unit"] == line["unit"] == line["e2e"]["unit"]
    assert line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_cpu_baseline_sample_is_bounded():
    import synth
    wl = synth.make("tiny")
    cpu = bench.cpu_oracle_sample(wl, 0.2)
    assert cpu["kind"] == "oracle" and cpu["unit"] == "GB/s" and cpu["cores"] >= 1
    assert cpu["value"] > 0 and "256 consecutive output rows" in cpu["sample"]
