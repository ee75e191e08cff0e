"""Multi-process plumbing of bench.py on CPU (gloo, world size 2): the path does not shard across GPUs (every
rank runs its own replica of the batch, no collective on the data path), so what runs across ranks is the
timing reduction (max over ranks) and the whole-job aggregation (units of all ranks over the slowest time)."""
import os
import tempfile

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _worker(rank, world, store_path, times, q):
    # File rendezvous: no TCP port to pick, so nothing else on the machine can take it between the pick and
    # the bind (bench.py itself uses torchrun's env:// rendezvous, covered by dist_env below).
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"file://{store_path}", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        mx = bench.reduce_max(times[rank], world)
        dist.barrier()
        q.put((rank, mx))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [1.25, 3.5]
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_worker, args=(2, os.path.join(d, "store"), times, q), nprocs=2, join=True)
    got = dict(q.get(timeout=30) for _ in range(2))
    assert got == {0: 3.5, 1: 3.5}


def test_aggregate_is_whole_job_over_slowest_rank():
    # 2 ranks, each 10 units, slowest 2 s: 10 units/s for the whole job
    assert bench.aggregate(10.0, 2, 2.0) == pytest.approx(10.0)
    assert bench.aggregate(5.0, 1, 0.5) == pytest.approx(10.0)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.parse_args(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_line(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"])
    assert bench.run_reference(args) == 0
    import json
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["workload"] == "tiny"


def test_decode_reference_arm_line(monkeypatch, capsys):
    """The decode workloads have their own metric (GB/s of algorithmic bytes); the reference arm times the
    oracle on a few sequences and prints one line."""
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    import json
    assert bench.main(["--impl", "reference", "--workload", "decode_tiny", "--steps", "1", "--warmup", "0"]) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["metric"] == bench.DECODE_METRIC and line["unit"] == "GB/s" and line["value"] > 0
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"


def test_prologue_reference_arm_line(monkeypatch, capsys):
    """The prologue workloads report GB/s of algorithmic bytes (forward + backward); the reference arm times the
    oracle's prologue and its backward on a bounded sample and prints one line."""
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    import json
    assert bench.main(["--impl", "reference", "--workload", "rope_tiny", "--steps", "1", "--warmup", "0"]) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["metric"] == bench.PROLOGUE_METRIC and line["unit"] == "GB/s" and line["value"] > 0
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


@pytest.mark.parametrize("workload", ["decode_tiny", "rope_tiny"])
def test_extra_reference_arms_run_on_rank0_only(monkeypatch, capsys, workload):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--workload", workload, "--gpus", "2", "--steps", "1",
                       "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""
