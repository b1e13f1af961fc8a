"""Host logic of the multi-rank bench on CPU: two gloo ranks take the element-wise max
of their timings (the job's time is the slowest rank's), the whole-job rate counts
every rank's tokens, and the reference arm runs on rank 0 alone."""

import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        # rank 0 is slower on the first timing, rank 1 on the second
        out = bench.max_over_ranks([100.0 + 7.0 * (rank == 0), 40.0 + 3.0 * (rank == 1)], ws, "cpu")
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: [107.0, 43.0], 1: [107.0, 43.0]}


def test_max_over_ranks_on_one_rank_is_identity():
    assert bench.max_over_ranks([3.5, 1.25], 1, "cpu") == [3.5, 1.25]


def test_job_rate_counts_every_rank():
    # 2 ranks x 32768 tokens x 5 steps in 0.5 ms of the slowest rank
    assert bench.job_rate(2, 32768, 5, 0.5) == pytest.approx(2 * 32768 * 5 / 0.5e-3)
    assert bench.job_rate(1, 100, 1, 1000.0) == pytest.approx(100.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        warmup, steps, gpus, layers = 3, 1, 2, 1

    assert bench.run_reference(Args(), bench.get_config("c0_tiny")) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    """The reference arm (the fp64 oracle on host cores) prints one JSON line with the
    driver's keys, on the tiny workload."""
    import json
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    import time
    t0 = time.perf_counter()
    assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "3", "--workload", "c0_tiny"]) == 0
    wall = time.perf_counter() - t0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "c0_tiny"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    # whole steps are timed, nothing is extrapolated: the claimed timed region fits in the run
    assert d["ms_per_step"] * d["steps"] / 1e3 <= wall
    assert "nothing extrapolated" in d["cpu_baseline"]["sample"]
