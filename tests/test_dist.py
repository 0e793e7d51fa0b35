"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the step time
is the maximum over ranks and the whole-job rate counts every rank's work.
The path shards into independent replicas, so there is no data-path
collective to test; only the timing reduction crosses ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        local_ms = 1.0 + rank * 0.5   # rank 1 is the slow one
        ms = bench.reduce_step_time(local_ms, device="cpu")
        rate = bench.whole_job_rate(210.125e9, ws, ms)
        q.put((rank, ws, r, local, ms, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ws, r, local, ms, rate in res:
        assert ws == 2 and r == rank and local == rank
        assert ms == pytest.approx(1.5)          # max over ranks
        assert rate == pytest.approx(2 * 210.125e9 / 1.5e-3)


def test_single_process_needs_no_group():
    import bench
    assert bench.reduce_step_time(2.5) == 2.5
    assert bench.whole_job_rate(10.0, 1, 1000.0) == pytest.approx(10.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0", "--gpus", "2"]) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_line(monkeypatch, capsys):
    import json

    import bench
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "1"]) == 0
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


@pytest.mark.parametrize("workload,metric_word", [("q8_tiny", "Q8_0"), ("drafter", "drafter"), ("verify", "verify")])
def test_reference_arm_small_workloads(monkeypatch, capsys, workload, metric_word):
    """The whole-step oracle of the decoder-side workloads, same line format."""
    import json

    import bench
    for key in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(key, raising=False)
    assert bench.main(["--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "0"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and metric_word in line["metric"] and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
