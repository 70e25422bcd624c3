"""Host logic of the N>1 bench path, run as two gloo ranks on the CPU.

The layer has no data-path collective: ``bench.py --gpus N`` runs one
independent replica per GPU.  The only cross-rank steps are a barrier around
the timed region and the maximum of the per-rank device times; throughput
counts every rank's units over the slowest rank's time.
"""
import datetime
import multiprocessing as mp
import os
import socket

import pytest

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports (1 + r, 10 - r) ms: the maxima are (world, 10)
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank], world)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    assert all(p.exitcode == 0 for p in procs)
    results = dict(q.get(timeout=5) for _ in procs)
    assert results == {0: [2.0, 10.0], 1: [2.0, 10.0]}


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks([3.0, 4.5], 1) == [3.0, 4.5]


def test_whole_job_throughput_counts_every_rank():
    # 2 ranks x 10 steps x 1e12 FLOP over the slowest rank's 1000 ms
    assert bench.whole_job_tflops(2, 1e12, 10, 1000.0) == pytest.approx(20.0)
    # weak scaling: same per-rank time -> throughput grows with the rank count
    one = bench.whole_job_tflops(1, 2.66e11, 100, 11.17)
    four = bench.whole_job_tflops(4, 2.66e11, 100, 11.17)
    assert four == pytest.approx(4 * one)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup, ref_rows, ref_cols = 1, 3, 8, 8

    assert bench.run_reference(Args()) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_rank_zero(monkeypatch, capsys):
    """Rank 0 times the oracle on a small sample of the same workload and
    prints one line with the main arm's metric, the reference marker, its
    own CPU-baseline description and a zero-copy end-to-end figure."""
    import json
    monkeypatch.setenv("RANK", "0")

    class Args:
        steps, warmup, ref_rows, ref_cols = 1, 3, 16, 32

    bench.run_reference(Args())
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOPS"
    assert d["value"] > 0 and d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"] == bench.WORKLOAD["workload"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and "16 of" in cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
