"""The benchmark's multi-rank harness on the CPU: world size 2 over gloo.

The step itself has no exchange between GPUs (the Nd data-parallel ranks are
simulated inside one GPU), so N GPUs run independent replicas.  What is shared
is the harness: the slowest rank's time sets the whole-job throughput, every
rank takes the same collective steps, and only rank 0 reports."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        owned, steps = 1_557_611_200, 50
        ms_local = 400.0 + 100.0 * rank          # rank 1 is the slower one
        ms_max, value = bench.aggregate(owned, steps, ms_local, world, device="cpu")
        kernel_max = bench.max_over_ranks(9.8 - rank, world, device="cpu")
        out.put((rank, ms_max, value, kernel_max))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_over_the_slowest():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, value, kernel_max in results:
        assert ms_max == 500.0
        assert value == pytest.approx(2 * 1_557_611_200 * 50 / 0.5)
        assert kernel_max == pytest.approx(9.8)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    ms_max, value = bench.aggregate(1000, 10, 20.0, 1)
    assert ms_max == 20.0 and value == pytest.approx(1000 * 10 / 0.02)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, ref_sample, storage = 1, 3, 1000, "fp16"
    wl = bench._workloads()["gpt2-1.5b-stage2-nd8"]
    assert bench.run_reference(Args, "gpt2-1.5b-stage2-nd8", wl) == 0
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    assert bench.run_reference(Args, "gpt2-1.5b-stage2-nd8", wl) == 0
    import json
    line = json.loads(capsys.readouterr().out)
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
