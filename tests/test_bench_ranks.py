"""The multi-process side of bench.py on CPU: two gloo ranks (no GPU).

With --gpus N every rank runs the whole workload on its own GPU (replicas, weak
scaling) and the only exchange is the timing: the slowest rank's time decides,
and the reported value counts the keys of all ranks.
"""

from __future__ import annotations

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, results):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        e2e = bench.max_over_ranks(2 * times[rank], dist, torch.device("cpu"))
        results[rank] = (ms, e2e)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    times = [3.25, 7.5]
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), times, results), nprocs=world,
                           start_method="spawn", join=True)
        got = dict(results)
    assert got[0] == got[1] == (7.5, 15.0)


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(4.0, None, None) == 4.0


def test_result_line_counts_all_ranks():
    n, steps = 1000, 10
    kw = dict(n=n, steps=steps, warmup=3, ms=20.0, q_ms=1.5, l_ms=0.4, e2e_ms=8.0, h2d=123, d2h=45,
              clocks={"sm_mhz": 1.0, "sm_max_mhz": 1.0, "reasons": []})
    one = bench.result_line(world=1, **kw)
    two = bench.result_line(world=2, **kw)
    # per-step time is the slowest rank's; the value counts every rank's keys
    assert one["ms_per_step"] == two["ms_per_step"] == pytest.approx(2.0)
    assert one["value"] == pytest.approx(n / 2.0 * 1e3)
    assert two["value"] == pytest.approx(2 * one["value"])
    assert two["e2e"]["value"] == pytest.approx(2 * n / 8.0 * 1e3)
    assert two["n_gpus"] == 2 and two["scaling"] == "weak"
    assert two["config"]["global_batch"] == 2 * bench.B
    assert two["config"]["parallelism"] == "replicas x2"
    # the dominant kernel's roofline uses the algorithmic bytes per key
    assert one["roofline"]["kernel"] == "tq_quantize"
    bpk = bench.bytes_per_key()
    assert one["roofline"]["achieved"] == pytest.approx(n * (bpk["quantize_in"] + bpk["quantize_out"]) / 1.5 / 1e6)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in one


def test_reference_arm_other_ranks_do_no_work(capsys):
    class Args:
        steps, warmup, gpus = 1, 0, 2

    assert bench.run_reference(Args, rank=1) == 0
    assert capsys.readouterr().out == ""
