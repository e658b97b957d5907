"""The benchmark's multi-rank host logic on CPU: two gloo ranks agree on the
slowest rank's time, the job value counts every rank's tokens, ranks draw
different prompts, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, local_ms, out):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.slowest_rank_ms(local_ms[rank], world, torch.device("cpu"))
        out.put((rank, ms, bench.job_value(world, 1000, ms)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    local_ms = [12.5, 20.0]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, local_ms, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in got:
        assert ms == max(local_ms)
        assert value == world * 1000 / (max(local_ms) / 1e3)


def test_single_rank_needs_no_process_group():
    assert bench.slowest_rank_ms(7.0, 1, None) == 7.0
    assert bench.job_value(1, 128, 250.0) == 512.0


def test_ranks_draw_different_prompts():
    wl = synth.WORKLOADS["llama1b_b1"]
    p0 = synth.make_prompts(wl.model.vocab, wl.batch, 16, wl.prompt_seed + 17 * 0)
    p1 = synth.make_prompts(wl.model.vocab, wl.batch, 16, wl.prompt_seed + 17 * 1)
    assert not np.array_equal(p0, p1)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    assert bench.run_reference(bench.parse()) == 0
    assert capsys.readouterr().out == ""
