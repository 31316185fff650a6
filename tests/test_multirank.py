"""The multi-rank host path of bench.py on CPU: two gloo ranks, as torchrun
would start them, take the same collective steps and agree on the slowest
rank's time; the whole-job rate counts every replica's queries."""
import json
import multiprocessing as mp
import os
import socket
import sys
import types

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# per-rank times (ms) of the three timed regions, in the order bench.py reduces them
RANK_TIMES = {0: (10.0, 31.0, 7.5), 1: (12.5, 29.0, 8.0)}


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        got = [bench.max_over_ranks(dist, torch.device("cpu"), ms) for ms in RANK_TIMES[rank]]
        dist.barrier()
        out.put((rank, got, bench.whole_job_rate(32, 20, world, got[0])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(world):
            rank, got, rate = out.get(timeout=120)
            results[rank] = (got, rate)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    want = [max(RANK_TIMES[r][i] for r in range(world)) for i in range(3)]
    for rank in range(world):
        got, rate = results[rank]
        assert got == want
        # 2 replicas x 32 queries x 20 steps in 12.5 ms
        assert rate == pytest.approx(2 * 32 * 20 / 12.5e-3)


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(None, torch.device("cpu"), 3.25) == 3.25
    assert bench.whole_job_rate(32, 20, 1, 10.0) == pytest.approx(64000.0)


def test_reference_arm_prints_on_rank_zero_only(capsys, monkeypatch):
    """Under torchrun the reference arm runs on rank 0 alone; the other ranks exit without work."""
    calls = []
    monkeypatch.setattr(bench, "cpu_baseline", lambda *a, **k: calls.append(a) or {})
    args = types.SimpleNamespace(steps=2, warmup=1, cpu_sample_queries=1, gpus=2)
    bench.run_reference(args, None, 1)
    assert capsys.readouterr().out == "" and calls == []


def test_reference_arm_line(capsys, monkeypatch):
    from sparse_gated_attention_b200 import synth

    fake = {"value": 1.0, "unit": bench.UNIT, "cores": 4, "kind": "oracle", "sample": "s", "seconds": 0.5}
    monkeypatch.setattr(bench, "cpu_baseline", lambda *a, **k: dict(fake))
    args = types.SimpleNamespace(steps=3, warmup=1, cpu_sample_queries=1, gpus=1)
    bench.run_reference(args, synth.WORKLOADS[synth.HEADLINE], 0)
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["value"] == pytest.approx(2.0)  # 1 query per 0.5 s
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["cpu_baseline"]["kind"] == "oracle" and line["config"]["workload"] == synth.HEADLINE


def test_replicas_draw_their_own_batches():
    from sparse_gated_attention_b200 import synth

    wl = synth.custom(batch=1, n_q=1, ctx=64, first_pos=63, name="tiny")
    a, b = synth.make_inputs(wl, seed=0), synth.make_inputs(wl, seed=1)
    assert not torch.equal(a["kv"], b["kv"])
