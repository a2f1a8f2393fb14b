"""The N > 1 host logic of bench.py on CPU: world-size-2 gloo ranks.

The decode path shards by tensor (every rank decodes its own weight matrix, as
the layers of a model are independent problems), so the only cross-rank step
is the timing reduction: every rank's step time goes through a max, and the
whole-job throughput is every rank's weights over that slowest time.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r is slower on the first value and faster on the second
        got = bench.reduce_max([1.0 + rank, 10.0 - rank, 0.5], world)
        # a second reduction in the same order, as bench.py takes one for the e2e time
        (e2e,) = bench.reduce_max([3.0 * (rank + 1)], world)
        dist.barrier()
        q.put((rank, got, e2e))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, got, e2e = q.get(timeout=120)
        out[rank] = (got, e2e)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the same maxima: the slowest rank's time per value
    for rank in range(world):
        assert out[rank][0] == [2.0, 10.0, 0.5]
        assert out[rank][1] == 6.0


def test_reduce_max_one_rank_is_identity():
    assert bench.reduce_max([1.5, 2], 1) == [1.5, 2.0]


def test_weak_value_counts_every_rank():
    numel = 3840 * 10240
    one = bench.weak_value(1, numel, 0.1)
    assert one == pytest.approx(numel / 1e-4 / 1e9)
    # weak scaling: N ranks, each with the same work, at the same slowest time: N times the value
    assert bench.weak_value(4, numel, 0.1) == pytest.approx(4 * one)
    # a slower slowest rank lowers the whole job's value
    assert bench.weak_value(2, numel, 0.2) == pytest.approx(one)


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    """Under torchrun the reference arm runs on rank 0 alone; the other ranks exit without work."""
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                                      "--warmup", "3"])
    called = []
    monkeypatch.setattr(bench, "run_reference", lambda args, world: called.append(args) or {})
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main()
    assert buf.getvalue() == "" and not called


def test_reference_arm_rank_zero_prints_one_line(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "0")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                                      "--warmup", "3"])
    monkeypatch.setattr(bench, "run_reference", lambda args, world: {"impl": "reference", "n_gpus": world})
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main()
    lines = buf.getvalue().strip().splitlines()
    assert len(lines) == 1 and json.loads(lines[0]) == {"impl": "reference", "n_gpus": 2}


def test_warmup_below_three_is_refused(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", "--warmup", "2"])
    with pytest.raises(SystemExit):
        bench.main()


def test_ranks_decode_distinct_tensors():
    from dit_weight_compression_ep_b200 import synth

    a, b = synth.headline(seed=7 + 0), synth.headline(seed=7 + 1)
    assert (a.rows, a.cols) == (b.rows, b.cols) and a.seed != b.seed


def test_gpus_must_match_the_launched_ranks(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "0")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--warmup", "3"])
    with pytest.raises(SystemExit):
        bench.main()


def test_gpus_two_without_a_launcher_starts_two_ranks(monkeypatch):
    """bench.py --gpus 2 run directly re-launches itself as two ranks; nothing runs here."""
    seen = []
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "2", "--steps", "5", "--warmup", "3"])
    monkeypatch.setattr(bench, "relaunch", lambda n, script, argv: seen.append((n, script, list(argv))) or
                        type("R", (), {"returncode": 0})())
    with pytest.raises(SystemExit) as ex:
        bench.main()
    assert ex.value.code == 0
    assert seen == [(2, os.path.abspath(bench.__file__), ["--gpus", "2", "--steps", "5", "--warmup", "3"])]


def test_relaunch_runs_two_gloo_ranks_with_the_timing_reduction():
    """The launch path itself: two ranks under torchrun on CPU (gloo), each timing its own step,
    the max over ranks taken by bench.reduce_max, one JSON line from rank 0 with n_gpus = 2."""
    probe = os.path.join(os.path.dirname(os.path.abspath(__file__)), "rank_probe.py")
    res = bench.relaunch(2, probe, ["--units", "1000000"], timeout_s=300, capture=True)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    out = json.loads(lines[0])
    assert out["n_gpus"] == 2 and out["ranks_seen"] == 2
    # rank 1 sleeps longer: the step time is the slower rank's, the value counts both ranks' units
    assert out["ms_per_step"] >= out["rank_ms"][1] >= out["rank_ms"][0]
    assert out["value"] == pytest.approx(bench.weak_value(2, 1000000, out["ms_per_step"]))


def test_workload_option_names_its_target_and_description():
    import argparse

    head = bench._workload(argparse.Namespace(workload="headline"))
    assert head == (bench.TARGET, bench.WORKLOAD)
    for name, (bpp, desc) in bench.OTHER_WORKLOADS.items():
        assert bench._workload(argparse.Namespace(workload=name)) == (bpp, desc)
        assert "8 bpp" in desc and "b = 12" in desc


def test_reference_arm_refuses_other_workloads(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "dit-qkv-8", "--warmup", "3"])
    with pytest.raises(SystemExit):
        bench.main()
