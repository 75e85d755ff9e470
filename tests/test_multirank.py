"""The multi-rank path of bench.py on CPU: two gloo ranks reduce their timed lengths to the
max and report the whole-job rate; the reference arm does its work on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bench():
    sys.path.insert(0, ROOT)
    import importlib.util

    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rank(rank, world, port, out):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        ms = b.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")  # rank 1 is the slow one
        out[rank] = (ms, b.whole_job_rate(world, 4, 50, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # 2 ranks x 4 queries x 50 steps in 15 ms
    assert res[0][1] == pytest.approx(2 * 4 * 50 / 0.015)


def test_single_rank_is_unchanged():
    b = _bench()
    assert b.max_over_ranks(12.5, 1, "cpu") == 12.5
    assert b.whole_job_rate(1, 4, 10, 2.0) == pytest.approx(4 * 10 / 0.002)


def test_reference_arm_does_nothing_on_other_ranks(monkeypatch, capsys):
    b = _bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1"])
    assert b.main() == 0
    assert capsys.readouterr().out == ""
