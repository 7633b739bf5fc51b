"""The N > 1 host logic of bench.py on CPU: two ranks over gloo.

The decode path does not shard (one sequence's attention is one GPU's work),
so N GPUs run N independent replicas.  What runs on more than one rank is
the host logic: the barriers around the timed region, every time taken as
the max over ranks, the whole-job value over all ranks' bytes, only rank 0
printing, and the reference arm running on rank 0 alone.  The same functions
run here with the gloo backend and world size 2.
"""
import importlib.util
import json
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    bench = _load_bench()
    bench.init_distributed(torch, "gloo", rank)
    try:
        bench.barrier()
        # rank r timed 4 steps of (1 + r) ms; its e2e and eager steps take 2 + r and 1.5 + r
        dec = {"step_ms": [1.0 + rank] * 4, "e2e_ms": [2.0 + rank] * 4,
               "eager_ms": [1.5 + rank] * 4}
        tot = bench.replica_totals(torch, dec, steps=4, world=world, step_bytes=1e9)
        bench.barrier()
        out_q.put((rank, tot))
    finally:
        bench._dist.destroy_process_group()


def test_replica_totals_take_the_max_over_ranks():
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
    assert got[0] == got[1]                       # every rank reports the same figures
    tot = got[0]
    # the slowest rank (rank 1: 2 ms per step) sets the time; 2 ranks x 1e9 bytes per step
    assert tot["ms_per_step"] == pytest.approx(2.0)
    assert tot["value"] == pytest.approx(2 * 1e9 / 2e-3 / 1e9)
    assert tot["e2e_ms"] == pytest.approx(3.0)
    assert tot["e2e_value"] == pytest.approx(2 * 1e9 / 3e-3 / 1e9)
    assert tot["eager_ms"] == pytest.approx(2.5)


def test_single_rank_needs_no_process_group():
    import torch
    bench = _load_bench()
    assert bench._dist is None
    bench.barrier()                               # a no-op without a group
    assert bench.max_over_ranks(torch, 3.25) == 3.25
    tot = bench.replica_totals(torch, {"step_ms": [1.0, 3.0], "e2e_ms": [4.0, 4.0],
                                       "eager_ms": [2.0, 2.0]}, steps=2, world=1, step_bytes=5e8)
    assert tot["ms_per_step"] == pytest.approx(2.0)
    assert tot["value"] == pytest.approx(5e8 / 2e-3 / 1e9)


def test_reference_arm_runs_on_rank_0_only(monkeypatch, capsys):
    """Under torchrun every rank starts `bench.py --impl reference`; ranks
    other than 0 exit at once without work and print nothing."""
    bench = _load_bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    called = []
    monkeypatch.setattr(bench, "decode_workload", lambda: called.append(1))
    assert bench.main() == 0
    assert called == []
    assert capsys.readouterr().out == ""
