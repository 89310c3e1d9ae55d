"""Multi-GPU bookkeeping of bench.py on two CPU processes over gloo (no GPU needed).

The layer runs as independent replicas, one per GPU: the process group carries only the
barriers around the timed region and the max over ranks of the measured times.  These tests run
that code path with world_size 2: both ranks see the slower rank's time, the whole-job value
counts every replica's tokens, and the reference arm's non-zero ranks exit without work.
"""
import contextlib
import io
import multiprocessing as mp
import os
import socket
import types

import pytest


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, step_ms, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r = bench.Replicas("gloo", timeout_s=60)
    r.barrier()
    m = r.max_over_ranks(step_ms[rank])
    v = bench.replica_value(r.world, 1, m)
    q.put((rank, r.world, m, v))
    r.close()


def test_two_replicas_share_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    step_ms = [0.125, 0.25]                     # rank 1 is the slower replica
    ps = [ctx.Process(target=_worker, args=(r, 2, port, step_ms, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
    for p in ps:
        if p.is_alive():
            p.kill()
    assert [p.exitcode for p in ps] == [0, 0]
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, world, m, v in res:
        assert world == 2
        assert m == 0.25                        # max over ranks, on every rank
        assert v == pytest.approx(2 * 1 / 0.25e-3)   # both replicas' tokens over that time


def test_single_process_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    r = bench.Replicas("gloo")
    assert (r.world, r.rank) == (1, 0)
    assert r.max_over_ranks(3.5) == 3.5
    r.barrier()
    r.close()
    assert bench.replica_value(1, 4, 2.0) == pytest.approx(2000.0)


def test_reference_arm_nonzero_rank_does_no_work(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    import bench
    args = types.SimpleNamespace(workload="mixtral_8x7b:1", steps=1, warmup=0,
                                 cpu_sample_rows=None)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        assert bench.run_reference(args) is None
    assert out.getvalue() == ""


def test_reference_arm_line_keeps_the_contract(monkeypatch):
    # rank 0 of the reference arm (the oracle timed on the host) prints one JSON line with the
    # keys the bench contract asks for; tiny layer, one step
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    import json

    import bench
    args = types.SimpleNamespace(workload="tiny:4", steps=1, warmup=0, cpu_sample_rows=None,
                                 affinity=False, no_rewrite=False)
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        bench.run_reference(args)
    lines = [ln for ln in out.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]
    assert "T=4" in d["config"]["workload"]
