"""The multi-rank host logic of bench.py on CPU (gloo, world size 2): the
job's time is the max over ranks, and the reference arm prints one line from
rank 0 while the other ranks exit without work."""

import importlib.util
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        # rank r measured (1 + r, 10 - r, 0.5 * r) seconds
        got = b.reduce_max([1.0 + rank, 10.0 - rank, 0.5 * rank], dist, torch.device("cpu"))
        q.put((rank, got))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[0] == res[1] == [2.0, 10.0, 0.5]


def test_reduce_max_without_process_group():
    assert _bench().reduce_max([3, 1.5], None, None) == [3.0, 1.5]


@pytest.mark.timeout(600)
def test_reference_arm_two_ranks_prints_one_line():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "3",
           "--ref-step-seconds", "0.3"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=560)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["value"] == d["value"] and d["cpu_baseline"]["kind"] == "oracle"


def test_clock_parse_reports_median_and_active_reasons():
    b = _bench()
    lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1700, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1720, 1965, 999.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    r = b.ClockSampler.parse(lines)
    assert r["samples"] == 3 and r["sm_mhz"] == 1720.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    r = b.ClockSampler.parse(["0, 1200, 1965, 500, 0x0, Active, Not Active, Active, Not Active"])
    assert r["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert b.ClockSampler.parse([])["sm_mhz"] is None
