"""World-size-2 checks of the benchmark's multi-rank plumbing on CPU (gloo): rendezvous, barrier,
max-over-ranks timing and the weak-scaling aggregate.  The data path itself has no collective:
every rank runs its own copy of the problem."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(0.5 + rank, world, torch.device("cpu"))
        units = bench.aggregate_weak(10.0, world)
        out[rank] = (t, units)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == (1.5, 20.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    import bench

    class A:
        workload = "tiny"
        steps = 1
        warmup = 0

    assert bench.run_reference(A(), 2, 1) is None


def test_reference_arm_prints_the_contract_line():
    # the driver parses this line: one JSON object with the contract's keys, on the host cores
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["config"]["workload"] == "prefill_gate_up"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0


def test_clock_summary_uses_the_samples_under_load():
    """The bench reports the median SM clock of the samples taken under load (power at least half the
    window's maximum): the idle moments around the timed region run at the top clock and must not
    hide a power-capped clock; throttle reasons seen anywhere in the window are reported."""
    import bench
    c = bench.ClockSampler(0)
    c.out = ("0, 1965, 1965, 120.5, 0x0, Not Active, Not Active, Not Active, Not Active\n"
             "0, 1500, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active\n"
             "0, 1450, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n"
             "0, 1965, 1965, 130.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    s = c.summary()
    assert s["sm_mhz"] == 1475.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples_under_load"] == 2
    c.out = ""
    assert c.summary()["reasons"] == ["unsampled"]
