"""Host-side logic of bench.py that runs without a GPU: the max-over-ranks reduction with
world_size 2 on gloo, the reference arm under torchrun (only rank 0 prints, the other rank
exits 0 without work), and the clock-log parser."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q.put((rank, bench.reduce_max(10.0 + 5 * rank, "cpu")))
    finally:
        torch.distributed.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def test_reduce_max_without_process_group_is_identity():
    assert bench.reduce_max(3.5, "cpu") == 3.5


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--workload", "large_e2", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["n_gpus"] == 2


def test_clock_parser_reports_reasons_and_median():
    log = "\n".join([
        "0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1300, 1965, 998.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1320, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1340, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active",
    ])
    c = bench.ClockSampler.parse(log)
    assert c["sm_max_mhz"] == 1965.0 and c["reasons"] == ["sw_power_cap"]
    assert c["sm_mhz"] == 1330.0 and c["samples"] == 4
    assert bench.ClockSampler.parse("") is None


def test_nvml_sampler_summary_decodes_reason_bits():
    """The in-process NVML sampler's summary, on samples a fake NVML would return (no GPU):
    median SM clock, and the clock-event reason bits decoded by name."""
    s = bench.NvmlClockSampler.__new__(bench.NvmlClockSampler)
    s.stop_flag = bench.threading.Event()
    s.thread = None
    s.max_mhz = 1965
    s.samples = [(0.0, 1965, 0x0), (1.0, 1310, 0x4), (2.0, 1290, 0x4), (3.0, 1300, 0x4 | 0x8)]
    c = s.stop()
    assert c["sm_mhz"] == 1305.0 and c["sm_max_mhz"] == 1965.0 and c["samples"] == 4
    assert c["reasons"] == ["hw_slowdown", "sw_power_cap"]
    # only the samples inside the timed region count
    c = s.stop(window=(0.5, 2.5))
    assert c["sm_mhz"] == 1300.0 and c["samples"] == 2 and c["reasons"] == ["sw_power_cap"]
    s.samples = []
    assert s.stop() is None
