"""Host-side logic of bench.py, on CPU: the multi-rank timing reduction under a
world-size-2 gloo group, the reference arm's rank behaviour, and the
algorithmic work figures the roofline divides by."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(dist)
        # each rank's device time differs; the job time is the slowest rank's
        ms = bench.max_over_ranks(dist, 10.0 + 5.0 * rank, torch.device("cpu"))
        bench.barrier(dist)
        out.put((rank, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_world_size_2_gloo():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(out.get(timeout=5) for _ in range(2))
    assert got == {0: 15.0, 1: 15.0}


def _run_reference(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "2", "--warmup", "3"], env=env, capture_output=True,
                          text=True, timeout=600)


def test_reference_arm_rank0_prints_other_ranks_silent():
    r1 = _run_reference({"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_reference({"RANK": "0", "LOCAL_RANK": "0", "WORLD_SIZE": "2"})
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0


def test_algorithmic_work_figures():
    flops, bytes_, T = bench.prefill_work()
    assert T == 16384
    # per token H(2QP + 4NP) + G 2QN = 128 (16384 + 32768) + 8 * 32768
    assert flops == 16384 * 6553600
    # x 16384 + B, C 4096 + dt 512 + bf16 y 16384 per token, plus the fp32 final state
    assert bytes_ == 16384 * 37376 + 4 * 128 * 64 * 128 * 4 + 2 * 128 * 4
    _, dbytes, b = bench.decode_work()
    assert b == 64 and dbytes == 2 * 536870912 + 2097152 + 262144 + 65536 + 2048 + 2097152


def test_traffic_entry_requires_matching_source_hash(tmp_path, monkeypatch):
    # a kernel whose source changed since the capture reports no traffic
    monkeypatch.setattr(bench, "kernel_source_hash", lambda f: "0000000000000000")
    assert bench.measured_traffic("ssd_chunk_scan", "scan_tc.cu") is None


def test_oracle_sample_reports_measured_and_scaled_time():
    """The reference arm's step is a bounded sample: the sample's own time
    (what ms_per_step reports) and its scaling to one full step (what the
    tokens/s value uses) both come back, the second at least the first."""
    import bench
    step_s, desc, cores, took = bench.oracle_step_sample(5, 64, 2, 1)
    assert 0 < took <= step_s
    assert cores >= 1 and "scaled to one full step" in desc
