#!/usr/bin/env python
"""Throughput of the Mamba-2 selective-scan hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  * prefill: ssd_chunk_scan over 4 sequences x 4096 tokens, 128 heads,
    head_dim 64, d_state 128, 8 groups, 128-token chunks, bf16 x/B/C, fp32 dt,
    bf16 y, fp32 final state (zero initial state);
  * decode: one ssm_state_update token for a batch of 64 at the Nemotron-3
    Ultra layer shape (256 heads, head_dim 64, d_state 128, 8 groups), in place
    on a 512 MiB fp32 state, bf16 x/B/C, bf16 y; per-step inputs cycle through
    a ring of 8 seeded input sets.
``value`` is tokens/s over both (16384 prefill + 64 decode tokens per step and
per GPU); the numbers the metric names (prefill ms, TFLOP/s and % of tensor
peak, decode GB/s and % of HBM peak) are top-level keys of the headline line.
Timed beside the step: the long prefill at the Ultra layer shape (1 x 32768
tokens, 256 heads, nonzero initial state) and the mixed workload (8 packed
sequences of 512..16384 tokens, then 128 decode steps), both summarised in the
headline; the causal conv1d that feeds the scan, speculative decode, the
fused steps and fp16 state pools, detailed on a separate JSON line printed
just before the headline (``bench_parts``).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun each rank runs its own batch (weak scaling, no data-path
collective); timing is max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("Mamba-2 prefill SSD tokens/s (% tensor peak); "
          "decode update HBM GB/s (% peak)")
PREFILL = dict(nseq=4, seqlen=4096, H=128, P=64, N=128, G=8, Q=128)
DECODE = dict(batch=64, H=256, P=64, N=128, G=8)
RING = 8

# Fallback roofline denominators (used only if MEASURED_PEAKS.json is absent).
FALLBACK_PEAKS = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Long prefill at the Ultra layer shape (nonzero initial state, bf16 y) and
# the mixed prefill-then-decode workload (8 packed sequences of seeded
# lengths, then 128 decode steps each): timed beside the step.
ULTRA32K = dict(nseq=1, seqlen=32768, H=256, P=64, N=128, G=8, Q=128, h0=True)
MIXED = dict(nseq=8, lo=512, hi=16384, H=128, P=64, N=128, G=8, Q=128, decode_steps=128)


def prefill_work(p=PREFILL, y_bytes=2, T=None):
    """Algorithmic flops and bytes of one prefill launch.

    flops per token = H(2QP + 4NP) + G*2QN (full Q x Q masked tile, the four
    per-head contractions C.B^T-masked.X, X^T.B, C.H^T and the group's C.B^T);
    bytes = x + B + C + dt + y per token, plus the fp32 final state (and the
    initial state when the workload has one).
    """
    T = p["nseq"] * p["seqlen"] if T is None else T
    H, P, N, G, Q = p["H"], p["P"], p["N"], p["G"], p["Q"]
    flops = T * (H * (2 * Q * P + 4 * N * P) + G * 2 * Q * N)
    per_tok = H * P * 2 + 2 * G * N * 2 + H * 4 + H * P * y_bytes
    states = 2 if p.get("h0") else 1
    bytes_ = T * per_tok + states * p["nseq"] * H * P * N * 4 + 2 * H * 4
    return flops, bytes_, T


def decode_work(d=DECODE, y_bytes=2):
    """Algorithmic bytes of one decode launch: state read + write, x, B, C, dt,
    A, D, y.  ~5 flops per state element (plain ALU work)."""
    b, H, P, N, G = d["batch"], d["H"], d["P"], d["N"], d["G"]
    state = b * H * P * N * 4
    bytes_ = 2 * state + b * H * P * 2 + 2 * b * G * N * 2 + b * H * 4 + 2 * H * 4 + b * H * P * y_bytes
    flops = 5 * b * H * P * N
    return flops, bytes_, b


def kernel_source_hash(fname):
    path = os.path.join(ROOT, "hybrid_mamba_ssm_b200", "csrc", fname)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def measured_traffic(kernel, source_file):
    """DRAM bytes (read + write) per launch of the benchmark's own launch, from
    the committed ncu summary, or None if the kernel's source changed since the
    counters were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash(source_file)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel:
                if parts[1] == want:
                    return float(parts[2])
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.gpu_id:
            cmd.insert(1, f"--id={self.gpu_id}")
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                c = [x.strip() for x in line.split(",")]
                if len(c) >= 9:
                    rows.append(c)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def gpu_uuid(dev):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if args.impl == "reference":
        return world, rank, local, None   # rank 0 alone times the oracle
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    else:
        torch.cuda.set_device(local)
    return world, rank, local, pg


def max_over_ranks(pg, value, device):
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg, device=None):
    if pg is not None:
        if device is not None:
            pg.barrier(device_ids=[device.index])
        else:
            pg.barrier()


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and --impl reference)
# ---------------------------------------------------------------------------
def oracle_step_sample(rank_seed, prefill_tokens, prefill_heads, decode_rows):
    """Time the oracle on a bounded sample of one step; returns (seconds for a
    full step, scaled from the sample, description, threads, seconds the
    sample itself took)."""
    import oracle
    from hybrid_mamba_ssm_b200 import inputs as synth
    oracle.set_num_threads(os.cpu_count() or 1)
    p, d = PREFILL, DECODE
    inp = synth.make_scan_inputs(rank_seed, [prefill_tokens], prefill_heads, p["P"], p["N"],
                                 1, dtype="bf16")
    t = time.perf_counter()
    oracle.scan(inp.x.values, inp.dt, inp.A, inp.B.values, inp.C.values, inp.D, None)
    t_pre = time.perf_counter() - t
    A, D = synth.make_head_params(rank_seed + 1, d["H"])
    st = synth.make_state(rank_seed + 2, (decode_rows, d["H"], d["P"], d["N"]))
    dec = synth.make_decode_step(rank_seed + 3, decode_rows, d["H"], d["P"], d["N"], d["G"])
    t = time.perf_counter()
    oracle.state_update(st, dec.x.values, dec.dt, A, dec.B.values, dec.C.values, D)
    t_dec = time.perf_counter() - t
    full_pre = p["nseq"] * p["seqlen"] * p["H"]
    scale_pre = full_pre / (prefill_tokens * prefill_heads)
    scale_dec = d["batch"] / decode_rows
    step_s = t_pre * scale_pre + t_dec * scale_dec
    desc = (f"prefill {prefill_tokens} tokens x {prefill_heads} heads (of 16384 x 128) and "
            f"decode {decode_rows} of 64 batch rows x 256 heads, scaled to one full step")
    return step_s, desc, oracle.num_threads(), t_pre + t_dec


CONV_PREFILL = dict(nseq=4, seqlen=4096, dim=128 * 64 + 2 * 8 * 128, width=4)
CONV_DECODE = dict(batch=64, dim=256 * 64 + 2 * 8 * 128, width=4, ring=32)


def conv_prefill_work(c=CONV_PREFILL):
    """Algorithmic bytes of one causal_conv1d_fwd call (bf16 x and y, bf16
    state read and written, fp32 weight and bias)."""
    T = c["nseq"] * c["seqlen"]
    W = c["width"]
    return T * c["dim"] * 4 + 2 * c["nseq"] * c["dim"] * (W - 1) * 2 + c["dim"] * (W + 1) * 4, T


def conv_decode_work(c=CONV_DECODE):
    """Algorithmic bytes of one causal_conv1d_update call: x, y, the state
    window read and written (bf16), weight, bias, slot indices."""
    b, dim, W = c["batch"], c["dim"], c["width"]
    return b * dim * (4 + 4 * (W - 1)) + dim * (W + 1) * 4 + b * 4, b


def time_conv(dev, stream, seed, iters=50):
    """Device time of the conv1d entry points at the benchmark shapes (run
    beside the step, not inside it).  Prefill inputs exceed L2; decode cycles
    through a ring of pool rows and inputs larger than L2."""
    import torch
    from hybrid_mamba_ssm_b200 import inputs as synth
    from hybrid_mamba_ssm_b200 import ssm

    def bf16(t):
        return torch.from_numpy(np.ascontiguousarray(t.bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    cp, cd = CONV_PREFILL, CONV_DECODE
    inp = synth.make_conv_inputs(seed, [cp["seqlen"]] * cp["nseq"], cp["dim"], cp["width"])
    x = bf16(inp.x).view(cp["nseq"], cp["seqlen"], cp["dim"])
    w = torch.from_numpy(inp.weight).to(dev)
    b = torch.from_numpy(inp.bias).to(dev)
    st = bf16(inp.state)
    y = torch.empty_like(x)
    rng = np.random.Generator(np.random.PCG64(seed + 1))
    rows = cd["batch"] * cd["ring"]
    pool = torch.from_numpy(rng.standard_normal((rows, cd["dim"], cd["width"] - 1),
                                                dtype=np.float32)).to(dev).to(torch.bfloat16)
    dx = torch.from_numpy(rng.standard_normal((cd["ring"], cd["batch"], cd["dim"]),
                                              dtype=np.float32)).to(dev).to(torch.bfloat16)
    dw = torch.from_numpy(rng.uniform(-0.5, 0.5, (cd["dim"], cd["width"])).astype(np.float32)).to(dev)
    db = torch.from_numpy(rng.uniform(-0.5, 0.5, cd["dim"]).astype(np.float32)).to(dev)
    slots = torch.arange(rows, dtype=torch.int32, device=dev).view(cd["ring"], cd["batch"])
    dy = torch.empty((cd["batch"], cd["dim"]), dtype=torch.bfloat16, device=dev)

    def pre():
        ssm.causal_conv1d_fwd(x, w, b, conv_state=st, y=y, stream=stream)

    def dec(k):
        ssm.causal_conv1d_update(dx[k % cd["ring"]], dw, db, pool, slot_idx=slots[k % cd["ring"]],
                                 y=dy, stream=stream)

    out = {}
    # prefill: per-launch events (two kernels per call: convolution, state roll)
    for k in range(5):
        pre()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    for k in range(iters):
        ev[k][0].record(stream)
        pre()
        ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / iters
    nbytes, units = conv_prefill_work()
    out["conv1d_prefill"] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
                             "bytes_per_launch": nbytes, "tokens_per_s": units / (ms * 1e-3),
                             "launches": iters}
    # decode: a few microseconds per launch, so the launches are replayed from
    # a CUDA graph (the host's launch rate would otherwise set the time)
    for k in range(5):
        dec(k)
    torch.cuda.synchronize(dev)
    gs = torch.cuda.Stream(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(gs):
        with torch.cuda.graph(graph, stream=gs):
            for k in range(cd["ring"]):
                ssm.causal_conv1d_update(dx[k], dw, db, pool, slot_idx=slots[k], y=dy, stream=gs)
    graph.replay()
    torch.cuda.synchronize(dev)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(1, iters // 10)
    g0.record(stream)
    for _ in range(reps):
        graph.replay()
    g1.record(stream)
    torch.cuda.synchronize(dev)
    ms = g0.elapsed_time(g1) / (reps * cd["ring"])
    nbytes, units = conv_decode_work()
    out["conv1d_decode"] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
                            "bytes_per_launch": nbytes, "tokens_per_s": units / (ms * 1e-3),
                            "launches": reps * cd["ring"], "timing": "CUDA graph replay"}
    del graph
    return out


MTP = dict(batch=64, ntok=4, H=256, P=64, N=128, G=8)


def mtp_work(kind, m=MTP):
    """Algorithmic bytes of one speculative-decode call at the Ultra decode
    shape: the state (fp32) read once, plus per draft token x, B, C (bf16), dt
    (fp32) and y (bf16); the intermediate states written (``verify_inter``);
    the state read and written once (``replay``); or the accepted
    intermediate state read and the state written (``scatter``)."""
    b, n, H, P, N, G = m["batch"], m["ntok"], m["H"], m["P"], m["N"], m["G"]
    state = b * H * P * N * 4
    per_tok = b * (H * P * 2 + 2 * G * N * 2 + H * 4)
    y = b * n * H * P * 2
    if kind == "verify":
        return state + n * per_tok + y
    if kind == "verify_inter":
        return state + n * per_tok + y + n * state
    if kind == "replay":
        return 2 * state + n * per_tok
    return 2 * state + b * 4                                    # scatter


def time_mtp(dev, stream, seed, iters=20):
    """Device time of the speculative-decode entry points (beside the step)."""
    import torch
    from hybrid_mamba_ssm_b200 import inputs as synth
    from hybrid_mamba_ssm_b200 import ssm

    m = MTP
    b, n, H, P, N, G = m["batch"], m["ntok"], m["H"], m["P"], m["N"], m["G"]
    A, D = synth.make_head_params(seed, H)
    A, D = torch.from_numpy(A).to(dev), torch.from_numpy(D).to(dev)
    state = torch.from_numpy(synth.make_state(seed + 1, (b, H, P, N))).to(dev)
    steps = [synth.make_decode_step(seed + 2 + k, b, H, P, N, G) for k in range(n)]

    def stack16(f):
        return torch.stack([torch.from_numpy(np.ascontiguousarray(f(s).bits).view(np.int16))
                            for s in steps], dim=1).view(torch.bfloat16).contiguous().to(dev)

    x, B, C = stack16(lambda s: s.x), stack16(lambda s: s.B), stack16(lambda s: s.C)
    dt = torch.from_numpy(np.stack([s.dt for s in steps], axis=1)).contiguous().to(dev)
    y = torch.empty((b, n, H, P), dtype=torch.bfloat16, device=dev)
    inter = torch.empty((b, n, H, P, N), dtype=torch.float32, device=dev)
    # every row accepts at least one token, so every row's state is written
    acc = torch.from_numpy(np.random.default_rng(seed).integers(1, n + 1, b).astype(np.int32)).to(dev)
    calls = {
        "verify": lambda: ssm.ssm_state_update_multi(state, x, dt, A, B, C, D, y=y, stream=stream),
        "verify_inter": lambda: ssm.ssm_state_update_multi(state, x, dt, A, B, C, D, y=y,
                                                           inter_states=inter, stream=stream),
        "replay": lambda: ssm.ssm_state_update_multi(state, x, dt, A, B, C, D, accept_len=acc,
                                                     want_y=False, stream=stream),
        "scatter": lambda: ssm.ssm_state_commit(inter, acc, state, stream=stream),
    }
    out = {}
    for name, fn in calls.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(iters)]
        for e0, e1 in ev:
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / iters
        nbytes = mtp_work(name)
        out["mtp_" + name] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
                              "bytes_per_launch": nbytes, "launches": iters,
                              "draft": f"batch {b} x {n} tokens"}
    del inter
    return out


NORM = dict(prefill=dict(rows=16384, dim=128 * 64, group=1024),
            decode=dict(rows=64, dim=256 * 64, group=2048))


def time_fused(dev, stream, seed, iters=20):
    """Device time of the steps on either side of the scan: the gated group
    RMSNorm at the prefill and decode shapes (bf16 y, z, out; y, z read and
    out written once: 6 bytes per element), and the 4x4096 prefill fed the
    raw dt with dt_bias + softplus + clamp applied inside the kernel."""
    import torch
    from hybrid_mamba_ssm_b200 import inputs as synth
    from hybrid_mamba_ssm_b200 import ssm

    def bf16(t):
        return torch.from_numpy(np.ascontiguousarray(t.bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    def timed(fn, graph=False):
        """ms per call: per-launch events, or (for calls of a few microseconds,
        where the host's launch rate would set the time) the replay of a CUDA
        graph of `iters` calls."""
        for _ in range(3):
            fn(stream)
        torch.cuda.synchronize(dev)
        if graph:
            gs = torch.cuda.Stream(dev)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(gs):
                with torch.cuda.graph(g, stream=gs):
                    for _ in range(iters):
                        fn(gs)
            g.replay()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            return e0.elapsed_time(e1) / iters
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(iters)]
        for e0, e1 in ev:
            e0.record(stream)
            fn(stream)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        return sum(e0.elapsed_time(e1) for e0, e1 in ev) / iters

    out = {}
    for name, c in NORM.items():
        y, z, w = synth.make_gate(seed + len(out), c["rows"], c["dim"])
        yd, zd, wd = bf16(y), bf16(z), torch.from_numpy(w).to(dev)
        od = torch.empty_like(yd)
        ms = timed(lambda st: ssm.ssm_gated_rmsnorm(yd, zd, wd, c["group"], out=od, stream=st),
                   graph=(name == "decode"))
        nbytes = c["rows"] * c["dim"] * 6 + c["dim"] * 4
        out["gated_rmsnorm_" + name] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
                                        "bytes_per_launch": nbytes, "launches": iters,
                                        "timing": "CUDA graph replay" if name == "decode"
                                        else "per-launch events",
                                        "shape": f"{c['rows']} x {c['dim']}, groups of {c['group']}"}
    p = PREFILL
    inp = synth.make_scan_inputs(seed + 7, [p["seqlen"]] * p["nseq"], p["H"], p["P"], p["N"],
                                 p["G"], dtype="bf16")
    raw, bias = synth.make_raw_dt(seed + 8, (p["nseq"] * p["seqlen"], p["H"]), p["H"])
    L = p["seqlen"]
    x = bf16(inp.x).view(p["nseq"], L, p["H"], p["P"])
    B = bf16(inp.B).view(p["nseq"], L, p["G"], p["N"])
    C = bf16(inp.C).view(p["nseq"], L, p["G"], p["N"])
    dt = torch.from_numpy(raw).to(dev).view(p["nseq"], L, p["H"])
    A, D = torch.from_numpy(inp.A).to(dev), torch.from_numpy(inp.D).to(dev)
    pool = torch.zeros((p["nseq"], p["H"], p["P"], p["N"]), dtype=torch.float32, device=dev)
    fresh = torch.zeros(p["nseq"], dtype=torch.int32, device=dev)
    y = torch.empty_like(x)
    bias_d = torch.from_numpy(bias).to(dev)
    ms = timed(lambda st: ssm.ssd_chunk_scan_slots(x, dt, A, B, C, D, pool, None,
                                                   has_initial_state=fresh, y=y, stream=st,
                                                   dt_bias=bias_d, dt_softplus=True,
                                                   dt_limit=(1e-3, 0.1)))
    flops, nbytes, T = prefill_work()
    out["prefill_raw_dt"] = {"ms": ms, "tokens_per_s": T / (ms * 1e-3),
                             "tflops": flops / (ms * 1e-3) / 1e12, "launches": iters,
                             "dt": "raw dt; bias, softplus and clamp inside the scan"}
    return out


def time_f16_decode(dev, stream, seed, iters=20):
    """Device time of the Ultra decode step on an fp16 state pool, written back
    with stochastic rounding (Philox-4x32 with 5 and with 10 rounds) and with
    round-to-nearest.  Bytes: the fp16 state read and written, plus the
    step's inputs and bf16 y."""
    import torch
    from hybrid_mamba_ssm_b200 import inputs as synth
    from hybrid_mamba_ssm_b200 import ssm

    d = DECODE
    b, H, P, N, G = d["batch"], d["H"], d["P"], d["N"], d["G"]
    A, D = synth.make_head_params(seed, H)
    A, D = torch.from_numpy(A).to(dev), torch.from_numpy(D).to(dev)
    pool = torch.from_numpy(synth.make_state(seed + 1, (b, H, P, N))).to(dev).half()
    st = synth.make_decode_step(seed + 2, b, H, P, N, G)
    bf = lambda t: torch.from_numpy(np.ascontiguousarray(t.bits).view(np.int16)).view(
        torch.bfloat16).to(dev)
    x, B, C = bf(st.x), bf(st.B), bf(st.C)
    dt = torch.from_numpy(st.dt).to(dev)
    y = torch.empty((b, H, P), dtype=torch.bfloat16, device=dev)
    _, full_bytes, _ = decode_work()
    nbytes = full_bytes - b * H * P * N * 4          # fp16 instead of fp32 state
    out = {}
    for name, rnd in (("decode_f16_sr_philox5", (7, 0, 5)), ("decode_f16_sr_philox10", (7, 0, 10)),
                      ("decode_f16_nearest", None)):
        calls = [0]

        def call():
            calls[0] += 1
            r = None if rnd is None else (rnd[0], calls[0], rnd[2])   # fresh offset per step
            ssm.ssm_state_update_slots(pool, None, x, dt, A, B, C, D, y=y, stream=stream,
                                       rounding=r)

        for _ in range(3):
            call()
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(iters)]
        for e0, e1 in ev:
            e0.record(stream)
            call()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / iters
        out[name] = {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9, "bytes_per_launch": nbytes,
                     "launches": iters, "state": "fp16 [64,256,64,128]"}
    return out


def prefill_numbers(flops, nbytes, tokens, ms, peaks):
    """Throughput and roofline fractions of one prefill launch."""
    t_sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    tf = flops / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": ms, "tokens_per_s": tokens / (ms * 1e-3), "tflops": tf,
            "tensor_frac_burst": tf / peaks["bf16_tflops"], "tensor_frac_sustained": tf / t_sus,
            "gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "flops_per_launch": flops,
            "bytes_per_launch": nbytes}


def time_ultra32k(dev, stream, peaks, iters=10):
    """Long prefill, 1 x 32768 tokens at the Ultra layer shape (256 heads,
    nonzero fp32 initial state, bf16 y, fp32 final state): per-launch CUDA
    events; 2.3 GB of inputs and outputs per launch, larger than L2."""
    import torch
    from hybrid_mamba_ssm_b200 import inputs as synth
    from hybrid_mamba_ssm_b200 import ssm
    u = ULTRA32K
    inp = synth.make_scan_inputs(1000 + 3, [u["seqlen"]], u["H"], u["P"], u["N"], u["G"],
                                 dtype="bf16", init_state=True)
    b16 = lambda t: torch.from_numpy(np.ascontiguousarray(t.bits).view(np.int16)).view(
        torch.bfloat16).to(dev)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)
    L = u["seqlen"]
    x = b16(inp.x).view(1, L, u["H"], u["P"])
    B = b16(inp.B).view(1, L, u["G"], u["N"])
    C = b16(inp.C).view(1, L, u["G"], u["N"])
    dt = f32(inp.dt).view(1, L, u["H"])
    A, D, h0 = f32(inp.A), f32(inp.D), f32(inp.h0)
    del inp
    y = torch.empty_like(x)
    hT = torch.empty_like(h0)
    call = lambda: ssm.ssd_chunk_scan(x, dt, A, B, C, D, h0, chunk_size=u["Q"], y=y,
                                      final_state=hT, stream=stream)
    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    for e0, e1 in ev:
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / iters
    f, b, T = prefill_work(u)
    out = prefill_numbers(f, b, T, ms, peaks)
    out["launches"] = iters
    del x, B, C, dt, y
    torch.cuda.empty_cache()
    return out


def time_mixed(dev, stream, peaks, iters=5):
    """Mixed workload: 8 packed sequences (seeded lengths in 512..16384,
    128 heads, per-sequence fp32 initial states) prefilled with one varlen
    ssd_chunk_scan, then 128 ssm_state_update steps on the 8 final states.
    Prefill tokens/s from per-launch events; decode steps/s over the 128
    consecutive steps (fresh inputs each step)."""
    import torch
    from hybrid_mamba_ssm_b200 import inputs as synth
    from hybrid_mamba_ssm_b200 import ssm
    m = MIXED
    seed = 1000 + 4
    lens = synth.mixed_seqlens(seed, m["nseq"], m["lo"], m["hi"])
    inp = synth.make_scan_inputs(seed, lens, m["H"], m["P"], m["N"], m["G"], dtype="bf16",
                                 init_state=True)
    b16 = lambda t: torch.from_numpy(np.ascontiguousarray(t.bits).view(np.int16)).view(
        torch.bfloat16).to(dev)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)
    x, B, C, dt = b16(inp.x), b16(inp.B), b16(inp.C), f32(inp.dt)
    A, D, h0 = f32(inp.A), f32(inp.D), f32(inp.h0)
    cu = torch.from_numpy(inp.cu_seqlens.astype(np.int32)).to(dev)
    y = torch.empty_like(x)
    hT = torch.empty_like(h0)
    pre = lambda: ssm.ssd_chunk_scan(x, dt, A, B, C, D, h0, cu_seqlens=cu, chunk_size=m["Q"],
                                     y=y, final_state=hT, stream=stream)
    steps = [synth.make_decode_step(seed + 500 + k, m["nseq"], m["H"], m["P"], m["N"], m["G"])
             for k in range(m["decode_steps"])]
    dsteps = [(b16(s.x), f32(s.dt), b16(s.B), b16(s.C)) for s in steps]
    dy = torch.empty((m["nseq"], m["H"], m["P"]), dtype=torch.bfloat16, device=dev)
    state = torch.empty_like(hT)

    def decode_all():
        for xs, dts, Bs, Cs in dsteps:
            ssm.ssm_state_update(state, xs, dts, A, Bs, Cs, D, y=dy, stream=stream)

    for _ in range(3):
        pre()
    state.copy_(hT)
    decode_all()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    for e0, e1 in ev:
        e0.record(stream)
        pre()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    pre_ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / iters
    state.copy_(hT)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    decode_all()
    d1.record(stream)
    torch.cuda.synchronize(dev)
    dec_ms = d0.elapsed_time(d1)
    T = int(sum(lens))
    f, b, _ = prefill_work(dict(m, nseq=m["nseq"], h0=True), T=T)
    out = {"prefill": prefill_numbers(f, b, T, pre_ms, peaks),
           "decode_steps_per_s": m["decode_steps"] / (dec_ms * 1e-3),
           "decode_ms_per_step": dec_ms / m["decode_steps"], "tokens": T,
           "seqlens": [int(v) for v in lens]}
    out["prefill"]["launches"] = iters
    return out


def run_reference(args, world, rank, pg):
    if rank != 0:
        return 0
    tokens_per_step = PREFILL["nseq"] * PREFILL["seqlen"] + DECODE["batch"]
    for _ in range(args.warmup):
        oracle_step_sample(2000, 256, 4, 1)
    total = measured = 0.0
    desc = cores = None
    for k in range(args.steps):
        s, desc, cores, took = oracle_step_sample(2000 + k, 256, 4, 1)
        total += s
        measured += took
    value = tokens_per_step * args.steps / total
    # ms_per_step is what each (sample) step took on the host; the value is the
    # full workload's tokens/s, the sample's time scaled to a whole step.
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * measured / args.steps,
            "full_step_ms_equivalent": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": "prefill 4x4096 H128 P64 N128 G8 Q128 + decode 64x256x64x128 G8",
                       "reference": "fp64 CPU oracle (sequential recurrence), bounded sample per step"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU path
# ---------------------------------------------------------------------------
def run_ours(args, world, rank, local, pg):
    import torch
    from hybrid_mamba_ssm_b200 import inputs as synth
    from hybrid_mamba_ssm_b200 import ssm

    dev = torch.device("cuda", local)
    p, d = PREFILL, DECODE
    seed = 1000 + 2 + 7919 * rank

    def bf16(t, pin=False):
        a = torch.from_numpy(np.ascontiguousarray(t.bits).view(np.int16)).view(torch.bfloat16)
        return a.pin_memory() if pin else a.to(dev)

    def f32(a, pin=False):
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
        return t.pin_memory() if pin else t.to(dev)

    # prefill inputs (resident) and host copies (for the end-to-end leg)
    pin = synth.make_scan_inputs(seed, [p["seqlen"]] * p["nseq"], p["H"], p["P"], p["N"],
                                 p["G"], dtype="bf16")
    L = p["seqlen"]
    shp = lambda t, *s: t.view(p["nseq"], L, *s)
    px, pdt = bf16(pin.x), f32(pin.dt)
    pB, pC = bf16(pin.B), bf16(pin.C)
    pA, pD = f32(pin.A), f32(pin.D)
    py = torch.empty((p["nseq"], L, p["H"], p["P"]), dtype=torch.bfloat16, device=dev)
    phT = torch.empty((p["nseq"], p["H"], p["P"], p["N"]), dtype=torch.float32, device=dev)
    host_pre = dict(x=bf16(pin.x, True), dt=f32(pin.dt, True), B=bf16(pin.B, True),
                    C=bf16(pin.C, True))
    # scan workspace: the balanced schedule, where the chains do not fill whole
    # waves of SMs (both legs' scans run on one stream, so they share it)
    n_ws = ssm.ssd_chunk_scan_workspace_size(p["nseq"], L, p["H"], p["P"], p["N"], p["G"], p["Q"])
    pws = torch.empty(n_ws, dtype=torch.uint8, device=dev) if n_ws else None

    # decode: state, per-head params, a ring of per-step inputs
    dA, dD = synth.make_head_params(1001 + 7919 * rank, d["H"])
    dA, dD = f32(dA), f32(dD)
    state = f32(synth.make_state(1001 + 7919 * rank + 1, (d["batch"], d["H"], d["P"], d["N"])))
    ring, host_ring = [], []
    for k in range(RING):
        s = synth.make_decode_step(1001 + 7919 * rank + 100 + k, d["batch"], d["H"], d["P"],
                                   d["N"], d["G"])
        ring.append((bf16(s.x), f32(s.dt), bf16(s.B), bf16(s.C)))
        host_ring.append((bf16(s.x, True), f32(s.dt, True), bf16(s.B, True), bf16(s.C, True)))
    dy = torch.empty((d["batch"], d["H"], d["P"]), dtype=torch.bfloat16, device=dev)

    stream = torch.cuda.current_stream(dev)

    def prefill(x=px, dt=pdt, B=pB, C=pC):
        ssm.ssd_chunk_scan(shp(x, p["H"], p["P"]), shp(dt, p["H"]), pA,
                           shp(B, p["G"], p["N"]), shp(C, p["G"], p["N"]), pD, None,
                           chunk_size=p["Q"], y=py, final_state=phT, stream=stream,
                           workspace=pws)

    def decode(k, inp=None):
        x, dt, B, C = inp if inp is not None else ring[k % RING]
        ssm.ssm_state_update(state, x, dt, dA, B, C, dD, y=dy, stream=stream)

    for k in range(args.warmup):
        prefill()
        decode(k)
    torch.cuda.synchronize(dev)
    barrier(pg, dev)
    torch.cuda.synchronize(dev)

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(gpu_uuid(dev))
    clocks.start()
    time.sleep(0.3)
    start.record(stream)
    for k in range(K):
        ev[k][0].record(stream)
        prefill()
        ev[k][1].record(stream)
        ev[k][2].record(stream)
        decode(k)
        ev[k][3].record(stream)
    end.record(stream)
    torch.cuda.synchronize(dev)
    clock_info = clocks.stop()
    barrier(pg, dev)
    ms = max_over_ranks(pg, start.elapsed_time(end), dev)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / K
    dec_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / K
    pre_ms = max_over_ranks(pg, pre_ms, dev)
    dec_ms = max_over_ranks(pg, dec_ms, dev)

    # ---- end to end: pinned host inputs -> device, call, results -> host ----
    # Three streams form a two-slot pipeline: step k's inputs are copied in on
    # the H2D stream while step k-1 computes; step k's y, final state and
    # decode y are copied out on the D2H stream while step k+1 computes.  A
    # slot is reused only after the compute (inputs) or copy-out (outputs)
    # of the step two earlier has finished.
    out_host = [dict(y=torch.empty(py.shape, dtype=py.dtype, pin_memory=True),
                     hT=torch.empty(phT.shape, dtype=phT.dtype, pin_memory=True),
                     dy=torch.empty(dy.shape, dtype=dy.dtype, pin_memory=True)) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_pre.values()) + \
        sum(t.numel() * t.element_size() for t in host_ring[0])
    d2h = sum(t.numel() * t.element_size() for t in out_host[0].values())
    e2e_steps = max(1, min(K, 50))
    slots = [dict(x=torch.empty_like(px), dt=torch.empty_like(pdt), B=torch.empty_like(pB),
                  C=torch.empty_like(pC), dec=[torch.empty_like(t) for t in ring[0]],
                  y=torch.empty_like(py), hT=torch.empty_like(phT), dy=torch.empty_like(dy))
             for _ in range(2)]
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def e2e_step(k):
        sl = slots[k % 2]
        with torch.cuda.stream(s_in):
            if started[k % 2]:
                s_in.wait_event(ev_comp[k % 2])          # inputs of step k-2 consumed
            sl["x"].copy_(host_pre["x"], non_blocking=True)
            sl["dt"].copy_(host_pre["dt"], non_blocking=True)
            sl["B"].copy_(host_pre["B"], non_blocking=True)
            sl["C"].copy_(host_pre["C"], non_blocking=True)
            for dst, src in zip(sl["dec"], host_ring[k % RING]):
                dst.copy_(src, non_blocking=True)
            ev_in[k % 2].record(s_in)
        stream.wait_event(ev_in[k % 2])
        if started[k % 2]:
            stream.wait_event(ev_out[k % 2])             # outputs of step k-2 copied out
        ssm.ssd_chunk_scan(shp(sl["x"], p["H"], p["P"]), shp(sl["dt"], p["H"]), pA,
                           shp(sl["B"], p["G"], p["N"]), shp(sl["C"], p["G"], p["N"]), pD, None,
                           chunk_size=p["Q"], y=sl["y"], final_state=sl["hT"], stream=stream,
                           workspace=pws)
        x, dt, B, C = sl["dec"]
        ssm.ssm_state_update(state, x, dt, dA, B, C, dD, y=sl["dy"], stream=stream)
        ev_comp[k % 2].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[k % 2])
            oh = out_host[k % 2]
            oh["y"].copy_(sl["y"], non_blocking=True)
            oh["hT"].copy_(sl["hT"], non_blocking=True)
            oh["dy"].copy_(sl["dy"], non_blocking=True)
            ev_out[k % 2].record(s_out)
        started[k % 2] = True

    for k in range(2):
        e2e_step(k)
    torch.cuda.synchronize(dev)
    barrier(pg, dev)
    torch.cuda.synchronize(dev)
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(s_in)
    for k in range(e2e_steps):
        e2e_step(k)
    s_out.wait_event(ev_comp[(e2e_steps - 1) % 2])
    e2.record(s_out)
    torch.cuda.synchronize(dev)
    barrier(pg, dev)
    e2e_ms = max_over_ranks(pg, s2.elapsed_time(e2), dev)

    peaks, peak_kind = load_peaks()
    # the other prefill workloads, timed beside the step
    ultra = mixed = None
    if not args.no_parts:
        ultra = time_ultra32k(dev, stream, peaks)
        mixed = time_mixed(dev, stream, peaks)
    conv = {}
    if not args.no_parts:   # the steps around the scan, timed beside the step
        conv = time_conv(dev, stream, seed + 17)
        conv.update(time_mtp(dev, stream, seed + 29))
        conv.update(time_fused(dev, stream, seed + 41))
        conv.update(time_f16_decode(dev, stream, seed + 53))

    # ---- numbers ----
    for part in conv.values():
        if "gbs" in part:
            part["hbm_frac"] = part["gbs"] / peaks["hbm_gbs"]
    tok_step = p["nseq"] * p["seqlen"] + d["batch"]
    value = world * tok_step * K / (ms * 1e-3)
    e2e_value = world * tok_step * e2e_steps / (e2e_ms * 1e-3)
    pf, pb, ptok = prefill_work()
    df, db, _ = decode_work()
    hbm = peaks["hbm_gbs"]
    t_sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    pre = prefill_numbers(pf, pb, ptok, pre_ms, peaks)
    dec = {"gbs": db / (dec_ms * 1e-3) / 1e9, "ms": dec_ms,
           "hbm_frac": db / (dec_ms * 1e-3) / 1e9 / hbm,
           "hbm_frac_of_8TBs": db / (dec_ms * 1e-3) / 8e12,
           "tokens_per_s": d["batch"] / (dec_ms * 1e-3), "bytes_per_launch": db}
    # prefill is HBM-bound by arithmetic intensity (flops/byte below the ridge)
    if pre_ms >= dec_ms:
        ridge = t_sus * 1e12 / (hbm * 1e9)
        if pf / pb < ridge:
            roof = {"kernel": "ssd_chunk_scan", "bound": "hbm", "achieved": pre["gbs"],
                    "peak": hbm, "unit": "GB/s", "frac": pre["hbm_frac"],
                    "traffic": measured_traffic("ssd_chunk_scan", "scan_tc.cu")}
        else:
            roof = {"kernel": "ssd_chunk_scan", "bound": "tensor", "achieved": pre["tflops"],
                    "peak": t_sus, "unit": "TFLOP/s", "frac": pre["tensor_frac_sustained"],
                    "traffic": measured_traffic("ssd_chunk_scan", "scan_tc.cu")}
    else:
        roof = {"kernel": "ssm_state_update", "bound": "hbm", "achieved": dec["gbs"],
                "peak": hbm, "unit": "GB/s", "frac": dec["hbm_frac"],
                "traffic": measured_traffic("ssm_state_update", "state_update.cu")}
    roof["peak_source"] = peak_kind

    r3 = lambda v: float(f"{v:.4g}")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "prefill 4x4096 H128 P64 N128 G8 Q128 + decode 64x256x64x128 G8",
                       "l2": "inputs larger than L2 (about 1.7 GB touched per step)",
                       "parallelism": f"replicas x{world} (independent batches per GPU)"},
            # the two numbers the metric names: prefill (% tensor peak) and decode (% HBM)
            "prefill_ms": r3(pre_ms), "prefill_tokens_per_s": r3(pre["tokens_per_s"]),
            "prefill_tflops": r3(pre["tflops"]),
            "prefill_tensor_frac_burst": r3(pre["tensor_frac_burst"]),
            "prefill_tensor_frac_sustained": r3(pre["tensor_frac_sustained"]),
            "prefill_hbm_frac": r3(pre["hbm_frac"]),
            "decode_ms": r3(dec_ms), "decode_gbs": r3(dec["gbs"]),
            "decode_hbm_frac": r3(dec["hbm_frac"]), "decode_frac_of_8TBs": r3(dec["hbm_frac_of_8TBs"]),
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "pipeline": "H2D, compute and D2H on three streams, two buffer slots"},
            "gpu_launches": 2 * K,
            "clocks": clock_info}

    if ultra is not None:
        line["prefill_ultra_32k"] = {k: r3(ultra[k]) for k in ("ms", "tokens_per_s", "tflops",
                                                               "tensor_frac_burst", "hbm_frac")}
        line["mixed_varlen"] = {"prefill_tokens_per_s": r3(mixed["prefill"]["tokens_per_s"]),
                                "decode_steps_per_s": r3(mixed["decode_steps_per_s"])}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        step_s, desc, cores, _ = oracle_step_sample(3000, 1024, 8, 4)
        line["cpu_baseline"] = {"value": tok_step / step_s, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        # per-kernel detail on its own line first; the headline line, short,
        # is the last line printed
        detail = {"bench_parts": {"prefill": pre, "decode": dec, "prefill_ultra_32k": ultra,
                                  "mixed_varlen": mixed, **conv},
                  "workloads": {"prefill": dict(PREFILL, in_dtype="bf16", y_dtype="bf16",
                                                initial_state="zero"),
                                "decode": dict(DECODE, in_dtype="bf16", y_dtype="bf16",
                                               ring=RING),
                                "prefill_ultra_32k": ULTRA32K, "mixed_varlen": MIXED}}
        print(json.dumps(detail), flush=True)
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-parts", action="store_true",
                    help="skip the timings of the kernels around the scan (conv1d, "
                         "speculative decode, fused steps, fp16 pools)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)   # timing rule: at least 3 warm-up steps
    world, rank, local, pg = dist_setup(args)
    try:
        if args.impl == "reference":
            rc = run_reference(args, world, rank, pg)
        else:
            rc = run_ours(args, world, rank, local, pg)
    finally:
        if pg is not None:
            pg.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
