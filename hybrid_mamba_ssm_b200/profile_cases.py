"""Small, self-contained launches of each kernel for profiling (ncu).

    python -m hybrid_mamba_ssm_b200.profile_cases prefill --nseq 1 --seqlen 4096 --heads 128
    python -m hybrid_mamba_ssm_b200.profile_cases prefill --nseq 4 --seqlen 4096 --workspace
    python -m hybrid_mamba_ssm_b200.profile_cases decode --batch 16 --heads 256
    python -m hybrid_mamba_ssm_b200.profile_cases conv --nseq 1 --seqlen 8192
    python -m hybrid_mamba_ssm_b200.profile_cases conv_update --batch 64
    python -m hybrid_mamba_ssm_b200.profile_cases mtp --batch 16 --ntok 4 --mode verify

Each case draws seeded inputs, runs ``--warmup`` untimed launches and then
``--launches`` more, and prints the device time of the last ones.  Inputs are
sized by the flags; the defaults keep the working set above the 126 MB L2 while
holding only a few hundred MB on the device.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import inputs as synth
from . import ssm


def _bf16(t, dev):
    return torch.from_numpy(np.ascontiguousarray(t.bits).view(np.int16)).view(torch.bfloat16).to(dev)


def _f32(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


def prefill(args, dev):
    inp = synth.make_scan_inputs(77, [args.seqlen] * args.nseq, args.heads, args.head_dim,
                                 args.d_state, args.groups, dtype="bf16")
    n, L = args.nseq, args.seqlen
    x = _bf16(inp.x, dev).view(n, L, args.heads, args.head_dim)
    dt = _f32(inp.dt, dev).view(n, L, args.heads)
    B = _bf16(inp.B, dev).view(n, L, args.groups, args.d_state)
    C = _bf16(inp.C, dev).view(n, L, args.groups, args.d_state)
    A, D = _f32(inp.A, dev), _f32(inp.D, dev)
    y = torch.empty_like(x)
    hT = torch.empty((n, args.heads, args.head_dim, args.d_state), dtype=torch.float32, device=dev)
    ws = None
    if args.workspace:   # the balanced schedule, where it applies to these shapes
        nb = ssm.ssd_chunk_scan_workspace_size(n, L, args.heads, args.head_dim, args.d_state,
                                               args.groups, args.chunk)
        ws = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
    return lambda: ssm.ssd_chunk_scan(x, dt, A, B, C, D, None, chunk_size=args.chunk, y=y,
                                      final_state=hT, workspace=ws)


def decode(args, dev):
    b, H, P, N, G = args.batch, args.heads, args.head_dim, args.d_state, args.groups
    A, D = synth.make_head_params(78, H)
    A, D = _f32(A, dev), _f32(D, dev)
    state = _f32(synth.make_state(79, (b, H, P, N)), dev)
    s = synth.make_decode_step(80, b, H, P, N, G)
    x, dt, Bt, Ct = _bf16(s.x, dev), _f32(s.dt, dev), _bf16(s.B, dev), _bf16(s.C, dev)
    y = torch.empty((b, H, P), dtype=torch.bfloat16, device=dev)
    return lambda: ssm.ssm_state_update(state, x, dt, A, Bt, Ct, D, y=y)


def conv(args, dev):
    dim = synth.conv_dim(args.heads, args.head_dim, args.groups, args.d_state)
    inp = synth.make_conv_inputs(81, [args.seqlen] * args.nseq, dim, args.width)
    x = _bf16(inp.x, dev).view(args.nseq, args.seqlen, dim)
    w, b = _f32(inp.weight, dev), _f32(inp.bias, dev)
    st = _bf16(inp.state, dev)
    y = torch.empty_like(x)
    return lambda: ssm.causal_conv1d_fwd(x, w, b, conv_state=st, y=y)


def conv_update(args, dev):
    dim = synth.conv_dim(args.heads, args.head_dim, args.groups, args.d_state)
    inp = synth.make_conv_inputs(82, [1] * args.batch, dim, args.width)
    x = _bf16(inp.x, dev)
    w, b = _f32(inp.weight, dev), _f32(inp.bias, dev)
    st = _bf16(inp.state, dev)
    y = torch.empty_like(x)
    return lambda: ssm.causal_conv1d_update(x, w, b, st, y=y)


def mtp(args, dev):
    b, n, H, P, N, G = args.batch, args.ntok, args.heads, args.head_dim, args.d_state, args.groups
    A, D = synth.make_head_params(83, H)
    A, D = _f32(A, dev), _f32(D, dev)
    state = _f32(synth.make_state(84, (b, H, P, N)), dev)
    steps = [synth.make_decode_step(85 + k, b, H, P, N, G) for k in range(n)]
    x = torch.stack([_bf16(s.x, dev) for s in steps], dim=1).contiguous()
    Bt = torch.stack([_bf16(s.B, dev) for s in steps], dim=1).contiguous()
    Ct = torch.stack([_bf16(s.C, dev) for s in steps], dim=1).contiguous()
    dt = torch.stack([_f32(s.dt, dev) for s in steps], dim=1).contiguous()
    acc = torch.full((b,), n, dtype=torch.int32, device=dev)
    y = torch.empty((b, n, H, P), dtype=torch.bfloat16, device=dev)
    if args.mode == "replay":
        return lambda: ssm.ssm_state_update_multi(state, x, dt, A, Bt, Ct, D, accept_len=acc,
                                                  want_y=False)
    return lambda: ssm.ssm_state_update_multi(state, x, dt, A, Bt, Ct, D, y=y)


CASES = {"mtp": mtp, "prefill": prefill, "decode": decode, "conv": conv, "conv_update": conv_update}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=sorted(CASES))
    ap.add_argument("--nseq", type=int, default=1)
    ap.add_argument("--seqlen", type=int, default=4096)
    ap.add_argument("--batch", type=int, default=16)
    ap.add_argument("--heads", type=int, default=None)
    ap.add_argument("--head-dim", type=int, default=64)
    ap.add_argument("--d-state", type=int, default=128)
    ap.add_argument("--groups", type=int, default=8)
    ap.add_argument("--chunk", type=int, default=128)
    ap.add_argument("--width", type=int, default=4)
    ap.add_argument("--ntok", type=int, default=4)
    ap.add_argument("--mode", choices=["verify", "replay"], default="verify")
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--launches", type=int, default=1)
    ap.add_argument("--graph", action="store_true")
    ap.add_argument("--workspace", action="store_true",
                    help="prefill: pass the scan workspace (balanced schedule)")
    args = ap.parse_args()
    if args.heads is None:
        args.heads = 128 if args.case in ("prefill", "conv") else 256
    dev = torch.device("cuda", 0)
    run = CASES[args.case](args, dev)
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if args.graph:
        # launch-bound kernels: replay the launches from a CUDA graph so the
        # device time is not bounded by the host's launch rate
        stream = torch.cuda.Stream()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(graph, stream=stream):
                for _ in range(args.launches):
                    run()
        graph.replay()
        torch.cuda.synchronize()
        s.record()
        graph.replay()
        e.record()
    else:
        s.record()
        for _ in range(args.launches):
            run()
        e.record()
    torch.cuda.synchronize()
    print(json.dumps({"case": args.case, "ms_per_launch": s.elapsed_time(e) / args.launches,
                      "args": vars(args)}))


if __name__ == "__main__":
    main()
