"""Full-size workloads in the benchmark's launch configuration (the prefill
with the scan workspace, as bench.py passes it), checked on sampled heads (and
batch rows) that the oracle computes one by one.

* prefill 4 x 4096 tokens, 128 heads (bf16 in, bf16 y, zero initial state);
* long prefill 1 x 32768 tokens, 256 heads, nonzero initial state;
* decode at the Ultra layer shape, 1000 consecutive steps (ring of 8 inputs);
* mixed: 8 packed sequences of seeded lengths in 512..16384 prefilled, then
  128 decode steps each; final states equal one oracle run over both.
"""
import numpy as np
import pytest
import torch

from hybrid_mamba_ssm_b200 import inputs as synth
from tests.gpu_helpers import (TOL, dev_f32, dev_tensor, oracle_scan, rel_err, scan_on_gpu,
                               to_np)

pytestmark = pytest.mark.gpu


def _workload_inputs(name):
    w = synth.WORKLOADS[name]
    return synth.make_scan_inputs(synth.workload_seed(name), w["seqlens"], w["nheads"],
                                  w["head_dim"], w["d_state"], w["ngroups"], dtype=w["dtype"],
                                  init_state=w["init_state"])


# One whole group of heads (all heads sharing one B, C), plus heads of other
# groups: group 1 of the 128-head workload (heads 16..31), group 6 of the
# 256-head one (heads 192..223).
@pytest.mark.parametrize("name,heads", [("prefill_4x4096", list(range(16, 32)) + [0, 66, 127]),
                                        ("prefill_ultra_32k", list(range(192, 224)) + [0, 95])])
def test_full_prefill_sampled_heads(name, heads):
    inp = _workload_inputs(name)
    y, hT = scan_on_gpu(inp, chunk=128, y_dtype=torch.bfloat16, workspace=True)
    y = y[:, heads]
    hT = hT[:, heads]
    y_ref, h_ref = oracle_scan(inp, heads=heads)
    ey = rel_err(to_np(y), y_ref, bf16=True)
    eh = rel_err(to_np(hT), h_ref)
    assert ey < TOL, ey
    assert eh < TOL, eh
    # per (sequence, head) final-state slices
    hg = to_np(hT)
    for s in range(hg.shape[0]):
        for k in range(hg.shape[1]):
            assert rel_err(hg[s, k], h_ref[s, k]) < TOL


def test_full_decode_1000_steps_sampled():
    import oracle
    from hybrid_mamba_ssm_b200 import ssm
    w = synth.WORKLOADS["decode_ultra"]
    b, H, P, N, G = w["batch"], w["nheads"], w["head_dim"], w["d_state"], w["ngroups"]
    seed = synth.workload_seed("decode_ultra")
    A, D = synth.make_head_params(seed, H)
    state0 = synth.make_state(seed + 1, (b, H, P, N))
    ring = [synth.make_decode_step(seed + 100 + k, b, H, P, N, G) for k in range(8)]
    dev_ring = [(dev_tensor(r.x), dev_f32(r.dt), dev_tensor(r.B), dev_tensor(r.C)) for r in ring]
    state = dev_f32(state0)
    At, Dt = dev_f32(A), dev_f32(D)
    rows, heads = [0, 41], [0, 33, 130, 255]
    groups = [h // (H // G) for h in heads]
    ref = state0[rows][:, heads].astype(np.float64)
    y_last = None
    for k in range(w["steps"]):
        x, dt, B, C = dev_ring[k % 8]
        y_last = ssm.ssm_state_update(state, x, dt, At, B, C, Dt, y_dtype=torch.float32)
        r = ring[k % 8]
        yr, ref = oracle.state_update(ref, r.x.values[rows][:, heads], r.dt[rows][:, heads],
                                      A[heads], r.B.values[rows][:, groups],
                                      r.C.values[rows][:, groups], D[heads])
    torch.cuda.synchronize()
    got = to_np(state)[rows][:, heads]
    assert rel_err(got, ref) < TOL
    assert rel_err(to_np(y_last)[rows][:, heads], yr) < TOL


def test_mixed_prefill_then_decode():
    import oracle
    from hybrid_mamba_ssm_b200 import ssm
    w = synth.WORKLOADS["mixed_varlen"]
    seed = synth.workload_seed("mixed_varlen")
    lens = synth.mixed_seqlens(seed, w["nseq"], w["lo"], w["hi"])
    H, P, N, G = w["nheads"], w["head_dim"], w["d_state"], w["ngroups"]
    inp = synth.make_scan_inputs(seed, lens, H, P, N, G, dtype="bf16", init_state=True)
    y, hT = scan_on_gpu(inp, chunk=w["chunk"], y_dtype=torch.bfloat16, varlen=True)
    state = hT.clone()
    At, Dt = dev_f32(inp.A), dev_f32(inp.D)
    steps = [synth.make_decode_step(seed + 500 + k, w["nseq"], H, P, N, G)
             for k in range(w["decode_steps"])]
    for st in steps:
        yd = ssm.ssm_state_update(state, dev_tensor(st.x), dev_f32(st.dt), At, dev_tensor(st.B),
                                  dev_tensor(st.C), Dt, y_dtype=torch.float32)
    torch.cuda.synchronize()

    heads = [3, 64, 127]
    groups = [h // (H // G) for h in heads]
    # one sequential oracle run per sequence over prefill tokens then decode tokens
    xs, dts, Bs, Cs, cu = [], [], [], [], [0]
    for s in range(w["nseq"]):
        a, b = inp.cu_seqlens[s], inp.cu_seqlens[s + 1]
        xs.append(np.concatenate([inp.x.values[a:b][:, heads]] +
                                 [st.x.values[s:s + 1][:, heads] for st in steps]))
        dts.append(np.concatenate([inp.dt[a:b][:, heads]] + [st.dt[s:s + 1][:, heads] for st in steps]))
        Bs.append(np.concatenate([inp.B.values[a:b][:, groups]] +
                                 [st.B.values[s:s + 1][:, groups] for st in steps]))
        Cs.append(np.concatenate([inp.C.values[a:b][:, groups]] +
                                 [st.C.values[s:s + 1][:, groups] for st in steps]))
        cu.append(cu[-1] + xs[-1].shape[0])
    y_ref, h_ref = oracle.scan(np.concatenate(xs), np.concatenate(dts), inp.A[heads],
                               np.concatenate(Bs), np.concatenate(Cs), inp.D[heads],
                               inp.h0[:, heads], cu_seqlens=np.array(cu))
    got = to_np(state)[:, heads]
    assert rel_err(got, h_ref) < TOL
    # the last decode token's y of every sequence
    last = np.array(cu[1:]) - 1
    assert rel_err(to_np(yd)[:, heads], y_ref[last]) < TOL
    # prefill y of the sampled heads
    pre_idx = np.concatenate([np.arange(cu[s], cu[s] + lens[s]) for s in range(w["nseq"])])
    assert rel_err(to_np(y)[:, heads], y_ref[pre_idx], bf16=True) < TOL
