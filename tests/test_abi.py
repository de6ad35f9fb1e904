"""The C ABI: the library loads, exports every symbol include/*.h declares,
and rejects bad arguments on the host before launching anything.

No test here launches a kernel: every call either fails validation (which
happens before any CUDA call) or is a documented no-op (batch 0, nseq 0).
"""
import ctypes
import os
import re

import pytest

from hybrid_mamba_ssm_b200 import build as ssm_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm.h")
HEADERS = sorted(os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
                 if f.endswith(".h"))

OK, INVALID, UNSUPPORTED, MISALIGNED = 0, 1, 2, 3
F32, BF16 = 0, 1


@pytest.fixture(scope="module")
def lib():
    path = ssm_build.build()
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.ssd_chunk_scan.restype = i
    lib.ssd_chunk_scan.argtypes = [i, i, vp, i, i, i, i, i, i, vp, vp, vp, vp, vp,
                                   vp, vp, i, vp, vp, vp, sz, vp, vp]
    lib.ssm_state_update.restype = i
    lib.ssm_state_update.argtypes = [i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, vp, i,
                                     vp, vp]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_status_string.argtypes = [i]
    lib.ssd_chunk_scan_workspace_size.restype = sz
    lib.ssd_chunk_scan_workspace_size.argtypes = [i] * 7
    return lib


def declared_functions():
    names = []
    for h in HEADERS:
        names += re.findall(r"SSM_API\s+[\w\s\*]+?\b(\w+)\s*\(", open(h).read())
    return names


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("ssd_chunk_scan", "ssm_state_update", "ssd_chunk_scan_workspace_size",
                     "ssm_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libssm.so does not export {name}"


def test_status_strings(lib):
    for code in range(10):
        assert lib.ssm_status_string(code)
        assert b"unknown" not in lib.ssm_status_string(code)
    assert b"unknown" in lib.ssm_status_string(99)


def test_workspace_size(lib):
    # no workspace for shapes off the tensor-core path, nor for empty input
    assert lib.ssd_chunk_scan_workspace_size(4, 4096, 128, 32, 128, 8, 128) == 0
    assert lib.ssd_chunk_scan_workspace_size(4, 4096, 128, 64, 128, 8, 64) == 0
    assert lib.ssd_chunk_scan_workspace_size(4, 4096, 12, 64, 128, 4, 128) == 0   # 3 heads per group
    assert lib.ssd_chunk_scan_workspace_size(0, 4096, 128, 64, 128, 8, 128) == 0
    # otherwise one 2 x 64 x 128 fp32 slot and one flag per run (per SM of the
    # current device; no device here means no runs)
    n = lib.ssd_chunk_scan_workspace_size(4, 4096, 128, 64, 128, 8, 128)
    assert n % (65536 + 4) == 0


def test_noalloc_validates_like_ssd_chunk_scan(lib):
    # Without a device no shape needs the built-in scratch, so the call goes
    # straight to ssd_chunk_scan's host validation (nothing is launched).
    f = lib.ssd_chunk_scan_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    f.restype = i
    f.argtypes = [i, i, vp, i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp]
    args = [1, 128, None, 4, 64, 128, 1, 128, BF16, 0x10000, 0x20000, 0x30000, 0x40000,
            0x50000, None, None, BF16, 0x60000, 0x70000, None, None]
    bad = list(args)
    bad[0] = -1                       # nseq
    assert f(*bad) == INVALID
    bad = list(args)
    bad[3], bad[6] = 6, 4             # heads not a multiple of groups
    assert f(*bad) == INVALID
    bad = list(args)
    bad[17] = 0x60008                 # y only 8-byte aligned
    assert f(*bad) == MISALIGNED
    assert b"SCRATCH" in lib.ssm_status_string(9)


# Fake, never-dereferenced device addresses: validation rejects the call first.
A16 = 0x10000
A16b = 0x20000
A16c = 0x30000
ODD = 0x10008   # 8-byte aligned only


def scan(lib, nseq=1, seqlen=128, cu=None, H=4, P=64, N=128, G=1, Q=128, ind=BF16,
         x=A16, dt=A16b, A=A16c, B=0x40000, C=0x50000, D=None, h0=None, yd=BF16,
         y=0x60000, hT=0x70000, status=None):
    return lib.ssd_chunk_scan(nseq, seqlen, cu, H, P, N, G, Q, ind, x, dt, A, B, C, D,
                              h0, yd, y, hT, None, 0, status, None)


@pytest.mark.parametrize("kw,code", [
    (dict(H=6, G=4), INVALID),             # heads not a multiple of groups
    (dict(G=0), INVALID),
    (dict(nseq=-1), INVALID),
    (dict(seqlen=-5), INVALID),
    (dict(ind=7), INVALID),
    (dict(yd=3), INVALID),
    (dict(P=48), UNSUPPORTED),
    (dict(N=256), UNSUPPORTED),
    (dict(Q=96), UNSUPPORTED),
    (dict(A=None), INVALID),
    (dict(x=None), INVALID),
    (dict(y=None), INVALID),
    (dict(x=ODD), MISALIGNED),
    (dict(hT=ODD), MISALIGNED),
    (dict(y=0x10000 + 1024), INVALID),     # y overlaps x
    (dict(hT=0x40000 + 64), INVALID),      # final state overlaps B
    (dict(h0=0x70000 + 4096), INVALID),    # partial overlap of initial / final
])
def test_scan_rejects(lib, kw, code):
    assert scan(lib, **kw) == code


def test_scan_nseq_zero_is_noop(lib):
    assert scan(lib, nseq=0, x=None, dt=None, y=None, hT=None) == OK


def update(lib, batch=2, H=4, P=64, N=128, G=2, ind=BF16, state=0x100000, x=A16,
           dt=A16b, A=A16c, B=0x40000, C=0x50000, D=None, yd=F32, y=0x60000):
    return lib.ssm_state_update(batch, H, P, N, G, ind, state, x, dt, A, B, C, D, yd, y,
                                None)


@pytest.mark.parametrize("kw,code", [
    (dict(H=5, G=2), INVALID),
    (dict(batch=-1), INVALID),
    (dict(P=0), INVALID),
    (dict(P=300), UNSUPPORTED),
    (dict(N=24), UNSUPPORTED),
    (dict(N=512), UNSUPPORTED),
    (dict(ind=2), INVALID),
    (dict(state=None), INVALID),
    (dict(B=None), INVALID),
    (dict(state=ODD), MISALIGNED),
    (dict(y=0x100000 + 256), INVALID),     # y inside the state
    (dict(x=0x100000), INVALID),           # x inside the state
])
def test_update_rejects(lib, kw, code):
    assert update(lib, **kw) == code


def test_update_batch_zero_is_noop(lib):
    assert update(lib, batch=0, state=None, x=None) == OK


@pytest.fixture(scope="module")
def slib(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.ssd_chunk_scan_slots.restype = i
    lib.ssd_chunk_scan_slots.argtypes = [i, i, vp, i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, vp,
                                         vp, i, vp, i, vp, vp, i, vp, vp, vp]
    lib.ssm_state_update_slots.restype = i
    lib.ssm_state_update_slots.argtypes = [i, i, i, i, i, i, vp, i, vp, i, vp, vp, vp, vp, vp,
                                           vp, vp, vp, i, vp, vp, vp]
    return lib


def scan_slots(lib, nseq=2, seqlen=128, H=4, P=64, N=128, G=1, pool=0x200000, max_slots=8,
               slots=0x300000, has=None, x=A16, y=0x60000, dtp=None, sd=F32, rnd=None):
    return lib.ssd_chunk_scan_slots(nseq, seqlen, None, H, P, N, G, 128, BF16, x, A16b, A16c,
                                    0x40000, 0x50000, None, dtp, pool, sd, rnd, max_slots, slots,
                                    has, BF16, y, None, None)


class Rounding(ctypes.Structure):
    _fields_ = [("seed", ctypes.c_uint64), ("offset", ctypes.c_uint64),
                ("philox_rounds", ctypes.c_int)]


class DtParams(ctypes.Structure):
    _fields_ = [("dt_bias", ctypes.c_void_p), ("softplus", ctypes.c_int), ("clamp", ctypes.c_int),
                ("dt_min", ctypes.c_float), ("dt_max", ctypes.c_float)]


@pytest.mark.parametrize("kw,code", [
    (dict(max_slots=0), INVALID),
    (dict(pool=None), INVALID),
    (dict(slots=None, max_slots=1), INVALID),   # no slot map: one row per sequence needed
    (dict(slots=0x300004), MISALIGNED),
    (dict(dtp=ctypes.byref(DtParams(0x700004, 1, 0, 0.0, 0.0))), MISALIGNED),
    (dict(dtp=ctypes.byref(DtParams(None, 1, 1, 0.5, 0.1))), INVALID),      # dt_min > dt_max
    (dict(sd=BF16), INVALID),                                                 # bf16 pools: no
    (dict(sd=2, rnd=ctypes.byref(Rounding(1, 2, 0))), INVALID),               # 0 Philox rounds
    (dict(y=0x200000 + 4096), INVALID),     # y inside the pool
    (dict(P=96), UNSUPPORTED),
])
def test_scan_slots_rejects(slib, kw, code):
    assert scan_slots(slib, **kw) == code


def test_scan_slots_nseq_zero_is_noop(slib):
    assert scan_slots(slib, nseq=0, pool=None, slots=None, x=None, y=None) == OK


def update_slots(lib, batch=2, H=4, P=64, N=128, G=2, pool=0x200000, max_slots=8,
                 slots=0x300000, x=A16, y=0x60000, dtp=None, sd=F32, rnd=None):
    return lib.ssm_state_update_slots(batch, H, P, N, G, BF16, pool, sd, rnd, max_slots, slots,
                                      x, A16b, A16c, 0x40000, 0x50000, None, dtp, F32, y, None,
                                      None)


@pytest.mark.parametrize("kw,code", [
    (dict(max_slots=-1), INVALID),
    (dict(slots=None, max_slots=1), INVALID),
    (dict(dtp=ctypes.byref(DtParams(None, 0, 1, float("nan"), 1.0))), INVALID),
    (dict(sd=2, rnd=ctypes.byref(Rounding(1, 2, 17))), INVALID),              # > 16 rounds
    (dict(sd=2, x=0x200000 + 256), INVALID),                                  # x inside fp16 pool
    (dict(x=None), INVALID),
    (dict(pool=0x200008), MISALIGNED),
    (dict(x=0x200000 + 512), INVALID),      # x inside the pool
    (dict(N=48), UNSUPPORTED),
])
def test_update_slots_rejects(slib, kw, code):
    assert update_slots(slib, **kw) == code


@pytest.fixture(scope="module")
def clib(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.causal_conv1d_fwd.restype = i
    lib.causal_conv1d_fwd.argtypes = [i, i, vp, i, i, i, vp, vp, vp, i, vp, i, vp, vp, i, vp,
                                      vp, vp]
    lib.causal_conv1d_update.restype = i
    lib.causal_conv1d_update.argtypes = [i, i, i, i, vp, vp, vp, i, vp, i, vp, i, vp, vp, vp]
    return lib


def conv_fwd(lib, nseq=2, seqlen=64, cu=None, dim=256, width=4, ind=BF16, x=0x100000,
             w=0x200000, bias=None, act=1, state=0x300000, max_slots=0, slots=None, has=None,
             yd=BF16, y=0x400000):
    return lib.causal_conv1d_fwd(nseq, seqlen, cu, dim, width, ind, x, w, bias, act, state,
                                 max_slots, slots, has, yd, y, None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(dim=0), INVALID),
    (dict(width=0), INVALID),
    (dict(width=9), UNSUPPORTED),
    (dict(act=2), INVALID),
    (dict(ind=5), INVALID),
    (dict(w=None), INVALID),
    (dict(x=None), INVALID),
    (dict(y=0x400002), MISALIGNED),
    (dict(y=0x100000 + 64), INVALID),           # y overlaps x
    (dict(state=0x100000 + 4096), INVALID),     # state inside x
    (dict(slots=0x500000, state=None), INVALID),
    (dict(slots=0x500000, max_slots=0), INVALID),
    (dict(nseq=0, seqlen=5, cu=0x600000), INVALID),
])
def test_conv_fwd_rejects(clib, kw, code):
    assert conv_fwd(clib, **kw) == code


def test_conv_fwd_noops(clib):
    assert conv_fwd(clib, nseq=0, x=None, y=None, state=None) == OK
    assert conv_fwd(clib, seqlen=0, x=None, y=None, state=None) == OK


def conv_update(lib, batch=4, dim=256, width=4, x=0x100000, w=0x200000, state=0x300000,
                max_slots=0, slots=None, y=0x400000):
    return lib.causal_conv1d_update(batch, dim, width, BF16, x, w, None, 1, state, max_slots,
                                    slots, BF16, y, None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(batch=-1), INVALID),
    (dict(width=9), UNSUPPORTED),
    (dict(state=None), INVALID),
    (dict(slots=0x500000), INVALID),            # slot map without a pool size
    (dict(x=0x100008), MISALIGNED),
    (dict(y=0x300000 + 256), INVALID),          # y inside the state
])
def test_conv_update_rejects(clib, kw, code):
    assert conv_update(clib, **kw) == code


def test_conv_update_batch_zero_is_noop(clib):
    assert conv_update(clib, batch=0, x=None, y=None, state=None) == OK


@pytest.fixture(scope="module")
def mlib(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.ssm_state_update_multi.restype = i
    lib.ssm_state_update_multi.argtypes = [i, i, i, i, i, i, i, vp, i, vp, vp, vp, vp, vp, vp,
                                           vp, vp, vp, vp, i, vp, vp, vp]
    lib.ssm_state_commit.restype = i
    lib.ssm_state_commit.argtypes = [i, i, i, i, i, vp, vp, vp, i, vp, vp, vp]
    lib.causal_conv1d_update_multi.restype = i
    lib.causal_conv1d_update_multi.argtypes = [i, i, i, i, i, vp, vp, vp, i, vp, i, vp, vp, i,
                                               vp, vp, vp]
    return lib


def multi(lib, batch=2, ntok=3, H=4, P=64, N=128, G=2, state=0x1000000, max_slots=0, slots=None,
          x=0x100000, acc=None, inter=None, y=0x200000):
    return lib.ssm_state_update_multi(batch, ntok, H, P, N, G, BF16, state, max_slots, slots, x,
                                      0x300000, 0x310000, 0x320000, 0x330000, None, None, acc,
                                      inter, BF16, y, None, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ntok=-1), INVALID),
    (dict(state=None), INVALID),
    (dict(y=None), INVALID),                        # no output asked for
    (dict(slots=0x400000), INVALID),                # slot map without a pool size
    (dict(acc=0x400004), MISALIGNED),
    (dict(inter=0x1000000 + 4096), INVALID),        # intermediates inside the state
    (dict(N=48), UNSUPPORTED),
])
def test_multi_rejects(mlib, kw, code):
    assert multi(mlib, **kw) == code


def test_multi_noops(mlib):
    assert multi(mlib, ntok=0, state=None, x=None, y=None) == OK
    assert multi(mlib, batch=0, state=None, x=None, y=None) == OK


@pytest.mark.parametrize("kw,code", [
    (dict(inter=None), INVALID),
    (dict(acc=None), INVALID),
    (dict(state=0x500000 + 64), INVALID),           # state inside the intermediates
    (dict(d_state=100), UNSUPPORTED),
])
def test_commit_rejects(mlib, kw, code):
    args = dict(batch=2, ntok=3, H=4, P=64, d_state=128, inter=0x500000, acc=0x400000,
                state=0x9000000)
    args.update(kw)
    assert mlib.ssm_state_commit(args["batch"], args["ntok"], args["H"], args["P"],
                                 args["d_state"], args["inter"], args["acc"], args["state"], 0,
                                 None, None, None) == code


@pytest.mark.parametrize("kw,code", [
    (dict(y=None), INVALID),                        # neither y nor a commit
    (dict(width=9), UNSUPPORTED),
    (dict(state=None), INVALID),
    (dict(y=0x100000 + 32), INVALID),               # y overlaps x
])
def test_conv_multi_rejects(mlib, kw, code):
    args = dict(batch=2, ntok=3, dim=256, width=4, x=0x100000, state=0x300000, acc=None,
                y=0x400000)
    args.update(kw)
    assert mlib.causal_conv1d_update_multi(args["batch"], args["ntok"], args["dim"],
                                           args["width"], BF16, args["x"], 0x200000, None, 1,
                                           args["state"], 0, None, args["acc"], BF16, args["y"],
                                           None, None) == code


def test_gated_rmsnorm_rejects(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.ssm_gated_rmsnorm.restype = i
    lib.ssm_gated_rmsnorm.argtypes = [i, i, i, i, vp, i, vp, vp, ctypes.c_float, i, vp, vp]

    def call(rows=4, dim=2048, gs=1024, y=0x100000, z=0x200000, w=0x300000, eps=1e-5,
             out=0x400000, od=BF16):
        return lib.ssm_gated_rmsnorm(rows, dim, gs, BF16, y, BF16, z, w, eps, od, out, None)

    assert call(gs=1000) == INVALID              # dim not a multiple of the group
    assert call(dim=2000, gs=1000) == UNSUPPORTED  # group not whole warps of 8-channel threads
    assert call(gs=16384, dim=16384) == UNSUPPORTED
    assert call(eps=-1.0) == INVALID
    assert call(z=None) == INVALID
    assert call(out=0x400008) == MISALIGNED
    assert call(out=0x100010) == INVALID          # out partly overlaps y
    assert call(out=0x200000 + 64) == INVALID    # out overlaps z
    assert call(out=0x100000 + 2, od=BF16) == MISALIGNED
    assert call(rows=0, y=None, z=None, w=None, out=None) == OK


def test_testing_hooks_validate_on_the_host(lib):
    u64 = ctypes.c_ulonglong
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.ssm_testing_scan_stalled.restype = i
    lib.ssm_testing_scan_stalled.argtypes = [i, i, i, i, vp, vp, vp, vp, vp, vp, u64, vp, vp]
    lib.ssm_testing_conv1d_stalled.restype = i
    lib.ssm_testing_conv1d_stalled.argtypes = [i, i, i, i, vp, vp, vp, u64, vp, vp]
    args = (A16, A16b, A16c, 0x40000, 0x50000, 0x60000)
    # the status word is required, the wait limit bounded, the pointers aligned
    assert lib.ssm_testing_scan_stalled(1, 256, 4, 2, *args, 10**6, None, None) == INVALID
    assert lib.ssm_testing_scan_stalled(1, 256, 4, 2, *args, 10, 0x80000, None) == INVALID
    assert lib.ssm_testing_scan_stalled(1, 256, 4, 2, *args, 10**11, 0x80000, None) == INVALID
    assert lib.ssm_testing_scan_stalled(1, 256, 3, 2, *args, 10**6, 0x80000, None) == INVALID
    assert lib.ssm_testing_scan_stalled(1, 256, 4, 2, ODD, *args[1:], 10**6, 0x80000,
                                        None) == MISALIGNED
    assert lib.ssm_testing_conv1d_stalled(1, 64, 100, 4, A16, A16b, A16c, 10**6, 0x80000,
                                          None) == INVALID            # dim % 8
    assert lib.ssm_testing_conv1d_stalled(1, 64, 128, 9, A16, A16b, A16c, 10**6, 0x80000,
                                          None) == INVALID            # width
    assert lib.ssm_testing_conv1d_stalled(1, 64, 128, 4, A16, A16b, A16c, 10**6, None,
                                          None) == INVALID            # no status word


def test_balanced_schedule_rule(lib):
    """When a fixed-length batch is cut into one run per SM (host arithmetic,
    for a device of a given SM count): more chains than SMs, and a last wave
    of chains less than nine tenths full; one run per SM."""
    f = lib.ssm_testing_balanced_runs
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int] * 4
    assert f(4, 4096, 128, 148) == 148       # 256 chains: a second wave 108 wide
    assert f(2, 8192, 160, 148) == 148       # 160 chains
    assert f(1, 32768, 256, 148) == 0        # 128 chains: one wave, each its own critical path
    assert f(9, 1024, 32, 148) == 0          # 144 chains
    assert f(37, 1024, 16, 148) == 0         # 296 chains: two whole waves
    assert f(266, 512, 2, 148) == 148        # last wave 118 of 148 (< 9/10)
    assert f(267, 512, 2, 148) == 0          # last wave 119 of 148 (>= 9/10)
    assert f(4, 4096, 128, 132) == 0         # 132 SMs: last wave 124 of 132 (>= 9/10)
    assert f(4, 4096, 128, 160) == 160       # 160 SMs: last wave 96 of 160
    assert f(0, 4096, 128, 148) == 0 and f(4, 0, 128, 148) == 0 and f(4, 4096, 128, 0) == 0
