"""Pins of the oracle's Philox-4x32 generator and fp16 stochastic rounding:
Philox-4x32-10 against cuRAND's host Philox generator (a library routine,
run on the CPU); stochastic rounding against numpy's fp16 neighbours and its
defining property, an exact mean over the random word."""
import ctypes
import os

import numpy as np
import pytest

import oracle

CURAND = "/usr/local/cuda/lib64/libcurand.so"


def _curand_words(seed, n, offset=0):
    lib = ctypes.CDLL(CURAND)
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0   # PHILOX4_32_10
    assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
    assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(offset)) == 0
    buf = (ctypes.c_uint32 * n)()
    assert lib.curandGenerate(gen, buf, ctypes.c_size_t(n)) == 0
    lib.curandDestroyGenerator(gen)
    return list(buf)


@pytest.mark.skipif(not os.path.exists(CURAND), reason="cuRAND host library not present")
@pytest.mark.parametrize("seed", [0, 12345, 0xDEADBEEFCAFEF00D])
def test_philox_matches_curand_host_generator(seed):
    # The host generator lays its output out as 65536 interleaved streams:
    # 4-word block b is Philox(counter = (b // 65536, 0, b % 65536, 0), key = seed).
    words = _curand_words(seed, 4 * (65536 + 8))
    key = (seed & 0xFFFFFFFF, seed >> 32)
    for b in list(range(16)) + list(range(65536, 65536 + 8)):
        got = oracle.philox4x32((b // 65536, 0, b % 65536, 0), key, 10)
        assert got == words[4 * b:4 * b + 4], b


def _fp16_bracket(v):
    """The fp16 values toward and away from zero around the fp32 value v."""
    f = np.float16(v)
    if float(f) == float(np.float32(v)):
        return float(f), float(f)
    away = np.float16(np.inf) if v > 0 else np.float16(-np.inf)
    a = np.nextafter(f, np.float16(0.0) if abs(float(f)) > abs(float(np.float32(v))) else away)
    lo, hi = sorted([float(f), float(a)], key=abs)
    return lo, hi


def test_sr_returns_a_neighbour_and_keeps_exact_values():
    rng = np.random.default_rng(5)
    vals = np.concatenate([rng.standard_normal(200).astype(np.float32),
                           (rng.standard_normal(50) * 1e-6).astype(np.float32),
                           np.float16(rng.standard_normal(50)).astype(np.float32)])
    rs = rng.integers(0, 2**16, len(vals))
    for v, r in zip(vals, rs):
        got = oracle.sr_fp16(v, r)
        lo, hi = _fp16_bracket(v)
        assert got in (lo, hi), (v, got, lo, hi)
        if lo == hi:
            assert got == lo
    assert oracle.sr_fp16(70000.0, 0) == 65504.0
    assert oracle.sr_fp16(-1e9, 123) == -65504.0


@pytest.mark.parametrize("v", [1.0 + 3 * 2.0**-20, -0.3337, 1234.567, 3.1e-6, -5.9e-8])
def test_sr_mean_over_the_random_word_is_exact(v):
    v = float(np.float32(v))
    if abs(v) >= 2.0**-14:
        # normal range: 13 dropped mantissa bits decide, so u = r16 / 2^16 over
        # r16 = 8k, k < 8192, hits every threshold once: the mean is v exactly
        vals = np.array([oracle.sr_fp16(v, 8 * k) for k in range(1 << 13)])
        assert vals.mean() == v
    else:
        # fp16 subnormals: over all 2^16 draws the mean is v to within 2^-16
        # of a step (the fraction has more bits than the draw)
        vals = np.array([oracle.sr_fp16(v, k) for k in range(1 << 16)])
        lo, hi = _fp16_bracket(v)
        assert set(np.unique(vals)) <= {lo, hi}
        assert abs(vals.mean() - v) <= 2.0**-24 * 2.0**-16 * 1.0001


def test_round_state_draw_layout():
    """Element e of a pool draws half e % 2 (low half first) of word
    (e % 8) / 2 of Philox(counter = (e / 8, offset)): values exactly halfway
    between fp16 neighbours (1 + 2^-11) round up iff that half is below 2^15."""
    v = np.full(24, 1.0 + 2.0**-11)
    got = oracle.round_state_f16(v, np.arange(24), 7, 3)
    ref = []
    for e in range(24):
        w = oracle.philox4x32((e // 8, 0, 3, 0), (7, 0), 10)[(e % 8) // 2]
        r16 = (w >> 16) if e % 2 else (w & 0xFFFF)
        ref.append(1.0 + 2.0**-10 if r16 < 32768 else 1.0)
    assert list(got) == ref
    assert 0 < sum(g > 1.0 for g in got) < 24


def test_header_states_the_pinned_draw_layout():
    """The public header's description of the draw layout (ssm_rounding in
    include/ssm.h) is the one the oracle follows and the test above pins:
    its numbers are read from the comment and checked against the oracle."""
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    text = open(os.path.join(root, "include", "ssm.h")).read()
    block = text[text.index("Stochastic rounding of an fp16 state pool"):
                 text.index("uint64_t seed;")]
    block = " ".join(block.replace("*", " ").split())
    bits, scale = map(int, re.search(r"u = r(\d+) / 2\^(\d+)", block).groups())
    halves = int(re.search(r"half e % (\d+)", block).group(1))
    per_call, per_word = map(int, re.search(r"word \(e % (\d+)\) / (\d+)", block).groups())
    ctr_div = int(re.search(r"counter = \(e / (\d+)", block).group(1))
    assert (bits, scale, halves, per_call, per_word, ctr_div) == (16, 16, 2, 8, 2, 8)
    v = np.full(24, 1.0 + 2.0**-11)
    got = oracle.round_state_f16(v, np.arange(24), 11, 5)
    for e in range(24):
        w = oracle.philox4x32((e // ctr_div, 0, 5, 0), (11, 0), 10)[(e % per_call) // per_word]
        r = (w >> (bits * (e % halves))) & ((1 << bits) - 1)
        assert got[e] == (1.0 + 2.0**-10 if r < (1 << (scale - 1)) else 1.0), e
