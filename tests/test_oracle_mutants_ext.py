"""Planted mistakes in the oracle's conv1d, Philox and stochastic-rounding
code: each mutated copy of the C source is compiled and must be rejected by
at least one of the pins in tests/test_oracle_conv.py or
tests/test_oracle_sr.py (the same check tests/test_oracle.py makes for the
scan)."""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_conv as conv_pins
from tests import test_oracle_sr as sr_pins

CONV_MUTANTS = {
    "kernel_reversed": ("acc += w[(size_t)c * K + k] * v;",
                        "acc += w[(size_t)c * K + (K - 1 - k)] * v;"),
    "bias_dropped": ("double acc = bias ? bias[c] : 0.0;", "double acc = 0.0;"),
    "state_read_newest_first": ("else if (st) v = st[(K - 1) + (src - t0)];",
                                "else if (st) v = st[-(src - t0) - 1];"),
    "short_sequence_loses_history": ("win[k] = src >= 0 ? x[(size_t)(t0 + src) * dim + c] : st[(K - 1) + src];",
                                     "win[k] = src >= 0 ? x[(size_t)(t0 + src) * dim + c] : 0.0;"),
    "silu_sign": ("return act ? v / (1.0 + exp(-v)) : v;", "return act ? v / (1.0 + exp(v)) : v;"),
}

SR_MUTANTS = {
    "philox_wrong_word_multiplied": ("const uint64_t p0 = (uint64_t)0xD2511F53u * c0;",
                                     "const uint64_t p0 = (uint64_t)0xD2511F53u * c1;"),
    "philox_key_not_bumped": ("k0 += 0x9E3779B9u;", "k0 += 0u;"),
    "sr_always_toward_zero": ("double m = lo + (u < f ? s : 0.0);", "double m = lo;"),
    "sr_wrong_spacing": ("s = ldexp(1.0, e - 1 - 10);", "s = ldexp(1.0, e - 10);"),
    "sr_wrong_half_of_word": ("out[i] = oracle_sr_fp16((float)v[i], (e & 1) ? (word >> 16) : (word & 0xFFFFu));",
                              "out[i] = oracle_sr_fp16((float)v[i], (e & 1) ? (word & 0xFFFFu) : (word >> 16));"),
}


def _mutant_lib(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "ssm_oracle.c")).read()
    assert old in src, f"mutant {name}: pattern not found"
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src.replace(old, new, 1))
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    lib = ctypes.CDLL(str(so))
    real = oracle._load()
    for fn in ("oracle_scan", "oracle_state_update", "oracle_causal_conv1d", "oracle_philox4x32",
               "oracle_sr_fp16", "oracle_round_state_f16"):
        getattr(lib, fn).restype = getattr(real, fn).restype
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _caught(pins):
    caught = []
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught.append(pin)
    return caught


@pytest.mark.parametrize("name", sorted(CONV_MUTANTS))
def test_conv_pins_reject_planted_mistakes(tmp_path, name, monkeypatch):
    lib = _mutant_lib(tmp_path, name, *CONV_MUTANTS[name])
    monkeypatch.setattr(oracle, "_lib", lib)
    pins = [lambda: conv_pins.test_matches_numpy_correlate(17, 5, 4),
            conv_pins.test_silu_is_v_times_logistic,
            conv_pins.test_impulse_response_is_the_kernel,
            lambda: conv_pins.test_split_and_carry(1),
            lambda: conv_pins.test_split_and_carry(11),
            conv_pins.test_decode_steps_equal_prefill]
    assert _caught(pins), f"no pin rejects the planted mistake {name!r}"


@pytest.mark.skipif(not os.path.exists(sr_pins.CURAND), reason="cuRAND host library not present")
@pytest.mark.parametrize("name", sorted(SR_MUTANTS))
def test_sr_pins_reject_planted_mistakes(tmp_path, name, monkeypatch):
    lib = _mutant_lib(tmp_path, name, *SR_MUTANTS[name])
    monkeypatch.setattr(oracle, "_lib", lib)

    pins = [lambda: sr_pins.test_philox_matches_curand_host_generator(12345),
            sr_pins.test_sr_returns_a_neighbour_and_keeps_exact_values,
            lambda: sr_pins.test_sr_mean_over_the_random_word_is_exact(-0.3337),
            lambda: sr_pins.test_sr_mean_over_the_random_word_is_exact(1234.567),
            sr_pins.test_round_state_draw_layout]
    assert _caught(pins), f"no pin rejects the planted mistake {name!r}"
