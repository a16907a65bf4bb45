"""Pins for the oracle's scalar formats: bf16 rounding, OCP E4M3, sigmoid_spec.

Each check compares the oracle with something other than itself: a library
conversion (torch), an exact brute force over neighbouring grid points, the
format's published extreme values, or the fp64 definition of the sigmoid.
"""
import ctypes
import os
import subprocess
import tempfile
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


# ----------------------------------------------------------------------------- bf16

def test_bf16_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(5000) * 1e-38).astype(np.float32),      # subnormal range
        (rng.standard_normal(5000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], dtype=np.float32),
    ])
    ours = oracle.bf16_bits_from_f64_array(vals.astype(np.float64))
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def _bf16_exact(h):
    u = np.array([int(h) << 16], dtype=np.uint32).view(np.float32)[0]
    return Fraction(float(u))


def test_bf16_from_f64_is_nearest_even_brute_force():
    """Direct fp64 -> bf16 rounding against an exact search over neighbouring bf16 values."""
    rng = np.random.default_rng(2)
    vals = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-20, 20, 3000))
    # exact ties between two bf16 values, and values a hair away from ties
    for base in (1.0, 1.5, 3.25, 1e-3):
        b = np.float32(base)
        vals += [float(b) * (1 + 2 ** -8), float(b) * (1 + 3 * 2 ** -8), float(b) * (1 + 2 ** -8) + 1e-30]
    for v in vals:
        v = float(v)
        h = oracle.bf16_from_f64(v)
        target = Fraction(v)
        t32 = np.array([np.float32(v)], dtype=np.float32).view(np.uint32)[0] >> 16
        sign = 0x8000 if v < 0 else 0
        cands = []
        for c in range(int(t32 & 0x7FFF) - 2, int(t32 & 0x7FFF) + 3):
            if 0 <= c < 0x7F80:
                cands.append(sign | c)
        best = min(cands, key=lambda c: (abs(_bf16_exact(c) - target), c & 1))
        assert h == best, (v, hex(h), hex(best))


# ----------------------------------------------------------------------------- e4m3

def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([oracle.e4m3_to_f64(c) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert nan.sum() == 2                                   # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_published_extremes():
    assert oracle.e4m3_to_f64(0x7E) == 448.0               # largest finite
    assert oracle.e4m3_to_f64(0x08) == 2.0 ** -6           # smallest normal
    assert oracle.e4m3_to_f64(0x01) == 2.0 ** -9           # smallest subnormal
    assert oracle.e4m3_to_f64(0x38) == 1.0
    assert oracle.e4m3_from_f32(448.0) == 0x7E
    assert oracle.e4m3_from_f32(1000.0) == 0x7E            # saturation, no infinity
    assert oracle.e4m3_from_f32(-1e30) == 0xFE
    assert oracle.e4m3_from_f32(460.0) == 0x7E
    assert oracle.e4m3_from_f32(2.0 ** -11) == 0x00        # below half the smallest subnormal
    assert oracle.e4m3_from_f32(2.0 ** -10) == 0x00        # tie with 0 -> even (0)
    assert oracle.e4m3_from_f32(3 * 2.0 ** -10) == 0x02    # tie between 1 and 2 -> even (2)


def test_e4m3_round_trip_and_ties():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = oracle.e4m3_to_f64(c)
        back = oracle.e4m3_from_f32(v)
        assert back == c or (v == 0.0 and back in (0x00, 0x80)), c
    # midpoint between 1.0 (0x38, even mantissa) and 1.125 (0x39) rounds to 1.0;
    # midpoint between 1.125 and 1.25 (0x3A) rounds to 1.25
    assert oracle.e4m3_from_f32(1.0625) == 0x38
    assert oracle.e4m3_from_f32(1.1875) == 0x3A


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(3)
    vals = np.concatenate([
        (rng.standard_normal(20000) * 50).astype(np.float32),
        (rng.standard_normal(5000) * 1e-2).astype(np.float32),
        rng.uniform(-448, 448, 5000).astype(np.float32),
    ])
    vals = np.clip(vals, -448, 448).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_from_f32(v) for v in vals], dtype=np.uint8)
    # torch and the oracle may differ only in the sign of a zero result
    diff = ours != ref
    assert np.all((ours[diff] & 0x7F) == 0) and np.all((ref[diff] & 0x7F) == 0)


# ----------------------------------------------------------------------------- sigmoid

def _sweep_lib():
    src = os.path.join(HERE, "native", "sigmoid_sweep.c")
    libdir = os.path.dirname(oracle.build())
    out = os.path.join(tempfile.mkdtemp(prefix="sigsweep"), "libsweep.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", src, "-o", out,
                    f"-L{libdir}", "-l:liboracle.so", f"-Wl,-rpath,{libdir}", "-lm"], check=True)
    L = ctypes.CDLL(out)
    L.sigmoid_sweep.restype = ctypes.c_double
    L.sigmoid_sweep.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int64)]
    return L


def test_sigmoid_exhaustive_within_2p5ulp_and_monotone():
    """Every fp32 l in [-88, 88] (about 2.1e9 values) against the fp64 definition.

    Bound: exp_spec and 1 + e each round once (half an ulp of their result)
    and the divide rounds once; when e sits at the bottom of its binade,
    s = 1/(1+e) sits at the top of its own, so the first two count double in
    ulps of s: 2 * 0.5 + 2 * 0.5 + 0.5 = 2.5."""
    L = _sweep_lib()
    worst = ctypes.c_float()
    nonmono = ctypes.c_int64()
    mx = L.sigmoid_sweep(-88.0, 88.0, os.cpu_count() or 1, ctypes.byref(worst), ctypes.byref(nonmono))
    assert nonmono.value == 0
    assert mx <= 2.5, f"max error {mx} ulp at l={worst.value}"


def test_sigmoid_special_values():
    s = oracle.sigmoid(np.array([0.0, 100.0, 88.0, 30.0, -30.0], dtype=np.float32))
    assert s[0] == np.float32(0.5)
    assert s[1] == 1.0 and s[2] == 1.0 and s[3] == 1.0
    assert abs(float(s[4]) - 1.0 / (1.0 + np.exp(30.0))) <= 2 * np.spacing(np.float32(s[4]))
    rng = np.random.default_rng(4)
    l = rng.standard_normal(1000).astype(np.float32) * 8
    s1, s2 = oracle.sigmoid(l), oracle.sigmoid(-l)
    assert np.all(np.abs(s1.astype(np.float64) + s2 - 1.0) < 4e-7)
