"""Pins for the oracle's pre-norm ("DeepSeek-V3" llm-vis, "RMSNorm" box: unit RMS over
the features with eps 1e-6, cast to the activation dtype, then the per-feature gain).

Each case fixes a part of the definition by a value reached another way: a constant
row and a one-hot row have closed forms, the sign, the gain and a permutation of the
features act in known ways, and the output's RMS is 1 up to bf16 rounding."""
import numpy as np
import torch

import oracle


def bf16(vals) -> np.ndarray:
    """bf16 bit patterns of the given values (torch's round to nearest even)."""
    t = torch.as_tensor(np.asarray(vals, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def f64(bits) -> np.ndarray:
    return oracle.bf16_bits_to_f64_array(bits)


ONES = {d: bf16(np.ones(d)) for d in (256, 7168)}


def test_constant_rows():
    d = 256
    # |c| large: c / sqrt(c^2 + eps) is 1 to within far less than a bf16 ulp
    for c, want in ((2.0 ** 10, 1.0), (-3.0, -1.0), (1.0, 1.0)):
        out = oracle.rmsnorm(bf16(np.full((1, d), c)), ONES[d])
        assert np.all(f64(out) == want)
    # c^2 = 2^-20 is about eps: without eps the row would come out as exactly 1
    c = 2.0 ** -10
    out = f64(oracle.rmsnorm(bf16(np.full((1, d), c)), ONES[d]))
    assert np.all(out == out[0, 0])
    closed = c / np.sqrt(c * c + np.float64(np.float32(1e-6)))          # 0.6987...
    assert abs(out[0, 0] - closed) <= 2.0 ** -9 and out[0, 0] < 0.75


def test_all_zero_row_stays_zero():
    out = oracle.rmsnorm(bf16(np.zeros((2, 256))), ONES[256])
    assert np.all(out == 0)


def test_one_hot_row_is_sqrt_d():
    # mean over d, not sum: a lone 1.5 among 255 zeros normalises to sqrt(256) = 16
    d = 256
    h = np.zeros((1, d))
    h[0, 37] = 1.5
    out = f64(oracle.rmsnorm(bf16(h), ONES[d]))
    assert out[0, 37] == 16.0
    assert np.count_nonzero(out) == 1


def test_sign_symmetry_bitwise():
    rng = np.random.default_rng(0)
    h = rng.standard_normal((4, 7168))
    a = oracle.rmsnorm(bf16(h), ONES[7168])
    b = oracle.rmsnorm(bf16(-h), ONES[7168])
    nz = (a & 0x7FFF) != 0
    assert np.array_equal(a[nz] ^ 0x8000, b[nz])


def test_gain_power_of_two_is_exact_and_rounding_precedes_gain():
    rng = np.random.default_rng(1)
    h = bf16(rng.standard_normal((3, 7168)))
    one = f64(oracle.rmsnorm(h, ONES[7168]))
    two = f64(oracle.rmsnorm(h, bf16(np.full(7168, 2.0))))
    assert np.array_equal(two, 2 * one)
    # gain 3: the normalised value is rounded to bf16 first, then multiplied and rounded again
    three = oracle.rmsnorm(h, bf16(np.full(7168, 3.0)))
    want = bf16((3.0 * one).astype(np.float32))               # 3 x bf16 is exact in fp32
    assert np.array_equal(three, want)
    # a per-feature gain picks the feature's own g
    g = rng.uniform(0.5, 1.5, 7168)
    mixed = oracle.rmsnorm(h, bf16(g))
    assert np.array_equal(mixed, bf16((one * f64(bf16(g))).astype(np.float32)))


def test_feature_permutation_invariance():
    # values on a 2^-6 grid in [-4, 4): every square and every partial sum is exact
    # in fp64, so the mean does not depend on the order of the features
    rng = np.random.default_rng(2)
    h = rng.integers(-256, 256, (3, 7168)) / 64.0
    perm = rng.permutation(7168)
    a = oracle.rmsnorm(bf16(h), ONES[7168])
    b = oracle.rmsnorm(bf16(h[:, perm]), ONES[7168])
    assert np.array_equal(a[:, perm], b)


def test_output_rms_is_one():
    # unit RMS up to bf16 rounding; at small inputs eps pulls it below 1 by m / (m + eps)
    rng = np.random.default_rng(3)
    for scale, want in ((300.0, 1.0), (1.0, 1.0), (1e-2, 1e-4 / (1e-4 + 1e-6))):
        out = f64(oracle.rmsnorm(bf16(rng.standard_normal((5, 7168)) * scale), ONES[7168]))
        ms = np.mean(out * out, axis=1)
        assert np.all(np.abs(ms - want) < 2.0 ** -7)
        if scale < 1:
            assert np.all(ms < 0.995)
