"""Pins for the oracle's dense SwiGLU FFN ("SwiGLU MLP" box: the model's first layers
run a dense FFN, hidden 18432, in place of the experts): closed forms on one-hot
weights, and agreement with the expert evaluation it is built from."""
import math

import numpy as np
import torch

import oracle


def _bf16(a):
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _val(bits):
    return oracle.bf16_bits_to_f64_array(bits)


def _silu(z):
    return z / (1.0 + math.exp(-z))


def test_one_hot_closed_form():
    """W_gate = c * e_i rows, W_up = e_i rows, W_down = e_{p(i)} columns for a
    permutation p: y[p(i)] = bf16(SiLU(c * x_i) * x_i), i.e. gate and up are told
    apart and a transposed down projection lands on the wrong features."""
    d = Hd = 8
    c = 3.0
    perm = np.array([3, 0, 7, 1, 6, 2, 5, 4])
    wg, wu, wd = np.zeros((Hd, d)), np.zeros((Hd, d)), np.zeros((d, Hd))
    for i in range(Hd):
        wg[i, i] = c
        wu[i, i] = 1.0
        wd[perm[i], i] = 1.0
    x = np.array([[0.5, -1.25, 2.0, 0.75, 9.0, -9.0, 1.0, 3.0]], dtype=np.float32)
    y = oracle.dense_ffn(_bf16(x), _bf16(wg), _bf16(wu), _bf16(wd))[0]
    ref = np.zeros(d)
    for i in range(Hd):
        ref[perm[i]] = float(_val(_bf16(_silu(c * x[0, i]) * x[0, i])))
    np.testing.assert_allclose(y, ref, rtol=1e-15, atol=0)


def test_dense_equals_the_always_on_expert():
    """The dense FFN is the expert evaluation of the same weights, token by token."""
    rng = np.random.default_rng(0)
    d, Hd, T = 128, 256, 5
    wg, wu = _bf16(rng.normal(0, 0.05, (Hd, d))), _bf16(rng.normal(0, 0.05, (Hd, d)))
    wd = _bf16(rng.normal(0, 0.05, (d, Hd)))
    x = _bf16(rng.standard_normal((T, d)))
    y = oracle.dense_ffn(x, wg, wu, wd)
    L = oracle.Layer(d, 0, Hd, Hd, 0, 1.0, [], [], [], wg, wu, wd)
    for t in range(T):
        np.testing.assert_array_equal(y[t], oracle.expert_single(L, -1, _val(x[t])))
    # rows are independent: a subset of tokens gives the same rows
    np.testing.assert_array_equal(oracle.dense_ffn(x, wg, wu, wd, tokens=np.array([3, 1], np.int32)), y[[3, 1]])


def test_fp8_dense_matches_dequantised_bf16_path_on_exact_values():
    """e4m3 weights whose block scales are 1 and whose values are exact in bf16, and
    inputs that are exact e4m3 values with a block amax of 448 (activation scale 1):
    the FP8 dense FFN equals the bf16 one up to h's own storage (e4m3 vs bf16)."""
    d, Hd = 128, 128
    rng = np.random.default_rng(1)
    codes_g = rng.integers(0, 0x38, (Hd, d)).astype(np.uint8)    # small positive e4m3 values
    codes_u = rng.integers(0, 0x38, (Hd, d)).astype(np.uint8)
    codes_d = rng.integers(0, 0x38, (d, Hd)).astype(np.uint8)
    vals = lambda cds: np.vectorize(oracle.e4m3_to_f64)(cds)
    ones = np.ones((1, 1), np.float32)
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 448.0
    x[0, 1:5] = [1.0, -0.5, 0.25, 2.0]
    y8 = oracle.dense_ffn(_bf16(x), codes_g, codes_u, codes_d, ones, ones, ones)[0]
    y16 = oracle.dense_ffn(_bf16(x), _bf16(vals(codes_g)), _bf16(vals(codes_u)), _bf16(vals(codes_d)))[0]
    rms = float(np.sqrt(np.mean(y16 ** 2)))
    assert np.max(np.abs(y8 - y16)) <= 2.0 ** -3 * rms             # e4m3 h: 3 mantissa bits
    assert not np.array_equal(y8, y16)
