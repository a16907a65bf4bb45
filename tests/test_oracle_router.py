"""Pins of the oracle's router GEMM (S1, "MoE router" box: logits = x . W_r^T with high-precision
accumulation) against closed forms that do not restate its formula:
  - a one-hot x row (value v) selects v times one column of W_r, exactly;
  - with small-integer x and W_r every product and partial sum is an exact integer, so the logits
    must equal the integer matrix product computed in int64.
The shapes are rectangular (E != d), so a transposed operand or a row/column mix-up fails."""
import numpy as np

import oracle


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Values exactly representable in bf16 -> their bit patterns."""
    u = np.asarray(a, np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


def test_one_hot_rows_select_columns():
    rng = np.random.default_rng(0)
    E, d = 16, 256
    wr = rng.standard_normal((E, d)).astype(np.float32) * 0.02
    wr_bits = oracle.bf16_bits_from_f64_array(wr.astype(np.float64))
    wr_vals = oracle.bf16_bits_to_f64_array(wr_bits)
    cols = [0, 7, 255, 128]
    vals = [1.0, 3.0, -0.5, 0.25]
    x = np.zeros((len(cols), d), np.float32)
    for t, (c, v) in enumerate(zip(cols, vals)):
        x[t, c] = v
    for xin in (x, bf16_bits(x)):                       # fp32 activations and bf16 bit patterns
        l = oracle.router_logits(xin, wr_bits)
        assert l.shape == (len(cols), E) and l.dtype == np.float32
        for t, (c, v) in enumerate(zip(cols, vals)):
            assert np.array_equal(l[t], (v * wr_vals[:, c]).astype(np.float32))


def test_integer_inputs_give_the_exact_integer_product():
    rng = np.random.default_rng(1)
    T, E, d = 5, 24, 384
    xi = rng.integers(-8, 9, size=(T, d))
    wi = rng.integers(-8, 9, size=(E, d))
    exact = xi.astype(np.int64) @ wi.astype(np.int64).T  # |sum| <= 384 * 64: exact in fp32
    l = oracle.router_logits(bf16_bits(xi.astype(np.float32)), bf16_bits(wi.astype(np.float32)))
    assert np.array_equal(l.astype(np.int64), exact) and np.all(l == exact.astype(np.float32))
    l32 = oracle.router_logits(xi.astype(np.float32), bf16_bits(wi.astype(np.float32)))
    assert np.array_equal(l32, l)
