"""Pins for the oracle's permutation (S3) and expert math / combine (S4, S5, S6).

Permutation: against numpy's stable argsort (a library sort) and invariants.
Expert math: closed forms with one-hot weights (which tell gate from up and
catch transposed operands), a second, expert-major formulation written with
numpy matmuls, and the special cases of the combine (scale 0, zero shared
expert, equal weights).
"""
import math

import numpy as np
import pytest

import oracle


# ----------------------------------------------------------------------------- permutation

@pytest.mark.parametrize("T,E,k,seed", [(64, 16, 4, 0), (1, 256, 8, 1), (300, 256, 8, 2), (129, 16, 4, 3)])
def test_permute_matches_stable_sort(T, E, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, src, inv = oracle.permute(idx, E)
    flat = idx.ravel()
    order = np.argsort(flat, kind="stable")        # by expert, then by (t, j) position
    assert np.array_equal(src, order.astype(np.int32))
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(inv[src], np.arange(T * k))          # inv o src = id
    for e in range(E):
        toks = src[offsets[e]:offsets[e + 1]] // k
        assert np.all(np.diff(toks) > 0)                        # strictly ascending t
        assert np.all(flat[src[offsets[e]:offsets[e + 1]]] == e)


def test_permute_empty_and_skewed():
    counts, offsets, src, inv = oracle.permute(np.zeros((0, 8), np.int32), 256)
    assert counts.sum() == 0 and offsets[-1] == 0 and src.size == 0
    idx = np.tile(np.arange(8, dtype=np.int32), (50, 1))       # every token -> experts 0..7
    counts, offsets, src, inv = oracle.permute(idx, 256)
    assert list(counts[:8]) == [50] * 8 and counts[8:].sum() == 0
    assert np.array_equal(src[:50], np.arange(50) * 8)


def test_permute_rejects_bad_expert_id():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 16]], np.int32), 16)


# ----------------------------------------------------------------------------- experts

def _bf16(v):
    return oracle.bf16_bits_from_f64_array(np.asarray(v, dtype=np.float64))


def _bf16_val(v):
    return oracle.bf16_bits_to_f64_array(_bf16(v))


def _silu(z):
    return z / (1.0 + math.exp(-z))


def _layer(d, E, H, k, wg, wu, wd, sg, su, sd, scale=2.5, x_is_f32=False):
    return oracle.Layer(d, E, H, H, k, scale, [_bf16(w) for w in wg], [_bf16(w) for w in wu],
                        [_bf16(w) for w in wd], _bf16(sg), _bf16(su), _bf16(sd), x_is_f32=x_is_f32)


def test_one_hot_closed_form_tells_gate_from_up_and_catches_transposes():
    """W_gate = c * e_i rows, W_up = e_i rows, W_down = e_i columns, d != H:
    y_i = 2.5 * bf16(SiLU(c * x_i) * x_i) for i < H, 0 elsewhere (shared expert off)."""
    d, H, E, k, c = 8, 4, 2, 1, 3.0
    wg = np.zeros((H, d)); wu = np.zeros((H, d)); wd = np.zeros((d, H))
    for i in range(H):
        wg[i, i] = c; wu[i, i] = 1.0; wd[i, i] = 1.0
    z = np.zeros((H, d)), np.zeros((d, H))
    L = _layer(d, E, H, k, [wg, wg], [wu, wu], [wd, wd], z[0], z[0], z[1])
    x = np.array([0.5, -1.25, 2.0, 0.75, 9.0, -9.0, 1.0, 3.0], dtype=np.float32)
    xb = _bf16(x).reshape(1, d)
    y = oracle.expert_tokens(L, xb, np.array([[1]], np.int32), np.array([[1.0]], np.float32), [0])[0]
    ref = np.zeros(d)
    for i in range(H):
        ref[i] = 2.5 * float(_bf16_val(_silu(c * x[i]) * x[i]))
    np.testing.assert_allclose(y, ref, rtol=1e-15, atol=0)
    # swapping gate and up would give SiLU(x_i) * c x_i, which differs here
    swapped = np.array([2.5 * float(_bf16_val(_silu(x[i]) * c * x[i])) for i in range(H)])
    assert np.all(np.abs(swapped - ref[:H]) > 1e-3)


def test_zero_gate_gives_zero_output():
    """SiLU(0) = 0 (a sigmoid in place of SiLU would give 0.5 * up)."""
    rng = np.random.default_rng(0)
    d, H, E, k = 16, 8, 1, 1
    wg = np.zeros((H, d)); wu = rng.standard_normal((H, d)); wd = rng.standard_normal((d, H))
    L = _layer(d, E, H, k, [wg], [wu], [wd], wg, wu, wd)
    xb = _bf16(rng.standard_normal((1, d)))
    y = oracle.expert_tokens(L, xb, np.array([[0]], np.int32), np.array([[1.0]], np.float32), [0])
    assert np.all(y == 0.0)


def _expert_major(x64, idx, w, wg, wu, wd, sg, su, sd, scale):
    """Second formulation: per expert, gather its rows, matmul (numpy), scatter-add."""
    T, k = idx.shape
    y = np.zeros((T, x64.shape[1]))
    for e in np.unique(idx):
        rows, slots = np.nonzero(idx == e)
        xe = x64[rows]
        h = _bf16_val((xe @ wg[e].T) / (1 + np.exp(-(xe @ wg[e].T))) * (xe @ wu[e].T))
        y[rows] += scale * w[rows, slots][:, None] * (h @ wd[e].T)
    hs = _bf16_val((x64 @ sg.T) / (1 + np.exp(-(x64 @ sg.T))) * (x64 @ su.T))
    return y + hs @ sd.T


def test_token_major_equals_expert_major():
    rng = np.random.default_rng(1)
    T, d, H, E, k = 24, 32, 16, 6, 3
    bf = lambda a: _bf16_val(a)
    wg = bf(rng.standard_normal((E, H, d)) * 0.2); wu = bf(rng.standard_normal((E, H, d)) * 0.2)
    wd = bf(rng.standard_normal((E, d, H)) * 0.2)
    sg = bf(rng.standard_normal((H, d)) * 0.2); su = bf(rng.standard_normal((H, d)) * 0.2)
    sd = bf(rng.standard_normal((d, H)) * 0.2)
    x = rng.standard_normal((T, d)).astype(np.float32)          # fp32 input, rounded to bf16 inside
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w = rng.uniform(0.1, 1, (T, k)).astype(np.float32)
    L = _layer(d, E, H, k, list(wg), list(wu), list(wd), sg, su, sd, scale=2.5, x_is_f32=True)
    y = oracle.expert_tokens(L, x, idx, w, np.arange(T))
    ref = _expert_major(bf(x), idx, w.astype(np.float64), wg, wu, wd, sg, su, sd, 2.5)
    np.testing.assert_allclose(y, ref, rtol=1e-9, atol=1e-12)


def test_combine_special_cases():
    rng = np.random.default_rng(2)
    T, d, H, E, k = 6, 16, 8, 4, 2
    bf = lambda a: _bf16_val(a)
    wg = bf(rng.standard_normal((E, H, d))); wu = bf(rng.standard_normal((E, H, d)))
    wd = bf(rng.standard_normal((E, d, H)))
    sg = bf(rng.standard_normal((H, d))); su = bf(rng.standard_normal((H, d)))
    sd = bf(rng.standard_normal((d, H)))
    xb = _bf16(rng.standard_normal((T, d)))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w = np.full((T, k), 0.5, np.float32)
    full = oracle.expert_tokens(_layer(d, E, H, k, list(wg), list(wu), list(wd), sg, su, sd), xb, idx, w, np.arange(T))
    # routed scale 0 leaves the shared expert alone
    only_shared = oracle.expert_tokens(_layer(d, E, H, k, list(wg), list(wu), list(wd), sg, su, sd, scale=0.0),
                                       xb, idx, w, np.arange(T))
    z = np.zeros_like(sd)
    only_routed = oracle.expert_tokens(_layer(d, E, H, k, list(wg), list(wu), list(wd), sg, su, z),
                                       xb, idx, w, np.arange(T))
    np.testing.assert_allclose(full, only_shared + only_routed, rtol=1e-12, atol=1e-12)
    # the routed part is linear in the scale and in each slot weight
    half = oracle.expert_tokens(_layer(d, E, H, k, list(wg), list(wu), list(wd), sg, su, z, scale=1.25),
                                xb, idx, w, np.arange(T))
    np.testing.assert_allclose(only_routed, 2 * half, rtol=1e-12, atol=1e-12)
    # sampled token subset equals the matching rows of the full run
    sub = oracle.expert_tokens(_layer(d, E, H, k, list(wg), list(wu), list(wd), sg, su, sd), xb, idx, w, [4, 1])
    assert np.array_equal(sub, full[[4, 1]])


# ----------------------------------------------------------------------------- FP8

def test_quant_act_codes_and_scales():
    rng = np.random.default_rng(3)
    T, d = 5, 256
    x = rng.standard_normal((T, d)) * 3
    x[2, :128] = 0.0                                          # amax 0 -> scale 1, codes 0
    x[3, 5] = 1000.0                                          # one outlier sets its block's scale
    xb = _bf16(x)
    q, sx = oracle.quant_act(xb)
    xv = oracle.bf16_bits_to_f64_array(xb)
    for t in range(T):
        for b in range(2):
            blk = xv[t, b * 128:(b + 1) * 128]
            amax = np.float32(np.abs(blk).max())
            scale = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
            assert sx[t, b] == scale
            codes = q[t, b * 128:(b + 1) * 128]
            deq = np.array([oracle.e4m3_to_f64(c) for c in codes]) * float(scale)
            # the amax element maps to 448 exactly (up to the fp32 divide)
            if amax > 0:
                assert np.max(np.abs([oracle.e4m3_to_f64(c) for c in codes])) == 448.0
            # every element within half an e4m3 step (relative 2^-4) or the subnormal floor
            err = np.abs(deq - blk)
            assert np.all(err <= np.maximum(np.abs(blk) * 2 ** -4, 2 ** -10 * float(scale)) + 1e-30)
    assert np.all(q[2, :128] == 0) and np.all(sx[2, 0] == 1.0)


def test_fp8_expert_closed_form():
    """e4m3 one-hot weights with block scales: y_i = 2.5 * h_i with h quantised
    per 128 channels, W_gate = c e_i (c on the e4m3 grid) times the block scale."""
    d, H, E, k = 256, 128, 1, 1
    c = 3.0                                                   # e4m3 exact
    wg = np.zeros((H, d), np.uint8); wu = np.zeros((H, d), np.uint8); wd = np.zeros((d, H), np.uint8)
    one, cc = oracle.e4m3_from_f32(1.0), oracle.e4m3_from_f32(c)
    for i in range(H):
        wg[i, i] = cc; wu[i, i] = one; wd[i, i] = one
    sgate = np.full((1, 2), 0.5, np.float32)                  # block scales
    sup = np.full((1, 2), 2.0, np.float32)
    sdown = np.full((2, 1), 0.25, np.float32)
    zq = np.zeros((H, d), np.uint8)
    L = oracle.Layer(d, E, H, H, k, 2.5, [wg], [wu], [wd], zq, zq, np.zeros((d, H), np.uint8),
                     s_gate=[sgate], s_up=[sup], s_down=[sdown], ss_gate=sgate, ss_up=sup, ss_down=sdown)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((1, d)) * 2
    xb = _bf16(x)
    q, sx = oracle.quant_act(xb)
    xh = np.array([oracle.e4m3_to_f64(v) for v in q[0]]) * np.repeat(sx[0].astype(np.float64), 128)
    y = oracle.expert_tokens(L, xb, np.array([[0]], np.int32), np.array([[1.0]], np.float32), [0])[0]
    a = np.array([_silu(c * 0.5 * xh[i]) * (2.0 * xh[i]) for i in range(H)])
    amax = np.abs(a).max()
    s = amax / 448.0
    hq = np.array([oracle.e4m3_to_f64(oracle.e4m3_from_f32(np.float32(v / s))) for v in a]) * s
    ref = np.zeros(d)
    ref[:H] = 2.5 * 0.25 * hq
    np.testing.assert_allclose(y, ref, rtol=1e-14, atol=1e-300)
