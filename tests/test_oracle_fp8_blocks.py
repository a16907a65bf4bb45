"""Pins for the oracle's FP8 weight block scales and for a shared expert whose width
differs from the routed experts'.

"Teardown: DeepSeek-V3" section 10 stores expert weights as e4m3 codes with one fp32
scale per 128x128 block: the weight at (r, c) of a [rows, cols] matrix is its code's
value times the scale of block (r // 128, c // 128).  The reference here builds that
matrix the textbook way, as the elementwise product of the codes' values with the
scale grid expanded by a Kronecker product, and evaluates the expert with numpy
matmuls.  Every 128x128 block gets a distinct power-of-two scale and the block grids
are not square (d = 384, H = 256: gate/up 2x3 blocks, down 3x2), so a lookup that swaps
the row and column block, or strides by the wrong block count, lands on another
scale; each test also checks that such a lookup would have been caught.

The shared expert's own hidden width ("Shared expert" box: one always-on expert; the
layer config carries its width separately) is pinned with Hs = 2 H, in bf16 and in
e4m3, so an oracle that evaluated it at the routed width would drop half its hidden
units.
"""
import math

import numpy as np

import oracle

D, H = 384, 256            # 3 column blocks x 2 row blocks for gate/up, 3 x 2 for down

E4M3 = np.array([oracle.e4m3_to_f64(c) for c in range(256)])


def _codes(rng, shape):
    """Random finite e4m3 codes of both signs, magnitudes 2^-6 .. 2^2."""
    mag = rng.integers(0x08, 0x48, size=shape)              # exponent fields 1..8
    sign = rng.integers(0, 2, size=shape) << 7
    return (mag | sign).astype(np.uint8)


def _scale_grid(rows, cols, base):
    """A distinct power of two per 128x128 block: 2^(base + i + rows/128 * j) for block (i, j)."""
    rb, cb = rows // 128, cols // 128
    return np.array([[2.0 ** (base + i + rb * j) for j in range(cb)] for i in range(rb)], np.float32)


def _dequant(codes, s):
    return E4M3[codes] * np.kron(s.astype(np.float64), np.ones((128, 128)))


def _silu(v):
    return v / (1.0 + np.exp(-v))


def _store_h_e4m3(a):
    """h kept as e4m3 with one scale per 128 hidden channels (amax / 448)."""
    out = np.empty_like(a)
    for b in range(0, a.size, 128):
        blk = a[b:b + 128]
        amax = np.abs(blk).max()
        s = amax / 448.0 if amax > 0 else 1.0
        out[b:b + 128] = np.array([oracle.e4m3_to_f64(oracle.e4m3_from_f32(np.float32(v / s))) for v in blk]) * s
    return out


def _ref_fp8_expert(xh, cg, cu, cd, sg, su, sd):
    g = _dequant(cg, sg) @ xh
    u = _dequant(cu, su) @ xh
    return _dequant(cd, sd) @ _store_h_e4m3(_silu(g) * u)


def _wrong_lookups(s, rows, cols):
    """Scale grids that a mis-indexed lookup would read, as full [rows/128, cols/128] grids:
    the row and column block swapped, and the row block strided by rows/128 (wrapping)."""
    rb, cb = rows // 128, cols // 128
    flat = s.ravel()
    swapped = np.array([[flat[(j * rb + i) % flat.size] for j in range(cb)] for i in range(rb)], np.float32)
    strided = np.array([[flat[(i * rb + j) % flat.size] for j in range(cb)] for i in range(rb)], np.float32)
    return [g for g in (swapped, strided) if not np.array_equal(g, s)]


def _fp8_layer(cg, cu, cd, sg, su, sd, shared, Hs=H):
    """One routed expert (slot 0) and the shared expert in e4m3."""
    scg, scu, scd, ssg, ssu, ssd = shared
    return oracle.Layer(D, 1, H, Hs, 1, 2.5, [cg], [cu], [cd], scg, scu, scd,
                        s_gate=[sg], s_up=[su], s_down=[sd], ss_gate=ssg, ss_up=ssu, ss_down=ssd)


def test_fp8_block_scales_select_the_block_of_each_element():
    rng = np.random.default_rng(11)
    cg, cu, cd = _codes(rng, (H, D)), _codes(rng, (H, D)), _codes(rng, (D, H))
    sg, su, sd = _scale_grid(H, D, -9), _scale_grid(H, D, -8), _scale_grid(D, H, -10)
    assert len(np.unique(sg)) == sg.size and len(np.unique(sd)) == sd.size and sg.shape != sd.shape
    zero = np.zeros((H, D), np.uint8), np.zeros((H, D), np.uint8), np.zeros((D, H), np.uint8)
    ones = np.ones((2, 3), np.float32), np.ones((2, 3), np.float32), np.ones((3, 2), np.float32)
    L = _fp8_layer(cg, cu, cd, sg, su, sd, zero + ones)
    xh = rng.standard_normal(D)
    o = oracle.expert_single(L, 0, xh)
    ref = _ref_fp8_expert(xh, cg, cu, cd, sg, su, sd)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert rms > 0
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12 * rms)
    # every mis-indexed lookup, in any one of the three projections, moves the output
    for which in range(3):
        grids = [sg, su, sd]
        shapes = [(H, D), (H, D), (D, H)]
        for wrong in _wrong_lookups(grids[which], *shapes[which]):
            g2 = list(grids)
            g2[which] = wrong
            alt = _ref_fp8_expert(xh, cg, cu, cd, *g2)
            assert np.max(np.abs(alt - o)) > 1e-3 * rms


def test_fp8_block_scales_through_the_layer():
    """The same expert reached through the layer (activation quantised per 1x128 tile,
    routed scale 2.5 x weight, plus the shared expert with its own distinct scales)."""
    rng = np.random.default_rng(12)
    cg, cu, cd = _codes(rng, (H, D)), _codes(rng, (H, D)), _codes(rng, (D, H))
    sg, su, sd = _scale_grid(H, D, -9), _scale_grid(H, D, -8), _scale_grid(D, H, -10)
    qg, qu, qd = _codes(rng, (H, D)), _codes(rng, (H, D)), _codes(rng, (D, H))
    tg, tu, td = _scale_grid(H, D, -10), _scale_grid(H, D, -7), _scale_grid(D, H, -9)
    L = _fp8_layer(cg, cu, cd, sg, su, sd, (qg, qu, qd, tg, tu, td))
    x = oracle.bf16_bits_from_f64_array(rng.standard_normal((2, D)) * 2.0)
    q, sx = oracle.quant_act(x)
    w = np.array([[1.0], [0.75]], np.float32)
    y = oracle.expert_tokens(L, x, np.zeros((2, 1), np.int32), w, [0, 1])
    for t in range(2):
        xh = E4M3[q[t]] * np.repeat(sx[t].astype(np.float64), 128)
        ref = 2.5 * float(w[t, 0]) * _ref_fp8_expert(xh, cg, cu, cd, sg, su, sd) + \
            _ref_fp8_expert(xh, qg, qu, qd, tg, tu, td)
        rms = float(np.sqrt(np.mean(ref ** 2)))
        np.testing.assert_allclose(y[t], ref, rtol=0, atol=1e-12 * rms)


def test_fp8_dense_block_scales():
    """The dense FFN in e4m3 ("SwiGLU MLP" box, the first layers) with distinct block scales."""
    rng = np.random.default_rng(13)
    cg, cu, cd = _codes(rng, (H, D)), _codes(rng, (H, D)), _codes(rng, (D, H))
    sg, su, sd = _scale_grid(H, D, -9), _scale_grid(H, D, -8), _scale_grid(D, H, -10)
    x = oracle.bf16_bits_from_f64_array(rng.standard_normal((3, D)))
    y = oracle.dense_ffn(x, cg, cu, cd, sg, su, sd)
    q, sx = oracle.quant_act(x)
    for t in range(3):
        xh = E4M3[q[t]] * np.repeat(sx[t].astype(np.float64), 128)
        ref = _ref_fp8_expert(xh, cg, cu, cd, sg, su, sd)
        rms = float(np.sqrt(np.mean(ref ** 2)))
        np.testing.assert_allclose(y[t], ref, rtol=0, atol=1e-12 * rms)
        alt = _ref_fp8_expert(xh, cg, cu, cd, sg.T.reshape(sg.shape), su, sd)   # row-major reread
        assert np.max(np.abs(alt - y[t])) > 1e-3 * rms


# ----------------------------------------------------------------------------- shared width

def _bf16(v):
    return oracle.bf16_bits_from_f64_array(np.asarray(v, dtype=np.float64))


def _val(bits):
    return oracle.bf16_bits_to_f64_array(bits)


def _ref_bf16_expert(xh, wg, wu, wd):
    a = _silu(_val(wg) @ xh) * (_val(wu) @ xh)
    return _val(wd) @ _val(_bf16(a))            # h stored in bf16


def test_shared_expert_has_its_own_width_bf16():
    d, Hr, Hs = 64, 32, 96
    rng = np.random.default_rng(14)
    wg, wu, wd = (_bf16(rng.normal(0, 0.1, s)) for s in ((Hr, d), (Hr, d), (d, Hr)))
    vg, vu, vd = (_bf16(rng.normal(0, 0.1, s)) for s in ((Hs, d), (Hs, d), (d, Hs)))
    L = oracle.Layer(d, 1, Hr, Hs, 1, 2.5, [wg], [wu], [wd], vg, vu, vd)
    x = _bf16(rng.standard_normal((3, d)))
    w = np.ones((3, 1), np.float32)
    y = oracle.expert_tokens(L, x, np.zeros((3, 1), np.int32), w, [0, 1, 2])
    for t in range(3):
        xh = _val(x[t])
        shared = _ref_bf16_expert(xh, vg, vu, vd)
        ref = 2.5 * _ref_bf16_expert(xh, wg, wu, wd) + shared
        rms = float(np.sqrt(np.mean(ref ** 2)))
        np.testing.assert_allclose(y[t], ref, rtol=0, atol=1e-12 * rms)
        # the shared expert's hidden units past the routed width carry real weight
        cut = _ref_bf16_expert(xh, vg[:Hr], vu[:Hr], vd[:, :Hr])
        assert np.max(np.abs(cut - shared)) > 1e-2 * rms
        np.testing.assert_allclose(oracle.expert_single(L, -1, xh), shared, rtol=0, atol=1e-12 * rms)


def test_shared_expert_has_its_own_width_fp8():
    Hs = 2 * H
    rng = np.random.default_rng(15)
    cg, cu, cd = _codes(rng, (H, D)), _codes(rng, (H, D)), _codes(rng, (D, H))
    sg, su, sd = _scale_grid(H, D, -9), _scale_grid(H, D, -8), _scale_grid(D, H, -10)
    qg, qu, qd = _codes(rng, (Hs, D)), _codes(rng, (Hs, D)), _codes(rng, (D, Hs))
    tg, tu, td = _scale_grid(Hs, D, -12), _scale_grid(Hs, D, -8), _scale_grid(D, Hs, -12)
    L = _fp8_layer(cg, cu, cd, sg, su, sd, (qg, qu, qd, tg, tu, td), Hs=Hs)
    xh = rng.standard_normal(D)
    shared = oracle.expert_single(L, -1, xh)
    ref = _ref_fp8_expert(xh, qg, qu, qd, tg, tu, td)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    np.testing.assert_allclose(shared, ref, rtol=0, atol=1e-12 * rms)
    routed = _ref_fp8_expert(xh, cg, cu, cd, sg, su, sd)
    np.testing.assert_allclose(oracle.expert_single(L, 0, xh), routed, rtol=0,
                               atol=1e-12 * math.sqrt(np.mean(routed ** 2)))
