"""GPU parity of the pre-norm (moe_rmsnorm) and of the MoE sublayer with pre-norm
and residual add (moe_forward_block) against the oracle.

- RMSNorm: bf16 outputs equal the oracle's except, rarely, by one bf16 ulp where
  the fp32 reduction and the oracle's fp64 one land on opposite sides of a
  rounding boundary; the fused e4m3 codes and scales are bit-exact against the
  quantisation of the norm's own output.
- Sublayer: y = bf16(h + MoE(RMSNorm(h))); the routing is compared bit for bit on
  the layer's own logits, the output within 1e-2 x RMS of the MoE part (FP8:
  5e-2) plus one bf16 ulp of y for the storage rounding of the stream.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import fine_grained_moe_gemm_b200 as moe
from moe_testlib import cfg_of, oracle_layer, u16, u8, weights_for_forward
from workloads import WORKLOADS, make_inputs, make_norm_gain, make_stream

pytestmark = pytest.mark.gpu
DEV = "cuda"

TINY16 = dataclasses.replace(WORKLOADS["tiny"], name="tiny_bf16", x_f32=False)

_cache = {}


def inputs(wl, device_gen):
    key = (wl.name, device_gen)
    if key not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        W = make_inputs(wl, device_gen)
        W["norm_g"] = make_norm_gain(wl, device_gen)
        _cache[key] = {k: v.to(DEV) for k, v in W.items()}
    return _cache[key]


def bf16_ulp(a):
    a = np.abs(a)
    return np.where(a > 0, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-300))) - 7), 0.0)


def f64(bits):
    return oracle.bf16_bits_to_f64_array(bits)


@pytest.mark.parametrize("T,d", [(1, 7168), (37, 7168), (300, 7168), (64, 256)])
def test_rmsnorm_vs_oracle(T, d):
    wl = dataclasses.replace(TINY16, d=d) if d == 256 else WORKLOADS["decode"]
    h = make_stream(wl, DEV, T=T)
    h[0, : d // 2] = 0.0                                      # a half-zero row
    g = make_norm_gain(wl, DEV)
    out = torch.empty_like(h)
    q = torch.empty((T, d), dtype=torch.uint8, device=DEV)
    sx = torch.empty((T, d // 128), dtype=torch.float32, device=DEV)
    moe.moe_rmsnorm(h, g, out, q, sx)
    torch.cuda.synchronize()
    ref = oracle.rmsnorm(u16(h), u16(g))
    got = u16(out)
    diff = np.abs(f64(got) - f64(ref))
    assert np.all(diff <= bf16_ulp(f64(ref)))
    assert np.count_nonzero(got != ref) <= max(2, got.size // 1000)
    # the fused quantisation is that of the norm's own output, bit for bit
    q2 = torch.empty_like(q)
    sx2 = torch.empty_like(sx)
    moe.moe_quantize_act(out, q2, sx2)
    torch.cuda.synchronize()
    assert torch.equal(q, q2) and torch.equal(sx.view(torch.int32), sx2.view(torch.int32))
    rq, rsx = oracle.quant_act(got)
    assert np.array_equal(u8(q), rq) and np.array_equal(sx.cpu().numpy().view(np.uint32), rsx.view(np.uint32))


def run_block(wl, W, h, y=None, routing=None, events=None):
    cfg = cfg_of(wl)
    T = h.shape[0]
    ws = torch.empty(moe.block_workspace_size(cfg, T), dtype=torch.uint8, device=DEV)
    y = torch.empty_like(h) if y is None else y
    moe.moe_forward_block(cfg, weights_for_forward({k: v for k, v in W.items() if k != "norm_g"}), W["norm_g"], h,
                          W["bias"], y, workspace=ws, routing_out=routing, stage_events=events)
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    return y


def block_reference(wl, W, h, tokens, rel):
    """Runs the block; returns (y_gpu rows, y_ref rows, MoE part of y_ref rows).  The
    routing the layer used (on its own logits) is checked against the oracle's
    selection bit for bit, and its logits against the oracle's router on the
    oracle's RMSNorm(h) within tolerance."""
    T = h.shape[0]
    E, k = wl.n_experts, wl.top_k
    r = {"logits": torch.empty((T, E), dtype=torch.float32, device=DEV),
         "topk_idx": torch.empty((T, k), dtype=torch.int32, device=DEV),
         "topk_w": torch.empty((T, k), dtype=torch.float32, device=DEV)}
    y = run_block(wl, W, h, routing=r)
    l = r["logits"].cpu().numpy()
    ridx, rw = oracle.select(l, W["bias"].cpu().numpy(), wl.n_groups, wl.topk_groups, wl.top_k)
    assert np.array_equal(r["topk_idx"].cpu().numpy(), ridx)
    assert np.array_equal(r["topk_w"].cpu().numpy().view(np.uint32), rw.view(np.uint32))
    xhat = oracle.rmsnorm(u16(h), u16(W["norm_g"]))
    rows = np.unique(np.linspace(0, T - 1, min(T, 8)).astype(np.int64))
    l_ref = oracle.router_logits(xhat[rows], u16(W["w_router"]))
    rms_l = float(np.sqrt(np.mean(l_ref.astype(np.float64) ** 2)))
    assert float(np.max(np.abs(l[rows] - l_ref))) <= 2e-3 * rms_l   # the norm's rare 1-ulp differences included
    L = oracle_layer(wl, W, np.unique(ridx[tokens]))
    moe_ref = oracle.expert_tokens(L, xhat, ridx, rw, tokens)
    h_rows = h[torch.from_numpy(tokens).long().to(DEV)].float().cpu().numpy().astype(np.float64)
    y_ref = h_rows + moe_ref
    y_rows = y[torch.from_numpy(tokens).long().to(DEV)].float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(moe_ref ** 2)))
    err = np.abs(y_rows - y_ref)
    bound = rel * rms + bf16_ulp(y_ref)
    assert np.all(np.isfinite(y_rows))
    assert np.all(err <= bound), f"worst excess {float((err - bound).max()):.4g}, MoE RMS {rms:.4g}"
    return y


@pytest.mark.parametrize("T", [64, 1, 1000])
def test_block_tiny_full(T):
    W = inputs(TINY16, "cpu")
    h = make_stream(TINY16, "cpu", T=T).to(DEV)
    block_reference(TINY16, W, h, np.arange(T, dtype=np.int32), 1e-2)


def test_block_decode_sampled():
    wl = WORKLOADS["decode"]
    W = inputs(wl, DEV)
    h = make_stream(wl, DEV)
    block_reference(wl, W, h, np.array([0, 5, 64, 127], dtype=np.int32), 1e-2)


def test_block_fp8_sampled():
    wl = WORKLOADS["fp8"]
    W = inputs(wl, DEV)
    h = make_stream(wl, DEV, T=300)
    block_reference(wl, W, h, np.array([0, 17, 299], dtype=np.int32), 5e-2)


def test_block_in_place_and_launches():
    """y may be h itself; the block launches the forward's kernels plus the norm
    (the FP8 layer's norm replaces its activation quantisation)."""
    for wl in (TINY16, WORKLOADS["fp8"]):
        W = inputs(wl, "cpu" if wl.d <= 1024 else DEV)
        T = 300
        h = make_stream(wl, DEV, T=T)
        n0 = moe.launch_count()
        y = run_block(wl, W, h)
        n1 = moe.launch_count()
        plan = moe.forward_plan(cfg_of(wl), T)
        assert n1 - n0 == plan["launches"] + 1
        h2 = h.clone()
        run_block(wl, W, h2, y=h2)
        # the combine's fp32 atomics may add in another order: one bf16 ulp of the larger
        # result, plus an fp32-sized slack where h and the MoE part nearly cancel
        a, b = y.float().cpu().numpy().astype(np.float64), h2.float().cpu().numpy().astype(np.float64)
        bound = bf16_ulp(np.maximum(np.abs(a), np.abs(b))) + 1e-6 * float(np.sqrt(np.mean(a * a)))
        excess = np.abs(a - b) - bound
        assert np.all(excess <= 0), f"{int((excess > 0).sum())} elements, worst excess {float(excess.max()):.3g}"
