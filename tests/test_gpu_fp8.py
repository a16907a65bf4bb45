"""GPU parity of the FP8 path ("Teardown: DeepSeek-V3", section 10).

- Activation quantisation (moe_quantize_act): codes and scales bit-exact
  against the oracle (both take every decision in the same fp32 arithmetic).
- Whole layer with e4m3 expert weights and 128x128 block scales: max |err| <=
  5e-2 x RMS(y_ref) against the oracle, which dequantises exactly and
  accumulates in fp64 (the FP8 layer-output bar).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import fine_grained_moe_gemm_b200 as moe
from moe_testlib import assert_close_bf16, assert_close_rms, cfg_of, oracle_layer, u16, weights_for_forward, x_host
from workloads import WORKLOADS, make_inputs, make_x

pytestmark = pytest.mark.gpu

DEV = "cuda"
REL = 5e-2


@pytest.mark.parametrize("T,d", [(1, 128), (7, 256), (300, 7168)])
def test_quant_act_bit_exact(T, d):
    rng = np.random.default_rng(T)
    x = rng.standard_normal((T, d)).astype(np.float32) * 3
    x[0, :128] = 0.0                                  # all-zero block: scale 1
    if T > 1:
        x[1, 5] = 3e4                                 # outlier sets its block's scale
        x[1, 130 % d] = -1e-8                         # rounds to a signed zero
    if T > 2:
        x[2] *= 1e-6                                  # values in the e4m3 subnormal range
    x[0, 129 % d] = -0.0
    xb = torch.from_numpy(x).to(torch.bfloat16).to(DEV)
    q = torch.empty((T, d), dtype=torch.uint8, device=DEV)
    sx = torch.empty((T, d // 128), dtype=torch.float32, device=DEV)
    moe.moe_quantize_act(xb, q, sx)
    torch.cuda.synchronize()
    rq, rsx = oracle.quant_act(u16(xb))
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), rsx.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), rq)


_cache = {}


def fp8_inputs(name):
    if name not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        if name == "tiny_fp8":
            wl = dataclasses.replace(WORKLOADS["tiny"], name="tiny_fp8", x_f32=False, fp8=True)
            W = {k: v.to(DEV) for k, v in make_inputs(wl, "cpu").items()}
        else:
            wl = WORKLOADS[name]
            W = {k: v.to(DEV) for k, v in make_inputs(wl, DEV).items()}
        _cache[name] = (wl, W)
    return _cache[name]


def run(wl, W, x, y_dtype):
    cfg = cfg_of(wl)
    T = x.shape[0]
    ws = torch.empty(moe.workspace_size(cfg, T), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, wl.d), dtype=y_dtype, device=DEV)
    moe.moe_forward(cfg, weights_for_forward(W), x, W["bias"], y, workspace=ws)
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    return y


def reference(wl, W, x, tokens):
    """Oracle output for `tokens`, routed as moe_forward routed (its own logits,
    checked bit for bit against the oracle's selection on them)."""
    cfg = cfg_of(wl)
    T = x.shape[0]
    r = {"logits": torch.empty((T, wl.n_experts), dtype=torch.float32, device=DEV),
         "topk_idx": torch.empty((T, wl.top_k), dtype=torch.int32, device=DEV),
         "topk_w": torch.empty((T, wl.top_k), dtype=torch.float32, device=DEV)}
    ws = torch.empty(moe.workspace_size(cfg, T), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, wl.d), dtype=torch.float32, device=DEV)
    moe.moe_forward(cfg, weights_for_forward(W), x, W["bias"], y, workspace=ws, routing_out=r)
    torch.cuda.synchronize()
    ridx, rw = oracle.select(r["logits"].cpu().numpy(), W["bias"].cpu().numpy(), wl.n_groups, wl.topk_groups,
                             wl.top_k)
    assert np.array_equal(r["topk_idx"].cpu().numpy(), ridx)
    assert np.array_equal(r["topk_w"].cpu().numpy().view(np.uint32), rw.view(np.uint32))
    L = oracle_layer(wl, W, np.unique(ridx[tokens]))
    return oracle.expert_tokens(L, x_host(x), ridx, rw, tokens)


@pytest.mark.parametrize("T", [64, 1, 129, 1000])
def test_fp8_tiny_full(T):
    wl, W = fp8_inputs("tiny_fp8")
    x = make_x(wl, "cpu", T=T).to(DEV)
    toks = np.arange(T, dtype=np.int32)
    ref = reference(wl, W, x, toks)
    assert_close_rms(run(wl, W, x, torch.float32).cpu().numpy(), ref, REL)
    assert_close_bf16(run(wl, W, x, torch.bfloat16), ref, REL)


@pytest.mark.parametrize("T", [8192, 1, 37, 300, 1000, 4096])
def test_fp8_deepseek_sampled(T):
    wl, W = fp8_inputs("fp8")
    x = W["x"] if T == wl.T else make_x(wl, DEV, T=T)
    rng = np.random.default_rng(T)
    toks = np.array(sorted(set([0, T - 1]) | set(rng.choice(T, min(T, 5), replace=False).tolist())), np.int32)
    ref = reference(wl, W, x, toks)
    yb = run(wl, W, x, torch.bfloat16)
    assert_close_bf16(yb[torch.from_numpy(toks).long().to(DEV)], ref, REL)
