"""moe_forward_noalloc: the layer with its scratch in the library's static
device array, for callers that cannot allocate device memory when they call
the layer.  Collected last on purpose (file name), so that a run stopping at
its first failure has run every other test first.

Each check calls the entry point through the C ABI twice in a row, on
different inputs, and compares both outputs with moe_forward (caller
workspace) at the layer tolerance, max |err| <= 1e-2 x RMS.  The second call
inherits whatever the first left in the array; it is also compared with the
CPU oracle, and the accumulating form (y += layer(x)) is checked after a call
of another batch size, for both output dtypes."""
import ctypes

import numpy as np
import pytest
import torch

import fine_grained_moe_gemm_b200 as moe
import oracle
from moe_testlib import assert_close_bf16, assert_close_rms, cfg_of, oracle_layer, u16, weights_for_forward, x_host
from workloads import WORKLOADS, make_inputs, make_x

pytestmark = pytest.mark.gpu

DEV = "cuda"
REL = 1e-2
NOALLOC_MAX_BYTES = 32 << 20


def _noalloc_fn():
    L = moe.lib()
    f = L.moe_forward_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.restype = I
    f.argtypes = [ctypes.POINTER(moe.MoeConfig), ctypes.POINTER(moe.MoeWeights), P, P, I, P, I, I, P]
    return f


def _noalloc(cfg, mw, x, bias, y, accumulate=False):
    st = _noalloc_fn()(ctypes.byref(cfg), ctypes.byref(mw), ctypes.c_void_p(x.data_ptr()),
                       ctypes.c_void_p(bias.data_ptr()), x.shape[0], ctypes.c_void_p(y.data_ptr()),
                       moe.MOE_F32 if y.dtype == torch.float32 else moe.MOE_BF16, int(accumulate),
                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _reference(cfg, weights, x, bias, y_dtype, y0=None):
    ws = torch.empty(moe.workspace_size(cfg, x.shape[0]), dtype=torch.uint8, device=DEV)
    y = y0.clone() if y0 is not None else torch.empty((x.shape[0], cfg.d), dtype=y_dtype, device=DEV)
    moe.moe_forward(cfg, weights, x, bias, y, accumulate=y0 is not None, workspace=ws)
    return y


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(b ** 2)))
    assert np.all(np.isfinite(a))
    assert float(np.max(np.abs(a - b))) <= REL * rms


@pytest.mark.parametrize("name,Ts", [("tiny", (64, 37)), ("decode", (128, 158))])
def test_noalloc_matches_forward_on_two_calls(name, Ts):
    wl = WORKLOADS[name]
    cfg = cfg_of(wl)
    W = {k: v.to(DEV) for k, v in make_inputs(wl, "cpu" if wl.d <= 1024 else DEV).items()}
    weights = weights_for_forward(W)
    mw = moe.make_weights(weights)
    for call, T in enumerate(Ts):
        x = make_x(wl, "cpu" if wl.d <= 1024 else DEV, seed=call + 1, T=T).to(DEV)
        assert moe.workspace_size(cfg, T) <= NOALLOC_MAX_BYTES
        for y_dtype in (torch.float32, torch.bfloat16):
            y = torch.full((T, wl.d), float("nan"), dtype=y_dtype, device=DEV)
            assert _noalloc(cfg, mw, x, W["bias"], y) == moe.MOE_OK
            ref = _reference(cfg, weights, x, W["bias"], y_dtype)
            torch.cuda.synchronize()
            _close(y, ref)
    assert moe.device_error() == 0


def test_noalloc_rejects_sizes_beyond_the_array():
    wl = WORKLOADS["decode"]
    cfg = cfg_of(wl)
    T = 4096
    assert moe.workspace_size(cfg, T) > NOALLOC_MAX_BYTES
    dummy = torch.zeros(16, dtype=torch.float32, device=DEV)
    mw = moe.MoeWeights()
    st = _noalloc_fn()(ctypes.byref(cfg), ctypes.byref(mw), ctypes.c_void_p(dummy.data_ptr()),
                       ctypes.c_void_p(dummy.data_ptr()), T, ctypes.c_void_p(dummy.data_ptr()), moe.MOE_BF16, 0,
                       None)
    assert st == moe.MOE_ERR_WORKSPACE


def _inputs(wl):
    gen = "cpu" if wl.d <= 1024 else DEV
    W = {k: v.to(DEV) for k, v in make_inputs(wl, gen).items()}
    return W, gen


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_noalloc_accumulate_after_a_call_of_another_size(y_dtype):
    """y += layer(x) on the static array, right after a call with another T: the fp32
    output accumulates in place, the bf16 output reads its residual from y."""
    wl = WORKLOADS["decode"]
    cfg = cfg_of(wl)
    W, gen = _inputs(wl)
    weights = weights_for_forward(W)
    mw = moe.make_weights(weights)
    x1 = make_x(wl, gen, seed=5, T=150).to(DEV)
    y1 = torch.empty((150, wl.d), dtype=torch.float32, device=DEV)
    assert _noalloc(cfg, mw, x1, W["bias"], y1) == moe.MOE_OK
    T = 96
    x = make_x(wl, gen, seed=6, T=T).to(DEV)
    y0 = (torch.randn((T, wl.d), generator=torch.Generator(DEV).manual_seed(7), device=DEV)).to(y_dtype)
    y = y0.clone()
    assert _noalloc(cfg, mw, x, W["bias"], y, accumulate=True) == moe.MOE_OK
    ref = _reference(cfg, weights, x, W["bias"], y_dtype, y0=y0)
    torch.cuda.synchronize()
    # the layer's part at the layer tolerance; a bf16 output may also land one bf16 ulp of
    # |y| apart, its own storage rounding of residual + layer
    got, want = y.double().cpu().numpy(), ref.double().cpu().numpy()
    part = want - y0.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(part ** 2)))
    ulp = 0.0
    if y_dtype == torch.bfloat16:
        a = np.abs(want)
        ulp = np.where(a > 0, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-300))) - 7), 0.0)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - want) <= REL * rms + ulp)
    assert moe.device_error() == 0


def test_noalloc_second_call_matches_the_oracle():
    """The tiny layer, twice: the second call (on the first call's leftovers) against
    the CPU oracle on every token, routed with the GPU's own logits."""
    wl = WORKLOADS["tiny"]
    cfg = cfg_of(wl)
    W, gen = _inputs(wl)
    mw = moe.make_weights(weights_for_forward(W))
    x1 = make_x(wl, gen, seed=3, T=64).to(DEV)
    y1 = torch.empty((64, wl.d), dtype=torch.float32, device=DEV)
    assert _noalloc(cfg, mw, x1, W["bias"], y1) == moe.MOE_OK
    T = 53
    x = make_x(wl, gen, seed=4, T=T).to(DEV)
    y = torch.full((T, wl.d), float("nan"), dtype=torch.float32, device=DEV)
    yb = torch.full((T, wl.d), float("nan"), dtype=torch.bfloat16, device=DEV)
    assert _noalloc(cfg, mw, x, W["bias"], y) == moe.MOE_OK
    assert _noalloc(cfg, mw, x, W["bias"], yb) == moe.MOE_OK
    logits = torch.empty((T, wl.n_experts), dtype=torch.float32, device=DEV)
    idx = torch.empty((T, wl.top_k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, wl.top_k), dtype=torch.float32, device=DEV)
    moe.moe_route(cfg, x, W["w_router"], logits, W["bias"], idx, w)
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    ridx, rw = oracle.select(logits.cpu().numpy(), W["bias"].cpu().numpy(), wl.n_groups, wl.topk_groups, wl.top_k)
    L = oracle_layer(wl, W, ridx.ravel())
    ref = oracle.expert_tokens(L, x_host(x), ridx, rw, np.arange(T))
    assert_close_rms(y.cpu().numpy(), ref, REL, "noalloc fp32")
    assert_close_bf16(yb, ref, REL, "noalloc bf16")
