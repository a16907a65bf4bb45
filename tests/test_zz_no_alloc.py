"""moe_forward_noalloc: the layer with its scratch in the library's static
device array, for callers that cannot allocate device memory when they call
the layer.  Collected last on purpose (file name), so that a run stopping at
its first failure has run every other test first.

Each check calls the entry point through the C ABI twice in a row, on
different inputs, and compares both outputs with moe_forward (caller
workspace) at the layer tolerance, max |err| <= 1e-2 x RMS."""
import ctypes

import numpy as np
import pytest
import torch

import fine_grained_moe_gemm_b200 as moe
from moe_testlib import cfg_of, weights_for_forward
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


def _reference(cfg, weights, x, bias, y_dtype):
    ws = torch.empty(moe.workspace_size(cfg, x.shape[0]), dtype=torch.uint8, device=DEV)
    y = torch.empty((x.shape[0], cfg.d), dtype=y_dtype, device=DEV)
    moe.moe_forward(cfg, weights, x, bias, y, workspace=ws)
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
