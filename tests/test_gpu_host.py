"""moe_forward_host (host x in, host y out, the copies inside the call) against the oracle,
and two calls on two streams with two workspaces overlapping on the GPU.

Tolerance as for moe_forward: max |err| <= 1e-2 x RMS(y_ref) (bf16 output: plus one
bf16 ulp of |y_ref|).  The host entry runs the same kernels on device copies of x
and y, so its result is also compared with moe_forward's on the same inputs; the
combine's fp32 atomics may add a token's expert outputs in another order, hence a
few-ulp bound rather than equality.
"""
import numpy as np
import pytest
import torch

import fine_grained_moe_gemm_b200 as moe
from moe_testlib import assert_close_bf16, assert_close_rms, cfg_of, weights_for_forward
from test_gpu_forward import inputs, oracle_y, run_forward
from workloads import WORKLOADS, make_residual, make_x

pytestmark = pytest.mark.gpu

DEV = "cuda"
REL = 1e-2


def host_forward(wl, W, x_host, y_host, accumulate=False, stream=None, ws=None):
    cfg = cfg_of(wl)
    T = x_host.shape[0]
    if ws is None:
        ws = torch.empty(moe.host_workspace_size(cfg, T, y_host.dtype), dtype=torch.uint8, device=DEV)
    moe.moe_forward_host(cfg, weights_for_forward(W), x_host, W["bias"], y_host, accumulate=accumulate,
                         workspace=ws, stream=stream)
    return ws


def close_to(a, b):
    """a and b (fp32) agree up to the order of a token's nine fp32 additions: a few ulps of
    the summands, whose size is that of the output's RMS (the sum may cancel below it)."""
    a64, b64 = a.double(), b.double()
    eps = torch.finfo(torch.float32).eps
    rms = float(b64.pow(2).mean().sqrt())
    tol = 64 * eps * rms + 4 * eps * b64.abs()
    assert bool(((a64 - b64).abs() <= tol).all())


@pytest.mark.parametrize("T", [64, 1, 129])
def test_tiny_host(T):
    wl = WORKLOADS["tiny"]
    W = inputs("tiny", "cpu")
    xh = make_x(wl, "cpu", T=T).pin_memory()
    ref = oracle_y(wl, W, xh.to(DEV), np.arange(T))
    for dt in (torch.float32, torch.bfloat16):
        yh = torch.empty((T, wl.d), dtype=dt).pin_memory()
        host_forward(wl, W, xh, yh)
        torch.cuda.synchronize()
        assert moe.device_error() == 0
        if dt == torch.float32:
            assert_close_rms(yh.numpy(), ref, REL)
        else:
            assert_close_bf16(yh.to(DEV), ref, REL)


def test_tiny_host_accumulate_and_pageable():
    """accumulate = 1 reads y_host as the residual; pageable host memory works too."""
    wl = WORKLOADS["tiny"]
    W = inputs("tiny", "cpu")
    xh = make_x(wl, "cpu")
    ref = oracle_y(wl, W, xh.to(DEV), np.arange(wl.T))
    r32 = make_residual(wl, "cpu", dtype=torch.float32)
    yh = r32.clone()                        # pageable
    host_forward(wl, W, xh, yh, accumulate=True)
    torch.cuda.synchronize()
    assert_close_rms(yh.numpy(), ref + r32.numpy().astype(np.float64), REL)


def test_decode_host_matches_device_entry():
    wl = WORKLOADS["decode"]
    W = inputs("decode", "cuda")
    x = W["x"]
    yd = run_forward(wl, W, x, torch.float32)
    xh = x.cpu().pin_memory()
    yh = torch.empty((wl.T, wl.d), dtype=torch.float32).pin_memory()
    host_forward(wl, W, xh, yh)
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    close_to(yh, yd.cpu())


def test_two_streams_overlap():
    """Calls alternating between two streams and two workspaces (the pipelined serving
    loop): each result equals the single-stream one on the same input."""
    wl = WORKLOADS["decode"]
    W = inputs("decode", "cuda")
    cfg = cfg_of(wl)
    T = wl.T
    xs = [make_x(wl, "cuda", T=T, seed=100 + i).cpu().pin_memory() for i in range(4)]
    solo = []
    for xh in xs:
        yh = torch.empty((T, wl.d), dtype=torch.float32).pin_memory()
        host_forward(wl, W, xh, yh)
        torch.cuda.synchronize()
        solo.append(yh.clone())
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    wss = [torch.empty(moe.host_workspace_size(cfg, T, torch.float32), dtype=torch.uint8, device=DEV)
           for _ in range(2)]
    outs = [torch.empty((T, wl.d), dtype=torch.float32).pin_memory() for _ in xs]
    for i, xh in enumerate(xs):
        host_forward(wl, W, xh, outs[i], stream=streams[i % 2], ws=wss[i % 2])
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    for a, b in zip(outs, solo):
        close_to(a, b)
