"""Shared helpers of the GPU parity tests: configs, oracle inputs from the
generated tensors, tolerance checks.  No arithmetic of the layer lives here."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import fine_grained_moe_gemm_b200 as moe
from workloads import Workload


def cfg_of(wl: Workload) -> moe.MoeConfig:
    return moe.MoeConfig(wl.d, wl.n_experts, wl.n_groups, wl.topk_groups, wl.top_k, wl.hidden, 1,
                         wl.shared_hidden, wl.routed_scale, moe.MOE_F32 if wl.x_f32 else moe.MOE_BF16,
                         moe.MOE_E4M3 if wl.fp8 else moe.MOE_BF16)


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> host uint16 bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def x_host(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().numpy() if x.dtype == torch.float32 else u16(x)


def oracle_layer(wl: Workload, W: dict, experts) -> oracle.Layer:
    """Oracle view of the layer holding only the listed routed experts."""
    E = wl.n_experts
    conv = u8 if wl.fp8 else u16
    wg, wu, wd = [None] * E, [None] * E, [None] * E
    sg = su = sd = None
    if wl.fp8:
        sg, su, sd = [None] * E, [None] * E, [None] * E
    for e in sorted(set(int(v) for v in experts)):
        wg[e], wu[e], wd[e] = conv(W["w_gate"][e]), conv(W["w_up"][e]), conv(W["w_down"][e])
        if wl.fp8:
            sg[e] = W["s_gate"][e].cpu().numpy()
            su[e] = W["s_up"][e].cpu().numpy()
            sd[e] = W["s_down"][e].cpu().numpy()
    kw = {}
    if wl.fp8:
        kw = dict(s_gate=sg, s_up=su, s_down=sd, ss_gate=W["ss_gate"].cpu().numpy(),
                  ss_up=W["ss_up"].cpu().numpy(), ss_down=W["ss_down"].cpu().numpy())
    return oracle.Layer(wl.d, E, wl.hidden, wl.shared_hidden, wl.top_k, wl.routed_scale, wg, wu, wd,
                        conv(W["ws_gate"]), conv(W["ws_up"]), conv(W["ws_down"]), x_is_f32=wl.x_f32, **kw)


def weights_for_forward(W: dict) -> dict:
    return {k: v for k, v in W.items() if k not in ("x", "bias")}


def assert_close_rms(y_gpu: np.ndarray, y_ref: np.ndarray, rel: float, what: str = "y"):
    """max |err| <= rel * RMS(y_ref)."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    rms = float(np.sqrt(np.mean(np.square(y_ref))))
    err = float(np.max(np.abs(y_gpu - y_ref)))
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite output"
    assert err <= rel * rms, f"{what}: max|err| {err:.4g} > {rel} * RMS {rms:.4g} (ratio {err / rms:.4g})"
    return err / rms


def assert_close_bf16(y_gpu_bf16: torch.Tensor, y_ref: np.ndarray, rel: float, what: str = "y"):
    """bf16 output: |err| <= rel * RMS(y_ref) + one bf16 ulp of |y_ref| (storage rounding)."""
    y = y_gpu_bf16.float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(np.square(y_ref))))
    a = np.abs(y_ref)
    ulp = np.where(a > 0, 2.0 ** (np.floor(np.log2(np.maximum(a, 1e-300))) - 7), 0.0)
    bound = rel * rms + ulp
    err = np.abs(y - y_ref)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements over bound; worst excess {float((err - bound).max()):.4g}"
