"""The C ABI library on the host (no GPU needed): it loads, exports every
entry point include/moe.h declares, and rejects invalid arguments before it
touches a device."""
import ctypes

import pytest

import fine_grained_moe_gemm_b200 as moe
from fine_grained_moe_gemm_b200 import build as moe_build
from moe_testlib import cfg_of
from workloads import WORKLOADS


@pytest.fixture(scope="module")
def L():
    moe_build.build()
    return moe.lib()


def test_exports_every_declared_symbol(L):
    names = moe.declared_symbols()
    assert set(names) >= {"moe_route", "moe_permute", "moe_forward", "moe_workspace_size", "moe_device_error",
                          "moe_status_string", "moe_abi_version"}
    for n in names:
        assert hasattr(L, n), n
    assert L.moe_abi_version() == 1


def test_status_strings(L):
    assert moe.status_string(moe.MOE_OK) == "MOE_OK"
    assert moe.status_string(moe.MOE_ERR_WORKSPACE) == "MOE_ERR_WORKSPACE"
    assert moe.status_string(99) == "MOE_ERR_UNKNOWN"


def test_workspace_size(L):
    cfg = cfg_of(WORKLOADS["decode"])
    assert moe.workspace_size(cfg, 0) > 0
    s128, s4096 = moe.workspace_size(cfg, 128), moe.workspace_size(cfg, 4096)
    assert s4096 > s128
    # dominated by the permuted activations (9T x d bf16), h (9T x H bf16) and the fp32 combine buffer
    T = 4096
    core = 9 * T * 7168 * 2 + 9 * T * 2048 * 2 + T * 7168 * 4
    assert core <= s4096 <= core * 1.05
    bad = cfg_of(WORKLOADS["decode"])
    bad.n_groups = 7
    assert moe.workspace_size(bad, 128) == 0


@pytest.mark.parametrize("field,value,status", [
    ("d", 100, moe.MOE_ERR_INVALID_ARG),           # not a multiple of 128
    ("n_groups", 7, moe.MOE_ERR_INVALID_ARG),      # 256 % 7 != 0
    ("topk_groups", 9, moe.MOE_ERR_INVALID_ARG),
    ("top_k", 0, moe.MOE_ERR_INVALID_ARG),
    ("hidden", 1000, moe.MOE_ERR_INVALID_ARG),
    ("n_shared", 2, moe.MOE_ERR_INVALID_ARG),
    ("act_dtype", moe.MOE_E4M3, moe.MOE_ERR_UNSUPPORTED),
])
def test_invalid_config_rejected_before_device(L, field, value, status):
    cfg = cfg_of(WORKLOADS["decode"])
    setattr(cfg, field, value)
    P = ctypes.c_void_p
    st = L.moe_route(ctypes.byref(cfg), None, None, P(16), P(16), 4, P(16), P(16), None)
    assert st == status
    st = L.moe_permute(ctypes.byref(cfg), P(16), 4, P(16), P(16), P(16), P(16), None)
    assert st == status
    w = moe.MoeWeights()
    st = L.moe_forward(ctypes.byref(cfg), ctypes.byref(w), P(16), P(16), 4, P(16), moe.MOE_BF16, 0, P(1024),
                       1 << 30, None)
    assert st == status


def test_null_and_negative_arguments(L):
    cfg = cfg_of(WORKLOADS["decode"])
    P = ctypes.c_void_p
    assert L.moe_route(ctypes.byref(cfg), None, None, None, P(16), 4, P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route(ctypes.byref(cfg), None, None, P(16), P(16), -1, P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_permute(ctypes.byref(cfg), None, 4, P(16), P(16), P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    # T = 0 is a valid no-op even without a device
    assert L.moe_permute(ctypes.byref(cfg), None, 0, None, None, None, None, None) == moe.MOE_OK
    w = moe.MoeWeights(w_router=16, w_gate=16, w_up=16, w_down=16, ws_gate=16, ws_up=16, ws_down=16)
    # misaligned x
    assert L.moe_forward(ctypes.byref(cfg), ctypes.byref(w), P(18), P(16), 4, P(16), moe.MOE_BF16, 0, P(1024),
                         1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small
    assert L.moe_forward(ctypes.byref(cfg), ctypes.byref(w), P(16), P(16), 4, P(16), moe.MOE_BF16, 0, P(1024),
                         1024, None) == moe.MOE_ERR_WORKSPACE
    # bad output dtype / accumulate flag
    assert L.moe_forward(ctypes.byref(cfg), ctypes.byref(w), P(16), P(16), 4, P(16), moe.MOE_E4M3, 0, P(1024),
                         1 << 30, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_forward(ctypes.byref(cfg), ctypes.byref(w), P(16), P(16), 4, P(16), moe.MOE_BF16, 2, P(1024),
                         1 << 30, None) == moe.MOE_ERR_INVALID_ARG


def test_no_device_means_unsupported_not_fallback(L):
    """Valid arguments on a machine without an sm_100 device: the library refuses
    (there is no CPU fallback).  On a B200 this test is skipped."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    cfg = cfg_of(WORKLOADS["decode"])
    P = ctypes.c_void_p
    st = L.moe_permute(ctypes.byref(cfg), P(16), 4, P(16), P(16), P(16), P(16), None)
    assert st == moe.MOE_ERR_UNSUPPORTED
    # the static-scratch forward refuses the same way, before it looks up its array
    f = L.moe_forward_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(moe.MoeConfig), ctypes.POINTER(moe.MoeWeights), P, P, ctypes.c_int, P,
                  ctypes.c_int, ctypes.c_int, P]
    mw = moe.MoeWeights()
    st = f(ctypes.byref(cfg), ctypes.byref(mw), P(16), P(16), 4, P(16), moe.MOE_BF16, 0, None)
    assert st == moe.MOE_ERR_UNSUPPORTED


def test_prenorm_and_block_arguments(L):
    cfg = cfg_of(WORKLOADS["decode"])
    P = ctypes.c_void_p
    F = ctypes.c_float
    # moe_rmsnorm: negative T, d not a multiple of 8, q without sx, fp8 outputs with d % 128, misaligned h
    assert L.moe_rmsnorm(P(16), P(16), F(1e-6), -1, 7168, P(16), None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(P(16), P(16), F(1e-6), 4, 7164, P(16), None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(P(16), P(16), F(1e-6), 4, 7168, P(16), P(16), None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(P(16), P(16), F(1e-6), 4, 200, P(16), P(16), P(16), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(P(18), P(16), F(1e-6), 4, 7168, P(16), None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(P(16), P(16), F(-1.0), 4, 7168, P(16), None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_rmsnorm(None, None, F(1e-6), 0, 7168, None, None, None, None) == moe.MOE_OK
    # the block workspace holds the forward's plus the normalised activations
    for T in (1, 128, 4096):
        assert L.moe_block_workspace_size(ctypes.byref(cfg), T) >= moe.workspace_size(cfg, T) + T * 7168 * 2
    w = moe.MoeWeights(w_router=16, w_gate=16, w_up=16, w_down=16, ws_gate=16, ws_up=16, ws_down=16)
    blk = lambda c, g, ws: L.moe_forward_block(ctypes.byref(c), ctypes.byref(w), g, F(1e-6), P(16), P(16), 4, P(16),
                                              P(1024), ws, None, None, None)
    assert blk(cfg, P(16), 1024) == moe.MOE_ERR_WORKSPACE
    assert blk(cfg, None, 1 << 30) == moe.MOE_ERR_INVALID_ARG          # no gain
    assert blk(cfg, P(20), 1 << 30) == moe.MOE_ERR_INVALID_ARG         # misaligned gain
    f32 = cfg_of(WORKLOADS["tiny"])                                     # fp32 activations: not a bf16 stream
    assert blk(f32, P(16), 1 << 30) == moe.MOE_ERR_UNSUPPORTED


def test_dense_arguments(L):
    P = ctypes.c_void_p
    B, F, E8 = moe.MOE_BF16, moe.MOE_F32, moe.MOE_E4M3
    assert moe.dense_workspace_size(7168, 18432, B, B, 128) > 128 * 18432 * 2
    assert moe.dense_workspace_size(7168, 100, B, B, 128) == 0          # hidden not a multiple of 128
    assert moe.dense_workspace_size(7168, 18432, F, E8, 128) == 0       # FP8 needs bf16 activations
    call = lambda d, h, act, wdt, ws: L.moe_dense_ffn(d, h, act, wdt, P(16), P(16), P(16), P(16), P(16), P(16),
                                                      P(16), 4, P(16), B, 0, P(1024), ws, None, None)
    assert call(7168, 100, B, B, 1 << 30) == moe.MOE_ERR_INVALID_ARG
    assert call(7168, 18432, F, E8, 1 << 30) == moe.MOE_ERR_UNSUPPORTED
    assert call(7168, 18432, B, B, 1024) == moe.MOE_ERR_WORKSPACE
    assert L.moe_dense_ffn(7168, 18432, B, E8, P(16), P(16), P(16), None, None, None, P(16), 4, P(16), B, 0,
                           P(1024), 1 << 30, None, None) == moe.MOE_ERR_INVALID_ARG   # FP8 without scales
    assert L.moe_dense_ffn(7168, 18432, B, B, None, None, None, None, None, None, None, 0, None, B, 0, None, 0,
                           None, None) == moe.MOE_OK                          # T = 0


def test_selftest_arguments(L):
    assert L.moe_selftest_wait_timeout(0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_wait_timeout(2_000_000_000, None) == moe.MOE_ERR_INVALID_ARG


def test_host_entry_arguments(L):
    """moe_forward_host: every argument is checked before anything is enqueued, so the
    errors below come back without a device."""
    cfg = cfg_of(WORKLOADS["decode"])
    P = ctypes.c_void_p
    for T in (1, 128, 4096):
        for yd, yb in ((moe.MOE_BF16, 2), (moe.MOE_F32, 4)):
            need = L.moe_host_workspace_size(ctypes.byref(cfg), T, yd)
            base = (moe.workspace_size(cfg, T) + 255) // 256 * 256
            assert need == base + (T * 7168 * 2 + 255) // 256 * 256 + (T * 7168 * yb + 255) // 256 * 256
    assert L.moe_host_workspace_size(ctypes.byref(cfg), 4, moe.MOE_E4M3) == 0
    w = moe.MoeWeights(w_router=16, w_gate=16, w_up=16, w_down=16, ws_gate=16, ws_up=16, ws_down=16)
    host = lambda T, x, y, yd, acc, ws: L.moe_forward_host(ctypes.byref(cfg), ctypes.byref(w), x, P(16), T, y, yd,
                                                           acc, P(1 << 20), ws, None)
    assert host(4, P(16), P(16), moe.MOE_BF16, 0, 1024) == moe.MOE_ERR_WORKSPACE
    assert host(4, None, P(16), moe.MOE_BF16, 0, 1 << 30) == moe.MOE_ERR_INVALID_ARG     # no x
    assert host(4, P(16), None, moe.MOE_BF16, 0, 1 << 30) == moe.MOE_ERR_INVALID_ARG     # no y
    assert host(4, P(16), P(16), moe.MOE_E4M3, 0, 1 << 30) == moe.MOE_ERR_INVALID_ARG    # output dtype
    assert host(4, P(16), P(16), moe.MOE_BF16, 2, 1 << 30) == moe.MOE_ERR_INVALID_ARG    # accumulate flag
    assert host(-1, P(16), P(16), moe.MOE_BF16, 0, 1 << 30) == moe.MOE_ERR_INVALID_ARG
    assert host(0, None, None, moe.MOE_BF16, 0, 0) == moe.MOE_OK                         # T = 0: a no-op
    # host buffers need no alignment (they are copy sources and targets only)
    nodev = L.moe_forward_host(ctypes.byref(cfg), ctypes.byref(moe.MoeWeights()), P(17), P(16), 4, P(19),
                               moe.MOE_BF16, 0, P(1 << 20), 1 << 30, None)
    assert nodev == moe.MOE_ERR_INVALID_ARG                                              # no weights


def test_binding_argument_counts_match_the_header(L):
    """Every entry point the binding declares argument types for takes as many parameters as its
    declaration in include/moe.h (a drift between the two would pass wrong values silently)."""
    import re
    text = open(moe.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    decls = dict(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(([^)]*)\)\s*;", text))
    assert set(decls) == set(moe.declared_symbols())
    checked = 0
    for name, params in decls.items():
        argtypes = getattr(L, name).argtypes
        if argtypes is None:
            continue
        n = 0 if params.strip() in ("", "void") else params.count(",") + 1
        assert len(argtypes) == n, f"{name}: header {n} parameters, binding {len(argtypes)}"
        checked += 1
    assert checked >= 20
