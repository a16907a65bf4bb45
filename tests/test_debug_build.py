"""The checking build (libmoe_b200_debug.so, the sources compiled with MOE_DEBUG).

Its kernels check every access that depends on a device-built table before making
it: the token of each permuted row (x rows in the gather, y rows in the combine),
the permuted row count, and each grouped-GEMM work item's row range and weight
tile.  A failed check sets MOE_DEVERR_BOUNDS and the access is skipped or replaced
by an in-bounds one; nothing traps.

CPU tests: both libraries load, export every declared entry point, and report
which build they are; the corruption hook is refused by the regular build.
GPU tests: with no corruption the checking build computes the same layer as the
regular one and flags nothing; then a table is corrupted on the device after the
permutation (moe_debug_corrupt_next: a token id past the batch, a row count past
the permuted buffers, a negative group start), the call completes, the bit is set,
and the next clean call on the same context is correct again.  Each kernel family
that reads the tables is reached: the single-CTA bf16 GEMMs (tiny, decode), the
CTA-pair bf16 GEMMs (T=4096), the single-CTA and CTA-pair e4m3 GEMMs.
"""
import ctypes

import numpy as np
import pytest
import torch

import fine_grained_moe_gemm_b200 as moe
from moe_testlib import cfg_of, weights_for_forward
from workloads import WORKLOADS, make_inputs, make_x

DEV = "cuda"


@pytest.fixture(scope="module")
def D():
    return moe.debug_lib()


def test_both_builds_export_every_entry_point_and_say_which_they_are(D):
    L = moe.lib()
    for n in moe.declared_symbols():
        assert hasattr(L, n), n
        assert hasattr(D, n), n
    assert L.moe_debug_build() == 0 and D.moe_debug_build() == 1
    assert L.moe_abi_version() == D.moe_abi_version()


def test_corruption_hook_host_side(D):
    L = moe.lib()
    assert L.moe_debug_corrupt_next(moe.MOE_DEBUG_TABLE_ROW_TOK, 0, 0) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_debug_corrupt_next(7, 0, 0) == moe.MOE_ERR_INVALID_ARG
    assert D.moe_debug_corrupt_next(7, 0, 0) == moe.MOE_ERR_INVALID_ARG
    assert D.moe_debug_corrupt_next(moe.MOE_DEBUG_TABLE_ROW_OFF, 3, -5) == moe.MOE_OK
    assert D.moe_debug_corrupt_next(-1, 0, 0) == moe.MOE_OK          # disarmed again


# ----------------------------------------------------------------------------- GPU

def _forward(L, cfg, W, x, y_dtype=torch.float32):
    T = x.shape[0]
    ws = torch.empty(L.moe_workspace_size(ctypes.byref(cfg), T), dtype=torch.uint8, device=DEV)
    y = torch.full((T, cfg.d), float("nan"), dtype=y_dtype, device=DEV)
    mw = moe.make_weights(weights_for_forward(W))
    P = ctypes.c_void_p
    st = L.moe_forward(ctypes.byref(cfg), ctypes.byref(mw), P(x.data_ptr()), P(W["bias"].data_ptr()), T,
                       P(y.data_ptr()), moe.MOE_F32 if y_dtype == torch.float32 else moe.MOE_BF16, 0,
                       P(ws.data_ptr()), ws.numel(), P(torch.cuda.current_stream().cuda_stream))
    assert st == moe.MOE_OK
    return y


def _flags(L):
    f = ctypes.c_uint(0)
    L.moe_device_error(ctypes.byref(f), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return int(f.value)


def _close(a, b, rel=1e-3):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(b ** 2)))
    assert np.all(np.isfinite(a)) and float(np.max(np.abs(a - b))) <= rel * rms


_CASES = [("tiny", 64), ("tiny", 700), ("decode", 128), ("prefill", 4096), ("fp8", 37), ("fp8", 4096)]


@pytest.mark.gpu
@pytest.mark.parametrize("name,T", _CASES)
def test_checking_build_flags_corrupted_tables(D, name, T):
    wl = WORKLOADS[name].with_T(T)
    cfg = cfg_of(wl)
    gen = "cpu" if wl.d <= 1024 else DEV
    W = {k: v.to(DEV) for k, v in make_inputs(wl, gen).items()}
    x = make_x(wl, gen, seed=11, T=T).to(DEV)
    E, k = wl.n_experts, wl.top_k
    rows = T * k + T
    plan = moe.forward_plan(cfg, T)

    assert _flags(D) == 0
    ref = _forward(moe.lib(), cfg, W, x)
    y = _forward(D, cfg, W, x)
    torch.cuda.synchronize()
    assert _flags(D) == 0, "a clean call flagged a bound"
    _close(y, ref)                                 # same kernels, same arithmetic; combine order may differ

    corruptions = [
        (moe.MOE_DEBUG_TABLE_ROW_TOK, rows // 3, T + 1000),     # a permuted row's token past the batch
        (moe.MOE_DEBUG_TABLE_ROW_TOK, rows - 1, -7),            # the shared expert's last row: negative token
        (moe.MOE_DEBUG_TABLE_ROW_OFF, E + 1, rows + 4096),      # more rows than the permuted buffers hold
        (moe.MOE_DEBUG_TABLE_ROW_OFF, 1, -5),                   # a negative group start
    ]
    for table, index, value in corruptions:
        assert D.moe_debug_corrupt_next(table, index, value) == moe.MOE_OK
        _forward(D, cfg, W, x)
        torch.cuda.synchronize()
        got = _flags(D)
        assert got & moe.MOE_DEVERR_BOUNDS, (table, index, value, got, plan)
        # the context is still usable and the next call is clean and correct
        y = _forward(D, cfg, W, x)
        torch.cuda.synchronize()
        assert _flags(D) == 0
        _close(y, ref)
