"""GPU parity of the dense SwiGLU FFN (moe_dense_ffn) against the oracle: the
expert GEMM kernels on one group of all T rows.  Tolerance as the layer's:
max |err| <= 1e-2 x RMS(y_ref) (e4m3 weights: 5e-2), a bf16 output adding one
bf16 ulp of |y_ref|."""
import numpy as np
import pytest
import torch

import oracle
import fine_grained_moe_gemm_b200 as moe
from moe_testlib import assert_close_bf16, assert_close_rms, u16, u8
from workloads import DENSE_HIDDEN, make_dense_weights

pytestmark = pytest.mark.gpu
DEV = "cuda"

_cache = {}


def weights(d, hidden, fp8):
    key = (d, hidden, fp8)
    if key not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        gen_dev = "cpu" if d * hidden < 4 * 2**20 else DEV
        _cache[key] = {k: v.to(DEV) for k, v in make_dense_weights(d, hidden, fp8, gen_dev).items()}
    return _cache[key]


def make_x(T, d, seed, f32=False):
    g = torch.Generator(device="cpu").manual_seed(1000 + 7 * T + seed)
    x = torch.randn((T, d), generator=g, dtype=torch.float32)
    return (x if f32 else x.to(torch.bfloat16)).to(DEV)


def run(W, x, y_dtype, accumulate=False, y0=None):
    hidden, d = W["w_gate"].shape
    fp8 = W["w_gate"].dtype == torch.uint8
    T = x.shape[0]
    act = moe.MOE_F32 if x.dtype == torch.float32 else moe.MOE_BF16
    ws = torch.empty(moe.dense_workspace_size(d, hidden, act, moe.MOE_E4M3 if fp8 else moe.MOE_BF16, T),
                     dtype=torch.uint8, device=DEV)
    y = y0.clone() if y0 is not None else torch.empty((T, d), dtype=y_dtype, device=DEV)
    n0 = moe.launch_count()
    moe.moe_dense_ffn(W["w_gate"], W["w_up"], W["w_down"], x, y, W.get("s_gate"), W.get("s_up"), W.get("s_down"),
                      accumulate=accumulate, workspace=ws)
    n = moe.launch_count() - n0
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    # the tables, a copy of x into row order only for fp32 x (the bf16 cast) or e4m3 weights (the
    # quantisation), the two GEMMs, the bf16 cast of y
    copy = 1 if (fp8 or x.dtype == torch.float32) else 0
    assert n == 1 + copy + 2 + (1 if y.dtype == torch.bfloat16 else 0)
    return y


def reference(W, x, tokens):
    fp8 = W["w_gate"].dtype == torch.uint8
    conv = u8 if fp8 else u16
    xs = x.cpu().numpy() if x.dtype == torch.float32 else u16(x)
    kw = {}
    if fp8:
        kw = dict(s_gate=W["s_gate"].cpu().numpy(), s_up=W["s_up"].cpu().numpy(), s_down=W["s_down"].cpu().numpy())
    return oracle.dense_ffn(xs, conv(W["w_gate"]), conv(W["w_up"]), conv(W["w_down"]), tokens=tokens,
                            x_is_f32=x.dtype == torch.float32, **kw)


@pytest.mark.parametrize("d,hidden,T", [(256, 512, 64), (256, 512, 1), (256, 512, 300), (512, 256, 300), (512, 2048, 100),
                                        (256, 384, 1000)])
def test_dense_small_full(d, hidden, T):
    W = weights(d, hidden, False)
    x = make_x(T, d, 0)
    ref = reference(W, x, np.arange(T, dtype=np.int32))
    assert_close_rms(run(W, x, torch.float32).cpu().numpy(), ref, 1e-2)
    assert_close_bf16(run(W, x, torch.bfloat16), ref, 1e-2)


def test_dense_fp32_input_and_accumulate():
    W = weights(256, 512, False)
    x = make_x(64, 256, 1, f32=True)
    ref = reference(W, x, np.arange(64, dtype=np.int32))
    r = make_x(64, 256, 2, f32=True)
    y = run(W, x, torch.float32, accumulate=True, y0=r)
    assert_close_rms(y.cpu().numpy() - r.cpu().numpy(), ref, 1e-2)


@pytest.mark.parametrize("T", [40, 300])
def test_dense_fp8_small(T):
    W = weights(256, 512, True)
    x = make_x(T, 256, 3)
    ref = reference(W, x, np.arange(T, dtype=np.int32))
    assert_close_bf16(run(W, x, torch.bfloat16), ref, 5e-2)


@pytest.mark.parametrize("T,fp8", [(128, False), (4096, False), (300, True)])
def test_dense_deepseek_sampled(T, fp8):
    W = weights(7168, DENSE_HIDDEN, fp8)
    x = make_x(T, 7168, 4)
    toks = np.array(sorted({0, T // 2, T - 1}), dtype=np.int32)
    ref = reference(W, x, toks)
    yb = run(W, x, torch.bfloat16)
    assert_close_bf16(yb[torch.from_numpy(toks).long().to(DEV)], ref, 5e-2 if fp8 else 1e-2)
