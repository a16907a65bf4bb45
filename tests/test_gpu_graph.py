"""The layer under CUDA-graph capture: moe_forward enqueues only kernels, memsets
and (optional) event records on the caller's stream, with no host synchronisation
and no allocation, so a captured forward replays with the same results."""
import numpy as np
import pytest
import torch

import fine_grained_moe_gemm_b200 as moe
from moe_testlib import cfg_of, weights_for_forward
from workloads import WORKLOADS, make_inputs, make_x

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,T", [("tiny", 64), ("decode", 128)])
def test_captured_forward_replays_the_eager_result(name, T):
    wl = WORKLOADS[name]
    W = {k: v.to(DEV) for k, v in make_inputs(wl, "cpu" if wl.d <= 1024 else DEV).items()}
    cfg = cfg_of(wl)
    x = make_x(wl, "cpu", T=T).to(DEV)
    ws = torch.empty(moe.workspace_size(cfg, T), dtype=torch.uint8, device=DEV)
    wts = weights_for_forward(W)
    r = {"topk_idx": torch.empty((T, wl.top_k), dtype=torch.int32, device=DEV)}
    y_eager = torch.empty((T, wl.d), dtype=torch.bfloat16, device=DEV)
    moe.moe_forward(cfg, wts, x, W["bias"], y_eager, workspace=ws, routing_out=r)
    torch.cuda.synchronize()
    idx_eager = r["topk_idx"].clone()

    y = torch.empty_like(y_eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        moe.moe_forward(cfg, wts, x, W["bias"], y, workspace=ws, routing_out=r, stream=s)
    r["topk_idx"].zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    assert torch.equal(r["topk_idx"], idx_eager)                  # routing: bit for bit
    a, b = y.float().cpu().numpy(), y_eager.float().cpu().numpy()
    # the combine's fp32 atomics may add in another order: one bf16 ulp at most
    ulp = np.where(np.abs(a) > 0, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(a), 1e-30))) - 7), 0)
    assert np.all(np.abs(a - b) <= ulp + 1e-6 * float(np.sqrt(np.mean(b * b))))
    # a new input in the captured buffer is picked up by the replay
    x.copy_(make_x(wl, "cpu", T=T, seed=1).to(DEV))
    g.replay()
    moe.moe_forward(cfg, wts, x, W["bias"], y_eager, workspace=ws)
    torch.cuda.synchronize()
    a, b = y.float().cpu().numpy(), y_eager.float().cpu().numpy()
    assert np.all(np.abs(a - b) <= np.where(np.abs(a) > 0, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(a), 1e-30))) - 7), 0)
                  + 1e-6 * float(np.sqrt(np.mean(b * b))))
