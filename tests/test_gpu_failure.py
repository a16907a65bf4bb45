"""The failure path of the in-kernel waits, on the GPU: a bounded wait that nothing
completes gives up after its limit, sets MOE_DEVERR_TIMEOUT, and the context stays
usable (the next layer call is correct).  No fault, trap or hang is involved: the
kernel only waits on an mbarrier of its own for a few milliseconds."""
import numpy as np
import pytest
import torch

import oracle
import fine_grained_moe_gemm_b200 as moe
from moe_testlib import assert_close_rms, cfg_of, oracle_layer, weights_for_forward, x_host
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_bounded_wait_times_out_and_the_context_survives():
    assert moe.device_error() == 0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    moe.selftest_wait_timeout(3_000_000)                 # 3 ms
    b.record()
    torch.cuda.synchronize()
    assert a.elapsed_time(b) >= 2.9                       # it waited its limit out ...
    assert moe.device_error() == moe.MOE_DEVERR_TIMEOUT   # ... and said so
    assert moe.device_error() == 0                        # the word is cleared by the read
    # the layer still runs correctly in the same context
    wl = WORKLOADS["tiny"]
    W = {k: v.to(DEV) for k, v in make_inputs(wl, "cpu").items()}
    cfg = cfg_of(wl)
    ws = torch.empty(moe.workspace_size(cfg, wl.T), dtype=torch.uint8, device=DEV)
    y = torch.empty((wl.T, wl.d), dtype=torch.float32, device=DEV)
    r = {"topk_idx": torch.empty((wl.T, wl.top_k), dtype=torch.int32, device=DEV),
         "topk_w": torch.empty((wl.T, wl.top_k), dtype=torch.float32, device=DEV)}
    moe.moe_forward(cfg, weights_for_forward(W), W["x"], W["bias"], y, workspace=ws, routing_out=r)
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    idx, w = r["topk_idx"].cpu().numpy(), r["topk_w"].cpu().numpy()
    L = oracle_layer(wl, W, np.unique(idx))
    ref = oracle.expert_tokens(L, x_host(W["x"]), idx, w, np.arange(wl.T, dtype=np.int32))
    assert_close_rms(y.cpu().numpy(), ref, 1e-2)


def test_selftest_limits():
    for bad in (0, 2_000_000_000):
        with pytest.raises(moe.MoeError):
            moe.selftest_wait_timeout(bad)
