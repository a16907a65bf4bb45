"""moe_forward_plan describes what moe_forward launches: the launch counter
advances by exactly the planned number of kernels, and the token tile and
CTA-pair choice follow the rows per expert."""
import pytest
import torch

import fine_grained_moe_gemm_b200 as moe
from moe_testlib import cfg_of, weights_for_forward
from workloads import WORKLOADS, make_inputs, make_x

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def tiny():
    wl = WORKLOADS["tiny"]
    return wl, {k: v.to(DEV) for k, v in make_inputs(wl, "cpu").items()}


@pytest.mark.parametrize("T", [1, 16, 300, 1025, 3000])
@pytest.mark.parametrize("y_dtype", [torch.bfloat16, torch.float32])
def test_launch_count_matches_plan(tiny, T, y_dtype):
    wl, W = tiny
    cfg = cfg_of(wl)
    plan = moe.forward_plan(cfg, T, y_dtype)
    x = make_x(wl, "cpu", T=T).to(DEV)
    ws = torch.empty(moe.workspace_size(cfg, T), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, wl.d), dtype=y_dtype, device=DEV)
    n0 = moe.launch_count()
    moe.moe_forward(cfg, weights_for_forward(W), x, W["bias"], y, workspace=ws)
    n1 = moe.launch_count()
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    assert n1 - n0 == plan["launches"]
    assert plan["permute_ctas"] == 1 if T <= 1024 else plan["permute_ctas"] > 1
    assert plan["router_splits"] >= 1


def test_plan_tiles_follow_rows_per_expert():
    wl = WORKLOADS["decode"]
    cfg = cfg_of(wl)
    assert moe.forward_plan(cfg, 0) == {k: 0 for k in moe.forward_plan(cfg, 0)}
    tiles = [moe.forward_plan(cfg, T)["token_tile"] for T in (1, 128, 512, 1024, 4096)]
    assert tiles == sorted(tiles) and tiles[0] == 32 and tiles[-1] == 256
    assert moe.forward_plan(cfg, 4096)["cta_pair"] == 1 and moe.forward_plan(cfg, 128)["cta_pair"] == 0
    p8 = moe.forward_plan(cfg_of(WORKLOADS["fp8"]), 8192)
    assert p8["fp8"] == 1 and p8["cta_pair"] == 1 and p8["token_tile"] == 128
