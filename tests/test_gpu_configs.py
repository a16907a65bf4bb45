"""Layer configurations beyond the five workloads, checked in full against the oracle:
no shared expert (bf16 x, fp32 x, e4m3 weights), other expert / group / top-k counts, a shared expert wider than the
routed ones, no group limiting (one group), and every token routed to the same eight
experts (the largest per-expert row count, T rows each, on the CTA-pair kernels)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import fine_grained_moe_gemm_b200 as moe
from moe_testlib import assert_close_bf16, assert_close_rms, oracle_layer, u16, u8, weights_for_forward, x_host
from workloads import WORKLOADS, make_inputs, make_x

pytestmark = pytest.mark.gpu
DEV = "cuda"
TINY = WORKLOADS["tiny"]

CASES = {
    # name: (workload fields, n_shared)
    "no_shared": (dict(x_f32=False), 0),
    "e64_g8_k6": (dict(d=512, n_experts=64, n_groups=8, topk_groups=3, top_k=6, hidden=256, shared_hidden=384,
                       x_f32=False), 1),
    "one_group_k1": (dict(n_experts=32, n_groups=1, topk_groups=1, top_k=1, x_f32=False), 1),
    "fp8_e32": (dict(d=512, n_experts=32, n_groups=4, topk_groups=2, top_k=4, hidden=256, shared_hidden=256,
                     x_f32=False, fp8=True), 1),
    # no shared row in the copy into expert order: fp32 x (converted in the copy) and e4m3 weights
    # (quantised in the copy)
    "no_shared_f32": (dict(x_f32=True), 0),
    "fp8_e32_no_shared": (dict(d=512, n_experts=32, n_groups=4, topk_groups=2, top_k=4, hidden=256,
                               shared_hidden=256, x_f32=False, fp8=True), 0),
}


def cfg_for(wl, n_shared):
    return moe.MoeConfig(wl.d, wl.n_experts, wl.n_groups, wl.topk_groups, wl.top_k, wl.hidden, n_shared,
                         wl.shared_hidden, wl.routed_scale, moe.MOE_F32 if wl.x_f32 else moe.MOE_BF16,
                         moe.MOE_E4M3 if wl.fp8 else moe.MOE_BF16)


def run_case(wl, n_shared, W, x, bias, y_dtype, rel):
    cfg = cfg_for(wl, n_shared)
    T = x.shape[0]
    ws = torch.empty(moe.workspace_size(cfg, T), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, wl.d), dtype=y_dtype, device=DEV)
    wts = weights_for_forward(W)
    if not n_shared:
        wts = {k: v for k, v in wts.items() if not k.startswith(("ws_", "ss_"))}
    E, k = wl.n_experts, wl.top_k
    r = {"logits": torch.empty((T, E), dtype=torch.float32, device=DEV),
         "topk_idx": torch.empty((T, k), dtype=torch.int32, device=DEV),
         "topk_w": torch.empty((T, k), dtype=torch.float32, device=DEV),
         "counts": torch.empty(E, dtype=torch.int32, device=DEV)}
    moe.moe_forward(cfg, wts, x, bias, y, workspace=ws, routing_out=r)
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    idx, w = oracle.select(r["logits"].cpu().numpy(), bias.cpu().numpy(), wl.n_groups, wl.topk_groups, k)
    assert np.array_equal(r["topk_idx"].cpu().numpy(), idx)
    assert np.array_equal(r["topk_w"].cpu().numpy().view(np.uint32), w.view(np.uint32))
    assert np.array_equal(r["counts"].cpu().numpy(), oracle.permute(idx, E)[0])
    Wo = dict(W)
    if not n_shared:  # the oracle always adds the shared expert: give it zero weights
        for name in ("ws_gate", "ws_up", "ws_down"):
            Wo[name] = torch.zeros_like(W[name])
    L = oracle_layer(wl, Wo, np.unique(idx))
    ref = oracle.expert_tokens(L, x_host(x), idx, w, np.arange(T, dtype=np.int32))
    if y_dtype == torch.float32:
        assert_close_rms(y.cpu().numpy(), ref, rel)
    else:
        assert_close_bf16(y, ref, rel)
    return r["counts"].cpu().numpy()


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("T", [1, 64, 700])
def test_config(name, T):
    fields, n_shared = CASES[name]
    wl = dataclasses.replace(TINY, name=name, **fields)
    W = {k: v.to(DEV) for k, v in make_inputs(wl, "cpu").items()}
    x = make_x(wl, "cpu", T=T).to(DEV)
    rel = 5e-2 if wl.fp8 else 1e-2
    run_case(wl, n_shared, W, x, W["bias"], torch.bfloat16, rel)
    if not wl.fp8:
        run_case(wl, n_shared, W, x, W["bias"], torch.float32, rel)


def test_every_token_to_the_same_eight_experts():
    """A bias of +10 on experts 0-7 (all in group 0) sends every token there: each
    of the eight holds all T rows, the largest grouped-GEMM problem the layer has."""
    wl = dataclasses.replace(TINY, name="same8", d=512, n_experts=64, n_groups=8, topk_groups=4, top_k=8,
                             hidden=256, shared_hidden=256, x_f32=False)
    W = {k: v.to(DEV) for k, v in make_inputs(wl, "cpu").items()}
    bias = torch.zeros(64, dtype=torch.float32, device=DEV)
    bias[:8] = 10.0
    T = 1500
    x = make_x(wl, "cpu", T=T).to(DEV)
    counts = run_case(wl, 1, W, x, bias, torch.float32, 1e-2)
    assert np.all(counts[:8] == T) and counts[8:].sum() == 0
