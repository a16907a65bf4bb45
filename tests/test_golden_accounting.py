"""The workload definitions and the byte/flop accounting against the figures the pages print."""
import json
import os

from workloads import WORKLOADS

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "deepseek_v3_moe_dims.json")))


def test_decode_workload_matches_printed_dimensions():
    wl = WORKLOADS["decode"]
    assert wl.d == G["d_model"]["value"]
    assert wl.n_experts == G["routed_experts"]["value"]
    assert wl.top_k == G["experts_per_token"]["value"]
    assert wl.hidden == wl.shared_hidden == G["expert_hidden"]["value"]
    assert wl.n_groups == G["groups"]["value"] and wl.n_experts // wl.n_groups == G["groups"]["group_size"]
    assert wl.topk_groups == G["groups"]["eligible"]
    assert wl.routed_scale == G["routed_scale"]["value"]
    for name in ("prefill", "skewed", "fp8"):
        w2 = WORKLOADS[name]
        assert (w2.d, w2.n_experts, w2.top_k, w2.hidden) == (wl.d, wl.n_experts, wl.top_k, wl.hidden)


def test_parameter_counts_reproduce_printed_figures():
    wl = WORKLOADS["decode"]
    per_expert = wl.params_per_expert
    assert round(per_expert / 1e6, 1) == G["params_per_expert_millions"]["value"]
    per_layer = (wl.n_experts + 1) * per_expert
    assert round(per_layer / 1e9, 1) == G["expert_params_per_layer_billions"]["value"]
    layers = G["expert_params_all_moe_layers_billions"]["moe_layers"]
    assert round(per_layer * layers / 1e9, 1) == G["expert_params_all_moe_layers_billions"]["value"]
    active = (wl.top_k + 1) * per_expert * layers
    assert round(active / 1e9, 1) == G["active_expert_params_per_token_billions"]["value"]
    assert wl.n_experts // wl.top_k == G["stored_to_exercised_ratio"]["value"]


def test_flops_per_token():
    wl = WORKLOADS["decode"]
    # 2 x (router 256 x 7168 + 9 experts x 3 x 7168 x 2048) multiply-adds
    assert wl.flops_per_token == 796_393_472
    assert WORKLOADS["tiny"].flops_per_token == 2 * (16 * 256 + 5 * 3 * 256 * 128)
