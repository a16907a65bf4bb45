"""GPU parity of the whole layer (moe_forward through the C ABI) against the oracle.

Tolerance (the layer-output bar): max |err| <= 1e-2 x RMS(y_ref) for the fp32
output against the oracle's unrounded fp64 output; the bf16 output adds one
bf16 ulp of |y_ref| for its own storage rounding.  The oracle consumes the
GPU's router logits (checked separately within tolerance) so that both sides
route identically; the routing itself is compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import fine_grained_moe_gemm_b200 as moe
from moe_testlib import assert_close_bf16, assert_close_rms, cfg_of, oracle_layer, u16, weights_for_forward, x_host
from workloads import WORKLOADS, make_inputs, make_residual, make_x

pytestmark = pytest.mark.gpu

DEV = "cuda"
REL = 1e-2

_cache = {}


def inputs(name, device_gen):
    """Full-size inputs are generated once per workload on the GPU (weights do not depend on T)."""
    key = (name, device_gen)
    if key not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        wl = WORKLOADS[name]
        W = make_inputs(wl, device_gen)
        _cache[key] = {k: v.to(DEV) for k, v in W.items()}
    return _cache[key]


def run_forward(wl, W, x, y_dtype=torch.float32, accumulate=False, y0=None, routing=None):
    cfg = cfg_of(wl)
    T = x.shape[0]
    ws = torch.empty(moe.workspace_size(cfg, T), dtype=torch.uint8, device=DEV)
    y = y0.clone() if y0 is not None else torch.empty((T, wl.d), dtype=y_dtype, device=DEV)
    moe.moe_forward(cfg, weights_for_forward(W), x, W["bias"], y, accumulate=accumulate, workspace=ws,
                    routing_out=routing)
    torch.cuda.synchronize()
    assert moe.device_error() == 0
    return y


def forward_routing(wl, W, x):
    """The routing moe_forward used (its own logits), checked bit for bit against
    the oracle's selection on those logits, and its logits against the oracle's
    fp64 router within tolerance."""
    T = x.shape[0]
    E, k = wl.n_experts, wl.top_k
    r = {"logits": torch.empty((T, E), dtype=torch.float32, device=DEV),
         "topk_idx": torch.empty((T, k), dtype=torch.int32, device=DEV),
         "topk_w": torch.empty((T, k), dtype=torch.float32, device=DEV),
         "counts": torch.empty(E, dtype=torch.int32, device=DEV),
         "offsets": torch.empty(E + 1, dtype=torch.int32, device=DEV),
         "src": torch.empty(T * k, dtype=torch.int32, device=DEV),
         "inv": torch.empty(T * k, dtype=torch.int32, device=DEV)}
    run_forward(wl, W, x, routing=r)
    l = r["logits"].cpu().numpy()
    ridx, rw = oracle.select(l, W["bias"].cpu().numpy(), wl.n_groups, wl.topk_groups, wl.top_k)
    assert np.array_equal(r["topk_idx"].cpu().numpy(), ridx)
    assert np.array_equal(r["topk_w"].cpu().numpy().view(np.uint32), rw.view(np.uint32))
    # the layer's own permutation (single- or multi-CTA), bit-exact
    for got, ref in zip((r["counts"], r["offsets"], r["src"], r["inv"]), oracle.permute(ridx, E)):
        assert np.array_equal(got.cpu().numpy(), ref)
    rows = np.unique(np.linspace(0, T - 1, min(T, 16)).astype(np.int64))
    l_ref = oracle.router_logits(x_host(x[torch.from_numpy(rows).to(DEV)]), u16(W["w_router"]))
    rms = float(np.sqrt(np.mean(l_ref.astype(np.float64) ** 2)))
    assert float(np.max(np.abs(l[rows] - l_ref))) <= 1e-5 * np.sqrt(wl.d) * rms
    return ridx, rw


def oracle_y(wl, W, x, tokens, chunk=16):
    """The oracle's output for the listed tokens, routed as the forward routed.  The
    tokens go in chunks, each with a host copy of only the experts it uses, so the
    host memory stays bounded however many tokens are checked."""
    idx, w = forward_routing(wl, W, x)
    xh = x_host(x)
    out = []
    tokens = np.asarray(tokens, dtype=np.int32)
    for c0 in range(0, tokens.size, chunk):
        part = tokens[c0:c0 + chunk]
        L = oracle_layer(wl, W, np.unique(idx[part]))
        out.append(oracle.expert_tokens(L, xh, idx, w, part))
        del L
    return np.concatenate(out) if out else np.zeros((0, wl.d))


# ----------------------------------------------------------------------------- tiny workload (full check)

@pytest.mark.parametrize("T", [64, 1, 2, 3, 127, 129, 600])
def test_tiny_full(T):
    wl = WORKLOADS["tiny"]
    W = inputs("tiny", "cpu")
    x = make_x(wl, "cpu", T=T).to(DEV)
    ref = oracle_y(wl, W, x, np.arange(T))
    y = run_forward(wl, W, x, torch.float32)
    assert_close_rms(y.cpu().numpy(), ref, REL)
    yb = run_forward(wl, W, x, torch.bfloat16)
    assert_close_bf16(yb, ref, REL)


def test_tiny_accumulate_into_residual():
    wl = WORKLOADS["tiny"]
    W = inputs("tiny", "cpu")
    x = make_x(wl, "cpu").to(DEV)
    ref = oracle_y(wl, W, x, np.arange(wl.T))
    r32 = make_residual(wl, "cpu", dtype=torch.float32).to(DEV)
    y = run_forward(wl, W, x, accumulate=True, y0=r32)
    assert_close_rms(y.cpu().numpy(), ref + r32.cpu().numpy().astype(np.float64), REL)
    rb = make_residual(wl, "cpu", dtype=torch.bfloat16).to(DEV)
    yb = run_forward(wl, W, x, accumulate=True, y0=rb)
    assert_close_bf16(yb, ref + rb.float().cpu().numpy().astype(np.float64), REL)


# ----------------------------------------------------------------------------- DeepSeek-V3 sizes (sampled tokens)

def _sample(T, n, seed=0):
    rng = np.random.default_rng(seed)
    s = set([0, T - 1]) | set(rng.choice(T, min(n, T), replace=False).tolist())
    return np.array(sorted(s), dtype=np.int32)


def _spread(T, n, seed=0):
    """n tokens spread over the batch: one from each of n equal slices (so every token
    chunk of the GEMMs' schedules is hit), plus the first and the last."""
    rng = np.random.default_rng(seed)
    edges = np.linspace(0, T, n + 1).astype(np.int64)
    s = {0, T - 1} | {int(rng.integers(a, b)) for a, b in zip(edges[:-1], edges[1:]) if b > a}
    return np.array(sorted(s), dtype=np.int32)


def test_decode_every_token():
    """The benchmarked decode batch (T = 128): every token, every feature, fp32 and bf16
    outputs, against the oracle."""
    wl = WORKLOADS["decode"]
    W = inputs("decode", "cuda")
    x = W["x"]
    toks = np.arange(wl.T, dtype=np.int32)
    ref = oracle_y(wl, W, x, toks)
    y = run_forward(wl, W, x, torch.float32)
    assert_close_rms(y.cpu().numpy(), ref, REL)
    yb = run_forward(wl, W, x, torch.bfloat16)
    assert_close_bf16(yb, ref, REL)


@pytest.mark.parametrize("T", [1, 37])
def test_decode(T):
    wl = WORKLOADS["decode"]
    W = inputs("decode", "cuda")
    x = make_x(wl, "cuda", T=T) if T != wl.T else W["x"]
    toks = np.arange(T, dtype=np.int32)
    ref = oracle_y(wl, W, x, toks)
    y = run_forward(wl, W, x, torch.float32)
    assert_close_rms(y.cpu().numpy()[toks], ref, REL)
    yb = run_forward(wl, W, x, torch.bfloat16)
    assert_close_bf16(yb[torch.from_numpy(toks).long().to(DEV)], ref, REL)


@pytest.mark.parametrize("T", [1000, 2048])
def test_mid_batches_sampled(T):
    """The single-CTA kernels' wider token tiles at full size: ~31 rows per expert
    (64-row tiles) at T = 1000 and ~64 (128-row tiles) at T = 2048."""
    wl = WORKLOADS["prefill"]
    W = inputs("prefill", "cuda")
    x = make_x(wl, "cuda", T=T)
    toks = _spread(T, 8, seed=T)
    ref = oracle_y(wl, W, x, toks)
    yb = run_forward(wl, W, x, torch.bfloat16)
    assert_close_bf16(yb[torch.from_numpy(toks).long().to(DEV)], ref, REL)
    cfg = cfg_of(wl)
    assert moe.forward_plan(cfg, T)["token_tile"] == (64 if T == 1000 else 128)


def test_prefill_sampled():
    wl = WORKLOADS["prefill"]
    W = inputs("prefill", "cuda")
    x = W["x"]
    toks = _spread(wl.T, 32, seed=1)
    ref = oracle_y(wl, W, x, toks)
    yb = run_forward(wl, W, x, torch.bfloat16)
    assert_close_bf16(yb[torch.from_numpy(toks).long().to(DEV)], ref, REL)


def test_large_batch_sampled():
    """T = 65536, four times the skewed workload's batch: the multi-CTA permutation over
    256 blocks, 589,824 permuted rows, several token chunks for every expert; routing
    and permutation checked for all tokens, outputs on a sample."""
    wl = WORKLOADS["prefill"]
    W = inputs("prefill", "cuda")
    T = 65536
    x = make_x(wl, "cuda", T=T)
    toks = _spread(T, 16, seed=3)
    ref = oracle_y(wl, W, x, toks)
    yb = run_forward(wl, W, x, torch.bfloat16)
    assert_close_bf16(yb[torch.from_numpy(toks).long().to(DEV)], ref, REL)


def test_skewed_sampled():
    wl = WORKLOADS["skewed"]
    W = inputs("skewed", "cuda")
    x = W["x"]
    toks = _spread(wl.T, 32, seed=2)
    ref = oracle_y(wl, W, x, toks)
    y = run_forward(wl, W, x, torch.float32)
    assert_close_rms(y.cpu().numpy()[toks], ref, REL)


def test_forward_routing_repeatable_bitwise():
    """The split-K router sums its partials in a fixed order: the forward's logits,
    routing and permutation-dependent output are bit-identical run to run."""
    wl = WORKLOADS["decode"]
    W = inputs("decode", "cuda")
    x = W["x"]
    T = x.shape[0]
    outs = []
    for _ in range(3):
        r = {"logits": torch.empty((T, wl.n_experts), dtype=torch.float32, device=DEV),
             "topk_idx": torch.empty((T, wl.top_k), dtype=torch.int32, device=DEV),
             "topk_w": torch.empty((T, wl.top_k), dtype=torch.float32, device=DEV)}
        run_forward(wl, W, x, routing=r)
        outs.append({k: v.cpu().numpy() for k, v in r.items()})
    for o in outs[1:]:
        for k in o:
            assert np.array_equal(o[k].view(np.uint32), outs[0][k].view(np.uint32)), k
