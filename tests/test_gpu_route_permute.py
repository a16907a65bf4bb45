"""GPU parity of stages 1-3 through the C ABI: router logits (tolerance), selection
and permutation (bit-exact against the oracle on identical inputs)."""
import numpy as np
import pytest
import torch

import oracle
import fine_grained_moe_gemm_b200 as moe
from moe_testlib import cfg_of, u16, x_host
from workloads import WORKLOADS, make_bias, make_weights, make_x

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _route(cfg, x, w_router, logits, bias, T):
    k = cfg.top_k
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.moe_route(cfg, x, w_router, logits, bias, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


def _logits_with_ties(rng, T, E):
    l = (rng.standard_normal((T, E)) * 2).astype(np.float32)
    # exact ties inside and across groups, and a few large magnitudes
    l[::3, 5] = l[::3, 7]
    l[::5, 40 % E] = l[::5, (40 + E // 2) % E]
    l[1::7, :] = np.round(l[1::7, :])
    l[2::11, 3] = 30.0
    l[2::13, 4] = -30.0
    return l


@pytest.mark.parametrize("name", ["tiny", "decode"])
@pytest.mark.parametrize("T", [1, 7, 64, 1000, 4099])
def test_select_bit_exact(name, T):
    wl = WORKLOADS[name]
    cfg = cfg_of(wl)
    rng = np.random.default_rng(T)
    l = _logits_with_ties(rng, T, wl.n_experts)
    b = rng.uniform(-0.1, 0.1, wl.n_experts).astype(np.float32)
    b[::9] = 0.0
    idx, w = _route(cfg, None, None, torch.from_numpy(l).to(DEV), torch.from_numpy(b).to(DEV), T)
    ridx, rw = oracle.select(l, b, wl.n_groups, wl.topk_groups, wl.top_k)
    assert np.array_equal(idx, ridx)
    assert np.array_equal(w.view(np.uint32), rw.view(np.uint32))


def test_select_all_equal_logits():
    wl = WORKLOADS["decode"]
    T = 33
    l = np.zeros((T, wl.n_experts), np.float32)
    b = np.zeros(wl.n_experts, np.float32)
    idx, w = _route(cfg_of(wl), None, None, torch.from_numpy(l).to(DEV), torch.from_numpy(b).to(DEV), T)
    assert np.array_equal(idx, np.tile(np.arange(8, dtype=np.int32), (T, 1)))
    assert np.all(w == np.float32(0.125))


def test_select_nonfinite_logits_are_flagged_and_ids_stay_valid():
    """Logits must be finite (a precondition).  A NaN or infinite logit sets
    MOE_DEVERR_NONFINITE; the NaN ranks last, so every token still gets k distinct
    in-range ids, and tokens whose logits are finite route exactly as the oracle."""
    wl = WORKLOADS["decode"]
    T, E = 40, wl.n_experts
    rng = np.random.default_rng(9)
    l = (rng.standard_normal((T, E)) * 2).astype(np.float32)
    l[3, :] = np.nan                                    # a whole token
    l[5, :E // 2] = np.nan                              # half of the groups
    l[7, 17] = np.nan
    l[9, 40] = np.inf
    b = np.zeros(E, np.float32)
    assert moe.device_error() == 0
    idx, w = _route(cfg_of(wl), None, None, torch.from_numpy(l).to(DEV), torch.from_numpy(b).to(DEV), T)
    assert moe.device_error() & moe.MOE_DEVERR_NONFINITE
    assert np.all((idx >= 0) & (idx < E))
    assert all(len(set(r)) == wl.top_k for r in idx.tolist())
    clean = [t for t in range(T) if np.all(np.isfinite(l[t]))]
    ridx, rw = oracle.select(l[clean], b, wl.n_groups, wl.topk_groups, wl.top_k)
    assert np.array_equal(idx[clean], ridx)
    assert np.array_equal(w[clean].view(np.uint32), rw.view(np.uint32))
    assert moe.device_error() == 0                      # read and cleared


@pytest.mark.parametrize("name,T", [("tiny", 64), ("tiny", 129), ("decode", 128), ("decode", 300)])
def test_router_logits_and_selection(name, T):
    wl = WORKLOADS[name]
    cfg = cfg_of(wl)
    W = {"w_router": make_weights_router(wl)}
    x = make_x(wl, "cpu", T=T).to(DEV)
    bias = make_bias(wl, "cpu").to(DEV)
    logits = torch.empty((T, wl.n_experts), dtype=torch.float32, device=DEV)
    idx, w = _route(cfg, x, W["w_router"], logits, bias, T)
    l_gpu = logits.cpu().numpy()
    l_ref = oracle.router_logits(x_host(x), u16(W["w_router"]))
    rms = float(np.sqrt(np.mean(l_ref.astype(np.float64) ** 2)))
    err = float(np.max(np.abs(l_gpu.astype(np.float64) - l_ref)))
    assert err <= 1e-5 * np.sqrt(wl.d) * rms, (err, rms)
    # selection from the GPU's own logits is bit-exact
    ridx, rw = oracle.select(l_gpu, bias.cpu().numpy(), wl.n_groups, wl.topk_groups, wl.top_k)
    assert np.array_equal(idx, ridx)
    assert np.array_equal(w.view(np.uint32), rw.view(np.uint32))


def make_weights_router(wl):
    from workloads import _normal_bf16, _seed, WEIGHT_STD
    return _normal_bf16((wl.n_experts, wl.d), WEIGHT_STD, "cpu", _seed(0, wl.wid, "w_router")).to(DEV)


def _rand_idx(rng, T, E, k, skew=False):
    if skew:
        p = np.arange(1, E + 1, dtype=np.float64) ** -1.2
        p /= p.sum()
        return np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32) if T else np.zeros((0, k), np.int32)


def _permute(cfg, idx_np):
    T, k = idx_np.shape
    E = cfg.n_experts
    idx = torch.from_numpy(idx_np).to(DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    src = torch.empty(max(T * k, 1), dtype=torch.int32, device=DEV)
    inv = torch.empty(max(T * k, 1), dtype=torch.int32, device=DEV)
    moe.moe_permute(cfg, idx, counts, offsets, src, inv)
    torch.cuda.synchronize()
    return counts.cpu().numpy(), offsets.cpu().numpy(), src.cpu().numpy()[:T * k], inv.cpu().numpy()[:T * k]


@pytest.mark.parametrize("name", ["tiny", "decode"])
@pytest.mark.parametrize("T,skew", [(1, False), (3, False), (64, False), (127, False), (129, True), (1000, False),
                                    (4096, True), (16384, True)])
def test_permute_bit_exact(name, T, skew):
    wl = WORKLOADS[name]
    cfg = cfg_of(wl)
    rng = np.random.default_rng(T)
    idx = _rand_idx(rng, T, wl.n_experts, wl.top_k, skew)
    got = _permute(cfg, idx)
    ref = oracle.permute(idx, wl.n_experts)
    for g, r, n in zip(got, ref, ("counts", "offsets", "src", "inv")):
        assert np.array_equal(g, r), n
    assert moe.device_error() == 0


def test_permute_all_tokens_one_expert_set():
    wl = WORKLOADS["decode"]
    T = 5000
    idx = np.tile(np.arange(100, 108, dtype=np.int32), (T, 1))
    got = _permute(cfg_of(wl), idx)
    ref = oracle.permute(idx, wl.n_experts)
    for g, r in zip(got, ref):
        assert np.array_equal(g, r)


def test_permute_reports_bad_expert_id():
    """An id outside [0, E) is skipped and flagged in the device error word (no trap)."""
    wl = WORKLOADS["tiny"]
    cfg = cfg_of(wl)
    assert moe.device_error() == 0
    idx = _rand_idx(np.random.default_rng(0), 20, wl.n_experts, wl.top_k)
    idx[3, 1] = wl.n_experts + 5
    counts, offsets, src, inv = _permute(cfg, idx)
    assert moe.device_error() & moe.MOE_DEVERR_BAD_EXPERT
    assert moe.device_error() == 0                      # read-and-clear
    assert counts.sum() == 20 * wl.top_k - 1 and inv[3 * wl.top_k + 1] == -1


def test_zero_tokens_is_a_no_op():
    wl = WORKLOADS["decode"]
    cfg = cfg_of(wl)
    e = torch.empty(0, device=DEV)
    moe.moe_route(cfg, None, None, torch.empty((0, wl.n_experts), device=DEV), torch.zeros(wl.n_experts, device=DEV),
                  torch.empty((0, 8), dtype=torch.int32, device=DEV), torch.empty((0, 8), device=DEV))
    counts, offsets, src, inv = _permute(cfg, np.zeros((0, 8), np.int32))
    assert moe.device_error() == 0


def test_repeatable_bitwise():
    wl = WORKLOADS["decode"]
    cfg = cfg_of(wl)
    T = 512
    wr = make_weights_router(wl)
    x = make_x(wl, "cpu", T=T).to(DEV)
    bias = make_bias(wl, "cpu").to(DEV)
    outs = []
    for _ in range(3):
        logits = torch.empty((T, wl.n_experts), dtype=torch.float32, device=DEV)
        idx, w = _route(cfg, x, wr, logits, bias, T)
        outs.append((logits.cpu().numpy(), idx, w, _permute(cfg, idx)))
    for o in outs[1:]:
        assert np.array_equal(o[0].view(np.uint32), outs[0][0].view(np.uint32))
        assert np.array_equal(o[1], outs[0][1]) and np.array_equal(o[2], outs[0][2])
        for a, b in zip(o[3], outs[0][3]):
            assert np.array_equal(a, b)
