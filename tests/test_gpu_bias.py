"""GPU parity of the bias controller (moe_update_bias) against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import fine_grained_moe_gemm_b200 as moe
from moe_testlib import cfg_of
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,seed", [("decode", 0), ("decode", 1), ("tiny", 2)])
def test_update_bias_bit_exact(name, seed):
    wl = WORKLOADS[name]
    E = wl.n_experts
    rng = np.random.default_rng(seed)
    cases = [rng.integers(0, 60, E), np.full(E, 9), np.zeros(E), rng.poisson(4, E)]
    cases[3][3] = 10_000_000                          # a huge count (large fp32 sum)
    b0 = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    for gamma in (1e-3, 0.25):
        for c in cases:
            c = c.astype(np.int32)
            bias = torch.from_numpy(b0).to(DEV)
            moe.moe_update_bias(cfg_of(wl), torch.from_numpy(c).to(DEV), bias, gamma)
            torch.cuda.synchronize()
            ref = oracle.update_bias(c, b0, gamma)
            assert np.array_equal(bias.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_update_bias_from_the_layers_own_counts():
    """One controller step fed by the permutation of a real routing."""
    wl = WORKLOADS["decode"]
    rng = np.random.default_rng(3)
    T, E, k = 512, wl.n_experts, wl.top_k
    idx = np.stack([rng.choice(E, k, replace=False, p=np.arange(1, E + 1) ** -1.0 / np.sum(np.arange(1, E + 1) ** -1.0))
                    for _ in range(T)]).astype(np.int32)
    cfg = cfg_of(wl)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    src = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    moe.moe_permute(cfg, torch.from_numpy(idx).to(DEV), counts, offsets, src, inv)
    b0 = np.zeros(E, np.float32)
    bias = torch.from_numpy(b0).to(DEV)
    moe.moe_update_bias(cfg, counts, bias)
    torch.cuda.synchronize()
    ref = oracle.update_bias(oracle.permute(idx, E)[0], b0)
    assert np.array_equal(bias.cpu().numpy(), ref)
    assert (ref < 0).sum() > 0 and (ref > 0).sum() > 0
