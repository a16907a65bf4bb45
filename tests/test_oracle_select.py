"""Pins for the oracle's routing stage (S2: sigmoid, selection bias, group-limited top-k).

- Brute force: on tiny inputs, enumerate every set of ``topk_groups`` groups and
  then every k-subset of the eligible experts, maximising exact sums; the
  two-stage definition of the field guide's routing cutaway must come out.
- Special cases: one group (or all groups eligible) reduces to plain
  ``topk(sigmoid + bias)`` as in the router box's snippet, checked against torch.
- Invariants: k distinct experts from at most topk_groups groups, weights that
  sum to 1 before scaling, the bias moving selection but never the weights.
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _brute_force(l_row, bias, G, topk_groups, k):
    s = oracle.sigmoid(l_row)
    b = (s + bias.astype(np.float32)).astype(np.float32)          # fp32 add, as specified
    E = b.size
    gs = E // G
    # group score: the best pair of biased scores inside the group (fp32 sum)
    gscore = []
    for g in range(G):
        vals = b[g * gs:(g + 1) * gs]
        best = None
        for i, j in itertools.combinations(range(gs), 2):
            v = np.float32(vals[i]) + np.float32(vals[j])
            best = v if best is None or v > best else best
        gscore.append(np.float32(best))
    # group subsets: maximal exact sum, then lexicographically smallest index set
    best_sub, best_val = None, None
    for sub in itertools.combinations(range(G), topk_groups):
        v = sum(Fraction(float(gscore[g])) for g in sub)
        if best_val is None or v > best_val:
            best_sub, best_val = sub, v
    eligible = [e for g in best_sub for e in range(g * gs, (g + 1) * gs)]
    best_set, best_val = None, None
    for sub in itertools.combinations(sorted(eligible), k):
        v = sum(Fraction(float(b[e])) for e in sub)
        if best_val is None or v > best_val:
            best_set, best_val = sub, v
    order = sorted(best_set, key=lambda e: (-float(b[e]), e))
    S = sum(float(s[e]) for e in order)
    w = np.array([float(s[e]) / S for e in order])
    return np.array(order, dtype=np.int32), w


@pytest.mark.parametrize("E,G,tg,k,T,seed", [
    (16, 4, 2, 4, 64, 0),      # the tiny workload's shape
    (12, 3, 2, 3, 40, 1),
    (16, 8, 3, 4, 40, 2),
    (8, 2, 1, 2, 40, 3),
    (18, 6, 4, 5, 30, 4),
])
def test_select_matches_brute_force(E, G, tg, k, T, seed):
    rng = np.random.default_rng(seed)
    logits = (rng.standard_normal((T, E)) * 2).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    idx, w = oracle.select(logits, bias, G, tg, k)
    for t in range(T):
        bi, bw = _brute_force(logits[t], bias, G, tg, k)
        assert np.array_equal(idx[t], bi), (t, idx[t], bi)
        np.testing.assert_allclose(w[t], bw, rtol=2.5e-7, atol=0)


def test_brute_force_catches_a_global_topk_mistake():
    """The two-stage rule differs from a global top-k: a group with one very
    strong expert loses eligibility to groups with two good ones."""
    E, G, tg, k = 8, 4, 2, 2
    logits = np.full((1, E), -4.0, dtype=np.float32)
    logits[0, 0] = 6.0                          # group 0: one strong expert
    logits[0, 2:4] = 3.0                        # group 1: two good experts
    logits[0, 4:6] = 2.9                        # group 2: two good experts
    bias = np.zeros(E, dtype=np.float32)
    idx, _ = oracle.select(logits, bias, G, tg, k)
    bi, _ = _brute_force(logits[0], bias, G, tg, k)
    assert list(idx[0]) == list(bi) == [2, 3]
    assert 0 not in idx[0]


@pytest.mark.parametrize("G_all", [False, True])
def test_one_group_reduces_to_torch_topk(G_all):
    rng = np.random.default_rng(5)
    T, E, k = 200, 256, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    G, tg = (8, 8) if G_all else (1, 1)
    idx, w = oracle.select(logits, bias, G, tg, k)
    s = torch.from_numpy(oracle.sigmoid(logits))
    ref = torch.topk(s + torch.from_numpy(bias), k, dim=-1).indices.numpy()
    assert np.array_equal(idx, ref)
    ws = torch.gather(s, 1, torch.from_numpy(ref).long()).double()
    np.testing.assert_allclose(w, (ws / ws.sum(-1, keepdim=True)).numpy(), rtol=3e-7)


def test_ties_resolve_to_lower_index_and_equal_weights():
    T, E, G, tg, k = 3, 256, 8, 4, 8
    logits = np.zeros((T, E), dtype=np.float32)
    bias = np.zeros(E, dtype=np.float32)
    idx, w = oracle.select(logits, bias, G, tg, k)
    assert np.array_equal(idx, np.tile(np.arange(8, dtype=np.int32), (T, 1)))
    assert np.all(w == np.float32(0.125))                      # 1/8 exactly
    # a tie between groups: groups 3 and 5 identical and best -> both eligible,
    # experts then ranked by score with the lower index first
    l2 = np.full((1, E), -5.0, dtype=np.float32)
    l2[0, 3 * 32:3 * 32 + 4] = 2.0
    l2[0, 5 * 32:5 * 32 + 4] = 2.0
    idx2, _ = oracle.select(l2, bias, G, tg, k)
    assert list(idx2[0]) == [96, 97, 98, 99, 160, 161, 162, 163]


def _routing_invariants(idx, w, E, G, tg, k):
    gs = E // G
    for t in range(idx.shape[0]):
        assert len(set(idx[t].tolist())) == k
        assert len(set((idx[t] // gs).tolist())) <= tg
        S = np.float32(0)
        for j in range(k):
            S = np.float32(S + w[t, j])
        assert abs(float(S) - 1.0) <= 2 * 2 ** -23 * k


def test_invariants_decode_shape():
    rng = np.random.default_rng(6)
    T, E, G, tg, k = 512, 256, 8, 4, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    idx, w = oracle.select(logits, bias, G, tg, k)
    _routing_invariants(idx, w, E, G, tg, k)
    # slot order: descending biased score
    s = oracle.sigmoid(logits)
    bsel = np.take_along_axis(s + bias, idx, 1)
    assert np.all(np.diff(bsel, axis=1) <= 0)


def _per_expert(idx_row, w_row):
    return {int(e): w_row[j] for j, e in enumerate(idx_row)}


def test_bias_moves_selection_not_weights():
    rng = np.random.default_rng(7)
    T, E, G, tg, k = 512, 256, 8, 4, 8
    logits = rng.standard_normal((T, E)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    idx, w = oracle.select(logits, bias, G, tg, k)
    for trial in range(4):
        b2 = (bias + rng.uniform(-0.03, 0.03, E)).astype(np.float32)
        idx2, w2 = oracle.select(logits, b2, G, tg, k)
        same = np.all(np.sort(idx2, 1) == np.sort(idx, 1), axis=1)
        # the bias moves selection for some tokens ...
        assert 0 < same.sum() < T
        # ... and wherever the selected set is unchanged (even if the slot order
        # changed) each expert keeps a bit-identical weight
        for t in np.nonzero(same)[0]:
            a, b = _per_expert(idx[t], w[t]), _per_expert(idx2[t], w2[t])
            assert all(a[e] == b[e] for e in a), t
    # a large bias on one expert puts it in every token's first slot, while the
    # weights still follow the unbiased scores
    b3 = bias.copy()
    b3[17] += 5.0
    idx3, w3 = oracle.select(logits, b3, G, tg, k)
    assert np.all(idx3[:, 0] == 17)
    s = oracle.sigmoid(logits)
    ssel = np.take_along_axis(s, idx3, 1)
    assert np.array_equal(np.argmax(w3, 1), np.argmax(ssel, 1))
    np.testing.assert_allclose(w3, ssel / ssel.astype(np.float64).sum(1, keepdims=True), rtol=3e-7)


def test_invalid_sizes_rejected():
    l = np.zeros((1, 16), dtype=np.float32)
    b = np.zeros(16, dtype=np.float32)
    with pytest.raises(ValueError):
        oracle.select(l, b, 3, 2, 4)        # 16 % 3 != 0
    with pytest.raises(ValueError):
        oracle.select(l, b, 4, 1, 5)        # k > eligible experts
