"""Oracle pins: batch-union lists and the grouped-vs-per-token invariant."""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_coli_b200 import synth


def _brute(idx, E):
    T, k = idx.shape
    pairs = sorted(((int(idx[t, j]), t, t * k + j) for t in range(T) for j in range(k)))
    counts = np.bincount(idx.ravel(), minlength=E)
    return counts, [p for (_, _, p) in pairs]


@pytest.mark.parametrize("T,E,k", [(1, 16, 2), (4, 16, 2), (37, 64, 8), (200, 256, 8), (3, 5, 5)])
def test_union_matches_brute_force(T, E, k):
    rng = np.random.default_rng(T * 1000 + E)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    idx, _ = oracle.route(lg, k)
    un = oracle.union(idx, E)
    counts, pairs = _brute(idx, E)
    assert np.array_equal(un["counts"], counts)
    assert list(un["pairs"]) == pairs
    assert un["offsets"][0] == 0 and un["offsets"][E] == T * k
    assert np.array_equal(np.diff(un["offsets"]), counts)
    act = [e for e in range(E) if counts[e] > 0]
    assert un["n_active"] == len(act)
    assert list(un["active"][:len(act)]) == act
    # every pair appears exactly once; each list is ascending in token
    assert sorted(un["pairs"]) == list(range(T * k))
    for e in range(E):
        lst = un["pairs"][un["offsets"][e]:un["offsets"][e + 1]]
        assert np.all(np.diff(lst // k) > 0)
        assert np.all(idx.ravel()[lst] == e)


def test_union_empty_and_bad_index():
    un = oracle.union(np.zeros((0, 2), np.int32), 4)
    assert un["n_active"] == 0 and list(un["offsets"]) == [0, 0, 0, 0, 0]
    with pytest.raises(ValueError):
        oracle.union(np.array([[0, 4]], np.int32), 4)
    with pytest.raises(ValueError):
        oracle.union(np.array([[-1, 2]], np.int32), 4)


def test_grouped_equals_per_token():
    H, I, E, k, T = 256, 128, 16, 2, 9
    bank = synth.make_expert_bank(H, I, E + 1, seed=11)
    ex = oracle.Experts([bank.expert_numpy(e) for e in range(E + 1)])
    xb = synth.make_activations(T, H, seed=12).view(torch.int16).numpy().view(np.uint16)
    lg = synth.make_logits_normal(T, E, seed=13).numpy()
    idx, w = oracle.route(lg, k)
    un = oracle.union(idx, E)
    res = np.random.default_rng(0).standard_normal((T, H))
    per_tok = oracle.layer(H, I, E, k, 1, ex, xb, idx, w, residual=res)
    grouped = oracle.layer_grouped(H, I, E, k, 1, ex, xb, w, un, residual=res)
    err = np.linalg.norm(per_tok - grouped) / np.linalg.norm(per_tok)
    assert err <= 1e-12
