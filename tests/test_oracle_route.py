"""Oracle pins: top-k routing and renormalised softmax weights."""
import itertools
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "route_closed_forms.txt")


def _golden():
    cases = []
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, lg, idx, w = [f.strip() for f in line.split("|")]
        cases.append((int(k), np.array([float(v) for v in lg.split()], np.float32),
                      [int(v) for v in idx.split()], [float(v) for v in w.split()], lg))
    return cases


def case_text(case):
    return case[4].split()


@pytest.mark.parametrize("case", _golden())
def test_closed_forms(case):
    k, lg, idx, w, _ = case
    got_i, got_w = oracle.route(lg[None, :], k)
    assert list(got_i[0]) == idx
    # logits are stored as fp32: a closed form stated at a logit that fp32
    # cannot hold exactly (ln 3) is met up to that input rounding only
    lg64 = np.array([float(v) for v in case_text(case)], np.float64)
    finite = np.isfinite(lg64)
    exact = np.array_equal(lg64[finite], lg[finite].astype(np.float64))
    np.testing.assert_allclose(got_w[0], w, rtol=0, atol=1e-15 if exact else 1e-7)


def _brute_force(row, k):
    """Best k-subset by enumeration: compare the subsets' values sorted
    descending (NaN lowest), then their sorted indices (lower first)."""
    E = len(row)

    def key(i):  # larger is better; NaN below everything
        v = row[i]
        return (0, 0.0) if np.isnan(v) else (1, float(v))

    best = None
    for sub in itertools.combinations(range(E), k):
        ordered = sorted(sub, key=lambda i: (tuple(-x for x in key(i)), i))
        vals = [key(i) for i in ordered]
        cand = (vals, [-i for i in ordered])
        if best is None or cand > best[0]:
            best = (cand, ordered)
    return best[1]


def test_brute_force_small_with_ties():
    rng = np.random.default_rng(0)
    for trial in range(300):
        E = int(rng.integers(1, 9))
        k = int(rng.integers(1, E + 1))
        # small integer logits force many ties; sprinkle specials
        row = rng.integers(-2, 3, size=E).astype(np.float32)
        if trial % 5 == 0:
            row[rng.integers(0, E)] = np.nan
        if trial % 7 == 0:
            row[rng.integers(0, E)] = -np.inf
        if trial % 11 == 0:
            row[rng.integers(0, E)] = -0.0
        idx, _ = oracle.route(row[None, :], k)
        assert list(idx[0]) == _brute_force(row, k), (row, k)


def test_weights_sum_to_one_and_positive():
    rng = np.random.default_rng(1)
    lg = rng.standard_normal((64, 256)).astype(np.float32)
    idx, w = oracle.route(lg, 8)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    assert np.all(w > 0)
    # weights follow the slot order (descending logits)
    assert np.all(np.diff(w, axis=1) <= 0)


def test_k_equals_E_is_textbook_softmax():
    rng = np.random.default_rng(2)
    lg = rng.standard_normal((5, 16)).astype(np.float32)
    idx, w = oracle.route(lg, 16)
    for t in range(5):
        ref = softmax(lg[t].astype(np.float64))
        np.testing.assert_allclose(w[t], ref[idx[t]], rtol=1e-14)
        assert sorted(idx[t]) == list(range(16))


def test_weight_ratio_is_exp_of_logit_gap():
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((8, 32)).astype(np.float32)
    idx, w = oracle.route(lg, 4)
    for t in range(8):
        for j in range(1, 4):
            gap = float(lg[t, idx[t, 0]]) - float(lg[t, idx[t, j]])
            assert math.isclose(w[t, 0] / w[t, j], math.exp(gap), rel_tol=1e-13)


def test_route_rejects_bad_sizes():
    with pytest.raises(ValueError):
        oracle.route(np.zeros((1, 4), np.float32), 5)


def test_router_logits_match_numpy():
    from npref import bf16_bits_to_f64
    rng = np.random.default_rng(5)
    xb = (rng.standard_normal((3, 256)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    wr = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    got = oracle.router_logits(xb, wr)
    ref = bf16_bits_to_f64(xb) @ wr.astype(np.float64).T
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)
