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


# ---- router logits: closed forms ------------------------------------------
# The router scores every routed expert for each token, logits[t][e] =
# sum_h x[t][h] W_r[e][h] ("zhichai.net/topic/178503686", MoE-sparsity
# section).  Shapes below are non-square, so a transposed or mis-strided read
# of W_r or x cannot reproduce the expected values.

BF16_ONE = 0x3F80


def test_router_logits_golden_worked_example():
    xs, ws, ls = [], [], []
    for line in open(os.path.join(os.path.dirname(__file__), "golden", "router_logits.txt")):
        f = line.split("#")[0].split("[")[0].split()
        if not f:
            continue
        if f[0] == "x":
            xs.append([int(v, 16) for v in f[1:]])
        elif f[0] == "w":
            ws.append([float(v) for v in f[1:]])
        elif f[0] == "l":
            ls.append([float(v) for v in f[1:]])
    got = oracle.router_logits(np.array(xs, np.uint16), np.array(ws, np.float32))
    assert got.shape == (2, 4)
    assert np.array_equal(got, np.array(ls))


def test_router_logits_one_hot_tokens_pick_router_columns():
    """x[t] = one-hot at h_t (bf16 1.0): logits[t][e] = W_r[e][h_t] exactly."""
    T, H, E = 3, 7, 5
    hot = [2, 6, 0]
    x = np.zeros((T, H), np.uint16)
    for t, h in enumerate(hot):
        x[t, h] = BF16_ONE
    # distinct dyadic entries (exact in fp32): 1/8 steps per expert, 1/64 per column
    wr = np.array([[(e + 1) / 8 + h / 64 for h in range(H)] for e in range(E)], np.float32)
    got = oracle.router_logits(x, wr)
    for t, h in enumerate(hot):
        for e in range(E):
            assert got[t, e] == (e + 1) / 8 + h / 64


def test_router_logits_one_hot_router_rows_pick_token_elements():
    """W_r[e] = 1/8 at column c_e, 0 elsewhere: logits[t][e] = x[t][c_e] / 8."""
    T, H, E = 2, 6, 4
    cols = [5, 0, 3, 3]
    vals = [[0x4000, 0xBF80, 0x3F00, 0x4080, 0x0000, 0xC040],   # 2 -1 0.5 4 0 -3
            [0x3E80, 0x4120, 0xC100, 0x3F80, 0x8000, 0x3FC0]]   # .25 10 -8 1 -0 1.5
    decoded = [[2, -1, 0.5, 4, 0, -3], [0.25, 10, -8, 1, 0, 1.5]]
    wr = np.zeros((E, H), np.float32)
    for e, c in enumerate(cols):
        wr[e, c] = 0.125
    got = oracle.router_logits(np.array(vals, np.uint16), wr)
    for t in range(T):
        for e, c in enumerate(cols):
            assert got[t, e] == decoded[t][c] / 8


def test_router_logits_constant_token_signed_rows():
    """x = 0.5 everywhere (H = 8); row e of W_r holds e + 1 entries +2^-6 and
    the rest -2^-6, so logits[t][e] = 0.5 * 2^-6 * (2(e + 1) - 8)."""
    H, E = 8, 4
    x = np.full((2, H), 0x3F00, np.uint16)
    wr = np.full((E, H), -2.0 ** -6, np.float32)
    for e in range(E):
        wr[e, : e + 1] = 2.0 ** -6
    got = oracle.router_logits(x, wr)
    expect = [-0.046875, -0.03125, -0.015625, 0.0]
    assert np.array_equal(got, np.array([expect, expect]))
