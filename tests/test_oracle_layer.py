"""Oracle pins: symmetries of the whole layer."""
import numpy as np
import torch
from scipy.special import softmax

import oracle
from int4_routed_expert_coli_b200 import synth
from npref import bf16_bits_to_f64, swiglu_mlp

H, I, E, K = 256, 128, 16, 2


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _setup(T, seed):
    bank = synth.make_expert_bank(H, I, E + 1, seed=seed)
    exs = [bank.expert_numpy(e) for e in range(E + 1)]
    xb = _bits(synth.make_activations(T, H, seed=seed + 1))
    lg = synth.make_logits_normal(T, E, seed=seed + 2).numpy()
    return exs, xb, lg


def test_token_permutation_equivariance_exact():
    T = 7
    exs, xb, lg = _setup(T, 40)
    ex = oracle.Experts(exs)
    idx, w = oracle.route(lg, K)
    out = oracle.layer(H, I, E, K, 1, ex, xb, idx, w)
    perm = np.random.default_rng(0).permutation(T)
    idx2, w2 = oracle.route(lg[perm], K)
    out2 = oracle.layer(H, I, E, K, 1, ex, xb[perm], idx2, w2)
    assert np.array_equal(out2, out[perm])


def test_expert_relabelling_invariance_exact():
    T = 5
    exs, xb, lg = _setup(T, 50)
    idx, w = oracle.route(lg, K)
    out = oracle.layer(H, I, E, K, 1, oracle.Experts(exs), xb, idx, w)
    pi = np.random.default_rng(1).permutation(E)         # new id of old expert e is pi[e]
    exs2 = [None] * (E + 1)
    for e in range(E):
        exs2[pi[e]] = exs[e]
    exs2[E] = exs[E]
    lg2 = np.empty_like(lg)
    lg2[:, pi] = lg
    idx2, w2 = oracle.route(lg2, K)
    assert np.array_equal(idx2, pi[idx])
    out2 = oracle.layer(H, I, E, K, 1, oracle.Experts(exs2), xb, idx2, w2)
    assert np.array_equal(out, out2)


def test_dense_equivalence_at_k_equals_E():
    T = 3
    exs, xb, lg = _setup(T, 60)
    idx, w = oracle.route(lg, E)
    got = oracle.layer(H, I, E, E, 1, oracle.Experts(exs), xb, idx, w)
    x = bf16_bits_to_f64(xb)
    for t in range(T):
        p = softmax(lg[t].astype(np.float64))
        ref = sum(p[e] * swiglu_mlp(exs[e], x[t]) for e in range(E)) + swiglu_mlp(exs[E], x[t])
        np.testing.assert_allclose(got[t], ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())


def test_sampled_tokens_equal_full_rows():
    T = 6
    exs, xb, lg = _setup(T, 70)
    ex = oracle.Experts(exs)
    idx, w = oracle.route(lg, K)
    full = oracle.layer(H, I, E, K, 1, ex, xb, idx, w)
    part = oracle.layer(H, I, E, K, 1, ex, xb, idx, w, sample=np.array([4, 1]))
    assert np.array_equal(part, full[[4, 1]])
