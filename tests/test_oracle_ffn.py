"""Oracle pins: the SwiGLU expert FFN and the layer sum."""
import math

import numpy as np
import torch

import oracle
from int4_routed_expert_coli_b200 import synth
from npref import bf16_bits_to_f64, swiglu_mlp


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _const_expert(H, I, code_g, code_u, code_d, sbits):
    pack = lambda rows, K, c: np.full((rows, K // 2), ((c & 15) | ((c & 15) << 4)), np.uint8)
    return dict(gate_q=pack(I, H, code_g), up_q=pack(I, H, code_u), down_q=pack(H, I, code_d),
                gate_s=np.full((I, H // 64), sbits, np.uint16),
                up_s=np.full((I, H // 64), sbits, np.uint16),
                down_s=np.full((H, I // 64), sbits, np.uint16))


def test_closed_form_constant_expert():
    # all codes 1, scale 2^-6, x = 1, K = H = 256: g = u = 256 / 64 = 4 exactly;
    # h = silu(4) * 4; y[m] = I * 2^-6 * h for every m.
    H, I = 256, 128
    ex = _const_expert(H, I, 1, 1, 1, 0x3C80)
    y = oracle.expert_ffn(H, I, ex, np.ones(H))
    h = 4.0 / (1.0 + math.exp(-4.0)) * 4.0
    np.testing.assert_allclose(y, I * 2.0 ** -6 * h, rtol=I * 2.0 ** -53)


def test_zero_gate_gives_zero():
    H, I = 256, 128
    ex = _const_expert(H, I, 0, 3, -5, 0x3F80)
    y = oracle.expert_ffn(H, I, ex, np.linspace(-2, 2, H))
    assert np.all(y == 0.0)


def test_negative_codes_sign():
    # gate codes -1, up codes -1, down codes 1, scale 1/64, x = 1:
    # g = u = -4; h = silu(-4) * -4 > 0; y = I/64 * h
    H, I = 256, 128
    ex = _const_expert(H, I, -1, -1, 1, 0x3C80)
    y = oracle.expert_ffn(H, I, ex, np.ones(H))
    h = -4.0 / (1.0 + math.exp(4.0)) * -4.0
    np.testing.assert_allclose(y, I * 2.0 ** -6 * h, rtol=I * 2.0 ** -53)


def test_matches_numpy_dense_mlp_random():
    H, I = 256, 128
    bank = synth.make_expert_bank(H, I, 1, seed=5)
    ex = bank.expert_numpy(0)
    x = bf16_bits_to_f64(_bits(synth.make_activations(3, H, seed=6)))
    ref = swiglu_mlp(ex, x)
    for t in range(3):
        got = oracle.expert_ffn(H, I, ex, x[t])
        np.testing.assert_allclose(got, ref[t], rtol=1e-11, atol=1e-12 * np.abs(ref[t]).max())


def test_down_scale_linearity_exact():
    H, I = 256, 128
    bank = synth.make_expert_bank(H, I, 1, seed=7)
    ex = bank.expert_numpy(0)
    ex2 = dict(ex)
    # doubling a bf16 scale: add one to the exponent field (exact)
    ex2["down_s"] = (ex["down_s"].astype(np.uint32) + (1 << 7)).astype(np.uint16)
    x = bf16_bits_to_f64(_bits(synth.make_activations(1, H, seed=8)))[0]
    y1 = oracle.expert_ffn(H, I, ex, x)
    y2 = oracle.expert_ffn(H, I, ex2, x)
    assert np.array_equal(y2, 2.0 * y1)


def test_layer_single_expert_is_dense_mlp():
    # E = 1, k = 1, no shared expert: the layer is one dense SwiGLU MLP (w = 1)
    H, I = 256, 128
    bank = synth.make_expert_bank(H, I, 1, seed=9)
    ex = bank.expert_numpy(0)
    xb = _bits(synth.make_activations(4, H, seed=10))
    idx, w = oracle.route(np.zeros((4, 1), np.float32), 1)
    assert np.all(w == 1.0)
    got = oracle.layer(H, I, 1, 1, 0, oracle.Experts([ex]), xb, idx, w)
    ref = swiglu_mlp(ex, bf16_bits_to_f64(xb))
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())


def test_layer_matches_numpy_mixture_with_shared_and_residual():
    H, I, E, k, T = 256, 128, 16, 2, 5
    bank = synth.make_expert_bank(H, I, E + 1, seed=21)
    exs = [bank.expert_numpy(e) for e in range(E + 1)]
    xb = _bits(synth.make_activations(T, H, seed=22))
    lg = synth.make_logits_normal(T, E, seed=23).numpy()
    idx, w = oracle.route(lg, k)
    res = np.random.default_rng(1).standard_normal((T, H))
    got = oracle.layer(H, I, E, k, 1, oracle.Experts(exs), xb, idx, w, residual=res,
                       n_threads=3)
    x = bf16_bits_to_f64(xb)
    ref = res.copy()
    for t in range(T):
        for j in range(k):
            ref[t] += w[t, j] * swiglu_mlp(exs[idx[t, j]], x[t])
        ref[t] += swiglu_mlp(exs[E], x[t])
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())


def test_thread_count_does_not_change_result():
    H, I, E, k, T = 256, 128, 16, 2, 6
    bank = synth.make_expert_bank(H, I, E + 1, seed=31)
    ex = oracle.Experts([bank.expert_numpy(e) for e in range(E + 1)])
    xb = _bits(synth.make_activations(T, H, seed=32))
    idx, w = oracle.route(synth.make_logits_normal(T, E, seed=33).numpy(), k)
    a = oracle.layer(H, I, E, k, 1, ex, xb, idx, w, n_threads=1)
    b = oracle.layer(H, I, E, k, 1, ex, xb, idx, w, n_threads=4)
    assert np.array_equal(a, b)
