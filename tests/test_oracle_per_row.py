"""Oracle pins for the per-row int4 format: the codes of gs64, one bf16
scale per row ("ssnai.com/JustVugg_colibri.html", decision guide: the older
per-row int4 GLM-5.2 mirror; "yunpan.plus/t/30351-1-1", capability four:
gs64 against per-row int4).  Reading: W[n][k] = q[n][k] * s[n], scales
[rows][1]."""
import math

import numpy as np
import torch

import oracle
from npref import bf16_bits_to_f64, swiglu_mlp_rows
from int4_routed_expert_coli_b200 import synth


def test_hand_packed_row_uses_one_scale_across_groups():
    # row 0: bytes 0x8F (codes -1, -8), scale 0.5; row 1: bytes 0x12 (2, 1), scale -1
    q = np.zeros((2, 64), np.uint8)              # K = 128: two gs64 groups per row
    q[0, :] = 0x8F
    q[1, :] = 0x12
    s = np.array([0x3F00, 0xBF80], np.uint16)    # [rows][1]
    for k, v in [(0, -0.5), (1, -4.0), (64, -0.5), (127, -4.0)]:
        assert oracle.weight_per_row(q, s, 128, 0, k) == v
    for k, v in [(0, -2.0), (1, -1.0), (66, -2.0), (127, -1.0)]:
        assert oracle.weight_per_row(q, s, 128, 1, k) == v


def _rand_expert(H, I, seed, per_row):
    bank = synth.make_expert_bank(H, I, 1, seed=seed, per_row=per_row)
    return bank.expert_numpy(0)


def test_per_row_equals_gs64_with_the_row_scale_in_every_group():
    """Exact: a per-row expert and the gs64 expert whose every group scale is
    the row's scale dequantise to the same weights, so the FFN outputs are
    identical bit for bit."""
    H, I = 256, 128
    ex = _rand_expert(H, I, 5, per_row=True)
    assert ex["group"] == 0 and ex["gate_s"].shape == (I, 1) and ex["down_s"].shape == (H, 1)
    gs = dict(ex)
    gs["group"] = 64
    gs["gate_s"] = np.repeat(ex["gate_s"], H // 64, axis=1)
    gs["up_s"] = np.repeat(ex["up_s"], H // 64, axis=1)
    gs["down_s"] = np.repeat(ex["down_s"], I // 64, axis=1)
    x = bf16_bits_to_f64(synth.make_activations(1, H, seed=6).view(torch.int16).numpy()
                         .view(np.uint16))[0]
    assert np.array_equal(oracle.expert_ffn(H, I, ex, x), oracle.expert_ffn(H, I, gs, x))


def test_per_row_closed_form():
    """All codes 1, one scale 2^-6 per row, x = 1, K = H = 256: g = u = 4;
    y[m] = I * 2^-6 * silu(4) * 4."""
    H, I = 256, 128
    pack = lambda rows, K: np.full((rows, K // 2), 0x11, np.uint8)
    ex = dict(gate_q=pack(I, H), up_q=pack(I, H), down_q=pack(H, I),
              gate_s=np.full((I, 1), 0x3C80, np.uint16), up_s=np.full((I, 1), 0x3C80, np.uint16),
              down_s=np.full((H, 1), 0x3C80, np.uint16), group=0)
    y = oracle.expert_ffn(H, I, ex, np.ones(H))
    h = 4.0 / (1.0 + math.exp(-4.0)) * 4.0
    np.testing.assert_allclose(y, I * 2.0 ** -6 * h, rtol=I * 2.0 ** -53)


def test_per_row_matches_numpy_mlp():
    H, I = 384, 256
    ex = _rand_expert(H, I, 7, per_row=True)
    x = np.random.default_rng(8).standard_normal(H)
    ref = swiglu_mlp_rows(ex, x)
    np.testing.assert_allclose(oracle.expert_ffn(H, I, ex, x), ref, rtol=1e-12, atol=1e-12)
