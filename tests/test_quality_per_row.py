"""Quantisation quality of the two int4 formats on synthetic weights.  The
pages report the cosine similarity of dequantised to original weights on a
real model (Qwen3.6) rising from 0.98777 (per-row int4) to 0.99313 (gs64)
("yunpan.plus/t/30351-1-1", capability four).  Real weights are not in this
container, so the same comparison runs on Gaussian and on heavier-tailed
(Student-t, 4 degrees of freedom) matrices of the GLM-5.2 gate/up shape:
symmetric round-to-nearest int4 codes in [-8, 7] with the scale max|w| / 7
of the group (or row), rounded to bf16 first."""
import numpy as np
import torch


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()


def quantise(w, group):
    """Dequantised copy of w [rows][K] after int4 quantisation with one scale
    per `group` consecutive elements of a row (group = K: one per row)."""
    rows, K = w.shape
    g = w.reshape(rows, K // group, group)
    s = _bf16(np.abs(g).max(axis=2, keepdims=True) / 7.0)
    s = np.where(s == 0, 1.0, s)
    q = np.clip(np.rint(g / s), -8, 7)
    return (q * s).reshape(rows, K)


def cosine(a, b):
    return float(np.sum(a * b) / np.sqrt(np.sum(a * a) * np.sum(b * b)))


def _compare(w):
    return cosine(w, quantise(w, 64)), cosine(w, quantise(w, w.shape[1]))


def test_gs64_beats_per_row_on_synthetic_weights():
    rng = np.random.default_rng(0)
    gauss = rng.standard_normal((512, 6144))
    heavy = rng.standard_t(4, size=(512, 6144))
    for name, w in (("gaussian", gauss), ("student-t4", heavy)):
        c64, crow = _compare(w)
        print(f"{name}: cosine gs64 {c64:.5f}, per-row {crow:.5f}")
        assert 0.8 < crow < c64 < 1.0
    # Gaussian weights: the per-row step is ~0.6 sigma, the gs64 step ~0.35
    c64, crow = _compare(gauss)
    assert crow < 0.99 and c64 > 0.99
