"""Helpers for the GPU parity tests: CUDA path through the C ABI on one
side, the CPU oracle on the other, fed the same seeded inputs."""
import os

import numpy as np
import pytest
import torch

import oracle

REL_L2 = 2e-3        # FFN/layer output: relative L2 error bound
MAX_ABS_FRAC = 1e-2  # FFN/layer output: max |err| <= 1e-2 * max |ref|

requires_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def threads():
    return max(1, min(64, os.cpu_count() or 1))


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_experts(bank, needed) -> oracle.Experts:
    needed = set(int(e) for e in needed)
    return oracle.Experts([bank.expert_numpy(e) if e in needed else None for e in range(bank.n)])


def ulp32(x: np.ndarray) -> np.ndarray:
    x = np.abs(np.asarray(x, np.float32))
    return np.spacing(np.maximum(x, np.float32(np.finfo(np.float32).tiny)))


def assert_weights_close(w_gpu: np.ndarray, w_ref: np.ndarray):
    """GPU fp32 weights within 2 ulp of the oracle's double rounded to fp32."""
    ref32 = w_ref.astype(np.float32)
    diff = np.abs(w_gpu.astype(np.float64) - ref32.astype(np.float64))
    assert np.all(diff <= 2 * ulp32(ref32)), float(diff.max())


def assert_close(got: np.ndarray, ref: np.ndarray, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), what
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    mx = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300)
    assert rel <= REL_L2, f"{what}: rel L2 {rel:.3e} > {REL_L2}"
    assert mx <= MAX_ABS_FRAC, f"{what}: max abs frac {mx:.3e} > {MAX_ABS_FRAC}"
    return rel, mx


def reference_layer(bank, E, k, n_shared, x, logits, residual=None, sample=None):
    """Oracle output rows for `sample` tokens (all if None) from the same
    logits the GPU routed on.  Returns (out [n][H], idx, w)."""
    lg = logits.detach().float().cpu().numpy() if isinstance(logits, torch.Tensor) else logits
    idx, w = oracle.route(lg, k)
    T = lg.shape[0]
    sample = np.arange(T) if sample is None else np.asarray(sample)
    needed = set(idx[sample].ravel().tolist()) | {E + s for s in range(n_shared)}
    ex = oracle_experts(bank, needed)
    res = None
    if residual is not None:
        res = residual.detach().float().cpu().numpy().astype(np.float64)
    out = oracle.layer(bank.hidden, bank.inter, E, k, n_shared, ex, bits(x), idx, w, residual=res,
                       sample=sample.astype(np.int32), n_threads=threads())
    return out, idx, w


def covering_sample(idx: np.ndarray, n_total: int) -> np.ndarray:
    """A deterministic token sample in which every expert that ``idx``
    ([T][k]) routes to appears at least once: a greedy set cover (the token
    that adds the most uncovered experts, lowest index on ties), then evenly
    spaced tokens up to ``n_total``.  Sorted ascending."""
    T = idx.shape[0]
    E = int(idx.max()) + 1
    hit = np.zeros((T, E), dtype=bool)
    hit[np.arange(T)[:, None], idx] = True
    uncovered = hit.any(axis=0)
    chosen = []
    while uncovered.any():
        gain = hit[:, uncovered].sum(axis=1)
        t = int(np.argmax(gain))   # first maximum: the lowest token index
        chosen.append(t)
        uncovered &= ~hit[t]
    picked = set(chosen)
    for t in np.linspace(0, T - 1, n_total).round().astype(np.int64):
        if len(picked) >= n_total:
            break
        picked.add(int(t))
    return np.array(sorted(picked), dtype=np.int64)
