"""GPU routing (coli_moe_route) against the oracle: indices bit-exact,
weights within 2 fp32 ulp, on random and adversarial logits."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_weights_close, requires_gpu

pytestmark = [pytest.mark.gpu, requires_gpu]


def _run(lg: np.ndarray, k: int):
    from int4_routed_expert_coli_b200 import coli_moe as c
    T, E = lg.shape
    d = torch.from_numpy(np.ascontiguousarray(lg, np.float32)).cuda()
    idx = torch.full((max(T, 1), k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((max(T, 1), k), -7.0, dtype=torch.float32, device="cuda")
    c.coli_moe_route(T, E, k, d, idx, w)
    torch.cuda.synchronize()
    return idx[:T].cpu().numpy(), w[:T].cpu().numpy()


def _check(lg, k):
    gi, gw = _run(lg, k)
    ri, rw = oracle.route(lg, k)
    assert np.array_equal(gi, ri)
    assert_weights_close(gw, rw)
    ok = np.isfinite(rw).all(axis=1)
    np.testing.assert_allclose(gw[ok].astype(np.float64).sum(axis=1), 1.0, atol=1e-6)


@pytest.mark.parametrize("T,E,k", [(4, 16, 2), (1, 256, 8), (4096, 256, 8), (37, 37, 5),
                                   (64, 1024, 32), (5, 32, 32), (9, 100, 1), (3, 1, 1),
                                   (2, 33, 32)])
def test_route_normal_logits(T, E, k):
    lg = np.random.default_rng(T * 7 + E).standard_normal((T, E)).astype(np.float32)
    _check(lg, k)


def test_route_uniform_prefill_logits():
    lg = np.random.default_rng(4).random((4096, 256), dtype=np.float32)
    _check(lg, 8)


def test_route_ties_and_specials():
    rng = np.random.default_rng(5)
    rows = []
    for t in range(512):
        E = 64
        r = rng.integers(-3, 4, size=E).astype(np.float32)      # many ties
        if t % 3 == 0:
            r[rng.integers(0, E, size=3)] = np.nan
        if t % 4 == 0:
            r[rng.integers(0, E, size=2)] = -np.inf
        if t % 5 == 0:
            r[rng.integers(0, E, size=2)] = np.inf
        if t % 6 == 0:
            r[rng.integers(0, E, size=4)] = -0.0
        rows.append(r)
    rows.append(np.full(64, 2.5, np.float32))                 # all equal
    rows.append(np.full(64, np.nan, np.float32))              # all NaN
    rows.append(np.full(64, -np.inf, np.float32))             # all -inf
    rows.append(-np.arange(64, dtype=np.float32))             # l = -index
    lg = np.stack(rows)
    for k in (1, 2, 8, 32):
        _check(lg, k)


def test_route_zero_tokens():
    from int4_routed_expert_coli_b200 import coli_moe as c
    assert c.coli_moe_route(0, 16, 2, None, None, None) == c.COLI_OK


def test_route_deterministic():
    lg = np.random.default_rng(6).standard_normal((1000, 256)).astype(np.float32)
    a = _run(lg, 8)
    b = _run(lg, 8)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))
