"""coli_moe_layer_noalloc: the layer step for callers that cannot allocate.

Some callers cannot call cudaMalloc: their device memory is owned by a host
framework that plans every byte up front and forbids side allocations, or
they run a latency-critical decode loop where cudaMalloc (which can
synchronise the device) is not acceptable.  They cannot allocate a workspace
or create a handle, so this entry point takes neither: its scratch is a fixed
array inside the library.  These tests call it through the C ABI twice in a
row and compare each result with coli_moe_layer on the same inputs, to the
tolerance the other layer tests use; they also check its output against the
CPU oracle directly, and that a call's status word does not carry over into
the next call.
"""
import numpy as np
import pytest
import torch

from gpu_util import assert_close, reference_layer, requires_gpu
from int4_routed_expert_coli_b200 import synth

pytestmark = [pytest.mark.gpu, requires_gpu]


def _pair(layer, T, seed, out_bf16=False, residual=False):
    from int4_routed_expert_coli_b200 import coli_moe as c
    od = c.COLI_OUT_BF16 if out_bf16 else c.COLI_OUT_F32
    dt = torch.bfloat16 if out_bf16 else torch.float32
    x = synth.make_activations(T, layer.H, seed=seed, device="cuda")
    lg = synth.make_logits_normal(T, layer.E, seed=seed + 1, device="cuda")
    res = synth.make_residual(T, layer.H, seed=seed + 2, dtype=dt, device="cuda") if residual else None
    ref = layer.layer(x, logits=lg, residual=res, out_dtype=od)
    got = torch.full((T, layer.H), float("nan"), dtype=dt, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    c.coli_moe_layer_noalloc(layer.desc, T, x, lg, res, got, od, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == c.COLI_OK
    return got, ref


def test_noalloc_matches_layer_two_calls_glm_decode():
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(6144, 2048, 257, seed=60, device="cuda")
    layer = c.MoELayer(bank, n_routed=256, top_k=8, n_shared=1)
    for call, (T, seed) in enumerate([(1, 61), (8, 62)]):   # two calls in a row
        got, ref = _pair(layer, T, seed)
        assert_close(got.double().cpu().numpy(), ref.double().cpu().numpy(), f"call {call}")


def test_noalloc_matches_layer_tiny_bf16_residual():
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(256, 128, 17, seed=63, device="cuda")
    layer = c.MoELayer(bank, n_routed=16, top_k=2, n_shared=1)
    for T, seed in [(4, 64), (3, 65)]:
        got, ref = _pair(layer, T, seed, out_bf16=True, residual=True)
        assert_close(got.double().cpu().numpy(), ref.double().cpu().numpy(), "tiny")


def test_noalloc_rejects_oversize_calls():
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(256, 128, 17, seed=66, device="cuda")
    layer = c.MoELayer(bank, n_routed=16, top_k=2, n_shared=1)
    x = synth.make_activations(9, 256, seed=67, device="cuda")
    lg = synth.make_logits_normal(9, 16, seed=68, device="cuda")
    out = torch.empty(9, 256, device="cuda")
    s = c.coli_moe_layer_noalloc(layer.desc, 9, x, lg, None, out, c.COLI_OUT_F32,
                                 raise_on_error=False)
    assert s == c.COLI_ERR_WORKSPACE


def test_noalloc_matches_oracle_glm_decode():
    """GLM-5.2 shape, T = 1 and T = 8, against the oracle (not only against
    coli_moe_layer)."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(6144, 2048, 257, seed=70, device="cuda")
    layer = c.MoELayer(bank, n_routed=256, top_k=8, n_shared=1)
    for T, seed in [(1, 71), (8, 72)]:
        x = synth.make_activations(T, 6144, seed=seed, device="cuda")
        lg = synth.make_logits_normal(T, 256, seed=seed + 1, device="cuda")
        res = synth.make_residual(T, 6144, seed=seed + 2, device="cuda")
        got = torch.full((T, 6144), float("nan"), device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        c.coli_moe_layer_noalloc(layer.desc, T, x, lg, res, got, c.COLI_OUT_F32,
                                 status_out=status)
        torch.cuda.synchronize()
        assert int(status.item()) == c.COLI_OK
        ref, _, _ = reference_layer(bank, 256, 8, 1, x, lg, residual=res)
        assert_close(got.cpu().numpy(), ref, f"noalloc vs oracle T={T}")


def test_noalloc_status_word_is_per_call():
    """A call whose activations exceed the fp16 range reports COLI_ERR_RANGE;
    the next call on the same shared scratch starts from a clear status word
    and reports COLI_OK, with the same output as coli_moe_layer."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(256, 128, 17, seed=73, device="cuda")
    layer = c.MoELayer(bank, n_routed=16, top_k=2, n_shared=1)
    x = synth.make_activations(4, 256, seed=74, device="cuda")
    lg = synth.make_logits_normal(4, 16, seed=75, device="cuda")
    big = x.clone()
    big[1, 5] = 1.0e6   # outside fp16: clamped, reported
    out = torch.empty(4, 256, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    c.coli_moe_layer_noalloc(layer.desc, 4, big, lg, None, out, c.COLI_OUT_F32, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == c.COLI_ERR_RANGE
    got, ref = _pair(layer, 4, 74)
    assert_close(got.double().cpu().numpy(), ref.double().cpu().numpy(), "after a range error")
