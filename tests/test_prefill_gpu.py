"""Tensor-core (tcgen05) grouped-GEMM path against the oracle.

The path runs when T*k/E reaches the handle's prefill threshold; these tests
force it on small shapes with prefill_min_tokens=1 so that ragged token
tiles (1..128 tokens, several N tiles for the shared expert), several M tiles
and K blocks, and two shared experts are all covered."""
import numpy as np
import pytest
import torch

from gpu_util import assert_close, assert_weights_close, reference_layer, requires_gpu
from int4_routed_expert_coli_b200 import synth

pytestmark = [pytest.mark.gpu, requires_gpu]


def _run(layer, x, lg, residual=None, out_bf16=False):
    from int4_routed_expert_coli_b200 import coli_moe as c
    T = x.shape[0]
    idx = torch.empty(T, layer.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, layer.k, dtype=torch.float32, device="cuda")
    ws = layer.workspace(T)
    out = layer.layer(x, logits=lg, residual=residual, topk_idx_out=idx, topk_w_out=w, ws=ws,
                      out_dtype=c.COLI_OUT_BF16 if out_bf16 else c.COLI_OUT_F32)
    assert c.coli_moe_get_status(ws) == c.COLI_OK
    return out, idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T", [1, 37, 203, 700])
def test_prefill_path_tiny(T):
    from int4_routed_expert_coli_b200 import coli_moe as c
    H, I, E, k = 256, 128, 16, 2
    bank = synth.make_expert_bank(H, I, E + 1, seed=40, device="cuda")
    layer = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=1, prefill_min_tokens=1)
    x = synth.make_activations(T, H, seed=41 + T, device="cuda")
    lg = synth.make_logits_normal(T, E, seed=42 + T, device="cuda")
    out, idx, w = _run(layer, x, lg)
    ref, ri, rw = reference_layer(bank, E, k, 1, x, lg)
    assert np.array_equal(idx, ri)
    assert_weights_close(w, rw)
    assert_close(out.cpu().numpy(), ref, f"prefill tiny T={T}")


def test_prefill_path_ragged_two_shared_residual_bf16():
    from int4_routed_expert_coli_b200 import coli_moe as c
    H, I, E, k, T = 384, 384, 12, 3, 150
    bank = synth.make_expert_bank(H, I, E + 2, seed=43, device="cuda")
    layer = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=2, prefill_min_tokens=1)
    x = synth.make_activations(T, H, seed=44, device="cuda")
    lg = synth.make_logits_uniform(T, E, seed=45, device="cuda")
    res = synth.make_residual(T, H, seed=46, dtype=torch.bfloat16, device="cuda")
    out, idx, _ = _run(layer, x, lg, residual=res, out_bf16=True)
    ref, ri, _ = reference_layer(bank, E, k, 2, x, lg, residual=res)
    assert np.array_equal(idx, ri)
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert_close(out.double().cpu().numpy(), ref_bf16, "prefill ragged")


def test_prefill_and_gemv_paths_agree():
    """The same call through both FFN paths: each is checked against the
    oracle elsewhere; here they must agree with each other to the same bar."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    H, I, E, k, T = 512, 256, 16, 4, 96
    bank = synth.make_expert_bank(H, I, E + 1, seed=47, device="cuda")
    tc = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=1, prefill_min_tokens=1)
    gemv = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=1, prefill_min_tokens=10 ** 6)
    x = synth.make_activations(T, H, seed=48, device="cuda")
    lg = synth.make_logits_normal(T, E, seed=49, device="cuda")
    a = _run(tc, x, lg)[0].cpu().numpy()
    b = _run(gemv, x, lg)[0].cpu().numpy()
    assert_close(a, b.astype(np.float64), "tc vs gemv")


def test_prefill_deterministic():
    from int4_routed_expert_coli_b200 import coli_moe as c
    H, I, E, k, T = 256, 128, 16, 2, 500
    bank = synth.make_expert_bank(H, I, E + 1, seed=50, device="cuda")
    layer = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=1, prefill_min_tokens=1)
    x = synth.make_activations(T, H, seed=51, device="cuda")
    lg = synth.make_logits_uniform(T, E, seed=52, device="cuda")
    a = _run(layer, x, lg)[0]
    b = _run(layer, x, lg)[0]
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
