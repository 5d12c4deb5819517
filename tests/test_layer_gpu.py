"""GPU layer / FFN (coli_moe_layer, coli_moe_ffn) against the oracle.

Output bar: relative L2 <= 2e-3 and max |err| <= 1e-2 * max |ref| per call;
routing bit-exact on identical fp32 logits."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_close, assert_weights_close, bits, covering_sample, reference_layer,
                      requires_gpu)
from int4_routed_expert_coli_b200 import synth

pytestmark = [pytest.mark.gpu, requires_gpu]

GLM = dict(H=6144, I=2048, E=256, k=8)


@pytest.fixture(scope="module")
def tiny():
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(256, 128, 17, seed=0, device="cuda")
    return bank, c.MoELayer(bank, n_routed=16, top_k=2, n_shared=1)


@pytest.fixture(scope="module")
def glm():
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(GLM["H"], GLM["I"], GLM["E"] + 1, seed=1, device="cuda")
    return bank, c.MoELayer(bank, n_routed=GLM["E"], top_k=GLM["k"], n_shared=1)


def _layer(layer, x, logits=None, router_w=None, residual=None, out_bf16=False):
    from int4_routed_expert_coli_b200 import coli_moe as c
    T = x.shape[0]
    idx = torch.empty(T, layer.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, layer.k, dtype=torch.float32, device="cuda")
    ws = layer.workspace(T)
    out = layer.layer(x, logits=logits, router_w=router_w, residual=residual,
                      out_dtype=c.COLI_OUT_BF16 if out_bf16 else c.COLI_OUT_F32,
                      topk_idx_out=idx, topk_w_out=w, ws=ws)
    assert c.coli_moe_get_status(ws) == c.COLI_OK
    return out, idx.cpu().numpy(), w.cpu().numpy(), ws


def test_tiny_layer_with_router_weight(tiny):
    """Tiny layer: H 256, I 128, 16 experts top-2 + 1 shared, 4 tokens, router
    weight fp32 N(0, 0.02), seed 0."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank, layer = tiny
    x = synth.make_activations(4, 256, seed=0, device="cuda")
    wr = synth.make_router_weight(16, 256, seed=0, device="cuda")
    out, idx, w, ws = _layer(layer, x, router_w=wr)
    off = c.COLI_WS_LOGITS_OFFSET
    lg_gpu = ws[off:off + 4 * 16 * 4].view(torch.float32).view(4, 16).cpu().numpy()
    lg_ref = oracle.router_logits(bits(x), wr.cpu().numpy())
    assert np.linalg.norm(lg_gpu - lg_ref) / np.linalg.norm(lg_ref) <= 1e-5
    ref, ri, rw = reference_layer(bank, 16, 2, 1, x, lg_gpu)
    assert np.array_equal(idx, ri)
    assert_weights_close(w, rw)
    assert_close(out.cpu().numpy(), ref, "tiny layer")


def test_tiny_layer_bf16_out_with_residual(tiny):
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank, layer = tiny
    x = synth.make_activations(4, 256, seed=3, device="cuda")
    lg = synth.make_logits_normal(4, 16, seed=3, device="cuda")
    res = synth.make_residual(4, 256, seed=4, dtype=torch.bfloat16, device="cuda")
    out, idx, w, _ = _layer(layer, x, logits=lg, residual=res, out_bf16=True)
    ref, ri, _ = reference_layer(bank, 16, 2, 1, x, lg, residual=res)
    assert np.array_equal(idx, ri)
    ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert_close(out.double().cpu().numpy(), ref_bf16, "tiny bf16")


def test_tiny_layer_f32_residual_many_tokens(tiny):
    bank, layer = tiny
    T = 203                                   # ragged: 25 full N-tiles + 3
    x = synth.make_activations(T, 256, seed=5, device="cuda")
    lg = synth.make_logits_normal(T, 16, seed=5, device="cuda")
    res = synth.make_residual(T, 256, seed=6, device="cuda")
    out, idx, w, _ = _layer(layer, x, logits=lg, residual=res)
    ref, ri, rw = reference_layer(bank, 16, 2, 1, x, lg, residual=res)
    assert np.array_equal(idx, ri)
    assert_close(out.cpu().numpy(), ref, "tiny T=203")


@pytest.mark.parametrize("T", [19, 40])
def test_tiny_layer_small_batch(tiny, T):
    """Tiny layer on the small-batch kernels: H / 64 = 4 and I / 64 = 2 scale
    groups (scales read from global memory, down's only stage half full);
    T = 40 puts the shared expert's list in two column chunks."""
    bank, layer = tiny
    x = synth.make_activations(T, 256, seed=7 + T, device="cuda")
    lg = synth.make_logits_normal(T, 16, seed=8 + T, device="cuda")
    res = synth.make_residual(T, 256, seed=9 + T, device="cuda")
    out, idx, w, _ = _layer(layer, x, logits=lg, residual=res)
    ref, ri, _ = reference_layer(bank, 16, 2, 1, x, lg, residual=res)
    assert np.array_equal(idx, ri)
    assert_close(out.cpu().numpy(), ref, f"tiny small-batch T={T}")


@pytest.mark.parametrize("prefill_min", [0, 10 ** 6])  # default path / streaming forced
def test_ragged_dims_two_shared(prefill_min):
    """H, I multiples of 128 but not of 256; 12 experts top-3; 2 shared;
    both the default (tensor-core) path and the streaming dequant-GEMV."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    H, I, E, k, T = 384, 384, 12, 3, 19
    bank = synth.make_expert_bank(H, I, E + 2, seed=8, device="cuda")
    layer = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=2, prefill_min_tokens=prefill_min)
    x = synth.make_activations(T, H, seed=9, device="cuda")
    lg = synth.make_logits_normal(T, E, seed=9, device="cuda")
    out, idx, w, _ = _layer(layer, x, logits=lg)
    ref, ri, _ = reference_layer(bank, E, k, 2, x, lg)
    assert np.array_equal(idx, ri)
    assert_close(out.cpu().numpy(), ref, "ragged")


def test_glm_decode_steps(glm):
    """GLM-5.2-shaped decode: 256 experts top-8 + 1 shared, one token per
    step, logits N(0,1), x N(0,1); a few seeded steps."""
    bank, layer = glm
    for s in range(4):
        x = synth.make_activations(1, 6144, seed=1000 + s, device="cuda")
        lg = synth.make_logits_normal(1, 256, seed=2000 + s, device="cuda")
        out, idx, w, _ = _layer(layer, x, logits=lg)
        ref, ri, rw = reference_layer(bank, 256, 8, 1, x, lg)
        assert np.array_equal(idx, ri)
        assert_weights_close(w, rw)
        assert_close(out.cpu().numpy(), ref, f"decode step {s}")


@pytest.mark.parametrize("T,n_sample,path", [(4, 4, "default"), (32, 32, "default"),
                                              (32, 32, "gemm"), (32, 32, "stream")])
def test_glm_small_batch_zipf(glm, T, n_sample, path):
    """Speculative-verify / small batch: Zipf-1.1 routing, 71.6 % repeats
    (T = 32 on the default small-batch kernels, on the tensor-core grouped
    GEMM with small token tiles, and on the streaming path)."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank, layer = glm
    if path != "default":
        layer = c.MoELayer(bank, n_routed=GLM["E"], top_k=GLM["k"], n_shared=1,
                           prefill_min_tokens=1 if path == "gemm" else 10 ** 6)
    _, logits = synth.zipf_routing(T, 256, 8, steps=2, seed=T)
    for s, lg_np in enumerate(logits):
        x = synth.make_activations(T, 6144, seed=3000 + s, device="cuda")
        lg = torch.from_numpy(lg_np).cuda()
        out, idx, w, _ = _layer(layer, x, logits=lg)
        sample = np.linspace(0, T - 1, n_sample).round().astype(np.int64)
        ref, ri, _ = reference_layer(bank, 256, 8, 1, x, lg, sample=sample)
        assert np.array_equal(idx, ri)
        assert_close(out.cpu().numpy()[sample], ref, f"T={T} step {s}")


def test_glm_prefill_sampled(glm):
    """Prefill: 4096 tokens, uniform logits (~128 tokens per expert); routing
    checked in full, the output on a deterministic 256-token sample that
    contains at least one token of every active routed expert, so every
    expert's tensor-core tiles are compared with the oracle."""
    bank, layer = glm
    T = 4096
    x = synth.make_activations(T, 6144, seed=4000, device="cuda")
    lg = synth.make_logits_uniform(T, 256, seed=4001, device="cuda")
    out, idx, w, _ = _layer(layer, x, logits=lg)
    sample = covering_sample(idx, 256)
    assert len(sample) == 256
    assert set(idx[sample].ravel().tolist()) == set(idx.ravel().tolist())
    ref, ri, rw = reference_layer(bank, 256, 8, 1, x, lg, sample=sample)
    assert np.array_equal(idx, ri)
    assert_weights_close(w, rw)
    assert_close(out.cpu().numpy()[sample], ref, "prefill sample")


def test_glm_deterministic(glm):
    bank, layer = glm
    x = synth.make_activations(32, 6144, seed=5000, device="cuda")
    _, logits = synth.zipf_routing(32, 256, 8, steps=1, seed=5)
    lg = torch.from_numpy(logits[0]).cuda()
    a = _layer(layer, x, logits=lg)[0]
    b = _layer(layer, x, logits=lg)[0]
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_ffn_api_with_prepared_union(tiny):
    """coli_moe_route -> coli_moe_union -> coli_moe_ffn equals coli_moe_layer."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank, layer = tiny
    T, E, k = 9, 16, 2
    x = synth.make_activations(T, 256, seed=11, device="cuda")
    lg = synth.make_logits_normal(T, E, seed=11, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    c.coli_moe_route(T, E, k, lg, idx, w)
    i32 = dict(dtype=torch.int32, device="cuda")
    counts, offsets = torch.empty(E, **i32), torch.empty(E + 1, **i32)
    pairs, active, na = torch.empty(T * k, **i32), torch.empty(E, **i32), torch.empty(1, **i32)
    c.coli_moe_union(T, E, k, idx, counts, offsets, pairs, active, na)
    ws = layer.workspace(T)
    out = torch.empty(T, 256, dtype=torch.float32, device="cuda")
    c.coli_moe_ffn(layer.handle, T, x, w, counts, offsets, pairs, active, na, None, out,
                   c.COLI_OUT_F32, ws)
    assert c.coli_moe_get_status(ws) == c.COLI_OK
    ref_out = _layer(layer, x, logits=lg)[0]
    assert torch.equal(out, ref_out)
    # a corrupted active list is reported, not faulted on
    bad = active.clone()
    bad[0] = 999
    c.coli_moe_ffn(layer.handle, T, x, w, counts, offsets, pairs, bad, na, None, out,
                   c.COLI_OUT_F32, ws)
    assert c.coli_moe_get_status(ws) == c.COLI_ERR_BAD_INDEX
    c.coli_moe_workspace_clear(ws)
    assert c.coli_moe_get_status(ws) == c.COLI_OK


def test_host_errors_launch_nothing(tiny):
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank, layer = tiny
    x = synth.make_activations(4, 256, seed=12, device="cuda")
    lg = synth.make_logits_normal(4, 16, seed=12, device="cuda")
    out = torch.empty(4, 256, device="cuda")
    small = torch.zeros(layer.workspace_size(4) - 256, dtype=torch.uint8, device="cuda")
    assert c.coli_moe_layer(layer.handle, 4, x, lg, None, None, out, c.COLI_OUT_F32, None, None,
                            small, raise_on_error=False) == c.COLI_ERR_WORKSPACE
    ws = layer.workspace(4)
    xs = torch.empty(4 * 256 + 8, dtype=torch.bfloat16, device="cuda")[1:4 * 256 + 1]
    assert c.coli_moe_layer(layer.handle, 4, xs, lg, None, None, out, c.COLI_OUT_F32, None,
                            None, ws, raise_on_error=False) == c.COLI_ERR_ALIGN
    assert c.coli_moe_layer(layer.handle, 4, x, lg, lg, None, out, c.COLI_OUT_F32, None, None,
                            ws, raise_on_error=False) == c.COLI_ERR_INVALID_ARG
    assert c.coli_moe_layer(layer.handle, 0, x, lg, None, None, out, c.COLI_OUT_F32, None, None,
                            ws, raise_on_error=False) == c.COLI_OK


def test_glm_decode_eight_tokens(glm):
    """T = 8: every token is one of the 8 MMA columns of the fused decode path."""
    bank, layer = glm
    x = synth.make_activations(8, 6144, seed=6000, device="cuda")
    lg = synth.make_logits_normal(8, 256, seed=6001, device="cuda")
    res = synth.make_residual(8, 6144, seed=6002, device="cuda")
    out, idx, w, _ = _layer(layer, x, logits=lg, residual=res)
    ref, ri, rw = reference_layer(bank, 256, 8, 1, x, lg, residual=res)
    assert np.array_equal(idx, ri)
    assert_close(out.cpu().numpy(), ref, "decode T=8")


def test_glm_fused_decode_matches_streaming_path(glm):
    """The fused decode kernel (handle with tensor maps) and the streaming
    kernels (the no-handle entry point) on the same inputs."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank, layer = glm
    for T in (1, 3):
        x = synth.make_activations(T, 6144, seed=6100 + T, device="cuda")
        lg = synth.make_logits_normal(T, 256, seed=6200 + T, device="cuda")
        a = _layer(layer, x, logits=lg)[0]
        b = torch.empty_like(a)
        c.coli_moe_layer_noalloc(layer.desc, T, x, lg, None, b, c.COLI_OUT_F32)
        torch.cuda.synchronize()
        assert_close(a.cpu().numpy(), b.double().cpu().numpy(), f"fused vs streaming T={T}")


def test_glm_decode_deterministic(glm):
    bank, layer = glm
    x = synth.make_activations(1, 6144, seed=6300, device="cuda")
    lg = synth.make_logits_normal(1, 256, seed=6301, device="cuda")
    a = _layer(layer, x, logits=lg)[0]
    b = _layer(layer, x, logits=lg)[0]
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("E,k,T", [(64, 8, 7), (64, 2, 8), (64, 1, 5), (200, 8, 8), (256, 4, 8),
                                   (256, 8, 3)])
def test_fused_decode_routing_ties_and_specials(E, k, T):
    """The fused decode kernel routes inside the kernel (a butterfly top-k per
    token row; E <= 256, T * k < E): indices bit-exact and weights within 2
    ulp of the oracle on tied, NaN, +-inf and signed-zero logits and on rows
    that are all NaN or all -inf; the layer output against the oracle."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    H, I = 512, 512
    bank = synth.make_expert_bank(H, I, E + 1, seed=E + k, device="cuda")
    layer = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=1)
    rng = np.random.default_rng(E * 31 + k * 7 + T)
    rows = []
    for t in range(T):
        r = rng.integers(-3, 4, size=E).astype(np.float32)   # many ties
        kind = t % 7
        if kind == 1:
            r[rng.integers(0, E, size=3)] = np.nan
        elif kind == 2:
            r[rng.integers(0, E, size=2)] = -np.inf
        elif kind == 3:
            r[rng.integers(0, E, size=2)] = np.inf
        elif kind == 4:
            r[rng.integers(0, E, size=4)] = -0.0
            r[rng.integers(0, E, size=4)] = 0.0
        elif kind == 5:
            r[:] = np.nan
        elif kind == 6:
            r[:] = -np.inf
        rows.append(r)
    lg = torch.from_numpy(np.stack(rows)).cuda()
    x = synth.make_activations(T, H, seed=3, device="cuda")
    out, idx, w, _ = _layer(layer, x, logits=lg)
    ref, ri, rw = reference_layer(bank, E, k, 1, x, lg)
    assert np.array_equal(idx, ri)
    assert_weights_close(w, rw)
    assert_close(out.cpu().numpy(), ref, f"E={E} k={k} T={T}")
