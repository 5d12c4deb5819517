"""The per-row int4 format (one bf16 scale per row, group_size
COLI_GROUP_PER_ROW: "ssnai.com/JustVugg_colibri.html", decision guide, the
older GLM-5.2 mirror) on every kernel path, against the oracle's per-row
reading: the fused decode kernel (GLM-5.2 shape, T = 1 and 4), the
small-batch kernels (T = 32, scales from global memory), the tensor-core
grouped GEMM with small token tiles (T = 32) and large ones (T = 512), the
streaming dequant-GEMV (forced, and the tiny shape), and the entry point
without allocation.  Same tolerance as every layer test."""
import numpy as np
import pytest
import torch

from gpu_util import assert_close, covering_sample, reference_layer, requires_gpu
from int4_routed_expert_coli_b200 import synth

pytestmark = [pytest.mark.gpu, requires_gpu]


@pytest.fixture(scope="module")
def glm_rows():
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(6144, 2048, 257, seed=80, device="cuda", per_row=True)
    return bank, c.MoELayer(bank, n_routed=256, top_k=8, n_shared=1)


def _run(layer, x, lg, residual=None):
    from int4_routed_expert_coli_b200 import coli_moe as c
    T = x.shape[0]
    idx = torch.empty(T, layer.k, dtype=torch.int32, device="cuda")
    ws = layer.workspace(T)
    out = layer.layer(x, logits=lg, residual=residual, topk_idx_out=idx, ws=ws)
    assert c.coli_moe_get_status(ws) == c.COLI_OK
    return out, idx.cpu().numpy()


@pytest.mark.parametrize("T", [1, 4])
def test_per_row_fused_decode(glm_rows, T):
    bank, layer = glm_rows
    x = synth.make_activations(T, 6144, seed=81 + T, device="cuda")
    lg = synth.make_logits_normal(T, 256, seed=82 + T, device="cuda")
    res = synth.make_residual(T, 6144, seed=83, device="cuda")
    out, idx = _run(layer, x, lg, residual=res)
    ref, ri, _ = reference_layer(bank, 256, 8, 1, x, lg, residual=res)
    assert np.array_equal(idx, ri)
    assert_close(out.cpu().numpy(), ref, f"per-row fused decode T={T}")


@pytest.mark.parametrize("path", ["default", "gemm", "stream"])
def test_per_row_small_batch(glm_rows, path):
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank, layer = glm_rows
    if path != "default":
        layer = c.MoELayer(bank, n_routed=256, top_k=8, n_shared=1,
                           prefill_min_tokens=1 if path == "gemm" else 10 ** 6)
    T = 32
    _, logits = synth.zipf_routing(T, 256, 8, steps=1, seed=84)
    x = synth.make_activations(T, 6144, seed=85, device="cuda")
    lg = torch.from_numpy(logits[0]).cuda()
    out, idx = _run(layer, x, lg)
    ref, ri, _ = reference_layer(bank, 256, 8, 1, x, lg)
    assert np.array_equal(idx, ri)
    assert_close(out.cpu().numpy(), ref, f"per-row T=32 path={path}")


def test_per_row_large_tiles(glm_rows):
    bank, layer = glm_rows
    T = 512
    x = synth.make_activations(T, 6144, seed=86, device="cuda")
    lg = synth.make_logits_uniform(T, 256, seed=87, device="cuda")
    out, idx = _run(layer, x, lg)
    sample = covering_sample(idx, 96)
    ref, ri, _ = reference_layer(bank, 256, 8, 1, x, lg, sample=sample)
    assert np.array_equal(idx, ri)
    assert_close(out.cpu().numpy()[sample], ref, "per-row T=512")


@pytest.mark.parametrize("T", [4, 19, 40, 203])
def test_per_row_tiny_all_paths(T):
    """Tiny layer (H 256, I 128, 16 experts top-2 + 1 shared; too small for
    the fused decode kernel): T = 4, 19 and 40 run the small-batch kernels
    (40: two column chunks for the shared expert), T = 203 the tensor-core
    GEMM."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(256, 128, 17, seed=88, device="cuda", per_row=True)
    layer = c.MoELayer(bank, n_routed=16, top_k=2, n_shared=1)
    x = synth.make_activations(T, 256, seed=89 + T, device="cuda")
    lg = synth.make_logits_normal(T, 16, seed=90 + T, device="cuda")
    out, idx = _run(layer, x, lg)
    ref, ri, _ = reference_layer(bank, 16, 2, 1, x, lg)
    assert np.array_equal(idx, ri)
    assert_close(out.cpu().numpy(), ref, f"per-row tiny T={T}")


def test_per_row_noalloc(glm_rows):
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank, layer = glm_rows
    x = synth.make_activations(2, 6144, seed=91, device="cuda")
    lg = synth.make_logits_normal(2, 256, seed=92, device="cuda")
    out = torch.empty(2, 6144, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    c.coli_moe_layer_noalloc(layer.desc, 2, x, lg, None, out, c.COLI_OUT_F32, status_out=status)
    torch.cuda.synchronize()
    assert int(status.item()) == c.COLI_OK
    ref, _, _ = reference_layer(bank, 256, 8, 1, x, lg)
    assert_close(out.cpu().numpy(), ref, "per-row noalloc")
