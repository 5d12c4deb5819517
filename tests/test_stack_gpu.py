"""The 16-layer stack (x_(l+1) = x_l + MoE_l(x_l), bf16 stream, residual
added by the combine), teacher-forced: every layer's bf16 output is compared
with the oracle run on the GPU's own input to that layer, on sampled tokens,
so differences do not compound through the stack.  The stack's generator
settings (zero-mean codes, one eighth of the scales) keep the residual stream
O(1) through untrained layers.

Two cases: all 16 layers at GLM-5.2 layer shape with 32 routed experts per
layer (top-8, Zipf routing) + 1 shared; and 4 layers at the full width of the
stack workload (256 routed + 1 shared experts per layer), steps 0, 1 and 255
of the per-layer Zipf routing (step 255 after 255 steps of 71.6 % repeats)."""
import numpy as np
import pytest
import torch

from int4_routed_expert_coli_b200 import synth
from gpu_util import assert_close, reference_layer, requires_gpu

pytestmark = [pytest.mark.gpu, requires_gpu]

H, I, K, NSH, T = 6144, 2048, 8, 1, 64
SAMPLE = np.array([0, 3, 17, 26, 40, 45, 58, 63], dtype=np.int64)  # tokens checked per layer


def _run_stack(E, layers_n, steps, seed):
    from int4_routed_expert_coli_b200 import coli_moe as c
    banks = [synth.make_expert_bank(H, I, E + NSH, seed=seed + l, device="cuda",
                                    scale_range=synth.STACK_SCALE_RANGE,
                                    code_range=synth.STACK_CODE_RANGE)
             for l in range(layers_n)]
    layers = [c.MoELayer(b, n_routed=E, top_k=K, n_shared=NSH) for b in banks]
    n_steps = max(steps) + 1
    lgs = [synth.zipf_routing(T, E, K, steps=n_steps, seed=seed + 400 + l)[1]
           for l in range(layers_n)]
    ws = layers[0].workspace(T)
    for s in steps:
        x = synth.make_activations(T, H, seed=seed + 77 + s, device="cuda")
        for l in range(layers_n):
            lg = torch.from_numpy(lgs[l][s]).cuda()
            out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
            c.coli_moe_layer(layers[l].handle, T, x, lg, None, x, out, c.COLI_OUT_BF16,
                             None, None, ws)
            assert c.coli_moe_get_status(ws) == c.COLI_OK
            ref, _, _ = reference_layer(banks[l], E, K, NSH, x, lg, residual=x, sample=SAMPLE)
            ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
            got = out[torch.from_numpy(SAMPLE).cuda()].double().cpu().numpy()
            assert_close(got, ref_bf16, f"E={E} step {s} layer {l}")
            x = out  # the next layer reads this layer's own output
    del layers, banks
    torch.cuda.empty_cache()


def test_stack_teacher_forced():
    _run_stack(E=32, layers_n=16, steps=[0, 1], seed=500)


def test_stack_full_width_layers():
    _run_stack(E=256, layers_n=4, steps=[0, 1, 255], seed=7000)
