"""The 16-layer stack (x_(l+1) = x_l + MoE_l(x_l), bf16 stream, residual
added by the combine), teacher-forced: every layer's bf16 output is compared
with the oracle run on the GPU's own input to that layer, on sampled tokens,
so differences do not compound through the stack.  GLM-5.2 layer shape, 32
routed experts per layer (top-8, Zipf routing) + 1 shared, T = 64, two steps;
the stack's generator settings (zero-mean codes, one eighth of the scales)
keep the residual stream O(1) through untrained layers."""
import numpy as np
import pytest
import torch

from int4_routed_expert_coli_b200 import synth
from gpu_util import assert_close, reference_layer

pytestmark = pytest.mark.gpu

H, I, E, K, NSH, T, LAYERS, STEPS = 6144, 2048, 32, 8, 1, 64, 16, 2
SAMPLE = np.array([3, 40], dtype=np.int64)  # tokens checked per layer and step


def test_stack_teacher_forced():
    from int4_routed_expert_coli_b200 import coli_moe as c
    banks = [synth.make_expert_bank(H, I, E + NSH, seed=500 + l, device="cuda",
                                    scale_range=synth.STACK_SCALE_RANGE,
                                    code_range=synth.STACK_CODE_RANGE)
             for l in range(LAYERS)]
    layers = [c.MoELayer(b, n_routed=E, top_k=K, n_shared=NSH) for b in banks]
    lgs = [synth.zipf_routing(T, E, K, steps=STEPS, seed=900 + l)[1] for l in range(LAYERS)]
    ws = layers[0].workspace(T)
    for s in range(STEPS):
        x = synth.make_activations(T, H, seed=77 + s, device="cuda")
        for l in range(LAYERS):
            lg = torch.from_numpy(lgs[l][s]).cuda()
            out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
            c.coli_moe_layer(layers[l].handle, T, x, lg, None, x, out, c.COLI_OUT_BF16,
                             None, None, ws)
            assert c.coli_moe_get_status(ws) == c.COLI_OK
            ref, _, _ = reference_layer(banks[l], E, K, NSH, x, lg, residual=x, sample=SAMPLE)
            ref_bf16 = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
            got = out[torch.from_numpy(SAMPLE).cuda()].double().cpu().numpy()
            assert_close(got, ref_bf16, f"step {s} layer {l}")
            x = out  # the next layer reads this layer's own output
