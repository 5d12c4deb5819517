"""The expert-parallel layer step's GPU building blocks, at world size 1
(this pool gives one GPU per run): routing, the top-1 FFN over the rank's
expert partition on the rows it received, the shared expert on a one-expert
handle, and the fixed-order combine kernel (coli_moe_combine_rows), against
the oracle layer."""
import numpy as np
import pytest
import torch

from gpu_util import assert_close, reference_layer, requires_gpu
from int4_routed_expert_coli_b200 import synth

pytestmark = [pytest.mark.gpu, requires_gpu]


@pytest.mark.parametrize("H,I,E,k,T,out_bf16", [(256, 128, 16, 2, 5, False),
                                                (6144, 2048, 256, 8, 4, True)])
def test_ep_step_world_one_matches_oracle(H, I, E, k, T, out_bf16):
    from int4_routed_expert_coli_b200 import coli_moe as c
    from int4_routed_expert_coli_b200 import expert_parallel as ep
    bank = synth.make_expert_bank(H, I, E + 1, seed=90 + T, device="cuda")
    starts = ep.partition(E, 1)
    loc = ep.LocalExperts(bank, E, k, 1, starts, 0)
    x = synth.make_activations(T, H, seed=91, device="cuda")
    lg = synth.make_logits_normal(T, E, seed=92, device="cuda")
    dt = torch.bfloat16 if out_bf16 else torch.float32
    res = synth.make_residual(T, H, seed=93, dtype=dt, device="cuda")
    od = c.COLI_OUT_BF16 if out_bf16 else c.COLI_OUT_F32
    out, idx, w = ep.ep_layer_step(x, lg, k, starts, 1, loc.route, loc.local_ffn, loc.shared_out,
                                   lambda r, s, rr: loc.combine(r, s, rr, od), residual=res)
    torch.cuda.synchronize()
    ref, ri, _ = reference_layer(bank, E, k, 1, x, lg, residual=res)
    assert np.array_equal(idx.cpu().numpy(), ri)
    if out_bf16:
        ref = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert_close(out.double().cpu().numpy(), ref, "expert-parallel step, one rank")


def test_combine_rows_fixed_order_exact():
    """out = ((sum_j rows[t*k+j]) + shared) + residual in fp32, that order:
    values chosen so another order would round differently."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    T, k, H = 3, 2, 8
    rows = torch.zeros(T * k, H, device="cuda")
    rows[:, 0] = torch.tensor([1.0, 2.0 ** -24, 1.0, 2.0 ** -24, 3.0, 5.0], device="cuda")
    shared = torch.zeros(T, H, device="cuda")
    shared[:, 0] = torch.tensor([2.0 ** -24, 1.0, -4.0], device="cuda")
    res = torch.ones(T, H, device="cuda")
    res[:, 0] = 0.0
    out = torch.empty(T, H, device="cuda")
    c.coli_moe_combine_rows(T, k, H, rows, shared, res, out, c.COLI_OUT_F32)
    torch.cuda.synchronize()
    # token 0: (1 + 2^-24) rounds to 1, then + 2^-24 rounds to 1 again; summing
    # the two small terms first would give 1 + 2^-23
    assert out[:, 0].cpu().numpy().tolist() == [1.0, 2.0, 4.0]
    assert torch.all(out[:, 1:] == 1.0)
