"""Failure detection on the GPU without faulting it: a staged tile that is
never filled makes the consumers' bounded wait (about one second) run out;
the kernel winds down, the status word reads COLI_ERR_TIMEOUT, and the
context stays usable for the next call."""
import numpy as np
import pytest
import torch

from gpu_util import assert_close, reference_layer, requires_gpu
from int4_routed_expert_coli_b200 import synth

pytestmark = [pytest.mark.gpu, requires_gpu]


def test_withheld_stage_times_out_and_context_survives():
    """The streaming kernels (forced: the tiny shape would take the grouped
    GEMM by default)."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    H, I, E, k, T = 256, 128, 16, 2, 4
    bank = synth.make_expert_bank(H, I, E + 1, seed=21, device="cuda")
    layer = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=1, prefill_min_tokens=10 ** 6)
    x = synth.make_activations(T, H, seed=22, device="cuda")
    lg = synth.make_logits_normal(T, E, seed=23, device="cuda")
    ws = layer.workspace(T)
    assert c.coli_moe_debug_inject(c.COLI_INJECT_WITHHOLD_STAGE) == c.COLI_OK
    try:
        layer.layer(x, logits=lg, ws=ws)
    finally:
        c.coli_moe_debug_inject(0)
    assert c.coli_moe_get_status(ws) == c.COLI_ERR_TIMEOUT
    # the context is still usable and the next call is correct
    c.coli_moe_workspace_clear(ws)
    out = layer.layer(x, logits=lg, ws=ws)
    assert c.coli_moe_get_status(ws) == c.COLI_OK
    ref, _, _ = reference_layer(bank, E, k, 1, x, lg)
    assert_close(out.cpu().numpy(), ref, "after timeout")


def test_bad_union_input_reports_not_faults():
    from int4_routed_expert_coli_b200 import coli_moe as c
    H, I, E, k, T = 256, 128, 16, 2, 4
    bank = synth.make_expert_bank(H, I, E + 1, seed=24, device="cuda")
    layer = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=1)
    x = synth.make_activations(T, H, seed=25, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    w = torch.full((T, k), 0.5, device="cuda")
    counts = torch.zeros(E, **i32)
    offsets = torch.zeros(E + 1, **i32)
    offsets[1:] = 8
    offsets[0] = 0
    counts[0] = 8
    pairs = torch.arange(T * k, **i32)
    pairs[3] = 10 ** 6                      # out of range pair id
    active = torch.full((E,), -1, **i32)
    active[0] = 0
    na = torch.tensor([1], **i32)
    ws = layer.workspace(T)
    out = torch.empty(T, H, device="cuda")
    c.coli_moe_ffn(layer.handle, T, x, w, counts, offsets, pairs, active, na, None, out,
                   c.COLI_OUT_F32, ws)
    assert c.coli_moe_get_status(ws) == c.COLI_ERR_BAD_INDEX
    na.fill_(5000)                          # n_active beyond E
    c.coli_moe_workspace_clear(ws)
    c.coli_moe_ffn(layer.handle, T, x, w, counts, offsets, pairs, active, na, None, out,
                   c.COLI_OUT_F32, ws)
    assert c.coli_moe_get_status(ws) == c.COLI_ERR_BAD_INDEX


def test_withheld_stage_in_fused_decode_times_out():
    """GLM-5.2 shape, one token: the fused decode kernel (one persistent
    launch for gate/up, down and combine) with one staged tile withheld; the
    stalled consumers and every down item waiting on that expert's h give up
    after their bounded waits."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(6144, 2048, 257, seed=26, device="cuda")
    layer = c.MoELayer(bank, n_routed=256, top_k=8, n_shared=1)
    x = synth.make_activations(1, 6144, seed=27, device="cuda")
    lg = synth.make_logits_normal(1, 256, seed=28, device="cuda")
    ws = layer.workspace(1)
    assert c.coli_moe_debug_inject(c.COLI_INJECT_WITHHOLD_STAGE) == c.COLI_OK
    try:
        layer.layer(x, logits=lg, ws=ws)
    finally:
        c.coli_moe_debug_inject(0)
    assert c.coli_moe_get_status(ws) == c.COLI_ERR_TIMEOUT
    c.coli_moe_workspace_clear(ws)
    out = layer.layer(x, logits=lg, ws=ws)
    assert c.coli_moe_get_status(ws) == c.COLI_OK
    ref, _, _ = reference_layer(bank, 256, 8, 1, x, lg)
    assert_close(out.cpu().numpy(), ref, "after timeout")


def test_fused_decode_refused_launch_takes_the_streaming_path():
    """GLM-5.2 shape, T = 1 and T = 4: when the fused decode kernel's
    cooperative launch is refused (its grid of one CTA per SM cannot be
    resident at once, as on a partitioned GPU; forced here by the test hook),
    the call runs on the streaming kernels and still matches the oracle, for
    the layer call and for the FFN call on a prepared union."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(6144, 2048, 257, seed=29, device="cuda")
    layer = c.MoELayer(bank, n_routed=256, top_k=8, n_shared=1)
    for T in (1, 4):
        x = synth.make_activations(T, 6144, seed=30 + T, device="cuda")
        lg = synth.make_logits_normal(T, 256, seed=40 + T, device="cuda")
        ws = layer.workspace(T)
        assert c.coli_moe_debug_inject(c.COLI_INJECT_NOT_RESIDENT) == c.COLI_OK
        try:
            out = layer.layer(x, logits=lg, ws=ws)
        finally:
            c.coli_moe_debug_inject(0)
        assert c.coli_moe_get_status(ws) == c.COLI_OK
        ref, _, _ = reference_layer(bank, 256, 8, 1, x, lg)
        assert_close(out.cpu().numpy(), ref, f"refused fused launch, layer T={T}")

        # the FFN entry point on a prepared union takes the same fallback
        k, E = 8, 256
        idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, k, dtype=torch.float32, device="cuda")
        c.coli_moe_route(T, E, k, lg, idx, w)
        i32 = dict(dtype=torch.int32, device="cuda")
        counts, offsets = torch.empty(E, **i32), torch.empty(E + 1, **i32)
        pairs, active, na = torch.empty(T * k, **i32), torch.empty(E, **i32), torch.empty(1, **i32)
        c.coli_moe_union(T, E, k, idx, counts, offsets, pairs, active, na)
        out2 = torch.empty(T, 6144, dtype=torch.float32, device="cuda")
        assert c.coli_moe_debug_inject(c.COLI_INJECT_NOT_RESIDENT) == c.COLI_OK
        try:
            c.coli_moe_ffn(layer.handle, T, x, w, counts, offsets, pairs, active, na, None,
                           out2, c.COLI_OUT_F32, ws)
        finally:
            c.coli_moe_debug_inject(0)
        assert c.coli_moe_get_status(ws) == c.COLI_OK
        assert_close(out2.cpu().numpy(), ref, f"refused fused launch, ffn T={T}")
