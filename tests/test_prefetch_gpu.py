"""coli_moe_prefetch (router-lookahead L2 prefetch): it only warms L2, so a
layer call made while it runs on a second stream must give the oracle's
result; a routing with an index outside [0, E) is reported in the status
word; a zero budget prefetches nothing and reports nothing."""
import numpy as np
import pytest
import torch

from gpu_util import assert_close, reference_layer, requires_gpu
from int4_routed_expert_coli_b200 import synth

pytestmark = [pytest.mark.gpu, requires_gpu]


def test_prefetch_beside_a_layer_call():
    from int4_routed_expert_coli_b200 import coli_moe as c
    H, I, E, k, T = 6144, 2048, 256, 8, 64
    banks = [synth.make_expert_bank(H, I, E + 1, seed=95 + l, device="cuda") for l in range(2)]
    layers = [c.MoELayer(b, n_routed=E, top_k=k, n_shared=1) for b in banks]
    _, lg = synth.zipf_routing(T, E, k, steps=2, seed=96)
    prev = torch.from_numpy(np.argsort(-lg[0], axis=1)[:, :k].astype(np.int32)).cuda()
    x = synth.make_activations(T, H, seed=97, device="cuda")
    lg1 = torch.from_numpy(lg[1]).cuda()
    ws0, ws1 = layers[0].workspace(T), layers[1].workspace(T)
    pf_ws = torch.zeros(c.COLI_WS_HEADER_BYTES, dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    start = torch.cuda.Event()
    start.record(main)
    side.wait_event(start)
    c.coli_moe_prefetch(layers[1].handle, T, k, prev, 96 << 20, pf_ws, side)
    out0 = layers[0].layer(x, logits=lg1, ws=ws0)          # runs beside the prefetch
    out1 = layers[1].layer(x, logits=lg1, ws=ws1)          # the layer that was prefetched
    torch.cuda.synchronize()
    assert c.coli_moe_get_status(pf_ws) == c.COLI_OK
    assert c.coli_moe_get_status(ws0) == c.COLI_OK and c.coli_moe_get_status(ws1) == c.COLI_OK
    sample = np.arange(0, T, 8)
    for l, out in enumerate((out0, out1)):
        ref, _, _ = reference_layer(banks[l], E, k, 1, x, lg1, sample=sample)
        assert_close(out.cpu().numpy()[sample], ref, f"layer {l} beside a prefetch")


def test_prefetch_reports_bad_index_and_zero_budget_is_quiet():
    from int4_routed_expert_coli_b200 import coli_moe as c
    bank = synth.make_expert_bank(256, 128, 17, seed=98, device="cuda")
    layer = c.MoELayer(bank, n_routed=16, top_k=2, n_shared=1)
    ws = torch.zeros(c.COLI_WS_HEADER_BYTES, dtype=torch.uint8, device="cuda")
    good = torch.tensor([[0, 5], [15, 3]], dtype=torch.int32, device="cuda")
    c.coli_moe_prefetch(layer.handle, 2, 2, good, 0, ws)
    assert c.coli_moe_get_status(ws) == c.COLI_OK
    bad = torch.tensor([[0, 16], [1, 2]], dtype=torch.int32, device="cuda")
    c.coli_moe_prefetch(layer.handle, 2, 2, bad, 1 << 30, ws)
    assert c.coli_moe_get_status(ws) == c.COLI_ERR_BAD_INDEX
    assert c.coli_moe_prefetch(layer.handle, -1, 2, good, 0, ws,
                               raise_on_error=False) == c.COLI_ERR_INVALID_ARG
