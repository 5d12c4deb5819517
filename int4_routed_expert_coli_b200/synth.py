"""Seeded synthetic inputs for the routed-expert MoE layer.

This module is the only code shared by the CUDA path and the CPU oracle's
tests.  It draws random numbers and lays them out in the storage formats of
the layer's inputs; it computes nothing of the layer itself (no routing, no
dequantisation, no matmul, no activation).

Formats (the layer's inputs, as the C-ABI header documents them):

* expert matrices ``gate_q``/``up_q`` ``[I][H/2]`` and ``down_q`` ``[H][I/2]``
  are uint8, two signed int4 codes per byte along the reduction dimension;
  a uniformly random byte gives two independent codes uniform over [-8, 7].
* scales ``gate_s``/``up_s`` ``[I][H/64]`` and ``down_s`` ``[H][I/64]`` are
  bf16, drawn from U(0.005, 0.02) in fp32 and rounded to bf16 (RNE); in the
  per-row format (``per_row=True``) one scale per row, ``[I][1]`` and
  ``[H][1]``, drawn the same way.
* activations ``x`` ``[T][H]`` are bf16 drawn from N(0, 1).
* router logits ``[T][E]`` are fp32; the router weight ``[E][H]`` is fp32
  N(0, 0.02).

The workloads follow the pages' GLM-5.2 numbers (256 routed experts, 8 + 1
active per layer, about 19 MB per int4 expert: "zhichai.net/topic/178503686",
section on MoE sparsity; "yunpan.plus/t/30351-1-1", memory-tier section).

Zipf-skewed routing (``zipf_routing``) realises a chosen expert set through
logits: chosen experts get 3 + |N(0,1)|, the rest min(N(0,1), 2.5), so any
correct top-k over those logits returns exactly the drawn set.  The 71.6 %
repeat probability is the pages' one-layer-ahead predictability figure
("yunpan.plus/t/30351-1-1", memory-tier section), reused as a step-to-step
repeat rate.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

GROUP = 64  # K elements per bf16 scale (the gs64 container)


@dataclasses.dataclass
class ExpertBank:
    """All experts of one layer: ``n`` = routed + shared, shared last.

    Each tensor's leading dim is the expert; one expert's matrix is a
    contiguous slice, so per-expert device pointers are plain offsets.
    """

    hidden: int
    inter: int
    n: int
    gate_q: torch.Tensor  # [n][I][H/2]  uint8
    up_q: torch.Tensor    # [n][I][H/2]  uint8
    down_q: torch.Tensor  # [n][H][I/2]  uint8
    gate_s: torch.Tensor  # [n][I][H/64] bf16
    up_s: torch.Tensor    # [n][I][H/64] bf16
    down_s: torch.Tensor  # [n][H][I/64] bf16
    per_row: bool = False  # scales [rows][1]: one per row instead of one per 64 codes

    def expert_numpy(self, e: int) -> dict:
        """Copy expert ``e`` to host numpy arrays (scales as raw bf16 bits;
        "group" 64 for gs64, 0 for one scale per row)."""
        out = {}
        for name in ("gate_q", "up_q", "down_q"):
            out[name] = getattr(self, name)[e].cpu().numpy()
        for name in ("gate_s", "up_s", "down_s"):
            out[name] = getattr(self, name)[e].cpu().view(torch.int16).numpy().view(np.uint16)
        out["group"] = 0 if self.per_row else GROUP
        return out

    def nbytes_per_expert(self) -> int:
        h, i = self.hidden, self.inter
        if self.per_row:
            return 3 * h * i // 2 + (2 * i + h) * 2
        return 3 * h * i // 2 + 3 * (h * i // GROUP) * 2


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


# Generator settings of the stacked-layers workload.  Untrained experts drawn
# as for a single layer make x_(l+1) = x_l + MoE_l(x_l) blow up: codes
# uniform over [-8, 7] have mean -1/2, so every layer adds the same offset to
# all H elements and the next layer's dot products grow with it, and U(.005,
# .02) scales multiply the stream's RMS by ~50 per layer.  Zero-mean codes
# over [-7, 7] and one eighth of the scales keep every layer's update near
# 7 % of an O(1) stream.
STACK_SCALE_RANGE = (0.005 / 8, 0.02 / 8)
STACK_CODE_RANGE = (-7, 7)


def make_expert_bank(hidden: int, inter: int, n_experts: int, seed: int,
                     device="cpu", scale_range=(0.005, 0.02),
                     code_range=(-8, 7), per_row: bool = False) -> ExpertBank:
    """Random int4 experts: codes uniform over code_range (default [-8, 7]:
    every nibble value), scales U(scale_range) rounded to bf16 (default
    U(.005, .02)), one per 64 codes of a row (gs64) or, with per_row, one per
    row."""
    if hidden % (2 * GROUP) or inter % (2 * GROUP):
        raise ValueError("hidden and inter must be multiples of 128")
    g = _gen(seed, device)
    kw = dict(dtype=torch.uint8, device=device)

    def codes(rows, cols):
        if tuple(code_range) == (-8, 7):  # all 16 nibble values: uniform bytes
            return torch.empty(n_experts, rows, cols, **kw).random_(0, 256, generator=g)
        lo, hi = code_range
        q = torch.empty(2, n_experts, rows, cols, **kw).random_(0, hi - lo + 1, generator=g)
        q = (q.to(torch.int16) + lo).bitwise_and(0xF).to(torch.uint8)
        return q[0] | (q[1] << 4)

    gate_q = codes(inter, hidden // 2)
    up_q = codes(inter, hidden // 2)
    down_q = codes(hidden, inter // 2)

    def scales(rows, cols):
        s = torch.empty(n_experts, rows, cols, dtype=torch.float32, device=device)
        s.uniform_(scale_range[0], scale_range[1], generator=g)
        return s.to(torch.bfloat16)

    gate_s = scales(inter, 1 if per_row else hidden // GROUP)
    up_s = scales(inter, 1 if per_row else hidden // GROUP)
    down_s = scales(hidden, 1 if per_row else inter // GROUP)
    return ExpertBank(hidden, inter, n_experts, gate_q, up_q, down_q, gate_s, up_s, down_s,
                      per_row)


def make_activations(tokens: int, hidden: int, seed: int, device="cpu") -> torch.Tensor:
    """x [T][H] bf16, N(0, 1)."""
    g = _gen(seed, device)
    return torch.randn(tokens, hidden, generator=g, device=device).to(torch.bfloat16)


def make_router_weight(n_routed: int, hidden: int, seed: int, device="cpu") -> torch.Tensor:
    """W_r [E][H] fp32, N(0, 0.02)."""
    g = _gen(seed, device)
    return torch.randn(n_routed, hidden, generator=g, device=device) * 0.02


def make_logits_normal(tokens: int, n_routed: int, seed: int, device="cpu") -> torch.Tensor:
    """Router logits [T][E] fp32, N(0, 1)."""
    g = _gen(seed, device)
    return torch.randn(tokens, n_routed, generator=g, device=device)


def make_logits_uniform(tokens: int, n_routed: int, seed: int, device="cpu") -> torch.Tensor:
    """Router logits [T][E] fp32, U[0, 1)."""
    g = _gen(seed, device)
    return torch.rand(tokens, n_routed, generator=g, device=device)


def make_residual(tokens: int, hidden: int, seed: int, dtype=torch.float32,
                  device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(tokens, hidden, generator=g, device=device).to(dtype)


def zipf_routing(tokens: int, n_routed: int, top_k: int, steps: int, seed: int,
                 exponent: float = 1.1, repeat: float = 0.716):
    """Zipf-skewed expert sets per step and logits that realise them.

    Returns ``(sets, logits)``: ``sets[s]`` is an int array [T][k] of the drawn
    experts (unordered), ``logits[s]`` a float32 array [T][E] whose top-k per
    row is exactly that set.
    """
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_routed)               # Zipf rank -> expert id
    p = np.arange(1, n_routed + 1, dtype=np.float64) ** (-exponent)
    p /= p.sum()

    def draw(exclude):
        while True:
            e = int(perm[rng.choice(n_routed, p=p)])
            if e not in exclude:
                return e

    sets, logits = [], []
    prev = None
    for s in range(steps):
        cur = np.empty((tokens, top_k), dtype=np.int64)
        for t in range(tokens):
            picked: list[int] = []
            for j in range(top_k):
                if prev is not None and rng.random() < repeat:
                    cand = int(prev[t, j])
                    if cand not in picked:
                        picked.append(cand)
                        continue
                excl = set(picked) | (set(prev[t].tolist()) if prev is not None else set())
                if len(excl) >= n_routed:
                    excl = set(picked)
                picked.append(draw(excl))
            cur[t] = picked
        lg = np.minimum(rng.standard_normal((tokens, n_routed)), 2.5)
        for t in range(tokens):
            lg[t, cur[t]] = 3.0 + np.abs(rng.standard_normal(top_k))
        sets.append(cur)
        logits.append(lg.astype(np.float32))
        prev = cur
    return sets, logits
