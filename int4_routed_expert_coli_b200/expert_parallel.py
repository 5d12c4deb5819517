"""Expert-parallel layer step: the routed experts partitioned over ranks, one
process per GPU.

The pages describe a local cluster in which a worker receives one layer's
routed batch-union and runs the FFN ("yunpan.plus/t/30351-1-1", capability
three, local cluster paragraph), and a multi-GPU run that keeps every expert
resident by spreading the experts over the cards (same page, the 6 x RTX 5090
figures).  This module is that split over torch.distributed:

1. every rank routes its own tokens (``coli_moe_route`` on the GPU);
2. dispatch: each (token, slot) pair goes to the rank that owns its expert:
   one all-to-all of the bf16 token rows, of the owner-local expert index and
   of the gate weight, into buffers on the receiving rank;
3. each rank runs its own experts over the rows it received as one batch
   (``coli_moe_union`` + ``coli_moe_ffn`` with top-1 over its local experts:
   every returned row is w * FFN_e(x), one read of each local expert for all
   rows that need it);
4. return: one all-to-all of those fp32 rows back, in the reverse split;
5. each rank runs the shared experts on its own tokens and sums, per token,
   the routed rows in slot order, then the shared output, then the residual
   (``coli_moe_combine_rows``).

Steps 2 and 4 are the only collectives; the rest runs in the library's
kernels on each rank.  Every rank takes the same collective steps in the same
order.  The split sizes of an all-to-all must be known on the host, so the
routing is read back once per layer step (a device-to-host copy of T*k
indices).  The exchange copies into local buffers: no kernel reads another
GPU's memory.

The compute steps are passed in as functions, so the same plumbing runs with
the library's kernels on GPUs (``LocalExperts``) or with any other per-rank
expert evaluation (the CPU tests use the oracle on gloo ranks).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


def partition(n_routed: int, world: int) -> np.ndarray:
    """Contiguous expert ranges: rank r owns experts [starts[r], starts[r+1]);
    sizes differ by at most one."""
    if world < 1 or n_routed < world:
        raise ValueError("need at least one routed expert per rank")
    return np.array([r * n_routed // world for r in range(world + 1)], dtype=np.int64)


def owner_of(experts: np.ndarray, starts: np.ndarray) -> np.ndarray:
    """Rank that owns each expert index."""
    return np.searchsorted(starts, np.asarray(experts), side="right") - 1


@dataclasses.dataclass
class DispatchPlan:
    order: np.ndarray        # [T*k] pair ids p = t*k + j, grouped by owner rank, ascending inside
    send_counts: np.ndarray  # [world] pairs sent to each rank
    local_eid: np.ndarray    # [T*k] owner-local expert index of each pair, in `order`


def plan_dispatch(idx: np.ndarray, starts: np.ndarray) -> DispatchPlan:
    """Which pairs go to which rank, from the routing idx [T][k]."""
    idx = np.asarray(idx, dtype=np.int64)
    world = len(starts) - 1
    flat = idx.reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= starts[-1]):
        raise ValueError("expert index outside [0, E)")
    dest = owner_of(flat, starts)
    order = np.argsort(dest, kind="stable")  # stable: ascending pair id within a rank
    send_counts = np.bincount(dest, minlength=world).astype(np.int64)
    local_eid = (flat[order] - starts[dest[order]]).astype(np.int32)
    return DispatchPlan(order=order, send_counts=send_counts, local_eid=local_eid)


def _exchange(t: torch.Tensor, send_counts, recv_counts, world: int, group=None) -> torch.Tensor:
    """all_to_all of the rows of t (split by send_counts along dim 0)."""
    if world == 1:
        return t.clone()
    import torch.distributed as dist
    out = torch.empty((int(sum(recv_counts)),) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_to_all_single(out, t.contiguous(), output_split_sizes=[int(c) for c in recv_counts],
                           input_split_sizes=[int(c) for c in send_counts], group=group)
    return out


def _exchange_counts(send_counts: np.ndarray, world: int, device, group=None) -> np.ndarray:
    if world == 1:
        return send_counts.copy()
    import torch.distributed as dist
    s = torch.tensor(send_counts, dtype=torch.int64, device=device)
    r = torch.empty_like(s)
    dist.all_to_all_single(r, s, group=group)
    return r.cpu().numpy()


def ep_layer_step(x: torch.Tensor, logits: torch.Tensor, k: int, starts: np.ndarray,
                  world: int, route_fn, local_ffn_fn, shared_fn, combine_fn, residual=None,
                  group=None):
    """One layer step of this rank's tokens with the experts partitioned as
    `starts` over `world` ranks (every rank calls it, with its own tokens).

      route_fn(logits) -> (idx [T][k] int tensor, w [T][k] float tensor)
      local_ffn_fn(rows [n][H] bf16, local_eid [n] int32, w [n]) -> [n][H]
          (w * FFN_e(row) for this rank's expert e)
      shared_fn(x) -> [T][H] (the shared experts' output) or None
      combine_fn(rows [T*k][H] in slot order, shared, residual) -> out [T][H]
    """
    T, H = x.shape
    dev = x.device
    idx, w = route_fn(logits)
    plan = plan_dispatch(idx.detach().cpu().numpy(), starts)
    order_t = torch.from_numpy(plan.order).to(dev)
    recv_counts = _exchange_counts(plan.send_counts, world, dev, group)

    # dispatch: token rows (as bytes), owner-local expert ids, gate weights
    tok = order_t // k
    rows_send = x.index_select(0, tok).contiguous().view(torch.uint8)
    w_send = w.reshape(-1).index_select(0, order_t).contiguous()
    eid_send = torch.from_numpy(plan.local_eid).to(dev)
    rows_recv = _exchange(rows_send, plan.send_counts, recv_counts, world, group)
    w_recv = _exchange(w_send, plan.send_counts, recv_counts, world, group)
    eid_recv = _exchange(eid_send, plan.send_counts, recv_counts, world, group)

    # this rank's experts over everything it received
    y_recv = local_ffn_fn(rows_recv.view(x.dtype).view(-1, H), eid_recv, w_recv)

    # return in the reverse split, then back into slot order
    y_back = _exchange(y_recv.contiguous(), recv_counts, plan.send_counts, world, group)
    rows = torch.empty((T * k, H), dtype=y_back.dtype, device=dev)
    rows.index_copy_(0, order_t, y_back)
    return combine_fn(rows, shared_fn(x), residual), idx, w


class LocalExperts:
    """This rank's share of a layer on its GPU, for ``ep_layer_step``: a
    library handle over its routed experts (top-1, no shared expert) and one
    over the shared expert (a single routed expert, top-1, zero logits: every
    token takes it with weight 1)."""

    def __init__(self, bank, n_routed: int, k: int, n_shared: int, starts: np.ndarray,
                 rank: int):
        from . import coli_moe as c
        if n_shared != 1:
            raise ValueError("the expert-parallel step supports one shared expert")
        self.c = c
        self.k = k
        self.H = bank.hidden
        lo, hi = int(starts[rank]), int(starts[rank + 1])
        self.n_local = hi - lo
        self.local = c.MoELayer(_sub_bank(bank, lo, hi), n_routed=self.n_local, top_k=1,
                                n_shared=0)
        self.shared = c.MoELayer(_sub_bank(bank, n_routed, n_routed + 1), n_routed=1, top_k=1,
                                 n_shared=0)
        self.E = n_routed

    def route(self, logits):
        T = logits.shape[0]
        idx = torch.empty(T, self.k, dtype=torch.int32, device=logits.device)
        w = torch.empty(T, self.k, dtype=torch.float32, device=logits.device)
        self.c.coli_moe_route(T, self.E, self.k, logits, idx, w)
        return idx, w

    def local_ffn(self, rows, eid, w):
        c, n = self.c, rows.shape[0]
        dev = rows.device
        out = torch.empty(n, self.H, dtype=torch.float32, device=dev)
        if n == 0:
            return out
        E = self.n_local
        i32 = dict(dtype=torch.int32, device=dev)
        counts, offsets = torch.empty(E, **i32), torch.empty(E + 1, **i32)
        pairs, active, na = torch.empty(n, **i32), torch.empty(E, **i32), torch.empty(1, **i32)
        c.coli_moe_union(n, E, 1, eid.view(n, 1).contiguous(), counts, offsets, pairs, active, na)
        ws = self.local.workspace(n, dev)
        c.coli_moe_ffn(self.local.handle, n, rows.contiguous(), w.float().contiguous(), counts,
                       offsets, pairs, active, na, None, out, c.COLI_OUT_F32, ws)
        return out

    def shared_out(self, x):
        T = x.shape[0]
        zeros = torch.zeros(T, 1, dtype=torch.float32, device=x.device)
        return self.shared.layer(x, logits=zeros, ws=self.shared.workspace(T, x.device))

    def combine(self, rows, shared, residual, out_dtype=None):
        c = self.c
        T = shared.shape[0]
        od = c.COLI_OUT_F32 if out_dtype is None else out_dtype
        dt = torch.float32 if od == c.COLI_OUT_F32 else torch.bfloat16
        out = torch.empty(T, self.H, dtype=dt, device=rows.device)
        c.coli_moe_combine_rows(T, self.k, self.H, rows, shared, residual, out, od)
        return out


def _sub_bank(bank, lo, hi):
    from .synth import ExpertBank
    return ExpertBank(bank.hidden, bank.inter, hi - lo, bank.gate_q[lo:hi], bank.up_q[lo:hi],
                      bank.down_q[lo:hi], bank.gate_s[lo:hi], bank.up_s[lo:hi],
                      bank.down_s[lo:hi], bank.per_row)
