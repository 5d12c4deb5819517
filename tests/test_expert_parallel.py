"""Expert-parallel plumbing (experts partitioned over ranks, all-to-all
dispatch and return) on CPU: gloo ranks at world size 2 and 3, each rank's
expert evaluation done by the oracle, compared with the single-rank oracle
layer on the same tokens; plus the host-side dispatch plan on its own."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_partition_and_owner():
    from int4_routed_expert_coli_b200 import expert_parallel as ep
    st = ep.partition(16, 3)
    assert st.tolist() == [0, 5, 10, 16]
    assert ep.owner_of(np.arange(16), st).tolist() == [0] * 5 + [1] * 5 + [2] * 6
    with pytest.raises(ValueError):
        ep.partition(2, 3)


def test_plan_dispatch_groups_pairs_by_owner():
    from int4_routed_expert_coli_b200 import expert_parallel as ep
    st = ep.partition(8, 2)            # rank 0: experts 0-3, rank 1: 4-7
    idx = np.array([[5, 1], [0, 7], [4, 3]])
    plan = ep.plan_dispatch(idx, st)
    # pairs p = t*k + j: owners 1,0,0,1,1,0 -> rank 0 gets p 1,2,5; rank 1 gets 0,3,4
    assert plan.order.tolist() == [1, 2, 5, 0, 3, 4]
    assert plan.send_counts.tolist() == [3, 3]
    assert plan.local_eid.tolist() == [1, 0, 3, 1, 3, 0]
    with pytest.raises(ValueError):
        ep.plan_dispatch(np.array([[8, 0]]), st)


def _rank_main(rank, world, port, q, T, seed_base):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    import oracle
    from int4_routed_expert_coli_b200 import expert_parallel as ep
    from int4_routed_expert_coli_b200 import synth
    from gpu_util import bits
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    try:
        H, I, E, k = 256, 128, 16, 2
        bank = synth.make_expert_bank(H, I, E + 1, seed=31, device="cpu")
        experts = [bank.expert_numpy(e) for e in range(E + 1)]
        starts = ep.partition(E, world)
        lo, hi = int(starts[rank]), int(starts[rank + 1])
        x = synth.make_activations(T, H, seed=seed_base + rank, device="cpu")
        lg = synth.make_logits_normal(T, E, seed=seed_base + 100 + rank, device="cpu")
        res = synth.make_residual(T, H, seed=seed_base + 200 + rank, device="cpu").double()

        def route_fn(logits):
            idx, w = oracle.route(logits.numpy(), k)
            return torch.from_numpy(idx), torch.from_numpy(w)

        def ffn(e, row_bf16):
            return oracle.expert_ffn(H, I, experts[e], bits_to_f64(bits(row_bf16[None]))[0])

        def local_ffn_fn(rows, eid, w):
            out = torch.zeros(rows.shape[0], H, dtype=torch.float64)
            for i in range(rows.shape[0]):
                e = lo + int(eid[i])
                assert lo <= e < hi, "a pair reached a rank that does not own its expert"
                out[i] = float(w[i]) * torch.from_numpy(ffn(e, rows[i]))
            return out

        def shared_fn(xx):
            return torch.stack([torch.from_numpy(ffn(E, xx[t])) for t in range(xx.shape[0])])

        def combine_fn(rows, shared, residual):
            out = rows.view(-1, k, H)[:, 0].clone()
            for j in range(1, k):
                out += rows.view(-1, k, H)[:, j]
            return out + shared + residual

        out, idx, w = ep.ep_layer_step(x, lg, k, starts, world, route_fn, local_ffn_fn, shared_fn,
                                       combine_fn, residual=res)
        ref = oracle.layer(H, I, E, k, 1, oracle.Experts(experts), bits(x), idx.numpy(),
                           w.numpy(), residual=res.numpy(), n_threads=1)
        err = float(np.abs(out.numpy() - ref).max() / np.abs(ref).max())
        q.put((rank, err, int(idx.numel())))
    finally:
        dist.destroy_process_group()


def bits_to_f64(b):
    b = np.asarray(b, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


@pytest.mark.parametrize("world,T", [(2, 5), (3, 4)])
def test_ep_layer_step_matches_single_rank_oracle(world, T):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, T, 40 + world))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, (e, n)) for r, e, n in (q.get(timeout=300) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(got) == list(range(world))
    for r, (err, n) in got.items():
        assert n == T * 2
        assert err <= 1e-12, (r, err)
