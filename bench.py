#!/usr/bin/env python
"""Benchmark of one routed int4 gs64 MoE layer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle, same workload

Default workload: GLM-5.2-shaped single-token decode (H 6144, I 2048, 256
routed experts top-8 + 1 shared, about 19 MB per int4 gs64 expert, all 257
experts resident in HBM), fresh seeded token and N(0,1) router logits every
step.  A step is one full layer call through the C ABI (route, batch-union,
gate/up, down, combine).  Inputs for every step sit in HBM before the timed
region; L2 is flushed between timed steps by reading a 256 MiB buffer (a
read leaves no dirty lines behind to be written back during the next step)
and each step is timed alone with CUDA events on the launching stream.

Multi-GPU (torchrun): every rank runs its own replica on its own token
stream (no data-path collective); the timed total is the max over ranks and
`value` counts the tokens of all ranks ("scaling": "weak").

Without --workload the run measures every workload: the decode line is the
headline and the others (verify4, batch32, prefill, stack) are attached to it
under "workloads", each with its own roofline, CPU baseline, end-to-end
figure and clock record.  --workload NAME measures that one alone.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int4_routed_expert_coli_b200 import synth  # noqa: E402

GLM = dict(H=6144, I=2048, E=256, k=8, n_shared=1)
WORKLOADS = {
    # name: (tokens per step, routing kind, description)
    "decode": (1, "normal", "GLM-5.2-shaped single-token decode: H 6144, I 2048, 256 routed "
                            "experts top-8 + 1 shared, int4 gs64, T=1, logits N(0,1)"),
    "verify4": (4, "zipf", "GLM-5.2-shaped speculative verify: T=4, Zipf-1.1 routing, "
                           "71.6% step-to-step expert repeats"),
    "batch32": (32, "zipf", "GLM-5.2-shaped small-batch decode: T=32, Zipf-1.1 routing, "
                            "71.6% step-to-step expert repeats"),
    "prefill": (4096, "uniform", "GLM-5.2-shaped prefill: T=4096, logits U[0,1)"),
    "stack": (64, "zipf", "16 independent GLM-5.2-shaped layers (16 x 257 experts resident), "
                          "T=64, per-layer Zipf-1.1 routing, x_(l+1) = x_l + MoE_l(x_l) in bf16"),
}
STACK_LAYERS = 16
# L2 budget of the stack's lookahead prefetch (--prefetch-mb): the shared
# expert (always used).  Measured with 0, 20 and 40 MiB: no budget made a step
# faster (larger budgets slow it down), so the stack line's value is the step
# with the prefetch off and the "on" time is reported beside it.
PREFETCH_BYTES = 20 << 20
METRIC = "MoE-layer tokens/s and achieved HBM GB/s (or TC util) vs B200 roofline"
L2_FLUSH_BYTES = 256 << 20
PAIR_FLOP = 75_497_472  # 2 * 3 * H * I for the GLM-5.2 shape
# DRAM bytes (read + write) of a workload's dominant kernel, from one ncu
# launch-list capture (dram__bytes_read.sum + dram__bytes_write.sum), as bytes
# per unit of work: a launch, or an expert the launch streams (the kernels'
# traffic grows with the experts they stream, so a capture on a smaller bank
# scales to the workload's own streamed experts).  Each entry names the
# kernel's source file and its SHA-256 at capture time; when the file has
# changed since, the bench reports traffic as null.
# workload -> (source file, sha256, bytes per unit, unit, how it was measured)
_DECODE_SRC = ("int4_routed_expert_coli_b200/csrc/decode.cu",
               "4b2566a371c85094c21a668a748004e16efadabc12e262cffc246356d1698882")
_BATCH_SRC = ("int4_routed_expert_coli_b200/csrc/batch.cu",
              "915e7e0caeea9571397e94c19bb28624199bc941cf5f45f145b0d74d4e9cbbaa")
_BATCH = (*_BATCH_SRC, 13_331_461, "streamed expert",
          "ncu launch list, 12 launches of the small-batch gate/up kernel on a 64-expert bank "
          "at T=32: bytes per streamed expert (unique routed + shared)")
DRAM_TRAFFIC = {
    "decode": (*_DECODE_SRC, 183_850_410, "launch",
               "ncu launch list, 18 launches of the fused decode kernel on a 64-expert bank "
               "(a T=1 step streams 8 + 1 experts on any bank)"),
    "verify4": (*_DECODE_SRC, 183_850_410 // 9, "streamed expert",
                "the T=1 fused-kernel capture, bytes per streamed expert"),
    "batch32": _BATCH,
}


def expert_bytes(H, I):
    return 3 * H * I // 2 + 3 * (H * I // 64) * 2


def gateup_bytes(H, I):
    return 2 * (H * I // 2) + 2 * (H * I // 64) * 2


def _sha256(path):
    import hashlib
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def traffic_for(workload, units):
    """(DRAM bytes per launch of the workload's dominant kernel, or None, and
    a note on the source); `units`: the launch's streamed experts."""
    ent = DRAM_TRAFFIC.get(workload)
    if ent is None:
        return None, "no ncu capture whose bytes scale to this workload"
    src, sha, per_unit, unit, how = ent
    if _sha256(os.path.join(ROOT, src)) != sha:
        return None, f"stale: {src} changed since the ncu capture"
    return (per_unit if unit == "launch" else per_unit * units), how


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def make_inputs(name, steps, seed, device):
    """Per-step activations and logits (lists of device tensors)."""
    T, kind, _ = WORKLOADS[name]
    xs, lgs = [], []
    if kind == "zipf":
        _, lg_np = synth.zipf_routing(T, GLM["E"], GLM["k"], steps=steps, seed=seed)
    for s in range(steps):
        xs.append(synth.make_activations(T, GLM["H"], seed=seed * 100003 + s, device=device))
        if kind == "normal":
            lgs.append(synth.make_logits_normal(T, GLM["E"], seed=seed * 100019 + s, device=device))
        elif kind == "uniform":
            lgs.append(synth.make_logits_uniform(T, GLM["E"], seed=seed * 100019 + s, device=device))
        else:
            lgs.append(torch.from_numpy(lg_np[s]).to(device))
    return xs, lgs


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.file = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
        sel = []
        try:
            bus = torch.cuda.get_device_properties(device_index).pci_bus_id
            sel = ["--id=" + bus]
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            sel = ["-i", vis.split(",")[device_index]] if vis else ["-i", str(device_index)]
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = list(csv.reader(io.StringIO(self.file.read())))
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        load = [v for v in sm if v > 0.5 * (mx or max(sm))] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    """One process per GPU under torchrun (NCCL); without a GPU (the CPU-only
    reference arm, or tests of this plumbing) the ranks use gloo."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=300)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout,
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time: every rank calls this with its own value."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
def oracle_steps(bank, xs, lgs, n_threads):
    """Oracle on the given steps (every token of every step); returns
    (seconds, tokens)."""
    import oracle
    E, k, n_sh = GLM["E"], GLM["k"], GLM["n_shared"]
    routes = [oracle.route(lg.float().cpu().numpy(), k) for lg in lgs]
    needed = set(range(E, E + n_sh))
    for idx, _ in routes:
        needed |= set(idx.ravel().tolist())
    ex = oracle.Experts([bank.expert_numpy(e) if e in needed else None for e in range(bank.n)])
    xb = [x.view(torch.int16).cpu().numpy().view(np.uint16) for x in xs]
    # all steps' tokens in one batch: the oracle is per token, so this is the
    # same work as running the steps one after another, spread over threads
    X = np.concatenate(xb, axis=0)
    IDX = np.concatenate([r[0] for r in routes], axis=0)
    W = np.concatenate([r[1] for r in routes], axis=0)
    t0 = time.perf_counter()
    oracle.layer(GLM["H"], GLM["I"], E, k, n_sh, ex, X, IDX, W, n_threads=n_threads)
    return time.perf_counter() - t0, X.shape[0]


def run_reference_stack(args):
    """The CPU oracle on the stack: each step takes a 2-token sample through
    all 16 layers (each layer's bf16 output feeds the next), timed on the
    host cores; the layers' weights are generated one at a time."""
    import oracle
    T, _, desc = WORKLOADS["stack"]
    H, I, E, k, n_sh = GLM["H"], GLM["I"], GLM["E"], GLM["k"], GLM["n_shared"]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    cores = os.cpu_count() or 1
    n = args.warmup + args.steps
    tok = 2
    xs, lgs = stack_inputs(n, seed=7, device="cpu")
    x = [xs[i][:tok].clone() for i in range(n)]
    sec = 0.0
    for l in range(STACK_LAYERS):
        bank = synth.make_expert_bank(H, I, E + n_sh, seed=7000 + l, device=dev,
                                      scale_range=synth.STACK_SCALE_RANGE,
                                      code_range=synth.STACK_CODE_RANGE)
        routes = [oracle.route(lgs[l][i][:tok].float().numpy(), k) for i in range(n)]
        needed = set(range(E, E + n_sh))
        for idx, _ in routes:
            needed |= set(idx.ravel().tolist())
        ex = oracle.Experts([bank.expert_numpy(e) if e in needed else None for e in range(bank.n)])
        del bank
        for i in range(n):
            xb = x[i].view(torch.int16).numpy().view(np.uint16)
            t0 = time.perf_counter()
            y = oracle.layer(H, I, E, k, n_sh, ex, xb, routes[i][0], routes[i][1],
                             n_threads=cores)
            if i >= args.warmup:
                sec += time.perf_counter() - t0
            x[i] = (x[i].double() + torch.from_numpy(np.asarray(y))).to(torch.bfloat16)
    value = tok * args.steps / sec
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": desc, "tokens_per_step": tok, "layers": STACK_LAYERS},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} steps of {tok} tokens through all "
                                   f"{STACK_LAYERS} layers, every routed + shared expert"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference(args, rank, world):
    """The CPU oracle on the same workload: each step is one full layer step
    of the workload (all its tokens), timed on the host cores."""
    if rank != 0:
        return
    name = args.workload
    if name == "stack":
        run_reference_stack(args)
        return
    T, _, desc = WORKLOADS[name]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    bank = synth.make_expert_bank(GLM["H"], GLM["I"], GLM["E"] + 1, seed=1, device=dev)
    cores = os.cpu_count() or 1
    n = args.warmup + args.steps
    sample_tokens = min(T, 8)  # tokens per step the oracle computes (prefill: a sample)
    xs, lgs = make_inputs(name, n, seed=7, device=dev)
    xs = [x[:sample_tokens] for x in xs]
    lgs = [lg[:sample_tokens] for lg in lgs]
    sec = 0.0
    toks = 0
    for i in range(n):
        s, t = oracle_steps(bank, [xs[i]], [lgs[i]], n_threads=cores)
        if i >= args.warmup:
            sec += s
            toks += t
    value = toks / sec
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": desc, "tokens_per_step": sample_tokens},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} steps of {sample_tokens} token(s) each, "
                                   f"all {GLM['k']}+{GLM['n_shared']} experts per token"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
def stack_inputs(n, seed, device):
    """Per-step layer-0 activations and per-layer, per-step Zipf logits."""
    T = WORKLOADS["stack"][0]
    xs = [synth.make_activations(T, GLM["H"], seed=seed * 100003 + s, device=device)
          for s in range(n)]
    lgs = []
    for l in range(STACK_LAYERS):
        _, lg_np = synth.zipf_routing(T, GLM["E"], GLM["k"], steps=n, seed=seed * 1009 + l)
        lgs.append([torch.from_numpy(lg_np[s]).to(device) for s in range(n)])
    return xs, lgs


def oracle_stack_sample(banks, x0, lgs_step, n_threads, tok=2):
    """The oracle on `tok` tokens of one stack step through every layer (each
    layer's bf16 output feeds the next, as on the GPU); returns the seconds
    spent in the oracle and the tokens."""
    import oracle
    E, k, n_sh = GLM["E"], GLM["k"], GLM["n_shared"]
    H, I = GLM["H"], GLM["I"]
    x = x0[:tok].cpu()
    sec = 0.0
    for l, bank in enumerate(banks):
        idx, w = oracle.route(lgs_step[l][:tok].float().cpu().numpy(), k)
        needed = set(idx.ravel().tolist()) | set(range(E, E + n_sh))
        ex = oracle.Experts([bank.expert_numpy(e) if e in needed else None for e in range(bank.n)])
        xb = x.view(torch.int16).numpy().view(np.uint16)
        t0 = time.perf_counter()
        y = oracle.layer(H, I, E, k, n_sh, ex, xb, idx, w, n_threads=n_threads)
        sec += time.perf_counter() - t0
        x = (x.double() + torch.from_numpy(np.asarray(y))).to(torch.bfloat16)
    return sec, tok


def run_stack(args, rank, world, local, with_cpu=True):
    """Config 5: 16 independent layers, each step runs them in sequence on
    one token batch, x_(l+1) = x_l + MoE_l(x_l) (bf16 stream, residual added
    in fp32 by the combine).  Returns the JSON line (rank 0) or None."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    T, _, desc = WORKLOADS["stack"]
    H, I, E, k, n_sh = GLM["H"], GLM["I"], GLM["E"], GLM["k"], GLM["n_shared"]
    L = STACK_LAYERS
    dev = torch.device("cuda", local if world > 1 else 0)
    banks = [synth.make_expert_bank(H, I, E + n_sh, seed=7000 + l, device=dev,
                                    scale_range=synth.STACK_SCALE_RANGE,
                                    code_range=synth.STACK_CODE_RANGE) for l in range(L)]
    layers = [c.MoELayer(b, n_routed=E, top_k=k, n_shared=n_sh) for b in banks]
    n = args.warmup + args.steps
    xs, lgs = stack_inputs(n, seed=7 + rank, device=dev)
    ws = layers[0].workspace(T, dev)
    acts = [torch.empty(T, H, dtype=torch.bfloat16, device=dev) for _ in range(L)]
    flush_buf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    fence_buf = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush_l2():
        flush_buf.sum()
        fence_buf.zero_()

    # Router-lookahead L2 prefetch: while layer l runs, a side stream
    # prefetches the experts layer l + 1 used in the previous step (the
    # prediction), whole experts in the order layer l + 1 streams them, up to
    # PREFETCH_BYTES.  Routings are double-buffered by step parity; the main
    # stream joins the side stream at the end of every step.
    side = torch.cuda.Stream(dev)
    idx_bufs = [[torch.zeros(T, k, dtype=torch.int32, device=dev) for _ in range(L)]
                for _ in range(2)]
    starts = [torch.cuda.Event() for _ in range(L)]
    side_done = torch.cuda.Event()

    def step(i, x0, out_last=None, prefetch=False):
        x = x0
        cur, prev = idx_bufs[i % 2], idx_bufs[(i - 1) % 2]
        for l in range(L):
            if prefetch and i > 0 and l + 1 < L:
                starts[l].record(stream)
                side.wait_event(starts[l])
                c.coli_moe_prefetch(layers[l + 1].handle, T, k, prev[l + 1], PREFETCH_BYTES,
                                    None, side)
            out = acts[l] if (l < L - 1 or out_last is None) else out_last
            c.coli_moe_layer(layers[l].handle, T, x, lgs[l][i], None, x, out, c.COLI_OUT_BF16,
                             cur[l], None, ws, stream)
            x = out
        if prefetch:
            side_done.record(side)
            stream.wait_event(side_done)
        return x

    for i in range(args.warmup):
        step(i, xs[i], prefetch=(i % 2 == 1))
        flush_l2()
    torch.cuda.synchronize(dev)
    if c.coli_moe_get_status(ws) != c.COLI_OK:
        raise RuntimeError("device status after warm-up: " + c.status_string(c.coli_moe_get_status(ws)))
    sets = [[set(torch.topk(lgs[l][i], k, dim=1).indices.flatten().tolist()) for l in range(L)]
            for i in range(n)]
    uniq = [[len(sets[i][l]) for l in range(L)] for i in range(args.warmup, n)]

    def timed(prefetch):
        barrier(world)
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for j in range(args.steps):
            ev[j][0].record(stream)
            step(args.warmup + j, xs[args.warmup + j], prefetch=prefetch)
            ev[j][1].record(stream)
            flush_l2()
        torch.cuda.synchronize(dev)
        barrier(world)
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world)

    sampler = ClockSampler(dev.index) if rank == 0 else None
    total_ms = timed(False)
    clocks = sampler.stop() if sampler else None
    on_ms = timed(True)
    if c.coli_moe_get_status(ws) != c.COLI_OK:
        raise RuntimeError("device status: " + c.status_string(c.coli_moe_get_status(ws)))
    # realised prediction: the share of layer l+1's experts (l + 1 >= 1) that
    # the previous step had used, and of the experts actually prefetched
    # (whole experts within the budget, ascending) the share that was used
    per_expert = expert_bytes(H, I)
    n_pf = max(0, PREFETCH_BYTES // per_expert - n_sh)
    hit_all, hit_pf = [], []
    for i in range(args.warmup, n):
        for l in range(1, L):
            act, pred = sets[i][l], sets[i - 1][l]
            hit_all.append(len(act & pred) / len(act))
            pf = sorted(pred)[:n_pf]
            if pf:
                hit_pf.append(len(act & set(pf)) / len(pf))

    torch.cuda.synchronize(dev)
    c.coli_moe_profile_enable(True)
    for j in range(args.steps):
        step(args.warmup + j, xs[args.warmup + j])
        flush_l2()
    torch.cuda.synchronize(dev)
    c.coli_moe_profile_enable(False)
    phase_ms, n_calls = c.coli_moe_profile_read()

    # end to end: layer-0 input from pinned host memory, last output back
    x_host = torch.stack([x.cpu() for x in xs[args.warmup:]]).pin_memory()
    out_host = torch.empty(args.steps, T, H, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    out_dev = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    for j in range(args.steps):
        ev2[j][0].record(stream)
        x_dev.copy_(x_host[j], non_blocking=True)
        step(args.warmup + j, x_dev, out_last=out_dev)
        out_host[j].copy_(out_dev, non_blocking=True)
        ev2[j][1].record(stream)
        flush_l2()
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev2), world)

    cpu = None
    if rank == 0 and world == 1 and with_cpu and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        sec, toks = oracle_stack_sample(banks, xs[args.warmup],
                                        [lgs[l][args.warmup] for l in range(L)], cores)
        cpu = {"value": toks / sec, "unit": "tokens/s", "cores": min(cores, toks * (k + n_sh)),
               "kind": "oracle",
               "sample": f"{toks} tokens of one step through all {L} layers (each layer's "
                         f"output feeds the next), every routed + shared expert, double "
                         f"precision, {sec:.1f} s"}
    del layers, banks
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    P = peaks()
    tokens = T * args.steps * world
    value = tokens / (total_ms / 1e3)
    step_bytes = statistics.mean(sum(u + n_sh for u in us) for us in uniq) * expert_bytes(H, I)
    k_ms = phase_ms[1] / max(n_calls, 1)
    k_bytes = statistics.mean(statistics.mean(us) for us in uniq) * gateup_bytes(H, I) + \
        n_sh * gateup_bytes(H, I)
    achieved = k_bytes / (k_ms / 1e3) / 1e9
    traffic, traffic_src = traffic_for(
        "stack", statistics.mean(statistics.mean(us) for us in uniq) + n_sh)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4xbf16/f16->f32", "data": "synthetic",
        "config": {"workload": desc, "tokens_per_step": T, "layers": L, "hidden": H, "inter": I,
                   "routed_experts": E, "top_k": k, "shared_experts": n_sh,
                   "resident_bytes": L * (E + n_sh) * expert_bytes(H, I),
                   "unique_routed_experts_per_layer": statistics.mean(
                       statistics.mean(us) for us in uniq),
                   "l2": "flushed between timed steps (256 MiB read); the stack itself "
                         "streams far more than L2 per step",
                   "parallelism": f"replicas x{world}"},
        "achieved_gbs_step": step_bytes / (total_ms / args.steps / 1e3) / 1e9,
        "roofline": {"bound": "hbm",
                     "kernel": "decode_fused_kernel" if T <= 8 and T * k < E
                     else "batch_ffn_kernel<gate/up>" if T <= 64 else "prefill_gemm_kernel<gate/up>",
                     "achieved": achieved,
                     "peak": P["hbm"], "unit": "GB/s", "frac": achieved / P["hbm"],
                     "peak_source": P["src"], "traffic": traffic, "traffic_source": traffic_src,
                     "algorithmic_bytes_per_launch": k_bytes, "avg_launch_ms": k_ms},
        "phase_ms_per_layer_call": {"before": phase_ms[0] / max(n_calls, 1), "main": k_ms,
                                    "after": phase_ms[2] / max(n_calls, 1)},
        "l2_prefetch": {"budget_bytes": PREFETCH_BYTES, "experts_per_layer": n_pf + n_sh,
                        "ms_per_step_on": on_ms / args.steps,
                        "ms_per_step_off": total_ms / args.steps,
                        "predicted_share_of_next_layer_experts": statistics.mean(hit_all),
                        "prefetched_experts_used_share": statistics.mean(hit_pf) if hit_pf
                        else None},
        "cpu_baseline": cpu,
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2},
        "gpu_launches": (1 if T <= 8 and T * k < E else 4 if T <= 64 else 7 if T * k >= 4096
                         else 6) * L * args.steps,
        "clocks": clocks,
    }
    return line


def run_ours(args, rank, world, local, name, with_cpu=True):
    """One workload through coli_moe_layer; returns the JSON line (rank 0) or
    None."""
    from int4_routed_expert_coli_b200 import coli_moe as c
    T, kind, desc = WORKLOADS[name]
    H, I, E, k, n_sh = GLM["H"], GLM["I"], GLM["E"], GLM["k"], GLM["n_shared"]
    if E != 256:  # a smaller resident bank (profiling runs) says so in the label
        desc = desc.replace("256 routed", f"{E} routed") + f", {E} routed experts resident"
    dev = torch.device("cuda", local if world > 1 else 0)
    bank = synth.make_expert_bank(H, I, E + n_sh, seed=1, device=dev)
    layer = c.MoELayer(bank, n_routed=E, top_k=k, n_shared=n_sh)
    n = args.warmup + args.steps
    xs, lgs = make_inputs(name, n, seed=1000 + rank, device=dev)
    ws = layer.workspace(T, dev)
    out = torch.empty(T, H, dtype=torch.float32, device=dev)
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    flush_buf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    fence_buf = torch.zeros(1, dtype=torch.int32, device=dev)

    def flush_l2():
        # a read of 256 MiB evicts the weights from L2; the one-element kernel
        # after it is what the layer's first kernel (launched as a programmatic
        # dependent, so it may start early) overlaps, instead of the flush
        flush_buf.sum()
        fence_buf.zero_()
    stream = torch.cuda.current_stream(dev)

    def step(i):
        c.coli_moe_layer(layer.handle, T, xs[i], lgs[i], None, None, out, c.COLI_OUT_F32, idx,
                         None, ws, stream)

    for i in range(args.warmup):
        step(i)
        flush_l2()
    torch.cuda.synchronize(dev)
    if c.coli_moe_get_status(ws) != c.COLI_OK:
        raise RuntimeError("device status after warm-up: " + c.status_string(c.coli_moe_get_status(ws)))

    # unique routed experts per timed step (sets the algorithmic bytes)
    uniq = []
    for i in range(args.warmup, n):
        uniq.append(len(set(torch.topk(lgs[i], k, dim=1).indices.flatten().tolist())))

    sampler = ClockSampler(dev.index) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for j in range(args.steps):
        ev[j][0].record(stream)
        step(args.warmup + j)
        ev[j][1].record(stream)
        flush_l2()
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms_steps = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(ms_steps), world)
    if c.coli_moe_get_status(ws) != c.COLI_OK:
        raise RuntimeError("device status: " + c.status_string(c.coli_moe_get_status(ws)))

    # ---- per-kernel durations: the same steps again with the library's
    # phase events on the launching stream (events between kernels stop the
    # kernels from overlapping, so this pass is not the headline) ------------
    torch.cuda.synchronize(dev)
    c.coli_moe_profile_enable(True)
    for j in range(args.steps):
        step(args.warmup + j)
        flush_l2()
    torch.cuda.synchronize(dev)
    c.coli_moe_profile_enable(False)
    phase_ms, n_calls = c.coli_moe_profile_read()

    # ---- end to end through the C ABI with host buffers --------------------
    # a step's inputs (x, then the logits) sit back to back in one pinned host
    # buffer and cross to the device in one copy; the output comes back in one
    nx, nl = T * H * 2, T * E * 4  # both multiples of 16: the logits view stays aligned
    in_host = torch.empty(args.steps, nx + nl, dtype=torch.uint8).pin_memory()
    for j in range(args.steps):
        in_host[j, :nx].copy_(xs[args.warmup + j].cpu().contiguous().view(torch.uint8).flatten())
        in_host[j, nx:].copy_(lgs[args.warmup + j].cpu().contiguous().view(torch.uint8).flatten())
    out_host = torch.empty(args.steps, T, H, dtype=torch.float32).pin_memory()
    in_dev = torch.empty(nx + nl, dtype=torch.uint8, device=dev)
    x_dev = in_dev[:nx].view(torch.bfloat16).view(T, H)
    lg_dev = in_dev[nx:].view(torch.float32).view(T, E)
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    for j in range(args.steps):
        ev2[j][0].record(stream)
        in_dev.copy_(in_host[j], non_blocking=True)
        c.coli_moe_layer(layer.handle, T, x_dev, lg_dev, None, None, out, c.COLI_OUT_F32, None,
                         None, ws, stream)
        out_host[j].copy_(out, non_blocking=True)
        ev2[j][1].record(stream)
        flush_l2()
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev2), world)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1) --------
    cpu = None
    if rank == 0 and world == 1 and with_cpu and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        tok = min(T, 8)
        # about 600 (token, expert) evaluations: ~10 s on 16 host cores
        n_s = max(1, min(args.steps, 600 // (tok * (k + n_sh))))
        sec, toks = oracle_steps(bank, [x[:tok] for x in xs[args.warmup:args.warmup + n_s]],
                                 [lg[:tok] for lg in lgs[args.warmup:args.warmup + n_s]],
                                 n_threads=cores)
        cpu = {"value": toks / sec, "unit": "tokens/s",
               "cores": min(cores, toks * (k + n_sh)), "kind": "oracle",
               "sample": f"{n_s} steps x {tok} token(s), every routed + shared expert of each "
                         f"token, double precision, {sec:.1f} s"}

    del layer, bank
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    P = peaks()
    tokens = T * args.steps * world
    value = tokens / (total_ms / 1e3)
    n_uniq = statistics.mean(uniq)
    step_bytes = (n_uniq + n_sh) * expert_bytes(H, I)
    # dominant kernel: up to 8 tokens with T*k < E the fused decode kernel
    # (routing, gate/up, down and combine; it streams every active expert
    # whole), other calls of up to 64 tokens the small-batch gate/up kernel,
    # larger ones the gate/up kernel of the tensor-core grouped GEMM (the
    # library's default paths)
    fused = T <= 8 and T * k < E
    small = not fused and T <= 64
    tensor = kind == "uniform"  # prefill: tensor-bound
    k_ms = phase_ms[1] / max(n_calls, 1)
    traffic, traffic_src = traffic_for(name, n_uniq + n_sh)
    if tensor:
        # gate/up GEMM: 2/3 of the pair FLOPs over all (token, expert) pairs + shared
        k_work = (T * k + T * n_sh) * PAIR_FLOP * 2 / 3
        achieved = k_work / (k_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": "prefill_gemm_kernel<gate/up>",
                "achieved": achieved, "peak": P["bf16"], "unit": "TFLOP/s",
                "frac": achieved / P["bf16"], "peak_source": P["src"] + " (bf16 burst; fp16 taken equal)",
                "traffic": traffic, "traffic_source": traffic_src,
                "algorithmic_flop_per_launch": k_work, "avg_launch_ms": k_ms}
    else:
        k_bytes = step_bytes if fused else (n_uniq + n_sh) * gateup_bytes(H, I)
        achieved = k_bytes / (k_ms / 1e3) / 1e9
        roof = {"bound": "hbm",
                "kernel": "decode_fused_kernel" if fused else "batch_ffn_kernel<gate/up>" if small
                else "prefill_gemm_kernel<gate/up>",
                "achieved": achieved, "peak": P["hbm"], "unit": "GB/s",
                "frac": achieved / P["hbm"], "peak_source": P["src"],
                "traffic": traffic, "traffic_source": traffic_src,
                "algorithmic_bytes_per_launch": k_bytes, "avg_launch_ms": k_ms}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4xbf16/f16->f32", "data": "synthetic",
        "config": {"workload": desc, "tokens_per_step": T, "hidden": H, "inter": I,
                   "routed_experts": E, "top_k": k, "shared_experts": n_sh,
                   "expert_bytes": expert_bytes(H, I), "unique_routed_experts_per_step": n_uniq,
                   "l2": "flushed between timed steps (256 MiB read), steps timed alone",
                   "parallelism": f"replicas x{world}"},
        "achieved_gbs_step": step_bytes / (total_ms / args.steps / 1e3) / 1e9,
        "roofline": roof,
        "phase_ms_per_step": {"before": phase_ms[0] / max(n_calls, 1), "main": k_ms,
                              "after": phase_ms[2] / max(n_calls, 1)},
        "cpu_baseline": cpu,
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * 2 + T * E * 4, "d2h_bytes_per_step": T * H * 4},
        # small-batch path: preparation (routing, union, activation operand),
        # gate/up, down, combine; grouped-GEMM path: route, union (two launches
        # from 4096 pairs on), gather, gate/up, down, combine
        "gpu_launches": (1 if fused else 4 if small else 7 if T * k >= 4096 else 6)
        * args.steps,
        "clocks": clocks,
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=None,
                    help="measure one workload alone (default: decode as the headline line, "
                         "the others attached under \"workloads\")")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefetch-mb", type=int, default=None,
                    help="L2 budget (MiB) of the stack's router-lookahead prefetch")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's tokens per step (small profiler cases)")
    ap.add_argument("--routed-experts", type=int, default=GLM["E"],
                    help="resident routed experts (default 256); fewer keeps a profiler "
                         "capture small while every step still runs 8 + 1 experts")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    GLM["E"] = args.routed_experts
    if args.prefetch_mb is not None:
        global PREFETCH_BYTES
        PREFETCH_BYTES = args.prefetch_mb << 20
    if args.tokens > 0:
        name = args.workload or "decode"
        T0, kind, desc = WORKLOADS[name]
        WORKLOADS[name] = (args.tokens, kind, desc.replace(f"T={T0}", f"T={args.tokens}"))
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            if args.workload is None:
                args.workload = "decode"
            run_reference(args, rank, world)
            return

        def one(name):
            if name == "stack":
                return run_stack(args, rank, world, local)
            return run_ours(args, rank, world, local, name)

        line = one(args.workload or "decode")
        if args.workload is None:
            extra = {}
            for name in ("verify4", "batch32", "prefill", "stack"):
                sub = one(name)
                if sub is not None:
                    for key in ("metric", "n_gpus", "steps", "warmup", "higher_is_better",
                                "scaling", "vs_baseline", "data"):
                        sub.pop(key, None)
                    extra[name] = sub
            if line is not None:
                line["workloads"] = extra
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
