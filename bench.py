#!/usr/bin/env python
"""Throughput of block-causal linear attention on B200, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step is one of the workloads run once through the library from a zero
state, with every input already resident in HBM.  The default is the largest
one that fits a GPU: batched 720p block-autoregressive streaming, B 4 x 64
heads x d 32, 7 blocks of 3 latent frames x 45 x 80 = 10,800 tokens, 4
denoising passes per block (the last one commits), 3D RoPE, bf16 (28
la_block_forward calls per step).  --config 2 is the 5 s 480p latent as one
bidirectional block (8190 tokens), 3 the 720p latent as one block, 4 the
minute-long 480p stream.  L2 is flushed before every timed step: a 256 MiB device
write, then a read of another 256 MiB buffer, so that no input line is in L2
and the flush's own dirty lines are written back before the step starts (a
write alone leaves ~126 MB of them to be written back inside the step); the
step time is the device time between CUDA events recorded before
its first and after its last kernel, so the flush is not in it.  The metric
is token*heads per second (every pass counts), whole job over all ranks.

Multi-GPU: one process per GPU (torchrun), no data-path collective.  By
default each rank runs an independent problem of the same shape (its own
seed): weak scaling.  With --shard heads the 64 heads of one problem are split
over the ranks (each owns its heads' tensors and state): strong scaling.  The
timed totals are reduced with MAX over ranks.

--impl reference times the fp64 CPU oracle (the test oracle, unchanged) on
the host cores on a bounded sample of the same workload; only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_causal_linear_b200 import ranks, synth  # noqa: E402

METRIC = "block linear-attn tokens·heads/s and achieved HBM GB/s vs B200 peak (1 GPU)"
METRIC_BWD = "block linear-attn backward tokens·heads/s and achieved HBM GB/s vs B200 peak (1 GPU)"
UNIT = "token·heads/s"
FLUSH_BYTES = 256 << 20          # > 2x the 126 MB L2 of a B200
FALLBACK_HBM_GBS = 6650.0
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=5, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--pass", dest="pass_", default="forward", choices=["forward", "backward"],
                    help="backward: la_full_backward over the workload's whole sequence (dq, dk, dv)")
    ap.add_argument("--op", default="attention", choices=["attention", "dwconv"],
                    help="dwconv: the Mix-FFN depthwise convolutions (1x3x3 then 3x1x1) on the workload's "
                         "latent grid, DWCONV_C channels")
    ap.add_argument("--input", default="native", choices=["native", "e4m3", "nvfp4"],
                    help="e4m3: q, k, v as FP8 E4M3 codes with per-tensor scales (la_*_forward_e4m3); nvfp4: "
                         "E2M1 codes with an E4M3 scale per 16 features and a per-tensor scale "
                         "(la_*_forward_nvfp4); bf16 out")
    ap.add_argument("--blocks", type=int, default=None,
                    help="streaming workloads: run only the first N blocks (small cases for profiling)")
    ap.add_argument("--shard", default="problem", choices=["problem", "heads", "tokens"],
                    help="problem: an independent problem per rank (weak scaling); "
                         "heads: one problem's heads split over the ranks (strong scaling); "
                         "tokens: every block's tokens split over the ranks, la_block_reduce -> all-gather of "
                         "the [S | Z] partials -> la_block_apply (strong scaling)")
    ap.add_argument("--emulate-ranks", type=int, default=1,
                    help="--shard tokens on one process: run this many ranks' slices one after another on "
                         "the GPU (the gather is then a view of one buffer)")
    return ap.parse_args()


def workload_config(w: synth.Workload, extra=None):
    c = {"workload": w.name, "B": w.B, "N_per_call": w.n_blk if w.mode == "stream" else w.n_total,
         "H": w.H, "d": w.d, "blocks": w.n_blocks, "passes_per_block": w.passes,
         "calls_per_step": w.calls, "api": "la_full_forward" if w.mode == "full" else "la_block_forward",
         "rope": "3d 8/12/12 base 1e4" if w.rope else None, "input_dtype": w.dtype,
         "accumulate": "f32", "state": "f32",
         "l2": "flushed before every timed step (256 MiB device write, then a 256 MiB device read so that "
               "the write's dirty lines leave L2 too; outside the step's events)"}
    if extra:
        c.update(extra)
    return c


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# the source files each timed kernel is built from (the shared headers too)
KERNEL_SOURCES = {
    "reduce": ["k_tc.cu"], "apply": ["k_tc.cu"], "finish": ["k_finish.cu"],
    "reduce_tc_rope": ["k_rope_tc.cu"], "apply_tc_rope": ["k_rope_tc.cu"],
    "reduce_tc_e4m3_rope": ["k_rope_tc.cu"], "apply_tc_e4m3_rope": ["k_rope_tc.cu"],
    "reduce_tc_nvfp4_rope": ["k_rope_tc.cu"], "apply_tc_nvfp4_rope": ["k_rope_tc.cu"],
    "bwd_q": ["k_bwd_q_tc.cu"], "bwd_k": ["k_bwd_tc.cu"], "dwconv": ["k_conv.cu"],
    "bwd_q_rope": ["k_bwd.cu"], "bwd_k_rope": ["k_bwd_tc.cu"],
}
SHARED_SOURCES = ["la_internal.cuh", "la_sm100.cuh", "la_rope.cuh"]


def kernel_sources_sha(kernel: str) -> str:
    """Hash of the sources of `kernel` (by the longest known prefix of its name), so that a
    stored ncu figure is dropped when, and only when, that kernel changed."""
    csrc = os.path.join(ROOT, "block_causal_linear_b200", "csrc")
    key = max((k for k in KERNEL_SOURCES if kernel.startswith(k)), key=len, default=None)
    files = sorted(os.listdir(csrc)) if key is None else KERNEL_SOURCES[key] + SHARED_SOURCES
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, units_per_launch: int):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, scaled
    to this launch by its units (token-heads, or elements for the convolution),
    or None when the kernel changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(kernel)
    if not e or e.get("sources_sha") != kernel_sources_sha(kernel):
        return None
    return e["dram_bytes_per_unit"] * units_per_launch


class ClockSampler:
    def __init__(self):
        self.proc = None
        self.path = None

    def start(self, device):
        """Sample the GPU behind `device` (selected by UUID, since nvidia-smi
        numbers the machine's GPUs regardless of CUDA_VISIBLE_DEVICES)."""
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", *sel, f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            self.filtered = bool(sel)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self, device_index: int):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, power, reasons = [], [], [], set()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9 or not parts[0].isdigit():
                    continue
                if not self.filtered and int(parts[0]) != device_index:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for nm, val in zip(names[1:], parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- oracle timing

def oracle_sample(w: synth.Workload, budget_s: float, orc, backward=False):
    """Time the oracle on the first call's inputs of the workload: all tokens of
    that call, a head subset sized to take about budget_s (backward: the fp64
    backward of that block).  Returns (token_heads, seconds, description)."""
    import numpy as np  # noqa: F401

    _, _, q, k, v = next(iter(synth.stream(w, "cpu", blocks=1)))
    rope = (orc.make_rope(Hg=w.Hg, Wg=w.Wg, t_offset=0, dims=w.rope_dims, base=w.rope_base)
            if w.rope else None)

    def run(nh):
        qs, ks, vs = (t[:, :, :nh].contiguous() for t in (q, k, v))
        st = orc.State(w.B, nh, w.d)
        t0 = time.perf_counter()
        if backward:
            orc.full_backward(qs, ks, vs, vs, 0, rope=rope, eps=w.eps)
        else:
            orc.block_forward(qs, ks, vs, st, commit=True, rope=rope, eps=w.eps)
        return time.perf_counter() - t0

    t1 = run(1)
    nh = int(max(1, min(w.H, budget_s / max(t1, 1e-6))))
    dt = run(nh)
    th = w.B * q.shape[1] * nh
    desc = (f"first call of the workload ({w.B}x{q.shape[1]} tokens) on {nh} of {w.H} heads, "
            + ("the fp64 backward of that block (state, dq and state gradients, dk, dv)" if backward else
               "one recurrence pass (block KV, state combine, apply, commit) in fp64"))
    return th, dt, desc


def run_reference(args, rank):
    if rank != 0:
        return
    import oracle as orc

    orc.build()
    w = synth.WORKLOADS[args.config]
    total_steps = args.steps if args.steps is not None else 10
    per_step = min(10.0, 150.0 / max(1, total_steps + args.warmup))
    _, _, q, k, v = next(iter(synth.stream(w, "cpu", blocks=1)))
    rope = (orc.make_rope(Hg=w.Hg, Wg=w.Wg, t_offset=0, dims=w.rope_dims, base=w.rope_base)
            if w.rope else None)
    # calibrate tokens per step on one head
    ntok = q.shape[1]
    t0 = time.perf_counter()
    orc.block_forward(q[:, :, :1].contiguous(), k[:, :, :1].contiguous(), v[:, :, :1].contiguous(),
                      orc.State(w.B, 1, w.d), rope=rope, eps=w.eps)
    per_th = (time.perf_counter() - t0) / (w.B * ntok)
    want = max(1, int(per_step / per_th))            # token-heads per step
    nh = max(1, min(w.H, want // (w.B * ntok)))
    nt = ntok if nh > 1 else max(1, min(ntok, want // w.B))
    qs, ks, vs = (t[:, :nt, :nh].contiguous() for t in (q, k, v))

    def step():
        orc.block_forward(qs, ks, vs, orc.State(w.B, nh, w.d), rope=rope, eps=w.eps)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(total_steps):
        step()
    dt = time.perf_counter() - t0
    th = w.B * nt * nh * total_steps
    value = th / dt
    sample = (f"each step: {w.B}x{nt} tokens of the workload's first call on {nh} of {w.H} heads, "
              f"fp64 recurrence (block KV, state combine, apply, commit)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": total_steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / total_steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, {"l2": "n/a (CPU)"}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.get_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- Mix-FFN convolutions

DWCONV_C = 5120   # MLP channels: 2.5 x the 2048-wide attention (the pages give no width)


def run_token_split(args, w, world, rank, dist, dev, la):
    """--shard tokens: every call's block is split over the ranks by tokens
    (whole frames with RoPE, so that positions continue across the slices).
    Per call: la_block_reduce of each local rank's k, v slice, one all-gather
    of the [S | Z] partials (NCCL, 4,224 bytes per (b, h) and rank), then
    la_block_apply of each local rank's q slice, which adds the gathered
    partials in rank order and commits the same state on every rank.  With one
    process, --emulate-ranks R runs R ranks' slices one after another on the
    GPU; the partials are then written straight into the gathered buffer.
    Strong scaling: the job's work is the unsplit workload."""
    if args.pass_ != "forward" or args.input != "native" or args.op != "attention":
        raise SystemExit("--shard tokens times the native forward path")
    if args.blocks is not None:
        if w.mode != "stream" or not 1 <= args.blocks <= w.n_blocks:
            raise SystemExit("--blocks needs a streaming workload and 1 <= N <= its block count")
        w = w.shrink(n_blocks=args.blocks)
    if w.mode == "full" and w.n_blocks != 1:
        raise SystemExit("--shard tokens: a one-call workload must be one block")
    R_local = args.emulate_ranks if world == 1 else 1
    R = world * R_local
    if R_local < 1 or R > 32:
        raise SystemExit("--emulate-ranks: 1 .. 32 ranks in all")
    N = w.n_blk if w.mode == "stream" else w.n_total
    align = w.Hg * w.Wg if w.rope else 1
    if (N + align - 1) // align < R:
        raise SystemExit(f"--shard tokens: a block of {N} tokens has fewer "
                         f"{'frames' if w.rope else 'tokens'} than the {R} ranks")
    frames_blk = N // align if w.rope else 0
    if w.mode == "stream":
        calls = list(synth.stream(w, device=dev))
    else:
        calls = [(0, 0, *synth.full_sequence(w, device=dev))]
    passes = w.passes if w.mode == "stream" else 1
    local = [rank * R_local + j for j in range(R_local)]          # global rank of each local rank
    slices = [ranks.token_slice(N, R, r, align) for r in local]
    # each rank owns its slices (what a token-parallel producer leaves on its GPU)
    ins = [[tuple(t[:, t0:t1].contiguous() for t in c[2:5]) for (t0, t1) in slices] for c in calls]
    del calls
    outs = [[torch.empty_like(x[0]) for x in c] for c in ins]
    states = [la.State(w.B, w.H, w.d, device=dev) for _ in local]
    ws = [la.alloc_workspace(w.B, t1 - t0, w.H, w.d, t1 - t0, device=dev) for (t0, t1) in slices]
    part_shape = (w.B, w.H, w.d * w.d + w.d)
    gathered = torch.empty((R,) + part_shape, dtype=torch.float32, device=dev)
    mine = torch.empty(part_shape, dtype=torch.float32, device=dev)
    exchange_bytes = gathered.numel() * 4                        # what every rank holds after one gather
    launches = [0]

    def rope_for(j, frames_before, reduce_side):
        if not w.rope:
            return None
        first_frame = ranks.split_frame_offsets(frames_before, N, R, align)[local[j]][2]
        T = 0 if reduce_side else frames_blk                      # apply: a commit advances by the block
        return la.make_rope(Hg=w.Hg, Wg=w.Wg, T=T, t_offset=first_frame, dims=w.rope_dims, base=w.rope_base)

    n_calls = len(ins)
    # external: recorded inside a captured graph as event-record nodes
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(n_calls)]

    def step(timed=False):
        n = 0
        for st in states:
            rc = la.la_state_init(st.c, st.S.data_ptr(), st.Z.data_ptr(), w.B, w.H, w.d, la._stream_ptr(None))
            if rc != la.LA_OK:
                raise la.LAError(rc, "la_state_init")
        for i, sl in enumerate(ins):
            commit = i % passes == passes - 1
            frames_before = states[0].t_next           # host counter, the same on every rank
            e = ev[i]

            def reduce_fn(j, k, v):
                nonlocal n
                dst = gathered[local[j]] if world == 1 else mine
                la.block_reduce(k, v, rope=rope_for(j, frames_before, True), ws=ws[j], partial=dst)
                n += la.la_last_launch_count()
                return dst

            def gather_fn(parts):
                if timed:
                    e[1].record()
                if world > 1:
                    dist.all_gather_into_tensor(gathered, parts[0])
                if timed:
                    e[2].record()
                return gathered

            def apply_fn(j, q, g):
                nonlocal n
                la.block_apply(q, g, states[j], commit=commit, rope=rope_for(j, frames_before, False), eps=w.eps,
                               ws=ws[j], out=outs[i][j])
                n += la.la_last_launch_count()

            if timed:
                e[0].record()
            ranks.split_call([x[0] for x in sl], [(x[1], x[2]) for x in sl], reduce_fn, gather_fn, apply_fn)
            if timed:
                e[3].record()
        launches[0] = n

    flush_w = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    acc = torch.empty((), dtype=torch.float32, device=dev)

    def flush(x):
        flush_w.fill_(x)
        torch.sum(flush_r, dim=0, out=acc)

    for i in range(max(3, args.warmup)):                # eager warm-up (also brings up NCCL before capture)
        step()
    torch.cuda.synchronize()
    la.device_status()
    # One step as a CUDA graph (NCCL's all-gather is captured with it), timed
    # between event nodes inside the graph; a second graph with events between
    # the reduce, gather and apply of every call gives the stage times.
    g0 = torch.cuda.Event(enable_timing=True, external=True)
    g1 = torch.cuda.Event(enable_timing=True, external=True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        g0.record()
        step()
        g1.record()
    graph_st = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_st):
        step(timed=True)
    torch.cuda.synchronize()
    for i in range(max(3, args.warmup)):
        flush(float(i))
        graph.replay()
    torch.cuda.synchronize()
    K = ranks.agree_steps(args.steps or 20, dist, dev)
    sampler = ClockSampler()
    if rank == 0:
        sampler.start(dev)
        time.sleep(0.3)
    t = [0.0, 0.0, 0.0, 0.0]                          # total, reduce, gather, apply (ms)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for it in range(K):
        flush(float(it))
        graph.replay()
        g1.synchronize()
        t[0] += g0.elapsed_time(g1)
    for it in range(K):
        flush(float(it))
        graph_st.replay()
        torch.cuda.synchronize()
        for e in ev:
            t[1] += e[0].elapsed_time(e[1])
            t[2] += e[1].elapsed_time(e[2])
            t[3] += e[2].elapsed_time(e[3])
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop(dev.index or 0) if rank == 0 else None
    la.device_status()                                  # raises if a bounded device wait gave up
    t = ranks.max_over_ranks(t, dist, dev)
    units = w.token_heads                               # the unsplit workload, once per step
    value = units * K / (t[0] / 1e3)
    peak, peak_kind = measured_peaks()
    step_gbs = w.alg_bytes / (t[0] / K / 1e3) / 1e9
    bytes_per_side = units * 2 * w.d * w.elem_bytes     # reduce: k, v; apply: q, out
    dom, dom_ms = ("reduce", t[1]) if t[1] >= t[3] else ("apply", t[3])
    path = la.la_last_path()
    kname = f"{dom}_{path}" + ("_rope" if w.rope and path == "tc" else "")
    achieved = bytes_per_side / (dom_ms / K / 1e3) / 1e9
    per_launch = w.B * (sum(t1 - t0 for t0, t1 in slices) // len(slices)) * w.H
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": max(3, args.warmup), "ms_per_step": t[0] / K, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": workload_config(w, {"pass": "forward", "input_dtype": w.dtype,
                                          "parallelism": f"tokens of every block split over {R} ranks "
                                                         f"({world} process{'es' if world > 1 else ''}"
                                                         f"{', emulated one after another' if R_local > 1 else ''})",
                                          "api": "la_block_reduce + all-gather + la_block_apply",
                                          "l2": "flushed before every timed step (256 MiB write, then 256 MiB read)"}),
            "achieved_hbm_gbs": step_gbs, "hbm_frac_of_" + peak_kind: step_gbs / peak,
            "stage_ms_per_step": {"reduce": t[1] / K, "gather": t[2] / K, "apply": t[3] / K},
            "exchange_bytes_per_call": exchange_bytes, "exchange_bytes_per_step": exchange_bytes * n_calls,
            "roofline": {"bound": "hbm", "kernel": f"{kname} (stage: kernel and its combine)", "achieved": achieved,
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": ncu_traffic(kname, per_launch)},
            "cpu_baseline": None, "e2e": None, "gpu_launches": launches[0] * K, "path": path, "clocks": clocks,
            "launch": "one CUDA graph per step (the all-gather captured with it); stage times from a second "
                      "graph with events between the reduce, gather and apply of every call",
        }
        print(json.dumps(line), flush=True)
    del graph, graph_st                                 # the graphs hold NCCL work: release them first
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def run_dwconv(args, w, world, rank, dist, dev, la):
    """One step = the two depthwise convolutions of the Spatial-Temporal
    Mix-FFN on one latent video: y1 = conv_1x3x3(x), y2 = conv_3x1x1(y1), bf16
    activations, fp32 weights, over the workload's frames (one call's frames
    for a streaming workload).  L2 flushed before every step.  Algorithmic
    bytes: each convolution reads and writes its activation once."""
    T = w.frames                  # one call's frames
    B, Hg, Wg, C = w.B, w.Hg, w.Wg, DWCONV_C
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 31)
    x = torch.randn((B, T, Hg, Wg, C), generator=g, device=dev).to(torch.bfloat16)
    w1 = (torch.randn((C, 1, 3, 3), generator=g, device=dev) / 3).contiguous()
    w2 = (torch.randn((C, 3, 1, 1), generator=g, device=dev) / 2).contiguous()
    b1 = torch.randn(C, generator=g, device=dev)
    b2 = torch.randn(C, generator=g, device=dev)
    y1, y2 = torch.empty_like(x), torch.empty_like(x)
    flush_w = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    acc = torch.empty(1, dtype=torch.float32, device=dev)

    def flush(v):
        flush_w.fill_(v)
        torch.sum(flush_r, dim=0, out=acc)

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]

    def step(record=False):
        if record:
            ev[0].record()
        la.dwconv3d(x, w1, b1, out=y1)
        if record:
            ev[1].record()
        la.dwconv3d(y1, w2, b2, out=y2)
        if record:
            ev[2].record()

    for i in range(max(3, args.warmup)):
        flush(float(i))
        step()
    torch.cuda.synchronize()
    K = args.steps or 200
    K = ranks.agree_steps(K, dist, dev)
    sampler = ClockSampler()
    if rank == 0:
        sampler.start(dev)
        time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_all, t1, t2 = 0.0, 0.0, 0.0
    for i in range(K):
        flush(float(i))
        step(record=True)
        ev[2].synchronize()
        t_all += ev[0].elapsed_time(ev[2])
        t1 += ev[0].elapsed_time(ev[1])
        t2 += ev[1].elapsed_time(ev[2])
    torch.cuda.synchronize()
    clocks = sampler.stop(dev.index or 0) if rank == 0 else None
    t_all, t1, t2 = ranks.max_over_ranks([t_all, t1, t2], dist, dev)
    tokens = B * T * Hg * Wg
    value = ranks.job_throughput(tokens, world, K, t_all)
    peak, peak_kind = measured_peaks()
    conv_bytes = tokens * C * 2 * 2                     # read + write, bf16
    dom, dom_ms = ("dwconv_1x3x3", t1) if t1 >= t2 else ("dwconv_3x1x1", t2)
    achieved = conv_bytes / (dom_ms / K / 1e3) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle as orc

        orc.build()
        nc = 64
        xs = x[..., :nc].contiguous().cpu()
        t0 = time.perf_counter()
        orc.dwconv3d(xs, w1[:nc].double().cpu().numpy(), b1[:nc].double().cpu().numpy())
        dt = time.perf_counter() - t0
        cpu = {"value": tokens * nc / C / dt, "unit": "tokens/s", "cores": orc.get_threads(), "kind": "oracle",
               "sample": f"the 1x3x3 convolution of the same grid on {nc} of {C} channels, fp64, scaled to {C}"}
    if rank == 0:
        line = {"metric": "Mix-FFN depthwise convolutions (1x3x3 then 3x1x1) tokens/s", "value": value,
                "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": max(3, args.warmup),
                "ms_per_step": t_all / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16 activations, fp32 weights and accumulation", "data": "synthetic",
                "config": {"workload": f"{w.name} latent grid", "B": B, "T": T, "Hg": Hg, "Wg": Wg, "C": C,
                           "l2": "flushed before every step (256 MiB write then 256 MiB read)"},
                "achieved_hbm_gbs": 2 * conv_bytes / (t_all / K / 1e3) / 1e9,
                "hbm_frac_of_" + peak_kind: 2 * conv_bytes / (t_all / K / 1e3) / 1e9 / peak,
                "stage_ms_per_step": {"dwconv_1x3x3": t1 / K, "dwconv_3x1x1": t2 / K},
                "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                             "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                             "traffic": ncu_traffic(dom, tokens * C)},
                "cpu_baseline": cpu, "e2e": None, "gpu_launches": 2 * K, "path": "dwconv", "clocks": clocks}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------- our arm

def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))

    from block_causal_linear_b200 import build as la_build

    la_build.build()
    from block_causal_linear_b200 import la
    from block_causal_linear_b200.runner import BackwardRunner, Runner

    base = synth.WORKLOADS[args.config]
    if args.shard == "tokens":
        return run_token_split(args, base, world, rank, dist, torch.device("cuda", local_rank), la)
    if args.shard == "heads":
        h0, h1 = ranks.head_slice(base.H, world, rank)
        if h1 <= h0:
            raise SystemExit(f"--shard heads: rank {rank} of {world} has no heads of {base.H}")
        w = ranks.rank_workload(base, rank).shrink(H=h1 - h0)
    else:
        w = ranks.rank_workload(base, rank)
    dev = torch.device("cuda", local_rank)
    if args.op == "dwconv":
        return run_dwconv(args, w, world, rank, dist, dev, la)
    if args.blocks is not None:
        if w.mode != "stream" or not 1 <= args.blocks <= w.n_blocks:
            raise SystemExit("--blocks needs a streaming workload and 1 <= N <= its block count")
        w = w.shrink(n_blocks=args.blocks)
    bwd = args.pass_ == "backward"
    f8 = args.input == "e4m3"
    f4 = args.input == "nvfp4"
    if (f8 or f4) and bwd:
        raise SystemExit(f"--input {args.input} is a forward path")
    runner = BackwardRunner(w, dev) if bwd else Runner(w, dev, e4m3=f8, nvfp4=f4)
    w = runner.w
    flush_w = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_acc = torch.empty((), dtype=torch.float32, device=dev)

    class _Flush:
        @staticmethod
        def fill_(x):
            flush_w.fill_(x)
            torch.sum(flush_r, dim=0, out=flush_acc)

    flush = _Flush()
    stream = torch.cuda.current_stream()
    n_calls = len(runner.calls)

    def barrier():
        if dist is not None:
            dist.barrier()

    # warm-up (untimed)
    for _ in range(args.warmup):
        flush.fill_(1.0)
        runner.step()
    torch.cuda.synchronize()
    # steps: about 2 s of timed region unless given
    if args.steps is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.fill_(2.0)
        e0.record()
        runner.step()
        e1.record()
        torch.cuda.synchronize()
        est = e0.elapsed_time(e1) / 1e3 + 1e-4
        args.steps = int(min(20000, max(20, 2.0 / est)))
        args.steps = ranks.agree_steps(args.steps, dist, dev)
    K = args.steps

    # one step captured as a CUDA graph (the library is capture-safe: it never
    # allocates or synchronises); kernels inside keep their programmatic
    # dependent-launch edges
    # One step captured as a CUDA graph (the library is capture-safe: it never
    # allocates or synchronises); kernels inside keep their programmatic
    # dependent-launch edges.  The step's device time is taken between two
    # event-record nodes inside the graph, before its first and after its last
    # kernel, so it excludes the host's graph-launch latency; the time between
    # events recorded on the stream around the replay, which includes it, is
    # reported beside it.
    g_start = torch.cuda.Event(enable_timing=True, external=True)
    g_end = torch.cuda.Event(enable_timing=True, external=True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        g_start.record()
        runner.step()
        g_end.record()
    launches_per_step = runner.launches_per_step
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        flush.fill_(3.0)
        graph.replay()
    torch.cuda.synchronize()

    o_start = torch.cuda.Event(enable_timing=True)
    o_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler()
    barrier()
    torch.cuda.synchronize()
    if rank == 0:
        sampler.start(dev)
        time.sleep(0.3)
    step_ms, outer_ms = [], []
    for kk in range(K):
        flush.fill_(float(kk))
        o_start.record(stream)
        graph.replay()
        o_end.record(stream)
        o_end.synchronize()
        step_ms.append(g_start.elapsed_time(g_end))
        outer_ms.append(o_start.elapsed_time(o_end))
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop(local_rank) if rank == 0 else None
    launches = K * launches_per_step
    la.device_status()

    # per-kernel durations: a second graph of the same step with the library's
    # stage events between its kernels (they serialise the kernels, so this
    # region is timed separately and only feeds the per-kernel roofline)
    Ks = min(K, 200)
    stage_ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(n_calls)]
    for e in stage_ev:
        for x in e:
            x.record()
    torch.cuda.synchronize()

    def set_stage(i):
        la.la_set_stage_events(*(x.cuda_event for x in stage_ev[i]))

    graph2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph2):
        set_stage(0)
        runner.step(after_call=lambda i: set_stage(i + 1) if i + 1 < n_calls else None)
    la.la_set_stage_events(None, None, None, None)
    stage_ms = [0.0, 0.0, 0.0]
    for kk in range(Ks):
        flush.fill_(float(kk))
        graph2.replay()
        torch.cuda.synchronize()
        for e in stage_ev:
            for j in range(3):
                stage_ms[j] += e[j].elapsed_time(e[j + 1])
    stage_ms = [x * K / Ks for x in stage_ms]      # scaled to K steps like total_ms

    # The step's last writes can still sit dirty in L2 when its last kernel
    # ends; they reach DRAM during the next (untimed) flush.  A second timing
    # counts them: the step followed by a read of a buffer twice the size of
    # L2 (which evicts every dirty line) between event nodes of one graph,
    # minus the same read alone after a flush.
    wb_start = torch.cuda.Event(enable_timing=True, external=True)
    wb_end = torch.cuda.Event(enable_timing=True, external=True)
    rd_start = torch.cuda.Event(enable_timing=True, external=True)
    rd_end = torch.cuda.Event(enable_timing=True, external=True)
    evict = torch.empty((), dtype=torch.float32, device=dev)
    graph_wb, graph_rd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_wb):
        wb_start.record()
        runner.step()
        torch.sum(flush_r, dim=0, out=evict)
        wb_end.record()
    with torch.cuda.graph(graph_rd):
        rd_start.record()
        torch.sum(flush_r, dim=0, out=evict)
        rd_end.record()
    Kw = min(K, 100)
    wb_ms = rd_ms = 0.0
    for kk in range(Kw):
        flush.fill_(float(kk))
        graph_wb.replay()
        flush.fill_(float(kk))
        graph_rd.replay()
        torch.cuda.synchronize()
        wb_ms += wb_start.elapsed_time(wb_end)
        rd_ms += rd_start.elapsed_time(rd_end)
    wb_step_ms = (wb_ms - rd_ms) / Kw
    total_ms = sum(step_ms)
    total_ms, outer_total_ms, red_ms, fin_ms, app_ms, wb_step_ms = ranks.max_over_ranks(
        [total_ms, sum(outer_ms)] + stage_ms + [wb_step_ms], dist, dev)

    th_step = w.token_heads                          # per rank per step
    value = ranks.job_throughput(th_step, world, K, total_ms)
    ms_per_step = total_ms / K
    peak, peak_kind = measured_peaks()
    # algorithmic bytes: forward reads q, k, v and writes out (4 tensors);
    # backward reads q, k, v, dout and writes dq, dk, dv (7 tensors)
    # E4M3 forward: q, k, v one byte per feature, out bf16; NVFP4 forward: q,
    # k, v half a byte per feature plus one scale byte per 16 features, out bf16
    if f8:
        alg_bytes = w.token_heads * w.d * (3 * 1 + 2) + (w.alg_bytes - w.token_heads * 4 * w.d * w.elem_bytes)
    elif f4:
        alg_bytes = w.token_heads * (3 * (w.d // 2 + w.d // 16) + 2 * w.d)
    else:
        alg_bytes = w.token_heads * (7 if bwd else 4) * w.d * w.elem_bytes if bwd else w.alg_bytes
    step_gbs = alg_bytes / (ms_per_step / 1e3) / 1e9

    launches_per_kernel = K * n_calls                # stage_ms is scaled to K steps
    per_call_th = w.B * runner.tokens_per_call(0) * w.H
    path = la.la_last_path()
    if bwd:
        # stages: forward state | query side (reads q, dout, writes dq) | key side
        # (reads k, v, writes dk, dv); the dominant one of the two sides
        side = [("bwd_q", fin_ms, 3), ("bwd_k", app_ms, 4)]
        dom, dom_ms, ntens = max(side, key=lambda x: x[1])
        kname = dom + ("_rope" if w.rope else "")   # with RoPE: the CUDA-core query side, the RoPE key side
    else:
        # dominant kernel: the larger of reduce (reads k, v) and apply (reads q, writes out)
        dom, dom_ms = ("reduce", red_ms) if red_ms >= app_ms else ("apply", app_ms)
        ntens = 2
        kname = f"{dom}_{path}" + ("_rope" if w.rope and path.startswith("tc") else "")
    if f8:   # reduce: k, v codes; apply: q codes and bf16 out
        kern_bytes = per_call_th * w.d * (2 if dom == "reduce" else 3)
    elif f4:   # reduce: k, v codes and block scales; apply: q codes and scales, bf16 out
        per_t = w.d // 2 + w.d // 16
        kern_bytes = per_call_th * (2 * per_t if dom == "reduce" else per_t + 2 * w.d)
    else:
        kern_bytes = per_call_th * ntens * w.d * w.elem_bytes
    avg_launch_s = dom_ms / launches_per_kernel / 1e3
    achieved = kern_bytes / avg_launch_s / 1e9

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(runner, w, dev, world, dist, steps=max(3, min(20, K)))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle as orc

        orc.build()
        th, dt, desc = oracle_sample(w, 12.0, orc, backward=bwd)
        cpu = {"value": th / dt, "unit": UNIT, "cores": orc.get_threads(), "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC_BWD if bwd else METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak", "vs_baseline": None,
            "dtype": ("e4m3 in, bf16 out" if f8 else "nvfp4 in, bf16 out" if f4 else
                      ("bf16" if w.dtype == "bf16" else "f32")), "data": "synthetic",
            "config": workload_config(w, {"pass": args.pass_,
                                          "input_dtype": ("e4m3 (per-tensor scale)" if f8 else
                                                          "nvfp4 (e2m1, e4m3 scale per 16, per-tensor scale)" if f4
                                                          else w.dtype),
                                          "parallelism": (f"heads of one problem split over {world} ranks"
                                                          if args.shard == "heads" else
                                                          f"independent problem per rank x{world}")}),
            "achieved_hbm_gbs": step_gbs, "hbm_frac_of_" + peak_kind: step_gbs / peak,
            "ms_per_step_incl_writeback": wb_step_ms,
            "hbm_frac_incl_writeback_of_" + peak_kind: alg_bytes / (wb_step_ms / 1e3) / 1e9 / peak,
            "stage_ms_per_step": ({"forward_state": red_ms / K, "query_side": fin_ms / K, "key_side": app_ms / K}
                                  if bwd else {"reduce": red_ms / K, "finish": fin_ms / K, "apply": app_ms / K}),
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": ncu_traffic(kname, per_call_th)},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "path": path, "clocks": clocks,
            "launch": "one CUDA graph per step (programmatic dependent launch between kernels); step time "
                      "between event nodes inside the graph",
            "ms_per_step_incl_graph_launch": outer_total_ms / K,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def measure_e2e(runner, w, dev, world, dist, steps):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory to the device, runs the workload, and
    copies every output back.  Copies and kernels run on three streams, call by
    call: the inputs of a call go up while earlier calls compute and earlier
    outputs come down (PCIe is full duplex); a call's device buffers are
    reused by the next step only after this step is done with them."""
    from block_causal_linear_b200 import la  # noqa: F401

    host_in = [tuple(t.cpu().pin_memory() for t in c) for c in runner.inputs]
    host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in runner.outs]
    h2d = sum(t.numel() * t.element_size() for c in host_in for t in c)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    n = len(runner.calls)
    main = torch.cuda.current_stream(dev)
    s_up, s_cmp, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    ev_up = [torch.cuda.Event() for _ in range(n)]
    ev_cmp = [torch.cuda.Event() for _ in range(n)]
    ev_down = [torch.cuda.Event() for _ in runner.outs]
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    state = {"first": True}

    def before_call(i):
        s_cmp.wait_event(ev_up[i])
        if not state["first"]:
            for j, c in enumerate(runner.out_call):
                if c == i:
                    s_cmp.wait_event(ev_down[j])   # call i's outputs of the previous step are on the host

    def after_call(i):
        ev_cmp[i].record(s_cmp)
        if i + 1 < n:
            before_call(i + 1)

    def one():
        for i, (hs, ds) in enumerate(zip(host_in, runner.inputs)):
            if not state["first"]:
                s_up.wait_event(ev_cmp[i])      # the previous step has read inputs i
            with torch.cuda.stream(s_up):
                for h_, d_ in zip(hs, ds):
                    d_.copy_(h_, non_blocking=True)
            ev_up[i].record(s_up)
        before_call(0)
        with torch.cuda.stream(s_cmp):
            runner.step(after_call=after_call, stream=s_cmp)
        for i, (ho, o) in enumerate(zip(host_out, runner.outs)):
            s_down.wait_event(ev_cmp[runner.out_call[i]])
            with torch.cuda.stream(s_down):
                ho.copy_(o, non_blocking=True)
            ev_down[i].record(s_down)
        state["first"] = False

    one()
    torch.cuda.synchronize()
    state["first"] = True
    e0.record(main)
    for s in (s_up, s_cmp, s_down):
        s.wait_stream(main)
    for _ in range(steps):
        one()
    for s in (s_up, s_cmp, s_down):
        main.wait_stream(s)
    e1.record(main)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    ms = ranks.max_over_ranks([ms], dist, dev)[0]
    return {"value": ranks.job_throughput(w.token_heads, world, steps, ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "overlap": "per call: H2D, kernels and D2H on three streams"}


if __name__ == "__main__":
    main()
