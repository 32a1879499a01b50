#!/usr/bin/env python
"""Benchmark of the rotated W4A4 linear layer on B200.

Default workload: the DiT action-head MLP stack (50 action tokens x batch 1,
hidden 1024, gate/up 1024->4096 and down 4096->1024, 4 layers, bf16 input,
10 denoising steps, per-step scale table [10][12], rotation block 64).
One timed step = one denoising step = 12 rotated W4A4 linears: one batched
rotate-quantise launch for all 12, then one batched W4A4 GEMM launch for all 12
(the step's linears are independent: each draws its own input), replayed from a
CUDA graph.  The same step with one launch per kernel and linear is reported
beside it.
The activation step index is a device scalar read by the rotate-quantise
kernel.  L2 is flushed (512 MB written, then read back) before every timed step, so every step
streams its packed weights from HBM.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle on the
same workload instead (the reference arm: the pages publish no code to run).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from w4a4_post_quantization_zigzag_b200 import inputs as I  # noqa: E402

METRIC = "µs per DiT denoise step"
UNIT = "us/step"
L2_FLUSH_BYTES = 512 << 20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="dit_mlp_stack",
                   choices=["dit_mlp_stack", "dit_mlp_stack_fused", "dit_denoise_loop",
                            "backbone_prefill", "single_linear"])
    p.add_argument("--rotation", default="composite", choices=["composite", "hadamard"],
                   help="composite: R = R_SVD.H (the method); hadamard: R_SVD = I variant")
    p.add_argument("--precision", default="w4a4", choices=["w4a4", "w8a8", "mix"],
                   help="w8a8: every linear W8A8 (dynamic per-token 8-bit activations); "
                        "mix: the down projections W8A8, the rest W4A4")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-sample-steps", type=int, default=0,
                   help="oracle steps for the CPU baseline (0: sized to ~15 s)")
    p.add_argument("--quick", action="store_true",
                   help="skip clocks, e2e and the CPU baseline (for profiler runs)")
    return p.parse_args()


def make_workload(name, rotation="composite"):
    wl = {"dit_mlp_stack": I.dit_mlp_stack, "dit_denoise_loop": I.dit_denoise_loop,
          "dit_mlp_stack_fused": lambda: I.dit_mlp_stack(fuse_gate_up=True),
          "backbone_prefill": I.backbone_prefill, "single_linear": I.single_linear}[name]()
    if rotation == "hadamard":
        wl.name += "_hadamard_only"
    wl.rotation = rotation
    return wl


def kernel_nodes(raw_graph):
    """Kernel nodes of a captured CUDA graph (every one a launch of this library)."""
    from cuda.bindings import runtime as rt
    if isinstance(raw_graph, int):
        raw_graph = rt.cudaGraph_t(init_value=raw_graph)
    err, _, n = rt.cudaGraphGetNodes(raw_graph)
    assert err == rt.cudaError_t.cudaSuccess, err
    err, nodes, n = rt.cudaGraphGetNodes(raw_graph, n)
    assert err == rt.cudaError_t.cudaSuccess, err
    kinds = [rt.cudaGraphNodeGetType(nd)[1] for nd in nodes[:n]]
    return sum(k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel for k in kinds)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = [r.split(",") for r in (self.out or "").strip().splitlines() if r.strip()]
        rows = [[c.strip() for c in r] for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ traffic record
def recorded_traffic(kernel, workload):
    """dram bytes per launch from a committed ncu summary, only while the kernel
    source is unchanged since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(f"{kernel}:{workload}")
    if not rec:
        return None
    src = os.path.join(ROOT, "w4a4_post_quantization_zigzag_b200", "csrc", rec["source"])
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != rec["sha256_16"]:
            return None
    return float(rec["dram_bytes_per_launch"])


# --------------------------------------------------------- replica timing
def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank timing over all ranks (identity without a process
    group).  Every rank must call it at the same point."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    if device is None:
        device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_time_per_unit(total_ms: float, steps: int, world: int) -> float:
    """Job-level microseconds per unit of work: N replicas each run `steps`
    units in (max over ranks) total_ms."""
    return total_ms * 1e3 / (steps * world)


# ------------------------------------------------------------- CPU oracle
def oracle_step(wl, packs, xs, t):
    from oracle import qvla_oracle as O
    out = []
    for lin, pk, x in zip(wl.linears, packs, xs[t]):
        if wl.mode == "table":
            r = O.linear_forward(x, pk, "table", wl.table, t, lin.layer)
        else:
            r = O.linear_forward(x, pk)
        out.append(r["y"])
    return out


def oracle_setup(wl, steps):
    from oracle import qvla_oracle as O
    pack = O.pack_linear_hadamard if getattr(wl, "rotation", "") == "hadamard" else O.pack_linear
    packs = [pack(l.make_w(), l.block, bias=l.make_bias()) for l in wl.linears]
    xs = [[l.make_x(seed_offset=t, std=(float(wl.sigmas[t]) if wl.sigmas is not None else None))
           for l in wl.linears] for t in range(steps)]
    return packs, xs


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(wl, sample_steps):
    T = max(1, wl.steps)
    packs, xs = oracle_setup(wl, min(T, max(1, sample_steps)))
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_step(wl, packs, xs, n % len(xs))
        n += 1
        el = time.perf_counter() - t0
        if (sample_steps and n >= sample_steps) or (not sample_steps and (el > 12.0 or n >= 50)):
            break
    us = el / n * 1e6
    return {"value": us, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} full denoise step(s) of {wl.name} ({len(wl.linears)} linears each); "
                      f"numpy fp64 rotation, fp32 RTN, int64 GEMM, fp64 dequant"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = make_workload(args.workload, args.rotation)
    packs, xs = oracle_setup(wl, min(max(1, wl.steps), 2))
    for i in range(args.warmup):
        oracle_step(wl, packs, xs, i % len(xs))
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_step(wl, packs, xs, i % len(xs))
    el = time.perf_counter() - t0
    us = el / args.steps * 1e6
    line = {"impl": "reference", "metric": METRIC, "value": us, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name},
            "cpu_baseline": {"value": us, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": f"each step: one full denoise step of {wl.name}"},
            "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- ours
def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    from w4a4_post_quantization_zigzag_b200 import build as B
    B.build()
    from w4a4_post_quantization_zigzag_b200 import qvla as Q

    wl = make_workload(args.workload, args.rotation)
    T = max(1, wl.steps)
    table = torch.from_numpy(wl.table).to(dev) if wl.table is not None else None
    steps_dev = torch.arange(T, dtype=torch.int32, device=dev)
    mode = Q.QVLA_SCALE_TABLE if wl.mode == "table" else Q.QVLA_SCALE_DYNAMIC

    # pack (offline step, timed for information)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    # which linears run W8A8 (dynamic 8-bit activations, one launch sequence
    # each) and which W4A4 (batched)
    w8 = [args.precision == "w8a8" or (args.precision == "mix" and lin.name.endswith("down"))
          for lin in wl.linears]
    packs = []
    for lin, is8 in zip(wl.linears, w8):
        W = torch.from_numpy(lin.make_w()).to(dev)
        pack = (Q.qvla_pack_weights_w8 if is8 else
                Q.qvla_pack_weights_hadamard if wl.rotation == "hadamard" else Q.qvla_pack_weights)
        packs.append(pack(W, lin.block, bias=torch.from_numpy(lin.make_bias()).to(dev)))
        del W
    torch.cuda.synchronize()
    pack_s = time.perf_counter() - t0

    # per-step inputs (device resident) and outputs
    xdt = torch.bfloat16 if wl.linears[0].x_dtype == "bf16" else torch.float32
    xs_host = [[torch.from_numpy(l.make_x(seed_offset=t, std=(float(wl.sigmas[t])
                                                              if wl.sigmas is not None else None)))
                .to(xdt).pin_memory() for l in wl.linears] for t in range(T)]
    xs = [[x.to(dev) for x in row] for row in xs_host]
    xq = [torch.empty(l.M, l.K, dtype=torch.int8, device=dev) if is8 else
          torch.empty(l.M, l.K // 2, dtype=torch.uint8, device=dev)
          for l, is8 in zip(wl.linears, w8)]
    sx = [torch.empty(l.M, dtype=torch.float32, device=dev) for l in wl.linears]
    ys = [torch.empty(l.M, l.N, dtype=torch.bfloat16, device=dev) for l in wl.linears]
    # scratch of the tensor-core rotation route (the permuted copy of x; for a
    # W8A8 linear also its fp32 rotated rows), one per linear since a batched
    # launch runs them together
    wss = [torch.empty(max(Q.qvla_rotate_quant_a8_workspace_bytes(l.M, l.K) if is8 else
                           Q.qvla_rotate_quant_workspace_bytes(l.M, l.K, l.block), 16),
                       dtype=torch.uint8, device=dev) for l, is8 in zip(wl.linears, w8)]
    nl = len(wl.linears)
    # one problem set per denoising step: same packed weights and buffers, the
    # step's own inputs and device step index
    probs = [[Q.LinearProblem(L, xs[t][i], mode, table=table, step=steps_dev[t:t + 1],
                              layer=lin.layer, xq=xq[i], s_x=sx[i], y=ys[i], workspace=wss[i])
              for i, (lin, L) in enumerate(zip(wl.linears, packs)) if not w8[i]]
             for t in range(T)]
    idx8 = [i for i in range(len(wl.linears)) if w8[i]]

    def w8_linears(t, phase):
        for i in idx8:
            if phase == 0:
                Q.qvla_rotate_quant_act_a8(xs[t][i], packs[i], xq8=xq[i], s_x=sx[i],
                                           workspace=wss[i])
            else:
                Q.qvla_w8a8_gemm(xq[i], sx[i], packs[i], y=ys[i])

    def step_batched(t, rec=None):
        if rec is not None:
            rec[0].record()
        if probs[t]:
            Q.qvla_rotate_quant_act_batched(probs[t])
        w8_linears(t, 0)
        if rec is not None:
            rec[1].record()
        if probs[t]:
            Q.qvla_w4a4_gemm_batched(probs[t])
        w8_linears(t, 1)
        if rec is not None:
            rec[2].record()

    def step_per_linear(t):
        for i, (lin, L) in enumerate(zip(wl.linears, packs)):
            if w8[i]:
                Q.qvla_rotate_quant_act_a8(xs[t][i], L, xq8=xq[i], s_x=sx[i], workspace=wss[i])
                Q.qvla_w8a8_gemm(xq[i], sx[i], L, y=ys[i])
                continue
            Q.qvla_rotate_quant_act(xs[t][i], L, mode, table=table, step=steps_dev[t:t + 1],
                                    layer=lin.layer, xq=xq[i], s_x=sx[i], workspace=wss[i])
            Q.qvla_w4a4_gemm(xq[i], sx[i], L, y=ys[i])

    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def l2_flush():
        """Cold L2 for the next step: write a buffer four times the L2, then
        read it back, so the write-backs of the flush itself happen here and
        not inside the timed step."""
        flush.zero_()
        flush.sum()

    def capture(fn):
        """One graph per denoising step; also returns the kernel nodes in each."""
        gs, nk = [], []
        for t in range(T):
            g = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(g, stream=stream):
                fn(t)
            nk.append(kernel_nodes(g.raw_cuda_graph()))
            g.instantiate()
            gs.append(g)
        return gs, nk

    with torch.cuda.stream(stream):
        step_batched(0)               # first calls resolve attributes outside capture
        step_per_linear(0)
        torch.cuda.synchronize()
        graphs, kernels_per_step = capture(step_batched)
        graphs_pl, _ = capture(step_per_linear)
    torch.cuda.synchronize()
    assert Q.qvla_read_error_word(clear=True) == 0

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def timed_replays(gs, n, flush_l2=True):
        starts = [ev() for _ in range(n)]
        ends = [ev() for _ in range(n)]
        with torch.cuda.stream(stream):
            for i in range(n):
                if flush_l2:
                    l2_flush()
                starts[i].record()
                gs[i % T].replay()
                ends[i].record()
        return starts, ends

    # ---- warm-up
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            l2_flush()
            graphs[i % T].replay()
            l2_flush()
            graphs_pl[i % T].replay()
    # ---- timed steps: graph replay of the batched step, L2 flushed before each
    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_uuid) if not args.quick else None
    barrier()
    if sampler:
        sampler.__enter__()
    starts, ends = timed_replays(graphs, args.steps)
    barrier()
    if sampler:
        sampler.__exit__()
    per_step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    tot_ms = max_over_ranks(sum(per_step_ms), dev)
    ms_per_step = tot_ms / args.steps
    us_job = job_time_per_unit(tot_ms, args.steps, world)

    # ---- the same steps, one launch per kernel and linear (informational)
    s2, e2 = timed_replays(graphs_pl, args.steps)
    torch.cuda.synchronize()
    per_linear_us = sum(a.elapsed_time(b) for a, b in zip(s2, e2)) * 1e3 / args.steps

    # ---- the batched step with a warm L2 (no flush between steps; informational)
    sw_, ew_ = timed_replays(graphs, args.steps, flush_l2=False)
    torch.cuda.synchronize()
    warm_us = sum(a.elapsed_time(b) for a, b in zip(sw_, ew_)) * 1e3 / args.steps

    # ---- per-kernel breakdown: eager launches with events on the launching
    # stream; a GPU sleep ahead of the events keeps host enqueue time out
    krot, kgemm = [], []
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            rec = [ev(), ev(), ev()]
            l2_flush()
            torch.cuda._sleep(2_000_000)
            step_batched(i % T, rec)
            stream.synchronize()
            krot.append(rec[0].elapsed_time(rec[1]))
            kgemm.append(rec[1].elapsed_time(rec[2]))
    assert Q.qvla_read_error_word(clear=True) == 0

    # ---- end to end: pinned-host inputs in, outputs back, every step
    e2e = None
    if not args.quick:
        y_host = [torch.empty(l.M, l.N, dtype=torch.bfloat16).pin_memory() for l in wl.linears]
        h2d = sum(x.numel() * x.element_size() for x in xs_host[0])
        d2h = sum(y.numel() * y.element_size() for y in y_host)
        e0, e1 = ev(), ev()
        barrier()
        with torch.cuda.stream(stream):
            e0.record()
            for i in range(args.steps):
                t = i % T
                for x_d, x_h in zip(xs[t], xs_host[t]):
                    x_d.copy_(x_h, non_blocking=True)
                graphs[t].replay()
                for y_d, y_h in zip(ys, y_host):
                    y_h.copy_(y_d, non_blocking=True)
            e1.record()
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e = {"value": job_time_per_unit(e2e_ms, args.steps, world), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # ---- roofline of the dominant kernel
    hbm, bf16_tf, peak_src = load_peaks()
    cb = [1.0 if is8 else 0.5 for is8 in w8]          # code bytes per element
    gemm_bytes = sum(int(l.N * l.K * c) + int(l.M * l.K * c) + 2 * l.M * l.N + 4 * l.M + 8 * l.N
                     for l, c in zip(wl.linears, cb))
    rot_bytes = sum((2 if l.x_dtype == "bf16" else 4) * l.M * l.K + int(l.M * l.K * c) + 4 * l.M
                    + (4 * l.K * l.block if wl.rotation != "hadamard" else 0) + 4 * l.K
                    for l, c in zip(wl.linears, cb))
    weight_bytes = sum(int(l.N * l.K * c) + 8 * l.N for l, c in zip(wl.linears, cb))
    t_gemm = sum(kgemm) / args.steps          # ms per step (one batched launch)
    t_rot = sum(krot) / args.steps
    dom = "w4a4_gemm" if t_gemm >= t_rot else "rotate_quant"
    if dom == "w4a4_gemm":
        per_launch_bytes, per_launch_ms = gemm_bytes, t_gemm
    else:
        per_launch_bytes, per_launch_ms = rot_bytes, t_rot
    achieved = per_launch_bytes / (per_launch_ms * 1e-3) / 1e9
    roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "peak_source": f"hbm_gbs ({peak_src})",
            "traffic": recorded_traffic(dom, wl.name),
            "algorithmic_bytes_per_launch": per_launch_bytes,
            "avg_launch_us": per_launch_ms * 1e3}

    ops = wl.ops_per_step()
    line = {
        "metric": METRIC, "value": us_job, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": {"workload": wl.name, "rotation": wl.rotation, "precision": args.precision,
                   "w8a8_linears": len(idx8), "tokens_M": wl.linears[0].M,
                   "linears_per_step": nl, "denoise_steps_T": T,
                   "block": wl.linears[0].block, "scale": wl.mode,
                   "l2": "flushed before every timed step (512 MB written, then read back: cold, clean L2)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single"},
        "roofline": roof,
        "tops": ops / (ms_per_step * 1e-3) / 1e12,
        "tops_frac_int8": ops / (ms_per_step * 1e-3) / 1e12 / (2.0 * bf16_tf),
        "int8_peak_tops": {"value": 2.0 * bf16_tf,
                           "source": f"2 x bf16_tflops ({peak_src}; dense int8 : bf16 = 2 : 1)"},
        "l2_warm_us_per_step": warm_us,
        "weight_gbs": weight_bytes / (ms_per_step * 1e-3) / 1e9,
        "kernels_us_per_step": {"rotate_quant": t_rot * 1e3, "w4a4_gemm": t_gemm * 1e3},
        "per_linear_launches_us_per_step": per_linear_us,
        "pack_s": pack_s,
        "gpu_launches": sum(kernels_per_step[i % T] for i in range(args.steps)),
        "kernels_per_step": kernels_per_step[0],
        "e2e": e2e,
    }
    if sampler:
        line["clocks"] = sampler.summary()
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.quick:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_sample_steps)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graphs, graphs_pl
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
