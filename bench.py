#!/usr/bin/env python
"""Benchmark of the rotated W4A4 linear layer on B200.

Default workload: the DiT action-head MLP stack (50 action tokens x batch 1,
hidden 1024, gate/up 1024->4096 and down 4096->1024, 4 layers, bf16 input,
10 denoising steps, per-step scale table [10][12], rotation block 64).
One timed step = one denoising step = 12 rotated W4A4 linears: one batched
rotate-quantise call for all 12 (it also writes the int8 image of the codes
that the GEMM reads), then one batched W4A4 GEMM launch for all 12 (the
step's linears are independent: each draws its own input), replayed from a
CUDA graph.  The same step with one call per kernel and linear is reported
beside it.
The activation step index is a device scalar read by the rotate-quantise
kernel.  L2 is flushed (512 MB written, then read back) before every timed
step, so every step streams its packed weights and rotations from HBM.

Besides the headline workload, the same line carries shorter measurements
of the backbone prefill linears (1024 tokens, 2048<->16384) and of the full
DiT denoise loop (512 tokens, 16 layers) under "secondary".

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

import numpy as np  # noqa: E402,F401

from w4a4_post_quantization_zigzag_b200 import inputs as I  # noqa: E402

METRIC = "µs per DiT denoise step"
UNIT = "us/step"
L2_FLUSH_BYTES = 512 << 20
WORKLOADS = ("dit_mlp_stack", "dit_mlp_stack_fused", "dit_denoise_loop",
             "dit_denoise_loop_fused", "backbone_prefill", "single_linear")
SECONDARY = ("backbone_prefill", "dit_denoise_loop")


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="dit_mlp_stack", choices=WORKLOADS)
    p.add_argument("--rotation", default="composite", choices=["composite", "hadamard"],
                   help="composite: R = R_SVD.H (the method); hadamard: R_SVD = I variant")
    p.add_argument("--precision", default="w4a4", choices=["w4a4", "w8a8", "mix"],
                   help="w8a8: every linear W8A8 (dynamic per-token 8-bit activations); "
                        "mix: the down projections W8A8, the rest W4A4")
    p.add_argument("--no-image", action="store_true",
                   help="batched GEMM unpacks the packed codes instead of reading the image")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-secondary", action="store_true")
    p.add_argument("--secondary-steps", type=int, default=3)
    p.add_argument("--cpu-sample-steps", type=int, default=0,
                   help="oracle steps for the CPU baseline (0: sized to ~15 s)")
    p.add_argument("--quick", action="store_true",
                   help="skip clocks, e2e, the CPU baseline and the secondary workloads "
                        "(for profiler runs)")
    return p.parse_args(argv)


def make_workload(name, rotation="composite"):
    wl = {"dit_mlp_stack": I.dit_mlp_stack, "dit_denoise_loop": I.dit_denoise_loop,
          "dit_mlp_stack_fused": lambda: I.dit_mlp_stack(fuse_gate_up=True),
          "dit_denoise_loop_fused": lambda: I.dit_denoise_loop(fuse_qkv=True),
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
    """(HBM GB/s, bf16 TFLOP/s burst, source) from the machine's measured peaks,
    else the recipe's fallback figures."""
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
        self.out = ""

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


# ------------------------------------------------------- roofline arithmetic
def algorithmic_work(wl, w8, rotation="composite"):
    """Per-step algorithmic bytes and ops of the two kernels (the work the
    method must do, not what an implementation happens to move):
      GEMM: N*K*c weights + M*K*c codes + 2*M*N bf16 out + 4*M s_x + 8*N s_w
            and bias (c = bytes per code: 1/2 for 4-bit, 1 for 8-bit);
            ops 2*M*N*K.
      rotate-quantise: e_x*M*K input + M*K*c codes + 4*M scales + 4*K*b
            R_SVD (fp32; none for the Hadamard-only variant) + 4*K perm."""
    cb = [1.0 if is8 else 0.5 for is8 in w8]
    gemm_bytes = sum(int(l.N * l.K * c) + int(l.M * l.K * c) + 2 * l.M * l.N + 4 * l.M + 8 * l.N
                     for l, c in zip(wl.linears, cb))
    gemm_ops = sum(2 * l.M * l.N * l.K for l in wl.linears)
    rot_bytes = sum((2 if l.x_dtype == "bf16" else 4) * l.M * l.K + int(l.M * l.K * c) + 4 * l.M
                    + (4 * l.K * l.block if rotation != "hadamard" else 0) + 4 * l.K
                    for l, c in zip(wl.linears, cb))
    weight_bytes = sum(int(l.N * l.K * c) + 8 * l.N for l, c in zip(wl.linears, cb))
    return gemm_bytes, gemm_ops, rot_bytes, weight_bytes


def roofline_entry(kernel, t_ms, nbytes, ops, hbm_gbs, int8_tops, peak_src, workload):
    """Achieved vs peak for one kernel's per-step launch(es).  The bound is the
    larger of bytes / HBM bandwidth and ops / int8 tensor peak."""
    t_hbm = nbytes / (hbm_gbs * 1e9)
    t_ten = ops / (int8_tops * 1e12) if ops else 0.0
    if t_ten > t_hbm:
        ach = ops / (t_ms * 1e-3) / 1e12
        ent = {"kernel": kernel, "bound": "tensor", "achieved": ach, "peak": int8_tops,
               "unit": "TOPS", "frac": ach / int8_tops,
               "peak_source": f"2 x bf16_tflops ({peak_src}; dense int8 : bf16 = 2 : 1)"}
    else:
        ach = nbytes / (t_ms * 1e-3) / 1e9
        ent = {"kernel": kernel, "bound": "hbm", "achieved": ach, "peak": hbm_gbs,
               "unit": "GB/s", "frac": ach / hbm_gbs, "peak_source": f"hbm_gbs ({peak_src})"}
    ent.update({"traffic": recorded_traffic(kernel, workload),
                "algorithmic_bytes_per_launch": nbytes, "ops_per_launch": ops,
                "avg_launch_us": t_ms * 1e3})
    return ent


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


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


THREADING_NOTE = ("numpy fp64 rotation products and Gram eigensolves on the BLAS/LAPACK "
                  "threads; the fp32 RTN, the int64 GEMM (numpy integer matmul, no BLAS) "
                  "and the dequantisation on one core")


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
    return {"value": us, "unit": UNIT, "cores": host_cores(), "blas_threads": blas_threads(),
            "threading": THREADING_NOTE, "kind": "oracle",
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
            "cpu_baseline": {"value": us, "unit": UNIT, "cores": host_cores(),
                             "blas_threads": blas_threads(), "threading": THREADING_NOTE,
                             "kind": "oracle",
                             "sample": f"each step: one full denoise step of {wl.name}"},
            "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- ours
class DeviceStep:
    """One workload on the device: packed linears, per-step inputs (device
    resident; each step's inputs are one contiguous buffer, mirrored in pinned
    host memory), outputs (one contiguous buffer), scratch, and the batched and
    per-linear step functions."""

    def __init__(self, wl, Q, dev, precision="w4a4", image=True, pack_fn=None):
        """pack_fn(lin, W, bias) -> packed linear replaces the default pack
        (tests pass one that feeds the oracle's permutation and R_SVD)."""
        import torch
        self.wl, self.Q, self.dev = wl, Q, dev
        self.T = T = max(1, wl.steps)
        self.table = torch.from_numpy(wl.table).to(dev) if wl.table is not None else None
        self.steps_dev = torch.arange(T, dtype=torch.int32, device=dev)
        self.mode = Q.QVLA_SCALE_TABLE if wl.mode == "table" else Q.QVLA_SCALE_DYNAMIC
        self.w8 = [precision == "w8a8" or (precision == "mix" and lin.name.endswith("down"))
                   for lin in wl.linears]
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        self.packs = []
        for lin, is8 in zip(wl.linears, self.w8):
            W = torch.from_numpy(lin.make_w()).to(dev)
            b = torch.from_numpy(lin.make_bias()).to(dev)
            if pack_fn is not None:
                self.packs.append(pack_fn(lin, W, b))
            else:
                pack = (Q.qvla_pack_weights_w8 if is8 else
                        Q.qvla_pack_weights_hadamard if wl.rotation == "hadamard" else
                        Q.qvla_pack_weights)
                self.packs.append(pack(W, lin.block, bias=b))
            del W
        torch.cuda.synchronize()
        self.pack_s = time.perf_counter() - t0

        xdt = torch.bfloat16 if wl.linears[0].x_dtype == "bf16" else torch.float32

        def carve(flat, shapes):
            """Row-major views [r, c] of a flat buffer, each 16-byte aligned."""
            out, off = [], 0
            step = 16 // flat.element_size()
            for r, c in shapes:
                out.append(flat[off:off + r * c].view(r, c))
                off += r * c + (-(r * c)) % step
            return out

        def total(shapes, esz):
            step = 16 // esz
            return sum(r * c + (-(r * c)) % step for r, c in shapes)

        xshapes = [(l.M, l.K) for l in wl.linears]
        xtot = total(xshapes, 2 if xdt == torch.bfloat16 else 4)
        self.x_host, self.x_dev, self.xs = [], [], []
        for t in range(T):
            hb = torch.empty(xtot, dtype=xdt).pin_memory()
            std = float(wl.sigmas[t]) if wl.sigmas is not None else None
            for v, l in zip(carve(hb, xshapes), wl.linears):
                v.copy_(torch.from_numpy(l.make_x(seed_offset=t, std=std)).to(xdt))
            db = hb.to(dev)
            self.x_host.append(hb)
            self.x_dev.append(db)
            self.xs.append(carve(db, xshapes))
        yshapes = [(l.M, l.N) for l in wl.linears]
        self.y_dev = torch.empty(total(yshapes, 2), dtype=torch.bfloat16, device=dev)
        self.ys = carve(self.y_dev, yshapes)
        self.xq = [torch.empty(l.M, l.K, dtype=torch.int8, device=dev) if is8 else
                   torch.empty(l.M, l.K // 2, dtype=torch.uint8, device=dev)
                   for l, is8 in zip(wl.linears, self.w8)]
        self.sx = [torch.empty(l.M, dtype=torch.float32, device=dev) for l in wl.linears]
        # scratch of the tensor-core rotation route (the permuted copy of x; for a
        # W8A8 linear also its fp32 rotated rows), one per linear since a batched
        # launch runs them together
        self.wss = [torch.empty(max(Q.qvla_rotate_quant_a8_workspace_bytes(l.M, l.K) if is8 else
                                    Q.qvla_rotate_quant_workspace_bytes(l.M, l.K, l.block), 16),
                                dtype=torch.uint8, device=dev)
                    for l, is8 in zip(wl.linears, self.w8)]
        # the int8 image of each W4A4 linear's codes: written by the batched
        # rotate-quantise, read by the batched GEMM
        self.img = [torch.empty(l.M, l.K, dtype=torch.int8, device=dev)
                    if (image and not is8) else None for l, is8 in zip(wl.linears, self.w8)]
        self.probs = [[Q.LinearProblem(L, self.xs[t][i], self.mode, table=self.table,
                                       step=self.steps_dev[t:t + 1], layer=lin.layer,
                                       xq=self.xq[i], s_x=self.sx[i], y=self.ys[i],
                                       workspace=self.wss[i], xq8=self.img[i])
                       for i, (lin, L) in enumerate(zip(wl.linears, self.packs)) if not self.w8[i]]
                      for t in range(T)]
        self.idx8 = [i for i in range(len(wl.linears)) if self.w8[i]]
        # the W8A8 linears as batched problems: xq8 holds their 8-bit codes
        # (the packed-code field is unused for them: one shared dummy each)
        dummy = {i: torch.empty(wl.linears[i].M, wl.linears[i].K // 2, dtype=torch.uint8,
                                device=dev) for i in self.idx8}
        self.probs8 = [[Q.LinearProblem(self.packs[i], self.xs[t][i], xq=dummy[i], s_x=self.sx[i],
                                        y=self.ys[i], workspace=self.wss[i], xq8=self.xq[i])
                        for i in self.idx8] for t in range(T)]

    def w8_linears(self, t, phase):
        """The W8A8 linears of the step: one batched 8-bit activation pass,
        then one batched W8A8 GEMM."""
        if not self.idx8:
            return
        if phase == 0:
            self.Q.qvla_rotate_quant_act_a8_batched(self.probs8[t])
        else:
            self.Q.qvla_w8a8_gemm_batched(self.probs8[t])

    def step_batched(self, t, rec=None):
        Q = self.Q
        if rec is not None:
            rec[0].record()
        if self.probs[t]:
            Q.qvla_rotate_quant_act_batched(self.probs[t])
        self.w8_linears(t, 0)
        if rec is not None:
            rec[1].record()
        if self.probs[t]:
            Q.qvla_w4a4_gemm_batched(self.probs[t])
        self.w8_linears(t, 1)
        if rec is not None:
            rec[2].record()

    def step_per_linear(self, t):
        Q = self.Q
        for i, (lin, L) in enumerate(zip(self.wl.linears, self.packs)):
            if self.w8[i]:
                Q.qvla_rotate_quant_act_a8(self.xs[t][i], L, xq8=self.xq[i], s_x=self.sx[i],
                                           workspace=self.wss[i])
                Q.qvla_w8a8_gemm(self.xq[i], self.sx[i], L, y=self.ys[i])
                continue
            Q.qvla_rotate_quant_act(self.xs[t][i], L, self.mode, table=self.table,
                                    step=self.steps_dev[t:t + 1], layer=lin.layer, xq=self.xq[i],
                                    s_x=self.sx[i], workspace=self.wss[i])
            Q.qvla_w4a4_gemm(self.xq[i], self.sx[i], L, y=self.ys[i])


def measure(ds, stream, steps, warmup, *, per_linear=True, warm=True, e2e=False,
            sampler=None, barrier=None):
    """Graph-replayed timing of one DeviceStep; returns a dict (ms values)."""
    import torch
    Q, T = ds.Q, ds.T
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=ds.dev)

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
        ds.step_batched(0)               # first calls resolve attributes outside capture
        if per_linear:
            ds.step_per_linear(0)
        torch.cuda.synchronize()
        graphs, kernels_per_step = capture(ds.step_batched)
        graphs_pl = capture(ds.step_per_linear)[0] if per_linear else None
    torch.cuda.synchronize()
    assert Q.qvla_read_error_word(clear=True) == 0
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    barrier = barrier or torch.cuda.synchronize

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

    with torch.cuda.stream(stream):
        for i in range(warmup):
            l2_flush()
            graphs[i % T].replay()
            if graphs_pl:
                l2_flush()
                graphs_pl[i % T].replay()
    barrier()
    if sampler:
        sampler.__enter__()
    starts, ends = timed_replays(graphs, steps)
    barrier()
    if sampler:
        sampler.__exit__()
    out = {"step_ms": [a.elapsed_time(b) for a, b in zip(starts, ends)],
           "kernels_per_step": kernels_per_step}
    if graphs_pl:
        s2, e2 = timed_replays(graphs_pl, steps)
        torch.cuda.synchronize()
        out["per_linear_ms"] = sum(a.elapsed_time(b) for a, b in zip(s2, e2)) / steps
    if warm:
        sw, ew = timed_replays(graphs, steps, flush_l2=False)
        torch.cuda.synchronize()
        out["warm_ms"] = sum(a.elapsed_time(b) for a, b in zip(sw, ew)) / steps
    # per-kernel breakdown: eager calls with events on the launching stream; a
    # GPU sleep ahead of the events keeps host enqueue time out
    krot, kgemm = [], []
    with torch.cuda.stream(stream):
        for i in range(steps):
            rec = [ev(), ev(), ev()]
            l2_flush()
            torch.cuda._sleep(2_000_000)
            ds.step_batched(i % T, rec)
            stream.synchronize()
            krot.append(rec[0].elapsed_time(rec[1]))
            kgemm.append(rec[1].elapsed_time(rec[2]))
    assert Q.qvla_read_error_word(clear=True) == 0
    out["rot_ms"] = sum(krot) / steps
    out["gemm_ms"] = sum(kgemm) / steps
    if e2e:
        # end to end: each step's inputs copied in from pinned host memory (one
        # contiguous copy), the step replayed, all outputs copied back (one
        # contiguous copy), inside the timed region
        y_host = torch.empty(ds.y_dev.shape, dtype=ds.y_dev.dtype).pin_memory()
        e0, e1 = ev(), ev()
        barrier()
        with torch.cuda.stream(stream):
            e0.record()
            for i in range(steps):
                t = i % T
                ds.x_dev[t].copy_(ds.x_host[t], non_blocking=True)
                graphs[t].replay()
                y_host.copy_(ds.y_dev, non_blocking=True)
            e1.record()
        barrier()
        out["e2e_ms"] = e0.elapsed_time(e1)
        out["h2d_bytes"] = ds.x_host[0].numel() * ds.x_host[0].element_size()
        out["d2h_bytes"] = y_host.numel() * y_host.element_size()
    del graphs, graphs_pl
    return out


def secondary_line(name, Q, dev, stream, steps, peaks):
    """Shorter measurement of another workload (graph replay, L2 flushed)."""
    import torch
    hbm, bf16_tf, src = peaks
    wl = make_workload(name)
    ds = DeviceStep(wl, Q, dev)
    m = measure(ds, stream, steps, 2, per_linear=False, warm=False)
    us = sum(m["step_ms"]) / steps * 1e3
    gb, gops, rb, _ = algorithmic_work(wl, ds.w8)
    r = {"workload": wl.name, "value": us, "unit": UNIT, "steps": steps,
         "kernels_us_per_step": {"rotate_quant": m["rot_ms"] * 1e3,
                                 "w4a4_gemm": m["gemm_ms"] * 1e3},
         "tops": gops / (us * 1e-6) / 1e12,
         "rooflines": [roofline_entry("rotate_quant", m["rot_ms"], rb, 0, hbm, 2 * bf16_tf, src,
                                      wl.name),
                       roofline_entry("w4a4_gemm", m["gemm_ms"], gb, gops, hbm, 2 * bf16_tf,
                                      src, wl.name)],
         "kernels_per_step": m["kernels_per_step"][0],
         "pack_s": ds.pack_s}
    del ds
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return r


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
    ds = DeviceStep(wl, Q, dev, args.precision, image=not args.no_image)
    stream = torch.cuda.Stream(device=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    gpu_uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_uuid) if not args.quick else None
    m = measure(ds, stream, args.steps, args.warmup, e2e=not args.quick, sampler=sampler,
                barrier=barrier)
    tot_ms = max_over_ranks(sum(m["step_ms"]), dev)
    ms_per_step = tot_ms / args.steps
    us_job = job_time_per_unit(tot_ms, args.steps, world)
    e2e = None
    if "e2e_ms" in m:
        e2e_ms = max_over_ranks(m["e2e_ms"], dev)
        e2e = {"value": job_time_per_unit(e2e_ms, args.steps, world), "unit": UNIT,
               "h2d_bytes_per_step": m["h2d_bytes"], "d2h_bytes_per_step": m["d2h_bytes"]}

    # ---- rooflines: every kernel of the step, the dominant one on top
    peaks = load_peaks()
    hbm, bf16_tf, peak_src = peaks
    gb, gops, rb, wb = algorithmic_work(wl, ds.w8, wl.rotation)
    roofs = [roofline_entry("rotate_quant", m["rot_ms"], rb, 0, hbm, 2 * bf16_tf, peak_src,
                            wl.name),
             roofline_entry("w4a4_gemm", m["gemm_ms"], gb, gops, hbm, 2 * bf16_tf, peak_src,
                            wl.name)]
    dom = max(roofs, key=lambda r: r["avg_launch_us"])
    ops = wl.ops_per_step()
    kps = m["kernels_per_step"]
    line = {
        "metric": METRIC, "value": us_job, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8", "data": "synthetic",
        "config": {"workload": wl.name, "rotation": wl.rotation, "precision": args.precision,
                   "w8a8_linears": len(ds.idx8), "tokens_M": wl.linears[0].M,
                   "linears_per_step": len(wl.linears), "denoise_steps_T": ds.T,
                   "block": wl.linears[0].block, "scale": wl.mode,
                   "gemm_activations": "packed codes" if args.no_image else "int8 image",
                   "l2": "flushed before every timed step (512 MB written, then read back: "
                         "cold, clean L2)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single"},
        "roofline": dom,
        "rooflines": roofs,
        "tops": ops / (ms_per_step * 1e-3) / 1e12,
        "tops_frac_int8": ops / (ms_per_step * 1e-3) / 1e12 / (2.0 * bf16_tf),
        "int8_peak_tops": {"value": 2.0 * bf16_tf,
                           "source": f"2 x bf16_tflops ({peak_src}; dense int8 : bf16 = 2 : 1)"},
        "weight_gbs": wb / (ms_per_step * 1e-3) / 1e9,
        "kernels_us_per_step": {"rotate_quant": m["rot_ms"] * 1e3,
                                "w4a4_gemm": m["gemm_ms"] * 1e3},
        "per_linear_launches_us_per_step": m.get("per_linear_ms", 0.0) * 1e3,
        "l2_warm_us_per_step": m.get("warm_ms", 0.0) * 1e3,
        "pack_s": ds.pack_s,
        "gpu_launches": sum(kps[i % ds.T] for i in range(args.steps)),
        "kernels_per_step": kps[0],
        "source_hash": Q.qvla_source_hash()[:16],
        "e2e": e2e,
    }
    if sampler:
        line["clocks"] = sampler.summary()
    del ds
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if not args.quick and not args.no_secondary and args.workload == "dit_mlp_stack" \
            and args.rotation == "composite" and args.precision == "w4a4":
        # every rank runs the same secondary work (no collectives inside)
        line["secondary"] = [secondary_line(n, Q, dev, stream, args.secondary_steps, peaks)
                             for n in SECONDARY]
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.quick:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_sample_steps)
    if rank == 0:
        print(json.dumps(line), flush=True)
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
