"""Seeded synthetic inputs for the rotated W4A4 linear layer.

This module is the only code shared by the CUDA path's tests/bench and the CPU
oracle.  It draws random numbers and rounds them to the storage type the layer
is fed (bf16 or fp32); it holds none of the layer's own arithmetic (no
permutation, rotation, scale selection, quantisation or GEMM).

Every generator takes an explicit seed and uses numpy's PCG64 bit generator, so
the same call returns the same array on any host.

Workload recipes follow the shapes and distributions of the Omega-QVLA DiT
action head and VLA backbone described on the pages ("Omega-QVLA: Nén VLA W4A4
trên Edge", section "Build DiT action head pack": block size 64, 4-bit weights
and activations, 8 or 10 denoising steps), with the synthetic stand-ins listed
in each recipe's docstring.  No public dataset or trained checkpoint is used.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

# two-sided 99.9th percentile of |z| for z ~ N(0, 1): P(|z| <= Z999) = 0.999
Z999 = 3.2905267314919255


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32
    holding exactly representable bf16 values.  Inputs here are finite."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exactly bf16."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def activations(seed: int, M: int, K: int, std: float = 1.0,
                n_outlier_cols: int = 0, outlier_scale: float = 20.0,
                heavy_tail_frac: float = 0.0, heavy_tail_nu: float = 3.0,
                heavy_tail_scale: float = 10.0, dtype: str = "bf16") -> np.ndarray:
    """x [M, K] ~ N(0, std^2).  `n_outlier_cols` columns (drawn without
    replacement) are multiplied by `outlier_scale`; a `heavy_tail_frac` share of
    columns is replaced by Student-t(nu) * heavy_tail_scale * std.  Returned as
    float32 holding values exact in `dtype` ("bf16" or "f32")."""
    g = rng(seed)
    x = g.standard_normal((M, K)) * std
    if n_outlier_cols:
        cols = g.choice(K, size=n_outlier_cols, replace=False)
        x[:, cols] *= outlier_scale
    if heavy_tail_frac > 0:
        n = max(1, int(round(heavy_tail_frac * K)))
        cols = g.choice(K, size=n, replace=False)
        x[:, cols] = g.standard_t(heavy_tail_nu, size=(M, n)) * heavy_tail_scale * std
    x = x.astype(np.float32)
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return x
    raise ValueError(dtype)


def weights(seed: int, N: int, K: int, std: float = 0.02, n_outlier_rows: int = 0,
            row_scale: float = 15.0, col_spread: float = 1.0) -> np.ndarray:
    """W [N, K] ~ N(0, std^2) (PyTorch Linear layout: out x in), fp32.
    `n_outlier_rows` rows are scaled by `row_scale`; with col_spread > 1 each
    column k is scaled by col_spread**u_k, u_k ~ U(0, 1) (log-uniform spread of
    column norms between 1x and col_spread x)."""
    g = rng(seed)
    W = g.standard_normal((N, K)) * std
    if n_outlier_rows:
        rows = g.choice(N, size=n_outlier_rows, replace=False)
        W[rows, :] *= row_scale
    if col_spread > 1.0:
        W *= col_spread ** g.uniform(0.0, 1.0, size=(1, K))
    return W.astype(np.float32)


def bias(seed: int, N: int, std: float = 0.01) -> np.ndarray:
    return (rng(seed).standard_normal(N) * std).astype(np.float32)


def step_sigmas(T: int, lo: float = 0.5, hi: float = 3.0) -> np.ndarray:
    """Activation std per denoising step, drifting linearly lo -> hi."""
    if T == 1:
        return np.array([lo])
    return lo + (hi - lo) * np.arange(T) / (T - 1)


def scale_table(seed: int, T: int, L: int, sigmas: np.ndarray, qmax: float = 7.0,
                jitter: float = 0.05) -> np.ndarray:
    """Synthetic per-step, per-layer activation step sizes, fp32 [T, L].

    Stand-in for a table calibrated offline at the 99.9th activation percentile:
    an orthogonal rotation keeps iid Gaussian activations Gaussian with the same
    std, so the percentile of |x'| at step t is Z999 * sigma_t.  Each entry is
    Z999 * sigma_t * (1 + jitter * u) / qmax, u ~ U(-1, 1) per (t, l)."""
    g = rng(seed)
    u = g.uniform(-1.0, 1.0, size=(T, L))
    tab = Z999 * np.asarray(sigmas, dtype=np.float64)[:, None] * (1.0 + jitter * u) / qmax
    return tab.astype(np.float32)


def int_codes(seed: int, rows: int, K: int, lo: int, hi: int) -> np.ndarray:
    """Uniform integer codes in [lo, hi], int8 [rows, K]."""
    return rng(seed).integers(lo, hi + 1, size=(rows, K), dtype=np.int64).astype(np.int8)


def positive_scales(seed: int, n: int, lo: float = 1e-3, hi: float = 1.0) -> np.ndarray:
    return rng(seed).uniform(lo, hi, size=n).astype(np.float32)


# --------------------------------------------------------------------------
# Workload recipes
# --------------------------------------------------------------------------

@dataclass
class Linear:
    """One rotated W4A4 linear: x [M, K] -> y [M, N]."""
    name: str
    M: int
    K: int
    N: int
    block: int
    x_seed: int
    w_seed: int
    b_seed: int
    x_kwargs: dict = field(default_factory=dict)
    w_kwargs: dict = field(default_factory=dict)
    x_dtype: str = "bf16"
    layer: int = 0          # column of the scale table

    def make_x(self, seed_offset: int = 0, std: Optional[float] = None) -> np.ndarray:
        kw = dict(self.x_kwargs)
        if std is not None:
            kw["std"] = std
        return activations(self.x_seed + seed_offset, self.M, self.K, dtype=self.x_dtype, **kw)

    def make_w(self) -> np.ndarray:
        return weights(self.w_seed, self.N, self.K, **self.w_kwargs)

    def make_bias(self) -> np.ndarray:
        return bias(self.b_seed, self.N)


@dataclass
class Workload:
    name: str
    linears: List[Linear]
    mode: str               # "dynamic" or "table"
    steps: int = 1
    table: Optional[np.ndarray] = None      # [T, L] fp32 for mode == "table"
    sigmas: Optional[np.ndarray] = None     # activation std per step

    def ops_per_step(self) -> int:
        return sum(2 * l.M * l.N * l.K for l in self.linears)

    def packed_weight_bytes(self) -> int:
        return sum(l.N * l.K // 2 for l in self.linears)


def single_linear(seed: int = 0) -> Workload:
    """Single W4A4 linear: x fp32 [16, 256] ~ N(0,1) with 4 outlier channels x20;
    W fp32 [256, 256] ~ N(0, 0.02) with 3 rows x15; bias ~ N(0, 0.01); block 64;
    per-token dynamic activation scale."""
    lin = Linear("single", M=16, K=256, N=256, block=64, x_seed=seed, w_seed=seed + 1,
                 b_seed=seed + 2, x_kwargs=dict(n_outlier_cols=4, outlier_scale=20.0),
                 w_kwargs=dict(n_outlier_rows=3, row_scale=15.0), x_dtype="f32")
    return Workload("single_linear_16x256x256_b64", [lin], mode="dynamic")


def dit_mlp_stack(seed: int = 1, layers: int = 4, M: int = 50, hidden: int = 1024,
                  ffn: int = 4096, steps: int = 10, block: int = 64,
                  fuse_gate_up: bool = False) -> Workload:
    """DiT action-head MLP stack: 50 action tokens x batch 1, hidden 1024,
    gate/up 1024->4096 and down 4096->1024, 4 layers, bf16 activations;
    10 denoising steps with a static act_scale_table[10][12]; activation std
    drifts 0.5 -> 3.0 across steps; block 64.  Every linear draws its own input
    (the MLP nonlinearity between up/gate and down is not part of the layer).

    fuse_gate_up: gate and up, which read the same input in the MLP, become one
    linear 1024->8192 (concatenated weights, one permutation and rotation, one
    activation pass); 8 linears and a table [10][8] per step."""
    lins = []
    li = 0
    shapes = ((("gate_up", hidden, 2 * ffn), ("down", ffn, hidden)) if fuse_gate_up else
              (("gate", hidden, ffn), ("up", hidden, ffn), ("down", ffn, hidden)))
    for layer in range(layers):
        for j, (nm, K, N) in enumerate(shapes):
            s = seed * 100000 + li * 10
            lins.append(Linear(f"l{layer}.{nm}", M=M, K=K, N=N, block=block, x_seed=s,
                               w_seed=s + 1, b_seed=s + 2, layer=li))
            li += 1
    sig = step_sigmas(steps)
    tab = scale_table(seed * 100000 + 99, steps, len(lins), sig)
    tag = "_gateup_fused" if fuse_gate_up else ""
    return Workload(f"dit_mlp_stack_M{M}_h{hidden}_f{ffn}_L{layers}_T{steps}_b{block}{tag}",
                    lins, mode="table", steps=steps, table=tab, sigmas=sig)


def backbone_prefill(seed: int = 2, M: int = 1024, d: int = 2048, f: int = 16384,
                     block: int = 128) -> Workload:
    """Backbone prefill linears (Gemma-2B-like widths): M = 1024 tokens, bf16
    x ~ N(0,1) with 1% heavy-tailed outlier channels (Student-t nu=3, x10);
    projections 2048->16384 and 16384->2048; per-token dynamic scale; block 128."""
    xk = dict(heavy_tail_frac=0.01, heavy_tail_nu=3.0, heavy_tail_scale=10.0)
    lins = [Linear("up", M=M, K=d, N=f, block=block, x_seed=seed * 1000, w_seed=seed * 1000 + 1,
                   b_seed=seed * 1000 + 2, x_kwargs=xk),
            Linear("down", M=M, K=f, N=d, block=block, x_seed=seed * 1000 + 10,
                   w_seed=seed * 1000 + 11, b_seed=seed * 1000 + 12, x_kwargs=xk)]
    return Workload(f"backbone_prefill_M{M}_{d}x{f}_b{block}", lins, mode="dynamic")


def dit_denoise_loop(seed: int = 3, layers: int = 16, tokens: int = 16, batch: int = 32,
                     d: int = 1536, f: int = 6144, steps: int = 8, block: int = 64,
                     fuse_qkv: bool = False) -> Workload:
    """Full DiT denoise loop, small-M regime: 16 layers x (q,k,v,o d->d; up d->f;
    down f->d), 16 action tokens x batch 32, 8 denoising steps, per-step scale
    table [8][96]; weights ~ N(0, 0.02) with a 1-30x log-uniform spread of
    column norms; block 64.

    fuse_qkv: q, k and v, which read the same normalised input, become one
    linear d -> 3d (concatenated weights, one permutation and rotation, one
    activation pass); 4 linears per layer and a table [8][64]."""
    M = tokens * batch
    lins = []
    li = 0
    shapes = ((("qkv", d, 3 * d), ("o", d, d), ("up", d, f), ("down", f, d)) if fuse_qkv else
              (("q", d, d), ("k", d, d), ("v", d, d), ("o", d, d), ("up", d, f), ("down", f, d)))
    for layer in range(layers):
        for nm, K, N in shapes:
            s = seed * 1000000 + li * 10
            lins.append(Linear(f"l{layer}.{nm}", M=M, K=K, N=N, block=block, x_seed=s,
                               w_seed=s + 1, b_seed=s + 2, layer=li,
                               w_kwargs=dict(col_spread=30.0)))
            li += 1
    sig = step_sigmas(steps)
    tab = scale_table(seed * 1000000 + 99, steps, len(lins), sig)
    tag = "_qkv_fused" if fuse_qkv else ""
    return Workload(f"dit_denoise_loop_M{M}_d{d}_f{f}_L{layers}_T{steps}_b{block}{tag}", lins,
                    mode="table", steps=steps, table=tab, sigmas=sig)


def sweep_point(M: int, KN: int, block: int, mode: str, seed: int = 5) -> Workload:
    """Roofline sweep point: square K = N, bf16 x ~ N(0,1) with 0.5% of channels
    x20; dynamic or per-step (table) scaling."""
    n_out = max(1, int(round(0.005 * KN)))
    s = seed * 1000 + M * 7 + KN * 13 + block
    lin = Linear("sq", M=M, K=KN, N=KN, block=block, x_seed=s, w_seed=s + 1, b_seed=s + 2,
                 x_kwargs=dict(n_outlier_cols=n_out, outlier_scale=20.0))
    sig = np.array([1.0])
    tab = scale_table(s + 3, 1, 1, sig) if mode == "table" else None
    return Workload(f"sweep_M{M}_KN{KN}_b{block}_{mode}", [lin], mode=mode, steps=1,
                    table=tab, sigmas=sig)


SWEEP_M = (1, 16, 64, 256, 1024, 4096, 8192)
SWEEP_KN = (1024, 2048, 4096, 8192)
SWEEP_BLOCK = (32, 64, 128, 256)
SWEEP_MODE = ("dynamic", "table")


def sweep_points() -> List[Tuple[int, int, int, str]]:
    return [(M, KN, b, m) for M in SWEEP_M for KN in SWEEP_KN for b in SWEEP_BLOCK
            for m in SWEEP_MODE]
