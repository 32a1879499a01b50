"""CPU oracle for the Omega-QVLA rotated W4A4 linear layer.

    y = s_x * s_w * ( q(R^T P^T x) . q(W P R)^T ) + b

TEST INFRASTRUCTURE ONLY.  This module is a plain, slow, double-precision
statement of what the layer computes, used by the test suite, by the package's
smoke check and by the benchmark's CPU-baseline leg.  The library's CUDA path
never imports, calls or links it, and it imports nothing from that path.

Sources (web pages on the method; page title, then section):
  [PT]  "{Omega}-QVLA: Robust Quantization for Vision-Language-Action Models via
        Composite Rotation and Per-step Scaling" (gist.science, Portuguese
        technical summary), Metodologia 1 "Rotacao Composta SVD.Hadamard"
        (bullets "Rotacao SVD", "Rotacao Hadamard", "Implementacao em Blocos")
        and 2 "Escalonamento de Ativacao DiT por Passo".
  [FR]  the same paper's French technical summary (gist.science), Methodologie
        1 "Rotation Composite SVD.Hadamard" and 2 "Mise a l'Echelle ... par Etape".
  [VN]  "Omega-QVLA: Nen VLA W4A4 tren Edge" (vnrobo.com), sections "Y tuong
        paper: xoay truoc, scale theo step sau" and "Build DiT action head pack"
        (flags --use-rtn, --w-bits 4, --a-bits 4, --act-percentile 99.9,
        --duquant-block-size 64).
  [ES]  "Omega-QVLA Reduce el Modelo de Vision de Robot por 71% Sin
        Reentrenamiento" (aiexpert.news): step-count mismatch / truncated table
        as a failure mode.
  [FQ]  "FoldQuantVLA: Native Low-Bit Quantization of Vision-Language-Action
        Models via Consistent Folding" (radar.vhtltd.com): dynamic per-token
        activation quantisation.

Readings taken where the pages are silent:
  * Layouts follow PyTorch Linear: W is [N, K] (out x in), x is [M, K].
  * R_SVD of a block is the matrix of right singular vectors of that block of
    W (eigenvectors of its Gram matrix), columns ordered by descending singular
    value, each column's largest-magnitude entry (first on ties) made positive.
  * H is the Sylvester Hadamard matrix of order b scaled by 1/sqrt(b).
  * The zigzag permutation sorts input channels by the L2 norm of their weight
    column, descending (ties: lower index first), and deals them to the blocks
    in a snake order, one channel per block per round.
  * Weights: symmetric per-output-channel RTN, s_w = max|W'|/7, codes in [-7, 7].
    Activations: s_x = max|x'|/7 per token (dynamic) or s = table[t][l]
    (per-step table), codes clamped to [-8, 7].  Rounding is to nearest, ties to
    even; the divisions that decide a code are IEEE fp32 divisions of fp32
    operands.  A scale of 0 gives all-zero codes.
  * Nibble packing: byte j holds code 2j in its low nibble and code 2j+1 in its
    high nibble, both as 4-bit two's complement.
"""
from __future__ import annotations

import numpy as np

WEIGHT_QMAX = 7
ACT_QMIN, ACT_QMAX = -8, 7
# W8A8 variant ("FoldQuantVLA": attention-output and FFN-down projections kept
# at W8A8): symmetric per-channel 8-bit weights, per-token dynamic 8-bit
# activations; the same RTN rule with the 8-bit ranges.
WEIGHT_QMAX8 = 127
ACT_QMIN8, ACT_QMAX8 = -128, 127


# --------------------------------------------------------------------------
# Zigzag channel permutation  ([PT] "Implementacao em Blocos"; [FR] "par Blocs")
# --------------------------------------------------------------------------

def column_norms(W: np.ndarray) -> np.ndarray:
    """c_k = ||W[:, k]||_2 in double."""
    W = np.asarray(W, dtype=np.float64)
    return np.sqrt(np.sum(W * W, axis=0))


def zigzag_permutation(W: np.ndarray, block: int) -> np.ndarray:
    """perm[j] = original input channel placed at permuted position j.

    Channels are ranked by weight-column norm (descending, ties to the lower
    index).  Rank r belongs to round r // nb and is dealt to block
    (r % nb) on even rounds and nb-1-(r % nb) on odd rounds, landing at
    position `round` inside that block.  Every block therefore receives one
    channel from each stratum of nb consecutive ranks, which spreads high- and
    low-norm channels evenly over the blocks."""
    K = W.shape[1]
    if K % block:
        raise ValueError("K must be a multiple of the block size")
    nb = K // block
    c = column_norms(W)
    order = sorted(range(K), key=lambda k: (-c[k], k))
    perm = np.empty(K, dtype=np.int64)
    for r, ch in enumerate(order):
        rnd, pos = divmod(r, nb)
        blk = pos if rnd % 2 == 0 else nb - 1 - pos
        perm[blk * block + rnd] = ch
    return perm


# --------------------------------------------------------------------------
# Composite rotation R = R_SVD . H  ([PT]/[FR] "Rotacao SVD", "Rotacao Hadamard")
# --------------------------------------------------------------------------

def hadamard(b: int) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix: H[i, j] = (-1)^popcount(i & j) / sqrt(b)."""
    if b < 1 or b & (b - 1):
        raise ValueError("Hadamard order must be a power of two")
    H = np.empty((b, b), dtype=np.float64)
    for i in range(b):
        for j in range(b):
            H[i, j] = -1.0 if bin(i & j).count("1") % 2 else 1.0
    return H / np.sqrt(b)


def _canonical_signs(V: np.ndarray) -> np.ndarray:
    V = V.copy()
    for j in range(V.shape[1]):
        i = int(np.argmax(np.abs(V[:, j])))      # first index on ties
        if V[i, j] < 0:
            V[:, j] = -V[:, j]
    return V


def svd_rotation_blocks(W: np.ndarray, perm: np.ndarray, block: int) -> np.ndarray:
    """R_SVD for every block, [nb, b, b] double.

    For block B, A_B = (W P)[:, B] is N x b.  Its SVD A_B = U S V^T gives the
    rotation whose columns are the right singular vectors: the columns of
    A_B V are U S, so each rotated weight channel carries exactly one singular
    value's energy.  V is obtained here as the eigenvectors of the Gram matrix
    A_B^T A_B (eigenvalues S^2), sorted by descending eigenvalue."""
    W = np.asarray(W, dtype=np.float64)
    K = W.shape[1]
    nb = K // block
    out = np.empty((nb, block, block), dtype=np.float64)
    for B in range(nb):
        A = W[:, perm[B * block:(B + 1) * block]]
        G = A.T @ A
        lam, V = np.linalg.eigh(G)               # ascending
        idx = sorted(range(block), key=lambda i: (-lam[i], i))
        out[B] = _canonical_signs(V[:, idx])
    return out


def composite_blocks(rsvd: np.ndarray) -> np.ndarray:
    """R_B = R_SVD,B . H_b for every block."""
    b = rsvd.shape[1]
    H = hadamard(b)
    return np.stack([r @ H for r in rsvd])


def rotate_weights(W: np.ndarray, perm: np.ndarray, R: np.ndarray) -> np.ndarray:
    """W' = W P R (block diagonal R), double [N, K]."""
    W = np.asarray(W, dtype=np.float64)
    nb, b, _ = R.shape
    out = np.empty_like(W)
    for B in range(nb):
        out[:, B * b:(B + 1) * b] = W[:, perm[B * b:(B + 1) * b]] @ R[B]
    return out


def rotate_activations(x: np.ndarray, perm: np.ndarray, R: np.ndarray) -> np.ndarray:
    """Row form of x' = R^T P^T x: x'[m, B] = x[m, perm[B]] . R_B, double [M, K]."""
    x = np.asarray(x, dtype=np.float64)
    nb, b, _ = R.shape
    out = np.empty_like(x)
    for B in range(nb):
        out[:, B * b:(B + 1) * b] = x[:, perm[B * b:(B + 1) * b]] @ R[B]
    return out


# --------------------------------------------------------------------------
# Round-to-nearest quantisation  ([VN] "Build DiT action head pack": --use-rtn,
# --w-bits 4, --a-bits 4; [FQ] dynamic per-token activation quantisation;
# [PT]/[FR] 2, per-step activation scale table)
# --------------------------------------------------------------------------

def _rtn_codes(v32: np.ndarray, s32: np.ndarray, qmin: int, qmax: int) -> np.ndarray:
    """clamp(rint(v / s), qmin, qmax) with an IEEE fp32 division; s == 0 gives 0."""
    v32 = np.asarray(v32, dtype=np.float32)
    s32 = np.asarray(s32, dtype=np.float32)
    safe = np.where(s32 == 0, np.float32(1), s32).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        r = np.rint(np.divide(v32, safe, dtype=np.float32))
    q = np.clip(r, qmin, qmax)
    q = np.where(s32 == 0, 0, q)
    return q.astype(np.int8)


def quantize_weights_fp32(Wr32: np.ndarray, qmax: int = WEIGHT_QMAX):
    """Symmetric per-output-channel RTN of fp32 rotated weights [N, K].
    s_w[n] = fp32(max_k |W'[n,k]| / qmax), codes in [-qmax, qmax] (qmax 7 for
    the 4-bit weights, 127 for the W8A8 variant)."""
    Wr32 = np.asarray(Wr32, dtype=np.float32)
    amax = np.max(np.abs(Wr32), axis=1)
    s = np.divide(amax, np.float32(qmax), dtype=np.float32)
    q = _rtn_codes(Wr32, s[:, None], -qmax, qmax)
    return q, s


def quantize_acts_dynamic_fp32(xr32: np.ndarray, qmin: int = ACT_QMIN, qmax: int = ACT_QMAX):
    """Per-token dynamic RTN of fp32 rotated activations [M, K].
    s_x[m] = fp32(max_k |x'[m,k]| / qmax), codes clamped to [qmin, qmax]
    ([-8, 7] for 4-bit activations, [-128, 127] for the W8A8 variant)."""
    xr32 = np.asarray(xr32, dtype=np.float32)
    amax = np.max(np.abs(xr32), axis=1) if xr32.shape[1] else np.zeros(xr32.shape[0], np.float32)
    s = np.divide(amax, np.float32(qmax), dtype=np.float32)
    q = _rtn_codes(xr32, s[:, None], qmin, qmax)
    return q, s


def table_scale(table: np.ndarray, step: int, layer: int) -> np.float32:
    """Per-step static activation scale: table[step][layer].  A step or layer
    outside the table is an error, never a clamp ([ES]: a step-count mismatch or
    a truncated table is a failure mode)."""
    T, L = table.shape
    if not (0 <= step < T) or not (0 <= layer < L):
        raise IndexError("step/layer outside the activation scale table")
    return np.float32(table[step, layer])


def quantize_acts_table_fp32(xr32: np.ndarray, s: np.float32):
    xr32 = np.asarray(xr32, dtype=np.float32)
    sv = np.full(xr32.shape[0], s, dtype=np.float32)
    q = _rtn_codes(xr32, sv[:, None], ACT_QMIN, ACT_QMAX)
    return q, sv


# --------------------------------------------------------------------------
# Nibble packing, integer GEMM, dequantisation
# --------------------------------------------------------------------------

def pack_nibbles(q: np.ndarray) -> np.ndarray:
    """[R, K] int codes in [-8, 7] -> [R, K/2] uint8; code 2j in the low nibble."""
    q = np.asarray(q, dtype=np.int64)
    if q.shape[-1] % 2:
        raise ValueError("K must be even")
    lo = q[..., 0::2] & 0xF
    hi = q[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_nibbles(p: np.ndarray) -> np.ndarray:
    p = np.asarray(p, dtype=np.int64)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def int_gemm(qx: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k qx[m, k] * qw[n, k] in int64."""
    return np.asarray(qx, dtype=np.int64) @ np.asarray(qw, dtype=np.int64).T


def dequantize(acc: np.ndarray, s_x: np.ndarray, s_w: np.ndarray, bias=None) -> np.ndarray:
    """y[m, n] = s_x[m] * s_w[n] * acc[m, n] + b[n] in double."""
    y = (np.asarray(s_x, np.float64)[:, None] * np.asarray(s_w, np.float64)[None, :]
         * np.asarray(acc, np.float64))
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    return y


# --------------------------------------------------------------------------
# Whole-layer compositions
# --------------------------------------------------------------------------

class PackedLinear:
    """What the offline pack step produces for one linear (all on the host)."""

    def __init__(self, perm, rsvd, R, Wr, qw, s_w, bias, bits=4):
        self.perm, self.rsvd, self.R, self.Wr = perm, rsvd, R, Wr
        self.qw, self.s_w, self.bias, self.bits = qw, s_w, bias, bits

    @property
    def wq(self):
        """Packed weight bytes: two 4-bit codes per byte, or one int8 code."""
        if self.bits == 8:
            return np.asarray(self.qw, dtype=np.int8).view(np.uint8)
        return pack_nibbles(self.qw)


def pack_linear_hadamard(W: np.ndarray, block: int, bias=None, perm=None) -> PackedLinear:
    """Hadamard-only variant: R_SVD = I for every block, so R_B = H_b and
    x'_B = H x_B ("FoldQuantVLA": Hadamard rotation of weights and activations;
    the composite rotation of "{Omega}-QVLA" Methodology 1 without its SVD
    factor).  The zigzag permutation is kept."""
    if perm is None:
        perm = zigzag_permutation(W, block)
    nb = np.asarray(W).shape[1] // block
    return pack_linear(W, block, bias=bias, perm=perm, rsvd=np.stack([np.eye(block)] * nb))


def pack_linear(W: np.ndarray, block: int, bias=None, perm=None, rsvd=None,
                bits: int = 4) -> PackedLinear:
    """Offline pack: zigzag P, per-block R_SVD, R = R_SVD.H, W' = W P R, then RTN
    of fp32(W') to 4-bit codes (8-bit for the W8A8 variant).  `perm` / `rsvd`
    may be given to pin the non-unique parts."""
    if perm is None:
        perm = zigzag_permutation(W, block)
    if rsvd is None:
        rsvd = svd_rotation_blocks(W, perm, block)
    R = composite_blocks(rsvd)
    Wr = rotate_weights(W, perm, R)
    qw, s_w = quantize_weights_fp32(Wr.astype(np.float32),
                                    WEIGHT_QMAX8 if bits == 8 else WEIGHT_QMAX)
    return PackedLinear(perm, rsvd, R, Wr, qw, s_w, bias, bits)


# --------------------------------------------------------------------------
# GPTQ weight rounding (the pages' LLM pack: "build_gptq_weights" with the
# composite rotation, 4-bit weights, block 128, damping 0.05): an alternative
# to round-to-nearest that quantises the rotated weight columns one at a time
# and moves each column's rounding error onto the columns not yet quantised,
# weighted by the inverse Hessian of the layer's calibration inputs.
# --------------------------------------------------------------------------

def gptq_hessian(xr_cal: np.ndarray) -> np.ndarray:
    """H = X'^T X' (K x K, double) of rotated calibration activations [T, K]."""
    X = np.asarray(xr_cal, dtype=np.float64)
    return X.T @ X


def gptq_inverse_factor(H: np.ndarray, damp: float = 0.05):
    """The upper Cholesky factor U of (H + damp * mean(diag H) * I)^-1 (so that
    U^T U is that inverse), after giving dead inputs (H[i,i] == 0) a unit
    diagonal.  Returns (U, dead)."""
    H = np.array(H, dtype=np.float64, copy=True)
    dead = np.diag(H) == 0
    H[dead, dead] = 1.0
    K = H.shape[0]
    H[np.arange(K), np.arange(K)] += damp * np.mean(np.diag(H))
    Hinv = np.linalg.inv(H)
    # upper factor: Hinv = U^T U  <=>  U = L^T with Hinv = L L^T
    U = np.linalg.cholesky(Hinv).T
    return U, dead


def gptq_quantize(Wr32: np.ndarray, U: np.ndarray, dead=None, qmax: int = WEIGHT_QMAX,
                  quotients: bool = False):
    """GPTQ rounding of fp32 rotated weights [N, K] with the inverse factor U.

    The per-row scale is the RTN one, s = fp32(max |W'[n,:]| / qmax).  Column
    by column, in order: q = clamp(rint(w / s), -qmax, qmax) in double, the
    error e = (w - q s) / U[j, j], and every later column k takes
    w_k -= e * U[j, k] (the block size of the pages only groups these updates
    and leaves the result unchanged).  Returns (codes int8 [N, K], s fp32 [N]),
    and with `quotients` also the double w / s that each code rounded."""
    W = np.asarray(Wr32, dtype=np.float32)
    s = np.divide(np.max(np.abs(W), axis=1), np.float32(qmax), dtype=np.float32)
    Wc = W.astype(np.float64)
    if dead is not None:
        Wc[:, np.asarray(dead, bool)] = 0.0
    s64 = s.astype(np.float64)
    safe = np.where(s64 == 0, 1.0, s64)
    N, K = Wc.shape
    Q = np.zeros((N, K), dtype=np.int8)
    T = np.zeros((N, K), dtype=np.float64)
    for j in range(K):
        w = Wc[:, j]
        T[:, j] = w / safe
        q = np.where(s64 == 0, 0.0, np.clip(np.rint(w / safe), -qmax, qmax))
        Q[:, j] = q.astype(np.int8)
        e = (w - q * s64) / U[j, j]
        if j + 1 < K:
            Wc[:, j + 1:] -= e[:, None] * U[j, j + 1:][None, :]
    return (Q, s, T) if quotients else (Q, s)


def pack_linear_gptq(W: np.ndarray, block: int, x_cal: np.ndarray, bias=None, perm=None,
                     rsvd=None, damp: float = 0.05, U=None) -> PackedLinear:
    """Offline pack with GPTQ rounding: zigzag P and composite R as
    pack_linear, the Hessian from the rotated calibration activations, codes
    by gptq_quantize.  `U` may be given (the inverse factor) to pin it."""
    pk = pack_linear(W, block, bias=bias, perm=perm, rsvd=rsvd)
    dead = None
    if U is None:
        xr = rotate_activations(np.asarray(x_cal, np.float64), pk.perm, pk.R)
        U, dead = gptq_inverse_factor(gptq_hessian(xr), damp)
    qw, s_w = gptq_quantize(pk.Wr.astype(np.float32), U, dead)
    pk.qw, pk.s_w = qw, s_w
    pk.U, pk.dead = U, dead
    return pk


def rotate_quant_act(x: np.ndarray, pk: PackedLinear, mode: str = "dynamic",
                     table=None, step: int = 0, layer: int = 0):
    """Activation side in double, quantised like the fp32 path but from the
    double x' (the end-to-end reference).  Returns (x' double, codes, s_x double)."""
    xr = rotate_activations(x, pk.perm, pk.R)
    qmin, qmax = (ACT_QMIN8, ACT_QMAX8) if pk.bits == 8 else (ACT_QMIN, ACT_QMAX)
    if mode == "dynamic":
        s = np.max(np.abs(xr), axis=1) / qmax
    elif mode == "table":
        s = np.full(xr.shape[0], float(table_scale(table, step, layer)))
    else:
        raise ValueError(mode)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.rint(xr / np.where(s == 0, 1.0, s)[:, None])
    q = np.where((s == 0)[:, None], 0, np.clip(r, qmin, qmax)).astype(np.int16)
    return xr, q, s


def linear_forward(x, pk: PackedLinear, mode="dynamic", table=None, step=0, layer=0):
    """End-to-end layer output (double) and the intermediates it used."""
    xr, qx, s_x = rotate_quant_act(x, pk, mode, table, step, layer)
    acc = int_gemm(qx, pk.qw)
    y = dequantize(acc, s_x, pk.s_w, pk.bias)
    return dict(xr=xr, qx=qx, s_x=s_x, acc=acc, y=y)
