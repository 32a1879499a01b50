"""Pins for the CPU oracle against what the pages and the mathematics fix.

Each check compares the oracle with something other than itself: hand-worked
fixtures under tests/golden/, closed forms, invariants, a different LAPACK
routine (SVD instead of the oracle's symmetric eigensolver), and brute force
with dense K x K matrices and scalar loops on tiny shapes.  The planted-mistake
test at the end shows that a plausible bug in each oracle stage trips a pin.
"""
import json
import os

import numpy as np
import pytest

from oracle import qvla_oracle as O
from w4a4_post_quantization_zigzag_b200 import inputs as I

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- Hadamard

def test_hadamard_golden_order4():
    g = gold("hadamard4.json")
    np.testing.assert_array_equal(O.hadamard(4) * 2.0, np.array(g["H_times_sqrt_b"], float))


@pytest.mark.parametrize("b", [1, 2, 4, 8, 32, 64, 128, 256])
def test_hadamard_orthonormal_symmetric(b):
    H = O.hadamard(b)
    assert np.abs(H @ H.T - np.eye(b)).max() <= 1e-14
    assert np.array_equal(H, H.T)
    assert np.allclose(np.abs(H), 1 / np.sqrt(b), rtol=0, atol=1e-16)
    # Sylvester recursion H_2b = [[H_b, H_b], [H_b, -H_b]] / sqrt(2)
    if b >= 2:
        h = O.hadamard(b // 2)
        rec = np.block([[h, h], [h, -h]]) / np.sqrt(2)
        assert np.abs(rec - H).max() <= 1e-15


def test_hadamard_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        O.hadamard(24)


# ------------------------------------------------------------------- zigzag

@pytest.mark.parametrize("case", gold("zigzag_cases.json")["cases"])
def test_zigzag_golden(case):
    W = np.array(case["W"], float)
    perm = O.zigzag_permutation(W, case["block"])
    assert perm.tolist() == case["perm"]
    c = O.column_norms(W)
    b = case["block"]
    sums = [float(c[perm[B * b:(B + 1) * b]].sum()) for B in range(W.shape[1] // b)]
    assert np.allclose(sums, case["block_norm_sums"])


def _ranks(W):
    c = O.column_norms(W)
    order = sorted(range(W.shape[1]), key=lambda k: (-c[k], k))
    rank = np.empty(W.shape[1], int)
    rank[order] = np.arange(W.shape[1])
    return c, rank


@pytest.mark.parametrize("K,b", [(256, 64), (1024, 64), (2048, 128), (512, 32), (512, 256)])
def test_zigzag_structure(K, b):
    W = I.weights(7 + K + b, 64, K, col_spread=30.0)
    perm = O.zigzag_permutation(W, b)
    assert sorted(perm.tolist()) == list(range(K))           # a permutation
    c, rank = _ranks(W)
    nb = K // b
    for B in range(nb):
        for pos in range(b):
            r = rank[perm[B * b + pos]]
            # position `pos` of every block holds a channel of stratum `pos`
            assert r // nb == pos
            # snake: even strata run left to right, odd strata right to left
            want = B if pos % 2 == 0 else nb - 1 - B
            assert r % nb == want
    sums = np.array([c[perm[B * b:(B + 1) * b]].sum() for B in range(nb)])
    # balance: the spread of block norm sums never exceeds c_max - c_min
    assert sums.max() - sums.min() <= c.max() - c.min() + 1e-12


# ------------------------------------------------------------------ R_SVD

@pytest.mark.parametrize("N,K,b", [(256, 256, 64), (96, 128, 32), (300, 256, 128), (512, 256, 256)])
def test_rsvd_against_library_svd(N, K, b):
    W = I.weights(11 + N + K, N, K, n_outlier_rows=3, col_spread=10.0).astype(np.float64)
    perm = O.zigzag_permutation(W, b)
    rs = O.svd_rotation_blocks(W, perm, b)
    for B in range(K // b):
        V = rs[B]
        assert np.abs(V.T @ V - np.eye(b)).max() <= 1e-12      # R_SVD^T R_SVD = I
        A = W[:, perm[B * b:(B + 1) * b]]
        AV = A @ V
        sv = np.linalg.svd(A, compute_uv=False)                 # a different LAPACK routine
        norms = np.linalg.norm(AV, axis=0)
        # each rotated channel carries one singular value's energy, descending
        assert np.allclose(norms, sv, rtol=1e-10, atol=1e-12 * sv[0])
        gram = AV.T @ AV
        off = gram - np.diag(np.diag(gram))
        assert np.abs(off).max() <= 1e-10 * sv[0] ** 2          # columns orthogonal
        # canonical sign: largest-magnitude entry of every column is positive
        idx = np.argmax(np.abs(V), axis=0)
        assert np.all(V[idx, np.arange(b)] > 0)


@pytest.mark.parametrize("N,K,b", [(256, 256, 64), (128, 256, 128), (64, 64, 32)])
def test_composite_equalises_channel_energy(N, K, b):
    """Columns of A_B R_SVD H all have squared norm ||A_B||_F^2 / b (closed form:
    A_B R_SVD = U S with orthonormal U, and every H entry squared is 1/b)."""
    W = I.weights(23 + K, N, K, n_outlier_rows=3, row_scale=15.0, col_spread=30.0).astype(np.float64)
    perm = O.zigzag_permutation(W, b)
    R = O.composite_blocks(O.svd_rotation_blocks(W, perm, b))
    for B in range(K // b):
        A = W[:, perm[B * b:(B + 1) * b]]
        assert np.abs(R[B].T @ R[B] - np.eye(b)).max() <= 1e-12
        n2 = np.sum((A @ R[B]) ** 2, axis=0)
        target = np.sum(A * A) / b
        assert np.allclose(n2, target, rtol=1e-10)


def test_rotation_preserves_the_product():
    """(W P R)(R^T P^T x) = W x before quantisation, within 1e-9 relative."""
    wl = I.single_linear()
    lin = wl.linears[0]
    W, x = lin.make_w().astype(np.float64), lin.make_x().astype(np.float64)
    pk = O.pack_linear(W, lin.block)
    xr = O.rotate_activations(x, pk.perm, pk.R)
    ref = x @ W.T
    got = xr @ pk.Wr.T
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-9


# -------------------------------------- Hadamard-only variant (R_SVD = I)

@pytest.mark.parametrize("K,b", [(256, 32), (512, 64), (1024, 128), (512, 256)])
def test_hadamard_only_pack_uses_the_library_hadamard(K, b):
    """R_B is SciPy's Sylvester Hadamard matrix scaled by 1/sqrt(b), entry for
    entry, and the zigzag permutation is the one the full method uses."""
    from scipy.linalg import hadamard as scipy_hadamard
    W = I.weights(7000 + K + b, 64, K, col_spread=10.0).astype(np.float64)
    pk = O.pack_linear_hadamard(W, b)
    Hs = scipy_hadamard(b).astype(np.float64) / np.sqrt(b)
    assert pk.R.shape == (K // b, b, b)
    for B in range(K // b):
        assert np.array_equal(pk.R[B], Hs)
    assert np.array_equal(pk.perm, O.zigzag_permutation(W, b))
    # W' = W P H block by block, against a dense product built from SciPy's H
    Wp = W[:, pk.perm]
    dense = np.concatenate([Wp[:, B * b:(B + 1) * b] @ Hs for B in range(K // b)], axis=1)
    np.testing.assert_allclose(pk.Wr, dense, rtol=0, atol=1e-12)


def test_hadamard_only_preserves_the_product_and_codes_range():
    """(W P H)(H^T P^T x) = W x, and the activation side is H applied to the
    gathered block (the fast Walsh-Hadamard transform)."""
    from scipy.linalg import hadamard as scipy_hadamard
    wl = I.single_linear()
    lin = wl.linears[0]
    W, x = lin.make_w().astype(np.float64), lin.make_x().astype(np.float64)
    pk = O.pack_linear_hadamard(W, lin.block)
    xr = O.rotate_activations(x, pk.perm, pk.R)
    ref = x @ W.T
    assert np.linalg.norm(xr @ pk.Wr.T - ref) / np.linalg.norm(ref) <= 1e-9
    b = lin.block
    Hs = scipy_hadamard(b).astype(np.float64) / np.sqrt(b)
    xp = x[:, pk.perm]
    for B in range(lin.K // b):
        np.testing.assert_allclose(xr[:, B * b:(B + 1) * b], xp[:, B * b:(B + 1) * b] @ Hs,
                                   rtol=0, atol=1e-12)
    assert pk.qw.min() >= -7 and pk.qw.max() <= 7


# ------------------------------------------------ dense brute force (tiny)

def _dense_P(perm):
    K = len(perm)
    P = np.zeros((K, K))
    P[perm, np.arange(K)] = 1.0          # (W P)[:, j] = W[:, perm[j]]
    return P


def _dense_R(Rb):
    nb, b, _ = Rb.shape
    R = np.zeros((nb * b, nb * b))
    for B in range(nb):
        R[B * b:(B + 1) * b, B * b:(B + 1) * b] = Rb[B]
    return R


@pytest.mark.parametrize("M,N,K,b,seed", [(1, 4, 8, 4, 0), (3, 4, 16, 4, 1), (2, 3, 16, 8, 2),
                                          (3, 4, 16, 8, 3)])
def test_tiny_pipeline_against_dense_matrices(M, N, K, b, seed):
    W = I.weights(seed, N, K, std=1.0).astype(np.float64)
    x = I.activations(seed + 50, M, K, dtype="f32").astype(np.float64)
    pk = O.pack_linear(W, b)
    P, R = _dense_P(pk.perm), _dense_R(pk.R)
    assert np.abs(P @ P.T - np.eye(K)).max() == 0
    assert np.abs(R.T @ R - np.eye(K)).max() <= 1e-12
    np.testing.assert_allclose(pk.Wr, W @ P @ R, rtol=0, atol=1e-12)
    xr = O.rotate_activations(x, pk.perm, pk.R)
    np.testing.assert_allclose(xr, (R.T @ P.T @ x.T).T, rtol=0, atol=1e-12)


# ------------------------------------------------------------------- RTN

def test_rtn_golden_scalars():
    g = gold("rtn_cases.json")
    for c in g["activation_cases"]:
        q, _ = O.quantize_acts_table_fp32(np.array([[c["v"]]], np.float32), np.float32(c["s"]))
        assert int(q[0, 0]) == c["q"], c
    for c in g["weight_cases"]:
        q = O._rtn_codes(np.float32(c["v"]), np.float32(c["s"]), -7, 7)
        assert int(q) == c["q"], c


def test_rtn_golden_rows():
    g = gold("rtn_cases.json")
    for c in g["dynamic_rows"]:
        q, s = O.quantize_acts_dynamic_fp32(np.array([c["x"]], np.float32))
        assert float(s[0]) == c["s"] and q[0].tolist() == c["q"]
    for c in g["weight_rows"]:
        q, s = O.quantize_weights_fp32(np.array([c["w"]], np.float32))
        assert int(s.view(np.uint32)[0]) == int(c["s_f32_hex"], 16)
        assert q[0].tolist() == c["q"]


def _brute_rtn(v, s, lo, hi):
    """Scalar loop: fp32 quotient, then ties-to-even by hand."""
    if s == 0:
        return 0
    t = float(np.float32(v) / np.float32(s))
    f = np.floor(t)
    d = t - f
    r = f + 1 if d > 0.5 else f if d < 0.5 else (f if f % 2 == 0 else f + 1)
    return int(min(max(r, lo), hi))


def test_rtn_brute_force_and_ranges():
    x = I.activations(5, 6, 64, n_outlier_cols=2, dtype="f32")
    q, s = O.quantize_acts_dynamic_fp32(x)
    for m in range(x.shape[0]):
        assert s[m] == np.float32(np.float32(np.abs(x[m]).max()) / np.float32(7))
        for k in range(x.shape[1]):
            assert q[m, k] == _brute_rtn(x[m, k], s[m], -8, 7)
    assert q.min() >= -8 and q.max() <= 7
    W = I.weights(6, 8, 64, n_outlier_rows=2)
    W[3] = 0.0
    qw, sw = O.quantize_weights_fp32(W)
    assert qw.min() >= -7 and qw.max() <= 7
    for n in range(W.shape[0]):
        if sw[n] == 0:
            assert not qw[n].any()
        else:
            assert np.abs(qw[n]).max() == 7          # the row max always lands on +-7
        for k in range(W.shape[1]):
            assert qw[n, k] == _brute_rtn(W[n, k], sw[n], -7, 7)


def test_rtn_8bit_brute_force_and_ranges():
    """The W8A8 reading: the same RTN rule with the 8-bit ranges, checked
    element by element against scalar fp32 arithmetic."""
    x = I.activations(15, 6, 64, n_outlier_cols=2, dtype="f32")
    q, s = O.quantize_acts_dynamic_fp32(x, O.ACT_QMIN8, O.ACT_QMAX8)
    for m in range(x.shape[0]):
        assert s[m] == np.float32(np.float32(np.abs(x[m]).max()) / np.float32(127))
        for k in range(x.shape[1]):
            assert q[m, k] == _brute_rtn(x[m, k], s[m], -128, 127)
        assert np.abs(q[m]).max() == 127              # the token max lands on +-127
    W = I.weights(16, 8, 64, n_outlier_rows=2)
    W[2] = 0.0
    qw, sw = O.quantize_weights_fp32(W, O.WEIGHT_QMAX8)
    assert qw.min() >= -127 and qw.max() <= 127
    for n in range(W.shape[0]):
        if sw[n] == 0:
            assert not qw[n].any()
        else:
            assert np.abs(qw[n]).max() == 127
            # every code is within half a step of the value it stands for
            err = np.abs(W[n].astype(np.float64) - qw[n] * np.float64(sw[n]))
            assert err.max() <= 0.5 * sw[n] * (1 + 1e-6)
        for k in range(W.shape[1]):
            assert qw[n, k] == _brute_rtn(W[n, k], sw[n], -127, 127)


def test_w8a8_layer_tracks_the_fp_layer_more_closely_than_w4a4():
    wl = I.single_linear()
    lin = wl.linears[0]
    W, x, b = lin.make_w(), lin.make_x(), lin.make_bias()
    ref = x.astype(np.float64) @ W.astype(np.float64).T + b
    errs = {}
    for bits in (4, 8):
        pk = O.pack_linear(W, lin.block, bias=b, bits=bits)
        out = O.linear_forward(x.astype(np.float64), pk)
        assert pk.bits == bits and np.abs(out["qx"]).max() <= (127 if bits == 8 else 8)
        errs[bits] = np.linalg.norm(out["y"] - ref) / np.linalg.norm(ref)
    assert errs[8] < errs[4] / 8
    assert O.pack_linear(W, lin.block, bits=8).wq.shape == (lin.N, lin.K)


# ------------------------------------------------------------------- GPTQ

def test_gptq_with_an_identity_hessian_is_round_to_nearest():
    """No correlation between inputs: the inverse factor is diagonal, no error
    moves between columns, and GPTQ rounds like RTN."""
    W = I.weights(40, 16, 64, n_outlier_rows=2).astype(np.float32)
    U, dead = O.gptq_inverse_factor(np.eye(64), damp=0.05)
    np.testing.assert_allclose(U, np.eye(64) / np.sqrt(1.05), rtol=1e-14, atol=0)
    q, s = O.gptq_quantize(W, U, dead)
    q_rtn, s_rtn = O.quantize_weights_fp32(W)
    assert np.array_equal(s, s_rtn) and np.array_equal(q, q_rtn)


def test_gptq_two_columns_by_hand():
    """K = 2 written out: damped H, its inverse and that inverse's upper
    Cholesky factor in closed form, then the two GPTQ steps."""
    H = np.array([[2.0, 0.9], [0.9, 1.5]])
    damp = 0.05
    mean = (H[0, 0] + H[1, 1]) / 2
    a, b, c = H[0, 0] + damp * mean, H[0, 1], H[1, 1] + damp * mean
    det = a * c - b * b
    i00, i01, i11 = c / det, -b / det, a / det            # inverse of [[a, b], [b, c]]
    u00 = np.sqrt(i00)
    u01 = i01 / u00
    u11 = np.sqrt(i11 - u01 * u01)
    U, _ = O.gptq_inverse_factor(H, damp)
    np.testing.assert_allclose(U, [[u00, u01], [0.0, u11]], rtol=1e-13, atol=1e-15)
    W = np.array([[0.70, -0.45], [0.10, 0.33], [-0.5, 0.5]], dtype=np.float32)
    q, s = O.gptq_quantize(W, U)
    for n in range(3):
        sn = float(np.float32(np.float32(np.abs(W[n]).max()) / np.float32(7)))
        w0, w1 = float(W[n, 0]), float(W[n, 1])
        q0 = min(7, max(-7, round(w0 / sn)))               # Python round: half to even
        e = (w0 - q0 * sn) / u00
        q1 = min(7, max(-7, round((w1 - e * u01) / sn)))
        assert (q[n, 0], q[n, 1]) == (q0, q1)


def test_gptq_dead_input_column_is_zero():
    W = I.weights(41, 8, 32).astype(np.float32)
    X = I.activations(42, 40, 32, dtype="f32").astype(np.float64)
    X[:, 5] = 0.0                                         # input 5 never active
    U, dead = O.gptq_inverse_factor(O.gptq_hessian(X))
    assert dead[5] and dead.sum() == 1
    q, _ = O.gptq_quantize(W, U, dead)
    assert not q[:, 5].any()


def test_gptq_lowers_the_calibration_output_error():
    W = I.weights(43, 128, 256, col_spread=10.0)
    x = I.activations(44, 300, 256, n_outlier_cols=3, dtype="f32")
    g = O.pack_linear_gptq(W, 64, x)
    r = O.pack_linear(W, 64)
    xr = O.rotate_activations(x.astype(np.float64), g.perm, g.R)
    err = lambda pk: np.linalg.norm((pk.Wr - pk.qw * pk.s_w[:, None].astype(np.float64)) @ xr.T)
    assert err(g) < 0.8 * err(r)
    assert np.abs(g.qw).max() <= 7 and np.array_equal(g.s_w, r.s_w)


def test_table_lookup_rejects_out_of_range():
    tab = np.ones((8, 3), np.float32)
    assert O.table_scale(tab, 7, 2) == 1.0
    for t, l in [(8, 0), (-1, 0), (0, 3)]:
        with pytest.raises(IndexError):
            O.table_scale(tab, t, l)


# -------------------------------------------------------- pack / GEMM / dequant

@pytest.mark.parametrize("case", gold("pack_cases.json")["cases"])
def test_pack_golden(case):
    assert O.pack_nibbles(np.array([case["q"]])).tolist() == [case["bytes"]]


def test_pack_roundtrip_all_bytes():
    b = np.arange(256, dtype=np.uint8)[None, :]
    q = O.unpack_nibbles(b)
    assert q.min() == -8 and q.max() == 7
    assert np.array_equal(O.pack_nibbles(q), b)


def test_int_gemm_brute_force():
    qx = I.int_codes(1, 3, 24, -8, 7)
    qw = I.int_codes(2, 5, 24, -7, 7)
    acc = O.int_gemm(qx, qw)
    for m in range(3):
        for n in range(5):
            assert acc[m, n] == sum(int(qx[m, k]) * int(qw[n, k]) for k in range(24))
    # extreme magnitudes stay far inside int32 at the largest K in use
    K = 16384
    assert 8 * 7 * K < 2 ** 31


def test_dequant_brute_force():
    acc = np.array([[3, -2], [0, 7]])
    sx, sw, b = np.array([0.5, 2.0]), np.array([0.25, 1.0]), np.array([0.1, -0.1])
    y = O.dequantize(acc, sx, sw, b)
    want = [[0.5 * 0.25 * 3 + 0.1, 0.5 * 1.0 * -2 - 0.1], [0.1, 2.0 * 7 - 0.1]]
    np.testing.assert_allclose(y, want, rtol=0, atol=1e-15)


def test_end_to_end_quantised_layer_is_close_to_fp_layer():
    """Sanity: the rotated W4A4 layer approximates the fp layer (what the method
    is for); rotation must beat no rotation on outlier-heavy inputs."""
    wl = I.single_linear()
    lin = wl.linears[0]
    W, x, bb = lin.make_w(), lin.make_x(), lin.make_bias()
    pk = O.pack_linear(W, lin.block, bias=bb)
    out = O.linear_forward(x, pk)
    ref = x.astype(np.float64) @ W.T.astype(np.float64) + bb
    err_rot = np.linalg.norm(out["y"] - ref) / np.linalg.norm(ref)
    # the same RTN without any rotation
    qw, sw = O.quantize_weights_fp32(W)
    qx, sx = O.quantize_acts_dynamic_fp32(x)
    y0 = O.dequantize(O.int_gemm(qx, qw), sx, sw, bb)
    err_plain = np.linalg.norm(y0 - ref) / np.linalg.norm(ref)
    assert err_rot < err_plain


# ------------------------------------- end-to-end activation quantiser

def _golden_pack(g):
    """The hand-worked linear: the fixture's permutation, R_SVD = I in every
    block (so R_B is the normalised Hadamard matrix), given weight codes."""
    b = g["block"]
    nb = g["K"] // b
    rsvd = np.stack([np.eye(b)] * nb)
    return O.PackedLinear(np.array(g["perm"]), rsvd, O.composite_blocks(rsvd), None,
                          np.array(g["qw"], np.int8), np.array(g["s_w"], np.float32),
                          np.array(g["bias"], np.float64))


def _golden_act_mismatches(g):
    """Which parts of the hand-worked case the oracle's end-to-end quantiser
    (rotate_quant_act) and layer (linear_forward) fail to reproduce."""
    pk = _golden_pack(g)
    x = np.array(g["x"], np.float64)
    table = np.array(g["table"], np.float32)
    bad = []
    xr, q, s = O.rotate_quant_act(x, pk, "table", table, g["step"], g["layer"])
    if not np.array_equal(xr, np.array(g["xr"], np.float64)):
        bad.append("xr")
    if q.tolist() != g["table_codes"] or not np.all(s == g["table_s"]):
        bad.append("table codes")
    out = O.linear_forward(x, pk, "table", table, g["step"], g["layer"])
    if out["acc"].tolist() != g["table_acc"] or not np.allclose(out["y"], g["table_y"],
                                                              rtol=0, atol=1e-15):
        bad.append("table layer")
    xr, q, s = O.rotate_quant_act(x, pk, "dynamic")
    want_s = [n / d for n, d in g["dynamic_s_fraction"]]
    if q.tolist() != g["dynamic_codes"] or not np.allclose(s, want_s, rtol=1e-15, atol=0):
        bad.append("dynamic codes")
    out = O.linear_forward(x, pk, "dynamic")
    want_y = [[n / d for n, d in row] for row in g["dynamic_y_fraction"]]
    if out["acc"].tolist() != g["dynamic_acc"] or not np.allclose(out["y"], want_y,
                                                                rtol=1e-14, atol=1e-15):
        bad.append("dynamic layer")
    return bad


def test_end_to_end_quantiser_golden():
    assert _golden_act_mismatches(gold("act_quant_cases.json")) == []


@pytest.mark.parametrize("mode", ["dynamic", "table"])
def test_end_to_end_quantiser_follows_the_fp32_rule(mode):
    """rotate_quant_act quantises the double x'; its codes must be the pinned
    fp32 rule applied to fp32(x') except within 1e-5 of a rounding boundary
    (where both roundings are correct), and its dynamic scale must be the
    token's max |x'| / 7 (scalar loop)."""
    lin = I.single_linear().linears[0]
    W = lin.make_w()
    pk = O.pack_linear(W, lin.block)
    x = I.activations(21, 64, 256, n_outlier_cols=4, dtype="f32").astype(np.float64)
    table = np.array([[0.9, 0.8], [0.5, 0.7]], np.float32)
    xr, q, s = O.rotate_quant_act(x, pk, mode, table, 1, 0)
    # x' is x P R with the dense matrices (pinned above)
    np.testing.assert_allclose(xr, x @ _dense_P(pk.perm) @ _dense_R(pk.R), rtol=0, atol=1e-12)
    xr32 = xr.astype(np.float32)
    if mode == "dynamic":
        q32, _ = O.quantize_acts_dynamic_fp32(xr32)
        for m in range(x.shape[0]):
            amax = 0.0
            for v in xr[m]:
                amax = max(amax, abs(float(v)))
            assert s[m] == amax / 7.0
            assert np.abs(q[m]).max() == 7 and q[m].min() >= -7   # -8 needs a table scale
    else:
        q32, _ = O.quantize_acts_table_fp32(xr32, np.float32(table[1, 0]))
        assert np.all(s == float(np.float32(table[1, 0])))
        assert q.min() == -8 and q.max() == 7                       # saturates both ways
    d = q.astype(np.int64) - q32.astype(np.int64)
    rows, cols = np.nonzero(d)
    assert np.abs(d).max(initial=0) <= 1
    t = xr[rows, cols] / s[rows]
    assert (np.abs(t - np.floor(t) - 0.5) < 1e-5).all()
    assert len(rows) <= max(1, 1e-4 * q.size)


def test_end_to_end_pins_catch_planted_mistakes(monkeypatch):
    """A dynamic divisor of 8, a clamp to [-7, 7], a transposed table read and
    a dropped permutation each break the hand-worked case."""
    g = gold("act_quant_cases.json")
    assert _golden_act_mismatches(g) == []
    with monkeypatch.context() as mp:
        mp.setattr(O, "ACT_QMAX", 8)
        assert "dynamic codes" in _golden_act_mismatches(g)
    with monkeypatch.context() as mp:
        mp.setattr(O, "ACT_QMIN", -7)
        assert "table codes" in _golden_act_mismatches(g)
    with monkeypatch.context() as mp:
        mp.setattr(O, "table_scale", lambda tab, step, layer: np.float32(tab[layer, step]))
        assert "table codes" in _golden_act_mismatches(g)
    rot = O.rotate_activations
    with monkeypatch.context() as mp:
        mp.setattr(O, "rotate_activations", lambda x, perm, R: rot(x, np.arange(len(perm)), R))
        assert "xr" in _golden_act_mismatches(g)
    assert _golden_act_mismatches(g) == []


# ------------------------------------------------------ planted mistakes

def test_pins_catch_planted_mistakes():
    """Plant a plausible bug in each oracle stage and show a pin fails."""
    W = I.weights(3, 128, 256, n_outlier_rows=3, col_spread=30.0).astype(np.float64)
    b = 64

    def composite_equal_norms(Rfun):
        perm = O.zigzag_permutation(W, b)
        R = Rfun(O.svd_rotation_blocks(W, perm, b))
        A = W[:, perm[:b]]
        n2 = np.sum((A @ R[0]) ** 2, axis=0)
        return np.allclose(n2, np.sum(A * A) / b, rtol=1e-10)

    assert composite_equal_norms(O.composite_blocks)
    # H applied on the wrong side (H . R_SVD instead of R_SVD . H)
    assert not composite_equal_norms(lambda rs: np.stack([O.hadamard(b) @ r for r in rs]))
    # R_SVD transposed
    assert not composite_equal_norms(lambda rs: np.stack([r.T @ O.hadamard(b) for r in rs]))

    # zigzag without the snake (plain round robin) breaks the golden case
    case = gold("zigzag_cases.json")["cases"][0]
    orig = O.zigzag_permutation

    def round_robin(Wm, block):
        K = Wm.shape[1]
        nb = K // block
        c = O.column_norms(Wm)
        order = sorted(range(K), key=lambda k: (-c[k], k))
        perm = np.empty(K, int)
        for r, ch in enumerate(order):
            perm[(r % nb) * block + r // nb] = ch
        return perm
    assert round_robin(np.array(case["W"], float), case["block"]).tolist() != case["perm"]
    assert orig(np.array(case["W"], float), case["block"]).tolist() == case["perm"]

    # Hadamard without its 1/sqrt(b) normalisation fails orthonormality
    Hn = O.hadamard(8) * np.sqrt(8)
    assert np.abs(Hn @ Hn.T - np.eye(8)).max() > 1e-3

    # double instead of fp32 division changes a golden RTN code
    v, s = np.float32(-3.0), np.float32(0.4)
    assert int(np.clip(np.rint(float(v) / float(s)), -8, 7)) != -8
    assert int(O._rtn_codes(v, s, -8, 7)) == -8

    # swapped nibble order fails the 0x78 pin
    q = np.array([[-8, 7]])
    swapped = ((q[:, 1::2] & 0xF) | ((q[:, 0::2] & 0xF) << 4)).astype(np.uint8)
    assert swapped.tolist() != [[0x78]] and O.pack_nibbles(q).tolist() == [[0x78]]
