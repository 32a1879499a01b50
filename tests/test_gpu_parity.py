"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact: packed weights and scales, activation codes and scales when both
sides quantise the same fp32 rotated inputs, and int32 accumulators for the
same codes.  Within tolerance: the fp32 rotation (vs fp64), end-to-end
activation codes (+-1 only at a rounding boundary), bf16 outputs
(2e-2 absolute + 1e-2 relative).
"""
import numpy as np
import pytest
import torch

from oracle import qvla_oracle as O
from w4a4_post_quantization_zigzag_b200 import inputs as I
from _parity import check_codes_near_boundary, check_y, unpack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    from w4a4_post_quantization_zigzag_b200 import qvla
    assert torch.cuda.is_available()
    qvla.qvla_read_error_word(clear=True)
    return qvla


def cu(a, dt=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dt is not None:
        t = t.to(dt)
    return t.cuda()


def x_dev(x32, dtype):
    return cu(x32).to(torch.bfloat16) if dtype == "bf16" else cu(x32)


def no_device_error(q):
    assert q.qvla_read_error_word(clear=True) == 0


# ------------------------------------------------------ quantisers (bit-exact)

@pytest.mark.parametrize("M,K", [(1, 32), (7, 256), (50, 1024), (33, 4096)])
def test_act_quant_from_fp32_is_bit_exact(q, M, K):
    xr = I.activations(100 + M, M, K, std=1.7, n_outlier_cols=2, dtype="f32")
    if M > 1:
        xr[M - 1, :] = 0.0                           # an all-zero row: s = 0, codes 0
    qx_ref, s_ref = O.quantize_acts_dynamic_fp32(xr)
    xq, s = q.qvla_quant_act_f32(cu(xr), q.QVLA_SCALE_DYNAMIC)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), O.pack_nibbles(qx_ref))
    # table mode with a small scale: saturation at -8 / 7
    tab = I.scale_table(3, 4, 5, I.step_sigmas(4)) * 0.25
    qx_t, _ = O.quantize_acts_table_fp32(xr, O.table_scale(tab, 2, 3))
    xq_t, s_t = q.qvla_quant_act_f32(cu(xr), q.QVLA_SCALE_TABLE, table=cu(tab), step=2, layer=3)
    assert np.array_equal(xq_t.cpu().numpy(), O.pack_nibbles(qx_t))
    assert (s_t.cpu().numpy() == tab[2, 3]).all()
    assert unpack(xq_t.cpu().numpy()).min() == -8
    no_device_error(q)


def _near_boundary_row(rng, s, K, hs, amax=None):
    """K fp32 values whose quotients by s sit on and within a few ulps of the
    half-integers hs (where rint flips), plus integers, zeros, subnormals and,
    without amax, saturating values; amax (dynamic mode) caps |v| and is
    placed once so that it is the row maximum."""
    s = np.float32(s)
    vals = []
    for h in hs:
        v = np.float32(np.float64(h) * np.float64(s))
        for k in range(-4, 5):
            w = v
            step = np.float32(np.inf) if k > 0 else np.float32(-np.inf)
            for _ in range(abs(k)):
                w = np.nextafter(w, step)
            vals.append(w)
    vals += [np.float32(0), np.float32(-0.0), np.float32(1e-40), np.float32(-1e-40)]
    vals += [np.float32(n) * s for n in range(-7, 8)]
    if amax is None:
        vals += [np.float32(x) * s for x in (7.49, 7.5, 7.51, -8.49, -8.5, -8.51, 9, -9, 40, -40)]
        vals += [np.float32(3e38), np.float32(-3e38)]
    v = np.array(vals, np.float32)
    if amax is not None:
        v = v[np.abs(v) <= np.float32(amax)]
    out = rng.uniform(-1, 1, K).astype(np.float32) * (np.float32(amax) if amax is not None else s * 6)
    pos = rng.permutation(K)
    n = min(len(v), K - 1)
    out[pos[:n]] = v[:n]
    if amax is not None:
        out[pos[n]] = np.float32(amax)
    return out


@pytest.mark.parametrize("K", [1024, 256])
def test_act_quant_near_rounding_boundaries_is_bit_exact(q, K):
    """The epilogue quantiser (fused clamp by a saturating FMA, paired FMAs,
    exact division only near a half-integer) against clamp(rint(fp32(v / s)))
    on quotients within a few ulps of every half-integer, in both modes."""
    rng = np.random.default_rng(77 + K)
    # dynamic: s = fp32(amax / 7) per row, a power of two and irregular ones
    amaxes = [7.0, 7.7, 1.0e-3 * 3.3, 5.0e4 + 0.3, 0.1, 123.456]
    rows = []
    for a in amaxes:
        s = np.float32(a) / np.float32(7)
        rows.append(_near_boundary_row(rng, s, K, np.arange(-6.5, 7.0, 1.0), amax=a))
    xr = np.stack(rows)
    qx_ref, s_ref = O.quantize_acts_dynamic_fp32(xr)
    xq, sx = q.qvla_quant_act_f32(cu(xr), q.QVLA_SCALE_DYNAMIC)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), O.pack_nibbles(qx_ref))
    # table: one irregular scale, quotients from -9.5 to 8.5 (saturation both ends)
    tab = np.full((2, 3), 0.01234567, np.float32)
    tab[1, 2] = np.float32(0.0123456789)
    st = O.table_scale(tab, 1, 2)
    xt = np.stack([_near_boundary_row(rng, st, K, np.arange(-9.5, 9.0, 1.0)) for _ in range(3)])
    qt_ref, _ = O.quantize_acts_table_fp32(xt, st)
    xq_t, s_t = q.qvla_quant_act_f32(cu(xt), q.QVLA_SCALE_TABLE, table=cu(tab), step=1, layer=2)
    assert (s_t.cpu().numpy() == st).all()
    assert np.array_equal(xq_t.cpu().numpy(), O.pack_nibbles(qt_ref))
    no_device_error(q)


def test_quant_near_rounding_boundaries_is_bit_exact(q):
    """Values at, and one or two ulp around, every half-integer multiple of the
    scale: the codes must equal clamp(rint(fp32(v / s))) exactly (ties to even),
    including where a reciprocal multiply would round the other way."""
    rows = []
    for s in (np.float32(0.1), np.float32(0.0123), np.float32(3.7), np.float32(1e-3)):
        v = []
        for j in range(-9, 9):
            c = np.float32((j + 0.5) * float(s))
            for d in (-2, -1, 0, 1, 2):
                v.append(c + np.float32(d) * np.spacing(c) if d else c)
        v = np.array(v, np.float32)
        # the row's max must pin s = max/7 exactly: append +-7 s and pad to 96
        row = np.zeros(96, np.float32)
        row[:len(v)] = v
        row[-1] = np.float32(7) * s
        rows.append(row)
    xr = np.stack(rows)
    # table mode (s taken as given) and dynamic mode (s = max/7)
    for mode in ("table", "dynamic"):
        if mode == "dynamic":
            qr, sr = O.quantize_acts_dynamic_fp32(xr)
            xq, sg = q.qvla_quant_act_f32(cu(xr), q.QVLA_SCALE_DYNAMIC)
            assert np.array_equal(sg.cpu().numpy(), sr)
            assert np.array_equal(xq.cpu().numpy(), O.pack_nibbles(qr))
        else:
            for i, s in enumerate((0.1, 0.0123, 3.7, 1e-3)):
                tab = np.full((1, 1), s, np.float32)
                qr, _ = O.quantize_acts_table_fp32(xr[i:i + 1], np.float32(s))
                xq, _ = q.qvla_quant_act_f32(cu(xr[i:i + 1]), q.QVLA_SCALE_TABLE, table=cu(tab),
                                             step=0, layer=0)
                assert np.array_equal(xq.cpu().numpy(), O.pack_nibbles(qr)), s
    no_device_error(q)


@pytest.mark.parametrize("N,K", [(3, 64), (256, 256), (1000, 1024)])
def test_weight_quant_from_fp32_is_bit_exact(q, N, K):
    Wr = I.weights(200 + N, N, K, n_outlier_rows=2)
    Wr[1] = 0.0
    qw_ref, s_ref = O.quantize_weights_fp32(Wr)
    wq, s = q.qvla_quant_pack_weights_f32(cu(Wr))
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(wq.cpu().numpy(), O.pack_nibbles(qw_ref))
    no_device_error(q)


# ----------------------------------------------------------------- pack

@pytest.mark.parametrize("N,K,b", [(256, 256, 64), (130, 512, 32), (256, 1024, 128),
                                   (96, 512, 256)])
def test_pack_parity(q, N, K, b):
    W = I.weights(300 + K + b, N, K, n_outlier_rows=3, col_spread=10.0)
    ref = O.pack_linear(W, b)
    # the GPU's own permutation and R_SVD
    pk = q.qvla_pack_weights(cu(W), b)
    assert np.array_equal(pk.perm.cpu().numpy(), ref.perm)
    rot = pk.rot.cpu().numpy().astype(np.float64)
    for B in range(K // b):
        A = W.astype(np.float64)[:, ref.perm[B * b:(B + 1) * b]]
        lam = np.linalg.eigvalsh(A.T @ A)[::-1]
        # columns with a simple, non-zero eigenvalue are unique up to the sign
        # rule and must match; with N < b the null space has no unique basis,
        # so there only orthonormality and A v = 0 are checked
        gap = np.minimum(np.r_[np.inf, lam[:-1] - lam[1:]], np.r_[lam[:-1] - lam[1:], np.inf])
        uniq = (lam > 1e-9 * lam[0]) & (gap > 1e-6 * lam[0])
        assert np.abs(rot[B][:, uniq] - ref.rsvd[B][:, uniq]).max() <= 1e-6
        assert np.abs(rot[B].T @ rot[B] - np.eye(b)).max() <= 1e-5
        null = lam <= 1e-9 * lam[0]
        if null.any():
            assert np.abs(A @ rot[B][:, null]).max() <= 1e-5 * np.sqrt(lam[0])
    # with the oracle's perm and R_SVD both sides quantise the same rotation
    pk2 = q.qvla_pack_weights(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    assert np.array_equal(pk2.w_scale.cpu().numpy().view(np.uint32), ref.s_w.view(np.uint32))
    flips = check_codes_near_boundary(unpack(pk2.wq.cpu().numpy()), ref.qw, ref.Wr,
                                      ref.s_w.astype(np.float64), "packed weights")
    assert flips == 0
    # the weight rotation alone: fp32(W P R) computed in fp64
    Wr = q.qvla_rotate_weights_f32(cu(W), b, pk2.perm, cu(ref.rsvd))
    assert np.array_equal(Wr.cpu().numpy(), ref.Wr.astype(np.float32))
    no_device_error(q)


# ----------------------------------------------------- activation rotation

@pytest.fixture(params=["auto", "fma"])
def path(request, monkeypatch):
    """auto: tensor cores where the linear has an image (bf16, block 64/128),
    else the CUDA-core kernels (the composite-R_B one for fp32 input at block
    64 in table / rotate-only mode); fma: always the R_SVD + Walsh-Hadamard
    CUDA-core kernel."""
    monkeypatch.setenv("QVLA_ROTATE_PATH", request.param)
    return request.param


def _unswizzle_tc_image(img, nb, b):
    """uint16 [nb*3*b*b] (128B-swizzled K-major R_B^T parts) -> float64 [nb, 3, b(i), b(j)]."""
    img = img.reshape(nb, 3, b * b)
    out = np.zeros((nb, 3, b, b))
    i = np.arange(b)[:, None]
    j = np.arange(b)[None, :]
    kc, c = i // 64, (i % 64) // 8
    off = kc * b * 64 + j * 64 + ((c ^ (j & 7)) * 8) + (i % 8)
    bits = img[:, :, off].astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


@pytest.mark.parametrize("K,b", [(256, 64), (512, 128)])
def test_tc_image_is_the_composite_rotation(q, K, b):
    """The tensor-core image holds hi + mid + lo = R_SVD,B . H_b to ~2^-25."""
    W = I.weights(450 + K, 96, K)
    ref = O.pack_linear(W, b)
    L = q.qvla_pack_weights(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    parts = _unswizzle_tc_image(L.rot_tc.cpu().numpy().view(np.uint16), K // b, b)
    recon = parts.sum(axis=1)
    assert np.abs(recon - ref.R).max() <= 2e-8 * np.abs(ref.R).max()
    assert np.abs(parts[:, 0] - ref.R).max() > 1e-5 * np.abs(ref.R).max()   # hi alone is coarse
    no_device_error(q)


@pytest.mark.parametrize("M,K,b,dt", [(16, 256, 64, "f32"), (50, 1024, 64, "bf16"),
                                      (5, 2048, 128, "bf16"), (3, 512, 32, "bf16"),
                                      (9, 1024, 256, "bf16"), (2, 16384, 128, "bf16"),
                                      (300, 1024, 64, "bf16"), (130, 512, 128, "bf16"),
                                      (33, 512, 64, "f32"), (100, 1024, 64, "f32"),
                                      (1, 4096, 64, "bf16")])
def test_rotation_fp32_vs_fp64(q, path, M, K, b, dt):
    W = I.weights(400 + K, 64, K)
    ref = O.pack_linear(W, b)
    L = q.qvla_pack_weights(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    x = I.activations(401 + M, M, K, n_outlier_cols=3, dtype=dt)
    xr = q.qvla_rotate_act_f32(x_dev(x, dt), L).cpu().numpy().astype(np.float64)
    xr_ref = O.rotate_activations(x, ref.perm, ref.R)
    scale = np.abs(xr_ref).max(axis=1, keepdims=True)
    assert (np.abs(xr - xr_ref) <= 2e-6 * scale).all()


@pytest.mark.parametrize("M,K,b,dt,mode", [
    (16, 256, 64, "f32", "dynamic"), (50, 1024, 64, "bf16", "table"),
    (50, 4096, 64, "bf16", "table"), (37, 2048, 128, "bf16", "dynamic"),
    (8, 1024, 32, "bf16", "dynamic"), (8, 1024, 256, "bf16", "table"),
    (3, 16384, 128, "bf16", "dynamic"), (300, 2048, 64, "bf16", "dynamic"),
    (257, 1536, 64, "bf16", "table"), (200, 4096, 128, "bf16", "table"),
    (1, 256, 64, "bf16", "table"), (33, 512, 64, "f32", "table"), (100, 1024, 64, "f32", "table"),
    (600, 1024, 64, "bf16", "table")])
@pytest.mark.parametrize("scratch", [False, True])
def test_rotate_quant_end_to_end(q, path, scratch, M, K, b, dt, mode):
    """scratch=True gives the call its workspace, which routes large bf16 inputs
    through the permuted copy + TMA-fed tensor-core kernel."""
    W = I.weights(500 + K + b, 96, K)
    ref = O.pack_linear(W, b)
    L = q.qvla_pack_weights(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    x = I.activations(501 + M, M, K, std=1.3, n_outlier_cols=4, dtype=dt)
    tab = I.scale_table(7, 10, 12, I.step_sigmas(10) * 1.3)
    ws = None
    if scratch:
        nbytes = q.qvla_rotate_quant_workspace_bytes(M, K, b, x_dev(x[:1], dt).dtype)
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    if mode == "dynamic":
        xq, s = q.qvla_rotate_quant_act(x_dev(x, dt), L, q.QVLA_SCALE_DYNAMIC, workspace=ws)
        xr_ref, qx_ref, s_ref = O.rotate_quant_act(x, ref, "dynamic")
        np.testing.assert_allclose(s.cpu().numpy(), s_ref, rtol=2e-6)
    else:
        step = torch.tensor([4], dtype=torch.int32, device="cuda")
        xq, s = q.qvla_rotate_quant_act(x_dev(x, dt), L, q.QVLA_SCALE_TABLE, table=cu(tab),
                                        step=step, layer=7, workspace=ws)
        xr_ref, qx_ref, s_ref = O.rotate_quant_act(x, ref, "table", tab, 4, 7)
        assert (s.cpu().numpy() == tab[4, 7]).all()
    check_codes_near_boundary(unpack(xq.cpu().numpy()), qx_ref, xr_ref, s_ref, "activations")
    no_device_error(q)


def test_rotate_quant_ragged_pitch_and_empty(q):
    M, K, b = 5, 512, 64
    W = I.weights(600, 64, K)
    ref = O.pack_linear(W, b)
    L = q.qvla_pack_weights(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    x = I.activations(601, M, K + 64, dtype="bf16")
    xd = x_dev(x, "bf16")[:, :K]                     # row pitch K + 64
    xq, s = q.qvla_rotate_quant_act(xd, L, q.QVLA_SCALE_DYNAMIC)
    xr_ref, qx_ref, s_ref = O.rotate_quant_act(x[:, :K], ref, "dynamic")
    check_codes_near_boundary(unpack(xq.cpu().numpy()), qx_ref, xr_ref, s_ref)
    e = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    xq0, s0 = q.qvla_rotate_quant_act(e, L, q.QVLA_SCALE_DYNAMIC)
    assert xq0.shape == (0, K // 2)


def test_device_step_out_of_range_sets_flag_and_zeroes(q):
    M, K, b = 4, 256, 64
    W = I.weights(700, 64, K)
    ref = O.pack_linear(W, b)
    L = q.qvla_pack_weights(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    x = x_dev(I.activations(701, M, K), "bf16")
    tab = cu(I.scale_table(1, 8, 3, I.step_sigmas(8)))
    q.qvla_read_error_word(clear=True)
    bad = torch.tensor([8], dtype=torch.int32, device="cuda")
    xq, s = q.qvla_rotate_quant_act(x, L, q.QVLA_SCALE_TABLE, table=tab, step=bad, layer=1)
    word = q.qvla_read_error_word(clear=True)
    assert word & q.QVLA_DEVERR_STEP_RANGE
    assert not xq.cpu().numpy().any() and not s.cpu().numpy().any()
    ok = torch.tensor([7], dtype=torch.int32, device="cuda")
    q.qvla_rotate_quant_act(x, L, q.QVLA_SCALE_TABLE, table=tab, step=ok, layer=1)
    assert q.qvla_read_error_word(clear=True) == 0


# ------------------------------------------------------------------ GEMM

GEMM_CASES = [
    # M, N, K, split_k
    (1, 256, 256, 0), (16, 256, 256, 1), (50, 4096, 1024, 0), (50, 1024, 4096, 0),
    (64, 384, 1024, 4), (64, 200, 512, 2), (100, 256, 2048, 8), (128, 512, 768, 1),
    (200, 384, 1024, 1), (256, 256, 512, 0), (300, 1000, 1056, 1), (520, 256, 2048, 0),
    (33, 640, 4096, 16), (120, 512, 1024, 2), (260, 384, 1024, 4),
    # small token tiles with long K: the tiles are split over K between the
    # two CTAs of a cluster (odd stage counts, a ragged last stage)
    (16, 256, 2048, 0), (30, 384, 1056, 0), (40, 512, 1056, 0), (64, 128, 8192, 0),
]


@pytest.mark.parametrize("M,N,K,split", GEMM_CASES)
def test_gemm_int32_accumulators_bit_exact(q, M, N, K, split):
    qx = I.int_codes(800 + M, M, K, -8, 7)
    qw = I.int_codes(801 + N, N, K, -7, 7)
    qx[0, :] = -8                                   # extreme magnitudes
    qw[0, :] = -7
    acc_ref = O.int_gemm(qx, qw)
    L = q.from_host_packed(O.pack_nibbles(qw), np.ones(N, np.float32),
                           np.arange(K, dtype=np.int32), np.zeros((K // 32, 32, 32)))
    acc = q.qvla_w4a4_gemm_s32(cu(O.pack_nibbles(qx)), L, split_k=split)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), acc_ref)
    no_device_error(q)


@pytest.mark.parametrize("M,N,K,split", [(50, 4096, 1024, 0), (16, 256, 256, 0),
                                         (300, 1000, 1056, 1), (64, 384, 1024, 4)])
def test_gemm_bf16_epilogue(q, M, N, K, split):
    qx = I.int_codes(900 + M, M, K, -8, 7)
    qw = I.int_codes(901 + N, N, K, -7, 7)
    s_x = I.positive_scales(902, M, 0.05, 0.6)
    s_w = I.positive_scales(903, N, 1e-3, 2e-2)
    b = I.bias(904, N)
    L = q.from_host_packed(O.pack_nibbles(qw), s_w, np.arange(K, dtype=np.int32),
                           np.zeros((K // 32, 32, 32)), bias=b)
    y = q.qvla_w4a4_gemm(cu(O.pack_nibbles(qx)), cu(s_x), L, split_k=split)
    y_ref = O.dequantize(O.int_gemm(qx, qw), s_x, s_w, b)
    check_y(y.float().cpu().numpy(), y_ref)
    # output row pitch larger than N
    yp = torch.zeros(M, N + 8, dtype=torch.bfloat16, device="cuda")
    q.qvla_w4a4_gemm(cu(O.pack_nibbles(qx)), cu(s_x), L, split_k=split, y=yp[:, :N])
    check_y(yp[:, :N].float().cpu().numpy(), y_ref)
    assert not yp[:, N:].float().abs().sum().item()
    no_device_error(q)


# ----------------------------------------------------- whole layer

def _layer(q, lin, mode="dynamic", tab=None, step=0, x_std=None):
    W, x, bb = lin.make_w(), lin.make_x(std=x_std), lin.make_bias()
    ref = O.pack_linear(W, lin.block, bias=bb)
    L = q.qvla_pack_weights(cu(W), lin.block, bias=cu(bb), perm_in=ref.perm.astype(np.int32),
                            rsvd_in=ref.rsvd)
    xd = x_dev(x, lin.x_dtype)
    if mode == "dynamic":
        xq, s = q.qvla_rotate_quant_act(xd, L, q.QVLA_SCALE_DYNAMIC)
        out = O.linear_forward(x, ref)
    else:
        xq, s = q.qvla_rotate_quant_act(xd, L, q.QVLA_SCALE_TABLE, table=cu(tab), step=step,
                                        layer=lin.layer)
        out = O.linear_forward(x, ref, "table", tab, step, lin.layer)
    y = q.qvla_w4a4_gemm(xq, s, L)
    qx_gpu = unpack(xq.cpu().numpy())
    check_codes_near_boundary(qx_gpu, out["qx"], out["xr"], out["s_x"])
    # several roundings are valid at a boundary: score y against the oracle's
    # dequantisation of the codes the GPU chose
    y_ref = O.dequantize(O.int_gemm(qx_gpu, ref.qw), out["s_x"], ref.s_w, bb)
    check_y(y.float().cpu().numpy(), y_ref)
    return y, out


def test_single_linear_layer(q):
    wl = I.single_linear()
    _layer(q, wl.linears[0])
    no_device_error(q)


def test_dit_mlp_layer_each_kind(q):
    wl = I.dit_mlp_stack()
    for lin in wl.linears[:3]:                       # gate, up, down of layer 0
        for step in (0, 9):
            _layer(q, lin, "table", wl.table, step, x_std=float(wl.sigmas[step]))
    no_device_error(q)


# ------------------------------------------------------------ batched calls

def test_batched_calls_match_single_calls(q):
    """Independent linears in one batched call give the same bytes and outputs
    as one call each (mixed block sizes, modes, dtypes, token tiles, M = 0)."""
    specs = [  # M, K, N, b, mode, dtype
        (50, 1024, 4096, 64, "table", "bf16"), (50, 4096, 1024, 64, "table", "bf16"),
        (50, 1024, 512, 64, "table", "bf16"), (16, 256, 256, 64, "dynamic", "f32"),
        (37, 2048, 384, 128, "dynamic", "bf16"), (200, 512, 256, 32, "table", "bf16"),
        (0, 256, 128, 64, "table", "bf16"), (3, 1024, 256, 256, "dynamic", "bf16"),
    ]
    tab = cu(I.scale_table(11, 6, 8, I.step_sigmas(6)))
    step = torch.tensor([5], dtype=torch.int32, device="cuda")
    probs, singles = [], []
    for i, (M, K, N, b, mode, dt) in enumerate(specs):
        W = I.weights(1100 + i, N, K)
        L = q.qvla_pack_weights(cu(W), b, bias=cu(I.bias(1150 + i, N)))
        x = x_dev(I.activations(1200 + i, max(M, 1), K, n_outlier_cols=2, dtype=dt), dt)[:M]
        md = q.QVLA_SCALE_TABLE if mode == "table" else q.QVLA_SCALE_DYNAMIC
        kw = dict(table=tab, step=step, layer=i) if mode == "table" else {}
        probs.append(q.LinearProblem(L, x, md, **kw))
        if M:
            xq, s = q.qvla_rotate_quant_act(x, L, md, **kw)
            singles.append((xq, s, q.qvla_w4a4_gemm(xq, s, L)))
        else:
            singles.append(None)
    q.qvla_rotate_quant_act_batched(probs)
    q.qvla_w4a4_gemm_batched(probs)
    torch.cuda.synchronize()
    for p, ref in zip(probs, singles):
        if ref is None:
            continue
        assert torch.equal(p.xq, ref[0]) and torch.equal(p.s_x, ref[1])
        assert torch.equal(p.y, ref[2])
    no_device_error(q)
