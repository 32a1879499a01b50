"""The W8A8 variant through the C ABI: 8-bit weight pack, 8-bit per-token
dynamic activations, the int8 GEMM with no unpack — against the oracle's
8-bit reading (codes +-1 only at a rounding boundary, int32 accumulators
bit-exact, bf16 outputs within tolerance, nothing written past N)."""
import numpy as np
import pytest
import torch

from oracle import qvla_oracle as O
from w4a4_post_quantization_zigzag_b200 import inputs as I
from _parity import BOUNDARY_8BIT, check_codes_near_boundary, check_y

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    from w4a4_post_quantization_zigzag_b200 import qvla
    qvla.qvla_read_error_word(clear=True)
    return qvla


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _w8_linear(q, qw, s_w, bias, K, block=32):
    """A packed W8 linear from host int8 codes (perm and rotation unused by the GEMM)."""
    N = qw.shape[0]
    return q.PackedLinear(N, K, block, cu(np.arange(K, dtype=np.int32)),
                          cu(np.zeros((K // block, block, block), np.float32)),
                          cu(qw.astype(np.int8)), cu(s_w.astype(np.float32)),
                          None if bias is None else cu(bias.astype(np.float32)))


@pytest.mark.parametrize("N,K,b", [(256, 256, 64), (130, 512, 32), (256, 1024, 128)])
def test_w8_pack_parity(q, N, K, b):
    W = I.weights(9300 + K + b, N, K, n_outlier_rows=3, col_spread=10.0)
    ref = O.pack_linear(W, b, bits=8)
    pk = q.qvla_pack_weights_w8(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    assert pk.wq.shape == (N, K) and pk.wq.dtype == torch.int8
    assert np.array_equal(pk.w_scale.cpu().numpy().view(np.uint32), ref.s_w.view(np.uint32))
    flips = check_codes_near_boundary(pk.wq.cpu().numpy().astype(np.int64), ref.qw, ref.Wr,
                                      ref.s_w.astype(np.float64), "int8 weights")
    assert flips == 0
    assert np.abs(pk.wq.cpu().numpy()).max() == 127
    assert q.qvla_read_error_word(clear=True) == 0


@pytest.mark.parametrize("M,K,b,dt", [(16, 256, 64, "f32"), (50, 1024, 64, "bf16"),
                                      (300, 2048, 128, "bf16"), (3, 512, 32, "bf16")])
def test_a8_activation_codes(q, M, K, b, dt):
    W = I.weights(9400 + K, 96, K)
    ref = O.pack_linear(W, b, bits=8)
    L = q.qvla_pack_weights_w8(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    x = I.activations(9401 + M, M, K, std=1.3, n_outlier_cols=4, dtype=dt)
    xd = cu(x) if dt == "f32" else cu(x).to(torch.bfloat16)
    xq8, s_x = q.qvla_rotate_quant_act_a8(xd, L)
    torch.cuda.synchronize()
    xr, qx, s = O.rotate_quant_act(x.astype(np.float64), ref)
    np.testing.assert_allclose(s_x.cpu().numpy(), s, rtol=2e-6)
    got = xq8.cpu().numpy().astype(np.int64)
    assert got.min() >= -128 and got.max() <= 127
    check_codes_near_boundary(got, qx, xr, s, "int8 activation codes", boundary=BOUNDARY_8BIT)
    assert q.qvla_read_error_word(clear=True) == 0


@pytest.mark.parametrize("M,K,b", [(50, 4096, 64), (3, 1024, 128), (200, 2048, 64), (520, 1024, 64)])
def test_a8_routes_agree(q, M, K, b):
    """A workspace of M*K*6 bytes (room for the permuted copy) and the minimum
    M*K*4 give identical codes and scales."""
    W = I.weights(9450 + K, 64, K)
    ref = O.pack_linear(W, b, bits=8)
    L = q.qvla_pack_weights_w8(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    x = cu(I.activations(9451 + M, M, K, std=1.3, n_outlier_cols=4)).to(torch.bfloat16)
    assert q.qvla_rotate_quant_a8_workspace_bytes(M, K) == M * K * 6
    big = torch.empty(M * K * 6, dtype=torch.uint8, device="cuda")
    small = torch.empty(M * K * 4, dtype=torch.uint8, device="cuda")
    a, sa = q.qvla_rotate_quant_act_a8(x, L, workspace=big)
    b8, sb = q.qvla_rotate_quant_act_a8(x, L, workspace=small)
    torch.cuda.synchronize()
    assert torch.equal(a, b8) and torch.equal(sa, sb)
    assert q.qvla_read_error_word(clear=True) == 0


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (16, 384, 512), (50, 1024, 4096),
                                   (64, 4096, 1024), (100, 256, 2048), (300, 1000, 1056),
                                   (520, 256, 2048), (33, 8, 32768)])
def test_w8a8_gemm_int32_bit_exact(q, M, N, K):
    qx = I.int_codes(9500 + M, M, K, -128, 127)
    qw = I.int_codes(9501 + N, N, K, -127, 127)
    qx[0, :] = -128                                 # extreme magnitudes
    qw[0, :] = -127
    qw[N - 1, :] = 127
    L = _w8_linear(q, qw, np.ones(N), None, K)
    acc = q.qvla_w8a8_gemm_s32(cu(qx.astype(np.int8)), L)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.int_gemm(qx, qw))
    assert q.qvla_read_error_word(clear=True) == 0


@pytest.mark.parametrize("M,N,K", [(50, 4096, 1024), (7, 3, 64), (16, 1001, 512),
                                   (300, 1000, 1056), (64, 133, 256)])
def test_w8a8_gemm_bf16_epilogue(q, M, N, K):
    qx = I.int_codes(9600 + M, M, K, -128, 127)
    qw = I.int_codes(9601 + N, N, K, -127, 127)
    s_x = I.positive_scales(9602, M, 1e-3, 1e-2)
    s_w = I.positive_scales(9603, N, 1e-4, 1e-3)
    b = I.bias(9604, N)
    L = _w8_linear(q, qw, s_w, b, K)
    pitch = (N + 7) // 8 * 8 + 8
    y = torch.full((M, pitch), float("nan"), dtype=torch.bfloat16, device="cuda")
    q.qvla_w8a8_gemm(cu(qx.astype(np.int8)), cu(s_x), L, y=y[:, :N])
    torch.cuda.synchronize()
    assert torch.isnan(y[:, N:].float()).all(), "wrote past N"
    yr = y[:, :N].float().cpu().numpy()
    assert np.isfinite(yr).all(), "an output element was not written"
    check_y(yr, O.dequantize(O.int_gemm(qx, qw), s_x, s_w, b))
    assert q.qvla_read_error_word(clear=True) == 0


@pytest.mark.parametrize("M,K,N,b", [(50, 4096, 1024, 64), (1, 1024, 512, 64),
                                     (300, 2048, 384, 128), (37, 1536, 256, 32)])
def test_w8a8_linear_end_to_end(q, M, K, N, b):
    W, bias = I.weights(9700 + K + N, N, K, col_spread=30.0), I.bias(9701, N)
    ref = O.pack_linear(W, b, bias=bias, bits=8)
    L = q.qvla_pack_weights_w8(cu(W), b, bias=cu(bias), perm_in=ref.perm.astype(np.int32),
                               rsvd_in=ref.rsvd)
    x = I.activations(9702 + M, M, K, std=1.3, n_outlier_cols=4)
    xq8, s_x = q.qvla_rotate_quant_act_a8(cu(x).to(torch.bfloat16), L)
    y = q.qvla_w8a8_gemm(xq8, s_x, L)
    torch.cuda.synchronize()
    out = O.linear_forward(x.astype(np.float64), ref)
    np.testing.assert_allclose(s_x.cpu().numpy(), out["s_x"], rtol=2e-6)
    qx = xq8.cpu().numpy().astype(np.int64)
    check_codes_near_boundary(qx, out["qx"], out["xr"], out["s_x"], "codes",
                              boundary=BOUNDARY_8BIT)
    y_ref = O.dequantize(O.int_gemm(qx, ref.qw), out["s_x"], ref.s_w, ref.bias)
    check_y(y.float().cpu().numpy(), y_ref)
    assert q.qvla_read_error_word(clear=True) == 0


def test_batched_w8a8_matches_single_calls(q):
    """qvla_rotate_quant_act_a8_batched + qvla_w8a8_gemm_batched over linears of
    different token tiles, widths, blocks and input types (both workspace
    sizes) give exactly the single-linear results."""
    shapes = [(50, 1024, 384, 64, "bf16", True), (50, 4096, 256, 64, "bf16", False),
              (16, 512, 200, 32, "f32", True), (130, 1024, 256, 128, "bf16", True),
              (7, 256, 136, 64, "f32", False)]
    probs, singles = [], []
    for i, (M, K, N, b, dt, full_ws) in enumerate(shapes):
        W = I.weights(9700 + i, N, K, n_outlier_rows=2)
        ref = O.pack_linear(W, b, bits=8)
        L = q.qvla_pack_weights_w8(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd,
                                   bias=cu(I.bias(9750 + i, N)))
        x = I.activations(9800 + i, M, K, std=1.1, n_outlier_cols=3, dtype=dt)
        xd = cu(x) if dt == "f32" else cu(x).to(torch.bfloat16)
        nbytes = q.qvla_rotate_quant_a8_workspace_bytes(M, K) if full_ws else M * K * 4
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        probs.append(q.LinearProblem(L, xd, workspace=ws, xq8=True))
        xq8, s_x = q.qvla_rotate_quant_act_a8(xd, L, workspace=ws.clone())
        singles.append((xq8, s_x, q.qvla_w8a8_gemm(xq8, s_x, L)))
    q.qvla_rotate_quant_act_a8_batched(probs)
    q.qvla_w8a8_gemm_batched(probs)
    torch.cuda.synchronize()
    for p, (xq8, s_x, y) in zip(probs, singles):
        assert torch.equal(p.xq8, xq8) and torch.equal(p.s_x, s_x)
        assert torch.equal(p.y, y)
    assert q.qvla_read_error_word(clear=True) == 0
