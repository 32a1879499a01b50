"""The Hadamard-only variant (R_SVD = I, R_B = H_b) through the C ABI:
pack parity against the oracle's Hadamard-only pack, the activation rotation
in fp32 against fp64, and whole linears (codes +-1 only at a rounding
boundary, bf16 outputs within tolerance)."""
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
    qvla.qvla_read_error_word(clear=True)
    return qvla


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("N,K,b", [(256, 256, 64), (130, 512, 32), (256, 1024, 128),
                                   (96, 512, 256)])
def test_hadamard_pack_parity(q, N, K, b):
    W = I.weights(8000 + K + b, N, K, n_outlier_rows=3, col_spread=10.0)
    ref = O.pack_linear_hadamard(W, b)
    pk = q.qvla_pack_weights_hadamard(cu(W), b)
    # R_SVD = I: no R_SVD blocks; the tensor-core image of R_B = H_b for b 64 / 128
    assert pk.rot is None and (pk.rot_tc is not None) == (b in (64, 128))
    assert np.array_equal(pk.perm.cpu().numpy(), ref.perm)
    assert np.array_equal(pk.w_scale.cpu().numpy().view(np.uint32), ref.s_w.view(np.uint32))
    flips = check_codes_near_boundary(unpack(pk.wq.cpu().numpy()), ref.qw, ref.Wr,
                                      ref.s_w.astype(np.float64), "packed weights")
    assert flips == 0
    assert q.qvla_read_error_word(clear=True) == 0


@pytest.mark.parametrize("M,K,b,dt,image", [(16, 256, 64, "f32", True), (50, 1024, 64, "bf16", True),
                                            (50, 1024, 64, "bf16", False),
                                            (3, 512, 32, "bf16", True), (9, 1024, 256, "bf16", True),
                                            (300, 2048, 128, "bf16", True),
                                            (300, 2048, 128, "bf16", False)])
def test_hadamard_rotation_fp32_vs_fp64(q, M, K, b, dt, image):
    """bf16 at blocks 64 / 128 with the image: the tensor-core route (R_B = H_b
    in three bf16 parts, of which only the first is non-zero); without it, or
    for fp32 input and blocks 32 / 256: the Walsh-Hadamard transform alone."""
    W = I.weights(8100 + K, 64, K)
    ref = O.pack_linear_hadamard(W, b)
    L = q.qvla_pack_weights_hadamard(cu(W), b, perm_in=ref.perm.astype(np.int32), image=image)
    x = I.activations(8101 + M, M, K, n_outlier_cols=3, dtype=dt)
    xd = cu(x) if dt == "f32" else cu(x).to(torch.bfloat16)
    xr = q.qvla_rotate_act_f32(xd, L).cpu().numpy().astype(np.float64)
    xr_ref = O.rotate_activations(x, ref.perm, ref.R)
    scale = np.abs(xr_ref).max(axis=1, keepdims=True)
    assert (np.abs(xr - xr_ref) <= 2e-6 * scale).all()
    assert q.qvla_read_error_word(clear=True) == 0


@pytest.mark.parametrize("M,K,N,b,mode", [(1, 1024, 512, 64, "dynamic"),
                                          (50, 1024, 4096, 64, "table"),
                                          (50, 4096, 1024, 64, "table"),
                                          (300, 2048, 384, 128, "dynamic"),
                                          (37, 1536, 256, 32, "table")])
def test_hadamard_linear_end_to_end(q, M, K, N, b, mode):
    W, bias = I.weights(8200 + K + N, N, K, col_spread=30.0), I.bias(8201, N)
    ref = O.pack_linear_hadamard(W, b, bias=bias)
    L = q.qvla_pack_weights_hadamard(cu(W), b, bias=cu(bias), perm_in=ref.perm.astype(np.int32))
    x = I.activations(8202 + M, M, K, std=1.3, n_outlier_cols=4)
    xd = cu(x).to(torch.bfloat16)
    if mode == "table":
        tab = I.scale_table(8203, 4, 3, I.step_sigmas(4) * 1.3)
        xq, s_x = q.qvla_rotate_quant_act(xd, L, q.QVLA_SCALE_TABLE, table=cu(tab), step=2,
                                          layer=1)
        out = O.linear_forward(x.astype(np.float64), ref, "table", tab, 2, 1)
    else:
        xq, s_x = q.qvla_rotate_quant_act(xd, L, q.QVLA_SCALE_DYNAMIC)
        out = O.linear_forward(x.astype(np.float64), ref)
    y = q.qvla_w4a4_gemm(xq, s_x, L)
    torch.cuda.synchronize()
    np.testing.assert_allclose(s_x.cpu().numpy(), out["s_x"], rtol=2e-6)
    qx = unpack(xq.cpu().numpy())
    check_codes_near_boundary(qx, out["qx"], out["xr"], out["s_x"], "codes")
    y_ref = O.dequantize(O.int_gemm(qx, ref.qw), out["s_x"], ref.s_w, ref.bias)
    check_y(y.float().cpu().numpy(), y_ref)
    assert q.qvla_read_error_word(clear=True) == 0
