"""The GPTQ pack through the C ABI: the device forms P, R and W' = W P R,
rotates the calibration rows, and the library rounds W' with GPTQ.  Against
the oracle's GPTQ pack of the same weights and calibration rows:
  * scales bit-identical (GPTQ keeps the RTN scale);
  * codes identical when the oracle's inverse factor U is passed in;
  * with the library's own factor (fp32-rotated calibration rows, so H and U
    differ from the oracle's by rounding) every row's first flipped code
    sits at a rounding boundary of the oracle's quotient, and the flips
    are few (the error feedback carries a flip along its row);
  * the calibration output error no worse than the oracle's codes';
  * end to end, a GPTQ-packed linear through the W4A4 path within the bf16
    tolerance of the oracle's dequantisation of the same codes."""
import numpy as np
import pytest
import torch

from oracle import qvla_oracle as O
from w4a4_post_quantization_zigzag_b200 import inputs as I
from _parity import check_codes_near_boundary, check_gptq_flips, check_y

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


def _recon_error(Wr, qw, s, xr):
    D = Wr.astype(np.float64) - qw.astype(np.float64) * s.astype(np.float64)[:, None]
    return np.linalg.norm(xr @ D.T)


def _case(seed, N, K, T):
    W = I.weights(seed, N, K, n_outlier_rows=2, col_spread=10.0)
    x = I.activations(seed + 1, T, K, std=1.3, n_outlier_cols=4)     # bf16-representable
    return W, x


@pytest.mark.parametrize("N,K,b,T", [(96, 512, 64, 700), (256, 1024, 128, 1200),
                                     (130, 256, 32, 300)])
def test_gptq_pack_given_factor(q, N, K, b, T):
    W, x = _case(2500 + K, N, K, T)
    ref = O.pack_linear_gptq(W, b, x)
    pk = q.qvla_pack_weights_gptq(cu(W), b, perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd,
                                  U=ref.U)
    torch.cuda.synchronize()
    assert np.array_equal(pk.w_scale.cpu().numpy().view(np.uint32), ref.s_w.view(np.uint32))
    qg = O.unpack_nibbles(pk.wq.cpu().numpy())
    # W' on the device is bit-exact and the column loop with the same U is a
    # fixed sequence of fp64 operations: no code may differ
    assert int((qg != ref.qw).sum()) == 0, "code flips with the oracle's own factor"
    assert q.qvla_read_error_word(clear=True) == 0


@pytest.mark.parametrize("N,K,b,T,dt", [(96, 512, 64, 700, "bf16"), (64, 1024, 128, 900, "f32")])
def test_gptq_pack_with_calibration(q, N, K, b, T, dt):
    W, x = _case(2600 + K, N, K, T)
    ref = O.pack_linear_gptq(W, b, x)
    xd = cu(x) if dt == "f32" else cu(x).to(torch.bfloat16)
    pk = q.qvla_pack_weights_gptq(cu(W), b, x_cal=xd, perm_in=ref.perm.astype(np.int32),
                                  rsvd_in=ref.rsvd)
    torch.cuda.synchronize()
    assert np.array_equal(pk.w_scale.cpu().numpy().view(np.uint32), ref.s_w.view(np.uint32))
    qg = O.unpack_nibbles(pk.wq.cpu().numpy())
    # the device rotates the calibration rows in fp32 (x' within ~2e-6 of each
    # row's max), so H and U differ from the oracle's at ~1e-6 relative and
    # a row's first flip must sit within 1e-3 of a rounding boundary
    _, _, t_ref = O.gptq_quantize(ref.Wr.astype(np.float32), ref.U, ref.dead, quotients=True)
    check_gptq_flips(qg, ref.qw, t_ref, boundary=1e-3, max_frac=2e-3)
    xr = O.rotate_activations(x.astype(np.float64), ref.perm, ref.R)
    Wr32 = ref.Wr.astype(np.float32)
    e_g = _recon_error(Wr32, qg, ref.s_w, xr)
    assert e_g <= 1.01 * _recon_error(Wr32, ref.qw, ref.s_w, xr)
    qr, sr = O.quantize_weights_fp32(Wr32)
    assert e_g < 0.8 * _recon_error(Wr32, qr, sr, xr), "GPTQ must beat RTN on its calibration set"
    assert q.qvla_read_error_word(clear=True) == 0


def test_gptq_linear_end_to_end(q):
    N, K, b, T, M = 384, 1024, 64, 800, 50
    W, x_cal = _case(2700, N, K, T)
    bias = I.bias(2701, N)
    ref = O.pack_linear_gptq(W, b, x_cal, bias=bias)
    L = q.qvla_pack_weights_gptq(cu(W), b, x_cal=cu(x_cal).to(torch.bfloat16), bias=cu(bias),
                                 perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    x = I.activations(2702, M, K, std=1.3, n_outlier_cols=4)
    xq, s_x = q.qvla_rotate_quant_act(cu(x).to(torch.bfloat16), L)
    y = q.qvla_w4a4_gemm(xq, s_x, L)
    torch.cuda.synchronize()
    out = O.linear_forward(x.astype(np.float64), ref)
    np.testing.assert_allclose(s_x.cpu().numpy(), out["s_x"], rtol=2e-6)
    qx = O.unpack_nibbles(xq.cpu().numpy()).astype(np.int64)
    check_codes_near_boundary(qx, out["qx"], out["xr"], out["s_x"], "activation codes")
    qw = O.unpack_nibbles(L.wq.cpu().numpy()).astype(np.int64)
    _, _, t_ref = O.gptq_quantize(ref.Wr.astype(np.float32), ref.U, ref.dead, quotients=True)
    check_gptq_flips(qw, ref.qw, t_ref, boundary=1e-3, max_frac=2e-3)
    check_y(y.float().cpu().numpy(), O.dequantize(O.int_gemm(qx, qw), out["s_x"], ref.s_w, bias))
    assert q.qvla_read_error_word(clear=True) == 0
