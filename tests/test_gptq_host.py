"""GPTQ weight rounding in the library's host code (the LLM pack of
"Omega-QVLA: Nen VLA W4A4 tren Edge", "Build LLM pack"), against the oracle.

With the same inverse factor U the column loop is a fixed sequence of IEEE
fp64 operations, so codes and scales must be bit-identical to the oracle's.
With the library's own factorisation of H the factor differs from the
oracle's only by rounding, and the codes must still agree (flips allowed
only where a row's first flip sits at a rounding boundary, counted and
bounded).  No GPU is used."""
import numpy as np
import pytest

from oracle import qvla_oracle as O
from w4a4_post_quantization_zigzag_b200 import inputs as I
from _parity import check_gptq_flips


@pytest.fixture(scope="module")
def q():
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    from w4a4_post_quantization_zigzag_b200 import qvla
    return qvla


def _case(seed, N, K, block, T, dead_cols=()):
    W = I.weights(seed, N, K, n_outlier_rows=2, col_spread=10.0)
    x = I.activations(seed + 1, T, K, std=1.3, n_outlier_cols=4)
    pk = O.pack_linear(W, block)
    xr = O.rotate_activations(x.astype(np.float64), pk.perm, pk.R)
    xr[:, list(dead_cols)] = 0.0               # rotated inputs that never fire
    return pk, xr


def _recon_error(Wr, qw, s, xr):
    """|| X' (W' - Q s)^T ||_F: the output error GPTQ minimises."""
    D = Wr.astype(np.float64) - qw.astype(np.float64) * s.astype(np.float64)[:, None]
    return np.linalg.norm(xr @ D.T)


@pytest.mark.parametrize("N,K,block,T", [(40, 128, 32, 300), (96, 512, 64, 700),
                                         (7, 256, 128, 64), (64, 1024, 128, 1500),
                                         (32, 256, 64, 100)])     # T < K: H singular
def test_given_factor_bit_identical(q, N, K, block, T):
    pk, xr = _case(2100 + K, N, K, block, T)
    U, dead = O.gptq_inverse_factor(O.gptq_hessian(xr), 0.05)
    qo, so = O.gptq_quantize(pk.Wr.astype(np.float32), U, dead)
    qg, sg = q.qvla_gptq_quantize_host(pk.Wr.astype(np.float32), U=U)
    assert np.array_equal(sg.view(np.uint32), so.view(np.uint32))
    assert np.array_equal(qg, qo)


@pytest.mark.parametrize("N,K,block,T,dead", [(96, 512, 64, 700, ()), (33, 256, 32, 100, (3, 200)),
                                              (64, 1024, 128, 1500, (0,)),
                                              (48, 512, 64, 200, ())])   # T < K: damping makes H definite
def test_own_factor_matches_oracle(q, N, K, block, T, dead):
    pk, xr = _case(2200 + K, N, K, block, T, dead)
    H = O.gptq_hessian(xr)
    Wr32 = pk.Wr.astype(np.float32)
    U, dd = O.gptq_inverse_factor(H, 0.05)
    qo, so, to = O.gptq_quantize(Wr32, U, dd, quotients=True)
    qg, sg = q.qvla_gptq_quantize_host(Wr32, H=H, damp=0.05)
    assert np.array_equal(sg.view(np.uint32), so.view(np.uint32))
    # the two fp64 factorisations differ by rounding only (~1e-12 relative)
    check_gptq_flips(qg, qo, to, boundary=1e-6, max_frac=5e-4)
    for j in dead:
        assert not qg[:, j].any(), "a dead input must get zero codes"
    e_g, e_o = _recon_error(Wr32, qg, sg, xr), _recon_error(Wr32, qo, so, xr)
    assert e_g <= 1.001 * e_o


@pytest.mark.parametrize("T,K", [(1, 64), (300, 256), (1000, 1024)])
def test_hessian(q, T, K):
    """Against the oracle's product of the same fp32 rows (fp64 sums in another order)."""
    xr = (I.activations(2150 + T, T, K, std=1.3, n_outlier_cols=4) * 0.7).astype(np.float32)
    Hg = q.qvla_gptq_hessian_host(xr)
    Ho = O.gptq_hessian(xr.astype(np.float64))
    assert np.array_equal(Hg, Hg.T)
    scale = np.sqrt(np.outer(np.diag(Ho), np.diag(Ho))) + 1e-300
    assert (np.abs(Hg - Ho) / scale).max() < 1e-12
    assert np.all(np.linalg.eigvalsh(Hg) > -1e-9 * np.abs(np.diag(Hg)).max())


def test_identity_hessian_is_rtn(q):
    """H = I with no damping: U = I, no error feedback, so GPTQ is RTN."""
    N, K = 50, 256
    Wr32 = I.weights(2300, N, K, col_spread=5.0)
    qg, sg = q.qvla_gptq_quantize_host(Wr32, H=np.eye(K), damp=0.0)
    qr, sr = O.quantize_weights_fp32(Wr32)
    assert np.array_equal(qg, qr) and np.array_equal(sg.view(np.uint32), sr.view(np.uint32))


def test_gptq_beats_rtn_on_the_calibration_output(q):
    pk, xr = _case(2400, 128, 512, 64, 800)
    Wr32 = pk.Wr.astype(np.float32)
    qg, sg = q.qvla_gptq_quantize_host(Wr32, H=O.gptq_hessian(xr), damp=0.05)
    qr, sr = O.quantize_weights_fp32(Wr32)
    assert _recon_error(Wr32, qg, sg, xr) < 0.8 * _recon_error(Wr32, qr, sr, xr)


def test_argument_errors(q):
    Wr = np.zeros((4, 64), np.float32)
    with pytest.raises(RuntimeError, match="ARG|argument"):
        q.qvla_gptq_quantize_host(Wr)                          # neither H nor U
    with pytest.raises(RuntimeError, match="ARG|argument"):
        q.qvla_gptq_quantize_host(Wr, H=-np.eye(64), damp=0.0)  # not positive definite
    with pytest.raises(RuntimeError, match="SHAPE|shape"):
        q.qvla_gptq_quantize_host(np.zeros((1, 4160), np.float32), U=np.eye(4160))
