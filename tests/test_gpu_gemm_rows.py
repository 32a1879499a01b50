"""The persistent small-M W4A4 GEMM (up to 64 tokens; weight rows split across
CTAs, no partial sums), selected with QVLA_GEMM_PATH=rows.  Checks, through the C ABI:
  * int32 accumulators bit-exact against the oracle's integer GEMM;
  * every output element written exactly once (outputs pre-filled with NaN,
    padding columns of a wider row pitch left alone);
  * bf16 outputs byte-identical to the one-tile-per-CTA kernel (same epilogue
    arithmetic) and within tolerance of the oracle's dequantisation;
  * batches of many linears with mixed token tiles, widths and depths.
"""
import numpy as np
import pytest
import torch

from oracle import qvla_oracle as O
from w4a4_post_quantization_zigzag_b200 import inputs as I
from _parity import check_y

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def rows_path(monkeypatch):
    """Every call in this file takes the row-split kernel unless a test
    switches to the tile kernel."""
    monkeypatch.setenv("QVLA_GEMM_PATH", "rows")


@pytest.fixture(scope="module")
def q():
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    from w4a4_post_quantization_zigzag_b200 import qvla
    qvla.qvla_read_error_word(clear=True)
    return qvla


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _operands(seed, M, N, K, extremes=True):
    qx = I.int_codes(seed, M, K, -8, 7)
    qw = I.int_codes(seed + 1, N, K, -7, 7)
    if extremes:
        qx[0, :] = -8
        qw[0, :] = -7
        qw[N - 1, :] = 7
    s_x = I.positive_scales(seed + 2, M, 0.05, 0.6)
    s_w = I.positive_scales(seed + 3, N, 1e-3, 2e-2)
    b = I.bias(seed + 4, N)
    return qx, qw, s_x, s_w, b


def _packed(q, qw, s_w, b, K):
    return q.from_host_packed(O.pack_nibbles(qw), s_w, np.arange(K, dtype=np.int32),
                              np.zeros((K // 32, 32, 32)), bias=b)


def _nan_out(M, N):
    pitch = (N + 7) // 8 * 8 + 8                    # wider than N, a multiple of 8
    return torch.full((M, pitch), float("nan"), dtype=torch.bfloat16, device="cuda")


CASES = [  # M, N, K
    (1, 256, 256), (7, 3, 64), (16, 1000, 1056), (17, 200, 32), (33, 640, 4096),
    (50, 4096, 1024), (50, 1024, 4096), (64, 16384, 256), (64, 136, 2048), (40, 8, 32768),
    (16, 1001, 512), (64, 133, 256), (20, 4099, 128),
]


@pytest.mark.parametrize("M,N,K", CASES)
def test_rows_int32_accumulators_bit_exact(q, M, N, K):
    qx, qw, *_ = _operands(1300 + M + N, M, N, K)
    L = _packed(q, qw, np.ones(N, np.float32), None, K)
    acc = q.qvla_w4a4_gemm_s32(cu(O.pack_nibbles(qx)), L, split_k=0)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.int_gemm(qx, qw))
    assert q.qvla_read_error_word(clear=True) == 0


@pytest.mark.parametrize("M,N,K", CASES)
def test_rows_bf16_matches_tile_kernel_and_oracle(q, monkeypatch, M, N, K):
    qx, qw, s_x, s_w, b = _operands(1400 + M + N, M, N, K)
    L = _packed(q, qw, s_w, b, K)
    xq = cu(O.pack_nibbles(qx))
    y = _nan_out(M, N)
    q.qvla_w4a4_gemm(xq, cu(s_x), L, split_k=0, y=y[:, :N])
    torch.cuda.synchronize()
    assert torch.isnan(y[:, N:].float()).all(), "wrote past N"
    yr = y[:, :N].float().cpu().numpy()
    assert np.isfinite(yr).all(), "an output element was not written"
    check_y(yr, O.dequantize(O.int_gemm(qx, qw), s_x, s_w, b))
    monkeypatch.setenv("QVLA_GEMM_PATH", "tiles")
    for split in (0, 2):
        if split > (K + 255) // 256:
            continue
        y_t = _nan_out(M, N)
        q.qvla_w4a4_gemm(xq, cu(s_x), L, split_k=split, y=y_t[:, :N])
        torch.cuda.synchronize()
        assert torch.isnan(y_t[:, N:].float()).all(), f"tile kernel (split {split}) wrote past N"
        assert torch.equal(y[:, :N], y_t[:, :N]), f"tile kernel (split {split}) differs"
    assert q.qvla_read_error_word(clear=True) == 0


def test_rows_batched_many_linears(q, monkeypatch):
    """More linears than one launch takes (16), mixed token tiles (16/32/64)."""
    rng = np.random.default_rng(1500)
    specs = []
    for i in range(21):
        M = int(rng.choice([1, 5, 16, 20, 32, 45, 64]))
        N = int(rng.choice([8, 96, 384, 1000, 2048]))
        K = int(rng.choice([32, 256, 768, 2048]))
        specs.append((M, N, K))
    probs, refs = [], []
    for i, (M, N, K) in enumerate(specs):
        qx, qw, s_x, s_w, b = _operands(1600 + 10 * i, M, N, K, extremes=i % 2 == 0)
        L = _packed(q, qw, s_w, b, K)
        y = _nan_out(M, N)
        p = q.LinearProblem(L, xq=cu(O.pack_nibbles(qx)), s_x=cu(s_x), y=y[:, :N])
        p.full_y = y
        probs.append(p)
        refs.append(O.dequantize(O.int_gemm(qx, qw), s_x, s_w, b))
    q.qvla_w4a4_gemm_batched(probs)
    torch.cuda.synchronize()
    for (M, N, K), p, ref in zip(specs, probs, refs):
        assert torch.isnan(p.full_y[:, N:].float()).all()
        yr = p.y.float().cpu().numpy()
        assert np.isfinite(yr).all(), f"unwritten output in {(M, N, K)}"
        check_y(yr, ref, f"{(M, N, K)}")
    monkeypatch.setenv("QVLA_GEMM_PATH", "tiles")
    for p in probs:
        assert torch.equal(p.y, q.qvla_w4a4_gemm(p.xq, p.s_x, p.L))
    assert q.qvla_read_error_word(clear=True) == 0
