"""Parity over the roofline sweep (square K = N, bf16 x with 0.5% outlier
channels): a deterministic subset of the points that covers every token count,
width, block size and scale mode at least once, through the single-linear
C-ABI calls with rotate-quantise scratch (the route a large-M call takes).
Codes, scales and bf16 outputs are checked on sampled token rows that the
oracle computes one by one."""
import numpy as np
import pytest
import torch

from oracle import qvla_oracle as O
from w4a4_post_quantization_zigzag_b200 import inputs as I
from _parity import check_codes_near_boundary, check_y, unpack

POINTS = [  # M, K = N, block, mode
    (1, 1024, 32, "dynamic"), (16, 2048, 64, "table"), (64, 4096, 128, "dynamic"),
    (256, 1024, 256, "table"), (1024, 2048, 32, "table"), (4096, 1024, 64, "dynamic"),
    (8192, 1024, 128, "table"), (256, 8192, 64, "dynamic"), (64, 2048, 256, "dynamic"),
    (1024, 4096, 128, "table"),
]


@pytest.fixture(scope="module")
def q():
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    from w4a4_post_quantization_zigzag_b200 import qvla
    qvla.qvla_read_error_word(clear=True)
    return qvla


def test_points_cover_every_sweep_axis():
    for axis, values in ((0, I.SWEEP_M), (1, I.SWEEP_KN), (2, I.SWEEP_BLOCK), (3, I.SWEEP_MODE)):
        assert set(values) <= {p[axis] for p in POINTS}
    assert set(POINTS) <= set(I.sweep_points())


@pytest.mark.gpu
@pytest.mark.parametrize("M,KN,b,mode", POINTS)
def test_sweep_point_parity(q, M, KN, b, mode):
    wl = I.sweep_point(M, KN, b, mode)
    lin = wl.linears[0]
    W, bias, x = lin.make_w(), lin.make_bias(), lin.make_x()
    ref = O.pack_linear(W, b, bias=bias)
    L = q.qvla_pack_weights(torch.from_numpy(W).cuda(), b, bias=torch.from_numpy(bias).cuda(),
                            perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    nbytes = q.qvla_rotate_quant_workspace_bytes(M, KN, b)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    if mode == "table":
        tab = torch.from_numpy(wl.table).cuda()
        xq, s_x = q.qvla_rotate_quant_act(xd, L, q.QVLA_SCALE_TABLE, table=tab, step=0, layer=0,
                                          workspace=ws)
    else:
        xq, s_x = q.qvla_rotate_quant_act(xd, L, q.QVLA_SCALE_DYNAMIC, workspace=ws)
    y = q.qvla_w4a4_gemm(xq, s_x, L)
    torch.cuda.synchronize()
    assert q.qvla_read_error_word(clear=True) == 0
    rows = np.unique(np.array([0, M // 3, M // 2, M - 1]))
    xs = x[rows].astype(np.float64)
    out = (O.linear_forward(xs, ref, "table", wl.table, 0, 0) if mode == "table"
           else O.linear_forward(xs, ref))
    np.testing.assert_allclose(s_x.cpu().numpy()[rows], out["s_x"], rtol=2e-6)
    qx = unpack(xq.cpu().numpy()[rows])
    check_codes_near_boundary(qx, out["qx"], out["xr"], out["s_x"], f"{(M, KN, b, mode)} codes")
    y_ref = O.dequantize(O.int_gemm(qx, ref.qw), out["s_x"], ref.s_w, ref.bias)
    check_y(y.float().cpu().numpy()[rows], y_ref, f"{(M, KN, b, mode)} y")
