"""The kernels' failure path: every wait on another agent (TMA, tensor core,
a peer CTA) is bounded, and an expired wait reports QVLA_DEVERR_TIMEOUT in
the device error word instead of hanging or trapping.  The self-test kernel
waits, with the same bounded wait, on a barrier that nothing arrives on and
with tensor memory held; the test checks that the wait gives up, reports the
timeout bit, frees its tensor memory, and that the next ordinary layer runs
clean and correct on the same context."""
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


@pytest.mark.parametrize("limit_ns", [50_000, 1_000_000])
def test_expired_wait_sets_the_timeout_bit_and_the_context_survives(q, limit_ns):
    assert q.qvla_read_error_word(clear=True) == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    q.qvla_selftest_wait_timeout(limit_ns)
    ev1.record()
    torch.cuda.synchronize()
    assert q.qvla_read_error_word(clear=True) == q.QVLA_DEVERR_TIMEOUT
    # it waited at least the limit and gave up soon after it
    ms = ev0.elapsed_time(ev1)
    assert limit_ns * 1e-6 * 0.9 <= ms < limit_ns * 1e-6 + 50.0, ms
    # the next ordinary layer on the same context: clean and correct
    lin = I.single_linear().linears[0]
    W, x, b = lin.make_w(), lin.make_x(), lin.make_bias()
    ref = O.pack_linear(W, lin.block, bias=b)
    L = q.qvla_pack_weights(torch.from_numpy(W).cuda(), lin.block, bias=torch.from_numpy(b).cuda(),
                            perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
    xq, s_x = q.qvla_rotate_quant_act(torch.from_numpy(x).cuda(), L)
    y = q.qvla_w4a4_gemm(xq, s_x, L)
    torch.cuda.synchronize()
    assert q.qvla_read_error_word(clear=True) == 0
    out = O.linear_forward(x.astype(np.float64), ref)
    qx = unpack(xq.cpu().numpy()).astype(np.int64)
    check_codes_near_boundary(qx, out["qx"], out["xr"], out["s_x"])
    check_y(y.float().cpu().numpy(), O.dequantize(O.int_gemm(qx, ref.qw), out["s_x"], ref.s_w, b))
