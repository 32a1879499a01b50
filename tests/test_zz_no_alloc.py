"""The allocation-free rotate-quantise entry point (qvla_rotate_quant_act_noalloc).

Some callers cannot allocate device memory while they run a layer: a control
loop that must not call cudaMalloc once started, code being captured into a
CUDA graph, or a host application that gives the library no allocator.  For
them the scratch of the fast large-M route lives in a fixed per-device array
inside the library.  These checks call that entry point through the C ABI and
compare it with the ordinary entry point (given its own scratch) on two calls
in a row: the codes and scales must be identical, since both run the same
kernels on the same route.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from w4a4_post_quantization_zigzag_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    from w4a4_post_quantization_zigzag_b200 import qvla
    assert torch.cuda.is_available()
    qvla.qvla_read_error_word(clear=True)
    return qvla


def _packed(q, N, K, b, seed):
    W = torch.from_numpy(I.weights(seed, N, K)).cuda()
    return q.qvla_pack_weights(W, b)


@pytest.mark.parametrize("M,K,b,mode", [(256, 2048, 128, "dynamic"), (300, 1536, 64, "table"),
                                        (40, 1024, 64, "table")])
def test_noalloc_matches_the_allocating_entry_point_twice(q, M, K, b, mode):
    L = _packed(q, 128, K, b, 9000 + K)
    tab = torch.from_numpy(I.scale_table(9001, 4, 3, I.step_sigmas(4))).cuda()
    need = q.qvla_rotate_quant_workspace_bytes(M, K, b)
    assert need <= q.QVLA_NOALLOC_SCRATCH_BYTES
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    kw = dict(table=tab, step=2, layer=1) if mode == "table" else {}
    md = q.QVLA_SCALE_TABLE if mode == "table" else q.QVLA_SCALE_DYNAMIC
    xq = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    for call in range(2):                     # two calls in a row share the array
        x = torch.from_numpy(I.activations(9100 + call, M, K, n_outlier_cols=3)).cuda()
        x = x.to(torch.bfloat16)
        ref_q, ref_s = q.qvla_rotate_quant_act(x, L, md, workspace=ws, **kw)
        q.qvla_rotate_quant_act_noalloc(x, L, xq, sx, md, **kw)
        torch.cuda.synchronize()
        assert torch.equal(xq, ref_q), f"codes differ on call {call}"
        assert torch.equal(sx, ref_s), f"scales differ on call {call}"
    assert q.qvla_read_error_word(clear=True) == 0


def test_noalloc_runs_the_permuted_copy_route(q):
    """The fixed array must really serve as the scratch: the call has to launch
    the permuted-copy kernel (without usable scratch the route would gather
    instead and give the same bits, so equal outputs alone do not show it).
    Kernel names come from the PyTorch profiler's CUDA activity trace."""
    M, K, b = 64, 1024, 64
    L = _packed(q, 128, K, b, 9300)
    x = torch.from_numpy(I.activations(9301, M, K, n_outlier_cols=3)).cuda().to(torch.bfloat16)
    xq = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    q.qvla_rotate_quant_act_noalloc(x, L, xq, sx)            # first call: set-up outside the trace
    torch.cuda.synchronize()
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        q.qvla_rotate_quant_act_noalloc(x, L, xq, sx)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    if not names:
        pytest.skip("no CUDA activity trace in this process")
    assert any("permute_rows_kernel" in n for n in names), names
    ref_q, ref_s = q.qvla_rotate_quant_act(x, L)
    torch.cuda.synchronize()
    assert torch.equal(xq, ref_q) and torch.equal(sx, ref_s)
    assert q.qvla_read_error_word(clear=True) == 0


def test_noalloc_at_the_array_size_keeps_the_one_launch_route(q):
    """A permuted copy that fills the array exactly (1024 x 8192 bf16 = 16 MiB)
    leaves no room for the row maxima of the two-launch dynamic route: the call
    still runs, on the cluster route, and gives the bits of the allocating
    entry point (which has room and takes the two-launch route)."""
    M, K, b = 1024, 8192, 128
    assert M * K * 2 == q.QVLA_NOALLOC_SCRATCH_BYTES
    assert q.qvla_rotate_quant_workspace_bytes(M, K, b) > q.QVLA_NOALLOC_SCRATCH_BYTES
    L = _packed(q, 128, K, b, 9400)
    x = torch.from_numpy(I.activations(9401, M, K, n_outlier_cols=5)).cuda().to(torch.bfloat16)
    ws = torch.empty(q.qvla_rotate_quant_workspace_bytes(M, K, b), dtype=torch.uint8, device="cuda")
    ref_q, ref_s = q.qvla_rotate_quant_act(x, L, q.QVLA_SCALE_DYNAMIC, workspace=ws)
    xq = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    q.qvla_rotate_quant_act_noalloc(x, L, xq, sx, q.QVLA_SCALE_DYNAMIC)
    torch.cuda.synchronize()
    assert torch.equal(xq, ref_q) and torch.equal(sx, ref_s)
    assert q.qvla_read_error_word(clear=True) == 0


def test_noalloc_rejects_sizes_beyond_its_array(q):
    M, K, b = 1024, 16384, 128                # needs 32 MiB of scratch
    assert q.qvla_rotate_quant_workspace_bytes(M, K, b) > q.QVLA_NOALLOC_SCRATCH_BYTES
    L = _packed(q, 128, K, b, 9200)
    x = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    xq = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    with pytest.raises(q.QvlaError) as e:
        q.qvla_rotate_quant_act_noalloc(x, L, xq, sx, q.QVLA_SCALE_DYNAMIC)
    assert e.value.code == q.QVLA_ERR_WORKSPACE
