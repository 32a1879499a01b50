"""Parity at the full workload sizes, in the launch configuration the benchmark
uses (batched calls, scratch for the large-M route), checked on sampled token
rows that the oracle computes one by one: rotated codes (+-1 only at a rounding
boundary), scales, and bf16 outputs against the oracle's dequantisation of the
codes the GPU chose."""
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


def _run_batched(q, lins, xs, mode, table=None, step=0, scratch=True, image=False):
    """Pack every linear (GPU pack fed the oracle's permutation and R_SVD),
    run the batched rotate-quantise and GEMM (with `image`, the GEMM reads the
    int8 image of the codes); return oracle packs and problems."""
    refs, probs = [], []
    steps = torch.tensor([step], dtype=torch.int32, device="cuda")
    tab = torch.from_numpy(table).cuda() if table is not None else None
    for lin, x in zip(lins, xs):
        W, b = lin.make_w(), lin.make_bias()
        ref = O.pack_linear(W, lin.block, bias=b)
        L = q.qvla_pack_weights(torch.from_numpy(W).cuda(), lin.block,
                                bias=torch.from_numpy(b).cuda(),
                                perm_in=ref.perm.astype(np.int32), rsvd_in=ref.rsvd)
        xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
        ws = None
        if scratch:
            nbytes = q.qvla_rotate_quant_workspace_bytes(lin.M, lin.K, lin.block)
            ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
        md = q.QVLA_SCALE_TABLE if mode == "table" else q.QVLA_SCALE_DYNAMIC
        kw = dict(table=tab, step=steps, layer=lin.layer) if mode == "table" else {}
        probs.append(q.LinearProblem(L, xd, md, workspace=ws, xq8=True if image else None, **kw))
        refs.append(ref)
    q.qvla_rotate_quant_act_batched(probs)
    q.qvla_w4a4_gemm_batched(probs)
    torch.cuda.synchronize()
    assert q.qvla_read_error_word(clear=True) == 0
    return refs, probs


def _check_sampled(lin, x, ref, prob, rows, mode, table=None, step=0):
    xs = x[rows].astype(np.float64)
    if mode == "table":
        out = O.linear_forward(xs, ref, "table", table, step, lin.layer)
    else:
        out = O.linear_forward(xs, ref)
    np.testing.assert_allclose(prob.s_x.cpu().numpy()[rows], out["s_x"], rtol=2e-6)
    qx = unpack(prob.xq.cpu().numpy()[rows])
    check_codes_near_boundary(qx, out["qx"], out["xr"], out["s_x"], f"{lin.name} codes")
    y_ref = O.dequantize(O.int_gemm(qx, ref.qw), out["s_x"], ref.s_w, ref.bias)
    check_y(prob.y.float().cpu().numpy()[rows], y_ref, f"{lin.name} y")


def test_dit_mlp_stack_step_full_size(q):
    wl = I.dit_mlp_stack()
    t = 9
    xs = [l.make_x(seed_offset=t, std=float(wl.sigmas[t])) for l in wl.linears]
    refs, probs = _run_batched(q, wl.linears, xs, "table", wl.table, t, scratch=False)
    rows = np.random.default_rng(0).choice(wl.linears[0].M, 6, replace=False)
    for lin, x, ref, p in zip(wl.linears, xs, refs, probs):
        _check_sampled(lin, x, ref, p, rows, "table", wl.table, t)


def test_dit_mlp_stack_gate_up_fused_full_size(q):
    """Shared-input fusion: gate and up as one 1024->8192 linear (one
    permutation and rotation from the concatenated weights, one activation
    pass), in the batched launches of the fused step."""
    wl = I.dit_mlp_stack(fuse_gate_up=True)
    assert [l.N for l in wl.linears[:2]] == [8192, 1024] and len(wl.linears) == 8
    t = 4
    xs = [l.make_x(seed_offset=t, std=float(wl.sigmas[t])) for l in wl.linears]
    refs, probs = _run_batched(q, wl.linears, xs, "table", wl.table, t, scratch=False)
    rows = np.random.default_rng(3).choice(wl.linears[0].M, 5, replace=False)
    for lin, x, ref, p in zip(wl.linears[:2], xs, refs, probs):
        _check_sampled(lin, x, ref, p, rows, "table", wl.table, t)


def test_dit_denoise_loop_qkv_fused_layer_full_size(q):
    """Shared-input fusion: q, k and v as one 1536->4608 linear (one
    permutation and rotation from the concatenated weights, one activation
    pass), with o, up and down of the same layer in the batched launches."""
    wl = I.dit_denoise_loop(fuse_qkv=True)
    lins = wl.linears[:4]                                   # qkv, o, up, down of layer 0
    assert [(l.K, l.N) for l in lins] == [(1536, 4608), (1536, 1536), (1536, 6144), (6144, 1536)]
    t = 5
    xs = [l.make_x(seed_offset=t, std=float(wl.sigmas[t])) for l in lins]
    refs, probs = _run_batched(q, lins, xs, "table", wl.table, t, image=True)
    rows = np.random.default_rng(4).choice(lins[0].M, 5, replace=False)
    for lin, x, ref, p in zip(lins, xs, refs, probs):
        _check_sampled(lin, x, ref, p, rows, "table", wl.table, t)


def test_backbone_prefill_full_size(q):
    wl = I.backbone_prefill()
    xs = [l.make_x() for l in wl.linears]
    refs, probs = _run_batched(q, wl.linears, xs, "dynamic", image=True)
    rows = np.sort(np.random.default_rng(1).choice(1024, 6, replace=False))
    rows[-1] = 1023                                         # the ragged last tile's edge
    for lin, x, ref, p in zip(wl.linears, xs, refs, probs):
        _check_sampled(lin, x, ref, p, rows, "dynamic")


def test_dit_denoise_loop_layer_full_size(q):
    wl = I.dit_denoise_loop()
    lins = wl.linears[:6]                                   # q, k, v, o, up, down of layer 0
    t = 7
    xs = [l.make_x(seed_offset=t, std=float(wl.sigmas[t])) for l in lins]
    refs, probs = _run_batched(q, lins, xs, "table", wl.table, t)
    rows = np.random.default_rng(2).choice(lins[0].M, 6, replace=False)
    for lin, x, ref, p in zip(lins, xs, refs, probs):
        _check_sampled(lin, x, ref, p, rows, "table", wl.table, t)
