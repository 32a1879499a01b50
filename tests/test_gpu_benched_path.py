"""Parity of the exact path the benchmark times.

bench.py's DeviceStep builds the step: every linear with its own
rotate-quantise workspace (so the permuted-copy + TMA tensor-core route
runs), the int8 image of the codes, one batched rotate-quantise call and one
batched GEMM call per denoising step, the step index a device scalar.  Here
the same object is captured into one CUDA graph per step and replayed, and
after every replay the codes, scales and bf16 outputs of sampled token rows
are checked against the oracle (the GPU pack is fed the oracle's permutation
and R_SVD, the non-unique parts of the pack).  Workloads: the DiT MLP stack
(50 tokens, 12 linears, all 10 steps) and one layer of the DiT denoise loop
(512 tokens, q/k/v/o/up/down, all 8 steps)."""
import numpy as np
import pytest
import torch

import bench
from oracle import qvla_oracle as O
from _parity import check_codes_near_boundary, check_y, unpack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    from w4a4_post_quantization_zigzag_b200 import qvla
    qvla.qvla_read_error_word(clear=True)
    return qvla


def _replay_and_check(q, wl, rows_per_linear, seed):
    refs = {}

    def pack_fn(lin, W, b):
        ref = O.pack_linear(W.cpu().numpy(), lin.block, bias=b.cpu().numpy())
        refs[lin.name] = ref
        return q.qvla_pack_weights(W, lin.block, bias=b, perm_in=ref.perm.astype(np.int32),
                                   rsvd_in=ref.rsvd)

    dev = torch.device("cuda")
    ds = bench.DeviceStep(wl, q, dev, pack_fn=pack_fn)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        ds.step_batched(0)                      # set-up calls outside capture
    torch.cuda.synchronize()
    graphs = []
    for t in range(ds.T):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            ds.step_batched(t)
        graphs.append(g)
    rng = np.random.default_rng(seed)
    for t in range(ds.T):
        with torch.cuda.stream(stream):
            graphs[t].replay()
        torch.cuda.synchronize()
        assert q.qvla_read_error_word(clear=True) == 0, f"device error at step {t}"
        for i, lin in enumerate(wl.linears):
            ref = refs[lin.name]
            rows = np.sort(rng.choice(lin.M, rows_per_linear, replace=False))
            x = ds.xs[t][i].float().cpu().numpy()[rows].astype(np.float64)
            out = O.linear_forward(x, ref, "table", wl.table, t, lin.layer)
            np.testing.assert_array_equal(ds.sx[i].cpu().numpy()[rows],
                                          out["s_x"].astype(np.float32))
            qx = unpack(ds.xq[i].cpu().numpy()[rows])
            check_codes_near_boundary(qx, out["qx"], out["xr"], out["s_x"],
                                      f"step {t} {lin.name} codes")
            img = ds.img[i].cpu().numpy()[rows].astype(np.int64).reshape(len(rows), -1, 32)
            g = qx.astype(np.int64).reshape(len(rows), -1, 32)
            assert np.array_equal(img, 16 * np.concatenate([g[:, :, 0::2], g[:, :, 1::2]], axis=2)), \
                f"step {t} {lin.name}: image differs from the codes"
            y_ref = O.dequantize(O.int_gemm(qx, ref.qw), out["s_x"], ref.s_w, ref.bias)
            check_y(ds.ys[i].float().cpu().numpy()[rows], y_ref, f"step {t} {lin.name} y")
    del graphs, ds


def test_dit_mlp_stack_graph_replay_every_step(q):
    _replay_and_check(q, bench.make_workload("dit_mlp_stack"), 4, 11)


def test_dit_denoise_loop_layer_graph_replay_every_step(q):
    wl = bench.make_workload("dit_denoise_loop")
    wl.linears = wl.linears[:6]                 # q, k, v, o, up, down of layer 0
    _replay_and_check(q, wl, 4, 12)


def test_mixed_precision_step_batched_equals_per_linear(q):
    """The benchmark's mixed-precision step (down projections at W8A8, through
    the batched 8-bit entry points) gives the same outputs, scales and codes as
    one call per linear, replayed from a graph."""
    wl = bench.make_workload("dit_mlp_stack")
    dev = torch.device("cuda")
    ds = bench.DeviceStep(wl, q, dev, precision="mix")
    assert ds.idx8 and all(wl.linears[i].name.endswith("down") for i in ds.idx8)
    stream = torch.cuda.Stream()
    t = 3
    with torch.cuda.stream(stream):
        ds.step_per_linear(t)
    torch.cuda.synchronize()
    ref = [(x.clone(), s.clone(), y.clone()) for x, s, y in zip(ds.xq, ds.sx, ds.ys)]
    for v in ds.ys:
        v.zero_()
    with torch.cuda.stream(stream):
        ds.step_batched(t)                      # set-up calls outside capture
    torch.cuda.synchronize()
    for v in ds.ys:
        v.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        ds.step_batched(t)
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    assert q.qvla_read_error_word(clear=True) == 0
    for i, (xq, s, y) in enumerate(ref):
        assert torch.equal(ds.xq[i], xq), wl.linears[i].name
        assert torch.equal(ds.sx[i], s), wl.linears[i].name
        assert torch.equal(ds.ys[i], y), wl.linears[i].name
    del g, ds
