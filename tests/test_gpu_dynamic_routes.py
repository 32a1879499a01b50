"""Per-token dynamic scale on the tensor-core route: the two ways its two passes
(row maximum, then quantisation) can run give the same codes, scales and int8
images, and both agree with the oracle.

- one launch, the row maximum reduced over a thread-block cluster along the
  rotation blocks (scratch of M * K * 2 bytes: the permuted copy only);
- two launches without clusters, every CTA's row maxima through the rest of
  the scratch (the full qvla_rotate_quant_workspace_bytes()), taken when it
  spreads the blocks better — wide and narrow linears in one batch, or few
  token tiles of a wide linear.

The scale is s = max_j |x'_j| / 7 per token (per-token absmax, symmetric
4-bit grid [-8, 7]); which launch computes the maximum must not change a bit
of it.
"""
import numpy as np
import pytest
import torch

from oracle import qvla_oracle as O
from w4a4_post_quantization_zigzag_b200 import inputs as I
from _parity import check_codes_near_boundary, unpack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    from w4a4_post_quantization_zigzag_b200 import qvla
    assert torch.cuda.is_available()
    qvla.qvla_read_error_word(clear=True)
    return qvla


def _linear(q, N, K, b, seed):
    W = I.weights(seed, N, K)
    ref = O.pack_linear(W, b)
    L = q.qvla_pack_weights(torch.from_numpy(W).cuda(), b, perm_in=ref.perm.astype(np.int32),
                            rsvd_in=ref.rsvd)
    return ref, L


def _launches(fn):
    """Kernel launches fn() makes: fn() runs once, then a second call is
    captured into a CUDA graph (not replayed) whose kernel nodes are counted."""
    from bench import kernel_nodes
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g, stream=torch.cuda.Stream()):
        fn()
    return kernel_nodes(g.raw_cuda_graph())


def _batch(q, specs, seed):
    """specs: (M, K, block) per linear; returns oracle refs, packed linears, inputs."""
    refs, Ls, xs = [], [], []
    for i, (M, K, b) in enumerate(specs):
        ref, L = _linear(q, 64, K, b, seed + 10 * i)
        refs.append(ref)
        Ls.append(L)
        xs.append(I.activations(seed + 10 * i + 1, M, K, std=1.2, n_outlier_cols=4,
                                heavy_tail_frac=0.01, heavy_tail_nu=3.0, heavy_tail_scale=10.0))
    return refs, Ls, xs


def _run(q, Ls, xs, full_scratch):
    probs = []
    for L, x in zip(Ls, xs):
        M, K = x.shape
        need = q.qvla_rotate_quant_workspace_bytes(M, K, L.block)
        assert need == M * K * 2 + M * (K // L.block) * 4
        nbytes = need if full_scratch else M * K * 2
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
        probs.append(q.LinearProblem(L, xd, q.QVLA_SCALE_DYNAMIC, workspace=ws, xq8=True))
    # the permuted copy (one launch for up to 16 linears), then the rotation
    n = _launches(lambda: q.qvla_rotate_quant_act_batched(probs)) - 1
    return probs, n


# (M, K, block) per linear of one batched call; the number of rotation
# launches each scratch size leads to (one per cluster size in the one-launch
# route, two per batch in the other)
CASES = [
    ([(3, 16384, 128)], 1, 2),                                   # one token tile, 128 blocks
    ([(300, 2048, 64)], 1, 2),
    ([(200, 2048, 128), (200, 8192, 128)], 1, 2),                # narrow and wide together
    ([(130, 1024, 64), (130, 4096, 64), (50, 1024, 64)], 1, 2),
    ([(37, 2048, 128)], 1, 1),                                   # the cluster route stays shorter
]


@pytest.mark.parametrize("specs,n_cluster,n_full", CASES)
def test_dynamic_routes_agree_and_match_the_oracle(q, specs, n_cluster, n_full):
    refs, Ls, xs = _batch(q, specs, 4400 + len(specs) * 97 + specs[0][1] // 64)
    p_small, n_small = _run(q, Ls, xs, full_scratch=False)
    p_full, n_full_seen = _run(q, Ls, xs, full_scratch=True)
    torch.cuda.synchronize()
    assert q.qvla_read_error_word(clear=True) == 0
    assert n_small == n_cluster
    assert n_full_seen == n_full
    for ref, x, a, b in zip(refs, xs, p_small, p_full):
        # the two routes: identical bits
        assert torch.equal(a.xq, b.xq)
        assert torch.equal(a.s_x.view(torch.int32), b.s_x.view(torch.int32))
        assert torch.equal(a.xq8, b.xq8)
        # and the oracle: scales within fp32 rounding of the fp64 rotation,
        # codes off by one only at a rounding boundary
        xr_ref, qx_ref, s_ref = O.rotate_quant_act(x, ref, "dynamic")
        np.testing.assert_allclose(b.s_x.cpu().numpy(), s_ref, rtol=2e-6)
        check_codes_near_boundary(unpack(b.xq.cpu().numpy()), qx_ref, xr_ref, s_ref, "activations")
        # the image is 16 * code, even codes of each 32 first, then the odd ones
        codes = unpack(b.xq.cpu().numpy()).astype(np.int32)
        M, K = codes.shape
        img = b.xq8.cpu().numpy().astype(np.int32).reshape(M, K // 32, 2, 16)
        c32 = codes.reshape(M, K // 32, 16, 2)
        assert np.array_equal(img[:, :, 0, :], 16 * c32[:, :, :, 0])
        assert np.array_equal(img[:, :, 1, :], 16 * c32[:, :, :, 1])


def test_dynamic_two_launch_route_zero_rows(q):
    """All-zero token rows (s = 0, codes 0) and a row with one huge entry, on
    the two-launch route: the maximum of a row comes from one CTA only."""
    M, K, b = 130, 8192, 128
    ref, L = _linear(q, 64, K, b, 4900)
    x = I.activations(4901, M, K, std=1.0, n_outlier_cols=2)
    x[5, :] = 0.0
    x[129, :] = 0.0
    x[64, 777] = 3072.0                       # exact in bf16
    probs, n = _run(q, [L], [x], full_scratch=True)
    torch.cuda.synchronize()
    assert q.qvla_read_error_word(clear=True) == 0
    assert n == 2
    p = probs[0]
    xr_ref, qx_ref, s_ref = O.rotate_quant_act(x, ref, "dynamic")
    s = p.s_x.cpu().numpy()
    assert s[5] == 0.0 and s[129] == 0.0
    assert not unpack(p.xq.cpu().numpy())[[5, 129]].any()
    np.testing.assert_allclose(s, s_ref, rtol=2e-6)
    check_codes_near_boundary(unpack(p.xq.cpu().numpy()), qx_ref, xr_ref, s_ref, "activations")
