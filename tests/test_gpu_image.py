"""The int8 image of the activation codes (qvla_linear_problem.xq8).

The header fixes the image as a rearrangement of the packed codes: byte k of a
row is 16 * q, and inside every aligned group of 32 codes the 16 even-indexed
codes come first, then the 16 odd-indexed ones.  Checks, through the C ABI:
  * the batched rotate-quantise writes exactly that image of the codes it
    packs, on the tensor-core route (bf16 x, block 64 / 128) and on the
    CUDA-core routes (fp32 x, blocks 32 / 256, which expand the packed codes);
  * the batched GEMM fed from the image gives bf16 outputs identical to the
    same GEMM unpacking xq, and within the bf16 tolerance of the oracle's
    dequantisation of the int64 product, over ragged M, N and K.
"""
import numpy as np
import pytest
import torch

from oracle import qvla_oracle as O
from w4a4_post_quantization_zigzag_b200 import inputs as I
from _parity import check_y, unpack

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


def image_of(codes):
    """The documented image of integer codes [M, K] (test-side restatement)."""
    c = np.asarray(codes, np.int64)
    M, K = c.shape
    g = c.reshape(M, K // 32, 32)
    return (np.concatenate([g[:, :, 0::2], g[:, :, 1::2]], axis=2).reshape(M, K) * 16).astype(np.int8)


def test_image_restatement_on_a_hand_case():
    codes = np.arange(64).reshape(1, 64) % 16 - 8
    img = image_of(codes)
    assert img[0, 0] == 16 * codes[0, 0] and img[0, 1] == 16 * codes[0, 2]
    assert img[0, 16] == 16 * codes[0, 1] and img[0, 31] == 16 * codes[0, 31]
    assert img[0, 32] == 16 * codes[0, 32] and img[0, 48] == 16 * codes[0, 33]


@pytest.mark.parametrize("M,K,b,dt,mode", [(50, 1024, 64, "bf16", "table"),
                                           (130, 512, 128, "bf16", "dynamic"),
                                           (16, 256, 64, "f32", "dynamic"),
                                           (40, 512, 32, "bf16", "table"),
                                           (9, 1024, 256, "bf16", "dynamic")])
def test_rotate_quant_writes_the_image_of_its_codes(q, M, K, b, dt, mode):
    W = I.weights(7000 + K + b, 96, K, col_spread=5.0)
    L = q.qvla_pack_weights(cu(W), b)
    x = I.activations(7001 + M, M, K, n_outlier_cols=3, dtype="f32")
    xd = cu(x) if dt == "f32" else cu(x).to(torch.bfloat16)
    tab = cu(I.scale_table(7002, 3, 2, I.step_sigmas(3)))
    kw = dict(table=tab, step=1, layer=1) if mode == "table" else {}
    md = q.QVLA_SCALE_TABLE if mode == "table" else q.QVLA_SCALE_DYNAMIC
    ws = torch.empty(max(q.qvla_rotate_quant_workspace_bytes(M, K, b), 16), dtype=torch.uint8,
                     device="cuda")
    p = q.LinearProblem(L, xd, md, workspace=ws, xq8=True, **kw)
    q.qvla_rotate_quant_act_batched([p])
    ref_q, ref_s = q.qvla_rotate_quant_act(xd, L, md, workspace=ws, **kw)
    torch.cuda.synchronize()
    assert torch.equal(p.xq, ref_q) and torch.equal(p.s_x, ref_s)
    assert np.array_equal(p.xq8.cpu().numpy(), image_of(unpack(p.xq.cpu().numpy())))
    assert q.qvla_read_error_word(clear=True) == 0


# M, N, K: ragged tokens (every token tile), N % 8 != 0, K % 128 != 0
IMAGE_GEMM_CASES = [(1, 256, 256), (16, 384, 1024), (50, 4096, 1024), (33, 1000, 1056),
                    (64, 200, 512), (100, 512, 2048), (128, 256, 256), (300, 640, 1024),
                    (520, 1024, 4096)]


@pytest.mark.parametrize("M,N,K", IMAGE_GEMM_CASES)
def test_gemm_from_the_image(q, M, N, K):
    qx = I.int_codes(7100 + M, M, K, -8, 7)
    qw = I.int_codes(7101 + N, N, K, -7, 7)
    qx[0, :] = -8
    qw[0, :] = -7
    s_x = I.positive_scales(7102, M, 0.05, 0.6)
    s_w = I.positive_scales(7103, N, 1e-3, 2e-2)
    b = I.bias(7104, N)
    L = q.from_host_packed(O.pack_nibbles(qw), s_w, np.arange(K, dtype=np.int32),
                           np.zeros((K // 32, 32, 32)), bias=b)
    xq = cu(O.pack_nibbles(qx))
    sx = cu(s_x)
    p_img = q.LinearProblem(L, xq=xq, s_x=sx, xq8=cu(image_of(qx)))
    p_pk = q.LinearProblem(L, xq=xq, s_x=sx)
    q.qvla_w4a4_gemm_batched([p_img])
    q.qvla_w4a4_gemm_batched([p_pk])
    torch.cuda.synchronize()
    assert torch.equal(p_img.y, p_pk.y), "image and packed activations disagree"
    check_y(p_img.y.float().cpu().numpy(), O.dequantize(O.int_gemm(qx, qw), s_x, s_w, b))
    assert q.qvla_read_error_word(clear=True) == 0


def test_gemm_batch_mixes_image_and_packed_problems(q):
    """One call with linears of different token tiles, some fed from the
    image and some from packed codes, each matching its own oracle."""
    shapes = [(50, 4096, 1024), (50, 1024, 4096), (16, 512, 512), (200, 384, 1024),
              (50, 256, 1056)]
    probs, refs = [], []
    for i, (M, N, K) in enumerate(shapes):
        qx = I.int_codes(7200 + i, M, K, -8, 7)
        qw = I.int_codes(7300 + i, N, K, -7, 7)
        s_x = I.positive_scales(7400 + i, M, 0.05, 0.6)
        s_w = I.positive_scales(7500 + i, N, 1e-3, 2e-2)
        L = q.from_host_packed(O.pack_nibbles(qw), s_w, np.arange(K, dtype=np.int32),
                               np.zeros((K // 32, 32, 32)))
        img = cu(image_of(qx)) if i % 2 == 0 else None
        probs.append(q.LinearProblem(L, xq=cu(O.pack_nibbles(qx)), s_x=cu(s_x), xq8=img))
        refs.append(O.dequantize(O.int_gemm(qx, qw), s_x, s_w))
    q.qvla_w4a4_gemm_batched(probs)
    torch.cuda.synchronize()
    for p, r in zip(probs, refs):
        check_y(p.y.float().cpu().numpy(), r)
    assert q.qvla_read_error_word(clear=True) == 0
