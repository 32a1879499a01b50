"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol include/qvla.h declares, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib_mod():
    from w4a4_post_quantization_zigzag_b200 import build
    build.build()
    from w4a4_post_quantization_zigzag_b200 import qvla
    return qvla


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "qvla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qvla_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("qvla_pack_weights", "qvla_rotate_quant_act", "qvla_w4a4_gemm"):
        assert s in syms


def test_library_exports_every_declared_symbol():
    q = _lib_mod()
    lib = ctypes.CDLL(q.LIB_PATH)
    for s in declared_symbols():
        assert hasattr(lib, s), s
    assert set(declared_symbols()) == set(q.EXPORTED)


def test_status_strings_and_version():
    q = _lib_mod()
    assert q.qvla_abi_version() == 2
    for code in range(9):
        assert q.qvla_status_str(code)
    assert q.qvla_status_str(q.QVLA_ERR_STEP_RANGE).startswith("denoising step")


def test_packed_sizes_and_shape_errors():
    q = _lib_mod()
    wq, rot, tc, ws = q.qvla_packed_sizes(4096, 1024, 64)
    assert wq == 4096 * 1024 // 2 and rot == 1024 * 64 * 4 and ws > 4096 * 1024 * 4
    assert tc == 6 * 1024 * 64
    assert q.qvla_packed_sizes(256, 512, 256)[2] == 0          # no tensor-core image
    assert q.qvla_packed_sizes(256, 512, 128)[2] == 6 * 512 * 128
    for args in ((4096, 1000, 64), (4096, 1024, 48), (0, 1024, 64), (16, 65536, 64),
                 (16, 1024, 512)):
        with pytest.raises(q.QvlaError) as e:
            q.qvla_packed_sizes(*args)
        assert e.value.code == q.QVLA_ERR_SHAPE


def test_argument_errors_before_any_cuda_call():
    q = _lib_mod()
    lib = q._lib
    # null packed linear
    assert lib.qvla_rotate_quant_act(None, 1, 4, 64, None, 0, None, 0, 0, None, 0, 0, None,
                                     None, None, 0, None) == q.QVLA_ERR_ARG
    L = q.qvla_packed_linear(128, 256, 64, 0, 0, None, 0, 0, None)
    assert lib.qvla_w4a4_gemm(None, None, 4, ctypes.byref(L), None, 128, 0, None) == q.QVLA_ERR_ARG
    # bad shape inside the struct
    Lbad = q.qvla_packed_linear(128, 250, 64, 16, 16, None, 16, 16, None)
    assert lib.qvla_rotate_act_f32(ctypes.c_void_p(16), 1, 4, 256, ctypes.byref(Lbad),
                                   ctypes.c_void_p(16), None) == q.QVLA_ERR_SHAPE
    # no permutation
    Lnop = q.qvla_packed_linear(128, 256, 64, 0, 16, 16, 16, 16, None)
    assert lib.qvla_rotate_act_f32(ctypes.c_void_p(16), 1, 4, 256, ctypes.byref(Lnop),
                                   ctypes.c_void_p(16), None) == q.QVLA_ERR_ARG
    # misaligned pointers
    Lmis = q.qvla_packed_linear(128, 256, 64, 16, 24, None, 16, 16, None)
    assert lib.qvla_rotate_act_f32(ctypes.c_void_p(16), 1, 4, 256, ctypes.byref(Lmis),
                                   ctypes.c_void_p(16), None) == q.QVLA_ERR_ALIGN
    # table mode: layer or host step outside the table -> STEP_RANGE, never a clamp
    Lok = q.qvla_packed_linear(128, 256, 64, 16, 16, None, 16, 16, None)
    args = lambda step, layer: (ctypes.c_void_p(16), 1, 4, 256, ctypes.byref(Lok),
                                q.QVLA_SCALE_TABLE, ctypes.c_void_p(16), 10, 12, None, step,
                                layer, ctypes.c_void_p(16), ctypes.c_void_p(16), None, 0, None)
    assert lib.qvla_rotate_quant_act(*args(10, 0)) == q.QVLA_ERR_STEP_RANGE
    assert lib.qvla_rotate_quant_act(*args(-1, 0)) == q.QVLA_ERR_STEP_RANGE
    assert lib.qvla_rotate_quant_act(*args(0, 12)) == q.QVLA_ERR_STEP_RANGE
    # table mode without a table
    assert lib.qvla_quant_act_f32(ctypes.c_void_p(16), 4, 256, q.QVLA_SCALE_TABLE, None, 10, 12,
                                  None, 0, 0, ctypes.c_void_p(16), ctypes.c_void_p(16),
                                  None) == q.QVLA_ERR_ARG
    # empty input is a no-op
    assert lib.qvla_rotate_quant_act(None, 1, 0, 256, ctypes.byref(Lok), 0, None, 0, 0, None, 0,
                                     0, None, None, None, 0, None) == q.QVLA_OK
    # scratch size query: the tensor-core route (bf16, block 64 / 128) uses it
    assert q.qvla_rotate_quant_workspace_bytes(1024, 2048, 128) == 1024 * 2048 * 2 + 1024 * 16 * 4
    assert q.qvla_rotate_quant_workspace_bytes(50, 2048, 64) == 50 * 2048 * 2 + 50 * 32 * 4
    assert q.qvla_rotate_quant_workspace_bytes(50, 2048, 64, torch.float32) == 0
    assert q.qvla_rotate_quant_workspace_bytes(0, 2048, 64) == 0
    assert q.qvla_rotate_quant_workspace_bytes(1024, 2048, 256) == 0
    # the W8A8 activation entry: fp32 rows plus the permuted copy
    assert q.qvla_rotate_quant_a8_workspace_bytes(50, 1024) == 50 * 1024 * 6
    assert lib.qvla_w4a4_gemm_s32(None, 0, ctypes.byref(Lok), None, 0, None) == q.QVLA_OK
    # split-K factor must be a power of two <= 16 and <= the number of 256-wide K tiles
    Lw = q.qvla_packed_linear(128, 256, 64, 16, 16, None, 16, 16, None)
    assert lib.qvla_w4a4_gemm_s32(ctypes.c_void_p(16), 4, ctypes.byref(Lw), ctypes.c_void_p(16),
                                  3, None) == q.QVLA_ERR_ARG
    assert lib.qvla_w4a4_gemm_s32(ctypes.c_void_p(16), 4, ctypes.byref(Lw), ctypes.c_void_p(16),
                                  2, None) == q.QVLA_ERR_SHAPE


def test_pack_workspace_check():
    q = _lib_mod()
    lib = q._lib
    assert lib.qvla_pack_weights(ctypes.c_void_p(16), 64, 256, 64, None, None,
                                 ctypes.c_void_p(16), ctypes.c_void_p(16), None,
                                 ctypes.c_void_p(16), ctypes.c_void_p(16), None, 0,
                                 None) == q.QVLA_ERR_WORKSPACE


def test_variant_entry_points_reject_bad_arguments():
    """The Hadamard-only, W8A8 and GPTQ entry points validate on the host,
    before any CUDA call (no GPU here)."""
    q = _lib_mod()
    lib = q._lib
    P = ctypes.c_void_p(16)
    big = 1 << 30
    # GPTQ pack: K beyond the host factorisation's limit; neither calibration
    # rows nor a factor; calibration scratch too small for T x K fp32 rows
    assert lib.qvla_pack_weights_gptq(P, 64, 8192, 64, P, 1, 100, 0.05, None, None, None, P, P,
                                      None, P, P, P, big, P, big, None) == q.QVLA_ERR_SHAPE
    assert lib.qvla_pack_weights_gptq(P, 64, 256, 64, None, 1, 0, 0.05, None, None, None, P, P,
                                      None, P, P, P, big, None, 0, None) == q.QVLA_ERR_ARG
    assert lib.qvla_pack_weights_gptq(P, 64, 256, 64, P, 1, 100, 0.05, None, None, None, P, P,
                                      None, P, P, P, big, P, 100 * 256 * 4 - 1,
                                      None) == q.QVLA_ERR_WORKSPACE
    # Hadamard-only and W8 packs: a block size outside {32, 64, 128, 256}
    assert lib.qvla_pack_weights_hadamard(P, 64, 256, 48, None, P, None, P, P, P, big,
                                          None) == q.QVLA_ERR_SHAPE
    assert lib.qvla_pack_weights_w8(P, 64, 256, 48, None, None, P, P, None, P, P, P, big,
                                    None) == q.QVLA_ERR_SHAPE
    # 8-bit activations: no packed linear; workspace below the M x K fp32 rows
    L = q.qvla_packed_linear(128, 256, 64, 16, 16, None, 16, 16, None)
    assert lib.qvla_rotate_quant_act_a8(P, 1, 4, 256, None, P, P, P, big,
                                        None) == q.QVLA_ERR_ARG
    assert lib.qvla_rotate_quant_act_a8(P, 1, 4, 256, ctypes.byref(L), P, P, P, 4 * 256 * 4 - 1,
                                        None) == q.QVLA_ERR_WORKSPACE
    # W8A8 GEMM: no output; no packed linear; nothing to do for M = 0
    assert lib.qvla_w8a8_gemm(P, P, 4, ctypes.byref(L), None, 256, None) == q.QVLA_ERR_ARG
    assert lib.qvla_w8a8_gemm_s32(P, 4, None, P, None) == q.QVLA_ERR_ARG
    assert lib.qvla_w8a8_gemm_s32(None, 0, ctypes.byref(L), None, None) == q.QVLA_OK


def test_batched_w8a8_entry_points_reject_bad_arguments():
    """The batched W8A8 entry points check every problem on the host: scratch
    below M * K * 4 bytes, overlapping scratch, missing outputs."""
    q = _lib_mod()
    lib = q._lib
    L = q.qvla_packed_linear(128, 256, 64, 16, 16, None, 16, 16, None)

    def prob(M, ws, ws_bytes, xq8=16, y=16):
        return q.qvla_linear_problem(ctypes.pointer(L), 16, q.QVLA_DTYPE_BF16, M, 256, 0, None, 0,
                                     0, None, 0, 0, 16, 16, y, 128, ws, ws_bytes, xq8)

    def call(fn, *ps):
        arr = (q.qvla_linear_problem * len(ps))(*ps)
        return fn(arr, len(ps), None)

    a8 = lib.qvla_rotate_quant_act_a8_batched
    g8 = lib.qvla_w8a8_gemm_batched
    assert a8(None, 1, None) == q.QVLA_ERR_ARG and g8(None, -1, None) == q.QVLA_ERR_ARG
    assert a8(None, 0, None) == q.QVLA_OK and g8(None, 0, None) == q.QVLA_OK
    assert call(a8, prob(4, 1 << 20, 4 * 256 * 4 - 1)) == q.QVLA_ERR_WORKSPACE
    assert call(a8, prob(4, None, 0)) == q.QVLA_ERR_WORKSPACE
    assert call(a8, prob(4, 1 << 20, 4 * 256 * 4, xq8=None)) == q.QVLA_ERR_ARG
    assert call(a8, prob(4, 1 << 20, 1 << 16), prob(4, (1 << 20) + 4096, 1 << 16)) == q.QVLA_ERR_ARG
    assert call(g8, prob(4, None, 0, y=None)) == q.QVLA_ERR_ARG
    assert call(a8, prob(0, None, 0)) == q.QVLA_OK


def test_selftest_wait_limit_is_checked_on_the_host():
    """Out-of-range wait limits are rejected before anything is launched."""
    q = _lib_mod()
    for ns in (0, 999, 10_000_001):
        with pytest.raises(q.QvlaError) as e:
            q.qvla_selftest_wait_timeout(ns, stream=0)
        assert e.value.code == q.QVLA_ERR_ARG


def test_library_carries_the_hash_of_its_sources():
    """build() rebuilds on any change of content (not of file times), and the
    loaded library reports the hash of exactly the sources on disk."""
    from w4a4_post_quantization_zigzag_b200 import build
    q = _lib_mod()
    h = build.source_hash()
    assert len(h) == 64 and q.qvla_source_hash() == h == build.library_stamp()
    assert build.up_to_date()
