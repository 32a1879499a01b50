"""ctypes binding of ``libqvla.so`` (the C ABI declared in ``include/qvla.h``).

Argument marshalling only: every function here validates Python-side types,
allocates output tensors with PyTorch (device memory is PyTorch's job) and calls
the C entry point of the same name.  No step of the layer's arithmetic runs in
Python.  Importing this module loads the library and raises ImportError when it
has not been built (``python -m w4a4_post_quantization_zigzag_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_double, c_int, c_int32, c_size_t, c_uint32, c_void_p
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqvla.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m w4a4_post_quantization_zigzag_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)


def _check_stamp():
    """The loaded library must be the build of the sources next to it."""
    from . import build as _build
    _lib.qvla_source_hash.restype = ctypes.c_char_p
    have = _lib.qvla_source_hash().decode()
    want = _build.source_hash()
    if have != want:
        raise ImportError(f"{LIB_PATH} was built from other sources (stamp {have[:12]}, "
                          f"sources {want[:12]}): rebuild it with "
                          "`python -m w4a4_post_quantization_zigzag_b200.build`")


_check_stamp()

QVLA_OK = 0
QVLA_ERR_ARG = 1
QVLA_ERR_SHAPE = 2
QVLA_ERR_ALIGN = 3
QVLA_ERR_STEP_RANGE = 4
QVLA_ERR_UNSUPPORTED = 5
QVLA_ERR_CUDA = 6
QVLA_ERR_DEVICE_FLAG = 7
QVLA_ERR_WORKSPACE = 8

QVLA_DTYPE_F32 = 0
QVLA_DTYPE_BF16 = 1
QVLA_SCALE_DYNAMIC = 0
QVLA_SCALE_TABLE = 1

QVLA_DEVERR_STEP_RANGE = 0x1
QVLA_DEVERR_TIMEOUT = 0x2
QVLA_DEVERR_TMEM = 0x4

# Every symbol include/qvla.h declares.
EXPORTED = (
    "qvla_status_str", "qvla_abi_version", "qvla_read_error_word", "qvla_packed_sizes",
    "qvla_pack_weights", "qvla_rotate_weights_f32", "qvla_quant_pack_weights_f32",
    "qvla_rotate_quant_act", "qvla_rotate_act_f32", "qvla_quant_act_f32", "qvla_w4a4_gemm",
    "qvla_w4a4_gemm_s32", "qvla_rotate_quant_act_batched", "qvla_w4a4_gemm_batched",
    "qvla_rotate_quant_workspace_bytes", "qvla_rotate_quant_act_noalloc",
    "qvla_pack_weights_hadamard", "qvla_pack_weights_w8", "qvla_rotate_quant_act_a8",
    "qvla_rotate_quant_a8_workspace_bytes", "qvla_w8a8_gemm", "qvla_w8a8_gemm_s32",
    "qvla_gptq_quantize_host", "qvla_pack_weights_gptq", "qvla_gptq_hessian_host",
    "qvla_selftest_wait_timeout", "qvla_source_hash", "qvla_rotate_quant_act_a8_batched",
    "qvla_w8a8_gemm_batched",
)

QVLA_NOALLOC_SCRATCH_BYTES = 16 << 20


class qvla_packed_linear(ctypes.Structure):
    _fields_ = [("N", c_int32), ("K", c_int32), ("block", c_int32),
                ("perm", c_void_p), ("rot", c_void_p), ("rot_tc", c_void_p), ("wq", c_void_p),
                ("w_scale", c_void_p), ("bias", c_void_p)]


class qvla_linear_problem(ctypes.Structure):
    _fields_ = [("L", POINTER(qvla_packed_linear)), ("x", c_void_p), ("xdt", c_int32),
                ("M", c_int32), ("ldx", c_int32), ("mode", c_int32), ("table", c_void_p),
                ("T", c_int32), ("Lcount", c_int32), ("step_dev", c_void_p),
                ("step_host", c_int32), ("layer", c_int32), ("xq", c_void_p), ("s_x", c_void_p),
                ("y", c_void_p), ("ldy", c_int32), ("workspace", c_void_p),
                ("ws_bytes", c_size_t), ("xq8", c_void_p)]


_P = POINTER(qvla_packed_linear)
_PP = POINTER(qvla_linear_problem)
_sig = {
    "qvla_status_str": (ctypes.c_char_p, [c_int]),
    "qvla_abi_version": (c_int, []),
    "qvla_source_hash": (ctypes.c_char_p, []),
    "qvla_read_error_word": (c_int, [POINTER(c_uint32), c_int]),
    "qvla_selftest_wait_timeout": (c_int, [ctypes.c_uint64, c_void_p]),
    "qvla_packed_sizes": (c_int, [c_int, c_int, c_int, POINTER(c_size_t), POINTER(c_size_t),
                                  POINTER(c_size_t), POINTER(c_size_t)]),
    "qvla_pack_weights": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                  c_void_p]),
    "qvla_pack_weights_hadamard": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p,
                                           c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                           c_void_p]),
    "qvla_pack_weights_w8": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                     c_void_p]),
    "qvla_gptq_hessian_host": (c_int, [c_void_p, c_int, c_int, c_void_p]),
    "qvla_gptq_quantize_host": (c_int, [c_void_p, c_int, c_int, c_void_p, ctypes.c_double,
                                        c_void_p, c_void_p, c_void_p]),
    "qvla_pack_weights_gptq": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_int, c_int,
                                       ctypes.c_double, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                       c_void_p, c_size_t, c_void_p]),
    "qvla_rotate_quant_act_a8": (c_int, [c_void_p, c_int, c_int, c_int, _P, c_void_p, c_void_p,
                                         c_void_p, c_size_t, c_void_p]),
    "qvla_rotate_quant_a8_workspace_bytes": (c_int, [c_int, c_int, POINTER(c_size_t)]),
    "qvla_w8a8_gemm": (c_int, [c_void_p, c_void_p, c_int, _P, c_void_p, c_int, c_void_p]),
    "qvla_w8a8_gemm_s32": (c_int, [c_void_p, c_int, _P, c_void_p, c_void_p]),
    "qvla_rotate_weights_f32": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p,
                                        c_void_p, c_void_p]),
    "qvla_quant_pack_weights_f32": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p,
                                            c_void_p]),
    "qvla_rotate_quant_act": (c_int, [c_void_p, c_int, c_int, c_int, _P, c_int, c_void_p, c_int,
                                      c_int, c_void_p, c_int, c_int, c_void_p, c_void_p,
                                      c_void_p, c_size_t, c_void_p]),
    "qvla_rotate_quant_workspace_bytes": (c_int, [c_int, c_int, c_int, c_int, POINTER(c_size_t)]),
    "qvla_rotate_quant_act_noalloc": (c_int, [c_void_p, c_int, c_int, c_int, _P, c_int, c_void_p,
                                              c_int, c_int, c_void_p, c_int, c_int, c_void_p,
                                              c_void_p, c_void_p]),
    "qvla_rotate_act_f32": (c_int, [c_void_p, c_int, c_int, c_int, _P, c_void_p, c_void_p]),
    "qvla_quant_act_f32": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_int, c_int,
                                   c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "qvla_w4a4_gemm": (c_int, [c_void_p, c_void_p, c_int, _P, c_void_p, c_int, c_int, c_void_p]),
    "qvla_w4a4_gemm_s32": (c_int, [c_void_p, c_int, _P, c_void_p, c_int, c_void_p]),
    "qvla_rotate_quant_act_batched": (c_int, [_PP, c_int, c_void_p]),
    "qvla_w4a4_gemm_batched": (c_int, [_PP, c_int, c_int, c_void_p]),
    "qvla_rotate_quant_act_a8_batched": (c_int, [_PP, c_int, c_void_p]),
    "qvla_w8a8_gemm_batched": (c_int, [_PP, c_int, c_void_p]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class QvlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {qvla_status_str(code)} (status {code})")


def qvla_status_str(code: int) -> str:
    return _lib.qvla_status_str(code).decode()


def qvla_abi_version() -> int:
    return _lib.qvla_abi_version()


def qvla_source_hash() -> str:
    return _lib.qvla_source_hash().decode()


def _check(rc: int, where: str):
    if rc != QVLA_OK:
        raise QvlaError(rc, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(stream) -> c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return c_void_p(stream.cuda_stream)
    return c_void_p(int(stream))


def qvla_read_error_word(clear: bool = True) -> int:
    v = c_uint32(0)
    _check(_lib.qvla_read_error_word(ctypes.byref(v), int(clear)), "qvla_read_error_word")
    return int(v.value)


def qvla_selftest_wait_timeout(limit_ns: int = 50_000, stream=None):
    """Launch the failure-path self-test: a wait that nothing ends, bounded
    by limit_ns; the error word then holds QVLA_DEVERR_TIMEOUT."""
    _check(_lib.qvla_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "qvla_selftest_wait_timeout")


def qvla_packed_sizes(N: int, K: int, block: int) -> Tuple[int, int, int, int]:
    """(wq_bytes, rot_bytes, rot_tc_bytes, workspace_bytes)."""
    a, b, t, c = c_size_t(), c_size_t(), c_size_t(), c_size_t()
    _check(_lib.qvla_packed_sizes(N, K, block, ctypes.byref(a), ctypes.byref(b), ctypes.byref(t),
                                  ctypes.byref(c)), "qvla_packed_sizes")
    return a.value, b.value, t.value, c.value


class PackedLinear:
    """Device buffers of one packed linear plus the C struct that points at them."""

    def __init__(self, N, K, block, perm, rot, wq, w_scale, bias=None, rot_tc=None):
        self.N, self.K, self.block = int(N), int(K), int(block)
        self.perm, self.rot, self.wq, self.w_scale, self.bias = perm, rot, wq, w_scale, bias
        self.rot_tc = rot_tc
        self._s = qvla_packed_linear(self.N, self.K, self.block, perm.data_ptr(),
                                     rot.data_ptr() if rot is not None else None,
                                     rot_tc.data_ptr() if rot_tc is not None else None,
                                     wq.data_ptr(), w_scale.data_ptr(),
                                     bias.data_ptr() if bias is not None else None)

    @property
    def struct(self):
        return ctypes.byref(self._s)

    def device_bytes(self) -> int:
        n = sum(t.numel() * t.element_size() for t in (self.perm, self.rot, self.wq, self.w_scale)
                if t is not None)
        n += self.rot_tc.numel() * 2 if self.rot_tc is not None else 0
        return n + (self.bias.numel() * 4 if self.bias is not None else 0)


def qvla_pack_weights(W: torch.Tensor, block: int, bias: Optional[torch.Tensor] = None,
                      perm_in: Optional[np.ndarray] = None, rsvd_in: Optional[np.ndarray] = None,
                      stream=None) -> PackedLinear:
    """W: cuda fp32 [N, K].  perm_in: host int32 [K]; rsvd_in: host float64 [nb, b, b]."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2
    N, K = W.shape
    wq_b, rot_b, tc_b, ws_b = qvla_packed_sizes(N, K, block)
    dev = W.device
    perm = torch.empty(K, dtype=torch.int32, device=dev)
    rot = torch.empty(rot_b // 4, dtype=torch.float32, device=dev)
    rot_tc = torch.empty(tc_b // 2, dtype=torch.int16, device=dev) if tc_b else None
    wq = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
    s_w = torch.empty(N, dtype=torch.float32, device=dev)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=dev)
    p_in = r_in = None
    if perm_in is not None:
        perm_in = np.ascontiguousarray(perm_in, dtype=np.int32)
        assert perm_in.shape == (K,)
        p_in = perm_in.ctypes.data_as(c_void_p)
    if rsvd_in is not None:
        rsvd_in = np.ascontiguousarray(rsvd_in, dtype=np.float64)
        assert rsvd_in.shape == (K // block, block, block)
        r_in = rsvd_in.ctypes.data_as(c_void_p)
    _check(_lib.qvla_pack_weights(_ptr(W), N, K, block, p_in, r_in, _ptr(perm), _ptr(rot),
                                  _ptr(rot_tc), _ptr(wq), _ptr(s_w), _ptr(ws), ws_b,
                                  _stream(stream)), "qvla_pack_weights")
    if bias is not None:
        assert bias.is_cuda and bias.dtype == torch.float32 and bias.shape == (N,)
        bias = bias.contiguous()
    return PackedLinear(N, K, block, perm, rot.view(K // block, block, block), wq, s_w, bias,
                        rot_tc=rot_tc)


def qvla_pack_weights_hadamard(W: torch.Tensor, block: int, bias: Optional[torch.Tensor] = None,
                               perm_in: Optional[np.ndarray] = None, image: bool = True,
                               stream=None) -> PackedLinear:
    """Hadamard-only pack (R_SVD = I): rot = None; with `image` (blocks 64 /
    128) the tensor-core image of R_B = H_b, else rot_tc = None."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2
    N, K = W.shape
    wq_b, _, tc_b, ws_b = qvla_packed_sizes(N, K, block)
    dev = W.device
    rot_tc = torch.empty(tc_b // 2, dtype=torch.int16, device=dev) if (tc_b and image) else None
    perm = torch.empty(K, dtype=torch.int32, device=dev)
    wq = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
    s_w = torch.empty(N, dtype=torch.float32, device=dev)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=dev)
    p_in = None
    if perm_in is not None:
        perm_in = np.ascontiguousarray(perm_in, dtype=np.int32)
        assert perm_in.shape == (K,)
        p_in = perm_in.ctypes.data_as(c_void_p)
    _check(_lib.qvla_pack_weights_hadamard(_ptr(W), N, K, block, p_in, _ptr(perm),
                                           _ptr(rot_tc), _ptr(wq), _ptr(s_w), _ptr(ws), ws_b,
                                           _stream(stream)),
           "qvla_pack_weights_hadamard")
    if bias is not None:
        assert bias.is_cuda and bias.dtype == torch.float32 and bias.shape == (N,)
        bias = bias.contiguous()
    return PackedLinear(N, K, block, perm, None, wq, s_w, bias, rot_tc=rot_tc)


def _host_f64(a, shape):
    if a is None:
        return None, None
    a = np.ascontiguousarray(a, dtype=np.float64)
    assert a.shape == shape
    return a, a.ctypes.data_as(c_void_p)


def qvla_gptq_hessian_host(xr: np.ndarray) -> np.ndarray:
    """H = X'^T X' (fp64 [K, K]) of host fp32 rotated calibration rows [T, K]."""
    xr = np.ascontiguousarray(xr, dtype=np.float32)
    T, K = xr.shape
    H = np.empty((K, K), np.float64)
    _check(_lib.qvla_gptq_hessian_host(xr.ctypes.data_as(c_void_p), T, K,
                                       H.ctypes.data_as(c_void_p)), "qvla_gptq_hessian_host")
    return H


def qvla_gptq_quantize_host(Wr: np.ndarray, H: Optional[np.ndarray] = None, damp: float = 0.05,
                            U: Optional[np.ndarray] = None):
    """GPTQ codes of host fp32 rotated weights Wr [N, K]; returns (int8 [N, K], fp32 [N])."""
    Wr = np.ascontiguousarray(Wr, dtype=np.float32)
    N, K = Wr.shape
    H, h_p = _host_f64(H, (K, K))
    U, u_p = _host_f64(U, (K, K))
    q = np.empty((N, K), np.int8)
    s = np.empty(N, np.float32)
    _check(_lib.qvla_gptq_quantize_host(Wr.ctypes.data_as(c_void_p), N, K, h_p, float(damp), u_p,
                                        q.ctypes.data_as(c_void_p), s.ctypes.data_as(c_void_p)),
           "qvla_gptq_quantize_host")
    return q, s


def qvla_pack_weights_gptq(W: torch.Tensor, block: int, x_cal: Optional[torch.Tensor] = None,
                           damp: float = 0.05, bias: Optional[torch.Tensor] = None,
                           perm_in: Optional[np.ndarray] = None,
                           rsvd_in: Optional[np.ndarray] = None, U: Optional[np.ndarray] = None,
                           stream=None) -> PackedLinear:
    """As qvla_pack_weights, with GPTQ weight codes (calibration rows x_cal [T, K] on the device,
    fp32 or bf16, or a given inverse-Hessian factor U)."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2
    N, K = W.shape
    wq_b, rot_b, tc_b, ws_b = qvla_packed_sizes(N, K, block)
    dev = W.device
    perm = torch.empty(K, dtype=torch.int32, device=dev)
    rot = torch.empty(rot_b // 4, dtype=torch.float32, device=dev)
    rot_tc = torch.empty(tc_b // 2, dtype=torch.int16, device=dev) if tc_b else None
    wq = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
    s_w = torch.empty(N, dtype=torch.float32, device=dev)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=dev)
    p_in = None
    if perm_in is not None:
        perm_in = np.ascontiguousarray(perm_in, dtype=np.int32)
        assert perm_in.shape == (K,)
        p_in = perm_in.ctypes.data_as(c_void_p)
    rsvd_in, r_in = _host_f64(rsvd_in, (K // block, block, block))
    U, u_p = _host_f64(U, (K, K))
    T, xdt, cal, cal_b = 0, QVLA_DTYPE_F32, None, 0
    if x_cal is not None:
        assert x_cal.is_cuda and x_cal.is_contiguous() and x_cal.dim() == 2 and x_cal.shape[1] == K
        xdt = _dtype_code(x_cal)
        T = x_cal.shape[0]
        cal = torch.empty(T * K, dtype=torch.float32, device=dev)
        cal_b = T * K * 4
    _check(_lib.qvla_pack_weights_gptq(_ptr(W), N, K, block, _ptr(x_cal), xdt, T, float(damp),
                                       p_in, r_in, u_p, _ptr(perm), _ptr(rot), _ptr(rot_tc),
                                       _ptr(wq), _ptr(s_w), _ptr(ws), ws_b, _ptr(cal), cal_b,
                                       _stream(stream)), "qvla_pack_weights_gptq")
    if bias is not None:
        assert bias.is_cuda and bias.dtype == torch.float32 and bias.shape == (N,)
        bias = bias.contiguous()
    return PackedLinear(N, K, block, perm, rot.view(K // block, block, block), wq, s_w, bias,
                        rot_tc=rot_tc)


def qvla_pack_weights_w8(W: torch.Tensor, block: int, bias: Optional[torch.Tensor] = None,
                         perm_in: Optional[np.ndarray] = None,
                         rsvd_in: Optional[np.ndarray] = None, image: bool = True,
                         stream=None) -> PackedLinear:
    """W8A8 variant: the same P and R (and, with `image`, the tensor-core image
    of R_B for blocks 64 / 128), int8 weight codes wq [N, K]."""
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2
    N, K = W.shape
    _, rot_b, tc_b, ws_b = qvla_packed_sizes(N, K, block)
    dev = W.device
    rot_tc = torch.empty(tc_b // 2, dtype=torch.int16, device=dev) if (tc_b and image) else None
    perm = torch.empty(K, dtype=torch.int32, device=dev)
    rot = torch.empty(rot_b // 4, dtype=torch.float32, device=dev)
    wq = torch.empty(N, K, dtype=torch.int8, device=dev)
    s_w = torch.empty(N, dtype=torch.float32, device=dev)
    ws = torch.empty(ws_b, dtype=torch.uint8, device=dev)
    p_in = r_in = None
    if perm_in is not None:
        perm_in = np.ascontiguousarray(perm_in, dtype=np.int32)
        assert perm_in.shape == (K,)
        p_in = perm_in.ctypes.data_as(c_void_p)
    if rsvd_in is not None:
        rsvd_in = np.ascontiguousarray(rsvd_in, dtype=np.float64)
        assert rsvd_in.shape == (K // block, block, block)
        r_in = rsvd_in.ctypes.data_as(c_void_p)
    _check(_lib.qvla_pack_weights_w8(_ptr(W), N, K, block, p_in, r_in, _ptr(perm), _ptr(rot),
                                     _ptr(rot_tc), _ptr(wq), _ptr(s_w), _ptr(ws), ws_b,
                                     _stream(stream)),
           "qvla_pack_weights_w8")
    if bias is not None:
        assert bias.is_cuda and bias.dtype == torch.float32 and bias.shape == (N,)
        bias = bias.contiguous()
    return PackedLinear(N, K, block, perm, rot.view(K // block, block, block), wq, s_w, bias,
                        rot_tc=rot_tc)


def qvla_rotate_quant_a8_workspace_bytes(M: int, K: int) -> int:
    b = c_size_t()
    _check(_lib.qvla_rotate_quant_a8_workspace_bytes(M, K, ctypes.byref(b)),
           "qvla_rotate_quant_a8_workspace_bytes")
    return b.value


def qvla_rotate_quant_act_a8(x: torch.Tensor, L: PackedLinear,
                             xq8: Optional[torch.Tensor] = None,
                             s_x: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None, stream=None):
    """8-bit per-token dynamic codes xq8 [M, K] int8 and s_x [M]."""
    M = x.shape[0]
    if xq8 is None:
        xq8 = torch.empty(M, L.K, dtype=torch.int8, device=x.device)
    if s_x is None:
        s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty(max(qvla_rotate_quant_a8_workspace_bytes(M, L.K), 16),
                                dtype=torch.uint8, device=x.device)
    _check(_lib.qvla_rotate_quant_act_a8(_ptr(x), _dtype_code(x), M, x.stride(0), L.struct,
                                         _ptr(xq8), _ptr(s_x), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)), "qvla_rotate_quant_act_a8")
    return xq8, s_x


def qvla_w8a8_gemm(xq8: torch.Tensor, s_x: torch.Tensor, L: PackedLinear,
                   y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M = xq8.shape[0]
    if y is None:
        y = torch.empty(M, L.N, dtype=torch.bfloat16, device=xq8.device)
    _check(_lib.qvla_w8a8_gemm(_ptr(xq8), _ptr(s_x), M, L.struct, _ptr(y), y.stride(0),
                               _stream(stream)), "qvla_w8a8_gemm")
    return y


def qvla_w8a8_gemm_s32(xq8: torch.Tensor, L: PackedLinear, stream=None) -> torch.Tensor:
    M = xq8.shape[0]
    acc = torch.empty(M, L.N, dtype=torch.int32, device=xq8.device)
    _check(_lib.qvla_w8a8_gemm_s32(_ptr(xq8), M, L.struct, _ptr(acc), _stream(stream)),
           "qvla_w8a8_gemm_s32")
    return acc


def qvla_rotate_weights_f32(W: torch.Tensor, block: int, perm: torch.Tensor,
                            rsvd64: torch.Tensor, stream=None) -> torch.Tensor:
    N, K = W.shape
    Wr = torch.empty(N, K, dtype=torch.float32, device=W.device)
    _check(_lib.qvla_rotate_weights_f32(_ptr(W), N, K, block, _ptr(perm), _ptr(rsvd64), _ptr(Wr),
                                        _stream(stream)), "qvla_rotate_weights_f32")
    return Wr


def qvla_quant_pack_weights_f32(Wr: torch.Tensor, stream=None):
    N, K = Wr.shape
    wq = torch.empty(N, K // 2, dtype=torch.uint8, device=Wr.device)
    s_w = torch.empty(N, dtype=torch.float32, device=Wr.device)
    _check(_lib.qvla_quant_pack_weights_f32(_ptr(Wr), N, K, _ptr(wq), _ptr(s_w), _stream(stream)),
           "qvla_quant_pack_weights_f32")
    return wq, s_w


def _dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return QVLA_DTYPE_BF16
    if x.dtype == torch.float32:
        return QVLA_DTYPE_F32
    raise TypeError(f"unsupported activation dtype {x.dtype}")


def _expect(t: torch.Tensor, dtype, shape, device, name: str):
    """Caller-given buffers: the kernels write exactly this shape, densely."""
    if (t.dtype != dtype or tuple(t.shape) != tuple(shape) or t.device != device
            or not t.is_contiguous()):
        raise ValueError(f"{name}: expected a contiguous {dtype} tensor of shape {tuple(shape)} "
                         f"on {device}, got {t.dtype} {tuple(t.shape)} on {t.device}"
                         f"{'' if t.is_contiguous() else ' (not contiguous)'}")


def _expect_rows(x: torch.Tensor, K: int, name: str = "x"):
    """Token rows [M, K] with unit stride along K (any row pitch)."""
    if x.dim() != 2 or x.shape[1] != K or (x.numel() and x.stride(1) != 1):
        raise ValueError(f"{name}: expected [M, {K}] rows with unit stride along K, "
                         f"got shape {tuple(x.shape)} strides {tuple(x.stride())}")


def _step_args(step):
    """int -> checked on the host; cuda int32 tensor -> read on the device."""
    if step is None:
        return None, 0
    if isinstance(step, torch.Tensor):
        assert step.is_cuda and step.dtype == torch.int32
        return _ptr(step), 0
    return None, int(step)


def qvla_rotate_quant_workspace_bytes(M: int, K: int, block: int, dtype=torch.bfloat16) -> int:
    b = c_size_t()
    code = QVLA_DTYPE_BF16 if dtype == torch.bfloat16 else QVLA_DTYPE_F32
    _check(_lib.qvla_rotate_quant_workspace_bytes(M, K, block, code, ctypes.byref(b)),
           "qvla_rotate_quant_workspace_bytes")
    return b.value


def qvla_rotate_quant_act(x: torch.Tensor, L: PackedLinear, mode: int = QVLA_SCALE_DYNAMIC,
                          table: Optional[torch.Tensor] = None, step=None, layer: int = 0,
                          xq: Optional[torch.Tensor] = None, s_x: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None, stream=None):
    """workspace: optional uint8 device scratch of qvla_rotate_quant_workspace_bytes() bytes."""
    _expect_rows(x, L.K)
    M = x.shape[0]
    if xq is None:
        xq = torch.empty(M, L.K // 2, dtype=torch.uint8, device=x.device)
    if s_x is None:
        s_x = torch.empty(M, dtype=torch.float32, device=x.device)
    _expect(xq, torch.uint8, (M, L.K // 2), x.device, "xq")
    _expect(s_x, torch.float32, (M,), x.device, "s_x")
    T, Lc = (table.shape if table is not None else (0, 0))
    sd, sh = _step_args(step)
    ws_n = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.qvla_rotate_quant_act(_ptr(x), _dtype_code(x), M, x.stride(0), L.struct, mode,
                                      _ptr(table), T, Lc, sd, sh, layer, _ptr(xq), _ptr(s_x),
                                      _ptr(workspace), ws_n, _stream(stream)),
           "qvla_rotate_quant_act")
    return xq, s_x


def qvla_rotate_quant_act_noalloc(x: torch.Tensor, L: PackedLinear, xq: torch.Tensor,
                                  s_x: torch.Tensor, mode: int = QVLA_SCALE_DYNAMIC,
                                  table: Optional[torch.Tensor] = None, step=None,
                                  layer: int = 0, stream=None):
    """qvla_rotate_quant_act for callers that cannot allocate device memory:
    the outputs are given, and the scratch is the library's fixed per-device
    array (at most QVLA_NOALLOC_SCRATCH_BYTES).  Calls that may overlap on the
    GPU race on that array."""
    _expect_rows(x, L.K)
    M = x.shape[0]
    _expect(xq, torch.uint8, (M, L.K // 2), x.device, "xq")
    _expect(s_x, torch.float32, (M,), x.device, "s_x")
    T, Lc = (table.shape if table is not None else (0, 0))
    sd, sh = _step_args(step)
    _check(_lib.qvla_rotate_quant_act_noalloc(_ptr(x), _dtype_code(x), M, x.stride(0), L.struct,
                                              mode, _ptr(table), T, Lc, sd, sh, layer, _ptr(xq),
                                              _ptr(s_x), _stream(stream)),
           "qvla_rotate_quant_act_noalloc")
    return xq, s_x


def qvla_rotate_act_f32(x: torch.Tensor, L: PackedLinear, stream=None) -> torch.Tensor:
    M = x.shape[0]
    xr = torch.empty(M, L.K, dtype=torch.float32, device=x.device)
    _check(_lib.qvla_rotate_act_f32(_ptr(x), _dtype_code(x), M, x.stride(0), L.struct, _ptr(xr),
                                    _stream(stream)), "qvla_rotate_act_f32")
    return xr


def qvla_quant_act_f32(xr: torch.Tensor, mode: int = QVLA_SCALE_DYNAMIC,
                       table: Optional[torch.Tensor] = None, step=None, layer: int = 0,
                       stream=None):
    M, K = xr.shape
    xq = torch.empty(M, K // 2, dtype=torch.uint8, device=xr.device)
    s_x = torch.empty(M, dtype=torch.float32, device=xr.device)
    T, Lc = (table.shape if table is not None else (0, 0))
    sd, sh = _step_args(step)
    _check(_lib.qvla_quant_act_f32(_ptr(xr), M, K, mode, _ptr(table), T, Lc, sd, sh, layer,
                                   _ptr(xq), _ptr(s_x), _stream(stream)), "qvla_quant_act_f32")
    return xq, s_x


def qvla_w4a4_gemm(xq: torch.Tensor, s_x: torch.Tensor, L: PackedLinear, split_k: int = 0,
                   y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M = xq.shape[0]
    if y is None:
        y = torch.empty(M, L.N, dtype=torch.bfloat16, device=xq.device)
    _check(_lib.qvla_w4a4_gemm(_ptr(xq), _ptr(s_x), M, L.struct, _ptr(y), y.stride(0), split_k,
                               _stream(stream)), "qvla_w4a4_gemm")
    return y


def qvla_w4a4_gemm_s32(xq: torch.Tensor, L: PackedLinear, split_k: int = 0,
                       stream=None) -> torch.Tensor:
    M = xq.shape[0]
    acc = torch.empty(M, L.N, dtype=torch.int32, device=xq.device)
    _check(_lib.qvla_w4a4_gemm_s32(_ptr(xq), M, L.struct, _ptr(acc), split_k, _stream(stream)),
           "qvla_w4a4_gemm_s32")
    return acc


def from_host_packed(wq: np.ndarray, s_w: np.ndarray, perm: np.ndarray, rsvd: np.ndarray,
                     bias: Optional[np.ndarray] = None, device="cuda") -> PackedLinear:
    """Uploads host arrays into a PackedLinear (e.g. to run the GEMM on given codes)."""
    N, Kh = wq.shape
    K = 2 * Kh
    block = rsvd.shape[-1]
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).to(device)
    return PackedLinear(N, K, block, t(perm, np.int32), t(rsvd, np.float32), t(wq, np.uint8),
                        t(s_w, np.float32), None if bias is None else t(bias, np.float32))


class LinearProblem:
    """One independent linear of a batched call; keeps its tensors alive."""

    def __init__(self, L: PackedLinear, x: Optional[torch.Tensor] = None,
                 mode: int = QVLA_SCALE_DYNAMIC, table: Optional[torch.Tensor] = None,
                 step=None, layer: int = 0, xq: Optional[torch.Tensor] = None,
                 s_x: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, xq8=None):
        """xq8: the int8 image of the codes that the batched rotate-quantise
        writes and the batched GEMM reads (a device int8 [M, K] tensor, or
        True to allocate one); None leaves the GEMM to unpack xq."""
        M = x.shape[0] if x is not None else xq.shape[0]
        dev = (x if x is not None else xq).device
        if x is not None:
            _expect_rows(x, L.K)
        self.L, self.x, self.table, self.step = L, x, table, step
        self.xq = xq if xq is not None else torch.empty(M, L.K // 2, dtype=torch.uint8, device=dev)
        self.s_x = s_x if s_x is not None else torch.empty(M, dtype=torch.float32, device=dev)
        self.y = y if y is not None else torch.empty(M, L.N, dtype=torch.bfloat16, device=dev)
        if xq8 is True:
            xq8 = torch.empty(M, L.K, dtype=torch.int8, device=dev)
        self.xq8 = xq8
        _expect(self.xq, torch.uint8, (M, L.K // 2), dev, "xq")
        _expect(self.s_x, torch.float32, (M,), dev, "s_x")
        if xq8 is not None:
            _expect(xq8, torch.int8, (M, L.K), dev, "xq8")
        if self.y.dim() != 2 or tuple(self.y.shape) != (M, L.N) or self.y.stride(1) != 1 \
                or self.y.dtype != torch.bfloat16:
            raise ValueError(f"y: expected bf16 [{M}, {L.N}] rows with unit stride")
        T, Lc = (table.shape if table is not None else (0, 0))
        sd, sh = _step_args(step)
        self.c = qvla_linear_problem(
            ctypes.pointer(L._s), x.data_ptr() if x is not None else None,
            _dtype_code(x) if x is not None else QVLA_DTYPE_BF16, M,
            x.stride(0) if x is not None else L.K, mode,
            table.data_ptr() if table is not None else None, T, Lc,
            sd.value if sd is not None else None, sh, layer, self.xq.data_ptr(),
            self.s_x.data_ptr(), self.y.data_ptr(), self.y.stride(0),
            workspace.data_ptr() if workspace is not None else None,
            workspace.numel() * workspace.element_size() if workspace is not None else 0,
            xq8.data_ptr() if xq8 is not None else None)
        self.workspace = workspace


def _problem_array(problems):
    arr = (qvla_linear_problem * len(problems))(*[p.c for p in problems])
    return arr


def qvla_rotate_quant_act_batched(problems, stream=None):
    arr = _problem_array(problems)
    _check(_lib.qvla_rotate_quant_act_batched(arr, len(problems), _stream(stream)),
           "qvla_rotate_quant_act_batched")


def qvla_w4a4_gemm_batched(problems, split_k: int = 0, stream=None):
    arr = _problem_array(problems)
    _check(_lib.qvla_w4a4_gemm_batched(arr, len(problems), split_k, _stream(stream)),
           "qvla_w4a4_gemm_batched")


def qvla_rotate_quant_act_a8_batched(problems, stream=None):
    """8-bit activation codes of W8A8 linears: each problem's xq8 (int8
    [M, K]) receives the codes themselves and s_x the per-token scales; each
    problem needs a workspace (qvla_rotate_quant_a8_workspace_bytes)."""
    arr = _problem_array(problems)
    _check(_lib.qvla_rotate_quant_act_a8_batched(arr, len(problems), _stream(stream)),
           "qvla_rotate_quant_act_a8_batched")


def qvla_w8a8_gemm_batched(problems, stream=None):
    """W8A8 GEMMs of the problems (xq8 holds 8-bit codes, L a W8 pack)."""
    arr = _problem_array(problems)
    _check(_lib.qvla_w8a8_gemm_batched(arr, len(problems), _stream(stream)),
           "qvla_w8a8_gemm_batched")
