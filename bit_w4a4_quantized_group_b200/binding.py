"""ctypes binding of libsvdq (argument marshalling only).

Every function keeps the name of the C entry point in ``include/svdq.h``.
The ``*_t`` helpers take torch tensors and pass their data pointers and the
current CUDA stream; they check nothing the library does not check itself.
Loading fails loudly when the library is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libsvdq.so")

SVDQ_OK, SVDQ_ERR_INVALID_ARG, SVDQ_ERR_UNSUPPORTED, SVDQ_ERR_CUDA, SVDQ_ERR_TIMEOUT = range(5)
SVDQ_FMT_NVFP4_G16 = 1
SVDQ_FMT_INT4_G64 = 2
SVDQ_FMT_MXFP4_G32 = 3
SVDQ_FMT_W8A8 = 4
FORMATS = {"nvfp4": SVDQ_FMT_NVFP4_G16, "int4": SVDQ_FMT_INT4_G64, "mxfp4": SVDQ_FMT_MXFP4_G32,
           "w8a8": SVDQ_FMT_W8A8}

EXPORTED = (
    "svdq_buffer_sizes", "svdq_pack_weight", "svdq_quantize_act_lowrank_down",
    "svdq_w4a4_gemm_lowrank_up", "svdq_status_string", "svdq_get_last_device_error",
    "svdq_last_launch_count", "svdq_last_cuda_error", "svdq_selftest_bounded_wait",
)


class svdq_sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("x", "a_codes", "a_scales", "z", "w_codes", "w_scales", "l1", "l2", "bias", "y")]


class SvdqError(RuntimeError):
    def __init__(self, status: int, what: str):
        detail = f" [{svdq_last_cuda_error()}]" if status == SVDQ_ERR_CUDA else ""
        super().__init__(f"{what}: {status_name(status)} ({status}){detail}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsvdq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libsvdq.so not found at {path}; run python -m bit_w4a4_quantized_group_b200.build")
    lib = ctypes.CDLL(path)
    vp, i64, c_int, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    lib.svdq_buffer_sizes.argtypes = [c_int, i64, i64, i64, c_int, ctypes.POINTER(svdq_sizes)]
    lib.svdq_pack_weight.argtypes = [c_int, i64, i64, c_int, f32, vp, vp, vp, vp, vp,
                                     ctypes.POINTER(ctypes.c_float), vp, vp]
    lib.svdq_quantize_act_lowrank_down.argtypes = [c_int, i64, i64, c_int, vp, vp, f32, vp, vp, vp, vp, vp]
    lib.svdq_w4a4_gemm_lowrank_up.argtypes = [c_int, i64, i64, i64, c_int, vp, vp, f32, vp, vp, f32,
                                              vp, vp, vp, vp, vp]
    lib.svdq_status_string.argtypes = [c_int]
    lib.svdq_status_string.restype = ctypes.c_char_p
    lib.svdq_get_last_device_error.argtypes = [vp, ctypes.POINTER(c_int)]
    lib.svdq_last_launch_count.argtypes = []
    lib.svdq_last_cuda_error.argtypes = []
    lib.svdq_last_cuda_error.restype = ctypes.c_char_p
    lib.svdq_selftest_bounded_wait.argtypes = [i64, vp]
    for name in EXPORTED:
        if name not in ("svdq_status_string", "svdq_last_cuda_error"):
            getattr(lib, name).restype = c_int
    _lib = lib
    return lib


def status_name(status: int) -> str:
    return load().svdq_status_string(int(status)).decode()


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


# ----------------------------------------------------------------- raw entry points

def svdq_buffer_sizes(fmt, M: int, N: int, K: int, rank: int) -> svdq_sizes:
    out = svdq_sizes()
    st = load().svdq_buffer_sizes(_fmt(fmt), M, N, K, rank, ctypes.byref(out))
    if st != SVDQ_OK:
        raise SvdqError(st, "svdq_buffer_sizes")
    return out


def svdq_pack_weight(fmt, N, K, rank, act_gscale, R, L1, L2, w_codes, w_scales, w_gscale, L1_bf16, L2_bf16) -> int:
    return load().svdq_pack_weight(_fmt(fmt), N, K, rank, act_gscale, R, L1, L2, w_codes, w_scales,
                                   w_gscale, L1_bf16, L2_bf16)


def svdq_quantize_act_lowrank_down(fmt, M, K, rank, X, lam, act_gscale, L1, a_codes, a_scales, Z, stream) -> int:
    return load().svdq_quantize_act_lowrank_down(_fmt(fmt), M, K, rank, X, lam, act_gscale, L1, a_codes,
                                                 a_scales, Z, stream)


def svdq_w4a4_gemm_lowrank_up(fmt, M, N, K, rank, a_codes, a_scales, act_gscale, w_codes, w_scales, w_gscale,
                              Z, L2, bias, Y, stream) -> int:
    return load().svdq_w4a4_gemm_lowrank_up(_fmt(fmt), M, N, K, rank, a_codes, a_scales, act_gscale, w_codes,
                                            w_scales, w_gscale, Z, L2, bias, Y, stream)


def svdq_get_last_device_error(stream=None):
    site = ctypes.c_int(0)
    st = load().svdq_get_last_device_error(stream, ctypes.byref(site))
    return st, site.value


def svdq_selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    return load().svdq_selftest_bounded_wait(int(limit_ns), stream)


def svdq_last_launch_count() -> int:
    return load().svdq_last_launch_count()


def svdq_last_cuda_error() -> str:
    return load().svdq_last_cuda_error().decode()


# ----------------------------------------------------------------- torch helpers

def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(st: int, what: str):
    if st != SVDQ_OK:
        raise SvdqError(st, what)


def pack_weight_np(fmt, R_nk, L1_rk, L2_nr, act_gscale: float = 1.0):
    """Host pack from NumPy float32 arrays; returns NumPy outputs and g_w."""
    import numpy as np
    N, K = R_nk.shape
    rank = 0 if L1_rk is None else L1_rk.shape[0]
    sz = svdq_buffer_sizes(fmt, 128, N, K, rank)
    R = np.ascontiguousarray(R_nk, dtype=np.float32)
    L1 = None if rank == 0 else np.ascontiguousarray(L1_rk, dtype=np.float32)
    L2 = None if rank == 0 else np.ascontiguousarray(L2_nr, dtype=np.float32)
    w_codes = np.zeros(sz.w_codes, np.uint8)
    w_scales = np.zeros(sz.w_scales, np.uint8)
    l1b = np.zeros(max(rank * K, 1), np.uint16)
    l2b = np.zeros(max(N * rank, 1), np.uint16)
    gw = ctypes.c_float(0.0)
    st = svdq_pack_weight(fmt, N, K, rank, act_gscale, R.ctypes.data,
                          None if L1 is None else L1.ctypes.data,
                          None if L2 is None else L2.ctypes.data,
                          w_codes.ctypes.data, w_scales.ctypes.data, ctypes.byref(gw),
                          l1b.ctypes.data, l2b.ctypes.data)
    _check(st, "svdq_pack_weight")
    return {"w_codes": w_codes, "w_scales": w_scales, "w_gscale": gw.value,
            "L1_bf16": l1b[: rank * K].reshape(rank, K), "L2_bf16": l2b[: N * rank].reshape(N, rank)}


def quantize_act_lowrank_down_t(fmt, X, lam, act_gscale, L1, a_codes, a_scales, Z, stream=None):
    """Device prologue on torch tensors (X [M, K] bf16, L1 [r, K] bf16 viewed as any 2-byte dtype).
    `stream` is a raw cudaStream_t handle; None means torch's current stream."""
    M, K = X.shape
    rank = 0 if L1 is None else L1.shape[0]
    st = svdq_quantize_act_lowrank_down(fmt, M, K, rank, _ptr(X), _ptr(lam), act_gscale, _ptr(L1),
                                        _ptr(a_codes), _ptr(a_scales), _ptr(Z),
                                        _stream() if stream is None else stream)
    _check(st, "svdq_quantize_act_lowrank_down")


def w4a4_gemm_lowrank_up_t(fmt, M, N, K, rank, a_codes, a_scales, act_gscale, w_codes, w_scales, w_gscale,
                           Z, L2, bias, Y, stream=None):
    st = svdq_w4a4_gemm_lowrank_up(fmt, M, N, K, rank, _ptr(a_codes), _ptr(a_scales), act_gscale,
                                   _ptr(w_codes), _ptr(w_scales), w_gscale, _ptr(Z), _ptr(L2), _ptr(bias),
                                   _ptr(Y), _stream() if stream is None else stream)
    _check(st, "svdq_w4a4_gemm_lowrank_up")
