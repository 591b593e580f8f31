"""Python binding of libbonsai.so, the B200 weight-only low-bit linear layer.

Argument marshalling only: every operation runs in the library's CUDA
kernels (see include/bonsai.h for the operations, the packed format and the
error codes).  PyTorch supplies device memory and the current stream.  There
is no fallback: if the library is missing or the device is not sm_100, calls
raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

BINARY = 1
TERNARY = 2
TERNARY_B3 = 3  # five trits per byte in 112-byte blocks of 4 groups (include/bonsai.h)
GROUP = 128

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbonsai.so")
_lock = threading.Lock()
_lib = None

# Every function the C header declares, with its ctypes signature.
_P = ctypes.c_void_p
_I64 = ctypes.c_int64


class GemmProblem(ctypes.Structure):
    """bonsai_gemm_problem: one GEMM of a bonsai_lowbit_gemm_batch call."""
    _fields_ = [("A", _P), ("packed", _P), ("scales", _P), ("out", _P), ("M", _I64), ("N", _I64), ("K", _I64)]


SIGNATURES = {
    "bonsai_packed_bytes": (ctypes.c_size_t, [_I64, _I64, ctypes.c_int]),
    "bonsai_scale_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "bonsai_pack": (ctypes.c_int, [_P, _I64, _I64, ctypes.c_int, _P, _P]),
    "bonsai_dequant": (ctypes.c_int, [_P, _P, _I64, _I64, ctypes.c_int, _P, _P]),
    "bonsai_lowbit_gemm": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _P, _P]),
    "bonsai_hqq4_packed_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "bonsai_hqq4_pack": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
    "bonsai_hqq4_dequant": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _P, _P]),
    "bonsai_hqq4_gemm": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "bonsai_lowbit_gemm_host": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, ctypes.c_int, _P, _P, _P, _P]),
    "bonsai_lowbit_gemm_batch": (ctypes.c_int, [ctypes.POINTER(GemmProblem), ctypes.c_int, ctypes.c_int, _P]),
    "bonsai_gemm_plan": (ctypes.c_int, [_I64, _I64, _I64, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                        ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                        ctypes.POINTER(ctypes.c_int)]),
    "bonsai_get_device_error": (ctypes.c_int, []),
    "bonsai_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bonsai_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint64]),
}


class BonsaiError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m bit_weight_gemm_b200.build`")
            handle = ctypes.CDLL(_LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().bonsai_status_string(int(status)).decode()


def _mode(mode) -> int:
    if mode in (BINARY, "binary"):
        return BINARY
    if mode in (TERNARY, "ternary"):
        return TERNARY
    if mode in (TERNARY_B3, "ternary_b3"):
        return TERNARY_B3
    raise ValueError(f"unknown mode {mode!r}")


def _check(status: int, what: str):
    if status != 0:
        raise BonsaiError(what, status)


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> ctypes.c_void_p:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def words_per_row(K: int, mode) -> int:
    m = _mode(mode)
    if m == TERNARY_B3:
        return -(-(K // GROUP) // 4) * 28
    return K // (32 if m == BINARY else 16)


def packed_bytes(N: int, K: int, mode) -> int:
    return int(lib().bonsai_packed_bytes(N, K, _mode(mode)))


def scale_bytes(N: int, K: int) -> int:
    return int(lib().bonsai_scale_bytes(N, K))


def pack(codes: torch.Tensor, mode, out: torch.Tensor | None = None) -> torch.Tensor:
    """int8 codes [N,K] on the device -> packed words (int32 view) [N, words_per_row(K, mode)]."""
    N, K = codes.shape
    m = _mode(mode)
    if out is None:
        out = torch.empty((N, words_per_row(K, m)), dtype=torch.int32, device=codes.device)
    _check(lib().bonsai_pack(_dev(codes, "codes", torch.int8), N, K, m, _dev(out, "out", torch.int32), _stream()),
           "bonsai_pack")
    return out


def dequant(packed: torch.Tensor, scales: torch.Tensor, K: int, mode, out: torch.Tensor | None = None):
    """-> FP16 [N,K] with w = t*s exactly."""
    N = packed.shape[0]
    m = _mode(mode)
    if out is None:
        out = torch.empty((N, K), dtype=torch.float16, device=packed.device)
    _check(lib().bonsai_dequant(_dev(packed, "packed"), _dev(scales, "scales", torch.float16), N, K, m,
                                _dev(out, "out", torch.float16), _stream()), "bonsai_dequant")
    return out


def lowbit_gemm(A: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, mode,
                out: torch.Tensor | None = None) -> torch.Tensor:
    """out[M,N] = A[M,K] * (s*t)^T in FP16 with FP32 accumulation."""
    M, K = A.shape
    N = packed.shape[0]
    m = _mode(mode)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(lib().bonsai_lowbit_gemm(_dev(A, "A", torch.float16), _dev(packed, "packed"),
                                    _dev(scales, "scales", torch.float16), M, N, K, m,
                                    _dev(out, "out", torch.float16), _stream()), "bonsai_lowbit_gemm")
    return out


def lowbit_gemm_batch(problems, mode, outs=None) -> list:
    """Independent GEMMs in one call: problems is a sequence of (A [M,K],
    packed, scales) device tensors of one mode; returns their FP16 outputs
    [M,N] (or fills `outs`).  Problems of up to 16 tokens share persistent
    launches; larger ones are launched one by one."""
    m = _mode(mode)
    n = len(problems)
    arr = (GemmProblem * max(n, 1))()
    result = []
    for i, (A, packed, scales) in enumerate(problems):
        M, K = A.shape
        N = packed.shape[0]
        out = outs[i] if outs is not None else torch.empty((M, N), dtype=torch.float16, device=A.device)
        if tuple(out.shape) != (M, N):
            raise ValueError(f"outs[{i}] must be [{M}, {N}]")
        arr[i] = GemmProblem(_dev(A, "A", torch.float16).value, _dev(packed, "packed").value,
                             _dev(scales, "scales", torch.float16).value, _dev(out, "out", torch.float16).value,
                             M, N, K)
        result.append(out)
    _check(lib().bonsai_lowbit_gemm_batch(arr, n, m, _stream()), "bonsai_lowbit_gemm_batch")
    return result


def _host(t: torch.Tensor, name: str) -> ctypes.c_void_p:
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != torch.float16:
        raise ValueError(f"{name} must be torch.float16, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def lowbit_gemm_host(A_host: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, mode,
                     out_host: torch.Tensor | None = None, A_dev: torch.Tensor | None = None,
                     out_dev: torch.Tensor | None = None) -> torch.Tensor:
    """The GEMM with A and out in (pinned) host memory: chunked copies in,
    GEMMs and copies out overlap on the library's streams; ordered on the
    current stream and not synchronised.  A_dev / out_dev are the device work
    buffers ([M,K] and [M,N] FP16), allocated here when not given."""
    M, K = A_host.shape
    N = packed.shape[0]
    m = _mode(mode)
    dev = packed.device
    if out_host is None:
        out_host = torch.empty((M, N), dtype=torch.float16, pin_memory=True)
    if A_dev is None:
        A_dev = torch.empty((M, K), dtype=torch.float16, device=dev)
    if out_dev is None:
        out_dev = torch.empty((M, N), dtype=torch.float16, device=dev)
    if A_dev.numel() < M * K or out_dev.numel() < M * N or out_host.numel() < M * N:
        raise ValueError("work or output buffer too small")
    _check(lib().bonsai_lowbit_gemm_host(_host(A_host, "A_host"), _dev(packed, "packed"),
                                         _dev(scales, "scales", torch.float16), M, N, K, m,
                                         _host(out_host, "out_host"), _dev(A_dev, "A_dev", torch.float16),
                                         _dev(out_dev, "out_dev", torch.float16), _stream()),
           "bonsai_lowbit_gemm_host")
    return out_host


# ------------------------------------------- 4-bit group-affine weights --
HQQ4 = 4  # mode value for gemm_plan
HQQ_GROUP = 64


def hqq4_pack(q: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """uint8 q [N,K] (0..15) on the device -> packed words (int32 view) [N, K/8]."""
    N, K = q.shape
    if out is None:
        out = torch.empty((N, K // 8), dtype=torch.int32, device=q.device)
    _check(lib().bonsai_hqq4_pack(_dev(q, "q", torch.uint8), N, K, _dev(out, "out", torch.int32), _stream()),
           "bonsai_hqq4_pack")
    return out


def hqq4_dequant(packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, K: int,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """-> FP16 [N,K] with w = fp16(fp16(q - z) * s), groups of 64 along K."""
    N = packed.shape[0]
    if out is None:
        out = torch.empty((N, K), dtype=torch.float16, device=packed.device)
    _check(lib().bonsai_hqq4_dequant(_dev(packed, "packed"), _dev(scales, "scales", torch.float16),
                                     _dev(zeros, "zeros", torch.float16), N, K, _dev(out, "out", torch.float16),
                                     _stream()), "bonsai_hqq4_dequant")
    return out


def hqq4_gemm(A: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
              out: torch.Tensor | None = None) -> torch.Tensor:
    """out[M,N] = A[M,K] * W^T with 4-bit group-affine weights."""
    M, K = A.shape
    N = packed.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=A.device)
    _check(lib().bonsai_hqq4_gemm(_dev(A, "A", torch.float16), _dev(packed, "packed"),
                                  _dev(scales, "scales", torch.float16), _dev(zeros, "zeros", torch.float16),
                                  M, N, K, _dev(out, "out", torch.float16), _stream()), "bonsai_hqq4_gemm")
    return out


def gemm_plan(M: int, N: int, K: int, mode) -> dict:
    """The launch bonsai_lowbit_gemm makes: tokens per tile, K split, CTAs,
    output tiles (fewer CTAs than tiles x split: the persistent form)."""
    bt, ks, ctas, tiles = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    m = HQQ4 if mode in (HQQ4, "hqq4") else _mode(mode)
    _check(lib().bonsai_gemm_plan(M, N, K, m, ctypes.byref(bt), ctypes.byref(ks), ctypes.byref(ctas),
                                  ctypes.byref(tiles)), "bonsai_gemm_plan")
    return {"block_t": bt.value, "ksplit": ks.value, "ctas": ctas.value, "tiles": tiles.value}


def get_device_error() -> int:
    return int(lib().bonsai_get_device_error())


def selftest_wait_timeout(limit_ns: int) -> int:
    return int(lib().bonsai_selftest_wait_timeout(int(limit_ns)))
