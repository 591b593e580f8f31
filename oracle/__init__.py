"""CPU oracle for the weight-only low-bit linear layer.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` import this package.  It shares
no code with ``bit_weight_gemm_b200`` and imports nothing from it.

The arithmetic lives in ``bonsai_oracle.c`` (plain C, doubles, one sequential
sum per output); this module only compiles it with gcc and marshals numpy
arrays through ctypes.  What it computes is stated, with its sources, in the
header of that file: w = scale_g * t, one FP16 scale per 128 consecutive
weights along K ("Cómo Bonsai Ternary 4B revoluciona la difusión
texto-imagen", section "Representación y almacenamiento de los pesos
ternarios"), out = A * W^T accumulated in double and rounded once to FP16.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

BINARY = 1
TERNARY = 2
TERNARY_B3 = 3  # five trits per byte, this project's denser format (see bonsai_oracle.c)
GROUP = 128

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bonsai_oracle.c")
_LIB = os.path.join(_HERE, "libbonsai_oracle.so")
_lock = threading.Lock()
_lib = None

_ERRORS = {1: "invalid argument", 2: "invalid shape", 4: "invalid code", 5: "out of memory"}


class OracleError(RuntimeError):
    pass


def build_oracle(force: bool = False) -> str:
    """Compile bonsai_oracle.c into libbonsai_oracle.so next to it."""
    stale = not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # A test may point the wrapper at another build of the oracle
            # (a copy with a planted mistake) to show that the pins catch it.
            path = os.environ.get("BONSAI_ORACLE_LIB") or build_oracle()
            lib = ctypes.CDLL(path)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.oracle_half_to_double.restype = ctypes.c_double
            lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_double_to_half.restype = ctypes.c_uint16
            lib.oracle_double_to_half.argtypes = [ctypes.c_double]
            lib.oracle_half_to_double_array.argtypes = [P, I64, P]
            lib.oracle_half_to_double_array.restype = None
            lib.oracle_double_to_half_array.argtypes = [P, I64, P]
            lib.oracle_double_to_half_array.restype = None
            lib.oracle_packed_bytes.argtypes = [I64, I64, ctypes.c_int]
            lib.oracle_packed_bytes.restype = I64
            lib.oracle_pack.argtypes = [P, I64, I64, ctypes.c_int, P]
            lib.oracle_pack.restype = ctypes.c_int
            lib.oracle_unpack.argtypes = [P, I64, I64, ctypes.c_int, P]
            lib.oracle_unpack.restype = ctypes.c_int
            lib.oracle_dequant.argtypes = [P, P, I64, I64, ctypes.c_int, P]
            lib.oracle_dequant.restype = ctypes.c_int
            lib.oracle_gemm.argtypes = [P, P, P, I64, I64, I64, ctypes.c_int, P, P, P, ctypes.c_int]
            lib.oracle_gemm.restype = ctypes.c_int
            lib.oracle_gemm_entries.argtypes = [P, P, P, I64, I64, I64, ctypes.c_int, P, P, I64, P, P, P]
            lib.oracle_gemm_entries.restype = ctypes.c_int
            lib.oracle_gemm_w16.argtypes = [P, P, I64, I64, I64, P, P, P, ctypes.c_int]
            lib.oracle_gemm_w16.restype = ctypes.c_int
            lib.oracle_hqq4_pack.argtypes = [P, I64, I64, P]
            lib.oracle_hqq4_pack.restype = ctypes.c_int
            lib.oracle_hqq4_unpack.argtypes = [P, I64, I64, P]
            lib.oracle_hqq4_unpack.restype = ctypes.c_int
            lib.oracle_hqq4_dequant.argtypes = [P, P, P, I64, I64, P]
            lib.oracle_hqq4_dequant.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: {_ERRORS.get(rc, rc)}")


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _mode(mode) -> int:
    if mode in (BINARY, "binary"):
        return BINARY
    if mode in (TERNARY, "ternary"):
        return TERNARY
    if mode in (TERNARY_B3, "ternary_b3"):
        return TERNARY_B3
    raise ValueError(f"unknown mode {mode!r}")


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------------ FP16 --
def half_bits_to_double(bits) -> np.ndarray:
    """binary16 bit patterns (uint16) -> exact float64 values."""
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    _load().oracle_half_to_double_array(_ptr(b), b.size, _ptr(out))
    return out


def double_to_half_bits(x) -> np.ndarray:
    """float64 -> binary16 bit patterns, round to nearest, ties to even."""
    d = _c(x, np.float64)
    out = np.empty(d.shape, np.uint16)
    _load().oracle_double_to_half_array(_ptr(d), d.size, _ptr(out))
    return out


# ---------------------------------------------------------------- format --
def packed_bytes(N: int, K: int, mode) -> int:
    return int(_load().oracle_packed_bytes(N, K, _mode(mode)))


def words_per_row(K: int, mode) -> int:
    m = _mode(mode)
    if m == TERNARY_B3:
        return -(-(K // GROUP) // 4) * 28  # one 112-byte block (28 words) per 4 groups
    return K // (32 if m == BINARY else 16)


def pack(codes, mode) -> np.ndarray:
    """int8 codes [N,K] -> uint32 packed words [N, K/32] (binary), [N, K/16]
    (INT2 ternary) or [N, 28 * ceil(K/512)] (base-3: 112-byte blocks of 4 groups)."""
    c = _c(codes, np.int8)
    N, K = c.shape
    out = np.zeros((N, words_per_row(K, mode)), np.uint32)
    _check(_load().oracle_pack(_ptr(c), N, K, _mode(mode), _ptr(out)), "oracle_pack")
    return out


def unpack(packed, K: int, mode) -> np.ndarray:
    p = _c(packed, np.uint32)
    N = p.shape[0]
    out = np.zeros((N, K), np.int8)
    _check(_load().oracle_unpack(_ptr(p), N, K, _mode(mode), _ptr(out)), "oracle_unpack")
    return out


def dequant(packed, scales, K: int, mode) -> np.ndarray:
    """-> fp16 bit patterns (uint16) of w = t*s, [N,K]."""
    p = _c(packed, np.uint32)
    s = _c(scales, np.uint16)
    N = p.shape[0]
    out = np.zeros((N, K), np.uint16)
    _check(_load().oracle_dequant(_ptr(p), _ptr(s), N, K, _mode(mode), _ptr(out)), "oracle_dequant")
    return out


# ------------------------------------------------------------------ GEMM --
def gemm(A_bits, packed, scales, K: int, mode, threads: int | None = None, want_acc: bool = True):
    """out = A * W^T.  A_bits: fp16 bit patterns [M,K].

    Returns (out_bits uint16 [M,N], acc float64 [M,N] or None, absacc or None)
    where acc is the double sum before rounding and absacc = sum |a*w|.
    """
    a = _c(A_bits, np.uint16)
    p = _c(packed, np.uint32)
    s = _c(scales, np.uint16)
    M = a.shape[0]
    N = p.shape[0]
    assert a.shape[1] == K
    out = np.zeros((M, N), np.uint16)
    acc = np.zeros((M, N), np.float64) if want_acc else None
    absacc = np.zeros((M, N), np.float64) if want_acc else None
    rc = _load().oracle_gemm(_ptr(a), _ptr(p), _ptr(s), M, N, K, _mode(mode), _ptr(out), _ptr(acc),
                             _ptr(absacc), threads or default_threads())
    _check(rc, "oracle_gemm")
    return out, acc, absacc


def gemm_entries(A_bits, packed, scales, K: int, mode, ms, ns):
    """The oracle's outputs at positions (ms[i], ns[i]), each computed alone."""
    a = _c(A_bits, np.uint16)
    p = _c(packed, np.uint32)
    s = _c(scales, np.uint16)
    ms = _c(ms, np.int64)
    ns = _c(ns, np.int64)
    M = a.shape[0]
    N = p.shape[0]
    out = np.zeros(ms.shape, np.uint16)
    acc = np.zeros(ms.shape, np.float64)
    absacc = np.zeros(ms.shape, np.float64)
    rc = _load().oracle_gemm_entries(_ptr(a), _ptr(p), _ptr(s), M, N, K, _mode(mode), _ptr(ms), _ptr(ns),
                                     ms.size, _ptr(out), _ptr(acc), _ptr(absacc))
    _check(rc, "oracle_gemm_entries")
    return out, acc, absacc


def gemm_w16(A_bits, w_bits, threads: int | None = None):
    """out = A * W^T for FP16 weights given as bit patterns [N,K]; returns
    (out_bits, acc, absacc) like gemm()."""
    a = _c(A_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    M, K = a.shape
    N = w.shape[0]
    assert w.shape[1] == K
    out = np.zeros((M, N), np.uint16)
    acc = np.zeros((M, N), np.float64)
    absacc = np.zeros((M, N), np.float64)
    rc = _load().oracle_gemm_w16(_ptr(a), _ptr(w), M, N, K, _ptr(out), _ptr(acc), _ptr(absacc),
                                 threads or default_threads())
    _check(rc, "oracle_gemm_w16")
    return out, acc, absacc


# ------------------------------------------- 4-bit group-affine weights --
HQQ_GROUP = 64


def hqq4_pack(q) -> np.ndarray:
    """uint8 q [N,K] in 0..15 -> uint32 words [N, K/8] (bonsai_oracle.c)."""
    c = _c(q, np.uint8)
    N, K = c.shape
    out = np.zeros((N, K // 8), np.uint32)
    _check(_load().oracle_hqq4_pack(_ptr(c), N, K, _ptr(out)), "oracle_hqq4_pack")
    return out


def hqq4_unpack(packed, K: int) -> np.ndarray:
    p = _c(packed, np.uint32)
    out = np.zeros((p.shape[0], K), np.uint8)
    _check(_load().oracle_hqq4_unpack(_ptr(p), p.shape[0], K, _ptr(out)), "oracle_hqq4_unpack")
    return out


def hqq4_dequant(packed, scales, zeros, K: int) -> np.ndarray:
    """-> fp16 bits of w = fp16(fp16(q - z) * s), groups of 64 along K."""
    p = _c(packed, np.uint32)
    s = _c(scales, np.uint16)
    z = _c(zeros, np.uint16)
    N = p.shape[0]
    out = np.zeros((N, K), np.uint16)
    _check(_load().oracle_hqq4_dequant(_ptr(p), _ptr(s), _ptr(z), N, K, _ptr(out)), "oracle_hqq4_dequant")
    return out


def hqq4_gemm(A_bits, packed, scales, zeros, K: int, threads: int | None = None):
    """out = A * W^T for 4-bit group-affine weights: the dequantised FP16
    weights, then one double sum per output."""
    return gemm_w16(A_bits, hqq4_dequant(packed, scales, zeros, K), threads)


def ulp16(ref_bits) -> np.ndarray:
    """One FP16 unit in the last place at each value: 2^(e-10) for |x| in
    [2^e, 2^(e+1)), e >= -14, and 2^-24 below 2^-14 (the subnormal spacing)."""
    x = np.abs(half_bits_to_double(ref_bits))
    out = np.full(x.shape, 2.0 ** -24)
    big = np.isfinite(x) & (x >= 2.0 ** -14)
    e = np.floor(np.log2(np.where(big, x, 1.0)))
    out[big] = np.exp2(e[big] - 10)
    return out


def within_tolerance(gpu_bits, ref_bits, absacc, rel: float = 1e-3) -> np.ndarray:
    """Element-wise GEMM acceptance: |gpu - ref| <= rel * sum|a*w| + ulp16(ref);
    an infinite or NaN reference must be matched exactly in kind."""
    g = half_bits_to_double(gpu_bits)
    r = half_bits_to_double(ref_bits)
    with np.errstate(invalid="ignore"):
        ok = np.abs(g - r) <= rel * np.asarray(absacc) + ulp16(ref_bits)
    inf = np.isinf(r)
    ok = np.where(inf, g == r, ok)
    nan = np.isnan(r)
    ok = np.where(nan, np.isnan(g), ok)
    return ok
