"""ctypes front end for the VBQ oracle (``vbq_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
use this module. The product package never imports it, and it never imports the product package.

The oracle is a plain fp64 CPU implementation of the VBQ dequantize-and-multiply path. It follows the VBQ paper
("Variable Bit-width Quantization", section 3.1: 64-weight groups with a per-group scale and a width from
{1,2,4,8}; section 6, "Fused kernels over packed weights": dequantize per group, then accumulate W x) and
FORMAT.md for the byte layout.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vbq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libvbq_oracle.so")

OK = 0
ERR_NULL, ERR_SHAPE, ERR_WIDTH, ERR_CODE_RANGE, ERR_BUFFER_TOO_SMALL = -1, -2, -3, -4, -5
ERR_BAD_MAGIC, ERR_VERSION, ERR_CRC, ERR_BATCH, ERR_ALIGN, ERR_CUDA = -6, -7, -8, -9, -10, -11
ERR_TILE, ERR_FORMAT = -12, -13


class OracleError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed with status {status}")
        self.status = status


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP) into oracle/_build. Returns the library path."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        os.makedirs(_BUILD, exist_ok=True)
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, u64, vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p
        L.vbqo_crc32.restype = ctypes.c_uint32
        L.vbqo_crc32.argtypes = [vp, u64]
        L.vbqo_half_to_double.restype = ctypes.c_double
        L.vbqo_half_to_double.argtypes = [ctypes.c_uint16]
        L.vbqo_bf16_to_double.restype = ctypes.c_double
        L.vbqo_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.vbqo_packed_size.argtypes = [i64, i64, i64, vp, ctypes.POINTER(u64)]
        L.vbqo_pack.argtypes = [i64, i64, i64, vp, vp, vp, vp, u64, ctypes.POINTER(u64)]
        L.vbqo_read_header.argtypes = [vp, u64, ctypes.POINTER(i64), ctypes.POINTER(i64),
                                       ctypes.POINTER(i64), ctypes.POINTER(u64)]
        L.vbqo_unpack.argtypes = [vp, u64, vp, vp, vp]
        L.vbqo_matvec.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, ctypes.c_int]
        L.vbqo_dequant.argtypes = [i64, i64, vp, vp, vp, vp]
        for f in ("vbqo_packed_size", "vbqo_pack", "vbqo_read_header", "vbqo_unpack", "vbqo_matvec",
                  "vbqo_dequant"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def crc32(data: bytes | np.ndarray) -> int:
    buf = np.frombuffer(bytes(data), dtype=np.uint8) if not isinstance(data, np.ndarray) else _c(data, np.uint8)
    return int(lib().vbqo_crc32(_p(buf), buf.size))


def half_to_double(bits: int) -> float:
    return float(lib().vbqo_half_to_double(bits))


def bf16_to_double(bits: int) -> float:
    return float(lib().vbqo_bf16_to_double(bits))


def packed_size(N: int, K: int, R: int, widths: np.ndarray) -> int:
    w = _c(widths, np.uint8)
    out = ctypes.c_uint64()
    st = lib().vbqo_packed_size(N, K, R, _p(w), ctypes.byref(out))
    if st:
        raise OracleError(st, "packed_size")
    return int(out.value)


def pack_status(N: int, K: int, R: int, widths, scales, codes, cap: int | None = None):
    """Returns (status, blob or None)."""
    w, s, c = _c(widths, np.uint8), _c(scales, np.uint16), _c(codes, np.uint8)
    if cap is None:
        try:
            cap = packed_size(N, K, R, w)
        except OracleError as e:
            return e.status, None
    out = np.zeros(max(cap, 1), dtype=np.uint8)
    n = ctypes.c_uint64()
    st = lib().vbqo_pack(N, K, R, _p(w), _p(s), _p(c), _p(out), cap, ctypes.byref(n))
    return st, (out[: n.value] if st == OK else None)


def pack(N: int, K: int, R: int, widths, scales, codes) -> np.ndarray:
    st, blob = pack_status(N, K, R, widths, scales, codes)
    if st:
        raise OracleError(st, "pack")
    return blob


def read_header(blob: np.ndarray):
    b = _c(blob, np.uint8)
    N, K, R, tot = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64(), ctypes.c_uint64()
    st = lib().vbqo_read_header(_p(b), b.size, ctypes.byref(N), ctypes.byref(K), ctypes.byref(R),
                                ctypes.byref(tot))
    return st, (N.value, K.value, R.value, tot.value)


def unpack_status(blob: np.ndarray):
    b = _c(blob, np.uint8)
    st, (N, K, R, _) = read_header(b)
    if st:
        return st, None
    G = K // 64
    widths = np.zeros((N, G), np.uint8)
    scales = np.zeros((N, G), np.uint16)
    codes = np.zeros((N, K), np.uint8)
    st = lib().vbqo_unpack(_p(b), b.size, _p(widths), _p(scales), _p(codes))
    return st, ((widths, scales, codes, R) if st == OK else None)


def unpack(blob: np.ndarray):
    """Returns (widths[N,G], scales[N,G] fp16 bits, codes[N,K], R)."""
    st, out = unpack_status(blob)
    if st:
        raise OracleError(st, "unpack")
    return out


def matvec(widths, scales, codes, x_bf16, nthreads: int | None = None):
    """fp64 y[B,N] and bound A[B,N] = sum |w||x| for x_bf16[B,K] (bf16 bit patterns, uint16)."""
    w, s, c = _c(widths, np.uint8), _c(scales, np.uint16), _c(codes, np.uint8)
    x = _c(x_bf16, np.uint16)
    if x.ndim == 1:
        x = x[None, :]
    N, K = c.shape
    B = x.shape[0]
    y = np.zeros((B, N), np.float64)
    a = np.zeros((B, N), np.float64)
    st = lib().vbqo_matvec(N, K, B, _p(w), _p(s), _p(c), _p(x), _p(y), _p(a), int(nthreads or 1))
    if st:
        raise OracleError(st, "matvec")
    return y, a


def dequant(widths, scales, codes) -> np.ndarray:
    w, s, c = _c(widths, np.uint8), _c(scales, np.uint16), _c(codes, np.uint8)
    N, K = c.shape
    out = np.zeros((N, K), np.float64)
    st = lib().vbqo_dequant(N, K, _p(w), _p(s), _p(c), _p(out))
    if st:
        raise OracleError(st, "dequant")
    return out


def within_tolerance(y_test: np.ndarray, y_ref: np.ndarray, bound: np.ndarray) -> np.ndarray:
    """Per-element parity bar of this project: |y - y_ref| <= 1e-3 * sum|w||x| + 1e-6."""
    return np.abs(np.asarray(y_test, np.float64) - y_ref) <= 1e-3 * bound + 1e-6


def silu(g) -> np.ndarray:
    """SiLU (swish) in fp64: g * logistic(g) = g / (1 + e^-g). The gate nonlinearity of the SwiGLU MLP that the
    VBQ paper's decoders use (section 4); plain definition, written as g * e^g / (1 + e^g) for negative g so that
    e^-g cannot overflow."""
    g = np.asarray(g, np.float64)
    e = np.exp(-np.abs(g))
    return np.where(g >= 0, g / (1.0 + e), g * e / (1.0 + e))


def swiglu(y_gate, y_up) -> np.ndarray:
    """h = silu(gate) * up, elementwise, fp64."""
    return silu(y_gate) * np.asarray(y_up, np.float64)


def swiglu_bound(y_gate, y_up, bound_gate, bound_up) -> np.ndarray:
    """Per-element bar for h computed from fp32 outputs that meet `within_tolerance` and rounded to bf16:
    2^-8 |h| (bf16 rounding, with margin) + 1.1 |u| tol_g + |silu(g)| tol_u + tol_g tol_u + 1e-6, where
    tol = 1e-3 * sum|w||x| + 1e-6 and 1.1 bounds |silu'|."""
    g, u = np.asarray(y_gate, np.float64), np.asarray(y_up, np.float64)
    tg, tu = 1e-3 * np.asarray(bound_gate) + 1e-6, 1e-3 * np.asarray(bound_up) + 1e-6
    h = swiglu(g, u)
    return 2.0 ** -8 * np.abs(h) + 1.1 * np.abs(u) * tg + np.abs(silu(g)) * tu + tg * tu + 1e-6
