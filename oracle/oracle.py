"""ctypes front end for the VBQ oracle (``vbq_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
use this module. The product package never imports it, and it never imports the product package.

The oracle is a plain fp64 CPU implementation of the VBQ dequantize-and-multiply path. It follows the VBQ paper
("Variable Bit-width Quantization", section 3.1: 64-weight groups with a per-group scale and a width from
{1,2,4,8}; section 6, "Fused kernels over packed weights": dequantize per group, then accumulate W x) and
packed format v1 for the byte layout (row tiles, one record per tile and group column, width buckets
inside each record).

Pins (tests/test_oracle_pins.py), besides those of the C part:
- silu: textbook values of the logistic function at 0 and +-1, large-argument limits, and the identity
  silu(g) - silu(-g) = g;
- swiglu_bound: admits the bf16 rounding of an exact h; its propagation term covers every admissible
  perturbation of (g, u) on a grid that reaches |g| = 30 and the peak of silu' (where 1.1 > sup|silu'| is checked
  against the textbook derivative and finite differences);
- quantize: weights that lie exactly on either grid come back as that scale and those codes; 1-bit groups give
  sign times the mean magnitude; every dequantized weight lies within half a step of its input (plus the
  scale's fp16 rounding); all-zero groups decode to zero; non-finite weights and scales beyond fp16 are
  refused.
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
ERR_TILE, ERR_FORMAT, ERR_FLAGS, ERR_VALUE = -12, -13, -16, -17
FLAG_GRID_SYMMETRIC = 1   # header flag bit 0: widths >= 2 on the paper's Eq. 1 integer grid


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
        L.vbqo_pack_ex.argtypes = [i64, i64, i64, vp, vp, vp, ctypes.c_uint, vp, u64, ctypes.POINTER(u64)]
        L.vbqo_read_header_ex.argtypes = [vp, u64, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i64),
                                          ctypes.POINTER(u64), ctypes.POINTER(ctypes.c_uint)]
        L.vbqo_matvec_ex.argtypes = [i64, i64, i64, vp, vp, vp, vp, ctypes.c_uint, vp, vp, ctypes.c_int]
        L.vbqo_dequant_ex.argtypes = [i64, i64, vp, vp, vp, ctypes.c_uint, vp]
        L.vbqo_read_header.argtypes = [vp, u64, ctypes.POINTER(i64), ctypes.POINTER(i64),
                                       ctypes.POINTER(i64), ctypes.POINTER(u64)]
        L.vbqo_unpack.argtypes = [vp, u64, vp, vp, vp]
        L.vbqo_matvec.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, ctypes.c_int]
        L.vbqo_dequant.argtypes = [i64, i64, vp, vp, vp, vp]
        for f in ("vbqo_packed_size", "vbqo_pack", "vbqo_read_header", "vbqo_unpack", "vbqo_matvec",
                  "vbqo_dequant", "vbqo_pack_ex", "vbqo_read_header_ex", "vbqo_matvec_ex", "vbqo_dequant_ex"):
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


def pack_status(N: int, K: int, R: int, widths, scales, codes, cap: int | None = None, flags: int = 0):
    """Returns (status, blob or None). flags: header flags (FLAG_GRID_SYMMETRIC selects Eq. 1's grid)."""
    w, s, c = _c(widths, np.uint8), _c(scales, np.uint16), _c(codes, np.uint8)
    if cap is None:
        try:
            cap = packed_size(N, K, R, w)
        except OracleError as e:
            return e.status, None
    out = np.zeros(max(cap, 1), dtype=np.uint8)
    n = ctypes.c_uint64()
    st = lib().vbqo_pack_ex(N, K, R, _p(w), _p(s), _p(c), flags, _p(out), cap, ctypes.byref(n))
    return st, (out[: n.value] if st == OK else None)


def pack(N: int, K: int, R: int, widths, scales, codes, flags: int = 0) -> np.ndarray:
    st, blob = pack_status(N, K, R, widths, scales, codes, flags=flags)
    if st:
        raise OracleError(st, "pack")
    return blob


def read_header(blob: np.ndarray):
    b = _c(blob, np.uint8)
    N, K, R, tot = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64(), ctypes.c_uint64()
    st = lib().vbqo_read_header(_p(b), b.size, ctypes.byref(N), ctypes.byref(K), ctypes.byref(R),
                                ctypes.byref(tot))
    return st, (N.value, K.value, R.value, tot.value)


def header_flags(blob: np.ndarray) -> int:
    b = _c(blob, np.uint8)
    f = ctypes.c_uint()
    st = lib().vbqo_read_header_ex(_p(b), b.size, None, None, None, None, ctypes.byref(f))
    if st:
        raise OracleError(st, "read_header")
    return int(f.value)


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


def matvec(widths, scales, codes, x_bf16, nthreads: int | None = None, flags: int = 0):
    """fp64 y[B,N] and bound A[B,N] = sum |w||x| for x_bf16[B,K] (bf16 bit patterns, uint16); flags selects the
    value grid as in the blob header."""
    w, s, c = _c(widths, np.uint8), _c(scales, np.uint16), _c(codes, np.uint8)
    x = _c(x_bf16, np.uint16)
    if x.ndim == 1:
        x = x[None, :]
    N, K = c.shape
    B = x.shape[0]
    y = np.zeros((B, N), np.float64)
    a = np.zeros((B, N), np.float64)
    st = lib().vbqo_matvec_ex(N, K, B, _p(w), _p(s), _p(c), _p(x), flags, _p(y), _p(a), int(nthreads or 1))
    if st:
        raise OracleError(st, "matvec")
    return y, a


def dequant(widths, scales, codes, flags: int = 0) -> np.ndarray:
    w, s, c = _c(widths, np.uint8), _c(scales, np.uint16), _c(codes, np.uint8)
    N, K = c.shape
    out = np.zeros((N, K), np.float64)
    st = lib().vbqo_dequant_ex(N, K, _p(w), _p(s), _p(c), flags, _p(out))
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
    """Per-element bar for h computed from fp32 outputs g', u' that meet `within_tolerance` (|g' - g| <= tol_g,
    |u' - u| <= tol_u with tol = 1e-3 * sum|w||x| + 1e-6) and rounded once to bf16:

        P   = 1.1 tol_g (|u| + tol_u) + |silu(g)| tol_u
        bar = P + 2^-8 (|h| + P) + 1e-6,  h = silu(g) u.

    P is the propagation term: silu(g') u' - silu(g) u = (silu(g') - silu(g)) u' + silu(g) (u' - u), and by the
    mean value theorem |silu(g') - silu(g)| <= sup|silu'| tol_g with sup|silu'| = 1.0998... < 1.1 (at g = 2.40),
    while |u'| <= |u| + tol_u. The computed h' lies within P of h; rounding it to bf16 moves it by at most
    2^-9 |h'| <= 2^-9 (|h| + P), and 2^-8 leaves the other half for the fp32 evaluation of silu(g') u'."""
    g, u = np.asarray(y_gate, np.float64), np.asarray(y_up, np.float64)
    tg, tu = 1e-3 * np.asarray(bound_gate) + 1e-6, 1e-3 * np.asarray(bound_up) + 1e-6
    h = swiglu(g, u)
    prop = 1.1 * tg * (np.abs(u) + tu) + np.abs(silu(g)) * tu
    return prop + 2.0 ** -8 * (np.abs(h) + prop) + 1e-6


def fp16_bits(v) -> np.ndarray:
    """fp16 bit patterns of fp64 values, round to nearest even (numpy's float64 -> float16 conversion)."""
    with np.errstate(over="ignore"):   # values beyond fp16 become inf, which the callers check for
        return np.asarray(v, np.float64).astype(np.float16).view(np.uint16)


def round_half_away(v) -> np.ndarray:
    """Nearest integer, ties away from zero (C's round()), exactly: integer part plus one step when the
    fraction is at least one half."""
    v = np.asarray(v, np.float64)
    t = np.trunc(v)
    return t + np.where(np.abs(v - t) >= 0.5, np.sign(v), 0.0)


def quantize(w, widths, flags: int = 0):
    """Quantize float32 weights w[N,K] to per-group codes for the given widths[N,G] (VBQ paper, section 3.1).

    Per group of 64 weights (values in fp64):
    - width 1: the scale is s = 2 * mean|w| (so that the two grid points +-s/2 are +-mean|w|: sign times the
      mean magnitude), with the mean taken as the sum of |w| in index order divided by 64; code = 1 where w >= 0.
    - width k >= 2, Eq. 1's symmetric grid (flags & FLAG_GRID_SYMMETRIC): L = 2^(k-1) - 1, s = max|w| / L,
      q = clip(round(w / s), -L, L), code = q + L.
    - width k >= 2, the default grid: c = (2^k - 1) / 2, s = max|w| / c, code = clip(round(w / s + c), 0,
      2^k - 1).
    The scale is rounded to fp16 (nearest even) first and the codes use that rounded scale; round() is to
    nearest with ties away from zero. A group whose scale is 0 gets code L (symmetric) or 2^(k-1) (default),
    i.e. the grid point nearest 0. Returns (status, scales[N,G] fp16 bits, codes[N,K]); status ERR_VALUE for a
    non-finite weight or a scale that does not fit in fp16.
    """
    w = np.asarray(w, np.float32).astype(np.float64)
    widths = np.asarray(widths, np.uint8)
    N, K = w.shape
    G = K // 64
    if not np.all(np.isfinite(w)):
        return ERR_VALUE, None, None
    wg = w.reshape(N, G, 64)
    a = np.abs(wg)
    k = widths.astype(np.int64)
    sym = bool(flags & FLAG_GRID_SYMMETRIC)
    seq_sum = np.add.accumulate(a, axis=2)[:, :, -1]          # index-order sum of |w| over the group
    amax = a.max(axis=2)
    L = np.where(sym, (1 << (k - 1)) - 1, 0).astype(np.float64)
    c = ((1 << k) - 1).astype(np.float64) / 2.0
    ratio = np.where(k == 1, seq_sum / 32.0, np.where(sym, amax / np.maximum(L, 1.0), amax / c))
    s16 = fp16_bits(ratio)
    sd = s16.astype(np.uint16).view(np.float16).astype(np.float64)
    if not np.all(np.isfinite(sd)):
        return ERR_VALUE, None, None
    sdx = sd[:, :, None]
    kx, Lx, cx = k[:, :, None], L[:, :, None], c[:, :, None]
    safe = np.where(sdx > 0, sdx, 1.0)
    q1 = (wg >= 0).astype(np.float64)
    qs = np.clip(round_half_away(wg / safe), -Lx, Lx) + Lx
    qh = np.clip(round_half_away(wg / safe + cx), 0.0, (1 << kx) - 1.0)
    zero_code = np.where(sym, Lx, (1 << (kx - 1)).astype(np.float64))
    q = np.where(kx == 1, q1, np.where(sdx > 0, np.where(sym, qs, qh), zero_code))
    return OK, s16.reshape(N, G), q.astype(np.uint8).reshape(N, K)
