"""Pins for the CPU oracle: each test checks the oracle against something other than itself.

- float decoders: numpy's binary16 and torch's bfloat16 conversions, over all 65536 bit patterns;
- CRC-32: the published check value and zlib;
- packing: hand-derived golden blobs of the packed format's worked example (default grid, and Eq. 1's
  symmetric grid flag with a top code), and a single-code bit-position sweep;
- matvec: exact rational arithmetic on tiny shapes, closed forms on uniform widths, one-hot columns, exact
  power-of-two scale invariance, and numpy's BLAS on weights rebuilt from the definition.

The method follows the VBQ paper ("Variable Bit-width Quantization", section 3.1, groups of 64 with a per-group
scale and width from {1,2,4,8}; section 6, "Fused kernels over packed weights").
"""
import math
import os
import zlib
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O
import vbq_synth as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "format_n2_k64_r16.txt")


def f16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def bf16(bits):
    t = torch.from_numpy(np.asarray(bits, np.uint16).astype(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


# ------------------------------------------------------------------------------------------------ decoders
def test_half_decoder_matches_numpy_all_patterns():
    ref = f16(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    got = np.array([O.half_to_double(b) for b in range(65536)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_decoder_matches_torch_all_patterns():
    ref = bf16(np.arange(65536, dtype=np.uint32).astype(np.uint16))
    got = np.array([O.bf16_to_double(b) for b in range(65536)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_crc32_check_value_and_zlib():
    assert O.crc32(b"123456789") == 0xCBF43926
    g = np.random.default_rng(1)
    for n in (0, 1, 7, 64, 1000):
        buf = g.integers(0, 256, n, dtype=np.uint8).tobytes()
        assert O.crc32(buf) == zlib.crc32(buf)


# ------------------------------------------------------------------------------------------------ packing
def golden_example():
    N, K, R = 2, 64, 16
    widths = np.array([[1], [2]], np.uint8)
    scales = np.array([[0x3C00], [0x3800]], np.uint16)
    codes = np.zeros((2, 64), np.uint8)
    codes[0] = np.arange(64) % 2
    codes[1] = np.arange(64) % 4
    return N, K, R, widths, scales, codes


def parse_golden(path):
    expect, crc_fields = {}, {}
    for line in open(path):
        line = line.split("#", 1)[0].strip() if line.lstrip().startswith("#") else line.strip()
        if not line:
            continue
        parts = line.split()
        off = int(parts[0])
        if parts[1].startswith("CRC32_"):
            crc_fields[parts[1]] = off
            continue
        for i, tok in enumerate(parts[1:]):
            try:
                b = int(tok, 16)
            except ValueError:
                break
            if len(tok) != 2:
                break
            expect[off + i] = b
    return expect, crc_fields


def test_golden_blob_bytes():
    N, K, R, w, s, c = golden_example()
    blob = O.pack(N, K, R, w, s, c).tobytes()
    expect, crc = parse_golden(GOLDEN)
    assert len(blob) == 144
    covered = set(expect) | {o + i for o in crc.values() for i in range(4)}
    assert covered == set(range(144)), "golden file must describe every byte"
    for off, b in expect.items():
        assert blob[off] == b, f"byte {off}: got {blob[off]:#04x} want {b:#04x}"
    assert int.from_bytes(blob[crc["CRC32_BODY"]:][:4], "little") == zlib.crc32(blob[64:144])
    assert int.from_bytes(blob[crc["CRC32_HEADER"]:][:4], "little") == zlib.crc32(blob[0:60])


GOLDEN_SYM = os.path.join(os.path.dirname(__file__), "golden", "format_n2_k64_r16_sym.txt")


def test_golden_blob_symmetric_grid_flag():
    """The worked example with header flag bit 0 (Eq. 1's grid) and a top-code (2 = 2^2 - 2) 2-bit row: every byte
    as derived by hand, the round trip, and the dequantized rows on one-hot activations."""
    N, K, R = 2, 64, 16
    w = np.array([[1], [2]], np.uint8)
    s = np.array([[0x3C00], [0x3800]], np.uint16)
    c = np.zeros((2, 64), np.uint8)
    c[0] = np.arange(64) % 2
    c[1] = np.arange(64) % 3
    blob = O.pack(N, K, R, w, s, c, flags=O.FLAG_GRID_SYMMETRIC)
    expect, crc = parse_golden(GOLDEN_SYM)
    b = blob.tobytes()
    assert len(b) == 144 and set(expect) | {o + i for o in crc.values() for i in range(4)} == set(range(144))
    for off, v in expect.items():
        assert b[off] == v, f"byte {off}: got {b[off]:#04x} want {v:#04x}"
    assert int.from_bytes(b[crc["CRC32_BODY"]:][:4], "little") == zlib.crc32(b[64:144])
    assert int.from_bytes(b[crc["CRC32_HEADER"]:][:4], "little") == zlib.crc32(b[0:60])
    assert O.header_flags(blob) == O.FLAG_GRID_SYMMETRIC
    w2, s2, c2, R2 = O.unpack(blob)
    assert R2 == R and np.array_equal(w2, w) and np.array_equal(s2, s) and np.array_equal(c2, c)
    for i in (0, 1, 2, 63):
        x = np.zeros((1, K), np.uint16); x[0, i] = 0x3F80
        y, _ = O.matvec(w, s, c, x, flags=O.FLAG_GRID_SYMMETRIC)
        assert y[0, 0] == (0.5 if i % 2 else -0.5) and y[0, 1] == 0.5 * (i % 3 - 1)


@pytest.mark.parametrize("k", [1, 2, 4, 8])
def test_single_code_bit_positions(k):
    # One 1-bit... 8-bit group (N=1, K=64, R=16): header 64 + directory 16 = 80; record: counts+width word
    # padded to 16, one scale padded to 16, then the group's 8k code bytes at record offset 32.
    code_start = 80 + 32
    for i in range(64):
        for v in sorted({1, (1 << k) - 1, (0x5A % (1 << k)) or 1}):
            codes = np.zeros((1, 64), np.uint8)
            codes[0, i] = v
            blob = O.pack(1, 64, 16, np.array([[k]], np.uint8), np.array([[0x3C00]], np.uint16), codes)
            bits = np.unpackbits(blob[code_start:code_start + 8 * k], bitorder="little")
            want = np.zeros(64 * k, np.uint8)
            for b in range(k):
                want[k * i + b] = (v >> b) & 1
            assert np.array_equal(bits, want), (k, i, v)


def random_logical(g, N, K, p=S.P_BASE):
    w = S.widths_iid(N, K // 64, p, g)
    s = S.scales_uniform(N, K // 64, g)
    c = S.codes_uniform(w, g)
    return w, s, c


@pytest.mark.parametrize("N,K,R", [(1, 64, 16), (17, 128, 16), (100, 320, 32), (1000, 256, 1024),
                                   (1030, 192, 512), (64, 64, 64)])
def test_pack_unpack_round_trip(N, K, R):
    g = np.random.default_rng(N * 1000 + K + R)
    w, s, c = random_logical(g, N, K)
    blob = O.pack(N, K, R, w, s, c)
    assert blob.size % 16 == 0
    assert O.packed_size(N, K, R, w) == blob.size
    w2, s2, c2, R2 = O.unpack(blob)
    assert R2 == R and np.array_equal(w, w2) and np.array_equal(s, s2) and np.array_equal(c, c2)
    blob2 = O.pack(N, K, R, w2, s2, c2)
    assert np.array_equal(blob, blob2)


def test_unpack_rejects_corruption():
    g = np.random.default_rng(7)
    N, K, R = 40, 128, 16
    w, s, c = random_logical(g, N, K)
    blob = O.pack(N, K, R, w, s, c)

    def refresh(b):
        b = b.copy()
        b[56:60] = np.frombuffer(zlib.crc32(b[64:].tobytes()).to_bytes(4, "little"), np.uint8)
        b[60:64] = np.frombuffer(zlib.crc32(b[:60].tobytes()).to_bytes(4, "little"), np.uint8)
        return b

    assert O.unpack_status(blob[:63])[0] == O.ERR_BUFFER_TOO_SMALL
    assert O.unpack_status(blob[:-16])[0] == O.ERR_BUFFER_TOO_SMALL
    b = blob.copy(); b[0] ^= 1
    assert O.unpack_status(b)[0] == O.ERR_BAD_MAGIC
    b = blob.copy(); b[4] = 2
    assert O.unpack_status(b)[0] == O.ERR_VERSION
    b = blob.copy(); b[-1] ^= 0x10
    assert O.unpack_status(b)[0] == O.ERR_CRC
    b = blob.copy(); b[20] = 17
    assert O.unpack_status(refresh(b))[0] == O.ERR_FORMAT
    # first record: the width word region of a 16-row tile is exactly one word, so bytes 12..15 are padding
    rec = 64 + ((4 * (3 * 2 + 1) + 15) // 16) * 16
    b = blob.copy(); b[rec + 12] = 1
    assert O.unpack_status(refresh(b))[0] == O.ERR_FORMAT
    b = blob.copy(); b[rec] ^= 1   # count n1 no longer matches the width codes
    assert O.unpack_status(refresh(b))[0] == O.ERR_FORMAT
    assert O.unpack_status(refresh(blob))[0] == O.OK


def test_pack_error_codes():
    g = np.random.default_rng(3)
    w, s, c = random_logical(g, 4, 128)
    assert O.pack_status(4, 100, 16, w, s, c)[0] == O.ERR_SHAPE
    assert O.pack_status(4, 128, 8, w, s, c)[0] == O.ERR_TILE
    assert O.pack_status(4, 128, 24, w, s, c)[0] == O.ERR_TILE
    bad = w.copy(); bad[1, 1] = 3
    assert O.pack_status(4, 128, 16, bad, s, c)[0] == O.ERR_WIDTH
    cc = c.copy(); r = int(np.argwhere(w[:, 0] == 1)[0][0]) if (w[:, 0] == 1).any() else None
    if r is None:
        w[0, 0] = 1; c[0, :64] &= 1; r = 0; cc = c.copy()
    cc[r, 5] = 2
    assert O.pack_status(4, 128, 16, w, s, cc)[0] == O.ERR_CODE_RANGE
    size = O.packed_size(4, 128, 16, w)
    assert O.pack_status(4, 128, 16, w, s, c, cap=size - 16)[0] == O.ERR_BUFFER_TOO_SMALL


# ------------------------------------------------------------------------------------------------ matvec
def grid_offset(k, symmetric):
    """The value-grid offset c of w = s (q - c), from its definition: (2^k - 1)/2 on the default half-integer grid;
    on Eq. 1's symmetric integer grid of the VBQ paper (section 3.1, header flag bit 0) 2^(k-1) - 1 for k >= 2,
    the 1-bit case (sign times the mean magnitude) staying +-s/2."""
    if symmetric and k >= 2:
        return Fraction((1 << (k - 1)) - 1)
    return Fraction((1 << k) - 1, 2)


def exact_y(w, s, c, xbits, flags=0):
    """Exact rational y and bound, decoding with numpy/torch (not the oracle)."""
    N, K = c.shape
    sym = bool(flags & O.FLAG_GRID_SYMMETRIC)
    sv = [[Fraction(float(v)) for v in row] for row in f16(s)]
    xv = [Fraction(float(v)) for v in bf16(xbits)]
    ys, bs = [], []
    for r in range(N):
        acc, a = Fraction(0), Fraction(0)
        for i in range(K):
            k = int(w[r, i // 64])
            wt = sv[r][i // 64] * (int(c[r, i]) - grid_offset(k, sym))
            acc += wt * xv[i]
            a += abs(wt) * abs(xv[i])
        ys.append(acc); bs.append(a)
    return ys, bs


def codes_on_grid(w, c, flags):
    """Codes valid on the flagged grid: at most 2^k - 2 for k >= 2 on the symmetric grid; a code at the top of
    each k >= 2 group so that the grid's extreme point is exercised."""
    if not flags & O.FLAG_GRID_SYMMETRIC:
        return c
    kk = np.repeat(w.astype(np.int64), 64, axis=1)
    top = np.where(kk >= 2, (1 << kk) - 2, 1)
    c = np.minimum(c, top).astype(np.uint8)
    c[:, ::64] = np.where(kk[:, ::64] >= 2, top[:, ::64], c[:, ::64])
    return c


@pytest.mark.parametrize("flags", [0, O.FLAG_GRID_SYMMETRIC])
def test_matvec_matches_exact_rationals_all_width_pairs(flags):
    # K=128 (2 groups): all 16 (width, width) pairs, one row each, on either value grid.
    g = np.random.default_rng(11)
    pairs = [(a, b) for a in (1, 2, 4, 8) for b in (1, 2, 4, 8)]
    w = np.array(pairs, np.uint8)
    s = S.scales_uniform(16, 2, g)
    s[3, 1] = 0xB555   # a negative scale
    s[5, 0] = 0x0003   # a subnormal scale
    c = codes_on_grid(w, S.codes_uniform(w, g), flags)
    x = S.x_normal(1, 128, g)
    x[0, 7] = 0x0001   # a subnormal activation
    x[0, 9] = 0x7F00   # a large one
    y, a = O.matvec(w, s, c, x, flags=flags)
    ys, bs = exact_y(w, s, c, x[0], flags)
    for r in range(16):
        assert abs(Fraction(y[0, r]) - ys[r]) <= Fraction(1, 2**50) * bs[r] + Fraction(1, 2**1000)
        assert abs(Fraction(a[0, r]) - bs[r]) <= Fraction(1, 2**50) * bs[r]


@pytest.mark.parametrize("flags", [0, O.FLAG_GRID_SYMMETRIC])
@pytest.mark.parametrize("N,K", [(1, 64), (3, 192), (5, 64)])
def test_matvec_brute_force_small(N, K, flags):
    g = np.random.default_rng(N + K)
    w, s, c = random_logical(g, N, K, p=(0.25, 0.25, 0.25, 0.25))
    c = codes_on_grid(w, c, flags)
    x = S.x_normal(2, K, g)
    y, a = O.matvec(w, s, c, x, flags=flags)
    for b in range(2):
        ys, bs = exact_y(w, s, c, x[b], flags)
        for r in range(N):
            assert abs(Fraction(y[b, r]) - ys[r]) <= Fraction(1, 2**50) * bs[r]


def test_symmetric_grid_closed_forms():
    """Eq. 1's grid at its extreme and middle codes, on a one-hot activation: code 2^k - 2 is +(2^(k-1) - 1) s,
    code 0 is -(2^(k-1) - 1) s, code 2^(k-1) - 1 is exactly 0; 1-bit codes stay +-s/2."""
    K = 64
    xe = np.zeros((1, K), np.uint16); xe[0, 5] = 0x3F80   # bf16 1.0 at column 5
    s = np.full((1, 1), 0x3400, np.uint16)                 # 0.25
    for k in (2, 4, 8):
        L = (1 << (k - 1)) - 1
        for code, want in ((2 * L, L * 0.25), (0, -L * 0.25), (L, 0.0)):
            c = np.full((1, K), code, np.uint8)
            y, a = O.matvec(np.full((1, 1), k, np.uint8), s, c, xe, flags=O.FLAG_GRID_SYMMETRIC)
            assert y[0, 0] == want and a[0, 0] == abs(want), (k, code)
    for code, want in ((1, 0.125), (0, -0.125)):
        y, _ = O.matvec(np.ones((1, 1), np.uint8), s, np.full((1, K), code, np.uint8), xe,
                        flags=O.FLAG_GRID_SYMMETRIC)
        assert y[0, 0] == want
    # codes above 2^k - 2 do not exist on the symmetric grid: the packer refuses them
    assert O.pack_status(1, K, 16, np.full((1, 1), 2, np.uint8), s, np.full((1, K), 3, np.uint8),
                         flags=O.FLAG_GRID_SYMMETRIC)[0] == O.ERR_CODE_RANGE


@pytest.mark.parametrize("k", [1, 2, 4, 8])
def test_closed_forms_uniform_width(k):
    N, K = 6, 256
    g = np.random.default_rng(100 + k)
    x = S.x_normal(1, K, g)
    xs = bf16(x[0])
    s0 = 0x2E66  # fp16 0.1
    s = np.full((N, K // 64), s0, np.uint16)
    w = np.full((N, K // 64), k, np.uint8)
    sv = float(f16(s0))
    tot = math.fsum(xs)
    top = np.full((N, K), (1 << k) - 1, np.uint8)
    y, _ = O.matvec(w, s, top, x)
    assert np.allclose(y[0], sv * ((1 << k) - 1) / 2 * tot, rtol=1e-13, atol=1e-13)
    y, _ = O.matvec(w, s, np.zeros((N, K), np.uint8), x)
    assert np.allclose(y[0], -sv * ((1 << k) - 1) / 2 * tot, rtol=1e-13, atol=1e-13)
    if k == 1:
        c = g.integers(0, 2, size=(N, K)).astype(np.uint8)
        y, _ = O.matvec(w, s, c, x)
        for r in range(N):
            want = sv / 2 * (math.fsum(xs[c[r] == 1]) - math.fsum(xs[c[r] == 0]))
            assert abs(y[0, r] - want) <= 1e-13 * (1 + abs(want))
    if k == 8:  # code 255 -> +127.5 s, code 0 -> -127.5 s, checked on a one-hot activation
        xe = np.zeros((1, K), np.uint16); xe[0, 3] = 0x3F80
        y, _ = O.matvec(w, s, top, xe)
        assert np.all(y[0] == 127.5 * sv)


def test_one_hot_columns_are_dequantized_weights():
    g = np.random.default_rng(5)
    N, K = 9, 192
    w, s, c = random_logical(g, N, K, p=(0.25, 0.25, 0.25, 0.25))
    sv = f16(s)
    for i in (0, 1, 63, 64, 100, 191):
        x = np.zeros((1, K), np.uint16); x[0, i] = 0x3F80   # bf16 1.0
        y, a = O.matvec(w, s, c, x)
        for r in range(N):
            k = int(w[r, i // 64])
            want = sv[r, i // 64] * (int(c[r, i]) - ((1 << k) - 1) / 2)
            assert y[0, r] == want and a[0, r] == abs(want)


def test_power_of_two_scale_invariance():
    g = np.random.default_rng(9)
    N, K = 20, 320
    w, s, c = random_logical(g, N, K)
    x = S.x_normal(3, K, g)
    y1, a1 = O.matvec(w, s, c, x)
    s2 = (s.astype(np.uint32) + (1 << 10)).astype(np.uint16)   # exponent + 1: exact doubling for normal fp16
    assert np.array_equal(f16(s2), 2 * f16(s))
    y2, a2 = O.matvec(w, s2, c, x)
    assert np.array_equal(y2, 2 * y1) and np.array_equal(a2, 2 * a1)


def test_matvec_against_an_independent_library_matmul():
    """T12, on the host: the weights rebuilt with numpy straight from the definition (fp16 scale times
    q - (2^k - 1)/2, no oracle code) and multiplied by numpy's BLAS. In fp64 the two sums differ only by
    rounding order (1e-12 of sum |w||x|); in fp32, BLAS stays inside the parity bar, as a fp32 kernel must."""
    g = np.random.default_rng(12)
    N, K, B = 384, 4096, 3
    w, s, c = random_logical(g, N, K)
    x = S.x_normal(B, K, g)
    y_ref, a = O.matvec(w, s, c, x, os.cpu_count() or 1)
    kk = np.repeat(w.astype(np.int64), 64, axis=1)
    W = np.repeat(f16(s), 64, axis=1) * (c.astype(np.float64) - ((1 << kk) - 1) / 2)
    X = bf16(x)
    y64 = X @ W.T
    assert np.all(np.abs(y64 - y_ref) <= 1e-12 * a + 1e-300)
    y32 = (X.astype(np.float32) @ W.astype(np.float32).T).astype(np.float64)
    assert np.array_equal(W.astype(np.float32).astype(np.float64), W)       # every weight exact in fp32
    assert np.all(O.within_tolerance(y32, y_ref, a))


def test_silu_pins_and_identities():
    """SiLU, the gate nonlinearity of the SwiGLU epilogue, pinned to textbook values of the logistic function
    sigma(t) = 1 / (1 + e^-t): sigma(1) = 0.7310585786300049, sigma(-1) = 0.2689414213699951."""
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(1.0) - 0.7310585786300049) < 1e-15
    assert abs(O.silu(-1.0) - (-0.2689414213699951)) < 1e-15
    assert abs(O.silu(40.0) - 40.0) < 1e-12                      # sigma(40) = 1 - 4e-18
    assert -1e-15 < O.silu(-40.0) < 0.0                           # -40 e^-40 / (1 + e^-40)
    assert np.isfinite(O.silu(-1000.0)) and O.silu(-1000.0) <= 0.0   # no overflow for very negative inputs
    t = np.linspace(-30, 30, 601)
    assert np.allclose(O.silu(t) - O.silu(-t), t, rtol=0, atol=1e-12)   # sigma(t) + sigma(-t) = 1
    assert np.array_equal(O.swiglu(t, 2 * np.ones_like(t)), 2 * O.silu(t))


def test_swiglu_bound_covers_bf16_rounding():
    """The h bar admits the bf16 rounding of an exact h (half an ulp is at most 2^-9 relative)."""
    rng = np.random.default_rng(0)
    g, u = rng.normal(0, 3, 1000), rng.normal(0, 3, 1000)
    h = O.swiglu(g, u)
    h_bf16 = (h.astype(np.float32).view(np.uint32) + 0x7FFF + ((h.astype(np.float32).view(np.uint32) >> 16) & 1)) \
        & 0xFFFF0000
    hq = h_bf16.astype(np.uint32).view(np.float32).astype(np.float64)
    bound = O.swiglu_bound(g, u, np.zeros_like(g), np.zeros_like(u))
    assert np.all(np.abs(hq - h) <= bound)


def silu_prime(g):
    """Textbook derivative of g * sigma(g): sigma(g) (1 + g (1 - sigma(g))), sigma the logistic function."""
    sg = 1.0 / (1.0 + np.exp(-np.asarray(g, np.float64)))
    return sg * (1.0 + g * (1.0 - sg))


def test_silu_derivative_is_below_the_bar_constant():
    """The 1.1 of the h bar bounds |silu'|: the textbook derivative on a fine grid peaks at 1.0998 (g = 2.3994), and
    central differences of the oracle's silu agree with it."""
    g = np.concatenate([np.linspace(-40, 40, 160001), np.linspace(2.3, 2.5, 20001)])
    d = silu_prime(g)
    assert 1.0995 < d.max() < 1.1 and abs(g[np.argmax(d)] - 2.3994) < 1e-3
    assert d.min() > -0.1
    h = 1e-5
    fd = (O.silu(g + h) - O.silu(g - h)) / (2 * h)
    assert np.max(np.abs(fd - d)) < 1e-8


def test_swiglu_bound_covers_every_admissible_perturbation():
    """The propagation term P of the h bar (the bar without its rounding terms 2^-8 (|h| + P) + 1e-6) bounds
    |silu(g') u' - silu(g) u| for every g' within tol_g of g and u' within tol_u of u: on a grid of (g, u) with |g|
    up to 30, dense around the peak of silu', each with the corners and 21 interior points of the tolerance box."""
    gs = np.concatenate([np.linspace(-30, 30, 241), np.linspace(2.2, 2.6, 41), [-1.2785]])
    us = np.array([-30.0, -3.0, -0.5, 0.0, 0.5, 3.0, 30.0])
    worst = 0.0
    for tg, tu in ((1e-3, 1e-3), (0.05, 0.02), (0.5, 0.5), (2.0, 1.0)):
        G, U = np.meshgrid(gs, us, indexing="ij")
        A_g, A_u = (tg - 1e-6) / 1e-3, (tu - 1e-6) / 1e-3   # sum|w||x| that gives these tolerances
        bar = O.swiglu_bound(G, U, np.full_like(G, A_g), np.full_like(U, A_u))
        h = O.swiglu(G, U)
        prop = (bar - 1e-6 - 2.0 ** -8 * np.abs(h)) / (1.0 + 2.0 ** -8)
        for dg in np.concatenate([np.linspace(-1, 1, 21), [-1.0, 1.0]]):
            for du in (-1.0, -0.5, 0.0, 0.5, 1.0):
                d = np.abs(O.swiglu(G + dg * tg, U + du * tu) - h)
                assert np.all(d <= prop * (1 + 1e-12) + 1e-12), (tg, tu, dg, du, float((d - prop).max()))
                worst = max(worst, float((d / np.maximum(prop, 1e-300)).max()))
    assert worst > 0.9   # the bar is tight somewhere: it is not loose by a large factor


def test_recipe_workload_shape():
    """The fixed-recipe workload has the widths the recipe fixes: 2-bit projections, a 4-bit first-block MLP, and
    a head whose tiers give 1.18 mean bits with rows in descending frequency order."""
    l0, l1 = S.cfg6_recipe_layer(0), S.cfg6_recipe_layer(1)
    assert all(np.all(m.widths == (4 if m.name in ("gate", "up", "down") else 2)) for m in l0)
    assert all(np.all(m.widths == 2) for m in l1)
    w = S.widths_head_tiered(32000, 64)
    assert abs(w.mean() - 1.18) < 1e-3
    assert np.all(np.diff(w[:, 0].astype(int)) <= 0)         # widths never increase down the frequency order
    assert (w[:, 0] == 8).sum() == 160 and (w[:, 0] == 4).sum() == 480 and (w[:, 0] == 2).sum() == 3200


def test_quantize_recovers_weights_on_either_grid_exactly():
    """Weights that lie exactly on a grid (with an fp16-exact scale and an extreme point present) come back as
    that scale and those codes: Eq. 1's symmetric grid (flag) and the default half-integer grid."""
    rng = np.random.default_rng(3)
    N, G = 6, 4
    for k in (2, 4, 8):
        Lk = (1 << (k - 1)) - 1
        q = rng.integers(-Lk, Lk + 1, size=(N, G, 64))
        q[:, :, 0] = Lk                                   # the extreme point fixes max|w| = L * s
        s = 0.5
        w = (s * q).reshape(N, G * 64).astype(np.float32)
        st, s16, codes = O.quantize(w, np.full((N, G), k, np.uint8), O.FLAG_GRID_SYMMETRIC)
        assert st == O.OK and np.all(s16 == 0x3800)
        assert np.array_equal(codes.reshape(N, G, 64), (q + Lk).astype(np.uint8))
        assert np.array_equal(O.dequant(np.full((N, G), k, np.uint8), s16, codes, flags=O.FLAG_GRID_SYMMETRIC), w)
        qh = rng.integers(0, 1 << k, size=(N, G, 64))
        qh[:, :, 0] = (1 << k) - 1
        wh = (0.25 * (qh - ((1 << k) - 1) / 2)).reshape(N, G * 64).astype(np.float32)
        st, s16, codes = O.quantize(wh, np.full((N, G), k, np.uint8))
        assert st == O.OK and np.all(s16 == 0x3400)
        assert np.array_equal(codes.reshape(N, G, 64), qh.astype(np.uint8))


def test_quantize_one_bit_is_sign_times_mean_magnitude():
    """1-bit groups: scale 2 * mean|w| (so the grid points are +-mean|w|), code 1 where w >= 0."""
    w = np.tile(np.array([0.125, -0.375, 0.25, -0.25], np.float32), 16)[None, :]   # mean |w| = 0.25
    st, s16, codes = O.quantize(w, np.ones((1, 1), np.uint8))
    assert st == O.OK and s16[0, 0] == 0x3800                                      # 0.5 = 2 * 0.25
    assert np.array_equal(codes[0], (w[0] >= 0).astype(np.uint8))
    assert np.array_equal(O.dequant(np.ones((1, 1), np.uint8), s16, codes)[0], np.where(w[0] >= 0, 0.25, -0.25))


def test_quantize_error_bound_zero_groups_and_bad_values():
    """Every weight lands within half a grid step of its value (the scale's fp16 rounding can push the largest
    one slightly out, by at most L * |s - s16|); all-zero groups decode to zero; non-finite weights and scales
    beyond fp16 are refused."""
    rng = np.random.default_rng(4)
    N, G = 8, 6
    w = rng.normal(0, 0.05, size=(N, G * 64)).astype(np.float32)
    w[0, :64] = 0.0
    widths = np.array([2, 4, 8, 2, 4, 8], np.uint8)[None, :].repeat(N, 0)
    for flags in (0, O.FLAG_GRID_SYMMETRIC):
        st, s16, codes = O.quantize(w, widths, flags)
        assert st == O.OK
        wq = O.dequant(widths, s16, codes, flags=flags)
        sd = np.repeat(s16.view(np.float16).astype(np.float64), 64, axis=1)
        kk = np.repeat(widths.astype(np.int64), 64, axis=1)
        Lc = ((1 << (kk - 1)) - 1) if flags else ((1 << kk) - 1) / 2
        amax = np.repeat(np.abs(w.astype(np.float64)).reshape(N, G, 64).max(axis=2), 64, axis=1)
        assert np.all(np.abs(wq - w) <= sd / 2 + np.abs(amax - Lc * sd) + 1e-12)
        assert np.all(wq[0, :64] == 0.0)
    bad = w.copy()
    bad[1, 5] = np.inf
    assert O.quantize(bad, widths)[0] == O.ERR_VALUE
    assert O.quantize(np.full((1, 64), 3e38, np.float32), np.full((1, 1), 2, np.uint8))[0] == O.ERR_VALUE
