"""Host-side tests of the C ABI (no GPU needed): symbol exports, the packer against the oracle (byte-exact),
unpack and validation error codes against the oracle's, and the argument checks of the device entry points
that run before any CUDA call."""
import ctypes
import os
import re
import zlib

import numpy as np
import pytest

import vbq_synth as S
from decode_vbq_gemv_b200 import vbq
from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    txt = open(os.path.join(ROOT, "include", "vbq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(vbq_[a-z_0-9]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    names = header_functions()
    assert "vbq_gemv" in names and "vbq_gemm_skinny" in names and "vbq_pack" in names
    L = ctypes.CDLL(vbq.library_path() if os.path.exists(vbq.library_path()) else vbq.lib()._name)
    for n in names:
        assert hasattr(L, n), f"libvbq.so does not export {n}"


def test_status_strings_and_version():
    for st in range(-17, 1):
        assert vbq.vbq_strerror(st) and "unknown" not in vbq.vbq_strerror(st)
    assert vbq.vbq_strerror(-99) == "unknown status"
    assert vbq.vbq_version() >> 16 == 1


def logical(seed, N, K, p=S.P_BASE):
    g = np.random.default_rng(seed)
    w = S.widths_iid(N, K // 64, p, g)
    return w, S.scales_uniform(N, K // 64, g), S.codes_uniform(w, g)


SHAPES = [(1, 64, 16), (5, 128, 16), (31, 192, 32), (100, 768, 64), (1030, 256, 1024), (1024, 64, 1024),
          (2049, 128, 512), (17, 320, 1024)]


@pytest.mark.parametrize("N,K,R", SHAPES)
@pytest.mark.parametrize("p", [S.P_BASE, (0.25, 0.25, 0.25, 0.25), (0, 0, 0, 1.0), (1.0, 0, 0, 0)])
def test_pack_matches_oracle_bytes(N, K, R, p):
    w, s, c = logical(N * 7 + K + R, N, K, p)
    blob, d = vbq.vbq_pack(N, K, R, w, s, c)
    ref = O.pack(N, K, R, w, s, c)
    assert np.array_equal(blob, ref)
    assert vbq.vbq_packed_size(N, K, R, w) == ref.size
    assert (d.N, d.K, d.G, d.R, d.T, d.total_bytes) == (N, K, K // 64, R, (N + R - 1) // R, ref.size)
    w2, s2, c2 = vbq.vbq_unpack(ref)
    assert np.array_equal(w2, w) and np.array_equal(s2, s) and np.array_equal(c2, c)


def test_pack_matches_oracle_on_workload_configs():
    for m in S.cfg1() + S.cfg2()[:1] + [S.cfg3(256, 512)[4]]:
        blob, _ = vbq.vbq_pack(m.N, m.K, 1024, m.widths, m.scales, m.codes)
        assert np.array_equal(blob, O.pack(m.N, m.K, 1024, m.widths, m.scales, m.codes))


def test_pack_error_codes_match_oracle():
    w, s, c = logical(1, 6, 128)
    cases = [(6, 100, 16, w, s, c), (6, 128, 8, w, s, c), (6, 128, 2048, w, s, c), (0, 128, 16, w, s, c)]
    bad_w = w.copy(); bad_w[2, 1] = 5
    cases.append((6, 128, 16, bad_w, s, c))
    bad_c = c.copy(); r, g = np.argwhere(w < 8)[0]; bad_c[r, 64 * g + 3] = 1 << int(w[r, g])
    cases.append((6, 128, 16, w, s, bad_c))
    for args in cases:
        st_lib = vbq.vbq_pack_status(*args)[0]
        st_ora = O.pack_status(*args)[0]
        assert st_lib == st_ora and st_lib < 0, (st_lib, st_ora)
    size = vbq.vbq_packed_size(6, 128, 16, w)
    assert vbq.vbq_pack_status(6, 128, 16, w, s, c, cap=size - 1)[0] == vbq.VBQ_ERR_BUFFER_TOO_SMALL


def _refresh_crc(b):
    b = b.copy()
    b[56:60] = np.frombuffer(zlib.crc32(b[64:].tobytes()).to_bytes(4, "little"), np.uint8)
    b[60:64] = np.frombuffer(zlib.crc32(b[:60].tobytes()).to_bytes(4, "little"), np.uint8)
    return b


def test_unpack_error_codes_match_oracle():
    w, s, c = logical(2, 70, 192)
    blob = O.pack(70, 192, 32, w, s, c)
    rng = np.random.default_rng(0)
    variants = [blob[:10], blob[:-16], blob.copy(), blob.copy(), blob.copy(), blob.copy()]
    variants[2][0] ^= 0xFF
    variants[3][4] = 9
    variants[4][100] ^= 1
    variants[5][-3] ^= 4
    # single-byte corruptions anywhere, with the CRCs made consistent again so the layout checks decide
    for _ in range(300):
        b = blob.copy()
        i = int(rng.integers(64, blob.size))
        b[i] ^= np.uint8(1 << int(rng.integers(0, 8)))
        variants.append(_refresh_crc(b))
    for b in variants:
        st_lib = vbq.vbq_unpack_status(b)[0]
        st_ora = O.unpack_status(b)[0]
        assert st_lib == st_ora, (st_lib, st_ora)
        if st_lib == 0:   # a corruption that still decodes must decode identically
            lw, ls, lc = vbq.vbq_unpack_status(b)[1]
            ow, os_, oc, _ = O.unpack_status(b)[1]
            assert np.array_equal(lw, ow) and np.array_equal(ls, os_) and np.array_equal(lc, oc)


def test_device_entry_argument_checks_need_no_gpu():
    w, s, c = logical(3, 40, 128)
    _, d = vbq.vbq_pack(40, 128, 16, w, s, c)
    L = vbq.lib()
    dp = ctypes.byref(d)
    assert L.vbq_gemv(dp, None, 16, 16, None, 0, None) == vbq.VBQ_ERR_NULL
    assert L.vbq_gemm_skinny(dp, 16, 16, 3, 16, None, 0, None) == vbq.VBQ_ERR_BATCH
    assert L.vbq_gemm_skinny(dp, 8, 16, 1, 16, None, 0, None) == vbq.VBQ_ERR_ALIGN
    assert L.vbq_gemm_skinny(dp, 16, 18, 1, 16, None, 0, None) == vbq.VBQ_ERR_ALIGN
    assert L.vbq_gemm_skinny(dp, 16, 16, 1, 18, None, 0, None) == vbq.VBQ_ERR_ALIGN
    bad = vbq.vbq_desc.from_buffer_copy(d)
    bad.K = 100
    assert L.vbq_gemv(ctypes.byref(bad), 16, 16, 16, None, 0, None) == vbq.VBQ_ERR_FORMAT
    out = ctypes.c_uint64()
    assert L.vbq_workspace_size(dp, 3, ctypes.byref(out)) == vbq.VBQ_ERR_BATCH
    assert L.vbq_workspace_size(dp, 16, ctypes.byref(out)) == vbq.VBQ_OK
    assert L.vbq_workspace_init(None, 0, None) == vbq.VBQ_ERR_NULL
    # the launch-options entry point: same checks, plus unknown option bits
    assert L.vbq_gemm_skinny_ex(dp, 16, 16, 1, 16, None, 0, 2, None) == vbq.VBQ_ERR_FLAGS
    assert L.vbq_gemm_skinny_ex(dp, 16, 16, 3, 16, None, 0, vbq.VBQ_LAUNCH_OVERLAP, None) == vbq.VBQ_ERR_BATCH
    assert L.vbq_gemm_skinny_ex(dp, 8, 16, 1, 16, None, 0, vbq.VBQ_LAUNCH_OVERLAP, None) == vbq.VBQ_ERR_ALIGN
    assert L.vbq_gemm_skinny_ex(dp, None, 16, 1, 16, None, 0, 0, None) == vbq.VBQ_ERR_NULL


def test_multi_entry_argument_checks_need_no_gpu():
    """vbq_gemm_skinny_multi / vbq_workspace_size_multi reject bad matrix sets before any CUDA call."""
    mk = lambda N, K, R, seed: vbq.vbq_pack(N, K, R, *logical(seed, N, K))[1]
    a, b = mk(40, 128, 16, 1), mk(70, 128, 16, 2)
    other_k, other_r = mk(40, 256, 16, 3), mk(40, 128, 32, 4)
    size = vbq.lib().vbq_workspace_size_multi
    out = ctypes.c_uint64()
    arr = vbq._desc_array
    assert size(2, arr([a, b]), 1, ctypes.byref(out)) == vbq.VBQ_OK
    one = ctypes.c_uint64()
    assert vbq.lib().vbq_workspace_size(ctypes.byref(a), 1, ctypes.byref(one)) == vbq.VBQ_OK
    assert out.value >= one.value
    assert size(0, arr([a]), 1, ctypes.byref(out)) == vbq.VBQ_ERR_SHAPE
    assert size(5, arr([a, b, a, b, a]), 1, ctypes.byref(out)) == vbq.VBQ_ERR_SHAPE
    assert size(2, arr([a, other_k]), 1, ctypes.byref(out)) == vbq.VBQ_ERR_SHAPE
    assert size(2, arr([a, other_r]), 1, ctypes.byref(out)) == vbq.VBQ_ERR_TILE
    assert size(2, arr([a, b]), 3, ctypes.byref(out)) == vbq.VBQ_ERR_BATCH
    assert size(2, None, 1, ctypes.byref(out)) == vbq.VBQ_ERR_NULL
    run = vbq.lib().vbq_gemm_skinny_multi
    P = lambda *v: (ctypes.c_void_p * len(v))(*v)
    assert run(2, arr([a, b]), P(16, 16), 16, 1, P(16, 16), None, 0, 0, None) == vbq.VBQ_ERR_WORKSPACE
    assert run(2, arr([a, b]), P(16, None), 16, 1, P(16, 16), None, 0, 0, None) == vbq.VBQ_ERR_NULL
    assert run(2, arr([a, b]), P(16, 16), 16, 1, P(16, 16), None, 0, 4, None) == vbq.VBQ_ERR_FLAGS
    assert run(2, arr([a, b]), P(16, 24), 16, 1, P(16, 16), None, 0, 0, None) == vbq.VBQ_ERR_ALIGN
    assert run(2, arr([a, b]), P(16, 16), 16, 1, P(16, 18), None, 0, 0, None) == vbq.VBQ_ERR_ALIGN
    assert run(2, arr([a, other_r]), P(16, 16), 16, 1, P(16, 16), None, 0, 0, None) == vbq.VBQ_ERR_TILE


def test_swiglu_entry_argument_checks_need_no_gpu():
    """vbq_gemm_swiglu rejects mismatched gate/up shapes, odd h and unknown flags before any CUDA call."""
    mk = lambda N, K, R, seed: vbq.vbq_pack(N, K, R, *logical(seed, N, K))[1]
    g, u = mk(40, 128, 16, 1), mk(40, 128, 16, 2)
    other_n, other_r = mk(48, 128, 16, 3), mk(40, 128, 32, 4)
    L = vbq.lib()
    r = ctypes.byref
    out = ctypes.c_uint64()
    assert L.vbq_workspace_size_swiglu(r(g), r(u), 1, r(out)) == vbq.VBQ_OK
    assert out.value == vbq.vbq_workspace_size_multi([g, u], 1)
    assert L.vbq_workspace_size_swiglu(r(g), r(other_n), 1, r(out)) == vbq.VBQ_ERR_SHAPE
    assert L.vbq_workspace_size_swiglu(r(g), r(other_r), 1, r(out)) == vbq.VBQ_ERR_TILE
    run = L.vbq_gemm_swiglu
    assert run(r(g), r(u), 16, 16, 16, 1, 16, 16, None, None, 0, 0, None) == vbq.VBQ_ERR_NULL
    assert run(r(g), r(u), 16, 16, 16, 3, 16, 16, 16, None, 0, 0, None) == vbq.VBQ_ERR_BATCH
    assert run(r(g), r(u), 16, 16, 16, 1, 16, 16, 16, None, 0, 2, None) == vbq.VBQ_ERR_FLAGS
    assert run(r(g), r(other_n), 16, 16, 16, 1, 16, 16, 16, None, 0, 0, None) == vbq.VBQ_ERR_SHAPE
    assert run(r(g), r(other_r), 16, 16, 16, 1, 16, 16, 16, None, 0, 0, None) == vbq.VBQ_ERR_TILE
    assert run(r(g), r(u), 16, 16, 16, 1, 16, 16, 17, None, 0, 0, None) == vbq.VBQ_ERR_ALIGN
    assert run(r(g), r(u), 16, 16, 16, 1, 16, 16, 16, None, 0, 0, None) == vbq.VBQ_ERR_WORKSPACE


def test_quantize_matches_oracle_bitwise_on_both_grids():
    """vbq_quantize (C++) and the oracle's quantize (numpy) give the same scales and codes, bit for bit: random
    weights over many magnitudes (fp16-subnormal scales included), every width, both grids, plus crafted
    groups whose scale ratio lies exactly halfway between two fp16 values and weights exactly halfway between
    two grid points."""
    rng = np.random.default_rng(21)
    N, G = 24, 8
    K = 64 * G
    w = (rng.normal(0, 1, size=(N, K)) * np.exp(rng.uniform(-14, 3, size=(N, 1)))).astype(np.float32)
    # ratio exactly halfway between fp16 1.0 and 1.0009765625 (k = 2 symmetric: L = 1, ratio = max|w|)
    w[0, :64] = 0.0
    w[0, 0] = np.float32(1.0 + 2.0 ** -11)
    # weights at x.5 steps of a power-of-two scale (ties for round())
    w[1, :64] = np.float32(0.5) * (np.arange(64) - 31.5).astype(np.float32) / np.float32(31.5) * np.float32(3.5)
    w[2, :64] = -w[1, :64]
    widths = rng.choice(np.array([1, 2, 4, 8], np.uint8), size=(N, G))
    widths[0, 0] = 2
    widths[1, 0] = widths[2, 0] = 8
    for flags in (0, vbq.VBQ_FLAG_GRID_SYMMETRIC):
        st_o, s_o, c_o = O.quantize(w, widths, flags)
        st_l, s_l, c_l = vbq.vbq_quantize_status(w, widths, flags)
        assert st_o == st_l == 0
        assert np.array_equal(s_o, s_l), np.argwhere(s_o != s_l)[:5]
        assert np.array_equal(c_o, c_l), np.argwhere(c_o != c_l)[:5]


def test_symmetric_grid_pack_unpack_and_errors():
    """Format flag bit 0 (Eq. 1's grid): the library's blob equals the oracle's byte for byte, carries the flag
    in its header and descriptor, and unpacks back; a code 2^k - 1 (outside the symmetric range) is refused by
    pack and, planted into a blob, by unpack; unknown format bits and bad weights are refused."""
    rng = np.random.default_rng(22)
    N, K = 70, 256
    widths = rng.choice(np.array([1, 2, 4, 8], np.uint8), size=(N, K // 64))
    w = rng.normal(0, 0.05, size=(N, K)).astype(np.float32)
    sym = vbq.VBQ_FLAG_GRID_SYMMETRIC
    scales, codes = vbq.vbq_quantize(w, widths, sym)
    blob, d = vbq.vbq_pack(N, K, 32, widths, scales, codes, format_flags=sym)
    assert d.flags == sym and vbq.vbq_describe(blob).flags == sym
    assert np.array_equal(blob, O.pack(N, K, 32, widths, scales, codes, flags=sym))
    assert O.header_flags(blob) == sym
    uw, us, uc = vbq.vbq_unpack(blob)
    assert np.array_equal(uw, widths) and np.array_equal(us, scales) and np.array_equal(uc, codes)
    r, g = np.argwhere(widths >= 2)[0]
    bad = codes.copy()
    bad[r, 64 * g] = (1 << int(widths[r, g])) - 1
    assert vbq.vbq_pack_status(N, K, 32, widths, scales, bad, format_flags=sym)[0] == vbq.VBQ_ERR_CODE_RANGE
    assert vbq.vbq_pack_status(N, K, 32, widths, scales, bad)[0] == vbq.VBQ_OK   # fine on the default grid
    plain, _ = vbq.vbq_pack(N, K, 32, widths, scales, bad)
    flagged = plain.copy()
    flagged[6] = sym                                            # claim the symmetric grid for that blob
    flagged = _refresh_crc(flagged)
    assert vbq.vbq_unpack_status(flagged)[0] == vbq.VBQ_ERR_FORMAT == O.unpack_status(flagged)[0]
    assert vbq.vbq_pack_status(N, K, 32, widths, scales, codes, format_flags=2)[0] == vbq.VBQ_ERR_FLAGS
    nan = w.copy()
    nan[3, 7] = np.nan
    assert vbq.vbq_quantize_status(nan, widths, 0)[0] == vbq.VBQ_ERR_VALUE
    assert vbq.vbq_quantize_status(np.full((1, 64), 1e38, np.float32), np.full((1, 1), 2, np.uint8), 0)[0] \
        == vbq.VBQ_ERR_VALUE


def test_suggest_tile_rows_rule():
    # the largest of 1024, 512, 256 rows that leaves every SM at least 7 records (tile, group column)
    assert vbq.suggest_tile_rows(4096, 4096, 148) == 256            # 1024 records at 256 rows: 6.9 per SM
    assert vbq.suggest_tile_rows(3 * 4096, 4096, 148) == 512        # fused q/k/v
    assert vbq.suggest_tile_rows(2 * 14336, 4096, 148) == 1024      # fused gate/up
    assert vbq.suggest_tile_rows(4096, 14336, 148) == 512           # down: 224 group columns
    assert vbq.suggest_tile_rows(32000, 4096, 148) == 1024          # LM head
    assert vbq.suggest_tile_rows(768, 768, 148) == 256              # too small for any: the smallest
    for rows, K in ((1, 64), (4096, 4096), (32000, 4096)):
        R = vbq.suggest_tile_rows(rows, K, 148)
        assert 16 <= R <= 1024 and R % 16 == 0


def test_pack_and_quantize_are_thread_safe():
    """The host entry points are pure (the bench packs layers on a thread pool): many threads packing and
    quantizing different matrices at once give the same bytes as one thread doing it alone."""
    import concurrent.futures as cf
    rng = np.random.default_rng(21)
    cases = []
    for i in range(12):
        N, K, R = int(rng.integers(1, 700)), 64 * int(rng.integers(1, 12)), 16 * int(rng.integers(1, 40))
        m = S.Matrix("t", N, K, S.widths_iid(N, K // 64, S.P_BASE, rng), S.scales_uniform(N, K // 64, rng),
                     np.zeros((N, K), np.uint8))
        m.codes[:] = S.codes_uniform(m.widths, rng)
        w = rng.normal(0, 0.05, size=(N, K)).astype(np.float32)
        cases.append((m, R, w))

    def work(c):
        m, R, w = c
        blob, _ = vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes)
        sc, co = vbq.vbq_quantize(w, m.widths)
        return blob.tobytes(), sc.tobytes(), co.tobytes()

    alone = [work(c) for c in cases]
    with cf.ThreadPoolExecutor(max_workers=8) as pool:
        for _ in range(3):
            assert list(pool.map(work, cases)) == alone


def test_packed_size_refuses_blobs_the_directory_cannot_address():
    """Directory entries count 16-byte units in 32 bits: an all-8-bit matrix of 65536 x 1048576 (66 bytes per
    group, 70 GB of records) is refused with VBQ_ERR_SHAPE; one of half the rows (35 GB) is sized normally."""
    psutil = pytest.importorskip("psutil")
    if psutil.virtual_memory().available < 4 << 30:
        pytest.skip("needs about 1.1 GB for the width array")
    G = 16384
    widths = np.full((65536, G), 8, np.uint8)
    L = vbq.lib()
    out = ctypes.c_uint64(0)
    st = L.vbq_packed_size(ctypes.c_int64(65536), ctypes.c_int64(64 * G), ctypes.c_int64(1024),
                           widths.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), ctypes.byref(out))
    assert st == vbq.VBQ_ERR_SHAPE
    half = widths[:32768]
    st = L.vbq_packed_size(ctypes.c_int64(32768), ctypes.c_int64(64 * G), ctypes.c_int64(1024),
                           half.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), ctypes.byref(out))
    assert st == 0 and out.value > 32 << 30


def pad_numpy(w, s, c, N_pad, K_pad):
    """Zero padding written independently of the library: 1-bit groups, scale +0, code 0."""
    N, G = w.shape
    K = c.shape[1]
    wp = np.ones((N_pad, K_pad // 64), np.uint8)
    sp = np.zeros((N_pad, K_pad // 64), np.uint16)
    cp = np.zeros((N_pad, K_pad), np.uint8)
    wp[:N, :G], sp[:N, :G], cp[:N, :K] = w, s, c
    return wp, sp, cp


@pytest.mark.parametrize("N,K,N_pad,K_pad,R", [(100, 192, 512, 512, 64), (1030, 256, 1536, 256, 512),
                                                (64, 448, 64, 512, 16), (7, 64, 7, 64, 16)])
def test_padded_pack_matches_oracle_pack_of_padded_arrays(N, K, N_pad, K_pad, R):
    """vbq_pack_padded equals the oracle's pack of the logical arrays padded with zero weights, and unpacks to
    them; the added weights dequantize to exactly 0 (VBQ paper, section 6, zero padding to a multiple of 512)."""
    w, s, c = logical(N + K + N_pad, N, K)
    for flags in (0, O.FLAG_GRID_SYMMETRIC):
        if flags:
            c = np.minimum(c, (1 << w.repeat(64, axis=1)) - 2 + (w.repeat(64, axis=1) == 1)).astype(np.uint8)
        blob, d = vbq.vbq_pack_padded(N, K, R, w, s, c, N_pad, K_pad, format_flags=flags)
        wp, sp, cp = pad_numpy(w, s, c, N_pad, K_pad)
        assert np.array_equal(blob, O.pack(N_pad, K_pad, R, wp, sp, cp, flags=flags))
        assert (d.N, d.K, d.flags) == (N_pad, K_pad, flags)
        assert vbq.lib().vbq_packed_size_padded is not None
        wq = O.dequant(wp, sp, cp, flags)
        assert not wq[N:, :].any() and not wq[:, K:].any()


def test_padded_pack_refuses_shrinking_or_unaligned_padding():
    w, s, c = logical(3, 10, 128)
    for N_pad, K_pad in ((9, 128), (10, 64), (10, 200), (0, 128)):
        st, blob, _ = vbq.vbq_pack_padded_status(10, 128, 16, w, s, c, N_pad, K_pad)
        assert st == vbq.VBQ_ERR_SHAPE and blob is None


def plan(descs, B, sms=148):
    return vbq.vbq_plan_info_get(descs, B, sms)


@pytest.mark.parametrize("B", [1, 2, 4, 8, 16])
def test_launch_plans_of_the_9b_linears_fit_the_sm(B):
    """Host-side launch plans (vbq_plan_info_get, no GPU): for every 9B-shaped linear at its suggested tile rows,
    a plan exists within 227 KB of shared memory per CTA, one CTA per SM, 16 warps at batch 1-2 and 12 at 4-16,
    1-7 records per batch, 2-3 batches in flight, two result sets below batch 8; records of similar size are
    split by count; the workspace holds one partial slot per CTA and tile plus two counters per tile and the
    status word."""
    for m in S.cfg4(("q", "gate", "down")):
        R = vbq.suggest_tile_rows(m.N, m.K, 148)
        _, d = vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes)
        p = plan(d, B)
        assert p["grid"] == 148 and p["threads"] == (512 if B <= 2 else 384)
        assert 0 < p["smem_bytes"] <= 227 * 1024
        assert 1 <= p["records_per_batch"] <= 7 and p["batches_in_flight"] in (2, 3)
        assert p["result_sets"] == 2 if B < 8 else p["result_sets"] in (1, 2)
        assert p["cost_split"] == 0
        ws = ((148 + d.T) * R * B * 4 + d.T * 8 + 4 + 15) // 16 * 16
        assert p["workspace_bytes"] == ws
        assert plan(d, B, 74)["workspace_bytes"] < ws and plan(d, B, 74)["grid"] == 74


def test_cost_split_is_chosen_for_uneven_records_only():
    """The launch splits records by estimated cost exactly when the largest record exceeds 1.3 times the mean:
    the LM head (frequent rows wider) and a matrix whose first rows are 8-bit, not the base-mix linears, alone or
    fused."""
    head = S.cfg5_head()
    _, dh = vbq.vbq_pack(head.N, head.K, 1024, head.widths, head.scales, head.codes)
    assert plan(dh, 1)["cost_split"] == 1
    w = np.ones((3000, 8), np.uint8)
    w[:300] = 8
    g = np.random.default_rng(1)
    _, du = vbq.vbq_pack(3000, 512, 64, w, S.scales_uniform(3000, 8, g), S.codes_uniform(w, g))
    assert plan(du, 4)["cost_split"] == 1
    gate, up = S.cfg4(("gate", "up"))
    dg = vbq.vbq_pack(gate.N, gate.K, 1024, gate.widths, gate.scales, gate.codes)[1]
    du2 = vbq.vbq_pack(up.N, up.K, 1024, up.widths, up.scales, up.codes)[1]
    assert plan(dg, 1)["cost_split"] == 0 and plan([dg, du2], 1)["cost_split"] == 0


def test_plan_of_the_largest_records_and_argument_errors():
    """All-8-bit 1024-row records (the largest a record gets) still plan at batch 16; bad batch sizes, SM counts,
    matrix counts and mismatched fused shapes are refused with the documented codes."""
    N, K = 2048, 512
    w = np.full((N, K // 64), 8, np.uint8)
    g = np.random.default_rng(2)
    _, d = vbq.vbq_pack(N, K, 1024, w, S.scales_uniform(N, K // 64, g), S.codes_uniform(w, g))
    p = plan(d, 16)
    assert p["records_per_batch"] >= 1 and p["smem_bytes"] <= 227 * 1024
    out = vbq.vbq_plan_info()
    L = vbq.lib()
    assert L.vbq_plan_info_get(1, vbq._desc_array([d]), 3, 148, ctypes.byref(out)) == vbq.VBQ_ERR_BATCH
    assert L.vbq_plan_info_get(1, vbq._desc_array([d]), 1, 0, ctypes.byref(out)) == vbq.VBQ_ERR_SHAPE
    assert L.vbq_plan_info_get(5, vbq._desc_array([d] * 5), 1, 148, ctypes.byref(out)) == vbq.VBQ_ERR_SHAPE
    _, d2 = vbq.vbq_pack(N, 256, 1024, w[:, :4], S.scales_uniform(N, 4, g), S.codes_uniform(w[:, :4], g))
    assert L.vbq_plan_info_get(2, vbq._desc_array([d, d2]), 1, 148, ctypes.byref(out)) == vbq.VBQ_ERR_SHAPE
    assert L.vbq_plan_info_get(1, None, 1, 148, ctypes.byref(out)) == vbq.VBQ_ERR_NULL
