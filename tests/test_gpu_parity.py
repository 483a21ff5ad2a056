"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element.

Bar: |y - y_ref| <= 1e-3 * sum_i |w_i||x_i| + 1e-6 per element (fp32 accumulation), bit-exact for one-hot
activations, bitwise identical across runs. Full-size matrices are checked on sampled rows, which the oracle
computes one by one.
"""
import os

import numpy as np
import pytest
import torch

import vbq_synth as S
from decode_vbq_gemv_b200 import vbq
from oracle import oracle as O

pytestmark = pytest.mark.gpu
NTH = os.cpu_count() or 1


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def to_dev_x(xbits: np.ndarray):
    t = torch.from_numpy(xbits.astype(np.int16)).view(torch.bfloat16)
    return t.to(dev()).contiguous()


def gpu_y(m, xbits, R=1024, mat=None):
    if mat is None:
        blob, _ = vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes)
        mat = vbq.DeviceMatrix(blob, dev())
    xd = to_dev_x(xbits)
    y = mat.matmul(xd)
    torch.cuda.synchronize()
    ws = mat.workspaces[xd.shape[0]]
    need = vbq.vbq_workspace_size(mat.desc, xd.shape[0])
    status = int(ws[need - 4:need].cpu().numpy().view(np.uint32)[0])
    assert status == 0, f"device status word {status:#x}"
    return y.cpu().numpy().astype(np.float64), mat


def check(y, yref, bound, what=""):
    ok = O.within_tolerance(y, yref, bound)
    if not ok.all():
        i = np.argwhere(~ok)[0]
        raise AssertionError(f"{what}: {int((~ok).sum())} elements out of tolerance; first {tuple(i)}: "
                             f"got {y[tuple(i)]!r} want {yref[tuple(i)]!r} bound {bound[tuple(i)]!r}")


def logical(seed, N, K, p):
    g = np.random.default_rng(seed)
    w = S.widths_iid(N, K // 64, p, g)
    return S.Matrix("t", N, K, w, S.scales_uniform(N, K // 64, g), S.codes_uniform(w, g))


SMALL = [(1, 64, 16), (31, 192, 16), (100, 768, 64), (1030, 256, 1024), (2100, 128, 512), (64, 1024, 32),
         (777, 2048, 256), (1000, 512, 208), (3000, 1024, 224)]
DISTS = {"base": S.P_BASE, "flat": (0.25, 0.25, 0.25, 0.25), "all8": (0, 0, 0, 1.0), "all1": (1.0, 0, 0, 0)}


@pytest.mark.parametrize("B", vbq.BATCHES)
@pytest.mark.parametrize("shape", SMALL)
@pytest.mark.parametrize("dist", list(DISTS))
def test_small_shapes_all_batches(shape, dist, B):
    N, K, R = shape
    m = logical(N + K + R + B, N, K, DISTS[dist])
    x = S.x_normal(B, K, np.random.default_rng(B + N))
    y, _ = gpu_y(m, x, R)
    yref, bound = O.matvec(m.widths, m.scales, m.codes, x, NTH)
    check(y, yref, bound, f"{shape} {dist} B={B}")


@pytest.mark.parametrize("B", vbq.BATCHES)
def test_config1_single_linear(B):
    m = S.cfg1()[0]
    x = S.make_x(1, "single", B, m.K)
    y, _ = gpu_y(m, x)
    yref, bound = O.matvec(m.widths, m.scales, m.codes, x, NTH)
    check(y, yref, bound, f"cfg1 B={B}")


@pytest.mark.parametrize("B", [1, 4, 16])
def test_config2_layer(B):
    for m in S.cfg2():
        x = S.make_x(2, m.name, B, m.K)
        y, _ = gpu_y(m, x)
        yref, bound = O.matvec(m.widths, m.scales, m.codes, x, NTH)
        check(y, yref, bound, f"cfg2 {m.name} B={B}")


@pytest.mark.parametrize("B", [1, 2, 8, 16])
def test_config3_uniform_widths_full(B):
    for m in S.cfg3():
        x = S.make_x(3, "single", B, m.K)
        y, _ = gpu_y(m, x)
        yref, bound = O.matvec(m.widths, m.scales, m.codes, x, NTH)
        check(y, yref, bound, f"cfg3 {m.name} B={B}")


@pytest.mark.parametrize("k", [1, 2, 4, 8])
@pytest.mark.parametrize("B", [1, 4, 16])
def test_closed_form_all_max_codes(k, B):
    N, K = 4096, 4096
    m = S.Matrix("cf", N, K, np.full((N, K // 64), k, np.uint8), np.full((N, K // 64), 0x2E66, np.uint16),
                 np.full((N, K), (1 << k) - 1, np.uint8))
    x = S.x_normal(B, K, np.random.default_rng(k))
    y, _ = gpu_y(m, x)
    xs = torch.from_numpy(x.astype(np.int16)).view(torch.bfloat16).double().numpy()
    s0 = float(np.uint16(0x2E66).view(np.float16))
    want = (s0 * ((1 << k) - 1) / 2 * xs.sum(axis=1))[:, None] * np.ones((1, N))
    bound = (s0 * ((1 << k) - 1) / 2 * np.abs(xs).sum(axis=1))[:, None] * np.ones((1, N))
    check(y, want, bound, f"closed form k={k} B={B}")
    assert np.all(y == y[:, :1]), "all rows are identical, so their outputs must be bitwise equal"


@pytest.mark.parametrize("R", [256, 1024])
@pytest.mark.parametrize("B", vbq.BATCHES)
def test_config4_full_size_sampled_rows(B, R):
    g = np.random.default_rng(B)
    for m in S.cfg4(("q", "gate", "down")):
        x = S.make_x(4, m.name, B, m.K)
        y, _ = gpu_y(m, x, R)
        rows = np.unique(np.concatenate([g.choice(m.N, 200, replace=False), [0, m.N - 1, 1023, 1024]]))
        yref, bound = O.matvec(m.widths[rows], m.scales[rows], m.codes[rows], x, NTH)
        check(y[:, rows], yref, bound, f"cfg4 {m.name} B={B}")


@pytest.mark.parametrize("B", [1, 2, 8, 16])
def test_lm_head_sampled_rows(B):
    m = S.cfg5_head()
    x = S.make_x(5, "head", B, m.K)
    y, _ = gpu_y(m, x)
    rows = np.unique(np.concatenate([np.arange(0, 3000, 7), np.random.default_rng(0).choice(m.N, 300), [m.N - 1]]))
    yref, bound = O.matvec(m.widths[rows], m.scales[rows], m.codes[rows], x, NTH)
    check(y[:, rows], yref, bound, f"head B={B}")


@pytest.mark.parametrize("B", vbq.BATCHES)
def test_one_hot_columns_bit_exact(B):
    m = logical(5, 300, 256, (0.25, 0.25, 0.25, 0.25))
    deq = O.dequant(m.widths, m.scales, m.codes)
    cols = [0, 63, 64, 130, 255][:B] + [7] * max(0, B - 5)
    x = np.zeros((B, m.K), np.uint16)
    for b, i in enumerate(cols):
        x[b, i] = 0x3F80
    y, _ = gpu_y(m, x, R=64)
    for b, i in enumerate(cols):
        assert np.array_equal(y[b], deq[:, i]), f"B={B} column {i}"


@pytest.mark.parametrize("B", vbq.BATCHES)
def test_deterministic_across_runs(B):
    m = S.cfg4(("gate",))[0]
    x = S.make_x(4, "gate", B, m.K)
    y1, mat = gpu_y(m, x)
    y2, _ = gpu_y(m, x, mat=mat)
    assert np.array_equal(y1, y2)


def test_output_guard_regions_untouched():
    m = logical(9, 1030, 512, S.P_BASE)
    blob, _ = vbq.vbq_pack(m.N, m.K, 1024, m.widths, m.scales, m.codes)
    mat = vbq.DeviceMatrix(blob, dev())
    for B in vbq.BATCHES:
        pad = 4096
        buf = torch.full((B * m.N + 2 * pad,), 12345.0, dtype=torch.float32, device=dev())
        y = buf[pad:pad + B * m.N].view(B, m.N)
        x = to_dev_x(S.x_normal(B, m.K, np.random.default_rng(B)))
        vbq.vbq_gemm_skinny(mat.desc, mat.blob, x, B, y, mat.workspaces[B])
        torch.cuda.synchronize()
        assert torch.all(buf[:pad] == 12345.0) and torch.all(buf[pad + B * m.N:] == 12345.0)
        assert torch.isfinite(y).all()


def test_abi_rejects_bad_device_arguments():
    m = logical(11, 100, 256, S.P_BASE)
    blob, _ = vbq.vbq_pack(m.N, m.K, 16, m.widths, m.scales, m.codes)
    mat = vbq.DeviceMatrix(blob, dev())
    x = torch.zeros(m.K + 8, dtype=torch.bfloat16, device=dev())
    y = torch.zeros(m.N, dtype=torch.float32, device=dev())
    st = vbq.vbq_gemm_skinny_status(mat.desc, mat.blob, x[1:1 + m.K], 1, y, mat.workspaces[1])
    assert st == vbq.VBQ_ERR_ALIGN
    need = vbq.vbq_workspace_size(mat.desc, 1)
    if need > 0:
        small = torch.zeros(need - 16, dtype=torch.uint8, device=dev())
        st = vbq.vbq_gemm_skinny_status(mat.desc, mat.blob, x[:m.K], 1, y, small)
        assert st == vbq.VBQ_ERR_WORKSPACE
        assert vbq.vbq_gemm_skinny_status(mat.desc, mat.blob, x[:m.K], 1, y, None) == vbq.VBQ_ERR_WORKSPACE
    torch.cuda.synchronize()


def test_overlapped_launch_chain_matches_plain_launches():
    """VBQ_LAUNCH_OVERLAP (programmatic dependent launch) on a chain of launches on one stream gives bitwise the
    results of plain launches. The chain reuses one matrix, its workspace and its output twice in a row with
    different activations, and feeds a launch with activations that a torch kernel writes just before it; the
    same chain is also captured in a CUDA graph and replayed."""
    import torch
    q, gate = S.cfg4(("q",))[0], S.cfg4(("gate",))[0]
    mq = vbq.DeviceMatrix(vbq.vbq_pack(q.N, q.K, 256, q.widths, q.scales, q.codes)[0], dev(), max_batch=1)
    mg = vbq.DeviceMatrix(vbq.vbq_pack(gate.N, gate.K, 256, gate.widths, gate.scales, gate.codes)[0], dev(),
                          max_batch=1)
    xa, xb = (to_dev_x(S.x_normal(1, q.K, np.random.default_rng(s))) for s in (1, 2))
    x_src = to_dev_x(S.x_normal(1, gate.K, np.random.default_rng(3)))

    def chain(flags, x_c):
        ys = [torch.full((1, m.N), np.nan, dtype=torch.float32, device=dev()) for m in (q, q, gate)]
        vbq.vbq_gemm_skinny_ex(mq.desc, mq.blob, xa, 1, ys[0], mq.workspaces[1], flags)
        vbq.vbq_gemm_skinny_ex(mq.desc, mq.blob, xb, 1, ys[1], mq.workspaces[1], flags)
        x_c.copy_(x_src)  # a kernel writes the next launch's activations
        vbq.vbq_gemm_skinny_ex(mg.desc, mg.blob, x_c, 1, ys[2], mg.workspaces[1], flags)
        return ys

    x_c = torch.zeros_like(x_src)
    want = [y.cpu() for y in chain(0, x_c)]
    torch.cuda.synchronize()
    for rep in range(3):
        x_c.zero_()
        got = chain(vbq.VBQ_LAUNCH_OVERLAP, x_c)
        torch.cuda.synchronize()
        for k in range(3):
            assert torch.equal(got[k].cpu(), want[k]), f"eager overlapped chain, rep {rep}, launch {k}"
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        x_c.zero_()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            x_c.zero_()
            ys = chain(vbq.VBQ_LAUNCH_OVERLAP, x_c)
        for rep in range(3):
            g.replay()
        torch.cuda.synchronize()
    for k in range(3):
        assert torch.equal(ys[k].cpu(), want[k]), f"graph-replayed overlapped chain, launch {k}"
    for m in (mq, mg):
        need = vbq.vbq_workspace_size(m.desc, 1)
        assert int(m.workspaces[1][need - 4:need].cpu().numpy().view(np.uint32)[0]) == 0


def fused_status(fused, B):
    ws = fused.workspaces[B]
    need = vbq.vbq_workspace_size_multi(fused.descs, B)
    return int(ws[need - 4:need].cpu().numpy().view(np.uint32)[0])


@pytest.mark.parametrize("B", vbq.BATCHES)
def test_fused_launch_ragged_matrices_all_batches(B):
    """One vbq_gemm_skinny_multi launch over three matrices with the same K but different row counts (ragged
    last tiles) and width mixes, element by element against the oracle."""
    K = 256
    spec = [(1030, "base"), (100, "flat"), (2100, "all8")]
    ms = [logical(100 + i + B, N, K, DISTS[d]) for i, (N, d) in enumerate(spec)]
    mats = [vbq.DeviceMatrix(vbq.vbq_pack(m.N, K, 64, m.widths, m.scales, m.codes)[0], dev(), max_batch=B)
            for m in ms]
    fused = vbq.FusedMatrices(mats, max_batch=B)
    x = S.x_normal(B, K, np.random.default_rng(7 + B))
    ys = fused.matmul(to_dev_x(x))
    torch_sync()
    assert fused_status(fused, B) == 0
    for m, y in zip(ms, ys):
        yref, bound = O.matvec(m.widths, m.scales, m.codes, x, NTH)
        check(y.cpu().numpy().astype(np.float64), yref, bound, f"fused ragged N={m.N} B={B}")


@pytest.mark.parametrize("B", [1, 4, 16])
def test_fused_qkv_and_gate_up_full_size(B):
    """The 9B-shaped fused projections (q/k/v share x; gate/up share x) in one launch each: sampled rows against
    the oracle, and bitwise identical across two runs."""
    g = np.random.default_rng(B)
    for names in (("q", "k", "v"), ("gate", "up")):
        ms = S.cfg4(names)
        mats = [vbq.DeviceMatrix(vbq.vbq_pack(m.N, m.K, 256, m.widths, m.scales, m.codes)[0], dev(), max_batch=B)
                for m in ms]
        fused = vbq.FusedMatrices(mats, max_batch=B)
        x = S.make_x(4, names[0], B, ms[0].K)
        xd = to_dev_x(x)
        y1 = [y.cpu().numpy().astype(np.float64) for y in fused.matmul(xd)]
        y2 = [y.cpu().numpy().astype(np.float64) for y in fused.matmul(xd)]
        assert fused_status(fused, B) == 0
        for m, a, b in zip(ms, y1, y2):
            assert np.array_equal(a, b), f"{m.name} B={B}: fused launch not deterministic"
            rows = np.unique(np.concatenate([g.choice(m.N, 150, replace=False), [0, m.N - 1, 255, 256]]))
            yref, bound = O.matvec(m.widths[rows], m.scales[rows], m.codes[rows], x, NTH)
            check(a[:, rows], yref, bound, f"fused {'/'.join(names)}: {m.name} B={B}")


def torch_sync():
    import torch
    torch.cuda.synchronize()


def bf16_to_f64(t):
    import torch
    return t.float().cpu().numpy().astype(np.float64)


def check_swiglu(h, g_ref, u_ref, bg, bu, what):
    want = O.swiglu(g_ref, u_ref)
    bar = O.swiglu_bound(g_ref, u_ref, bg, bu)
    ok = np.abs(h - want) <= bar
    if not ok.all():
        i = tuple(np.argwhere(~ok)[0])
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} h out of bar; first {i}: got {h[i]!r} "
                             f"want {want[i]!r} bar {bar[i]!r}")


@pytest.mark.parametrize("B", vbq.BATCHES)
def test_swiglu_epilogue_ragged_all_batches(B):
    """vbq_gemm_swiglu on a ragged gate/up pair (1030 rows, 64-row tiles): y_gate and y_up against the oracle,
    and the fused h = silu(y_gate) * y_up (bf16) against the oracle's fp64 h within its bar."""
    N, K = 1030, 256
    g_m = logical(200 + B, N, K, DISTS["base"])
    u_m = logical(300 + B, N, K, DISTS["flat"])
    mats = [vbq.DeviceMatrix(vbq.vbq_pack(m.N, K, 64, m.widths, m.scales, m.codes)[0], dev(), max_batch=B)
            for m in (g_m, u_m)]
    fused = vbq.FusedMatrices(mats, max_batch=B)
    x = S.x_normal(B, K, np.random.default_rng(11 + B))
    yg, yu, h = fused.swiglu(to_dev_x(x))
    torch_sync()
    assert fused_status(fused, B) == 0
    g_ref, bg = O.matvec(g_m.widths, g_m.scales, g_m.codes, x, NTH)
    u_ref, bu = O.matvec(u_m.widths, u_m.scales, u_m.codes, x, NTH)
    check(yg.cpu().numpy().astype(np.float64), g_ref, bg, f"swiglu gate B={B}")
    check(yu.cpu().numpy().astype(np.float64), u_ref, bu, f"swiglu up B={B}")
    check_swiglu(bf16_to_f64(h), g_ref, u_ref, bg, bu, f"swiglu h B={B}")


@pytest.mark.parametrize("B", [1, 4, 16])
def test_swiglu_epilogue_full_size(B):
    """The 9B-shaped gate/up pair (14336x4096 each) with the fused epilogue: sampled rows of y and h against the
    oracle; h bitwise identical across runs and equal to silu(y_gate) * y_up from the same launch, rounded to
    bf16."""
    import torch
    ms = S.cfg4(("gate", "up"))
    mats = [vbq.DeviceMatrix(vbq.vbq_pack(m.N, m.K, 256, m.widths, m.scales, m.codes)[0], dev(), max_batch=B)
            for m in ms]
    fused = vbq.FusedMatrices(mats, max_batch=B)
    x = S.make_x(4, "gate", B, ms[0].K)
    xd = to_dev_x(x)
    yg, yu, h1 = fused.swiglu(xd)
    h1 = h1.clone()
    _, _, h2 = fused.swiglu(xd)
    torch_sync()
    assert fused_status(fused, B) == 0
    assert torch.equal(h1, h2), "SwiGLU output differs between runs"
    # h is silu of this launch's own y_gate times its y_up, rounded once to bf16
    g32, u32 = yg.double(), yu.double()
    h_from_y = (g32 / (1 + torch.exp(-g32)) * u32).float().to(torch.bfloat16)
    assert (h1.float() - h_from_y.float()).abs().max().item() <= 2 ** -7 * h_from_y.float().abs().max().item()
    rows = np.unique(np.concatenate([np.random.default_rng(B).choice(ms[0].N, 150, replace=False),
                                     [0, 255, 256, ms[0].N - 1]]))
    g_m, u_m = ms
    g_ref, bg = O.matvec(g_m.widths[rows], g_m.scales[rows], g_m.codes[rows], x, NTH)
    u_ref, bu = O.matvec(u_m.widths[rows], u_m.scales[rows], u_m.codes[rows], x, NTH)
    check_swiglu(bf16_to_f64(h1)[:, rows], g_ref, u_ref, bg, bu, f"swiglu full-size h B={B}")


@pytest.mark.parametrize("B", [1, 4, 16])
def test_recipe_workload_layers_and_head(B):
    """The fixed-recipe workload (uniform width per projection; first-block MLP 4-bit, the rest 2-bit; tiered
    head at 1.18 mean bits) through the fused launches: sampled rows against the oracle."""
    g = np.random.default_rng(50 + B)

    def sampled(m):
        return np.unique(np.concatenate([g.choice(m.N, 100, replace=False), [0, 255, 256, m.N - 1]]))

    for layer in (0, 1):
        ms = {m.name: m for m in S.cfg6_recipe_layer(layer)}
        for names in (("q", "k", "v"), ("gate", "up")):
            group = [ms[n] for n in names]
            mats = [vbq.DeviceMatrix(vbq.vbq_pack(m.N, m.K, 256, m.widths, m.scales, m.codes)[0], dev(),
                                     max_batch=B) for m in group]
            fused = vbq.FusedMatrices(mats, max_batch=B)
            x = S.make_x(6, names[0], B, group[0].K, layer=layer)
            ys = fused.matmul(to_dev_x(x))
            torch_sync()
            assert fused_status(fused, B) == 0
            for m, y in zip(group, ys):
                rows = sampled(m)
                yref, bound = O.matvec(m.widths[rows], m.scales[rows], m.codes[rows], x, NTH)
                check(y.cpu().numpy().astype(np.float64)[:, rows], yref, bound, f"recipe layer {layer} {m.name} B={B}")
    head = S.cfg6_recipe_head()
    x = S.make_x(6, "head", B, head.K)
    y, _ = gpu_y(head, x, 256)
    rows = np.unique(np.concatenate([np.arange(0, 4000, 9), g.choice(head.N, 200), [head.N - 1]]))
    yref, bound = O.matvec(head.widths[rows], head.scales[rows], head.codes[rows], x, NTH)
    check(y[:, rows], yref, bound, f"recipe head B={B}")


def sym_matrix(seed, N, K, p):
    """Random widths, scales and codes on Eq. 1's symmetric grid (codes in [0, 2^k - 2] for k >= 2)."""
    g = np.random.default_rng(seed)
    w = S.widths_iid(N, K // 64, p, g)
    codes = S.codes_uniform(w, g)
    top = np.repeat(np.where(w >= 2, (1 << w.astype(np.int64)) - 2, 1), 64, axis=1)
    codes = np.minimum(codes, top).astype(np.uint8)
    return S.Matrix("sym", N, K, w, S.scales_uniform(N, K // 64, g), codes)


@pytest.mark.parametrize("B", vbq.BATCHES)
def test_symmetric_grid_all_batches(B):
    """Blobs flagged with Eq. 1's symmetric grid (VBQ_FLAG_GRID_SYMMETRIC) through every batch path (CUDA cores
    at B <= 2, tensor cores at B = 4, 8, 16) against the oracle's flag-aware matvec; and one fused launch mixing a
    flagged and an unflagged matrix."""
    sym = vbq.VBQ_FLAG_GRID_SYMMETRIC
    for (N, K, R, dist) in ((1030, 256, 64, "flat"), (777, 2048, 256, "base"), (300, 512, 1024, "all8")):
        m = sym_matrix(N + K + B, N, K, DISTS[dist])
        blob, d = vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes, format_flags=sym)
        assert d.flags == sym
        mat = vbq.DeviceMatrix(blob, dev(), max_batch=B)
        x = S.x_normal(B, K, np.random.default_rng(B + N))
        y, _ = gpu_y(m, x, mat=mat)
        yref, bound = O.matvec(m.widths, m.scales, m.codes, x, NTH, flags=sym)
        check(y, yref, bound, f"symmetric grid {N}x{K} R={R} B={B}")
    a = sym_matrix(7 + B, 500, 256, DISTS["flat"])
    b = logical(8 + B, 900, 256, DISTS["flat"])
    ma = vbq.DeviceMatrix(vbq.vbq_pack(a.N, a.K, 64, a.widths, a.scales, a.codes, format_flags=sym)[0], dev(),
                          max_batch=B)
    mb = vbq.DeviceMatrix(vbq.vbq_pack(b.N, b.K, 64, b.widths, b.scales, b.codes)[0], dev(), max_batch=B)
    fused = vbq.FusedMatrices([ma, mb], max_batch=B)
    x = S.x_normal(B, 256, np.random.default_rng(99 + B))
    ya, yb = fused.matmul(to_dev_x(x))
    torch_sync()
    assert fused_status(fused, B) == 0
    ra, ba = O.matvec(a.widths, a.scales, a.codes, x, NTH, flags=sym)
    rb, bb = O.matvec(b.widths, b.scales, b.codes, x, NTH)
    check(ya.cpu().numpy().astype(np.float64), ra, ba, f"fused symmetric+default: symmetric B={B}")
    check(yb.cpu().numpy().astype(np.float64), rb, bb, f"fused symmetric+default: default B={B}")


@pytest.mark.parametrize("B", [1, 16])
def test_quantize_pack_gemv_pipeline(B):
    """Float weights -> vbq_quantize (Eq. 1 grid, and the default grid) -> vbq_pack_ex -> device GEMV, against the
    oracle's matvec on the same codes."""
    rng = np.random.default_rng(30 + B)
    N, K = 1100, 1024
    w = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    widths = S.widths_iid(N, K // 64, S.P_BASE, rng)
    x = S.x_normal(B, K, rng)
    for flags in (vbq.VBQ_FLAG_GRID_SYMMETRIC, 0):
        scales, codes = vbq.vbq_quantize(w, widths, flags)
        blob, _ = vbq.vbq_pack(N, K, 256, widths, scales, codes, format_flags=flags)
        mat = vbq.DeviceMatrix(blob, dev(), max_batch=B)
        m = S.Matrix("q", N, K, widths, scales, codes)
        y, _ = gpu_y(m, x, mat=mat)
        yref, bound = O.matvec(widths, scales, codes, x, NTH, flags=flags)
        check(y, yref, bound, f"quantize pipeline flags={flags} B={B}")


def test_decode_step_in_the_bench_launch_configuration():
    """Two layers of the 9B-shaped decode step (layer 0 at the first-block MLP mix, layer 1 at the base mix) and
    the LM head, packed with vbq.suggest_tile_rows and launched as the bench times them: fused q/k/v, o, fused
    gate/up whose SwiGLU epilogue writes down's input, down, then the head, chained by programmatic dependent
    launch inside one CUDA graph at batch 1. Sampled rows of every output against the oracle. Down reads the
    epilogue's bf16 h, so its bar adds the propagated h bar: with E = sum |w| bar_h and A = sum |w||h_ref|,
    |y - y_ref| <= 1e-3 (A + E) + 1e-6 + E. A second replay must reproduce every output bit for bit."""
    import torch
    d = dev()
    sms = torch.cuda.get_device_properties(d).multi_processor_count
    B, flags = 1, vbq.VBQ_LAUNCH_OVERLAP
    rng = np.random.default_rng(5)
    launches, checks = [], []

    def rows_of(N, R):
        extra = [r for r in (0, R - 1, R, N - 1) if 0 <= r < N]
        return np.unique(np.concatenate([rng.choice(N, 120, replace=False), extra]))

    def add_group(ms, x_bits, h=None, x_dev=None):
        R = vbq.suggest_tile_rows(sum(m.N for m in ms), ms[0].K, sms)
        mats = [vbq.DeviceMatrix(vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes)[0], d, max_batch=B)
                for m in ms]
        fused = vbq.FusedMatrices(mats, max_batch=B) if len(mats) > 1 else None
        xd = x_dev if x_dev is not None else to_dev_x(x_bits)
        ys = [torch.empty((B, m.N), dtype=torch.float32, device=d) for m in ms]

        def run(st):
            if h is not None:
                fused.swiglu(xd, ys, h, flags, st)
            elif fused is not None:
                fused.matmul(xd, ys, flags, st)
            else:
                vbq.vbq_gemm_skinny_ex(mats[0].desc, mats[0].blob, xd, B, ys[0], mats[0].workspaces[B], flags, st)

        def status():
            if fused is not None:
                return fused_status(fused, B)
            ws, need = mats[0].workspaces[B], vbq.vbq_workspace_size(mats[0].desc, B)
            return int(ws[need - 4:need].cpu().numpy().view(np.uint32)[0])

        launches.append((run, status))
        return R, ys

    for layer in (0, 1):
        ms = {m.name: m for m in S.cfg5_layer(layer)}
        for names in (("q", "k", "v"), ("o",)):
            x = S.make_x(5, names[0], B, 4096, layer=layer)
            R, ys = add_group([ms[n] for n in names], x)
            checks += [("plain", ms[n], x, R, y, f"layer {layer} {n}") for n, y in zip(names, ys)]
        h = torch.empty((B, ms["down"].K), dtype=torch.bfloat16, device=d)
        x = S.make_x(5, "gate", B, 4096, layer=layer)
        R, (yg, yu) = add_group([ms["gate"], ms["up"]], x, h=h)
        checks += [("plain", ms["gate"], x, R, yg, f"layer {layer} gate"),
                   ("plain", ms["up"], x, R, yu, f"layer {layer} up"),
                   ("down", (ms["gate"], ms["up"], ms["down"]), x, None, h, f"layer {layer} h and down")]
        R, (yd,) = add_group([ms["down"]], None, x_dev=h)
        checks[-1] = checks[-1][:3] + (R, (h, yd), checks[-1][5])
    head = S.cfg5_head()
    x = S.make_x(5, "head", B, 4096)
    R, (yh,) = add_group([head], x)
    checks.append(("plain", head, x, R, yh, "LM head"))

    st = torch.cuda.Stream(d)
    with torch.cuda.stream(st):
        for run, _ in launches:
            run(st)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            for run, _ in launches:
                run(st)
        g.replay()
        torch.cuda.synchronize()
        first = [c[4].clone() if c[0] == "plain" else (c[4][0].clone(), c[4][1].clone()) for c in checks]
        g.replay()
    torch.cuda.synchronize()
    for (_, status) in launches:
        assert status() == 0
    for c, f in zip(checks, first):
        if c[0] == "plain":
            assert torch.equal(c[4], f), f"{c[5]}: second replay differs"
        else:
            assert torch.equal(c[4][0], f[0]) and torch.equal(c[4][1], f[1]), f"{c[5]}: second replay differs"

    for kind, m, x, R, out, what in checks:
        if kind == "plain":
            rows = rows_of(m.N, R)
            yref, bound = O.matvec(m.widths[rows], m.scales[rows], m.codes[rows], x, NTH)
            check(out.cpu().numpy().astype(np.float64)[:, rows], yref, bound, what)
            continue
        g_m, u_m, d_m = m
        h, yd = out
        g_ref, bg = O.matvec(g_m.widths, g_m.scales, g_m.codes, x, NTH)
        u_ref, bu = O.matvec(u_m.widths, u_m.scales, u_m.codes, x, NTH)
        check_swiglu(bf16_to_f64(h), g_ref, u_ref, bg, bu, what + " (h)")
        h_ref, bar_h = O.swiglu(g_ref, u_ref)[0], O.swiglu_bound(g_ref, u_ref, bg, bu)[0]
        rows = rows_of(d_m.N, R)
        W = O.dequant(d_m.widths[rows], d_m.scales[rows], d_m.codes[rows])
        y_ref, A, E = W @ h_ref, np.abs(W) @ np.abs(h_ref), np.abs(W) @ bar_h
        got = yd.cpu().numpy().astype(np.float64)[0, rows]
        bad = np.abs(got - y_ref) > 1e-3 * (A + E) + 1e-6 + E
        assert not bad.any(), f"{what} (down): {int(bad.sum())} rows out of bar; first row {rows[bad][0]}"


@pytest.mark.parametrize("B", [1, 4, 16])
def test_zero_padded_mlp_matches_unpadded_and_oracle(B):
    """The 8960-wide MLP (gate/up 8960x1536, down 1536x8960) packed as is and zero-padded to 9216 (a multiple of
    512; VBQ paper, section 6, "Granularity is deployment-friendly"): in both forms gate/up with the fused SwiGLU
    epilogue, then down on h. h against the oracle within its bar, the padded h exactly 0 past row 8960, and the
    down output against the oracle's fp64 down projection of the oracle's h within the propagated bar."""
    gm, um, dm = S.cfg7_mlp()
    I, H, I_pad = gm.N, gm.K, 9216
    R = vbq.suggest_tile_rows(I, H, 148)
    x = S.make_x(7, "gate", B, H)
    g_ref, bg = O.matvec(gm.widths, gm.scales, gm.codes, x, NTH)
    u_ref, bu = O.matvec(um.widths, um.scales, um.codes, x, NTH)
    h_ref, bar_h = O.swiglu(g_ref, u_ref), O.swiglu_bound(g_ref, u_ref, bg, bu)
    W = O.dequant(dm.widths, dm.scales, dm.codes)
    y_ref, A, E = h_ref @ W.T, np.abs(h_ref) @ np.abs(W).T, bar_h @ np.abs(W).T
    for pad in (False, True):
        if pad:
            pk = [vbq.vbq_pack_padded(m.N, m.K, R, m.widths, m.scales, m.codes, I_pad, H)[0] for m in (gm, um)]
            pd = vbq.vbq_pack_padded(dm.N, dm.K, 256, dm.widths, dm.scales, dm.codes, H, I_pad)[0]
        else:
            pk = [vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes)[0] for m in (gm, um)]
            pd = vbq.vbq_pack(dm.N, dm.K, 256, dm.widths, dm.scales, dm.codes)[0]
        fused = vbq.FusedMatrices([vbq.DeviceMatrix(b, dev(), max_batch=B) for b in pk], max_batch=B)
        down = vbq.DeviceMatrix(pd, dev(), max_batch=B)
        _, _, h = fused.swiglu(to_dev_x(x))
        y = down.matmul(h)
        torch_sync()
        assert fused_status(fused, B) == 0
        hh = bf16_to_f64(h)
        what = f"{'padded' if pad else 'unpadded'} MLP B={B}"
        assert hh.shape == (B, I_pad if pad else I)
        if pad:
            assert not hh[:, I:].any(), f"{what}: padded rows of h are not 0"
        check_swiglu(hh[:, :I], g_ref, u_ref, bg, bu, what + " (h)")
        got = y.cpu().numpy().astype(np.float64)
        bad = np.abs(got - y_ref) > 1e-3 * (A + E) + 1e-6 + E
        assert not bad.any(), f"{what} (down): {int(bad.sum())} outputs out of bar"


def uneven(seed, N, K, heavy_rows, heavy_width=8):
    """Rows [0, heavy_rows) at heavy_width bits, the rest 1-bit: records of very different sizes, as in an LM head
    whose frequent rows are wider (VBQ paper, section 6: frequency-grouped row buckets), so that CTAs split the
    records by bytes."""
    g = np.random.default_rng(seed)
    w = np.ones((N, K // 64), np.uint8)
    w[:heavy_rows] = heavy_width
    return S.Matrix("uneven", N, K, w, S.scales_uniform(N, K // 64, g), S.codes_uniform(w, g))


@pytest.mark.parametrize("B", [1, 4, 16])
def test_byte_split_on_uneven_records(B):
    """Matrices whose records differ up to eightfold in size, so the launch splits them among CTAs by bytes: a
    ragged 3000-row matrix, one with fewer records than CTAs (CTAs that own nothing), and a fused launch of an
    all-8-bit matrix with an all-1-bit one. Every output against the oracle."""
    cases = [(uneven(1 + B, 3000, 512, 300), 64), (uneven(2 + B, 100, 2048, 10), 16),
             (uneven(3 + B, 40, 256, 7), 16)]
    for m, R in cases:
        mat = vbq.DeviceMatrix(vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes)[0], dev(), max_batch=B)
        x = S.x_normal(B, m.K, np.random.default_rng(m.N + B))
        y, _ = gpu_y(m, x, mat=mat)
        yref, bound = O.matvec(m.widths, m.scales, m.codes, x, NTH)
        check(y, yref, bound, f"uneven {m.N}x{m.K} R={R} B={B}")
    a, b = uneven(5 + B, 500, 512, 500), uneven(6 + B, 2000, 512, 0)
    mats = [vbq.DeviceMatrix(vbq.vbq_pack(m.N, m.K, 64, m.widths, m.scales, m.codes)[0], dev(), max_batch=B)
            for m in (a, b)]
    fused = vbq.FusedMatrices(mats, max_batch=B)
    x = S.x_normal(B, 512, np.random.default_rng(77 + B))
    ys = fused.matmul(to_dev_x(x))
    torch_sync()
    assert fused_status(fused, B) == 0
    for m, y in zip((a, b), ys):
        yref, bound = O.matvec(m.widths, m.scales, m.codes, x, NTH)
        check(y.cpu().numpy().astype(np.float64), yref, bound, f"fused uneven {m.N} B={B}")
