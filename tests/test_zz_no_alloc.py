"""GPU tests of the allocation-free entry point, vbq_gemm_skinny_noalloc (C ABI, through the Python binding), and
of its status reader, vbq_noalloc_status.

Some callers cannot allocate device memory, for example plug-in hosts that own every device buffer and forbid new
allocations. For them the library keeps one fixed 16 MiB scratch buffer per device instead of taking a workspace.
The noalloc call runs the same kernel with the same launch plan as vbq_gemm_skinny, so its outputs must be bitwise
equal to the workspace path's; they are also checked against the fp64 oracle within the parity bar
|y - y_ref| <= 1e-3 * sum|w||x| + 1e-6. Calls of different shapes and batch sizes run back to back, so every call
must clear what the one before it left in the shared buffer. A call whose bounded wait runs out reports it through
vbq_noalloc_status. A problem too large for the buffer is refused. The file is named so that pytest collects it
last.
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


def x_dev(x):
    return torch.from_numpy(x.astype(np.int16)).view(torch.bfloat16).to(dev())


# back to back: large then small, batch up and down, a ragged last tile, the tensor-core batch among them
SEQUENCE = [
    ("gate 14336x4096", lambda: S.cfg4(("gate",))[0], 1, 256),
    ("single 768x768", lambda: S.cfg1()[0], 16, 256),
    ("ragged 1030x256", lambda: S.make_matrix(9, "single", 1030, 256, p=(0.25, 0.25, 0.25, 0.25)), 4, 64),
    ("gate 14336x4096", lambda: S.cfg4(("gate",))[0], 2, 1024),
    ("single 768x768", lambda: S.cfg1()[0], 1, 64),
]


def test_noalloc_sequence_matches_workspace_path_and_oracle():
    made = {}
    for name, make, B, R in SEQUENCE:
        if name not in made:
            made[name] = make()
        m = made[name]
        blob, _ = vbq.vbq_pack(m.N, m.K, R, m.widths, m.scales, m.codes)
        mat = vbq.DeviceMatrix(blob, dev(), max_batch=B)
        x = S.x_normal(B, m.K, np.random.default_rng(B + R))
        xd = x_dev(x)
        y_ws = torch.empty((B, m.N), dtype=torch.float32, device=dev())
        vbq.vbq_gemm_skinny(mat.desc, mat.blob, xd, B, y_ws, mat.workspaces[B])
        for call in range(2):
            y = torch.full((B, m.N), float("nan"), dtype=torch.float32, device=dev())
            vbq.vbq_gemm_skinny_noalloc(mat.desc, mat.blob, xd, B, y)
            assert vbq.vbq_noalloc_status() == 0, f"{name} B={B} call {call}: device status word"
            assert torch.equal(y, y_ws), f"{name} B={B} R={R} call {call}: differs from vbq_gemm_skinny"
        rows = np.arange(m.N) if m.N <= 2048 else np.unique(
            np.concatenate([np.random.default_rng(0).choice(m.N, 200, replace=False), [0, R - 1, R, m.N - 1]]))
        yref, bound = O.matvec(m.widths[rows], m.scales[rows], m.codes[rows], x, NTH)
        got = y.cpu().numpy().astype(np.float64)[:, rows]
        ok = O.within_tolerance(got, yref, bound)
        assert ok.all(), f"{name} B={B}: {int((~ok).sum())} outputs out of the oracle's bar"


@pytest.mark.parametrize("B", [1, 16])
def test_noalloc_status_reports_a_wait_that_ran_out(B):
    """With record 0's bulk copy withheld and a 1 ms wait limit (vbq_test_set_fault), the call returns, the kernel
    ends, and the status word read back through vbq_noalloc_status has bit 0 set; the next call, hook cleared,
    is clean and matches the workspace path."""
    m = S.make_matrix(11, "single", 1000, 512, p=S.P_BASE)
    blob, _ = vbq.vbq_pack(m.N, m.K, 256, m.widths, m.scales, m.codes)
    mat = vbq.DeviceMatrix(blob, dev(), max_batch=B)
    xd = x_dev(S.x_normal(B, m.K, np.random.default_rng(3)))
    y = torch.zeros((B, m.N), dtype=torch.float32, device=dev())
    try:
        vbq.vbq_test_set_fault(1_000_000, 0)
        vbq.vbq_gemm_skinny_noalloc(mat.desc, mat.blob, xd, B, y)
        torch.cuda.synchronize()
        assert vbq.vbq_noalloc_status() & 1 == 1
    finally:
        vbq.vbq_test_set_fault(0, -1)
    vbq.vbq_gemm_skinny_noalloc(mat.desc, mat.blob, xd, B, y)
    assert vbq.vbq_noalloc_status() == 0
    y_ws = torch.empty_like(y)
    vbq.vbq_gemm_skinny(mat.desc, mat.blob, xd, B, y_ws, mat.workspaces[B])
    torch.cuda.synchronize()
    assert torch.equal(y, y_ws)


def test_noalloc_rejects_problems_above_its_fixed_buffer():
    N, K, B = 200_000, 64, 16
    w = np.ones((N, 1), np.uint8)
    s = np.full((N, 1), 0x3C00, np.uint16)
    c = np.zeros((N, K), np.uint8)
    blob, desc = vbq.vbq_pack(N, K, 1024, w, s, c)
    assert vbq.vbq_workspace_size(desc, B) > 16 << 20
    blob_dev = torch.from_numpy(blob).to(dev())
    x = torch.zeros((B, K), dtype=torch.bfloat16, device=dev())
    y = torch.zeros((B, N), dtype=torch.float32, device=dev())
    st = vbq.vbq_gemm_skinny_noalloc_status(desc, blob_dev, x, B, y)
    assert st == vbq.VBQ_ERR_SCRATCH_LIMIT
    assert "16 MiB" in vbq.vbq_strerror(st)
    torch.cuda.synchronize()
