"""GPU test of the allocation-free entry point, vbq_gemm_skinny_noalloc (C ABI, through the Python binding).

Some callers cannot allocate device memory, for example plug-in hosts that own every device buffer and forbid
new allocations. For them the library keeps one fixed 16 MiB scratch buffer per device, instead of taking a
workspace. This test checks that the entry point gives the same results as vbq_gemm_skinny with its own
workspace, on two calls in a row, within the parity bar the other tests use:
|y_noalloc - y| <= 1e-3 * sum|w||x| + 1e-6. It also checks that a problem too large for the fixed buffer is
refused. The file is named so that pytest collects it last.
"""
import os

import numpy as np
import pytest
import torch

import vbq_synth as S
from decode_vbq_gemv_b200 import vbq
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


CASES = [
    ("gate 14336x4096", lambda: S.cfg4(("gate",))[0], 1),
    ("single 768x768", lambda: S.cfg1()[0], 16),
    ("ragged 1030x256", lambda: S.make_matrix(9, "single", 1030, 256, p=(0.25, 0.25, 0.25, 0.25)), 4),
]


@pytest.mark.parametrize("name,make,B", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_entry_point_twice(name, make, B):
    m = make()
    blob, _ = vbq.vbq_pack(m.N, m.K, vbq.DEFAULT_TILE_ROWS, m.widths, m.scales, m.codes)
    mat = vbq.DeviceMatrix(blob, dev(), max_batch=B)
    x = S.x_normal(B, m.K, np.random.default_rng(B))
    xd = torch.from_numpy(x.astype(np.int16)).view(torch.bfloat16).to(dev())
    y_ref = torch.empty((B, m.N), dtype=torch.float32, device=dev())
    vbq.vbq_gemm_skinny(mat.desc, mat.blob, xd, B, y_ref, mat.workspaces[B])
    torch.cuda.synchronize()
    y_ref = y_ref.cpu().numpy().astype(np.float64)
    _, bound = O.matvec(m.widths, m.scales, m.codes, x, os.cpu_count() or 1)
    for call in range(2):
        y = torch.full((B, m.N), float("nan"), dtype=torch.float32, device=dev())
        vbq.vbq_gemm_skinny_noalloc(mat.desc, mat.blob, xd, B, y)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64)
        ok = np.abs(got - y_ref) <= 1e-3 * bound + 1e-6
        assert ok.all(), f"{name} call {call}: {int((~ok).sum())} outputs differ from vbq_gemm_skinny"


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
