"""GPU tests of the failure-detection path, in the forms that fault no GPU.

The kernels check what they read before they use it and never trap: a record whose directory entry points past the
end of the records (status bit 1), or whose bucket counts disagree with its width codes (status bit 2), is refused
and the rest of the launch completes; a bounded wait that runs out (status bit 0) makes the CTA publish nothing and
return. The corruptions are made on the host in the bytes uploaded to the device, while the descriptor comes from
the clean blob (vbq_describe and vbq_unpack would refuse the corrupt one): a device copy that is not what its
descriptor promised.
A wait is made to run out by withholding one record's bulk copy (vbq_test_set_fault) with a 1 ms limit. After each
failure the same workspace, zeroed again by vbq_workspace_init, serves a clean call whose outputs match the oracle.
"""
import os
import zlib

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


def refresh_crcs(b):
    b = b.copy()
    total = int.from_bytes(b[48:56].tobytes(), "little")
    b[56:60] = np.frombuffer(zlib.crc32(b[64:total].tobytes()).to_bytes(4, "little"), np.uint8)
    b[60:64] = np.frombuffer(zlib.crc32(b[:60].tobytes()).to_bytes(4, "little"), np.uint8)
    return b


def case():
    m = S.make_matrix(12, "single", 700, 512, p=(0.4, 0.3, 0.2, 0.1))
    blob, d = vbq.vbq_pack(m.N, m.K, 256, m.widths, m.scales, m.codes)
    return m, blob, d


def run(blob, B, x, ws=None, device_bytes=None):
    """Launches blob (its device copy replaced by device_bytes if given) on x with workspace ws (a fresh, zeroed one
    if None); returns (y, status, workspace)."""
    d = vbq.vbq_describe(blob)
    up = blob if device_bytes is None else device_bytes
    assert up.size == blob.size
    blob_dev = torch.from_numpy(np.ascontiguousarray(up)).to(dev())
    need = vbq.vbq_workspace_size(d, B)
    if ws is None:
        ws = torch.zeros(need, dtype=torch.uint8, device=dev())
    xd = torch.from_numpy(x.astype(np.int16)).view(torch.bfloat16).to(dev())
    y = torch.zeros((B, d.N), dtype=torch.float32, device=dev())
    vbq.vbq_gemm_skinny(d, blob_dev, xd, B, y, ws)
    torch.cuda.synchronize()
    status = int(ws[need - 4:need].cpu().numpy().view(np.uint32)[0])
    return y, status, ws


def clean_call_after(ws, m, blob, B, x):
    vbq.vbq_workspace_init(ws)
    y, status, _ = run(blob, B, x, ws)
    assert status == 0
    yref, bound = O.matvec(m.widths, m.scales, m.codes, x, NTH)
    assert O.within_tolerance(y.cpu().numpy().astype(np.float64), yref, bound).all()


@pytest.mark.parametrize("B", [1, 4, 16])
def test_counts_that_disagree_with_width_codes_set_status_bit_2(B):
    m, blob, d = case()
    rec0 = int(d.rec_offset)
    bad = blob.copy()
    counts = bad[rec0:rec0 + 8].view(np.uint16).copy()
    assert counts[0] > 0 and counts.sum() == 256
    counts[0] -= 1      # one 1-bit group fewer, one 2-bit group more: still R_t groups, but not what the codes say
    counts[1] += 1
    bad[rec0:rec0 + 8] = counts.view(np.uint8)
    assert vbq.vbq_unpack_status(refresh_crcs(bad))[0] == vbq.VBQ_ERR_FORMAT   # the host validator refuses it
    x = S.x_normal(B, m.K, np.random.default_rng(B))
    _, status, ws = run(blob, B, x, device_bytes=bad)
    assert status == 4
    clean_call_after(ws, m, blob, B, x)


@pytest.mark.parametrize("B", [1, 4, 16])
def test_directory_entry_past_the_records_sets_status_bit_1(B):
    m, blob, d = case()
    bad = blob.copy()
    units = (int(d.total_bytes) - int(d.rec_offset)) // 16
    entry = int(d.dir_offset) + 4 * 3    # end of record 2 = start of record 3
    bad[entry:entry + 4] = np.frombuffer(np.uint32(units + 1).tobytes(), np.uint8)
    assert vbq.vbq_describe_status(refresh_crcs(bad))[0] == vbq.VBQ_ERR_FORMAT   # the host validator refuses it
    x = S.x_normal(B, m.K, np.random.default_rng(B))
    _, status, ws = run(blob, B, x, device_bytes=bad)
    assert status == 2
    clean_call_after(ws, m, blob, B, x)


@pytest.mark.parametrize("B", [1, 4, 16])
@pytest.mark.parametrize("record", [0, 5])
def test_a_wait_that_runs_out_sets_status_bit_0_and_the_kernel_returns(B, record):
    m, blob, d = case()
    x = S.x_normal(B, m.K, np.random.default_rng(B))
    try:
        vbq.vbq_test_set_fault(1_000_000, record)
        _, status, ws = run(blob, B, x)
    finally:
        vbq.vbq_test_set_fault(0, -1)
    assert status & 1 == 1 and status & ~1 == 0
    clean_call_after(ws, m, blob, B, x)
