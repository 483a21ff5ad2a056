"""Thin Python binding of libvbq (include/vbq.h): argument marshalling only.

Each ``vbq_*`` function here calls the C entry point of the same name. Host arrays are numpy arrays. Device
buffers and streams are torch CUDA tensors and streams, because PyTorch only provides device memory and streams.
All work runs inside libvbq: the packer in C++ and the products in the sm_100a CUDA kernels. Nothing falls back to
Python or to a CPU path. If the library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

VBQ_OK = 0
VBQ_ERR_NULL, VBQ_ERR_SHAPE, VBQ_ERR_WIDTH, VBQ_ERR_CODE_RANGE = -1, -2, -3, -4
VBQ_ERR_BUFFER_TOO_SMALL, VBQ_ERR_BAD_MAGIC, VBQ_ERR_VERSION, VBQ_ERR_CRC = -5, -6, -7, -8
VBQ_ERR_BATCH, VBQ_ERR_ALIGN, VBQ_ERR_CUDA, VBQ_ERR_TILE = -9, -10, -11, -12
VBQ_ERR_FORMAT, VBQ_ERR_WORKSPACE, VBQ_ERR_SCRATCH_LIMIT, VBQ_ERR_FLAGS, VBQ_ERR_VALUE = -13, -14, -15, -16, -17
VBQ_FLAG_GRID_SYMMETRIC = 1
VBQ_LAUNCH_OVERLAP = 1
BATCHES = (1, 2, 4, 8, 16)
DEFAULT_TILE_ROWS = 256


def suggest_tile_rows(rows: int, K: int, sms: int = 148) -> int:
    """Tile rows for packing a matrix (or the matrices of one fused launch, `rows` in total) on a GPU with `sms`
    SMs: the largest of 1024, 512 and 256 that still gives every SM at least 7 records (tile, group column).

    Larger tiles fill the width-bucket units better and cut per-record work; too few records per SM leave the
    CTAs' batches short. Graph-timed at batch 1 on B200, this picks the fastest size for each 9B-shaped launch:
    the lone 4096x4096 projection 256 rows (13.5 us; 128: 17.9, 512: 16.9), gate 14336x4096 512 (21.5 us; 256:
    26.3, 1024: 22.9), down 4096x14336 512 (23.7 us; 256: 26.1, 1024: 30.2), the LM head 1024 (30.0 us; 512:
    33.6) and fused gate/up 1024 (35.2 us; 512: 36.1)."""
    G = max(K // 64, 1)
    for R in (1024, 512, 256):
        if -(-rows // R) * G >= 7 * sms:
            return R
    return 256


class VbqError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {vbq_strerror(status)} (status {status})")
        self.status = status


class vbq_desc(ctypes.Structure):
    _fields_ = [("version", ctypes.c_uint32), ("flags", ctypes.c_uint32), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("G", ctypes.c_int64), ("R", ctypes.c_int64), ("T", ctypes.c_int64),
                ("dir_offset", ctypes.c_uint64), ("rec_offset", ctypes.c_uint64),
                ("total_bytes", ctypes.c_uint64), ("max_record_bytes", ctypes.c_uint64)]


class vbq_plan_info(ctypes.Structure):
    _fields_ = [("grid", ctypes.c_int32), ("threads", ctypes.c_int32), ("records_per_batch", ctypes.c_int32),
                ("batches_in_flight", ctypes.c_int32), ("result_sets", ctypes.c_int32), ("cost_split", ctypes.c_int32),
                ("smem_bytes", ctypes.c_uint32), ("workspace_bytes", ctypes.c_uint64)]


_lib = None


def library_path() -> str:
    return _build.LIB


def lib() -> ctypes.CDLL:
    """Loads libvbq.so, building it first if the sources are newer. Raises if it cannot be built or loaded."""
    global _lib
    if _lib is None:
        path = _build.build()
        if not os.path.exists(path):
            raise RuntimeError(f"libvbq.so missing at {path}")
        L = ctypes.CDLL(path)
        vp, i64, u64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int
        dp = ctypes.POINTER(vbq_desc)
        sig = {
            "vbq_strerror": (ctypes.c_char_p, [i32]),
            "vbq_version": (ctypes.c_uint32, []),
            "vbq_packed_size": (i32, [i64, i64, i64, vp, ctypes.POINTER(u64)]),
            "vbq_pack": (i32, [i64, i64, i64, vp, vp, vp, vp, u64, dp]),
            "vbq_pack_ex": (i32, [i64, i64, i64, vp, vp, vp, ctypes.c_uint, vp, u64, dp]),
            "vbq_quantize": (i32, [i64, i64, vp, vp, ctypes.c_uint, vp, vp]),
            "vbq_packed_size_padded": (i32, [i64, i64, i64, vp, i64, i64, ctypes.POINTER(u64)]),
            "vbq_pack_padded": (i32, [i64, i64, i64, vp, vp, vp, i64, i64, ctypes.c_uint, vp, u64, dp]),
            "vbq_describe": (i32, [vp, u64, dp]),
            "vbq_unpack": (i32, [vp, u64, vp, vp, vp]),
            "vbq_workspace_size": (i32, [dp, i32, ctypes.POINTER(u64)]),
            "vbq_plan_info_get": (i32, [i32, vp, i32, i32, ctypes.POINTER(vbq_plan_info)]),
            "vbq_workspace_init": (i32, [vp, u64, vp]),
            "vbq_gemv": (i32, [dp, vp, vp, vp, vp, u64, vp]),
            "vbq_gemm_skinny": (i32, [dp, vp, vp, i32, vp, vp, u64, vp]),
            "vbq_gemm_skinny_ex": (i32, [dp, vp, vp, i32, vp, vp, u64, ctypes.c_uint, vp]),
            "vbq_workspace_size_multi": (i32, [i32, vp, i32, ctypes.POINTER(u64)]),
            "vbq_gemm_skinny_multi": (i32, [i32, vp, vp, vp, i32, vp, vp, u64, ctypes.c_uint, vp]),
            "vbq_workspace_size_swiglu": (i32, [dp, dp, i32, ctypes.POINTER(u64)]),
            "vbq_gemm_swiglu": (i32, [dp, dp, vp, vp, vp, i32, vp, vp, vp, vp, u64, ctypes.c_uint, vp]),
            "vbq_gemm_skinny_noalloc": (i32, [dp, vp, vp, i32, vp, vp]),
            "vbq_noalloc_status": (i32, [vp, vp]),
            "vbq_test_set_fault": (i32, [u64, i64]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _np_ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dev_ptr(t) -> int:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream_ptr(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(st: int, where: str):
    if st != VBQ_OK:
        raise VbqError(st, where)


def vbq_strerror(status: int) -> str:
    return lib().vbq_strerror(status).decode()


def vbq_version() -> int:
    return int(lib().vbq_version())


def vbq_packed_size(N: int, K: int, R: int, widths: np.ndarray) -> int:
    w = np.ascontiguousarray(widths, np.uint8)
    out = ctypes.c_uint64()
    _check(lib().vbq_packed_size(N, K, R, _np_ptr(w), ctypes.byref(out)), "vbq_packed_size")
    return int(out.value)


def vbq_pack_status(N, K, R, widths, scales, codes, cap: int | None = None, format_flags: int = 0):
    """Returns (status, blob[uint8] or None, vbq_desc). format_flags: 0 or VBQ_FLAG_GRID_SYMMETRIC."""
    w = np.ascontiguousarray(widths, np.uint8)
    s = np.ascontiguousarray(scales, np.uint16)
    c = np.ascontiguousarray(codes, np.uint8)
    d = vbq_desc()
    if cap is None:
        out = ctypes.c_uint64()
        st = lib().vbq_packed_size(N, K, R, _np_ptr(w), ctypes.byref(out))
        if st != VBQ_OK:
            return st, None, d
        cap = int(out.value)
    blob = np.zeros(max(cap, 1), np.uint8)
    st = lib().vbq_pack_ex(N, K, R, _np_ptr(w), _np_ptr(s), _np_ptr(c), format_flags, _np_ptr(blob), cap,
                           ctypes.byref(d))
    return st, (blob[: d.total_bytes] if st == VBQ_OK else None), d


def vbq_pack(N: int, K: int, R: int, widths, scales, codes, format_flags: int = 0):
    """Packs a logical matrix (vbq_pack_ex). Returns (blob as uint8 numpy array, vbq_desc)."""
    st, blob, d = vbq_pack_status(N, K, R, widths, scales, codes, format_flags=format_flags)
    _check(st, "vbq_pack")
    return blob, d


def vbq_pack_padded_status(N, K, R, widths, scales, codes, N_pad, K_pad, format_flags: int = 0):
    """Returns (status, blob[uint8] or None, vbq_desc) of the N x K matrix packed as N_pad x K_pad with zero
    weights in the added rows and columns (vbq_pack_padded)."""
    w = np.ascontiguousarray(widths, np.uint8)
    s = np.ascontiguousarray(scales, np.uint16)
    c = np.ascontiguousarray(codes, np.uint8)
    d = vbq_desc()
    out = ctypes.c_uint64()
    st = lib().vbq_packed_size_padded(N, K, R, _np_ptr(w), N_pad, K_pad, ctypes.byref(out))
    if st != VBQ_OK:
        return st, None, d
    cap = int(out.value)
    blob = np.zeros(max(cap, 1), np.uint8)
    st = lib().vbq_pack_padded(N, K, R, _np_ptr(w), _np_ptr(s), _np_ptr(c), N_pad, K_pad, format_flags,
                               _np_ptr(blob), cap, ctypes.byref(d))
    return st, (blob[: d.total_bytes] if st == VBQ_OK else None), d


def vbq_pack_padded(N: int, K: int, R: int, widths, scales, codes, N_pad: int, K_pad: int, format_flags: int = 0):
    """Packs with zero padding to N_pad x K_pad (vbq_pack_padded). Returns (blob, vbq_desc)."""
    st, blob, d = vbq_pack_padded_status(N, K, R, widths, scales, codes, N_pad, K_pad, format_flags)
    _check(st, "vbq_pack_padded")
    return blob, d


def vbq_quantize_status(w, widths, format_flags: int = 0):
    """Returns (status, scales[N,G] fp16 bits or None, codes[N,K] or None) for float32 weights w[N,K]."""
    wf = np.ascontiguousarray(w, np.float32)
    wd = np.ascontiguousarray(widths, np.uint8)
    N, K = wf.shape
    scales = np.zeros((N, max(K // 64, 1)), np.uint16)
    codes = np.zeros((N, K), np.uint8)
    st = lib().vbq_quantize(N, K, _np_ptr(wf), _np_ptr(wd), format_flags, _np_ptr(scales), _np_ptr(codes))
    return st, (scales if st == VBQ_OK else None), (codes if st == VBQ_OK else None)


def vbq_quantize(w, widths, format_flags: int = 0):
    """Quantizes float32 weights w[N,K] for the given widths[N,G]. Returns (scales fp16 bits, codes)."""
    st, scales, codes = vbq_quantize_status(w, widths, format_flags)
    _check(st, "vbq_quantize")
    return scales, codes


def vbq_describe_status(blob: np.ndarray):
    b = np.ascontiguousarray(blob, np.uint8)
    d = vbq_desc()
    return lib().vbq_describe(_np_ptr(b), b.size, ctypes.byref(d)), d


def vbq_describe(blob: np.ndarray) -> vbq_desc:
    st, d = vbq_describe_status(blob)
    _check(st, "vbq_describe")
    return d


def vbq_unpack_status(blob: np.ndarray):
    b = np.ascontiguousarray(blob, np.uint8)
    st, d = vbq_describe_status(b)
    if st != VBQ_OK:
        return st, None
    widths = np.zeros((d.N, d.G), np.uint8)
    scales = np.zeros((d.N, d.G), np.uint16)
    codes = np.zeros((d.N, d.K), np.uint8)
    st = lib().vbq_unpack(_np_ptr(b), b.size, _np_ptr(widths), _np_ptr(scales), _np_ptr(codes))
    return st, ((widths, scales, codes) if st == VBQ_OK else None)


def vbq_unpack(blob: np.ndarray):
    """Returns (widths[N,G], scales[N,G] fp16 bits, codes[N,K])."""
    st, out = vbq_unpack_status(blob)
    _check(st, "vbq_unpack")
    return out


def vbq_plan_info_get(descs, B: int, sm_count: int = 148) -> dict:
    """The launch plan of a device call over the given descriptors (one, or the matrices of one fused launch) at
    batch B on a GPU with sm_count SMs (vbq_plan_info_get; host only, no GPU needed)."""
    ds = [descs] if isinstance(descs, vbq_desc) else list(descs)
    out = vbq_plan_info()
    _check(lib().vbq_plan_info_get(len(ds), _desc_array(ds), B, sm_count, ctypes.byref(out)), "vbq_plan_info_get")
    return {f: getattr(out, f) for f, _ in vbq_plan_info._fields_}


def vbq_workspace_size(desc: vbq_desc, B: int) -> int:
    out = ctypes.c_uint64()
    _check(lib().vbq_workspace_size(ctypes.byref(desc), B, ctypes.byref(out)), "vbq_workspace_size")
    return int(out.value)


def vbq_workspace_init(workspace, stream=None) -> None:
    if workspace is None or workspace.numel() == 0:
        return
    _check(lib().vbq_workspace_init(_dev_ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream_ptr(stream)), "vbq_workspace_init")


def vbq_gemm_skinny_status(desc, blob_dev, x_bf16, B, y, workspace=None, stream=None) -> int:
    ws_ptr = _dev_ptr(workspace) if workspace is not None and workspace.numel() > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return lib().vbq_gemm_skinny(ctypes.byref(desc), _dev_ptr(blob_dev), _dev_ptr(x_bf16), B, _dev_ptr(y),
                                 ws_ptr, ws_bytes, _stream_ptr(stream))


def vbq_gemm_skinny(desc, blob_dev, x_bf16, B, y, workspace=None, stream=None) -> None:
    """Y[B,N] = X[B,K] W^T on the device (asynchronous on `stream`, default: torch's current stream)."""
    _check(vbq_gemm_skinny_status(desc, blob_dev, x_bf16, B, y, workspace, stream), "vbq_gemm_skinny")


def vbq_gemm_skinny_ex_status(desc, blob_dev, x_bf16, B, y, workspace=None, flags=0, stream=None) -> int:
    ws_ptr = _dev_ptr(workspace) if workspace is not None and workspace.numel() > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return lib().vbq_gemm_skinny_ex(ctypes.byref(desc), _dev_ptr(blob_dev), _dev_ptr(x_bf16), B, _dev_ptr(y),
                                    ws_ptr, ws_bytes, flags, _stream_ptr(stream))


def vbq_gemm_skinny_ex(desc, blob_dev, x_bf16, B, y, workspace=None, flags=0, stream=None) -> None:
    """vbq_gemm_skinny with launch options; flags=VBQ_LAUNCH_OVERLAP enables programmatic dependent launch."""
    _check(vbq_gemm_skinny_ex_status(desc, blob_dev, x_bf16, B, y, workspace, flags, stream), "vbq_gemm_skinny_ex")


def _desc_array(descs):
    arr = (ctypes.POINTER(vbq_desc) * max(1, len(descs)))()
    for i, d in enumerate(descs):
        arr[i] = ctypes.pointer(d)
    return arr


def vbq_workspace_size_multi(descs, B: int) -> int:
    out = ctypes.c_uint64()
    _check(lib().vbq_workspace_size_multi(len(descs), _desc_array(descs), B, ctypes.byref(out)),
           "vbq_workspace_size_multi")
    return int(out.value)


def vbq_gemm_skinny_multi_status(descs, blobs_dev, x_bf16, B, ys, workspace=None, flags=0, stream=None) -> int:
    n = len(descs)
    blobs = (ctypes.c_void_p * max(1, n))(*[_dev_ptr(b) for b in blobs_dev])
    yv = (ctypes.c_void_p * max(1, n))(*[_dev_ptr(y) for y in ys])
    ws_ptr = _dev_ptr(workspace) if workspace is not None and workspace.numel() > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return lib().vbq_gemm_skinny_multi(n, _desc_array(descs), blobs, _dev_ptr(x_bf16), B, yv, ws_ptr, ws_bytes,
                                       flags, _stream_ptr(stream))


def vbq_gemm_skinny_multi(descs, blobs_dev, x_bf16, B, ys, workspace=None, flags=0, stream=None) -> None:
    """Fused launch over up to 4 matrices sharing x (same K and tile rows): ys[m][B, N_m] = X W_m^T."""
    _check(vbq_gemm_skinny_multi_status(descs, blobs_dev, x_bf16, B, ys, workspace, flags, stream),
           "vbq_gemm_skinny_multi")


def vbq_workspace_size_swiglu(gate: vbq_desc, up: vbq_desc, B: int) -> int:
    out = ctypes.c_uint64()
    _check(lib().vbq_workspace_size_swiglu(ctypes.byref(gate), ctypes.byref(up), B, ctypes.byref(out)),
           "vbq_workspace_size_swiglu")
    return int(out.value)


def vbq_gemm_swiglu_status(gate, up, blob_gate, blob_up, x_bf16, B, y_gate, y_up, h_bf16, workspace=None,
                           flags=0, stream=None) -> int:
    ws_ptr = _dev_ptr(workspace) if workspace is not None and workspace.numel() > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return lib().vbq_gemm_swiglu(ctypes.byref(gate), ctypes.byref(up), _dev_ptr(blob_gate), _dev_ptr(blob_up),
                                 _dev_ptr(x_bf16), B, _dev_ptr(y_gate), _dev_ptr(y_up), _dev_ptr(h_bf16), ws_ptr,
                                 ws_bytes, flags, _stream_ptr(stream))


def vbq_gemm_swiglu(gate, up, blob_gate, blob_up, x_bf16, B, y_gate, y_up, h_bf16, workspace=None, flags=0,
                    stream=None) -> None:
    """Gate/up projections with the fused SwiGLU epilogue: h = silu(X W_gate^T) * (X W_up^T), bf16."""
    _check(vbq_gemm_swiglu_status(gate, up, blob_gate, blob_up, x_bf16, B, y_gate, y_up, h_bf16, workspace,
                                  flags, stream), "vbq_gemm_swiglu")


def vbq_gemm_skinny_noalloc_status(desc, blob_dev, x_bf16, B, y, stream=None) -> int:
    """Allocation-free variant: the library's fixed 16 MiB device buffer replaces the workspace."""
    return lib().vbq_gemm_skinny_noalloc(ctypes.byref(desc), _dev_ptr(blob_dev), _dev_ptr(x_bf16), B,
                                         _dev_ptr(y), _stream_ptr(stream))


def vbq_gemm_skinny_noalloc(desc, blob_dev, x_bf16, B, y, stream=None) -> None:
    _check(vbq_gemm_skinny_noalloc_status(desc, blob_dev, x_bf16, B, y, stream), "vbq_gemm_skinny_noalloc")


def vbq_noalloc_status(stream=None) -> int:
    """Device status word of the last vbq_gemm_skinny_noalloc call on the current device (0: no device-side
    error). Enqueues the read on `stream` and synchronizes that stream."""
    import torch
    out = np.zeros(1, np.uint32)
    st = _stream_ptr(stream)
    _check(lib().vbq_noalloc_status(_np_ptr(out), st), "vbq_noalloc_status")
    (stream or torch.cuda.current_stream()).synchronize()
    return int(out[0])


def vbq_test_set_fault(wait_limit_ns: int = 0, withheld_record: int = -1) -> None:
    """Test hook of the failure-detection path: the kernels' wait limit and a record whose copy is withheld."""
    _check(lib().vbq_test_set_fault(wait_limit_ns, withheld_record), "vbq_test_set_fault")


def vbq_gemv(desc, blob_dev, x_bf16, y, workspace=None, stream=None) -> None:
    """y[N] = W x[K] on the device (batch 1)."""
    ws_ptr = _dev_ptr(workspace) if workspace is not None and workspace.numel() > 0 else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().vbq_gemv(ctypes.byref(desc), _dev_ptr(blob_dev), _dev_ptr(x_bf16), _dev_ptr(y), ws_ptr,
                          ws_bytes, _stream_ptr(stream)), "vbq_gemv")


class DeviceMatrix:
    """A packed VBQ matrix resident on one CUDA device, plus a workspace sized for the largest batch used.

    ``blob`` is a host numpy uint8 array (the canonical packed bytes). It is copied to the device once.
    """

    def __init__(self, blob: np.ndarray, device="cuda", max_batch: int = 16):
        import torch
        self.desc = vbq_describe(blob)
        self.N, self.K = int(self.desc.N), int(self.desc.K)
        self.device = torch.device(device)
        host = torch.from_numpy(np.ascontiguousarray(blob, np.uint8))
        self.blob = torch.empty(host.numel(), dtype=torch.uint8, device=self.device)
        self.blob.copy_(host)
        self.workspaces = {}
        for B in BATCHES:
            if B <= max_batch:
                self.workspaces[B] = self._alloc_ws(B)

    def _alloc_ws(self, B):
        import torch
        n = vbq_workspace_size(self.desc, B)
        ws = torch.zeros(max((n + 15) // 16, 1) * 16, dtype=torch.uint8, device=self.device)
        return ws

    @property
    def nbytes(self) -> int:
        return int(self.desc.total_bytes)

    def matmul(self, x_bf16, out=None, stream=None):
        """x_bf16: torch.bfloat16 [B, K] (or [K]) on the device. Returns fp32 [B, N] (or [N])."""
        import torch
        squeeze = x_bf16.dim() == 1
        x2 = x_bf16.reshape(-1, self.K)
        B = x2.shape[0]
        if out is None:
            out = torch.empty((B, self.N), dtype=torch.float32, device=self.device)
        ws = self.workspaces.get(B)
        if ws is None:
            ws = self.workspaces[B] = self._alloc_ws(B)
        vbq_gemm_skinny(self.desc, self.blob, x2, B, out, ws, stream)
        return out.reshape(self.N) if squeeze else out


class FusedMatrices:
    """Up to 4 DeviceMatrix objects that share their input (same K and tile rows), run as one launch
    (vbq_gemm_skinny_multi), plus a workspace per batch size for that launch."""

    def __init__(self, mats, max_batch: int = 16):
        import torch
        self.mats = list(mats)
        self.descs = [m.desc for m in self.mats]
        self.K = self.mats[0].K
        self.device = self.mats[0].device
        self.workspaces = {}
        for B in BATCHES:
            if B <= max_batch:
                n = vbq_workspace_size_multi(self.descs, B)
                self.workspaces[B] = torch.zeros(max((n + 15) // 16, 1) * 16, dtype=torch.uint8, device=self.device)

    @property
    def nbytes(self) -> int:
        return sum(m.nbytes for m in self.mats)

    def swiglu(self, x_bf16, outs=None, h=None, flags=0, stream=None):
        """Two matrices (gate, up) with the fused SwiGLU epilogue. Returns (y_gate, y_up, h bf16 [B, N])."""
        import torch
        x2 = x_bf16.reshape(-1, self.K)
        B = x2.shape[0]
        gate, up = self.mats
        if outs is None:
            outs = [torch.empty((B, m.N), dtype=torch.float32, device=self.device) for m in self.mats]
        if h is None:
            h = torch.empty((B, gate.N), dtype=torch.bfloat16, device=self.device)
        vbq_gemm_swiglu(gate.desc, up.desc, gate.blob, up.blob, x2, B, outs[0], outs[1], h, self.workspaces[B],
                        flags, stream)
        return outs[0], outs[1], h

    def matmul(self, x_bf16, outs=None, flags=0, stream=None):
        """x_bf16: torch.bfloat16 [B, K] on the device. Returns the list of fp32 [B, N_m] outputs."""
        import torch
        x2 = x_bf16.reshape(-1, self.K)
        B = x2.shape[0]
        if outs is None:
            outs = [torch.empty((B, m.N), dtype=torch.float32, device=self.device) for m in self.mats]
        vbq_gemm_skinny_multi(self.descs, [m.blob for m in self.mats], x2, B, outs, self.workspaces[B], flags,
                              stream)
        return outs
