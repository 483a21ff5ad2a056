"""B200-native VBQ mixed-bit GEMV / skinny GEMM.

The work runs in ``libvbq.so`` (C++ packer and hand-written sm_100a CUDA kernels; C ABI in include/vbq.h).
``decode_vbq_gemv_b200.vbq`` is its Python binding: the functions have the same names as the C entry points.
"""
from .vbq import (BATCHES, DEFAULT_TILE_ROWS, VBQ_FLAG_GRID_SYMMETRIC, VBQ_LAUNCH_OVERLAP, DeviceMatrix, FusedMatrices, VbqError, vbq_desc,
                  vbq_describe, vbq_gemm_skinny, vbq_gemm_skinny_ex, vbq_gemm_skinny_multi, vbq_gemm_skinny_noalloc,
                  vbq_gemm_swiglu, vbq_workspace_size_swiglu,
                  vbq_gemv, vbq_pack, vbq_packed_size, vbq_quantize, vbq_strerror, vbq_unpack, vbq_version, vbq_workspace_init,
                  vbq_workspace_size, vbq_workspace_size_multi)

__all__ = ["BATCHES", "DEFAULT_TILE_ROWS", "VBQ_FLAG_GRID_SYMMETRIC", "VBQ_LAUNCH_OVERLAP", "DeviceMatrix", "FusedMatrices", "VbqError",
           "vbq_desc", "vbq_describe", "vbq_gemm_skinny", "vbq_gemm_skinny_ex", "vbq_gemm_skinny_multi",
           "vbq_gemm_skinny_noalloc", "vbq_gemm_swiglu", "vbq_workspace_size_swiglu", "vbq_gemv", "vbq_pack", "vbq_packed_size", "vbq_quantize", "vbq_strerror", "vbq_unpack",
           "vbq_version", "vbq_workspace_init", "vbq_workspace_size", "vbq_workspace_size_multi"]
