// Device side of libvbq: fused dequantize-and-multiply GEMV and skinny GEMM over format-v1 VBQ blobs.
//
// What is computed (VBQ paper, "Variable Bit-width Quantization", section 3.1 and section 6, paragraph
// "Fused kernels over packed weights"): y[b][r] = sum_g s[r][g] * sum_i (q[r][64g+i] - (2^k-1)/2) * x[b][64g+i].
// The low-bit codes are expanded in registers. The dense matrix never exists in memory.
//
// Work decomposition (B200, sm_100a):
//  - The blob stores one record per (row tile, group column). Inside a record the tile's groups sit in four
//    width buckets (1, 2, 4, 8 bits), each in ascending row order (FORMAT.md).
//  - A CTA owns one row tile and a contiguous range of group columns (split-K across CTAs). Its partial
//    outputs go to a workspace. The last CTA of a tile to arrive (one atomic ticket, no waiting) adds the
//    partials in a fixed order. The result is deterministic.
//  - For each record, the CTA rebuilds the item -> row map from the 2-bit width codes (block-wide scan).
//    Warps then take "units" of 32 items of one bucket, so every warp instruction runs a single width.
//    This is the width-bucketed schedule: 1-bit groups never share a warp instruction with 8-bit groups.
//  - Batch 1: a lane owns one group (64 weights). It keeps the column's 64 activations in registers
//    (all lanes of the warp share the column). 1-bit groups use predicated adds of the activations whose bit
//    is set. 2/4-bit groups use a magic-number bit-to-float expansion with pre-scaled activations, and 8-bit
//    groups use byte permutes.
//  - Batch 2/4: same schedule. Activations for all batches are read from shared memory by broadcast.
//  - Batch 8/16: each lane dequantizes its group to exact bf16 integers 2q-(2^k-1) in shared memory. The warp
//    then runs mma.sync m16n8k16 (bf16 in, fp32 accumulate) against the activations and applies s/2 per row.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "vbq.h"

namespace vbq {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxTileRows = 1024;
constexpr int kAStride = 72;  // bf16 elements per staged A row (64 + 8 pad: ldmatrix rows hit distinct banks)

struct Params {
  const uint32_t* dir;     // record directory, 16-byte units from recs
  const uint8_t* recs;     // first record
  const uint16_t* x;       // bf16 bits, [B][K]
  float* y;                // [B][N]
  float* partial;          // [T][S][R][B] split-K partial sums
  unsigned* counters;      // [T] arrival tickets, zero between calls
  int N, K, G, R, T;
  int S;                   // column splits per tile (grid.x)
  int C;                   // group columns per split
};

__host__ __device__ constexpr int align16i(int v) { return (v + 15) & ~15; }

// ------------------------------------------------------------------------------------------ small helpers
__device__ __forceinline__ uint2 ld_stream2(const void* p) {
  uint2 v;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_stream4(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ float ld_scale(const uint8_t* p) {
  unsigned short h;
  asm("ld.global.nc.u16 %0, [%1];" : "=h"(h) : "l"(p));
  return __half2float(__ushort_as_half(h));
}

// d = a * b + c on two fp32 lanes at once (sm_100 packed FMA).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Bit position of code t inside its 32-bit source for the magic-number expansion: the code's bits must lie in
// [0, 23) so that OR-ing them into the mantissa of 2^23 gives exactly 2^23 + q * 2^shift. High codes are
// read from (word >> HI) instead of word.
template <int KB> struct Magic;
template <> struct Magic<2> { static constexpr int HI = 10; };
template <> struct Magic<4> { static constexpr int HI = 12; };
template <int KB> __host__ __device__ constexpr bool magic_hi(int t) { return KB * t + KB > 23; }
template <int KB> __host__ __device__ constexpr int magic_shift(int t) {
  return magic_hi<KB>(t) ? KB * t - Magic<KB>::HI : KB * t;
}
// Shift of code i (0..63) of a KB-bit group: code i is code t = i % (32/KB) of word i / (32/KB).
template <int KB> __host__ __device__ constexpr int code_shift(int i) { return magic_shift<KB>(i % (32 / KB)); }

__device__ __forceinline__ float magic_f(uint32_t src, uint32_t mask_shifted) {
  return __uint_as_float((src & mask_shifted) | 0x4B000000u);
}

// ---------------------------------------------------------------------------------- batch-1 inner loops
// Each returns sum_i (q_i - (2^k-1)/2) x_i for one 64-weight group; sg = sum_i x_i.

// 1-bit: sum of the activations whose bit is set, minus half the group sum.
__device__ __forceinline__ float dot_b1(uint2 w, const float (&xr)[64], float sg) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    if (w.x & (1u << i)) a0 += xr[i];
    if (w.x & (1u << (i + 1))) a1 += xr[i + 1];
    if (w.x & (1u << (i + 2))) a2 += xr[i + 2];
    if (w.x & (1u << (i + 3))) a3 += xr[i + 3];
  }
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    if (w.y & (1u << i)) a0 += xr[32 + i];
    if (w.y & (1u << (i + 1))) a1 += xr[33 + i];
    if (w.y & (1u << (i + 2))) a2 += xr[34 + i];
    if (w.y & (1u << (i + 3))) a3 += xr[35 + i];
  }
  return ((a0 + a1) + (a2 + a3)) - 0.5f * sg;
}

// 2- and 4-bit: xs holds x_i * 2^-shift(i). v - 2^23 = q * 2^shift exactly, so (v - 2^23) * xs_i = q * x_i.
template <int KB>
__device__ __forceinline__ float dot_magic(const uint32_t (&w)[2 * KB], const float (&xr)[64], float sg) {
  constexpr int CPW = 32 / KB;
  constexpr uint32_t M = (1u << KB) - 1u;
  const float2 neg = make_float2(-8388608.f, -8388608.f);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int m = 0; m < 2 * KB; ++m) {
    const uint32_t lo = w[m], hi = w[m] >> Magic<KB>::HI;
#pragma unroll
    for (int t = 0; t < CPW; t += 2) {
      const float va = magic_f(magic_hi<KB>(t) ? hi : lo, M << magic_shift<KB>(t));
      const float vb = magic_f(magic_hi<KB>(t + 1) ? hi : lo, M << magic_shift<KB>(t + 1));
      const float2 q = fadd2(make_float2(va, vb), neg);
      const int i = m * CPW + t;
      if ((t >> 1) & 1) acc1 = ffma2(q, make_float2(xr[i], xr[i + 1]), acc1);
      else acc0 = ffma2(q, make_float2(xr[i], xr[i + 1]), acc0);
    }
  }
  // sum q x - (2^(k-1) - 1/2) * sum x
  return ((acc0.x + acc0.y) + (acc1.x + acc1.y)) - (float((1 << (KB - 1))) - 0.5f) * sg;
}

// 8-bit: byte permute places q in the low mantissa byte of 2^23; subtracting 2^23 + 128 gives q - 128 exactly.
__device__ __forceinline__ float dot_b8(const uint32_t (&w)[16], const float (&xr)[64], float sg) {
  const float2 neg = make_float2(-8388736.f, -8388736.f);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const float2 q0 = fadd2(make_float2(__uint_as_float(__byte_perm(w[m], 0x4B000000u, 0x7440u)),
                                        __uint_as_float(__byte_perm(w[m], 0x4B000000u, 0x7441u))), neg);
    const float2 q1 = fadd2(make_float2(__uint_as_float(__byte_perm(w[m], 0x4B000000u, 0x7442u)),
                                        __uint_as_float(__byte_perm(w[m], 0x4B000000u, 0x7443u))), neg);
    acc0 = ffma2(q0, make_float2(xr[4 * m], xr[4 * m + 1]), acc0);
    acc1 = ffma2(q1, make_float2(xr[4 * m + 2], xr[4 * m + 3]), acc1);
  }
  return ((acc0.x + acc0.y) + (acc1.x + acc1.y)) + 0.5f * sg;
}

// --------------------------------------------------------------------------------------- generic decode
// q - 2^(k-1) of code i from a group's code words, as an exact float (any width, runtime index).
__device__ __forceinline__ float code_minus_half_range(const uint32_t* w, int k, int i) {
  const int bit = k * i;
  const uint32_t q = (w[bit >> 5] >> (bit & 31)) & ((1u << k) - 1u);
  return float(int(q) - (1 << (k - 1)));
}

// ------------------------------------------------------------------------------------- shared layout
template <int B>
struct Smem {
  // Offsets in bytes inside dynamic shared memory.
  static __host__ __device__ int ys(int) { return 0; }
  static __host__ __device__ int xs(int R) { return align16i(R * B * 4); }
  static __host__ __device__ int xcopies() { return B == 1 ? 3 : 1; }
  static __host__ __device__ int sg(int R, int C) { return xs(R) + (B >= 8 ? 0 : C * xcopies() * 64 * B * 4); }
  static __host__ __device__ int rows(int R, int C) { return sg(R, C) + (B >= 8 ? 0 : align16i(C * B * 4)); }
  static __host__ __device__ int astage(int R, int C) { return rows(R, C) + align16i(R * 2); }
  static __host__ __device__ int bytes(int R, int C) {
    return astage(R, C) + (B >= 8 ? kWarps * 32 * kAStride * 2 : 0);
  }
};

// Block-wide rebuild of rowlist[item] = row (within tile) for one record. Row j's 2-bit width code is bits
// 2(j%4) of byte j/4 of the width-code section. Thread tid handles rows 4*tid .. 4*tid+3.
__device__ __forceinline__ void build_rowlist(const uint8_t* rec, int Rt, int n1, int n2, int n4,
                                              uint16_t* rowlist, unsigned long long* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nrows = max(0, min(4, Rt - 4 * tid));
  uint32_t byte = 0;
  unsigned long long mine = 0;
  if (nrows > 0) {
    byte = rec[8 + tid];
    for (int jj = 0; jj < nrows; ++jj) mine += 1ull << (16 * ((byte >> (2 * jj)) & 3u));
  }
  unsigned long long incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  unsigned long long run = incl - mine;
  for (int w = 0; w < warp; ++w) run += warp_tot[w];
  const int base[4] = {0, n1, n1 + n2, n1 + n2 + n4};
  for (int jj = 0; jj < nrows; ++jj) {
    const int c = (byte >> (2 * jj)) & 3;
    rowlist[base[c] + int((run >> (16 * c)) & 0xFFFFull)] = uint16_t(4 * tid + jj);
    run += 1ull << (16 * c);
  }
}

struct RecordView {
  const uint8_t* rec;
  int n[4];
  int item0[4];          // first item index of each bucket
  const uint8_t* code[4];  // first code byte of each bucket
  const uint8_t* scale;    // fp16 scales in item order
  int units[4];          // units (32 items) per bucket
  int U;
};

__device__ __forceinline__ RecordView view_record(const Params& p, int t, int g, int Rt) {
  RecordView v;
  v.rec = p.recs + 16ull * p.dir[size_t(t) * p.G + g];
  const uint2 cnt = *reinterpret_cast<const uint2*>(v.rec);
  v.n[0] = cnt.x & 0xFFFF; v.n[1] = cnt.x >> 16; v.n[2] = cnt.y & 0xFFFF; v.n[3] = cnt.y >> 16;
  const int sc_off = align16i(8 + 4 * ((Rt + 15) / 16));
  const int cd_off = sc_off + align16i(2 * Rt);
  v.scale = v.rec + sc_off;
  v.code[0] = v.rec + cd_off;
  v.code[1] = v.code[0] + align16i(8 * v.n[0]);
  v.code[2] = v.code[1] + 16 * v.n[1];
  v.code[3] = v.code[2] + 32 * v.n[2];
  v.item0[0] = 0; v.item0[1] = v.n[0]; v.item0[2] = v.n[0] + v.n[1]; v.item0[3] = v.item0[2] + v.n[2];
  v.U = 0;
  for (int c = 0; c < 4; ++c) { v.units[c] = (v.n[c] + 31) >> 5; v.U += v.units[c]; }
  return v;
}

// Maps unit u (warp-uniform) to (bucket c, first item j0 of the unit within the bucket).
__device__ __forceinline__ int unit_bucket(const RecordView& v, int u, int& j0) {
  int c = 0, base = 0;
  while (c < 3 && u >= base + v.units[c]) { base += v.units[c]; ++c; }
  j0 = (u - base) << 5;
  return c;
}

// ----------------------------------------------------------------------------------------------- kernel
template <int B>
__global__ void __launch_bounds__(kThreads, 2) vbq_kernel(Params p) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ unsigned long long warp_tot[kWarps];
  __shared__ int last_flag;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t = blockIdx.y, s = blockIdx.x;
  const int g0 = s * p.C, g1 = min(p.G, g0 + p.C), ncols = g1 - g0;
  const int Rt = min(p.R, p.N - t * p.R);

  float* ys = reinterpret_cast<float*>(smem + Smem<B>::ys(p.R));
  float* xs = reinterpret_cast<float*>(smem + Smem<B>::xs(p.R));
  float* sgs = reinterpret_cast<float*>(smem + Smem<B>::sg(p.R, p.C));
  uint16_t* rowlist = reinterpret_cast<uint16_t*>(smem + Smem<B>::rows(p.R, p.C));

  for (int i = tid; i < Rt * B; i += kThreads) ys[i] = 0.f;

  // Stage activations of this CTA's columns as fp32 (bf16 -> fp32 is exact).
  // B == 1: three copies per column: raw, scaled for the 2-bit magic shifts, scaled for the 4-bit ones.
  // B >= 2: one copy, layout [column][i][b].
  if constexpr (B < 8) {
    for (int e = tid; e < ncols * 64 * B; e += kThreads) {
      const int b = e / (ncols * 64), rem = e - b * ncols * 64, c = rem >> 6, i = rem & 63;
      const float xv = __uint_as_float(uint32_t(p.x[size_t(b) * p.K + size_t(g0 + c) * 64 + i]) << 16);
      if (B == 1) {
        float* col = xs + c * 3 * 64;
        col[i] = xv;
        col[64 + i] = xv * __uint_as_float(uint32_t(127 - code_shift<2>(i)) << 23);
        col[128 + i] = xv * __uint_as_float(uint32_t(127 - code_shift<4>(i)) << 23);
      } else {
        xs[(c * 64 + i) * B + b] = xv;
      }
    }
    __syncthreads();
    // Group sums S[c][b] = sum_i x_b[64(g0+c) + i], one warp per (c, b), fixed reduction order.
    for (int pr = warp; pr < ncols * B; pr += kWarps) {
      const int c = pr / B, b = pr - c * B;
      float v;
      if (B == 1) v = xs[c * 192 + lane] + xs[c * 192 + 32 + lane];
      else v = xs[(c * 64 + lane) * B + b] + xs[(c * 64 + 32 + lane) * B + b];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
      if (lane == 0) sgs[c * B + b] = v;
    }
  }
  __syncthreads();

  for (int g = g0; g < g1; ++g) {
    const RecordView v = view_record(p, t, g, Rt);
    build_rowlist(v.rec, Rt, v.n[0], v.n[1], v.n[2], rowlist, warp_tot);
    __syncthreads();
    const int c = g - g0;

    if constexpr (B == 1) {
      // Units in bucket order; warp w takes a contiguous run of units so it switches width rarely.
      const int per = (v.U + kWarps - 1) / kWarps;
      const int ub = warp * per, ue = min(v.U, ub + per);
      int loaded = -1;
      float xr[64];
      const float sg = sgs[c];
      for (int u = ub; u < ue; ++u) {
        int j0;
        const int bk = unit_bucket(v, u, j0);
        const int copy = bk == 1 ? 1 : (bk == 2 ? 2 : 0);
        if (copy != loaded) {
          const float4* src = reinterpret_cast<const float4*>(xs + c * 192 + copy * 64);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float4 f = src[q];
            xr[4 * q] = f.x; xr[4 * q + 1] = f.y; xr[4 * q + 2] = f.z; xr[4 * q + 3] = f.w;
          }
          loaded = copy;
        }
        const int j = j0 + lane;
        if (j < v.n[bk]) {
          const int item = v.item0[bk] + j;
          float d;
          if (bk == 0) {
            d = dot_b1(ld_stream2(v.code[0] + 8 * j), xr, sg);
          } else if (bk == 1) {
            uint32_t w[4];
            const uint4 a = ld_stream4(v.code[1] + 16 * j);
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
            d = dot_magic<2>(w, xr, sg);
          } else if (bk == 2) {
            uint32_t w[8];
            const uint4 a = ld_stream4(v.code[2] + 32 * j), b2 = ld_stream4(v.code[2] + 32 * j + 16);
            w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b2.x; w[5] = b2.y; w[6] = b2.z; w[7] = b2.w;
            d = dot_magic<4>(w, xr, sg);
          } else {
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 a = ld_stream4(v.code[3] + 64 * j + 16 * q);
              w[4 * q] = a.x; w[4 * q + 1] = a.y; w[4 * q + 2] = a.z; w[4 * q + 3] = a.w;
            }
            d = dot_b8(w, xr, sg);
          }
          const float sc = ld_scale(v.scale + 2 * item);
          const int row = rowlist[item];
          ys[row] = fmaf(sc, d, ys[row]);
        }
      }
    } else if constexpr (B < 8) {
      // CUDA cores, B in {2, 4}: lane = group, activations of all batches read by broadcast from shared.
      const float* xc = xs + c * 64 * B;
      for (int u = warp; u < v.U; u += kWarps) {
        int j0;
        const int bk = unit_bucket(v, u, j0);
        const int j = j0 + lane;
        if (j >= v.n[bk]) continue;
        const int item = v.item0[bk] + j;
        const int k = 1 << bk;
        uint32_t w[16];
        const uint8_t* cp = v.code[bk] + size_t(8 * k) * j;
        if (bk == 0) {
          const uint2 a = ld_stream2(cp);
          w[0] = a.x; w[1] = a.y;
        } else {
          for (int q = 0; q < k / 2; ++q) {
            const uint4 a = ld_stream4(cp + 16 * q);
            w[4 * q] = a.x; w[4 * q + 1] = a.y; w[4 * q + 2] = a.z; w[4 * q + 3] = a.w;
          }
        }
        float acc[B];
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = 0.f;
        if (bk == 0) {
#pragma unroll 8
          for (int i = 0; i < 64; ++i) {
            if (w[i >> 5] & (1u << (i & 31))) {
#pragma unroll
              for (int b = 0; b < B; ++b) acc[b] += xc[i * B + b];
            }
          }
        } else {
#pragma unroll 4
          for (int i = 0; i < 64; ++i) {
            const float qv = code_minus_half_range(w, k, i);
#pragma unroll
            for (int b = 0; b < B; ++b) acc[b] = fmaf(qv, xc[i * B + b], acc[b]);
          }
        }
        const float sc = ld_scale(v.scale + 2 * item);
        const int row = rowlist[item];
        // sum (q - 2^(k-1)) x + 1/2 sum x  ==  sum (q - (2^k-1)/2) x; for k = 1 the first sum is sum_{q=1} x - S.
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float S = sgs[c * B + b];
          const float d = (bk == 0) ? acc[b] - 0.5f * S : acc[b] + 0.5f * S;
          ys[row * B + b] = fmaf(sc, d, ys[row * B + b]);
        }
      }
    } else {
      // Tensor cores, B in {8, 16}. Lane = group: dequantize to bf16 2q-(2^k-1) into this warp's A stage,
      // then two m16 tiles per unit through mma.sync m16n8k16 against x (bf16) of this column.
      constexpr int NT = B >= 8 ? B / 8 : 1;
      __nv_bfloat16* As = reinterpret_cast<__nv_bfloat16*>(smem + Smem<B>::astage(p.R, p.C)) + warp * 32 * kAStride;
      uint32_t bfr[4][NT][2];
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int n = nt * 8 + (lane >> 2);
          const uint16_t* xp = p.x + size_t(n) * p.K + size_t(g) * 64 + 16 * ks + 2 * (lane & 3);
          bfr[ks][nt][0] = *reinterpret_cast<const uint32_t*>(xp);
          bfr[ks][nt][1] = *reinterpret_cast<const uint32_t*>(xp + 8);
        }
      for (int u = warp; u < v.U; u += kWarps) {
        int j0;
        const int bk = unit_bucket(v, u, j0);
        const int k = 1 << bk;
        const int j = j0 + lane;
        const bool valid = j < v.n[bk];
        __nv_bfloat162* arow = reinterpret_cast<__nv_bfloat162*>(As + lane * kAStride);
        if (valid) {
          uint32_t w[16];
          const uint8_t* cp = v.code[bk] + size_t(8 * k) * j;
          if (bk == 0) {
            const uint2 a = ld_stream2(cp);
            w[0] = a.x; w[1] = a.y;
          } else {
            for (int q = 0; q < k / 2; ++q) {
              const uint4 a = ld_stream4(cp + 16 * q);
              w[4 * q] = a.x; w[4 * q + 1] = a.y; w[4 * q + 2] = a.z; w[4 * q + 3] = a.w;
            }
          }
          const float off = float((1 << k) - 1);
#pragma unroll 8
          for (int i = 0; i < 64; i += 2) {
            const int b0 = k * i, b1 = k * (i + 1);
            const uint32_t q0 = (w[b0 >> 5] >> (b0 & 31)) & ((1u << k) - 1u);
            const uint32_t q1 = (w[b1 >> 5] >> (b1 & 31)) & ((1u << k) - 1u);
            arow[i >> 1] = __floats2bfloat162_rn(2.f * float(q0) - off, 2.f * float(q1) - off);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) arow[i] = __floats2bfloat162_rn(0.f, 0.f);
        }
        __syncwarp();
        float scale_mine = 0.f;
        int row_mine = 0;
        if (valid) {
          scale_mine = 0.5f * ld_scale(v.scale + 2 * (v.item0[bk] + j));
          row_mine = rowlist[v.item0[bk] + j];
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          float acc[NT][4];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const int r = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int kk = ks * 16 + (lane >> 4) * 8;
            const uint32_t addr = uint32_t(__cvta_generic_to_shared(As + r * kAStride + kk));
            uint32_t a0, a1, a2, a3;
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3) : "r"(addr));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              asm volatile(
                  "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                  "{%0,%1,%2,%3};"
                  : "+f"(acc[nt][0]), "+f"(acc[nt][1]), "+f"(acc[nt][2]), "+f"(acc[nt][3])
                  : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(bfr[ks][nt][0]), "r"(bfr[ks][nt][1]));
          }
          // acc[nt][0..1]: tile row lane/4, batch nt*8 + 2(lane%4) + {0,1}; acc[nt][2..3]: tile row lane/4 + 8.
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int src = mt * 16 + (lane >> 2) + 8 * h;   // lane that owns this item
            const float sc = __shfl_sync(0xFFFFFFFFu, scale_mine, src);
            const int row = __shfl_sync(0xFFFFFFFFu, row_mine, src);
            if (j0 + src < v.n[bk]) {
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                const int b = nt * 8 + 2 * (lane & 3);
                ys[row * B + b] = fmaf(sc, acc[nt][2 * h], ys[row * B + b]);
                ys[row * B + b + 1] = fmaf(sc, acc[nt][2 * h + 1], ys[row * B + b + 1]);
              }
            }
          }
        }
        __syncwarp();
      }
    }
    __syncthreads();
  }

  // ---------------------------------------------------------------------------------------- output
  const int rbase = t * p.R;
  if (p.S == 1) {
    for (int e = tid; e < Rt * B; e += kThreads) {
      const int b = e / Rt, jj = e - b * Rt;
      p.y[size_t(b) * p.N + rbase + jj] = ys[jj * B + b];
    }
    return;
  }
  float* mine = p.partial + (size_t(t) * p.S + s) * size_t(p.R) * B;
  for (int e = tid; e < Rt * B; e += kThreads) mine[e] = ys[e];
  __threadfence();
  __syncthreads();
  if (tid == 0) last_flag = (atomicAdd(&p.counters[t], 1u) == unsigned(p.S - 1));
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
  const float* tile = p.partial + size_t(t) * p.S * size_t(p.R) * B;
  for (int e = tid; e < Rt * B; e += kThreads) {
    const int b = e / Rt, jj = e - b * Rt;
    float acc = 0.f;
    for (int s2 = 0; s2 < p.S; ++s2) acc += __ldcg(tile + size_t(s2) * p.R * B + jj * B + b);
    p.y[size_t(b) * p.N + rbase + jj] = acc;
  }
  if (tid == 0) p.counters[t] = 0u;
}

// ------------------------------------------------------------------------------------------ launch plan
struct Plan {
  int S, C;
  uint64_t ws_bytes;
  int smem;
};

inline int num_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

inline int smem_bytes(int B, int R, int C) {
  switch (B) {
    case 1: return Smem<1>::bytes(R, C);
    case 2: return Smem<2>::bytes(R, C);
    case 4: return Smem<4>::bytes(R, C);
    case 8: return Smem<8>::bytes(R, C);
    default: return Smem<16>::bytes(R, C);
  }
}

// Split the G group columns of each tile over S CTAs so that the grid covers about two CTAs per SM.
inline Plan make_plan(const vbq_desc& d, int B, int sms) {
  Plan pl;
  const int64_t target = 2LL * sms;
  int64_t S = (target + d.T - 1) / d.T;
  if (S > d.G) S = d.G;
  if (S < 1) S = 1;
  int64_t C = (d.G + S - 1) / S;
  S = (d.G + C - 1) / C;
  pl.S = int(S);
  pl.C = int(C);
  pl.ws_bytes = S > 1 ? uint64_t(d.T) * S * d.R * B * 4 + ((uint64_t(d.T) * 4 + 15) / 16) * 16 : 0;
  pl.smem = smem_bytes(B, int(d.R), pl.C);
  return pl;
}

inline bool desc_ok(const vbq_desc* d) {
  return d->version == 1 && d->N >= 1 && d->K >= 64 && d->K % 64 == 0 && d->G == d->K / 64 && d->R >= 16 &&
         d->R <= kMaxTileRows && d->R % 16 == 0 && d->T == (d->N + d->R - 1) / d->R && d->N <= INT32_MAX &&
         d->K <= INT32_MAX && d->dir_offset == 64 && d->rec_offset > d->dir_offset &&
         d->total_bytes > d->rec_offset;
}

template <int B>
int launch(const vbq_desc* d, const void* blob, const void* x, float* y, void* ws, uint64_t ws_bytes,
           cudaStream_t stream) {
  const Plan pl = make_plan(*d, B, num_sms());
  if (pl.ws_bytes > 0) {
    if (!ws) return VBQ_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 15) return VBQ_ERR_WORKSPACE;
    if (ws_bytes < pl.ws_bytes) return VBQ_ERR_WORKSPACE;
  }
  Params p;
  const uint8_t* base = static_cast<const uint8_t*>(blob);
  p.dir = reinterpret_cast<const uint32_t*>(base + d->dir_offset);
  p.recs = base + d->rec_offset;
  p.x = static_cast<const uint16_t*>(x);
  p.y = y;
  p.partial = static_cast<float*>(ws);
  p.counters = pl.ws_bytes ? reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) +
                                                         uint64_t(d->T) * pl.S * d->R * B * 4)
                           : nullptr;
  p.N = int(d->N); p.K = int(d->K); p.G = int(d->G); p.R = int(d->R); p.T = int(d->T);
  p.S = pl.S; p.C = pl.C;
  // Opt in to more than 48 KB of dynamic shared memory once per (device, batch size) and size.
  static int opted[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& done = opted[dev & 63];
  if (pl.smem > 48 * 1024 && pl.smem > done) {
    if (cudaFuncSetAttribute(vbq_kernel<B>, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem) != cudaSuccess)
      return VBQ_ERR_CUDA;
    done = pl.smem;
  }
  dim3 grid(unsigned(pl.S), unsigned(d->T));
  vbq_kernel<B><<<grid, kThreads, pl.smem, stream>>>(p);
  return cudaPeekAtLastError() == cudaSuccess ? VBQ_OK : VBQ_ERR_CUDA;
}

}  // namespace vbq

extern "C" {

int vbq_workspace_size(const vbq_desc* d, int B, uint64_t* out_bytes) {
  if (!d || !out_bytes) return VBQ_ERR_NULL;
  if (B != 1 && B != 2 && B != 4 && B != 8 && B != 16) return VBQ_ERR_BATCH;
  if (!vbq::desc_ok(d)) return VBQ_ERR_FORMAT;
  *out_bytes = vbq::make_plan(*d, B, vbq::num_sms()).ws_bytes;
  return VBQ_OK;
}

int vbq_workspace_init(void* workspace, uint64_t workspace_bytes, void* stream) {
  if (!workspace) return VBQ_ERR_NULL;
  if (workspace_bytes == 0) return VBQ_OK;
  return cudaMemsetAsync(workspace, 0, size_t(workspace_bytes), static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? VBQ_OK : VBQ_ERR_CUDA;
}

int vbq_gemm_skinny(const vbq_desc* d, const void* blob_dev, const void* x_bf16, int B, float* y,
                    void* workspace, uint64_t workspace_bytes, void* stream) {
  if (!d || !blob_dev || !x_bf16 || !y) return VBQ_ERR_NULL;
  if (B != 1 && B != 2 && B != 4 && B != 8 && B != 16) return VBQ_ERR_BATCH;
  if (!vbq::desc_ok(d)) return VBQ_ERR_FORMAT;
  if ((reinterpret_cast<uintptr_t>(blob_dev) & 15) || (reinterpret_cast<uintptr_t>(x_bf16) & 15) ||
      (reinterpret_cast<uintptr_t>(y) & 3))
    return VBQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (B) {
    case 1: return vbq::launch<1>(d, blob_dev, x_bf16, y, workspace, workspace_bytes, st);
    case 2: return vbq::launch<2>(d, blob_dev, x_bf16, y, workspace, workspace_bytes, st);
    case 4: return vbq::launch<4>(d, blob_dev, x_bf16, y, workspace, workspace_bytes, st);
    case 8: return vbq::launch<8>(d, blob_dev, x_bf16, y, workspace, workspace_bytes, st);
    default: return vbq::launch<16>(d, blob_dev, x_bf16, y, workspace, workspace_bytes, st);
  }
}

int vbq_gemv(const vbq_desc* d, const void* blob_dev, const void* x_bf16, float* y, void* workspace,
             uint64_t workspace_bytes, void* stream) {
  return vbq_gemm_skinny(d, blob_dev, x_bf16, 1, y, workspace, workspace_bytes, stream);
}

}  // extern "C"
