// Device side of libvbq: fused dequantize-and-multiply GEMV and skinny GEMM over format-v1 VBQ blobs.
//
// What is computed (VBQ paper, "Variable Bit-width Quantization", section 3.1 and section 6, paragraph
// "Fused kernels over packed weights"): y[b][r] = sum_g s[r][g] * sum_i (q[r][64g+i] - (2^k-1)/2) * x[b][64g+i].
// The low-bit codes are expanded in registers. The dense matrix never exists in memory.
//
// Kernel structure (B200, sm_100a), one persistent CTA per SM:
//  - The blob is one record per (row tile, group column), stored tile-major. Inside a record, the tile's groups
//    sit in four width buckets (1, 2, 4, 8 bits), each in ascending row order (FORMAT.md). CTA c owns the records
//    whose start offsets fall in the c-th equal slice of the record bytes, so every CTA streams the same number
//    of bytes.
//  - Warp specialization. One producer warp streams whole records into a ring of shared-memory stages with
//    cp.async.bulk (the TMA engine, no multicast). Completion is signaled through mbarrier transaction counts.
//    For each landed record it rebuilds the item -> row map from the 2-bit width codes and stages the column's
//    activations, then releases the stage to the consumer warps through a second mbarrier. Consumers hand the
//    stage back through a third. Every wait is bounded by a timer. On timeout the kernel sets a status bit in
//    the workspace and leaves.
//  - Consumer warps take units of 32 items of one bucket, so every warp instruction runs a single width (the
//    width-bucketed schedule). Units are dealt round-robin over the CTA's record sequence.
//    Batch 1: each consumer warp accumulates into its own copy of the tile's outputs. No barrier is needed
//    between records. Each lane owns one 64-weight group and holds the column's activations in registers.
//    1-bit groups add the activations whose bit is set (predicated adds). 2/4-bit groups expand codes with a
//    magic-number bit-to-float trick against pre-scaled activations. 8-bit groups use byte permutes.
//    Batch 2/4 (CUDA cores) and 8/16 (mma.sync bf16 tensor cores): all consumer warps share one accumulator
//    and synchronize once per record.
//  - A row tile split across CTAs is reduced without floating-point atomics. Each owner CTA writes its partial
//    sums to the workspace and counts itself in. Only the first and last tile of a CTA's range can be shared.
//    At the end of the kernel, each owner waits (bounded) until all owners of the tile are in. It then adds all
//    partials, in CTA order, for its own slice of the tile's rows. The launch is cooperative, so every CTA is
//    resident while others wait for it. Results are bitwise deterministic.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <mutex>

#include "vbq.h"

namespace vbq {

constexpr int kMaxTileRows = 1024;
constexpr int kAStride = 72;            // bf16 per staged A row for ldmatrix (64 + 8 pad: conflict-free rows)
constexpr int kMaxStages = 4;
constexpr int kSmemBudget = 227 * 1024;
constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded mbarrier waits: 2 s
constexpr unsigned kSuspendNs = 20000;                  // a waiting thread sleeps (no issue slots) up to 20 us per poll
constexpr unsigned kStatusTimeout = 1u, kStatusOversize = 2u;

template <int B> struct Cfg {
  // Batch 1: per-item results plus a lagged row pass, with no barrier between records. Other batches: the
  // consumers add straight into the tile accumulators and synchronize once per record.
  static constexpr bool kRowPass = (B == 1);
  static constexpr int kConsumers = (B == 1) ? 14 : 8;  // consumer warps
  static constexpr int kThreads = (kConsumers + 1) * 32;
  static constexpr int kCThreads = kConsumers * 32;
  // activations staged per record: B=1: raw, x*2^-shift for 2-bit, x*2^-shift for 4-bit (fp32);
  // B=2,4: fp32 [64][B]; B=8,16: none (the tensor-core path reads the bf16 copy directly)
  static constexpr int kXBytes = (B == 1) ? 3 * 64 * 4 : (B < 8 ? 64 * B * 4 : 0);
};

struct Params {
  const uint32_t* dir;     // record directory (16-byte units from recs), T*G+1 entries
  const uint8_t* recs;     // first record
  const uint16_t* x;       // bf16 bits, [B][K]
  float* y;                // [B][N]
  float* partial;          // [nCTA + T][R][B] partial sums of shared row tiles
  unsigned* arrive;        // [T] owners that have published their partial sums; zero between calls
  unsigned* depart;        // [T] owners done reducing; the last one resets both counters
  unsigned* status;        // device status word
  int N, K, G, R, T, nrec;
  uint32_t units_total;    // dir[nrec]
  int stage_bytes;         // record capacity of one stage (multiple of 128)
  int stage_size;          // full stage size, record + row list + activations + meta
  int NS;                  // stages
  int ys_cap;              // floats of the tile-accumulator region (>= R*B and >= the CTA count)
};

__host__ __device__ constexpr int align16i(int v) { return (v + 15) & ~15; }
__host__ __device__ constexpr int align128i(int v) { return (v + 127) & ~127; }

// Stage layout: [record bytes | bf16 activations of the column ([B][64], landed by bulk copy) | expanded
// activations | group sums (B f32) | width masks [4][32] u32 | item starts [4][32] i32 | item results (batch 1,
// R f32) | meta (16 int)]
struct StageOff {
  int xraw, xv, sg, masks, pref, res, meta;
  __host__ __device__ StageOff(int stage_bytes, int R, int xbytes, int B, bool rowpass) {
    xraw = stage_bytes;
    xv = xraw + 128 * B;
    sg = xv + align16i(xbytes);
    masks = sg + align16i(4 * B);
    pref = masks + 512;
    res = pref + 512;
    meta = res + (rowpass ? 4 * R : 0);
  }
  __host__ __device__ int size() const { return align128i(meta + 64); }
};
enum Meta { M_T = 0, M_G, M_RT, M_N0, M_N1, M_N2, M_N3, M_UBASE, M_U };

// ------------------------------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return uint32_t(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs) : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for the phase with the given parity to complete. Gives up after kWaitNs: sets the status word and the
// CTA's abort flag, after which every wait of the CTA returns at once and nothing more is written.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, unsigned* status, volatile int* abort) {
  if (*abort) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  for (unsigned it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort) return false;
      if (now_ns() - t0 > kWaitNs) {
        *abort = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}
// Drain wait used after an abort: waits (bounded, ignoring the abort flag) for a bulk copy this CTA issued, so
// that no copy into its shared memory is still in flight when the CTA exits.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, unsigned parity) {
  const unsigned long long t0 = now_ns();
  while (!mbar_try_wait(bar, parity))
    if (now_ns() - t0 > kWaitNs) return;
}
// Bulk copy global -> shared through the TMA engine; completes `bytes` transactions on `bar`.
__device__ __forceinline__ void tma_bulk_load(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Shared-memory accesses by 32-bit shared address (always LDS/STS, never generic loads). The "memory" clobber
// keeps them ordered with the mbarrier waits that publish the data.
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float4 lds128f(uint32_t a) {
  float4 v;
  asm("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float lds32f(uint32_t a) {
  float v;
  asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  unsigned short v;
  asm("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t a) {
  unsigned short v;
  asm("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void sts32f(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
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

// ------------------------------------------------------------------------------- batch-1 inner loops
// Bit position of code t inside its 32-bit source for the magic-number expansion: the code's bits must lie in
// [0, 23), so that OR-ing them into the mantissa of 2^23 gives exactly 2^23 + q * 2^shift. High codes are
// read from (word >> HI) instead of word.
template <int KB> struct Magic;
template <> struct Magic<2> { static constexpr int HI = 10; };
template <> struct Magic<4> { static constexpr int HI = 12; };
template <int KB> __host__ __device__ constexpr bool magic_hi(int t) { return KB * t + KB > 23; }
template <int KB> __host__ __device__ constexpr int magic_shift(int t) {
  return magic_hi<KB>(t) ? KB * t - Magic<KB>::HI : KB * t;
}
// Shift of code i (0..63) of a KB-bit group (code i is code i % (32/KB) of word i / (32/KB)).
template <int KB> __host__ __device__ constexpr int code_shift(int i) { return magic_shift<KB>(i % (32 / KB)); }

__device__ __forceinline__ float magic_f(uint32_t src, uint32_t mask_shifted) {
  return __uint_as_float((src & mask_shifted) | 0x4B000000u);
}

// Each returns sum_i (q_i - (2^k-1)/2) x_i for one 64-weight group; sg = sum_i x_i.
// a += x when (w & bit) != 0, as a predicated add (no branch).
__device__ __forceinline__ void add_if(float& a, uint32_t w, uint32_t bit, float x) {
  asm("{\n\t.reg .pred p;\n\t.reg .b32 t;\n\tand.b32 t, %1, %2;\n\tsetp.ne.b32 p, t, 0;\n\t"
      "@p add.f32 %0, %0, %3;\n\t}"
      : "+f"(a) : "r"(w), "r"(bit), "f"(x));
}
// 1-bit: sum of the activations whose bit is set, minus half the group sum.
__device__ __forceinline__ float dot_b1(uint2 w, const float (&xr)[64], float sg) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    add_if(a0, w.x, 1u << i, xr[i]);
    add_if(a1, w.x, 1u << (i + 1), xr[i + 1]);
    add_if(a2, w.x, 1u << (i + 2), xr[i + 2]);
    add_if(a3, w.x, 1u << (i + 3), xr[i + 3]);
  }
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    add_if(a0, w.y, 1u << i, xr[32 + i]);
    add_if(a1, w.y, 1u << (i + 1), xr[33 + i]);
    add_if(a2, w.y, 1u << (i + 2), xr[34 + i]);
    add_if(a3, w.y, 1u << (i + 3), xr[35 + i]);
  }
  return ((a0 + a1) + (a2 + a3)) - 0.5f * sg;
}

// 2- and 4-bit: xr holds x_i * 2^-shift(i). v - 2^23 = q * 2^shift exactly, so (v - 2^23) * xr_i = q * x_i.
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
  // sum q x - (2^(k-1) - 1/2) sum x
  return ((acc0.x + acc0.y) + (acc1.x + acc1.y)) - (float(1 << (KB - 1)) - 0.5f) * sg;
}

// 8-bit: a byte permute places q in the low mantissa byte of 2^23; subtracting 2^23 + 128 gives q - 128 exactly.
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

// q - 2^(k-1) of code i from a group's code words in shared memory (any width, runtime index).
__device__ __forceinline__ float code_centered(const uint32_t* w, int k, int i) {
  const int bit = k * i;
  const uint32_t q = (w[bit >> 5] >> (bit & 31)) & ((1u << k) - 1u);
  return float(int(q) - (1 << (k - 1)));
}

// Row (within the tile) of item `item` of bucket c. masks[c][w] marks the rows of 32-row word w whose width code
// is c; pref[c][w] is the item index of the first such row (bucket start + rows of code c in earlier words).
// Binary search for the word, then select the k-th set bit of its mask.
__device__ __forceinline__ int item_row(const uint32_t* masks, const int* pref, int c, int item) {
  const int* P = pref + c * 32;
  int w = 0;
#pragma unroll
  for (int step = 16; step > 0; step >>= 1)
    if (P[w + step] <= item) w += step;
  uint32_t m = masks[c * 32 + w];
  int k = item - P[w], pos = 0, cnt;
  cnt = __popc(m & 0xFFFFu); if (k >= cnt) { k -= cnt; m >>= 16; pos += 16; }
  cnt = __popc(m & 0xFFu);   if (k >= cnt) { k -= cnt; m >>= 8;  pos += 8; }
  cnt = __popc(m & 0xFu);    if (k >= cnt) { k -= cnt; m >>= 4;  pos += 4; }
  cnt = __popc(m & 0x3u);    if (k >= cnt) { k -= cnt; m >>= 2;  pos += 2; }
  if (k >= int(m & 1u)) pos += 1;
  return 32 * w + pos;
}

// ----------------------------------------------------------------------------------------- record view
// Offsets of the parts of a record with Rt rows and bucket counts n0..n3 (FORMAT.md).
struct Rec {
  int n0, n1, n2, n3;
  int sc, c0, c1, c2, c3;     // byte offsets: scales and the four code buckets
  int u0, u1, u2, U;          // cumulative unit counts (32 items per unit)
  __device__ __forceinline__ Rec(int Rt, int a, int b, int c, int d) : n0(a), n1(b), n2(c), n3(d) {
    sc = align16i(8 + 4 * ((Rt + 15) / 16));
    c0 = sc + align16i(2 * Rt);
    c1 = c0 + align16i(8 * n0);
    c2 = c1 + 16 * n1;
    c3 = c2 + 32 * n2;
    u0 = (n0 + 31) >> 5;
    u1 = u0 + ((n1 + 31) >> 5);
    u2 = u1 + ((n2 + 31) >> 5);
    U = u2 + ((n3 + 31) >> 5);
  }
  // unit -> bucket, first item of the unit within the bucket, item base, code base, count (branch-free)
  __device__ __forceinline__ void unit(int u, int& bk, int& j0, int& ibase, int& cbase, int& n) const {
    bk = (u >= u0) + (u >= u1) + (u >= u2);
    const int ub = bk == 0 ? 0 : bk == 1 ? u0 : bk == 2 ? u1 : u2;
    j0 = (u - ub) << 5;
    ibase = bk == 0 ? 0 : bk == 1 ? n0 : bk == 2 ? n0 + n1 : n0 + n1 + n2;
    cbase = bk == 0 ? c0 : bk == 1 ? c1 : bk == 2 ? c2 : c3;
    n = bk == 0 ? n0 : bk == 1 ? n1 : bk == 2 ? n2 : n3;
  }
};

// CTA c owns records [lo(c), lo(c+1)) with lo(c) = floor(c * nrec / nCTA): records of one matrix have similar
// sizes, so equal record counts give nearly equal bytes. No memory is read to compute ownership.
__device__ __forceinline__ int rec_lo(const Params& p, int c) {
  return int((long long)c * p.nrec / int(gridDim.x));
}
// Owner of record j: the largest c with lo(c) <= j.
__device__ __forceinline__ int owner(const Params& p, int j) {
  const long long c = ((long long)(j + 1) * gridDim.x + p.nrec - 1) / p.nrec - 1;
  return int(min(c, (long long)gridDim.x - 1));
}

// Gathers the even bits of a 64-bit word into 32 bits.
__device__ __forceinline__ uint32_t even_bits(unsigned long long x) {
  x &= 0x5555555555555555ull;
  x = (x | (x >> 1)) & 0x3333333333333333ull;
  x = (x | (x >> 2)) & 0x0F0F0F0F0F0F0F0Full;
  x = (x | (x >> 4)) & 0x00FF00FF00FF00FFull;
  x = (x | (x >> 8)) & 0x0000FFFF0000FFFFull;
  x = (x | (x >> 16)) & 0x00000000FFFFFFFFull;
  return uint32_t(x);
}

// ------------------------------------------------------------------------------------------------ kernel
template <int B>
__global__ void __launch_bounds__(Cfg<B>::kThreads, 1) vbq_kernel(Params p) {
  using C = Cfg<B>;
  constexpr int NW = C::kConsumers;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t bar_full[kMaxStages], bar_ready[kMaxStages], bar_empty[kMaxStages], bar_done[kMaxStages];
  __shared__ uint64_t bar_cons;
  __shared__ int range[2];
  __shared__ volatile int abort_flag;
  __shared__ int pending[2], npending;  // shared tiles published by this CTA (at most its first and last)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NS = p.NS;
  const StageOff so(p.stage_bytes, p.R, C::kXBytes, B, C::kRowPass);
  float* ys = reinterpret_cast<float*>(smem);                       // tile accumulators [R][B]
  const int ys_floats = p.ys_cap;
  unsigned char* astage = smem + align128i(ys_floats * 4);          // tensor-core A tiles (B >= 8)
  unsigned char* stages = astage + (B >= 8 ? align128i(NW * 32 * kAStride * 2) : 0);

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_ready[s], 32);
      mbar_init(&bar_empty[s], NW);
      mbar_init(&bar_done[s], NW);
    }
    mbar_init(&bar_cons, C::kCThreads);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
    npending = 0;
    range[0] = rec_lo(p, blockIdx.x);
    range[1] = rec_lo(p, blockIdx.x + 1);
  }
  for (int e = tid; e < ys_floats; e += C::kThreads) ys[e] = 0.f;
  __syncthreads();
  const int jbeg = range[0], jend = range[1], n = jend - jbeg;
  if (n <= 0) return;
  // Consumers fold record i's results into the tile accumulators one record later (lag 1), so that the row
  // pass never waits; with a single stage there is nothing to overlap, and the lag is 0.
  const int lag = (C::kRowPass && NS >= 2) ? 1 : 0;

  if (warp == NW) {
    // ================================================================ producer warp
    // Directory entries of this CTA's records, 32 at a time in lanes (records are issued in order).
    int win = 0;
    uint32_t dlane = lane <= n ? __ldg(p.dir + jbeg + lane) : 0u;
    auto dir_at = [&](int i) -> uint32_t {  // whole warp; i in [0, n]
      if (i >= win + 32) {
        win = i;
        dlane = win + lane <= n ? __ldg(p.dir + jbeg + win + lane) : 0u;
      }
      return __shfl_sync(0xFFFFFFFFu, dlane, i - win);
    };
    // Issue record i: one bulk copy of the record and B bulk copies of the column's bf16 activations (128 B).
    auto issue = [&](int i) {  // whole warp; lane 0 issues
      const uint32_t a = dir_at(i);
      const uint32_t b = i + 1 - win < 32 ? __shfl_sync(0xFFFFFFFFu, dlane, i + 1 - win) : __ldg(p.dir + jbeg + i + 1);
      if (lane != 0) return;
      const int j = jbeg + i, s = i % NS, g = j % p.G;
      const unsigned bytes = 16u * (b - a);
      unsigned char* dst = stages + s * p.stage_size;
      if (bytes > unsigned(p.stage_bytes)) {  // descriptor promised a smaller record: flag and skip the copy
        atomicOr(p.status, kStatusOversize);
        mbar_arrive(&bar_full[s]);
        return;
      }
      mbar_arrive_tx(&bar_full[s], bytes + 128u * B);
      tma_bulk_load(dst, p.recs + 16ull * a, bytes, &bar_full[s]);
#pragma unroll
      for (int bb = 0; bb < B; ++bb)
        tma_bulk_load(dst + so.xraw + 128 * bb, p.x + size_t(bb) * p.K + size_t(g) * 64, 128u, &bar_full[s]);
    };
    for (int i = 0; i < min(NS, n); ++i) issue(i);
    __syncwarp();
    int issued = min(NS, n);  // records whose bulk copy has been issued (warp-uniform)
    int unit_base = 0;
    for (int i = 0; i < n; ++i) {
      const int s = i % NS;
      unsigned char* st = stages + s * p.stage_size;
      if (!mbar_wait(&bar_full[s], (i / NS) & 1, p.status, &abort_flag)) {
        for (int r = i; r < issued; ++r) mbar_drain(&bar_full[r % NS], (r / NS) & 1);
        break;
      }
      // -- width masks and item starts per 32-row word (lane = word)
      const int j = jbeg + i, t = j / p.G, g = j - t * p.G;
      const int Rt = min(p.R, p.N - t * p.R);
      const uint2 cnt = *reinterpret_cast<const uint2*>(st);
      const int n0 = cnt.x & 0xFFFF, n1 = cnt.x >> 16, n2 = cnt.y & 0xFFFF, n3 = cnt.y >> 16;
      const int nvalid = max(0, min(32, Rt - 32 * lane));
      unsigned long long v = 0;
      if (nvalid > 0) v = *reinterpret_cast<const unsigned long long*>(st + 8 + 8 * lane);
      const unsigned long long lo = v & 0x5555555555555555ull, hi = (v >> 1) & 0x5555555555555555ull;
      const uint32_t valid = nvalid >= 32 ? 0xFFFFFFFFu : ((1u << nvalid) - 1u);
      const uint32_t m0 = even_bits(~hi & ~lo) & valid, m1 = even_bits(~hi & lo) & valid;
      const uint32_t m2 = even_bits(hi & ~lo) & valid, m3 = even_bits(hi & lo) & valid;
      const unsigned long long mine = (unsigned long long)__popc(m0) | ((unsigned long long)__popc(m1) << 16) |
                                      ((unsigned long long)__popc(m2) << 32) | ((unsigned long long)__popc(m3) << 48);
      unsigned long long incl = mine;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += u;
      }
      const unsigned long long pre = incl - mine;
      uint32_t* masks = reinterpret_cast<uint32_t*>(st + so.masks);
      int* pref = reinterpret_cast<int*>(st + so.pref);
      masks[lane] = m0; masks[32 + lane] = m1; masks[64 + lane] = m2; masks[96 + lane] = m3;
      pref[lane] = int(pre & 0xFFFFull);
      pref[32 + lane] = n0 + int((pre >> 16) & 0xFFFFull);
      pref[64 + lane] = n0 + n1 + int((pre >> 32) & 0xFFFFull);
      pref[96 + lane] = n0 + n1 + n2 + int(pre >> 48);
      // -- expand the column's activations (and group sums for the CUDA-core paths)
      const uint16_t* xg = reinterpret_cast<const uint16_t*>(st + so.xraw);  // [B][64] bf16, landed with the record
      if constexpr (B == 1) {
        float* xv = reinterpret_cast<float*>(st + so.xv);
        const float x0 = __uint_as_float(uint32_t(xg[lane]) << 16);
        const float x1 = __uint_as_float(uint32_t(xg[32 + lane]) << 16);
        xv[lane] = x0;
        xv[32 + lane] = x1;
        xv[64 + lane] = x0 * __uint_as_float(uint32_t(127 - code_shift<2>(lane)) << 23);
        xv[96 + lane] = x1 * __uint_as_float(uint32_t(127 - code_shift<2>(32 + lane)) << 23);
        xv[128 + lane] = x0 * __uint_as_float(uint32_t(127 - code_shift<4>(lane)) << 23);
        xv[160 + lane] = x1 * __uint_as_float(uint32_t(127 - code_shift<4>(32 + lane)) << 23);
        float sgv = x0 + x1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sgv += __shfl_xor_sync(0xFFFFFFFFu, sgv, off);
        if (lane == 0) reinterpret_cast<float*>(st + so.sg)[0] = sgv;
      } else if constexpr (B < 8) {
        float* xv = reinterpret_cast<float*>(st + so.xv);
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float x0 = __uint_as_float(uint32_t(xg[b * 64 + lane]) << 16);
          const float x1 = __uint_as_float(uint32_t(xg[b * 64 + 32 + lane]) << 16);
          xv[lane * B + b] = x0;
          xv[(32 + lane) * B + b] = x1;
          float sgv = x0 + x1;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) sgv += __shfl_xor_sync(0xFFFFFFFFu, sgv, off);
          if (lane == 0) reinterpret_cast<float*>(st + so.sg)[b] = sgv;
        }
      }
      const int U = ((n0 + 31) >> 5) + ((n1 + 31) >> 5) + ((n2 + 31) >> 5) + ((n3 + 31) >> 5);
      if (lane == 0) {
        int* meta = reinterpret_cast<int*>(st + so.meta);
        meta[M_T] = t; meta[M_G] = g; meta[M_RT] = Rt;
        meta[M_N0] = n0; meta[M_N1] = n1; meta[M_N2] = n2; meta[M_N3] = n3;
        meta[M_UBASE] = unit_base; meta[M_U] = U;
      }
      unit_base += U;
      __syncwarp();
      mbar_arrive(&bar_ready[s]);
      // -- refill a stage that the consumers release without needing a later record
      const int rs = NS == 1 ? i : i - min(2, NS - 1), r = rs + NS;
      if (rs >= 0 && r < n) {
        if (!mbar_wait(&bar_empty[rs % NS], (rs / NS) & 1, p.status, &abort_flag)) {
          for (int r2 = i + 1; r2 < issued; ++r2) mbar_drain(&bar_full[r2 % NS], (r2 / NS) & 1);
          break;
        }
        issue(r);
        ++issued;
        __syncwarp();
      }
    }
    return;
  }

  // ================================================================== consumer warps
  const int ctid = tid;  // 0 .. kCThreads-1

  // Bounded barrier of the consumer warps (an mbarrier with one arrival per consumer thread).
  unsigned cons_phase = 0;
  auto consumers_sync = [&]() -> bool {
    mbar_arrive(&bar_cons);
    const bool ok = mbar_wait(&bar_cons, cons_phase & 1u, p.status, &abort_flag);
    ++cons_phase;
    return ok;
  };

  // Owners of tile t. With at least as many records as CTAs every CTA owns a contiguous, non-empty record range,
  // so the owners are first..last. With fewer records than CTAs each CTA owns at most one record, so the owners
  // are the owners of the tile's G records, one each.
  const bool dense = p.nrec >= int(gridDim.x);
  auto tile_owners = [&](int t, int& first) -> int {
    first = owner(p, t * p.G);
    return dense ? owner(p, t * p.G + p.G - 1) - first + 1 : p.G;
  };
  auto kth_owner = [&](int t, int first, int k) -> int { return dense ? first + k : owner(p, t * p.G + k); };

  // Publishes the tile accumulators of tile t: straight into y when this CTA is the tile's only owner, otherwise
  // into its partial slot (owner + tile indexes the slots without collision, since (owner, tile) pairs increase
  // along the records) and counts itself in. Leaves the accumulators zeroed.
  auto publish = [&](int t) -> bool {
    if (!consumers_sync()) return false;
    int first;
    const int owners = tile_owners(t, first);
    const int Rt = min(p.R, p.N - t * p.R);
    const bool sole = owners == 1;
    float* slot = p.partial + size_t(blockIdx.x + t) * p.R * B;
    for (int e = ctid; e < Rt * B; e += C::kCThreads) {
      const float v = ys[e];
      ys[e] = 0.f;
      if (sole) {
        const int jj = e / B, b = e - jj * B;
        p.y[size_t(b) * p.N + size_t(t) * p.R + jj] = v;
      } else {
        slot[e] = v;
      }
    }
    if (!sole) {
      __threadfence();
      if (!consumers_sync()) return false;
      if (ctid == 0) {
        atomicAdd(&p.arrive[t], 1u);
        pending[npending < 2 ? npending : 1] = t;
        npending = min(npending + 1, 2);
      }
    }
    return consumers_sync();
  };

  // Final step for a shared tile: wait (bounded) until every owner has published, then add all owners' slots
  // in CTA order for this CTA's slice of the rows. All loads of a chunk are issued at once (one thread per
  // (owner, element)) into the free accumulator space, then summed per element in owner order. The last owner
  // to finish resets the tile's counters.
  auto reduce_shared = [&](int t) -> bool {
    int first;
    const int owners = tile_owners(t, first);
    if (ctid == 0) {
      const volatile unsigned* arr = p.arrive + t;
      const unsigned long long t0 = now_ns();
      while (*arr < unsigned(owners)) {
        if (abort_flag) break;
        if (now_ns() - t0 > kWaitNs) {
          abort_flag = 1;
          atomicOr(p.status, kStatusTimeout);
          break;
        }
        __nanosleep(32);
      }
    }
    if (!consumers_sync()) return false;
    __threadfence();
    const int rank = dense ? int(blockIdx.x) - first : rec_lo(p, blockIdx.x) - t * p.G;
    const int Rt = min(p.R, p.N - t * p.R);
    const int e0 = int((long long)Rt * rank / owners) * B, e1 = int((long long)Rt * (rank + 1) / owners) * B;
    const int chunk = max(1, ys_floats / owners);
    for (int c0 = e0; c0 < e1; c0 += chunk) {
      const int ne = min(chunk, e1 - c0);
      for (int q = ctid; q < ne * owners; q += C::kCThreads) {
        const int k = q / ne, e = q - k * ne;
        ys[q] = __ldcg(p.partial + size_t(kth_owner(t, first, k) + t) * p.R * B + c0 + e);
      }
      if (!consumers_sync()) return false;
      for (int e = ctid; e < ne; e += C::kCThreads) {
        float v = 0.f;
        for (int k = 0; k < owners; ++k) v += ys[k * ne + e];
        const int ee = c0 + e, jj = ee / B, b = ee - jj * B;
        p.y[size_t(b) * p.N + size_t(t) * p.R + jj] = v;
      }
      if (!consumers_sync()) return false;
    }
    for (int q = ctid; q < ys_floats; q += C::kCThreads) ys[q] = 0.f;
    if (ctid == 0 && atomicAdd(&p.depart[t], 1u) == unsigned(owners - 1)) {
      p.arrive[t] = 0u;
      p.depart[t] = 0u;
    }
    return true;
  };

  int cur_t = -1;
  // Publishes the current tile when record j (still resident) starts a new one.
  auto tile_switch = [&](int j) -> bool {
    const int t = reinterpret_cast<const int*>(stages + (j % NS) * p.stage_size + so.meta)[M_T];
    if (t != cur_t) {
      if (cur_t >= 0 && !publish(cur_t)) return false;
      cur_t = t;
    }
    return true;
  };

  // Batch 1: folds record j's item results into the tile accumulators. Each warp owns a fixed slice of rows,
  // so no two warps ever touch the same accumulator and every row sums its records in order. Row r's item is
  // its bucket's item start for its 32-row word plus the rows of the same width before it in that word.
  auto row_pass = [&](int j) -> bool {
    const int s = j % NS;
    const unsigned char* st = stages + s * p.stage_size;
    if (!mbar_wait(&bar_done[s], (j / NS) & 1, p.status, &abort_flag)) return false;
    if (!tile_switch(j)) return false;
    const int Rt = reinterpret_cast<const int*>(st + so.meta)[M_RT];
    const uint32_t sa = smem_u32(st);
    const int r0 = warp * Rt / NW, r1 = (warp + 1) * Rt / NW;
    for (int r = r0 + lane; r < r1; r += 32) {
      const int c = int(lds8(sa + 8 + (r >> 2)) >> (2 * (r & 3))) & 3;
      const int w = r >> 5;
      const int item = int(lds32(sa + so.pref + 4 * (c * 32 + w))) +
                       __popc(lds32(sa + so.masks + 4 * (c * 32 + w)) & ((1u << (r & 31)) - 1u));
      ys[r] += lds32f(sa + so.res + 4 * item);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_empty[s]);
    return true;
  };

  int loaded_rec = -1, loaded_copy = -1;
  float xr[B == 1 ? 64 : 1];
  for (int i = 0; i < n; ++i) {
    const int s = i % NS;
    unsigned char* st = stages + s * p.stage_size;
    if (!mbar_wait(&bar_ready[s], (i / NS) & 1, p.status, &abort_flag)) return;
    const int* meta = reinterpret_cast<const int*>(st + so.meta);
    const Rec rc(meta[M_RT], meta[M_N0], meta[M_N1], meta[M_N2], meta[M_N3]);
    const int ubase = meta[M_UBASE];
    const uint32_t* masks = reinterpret_cast<const uint32_t*>(st + so.masks);
    const int* pref = reinterpret_cast<const int*>(st + so.pref);
    const float* sgs = reinterpret_cast<const float*>(st + so.sg);
    const int u_first = ((warp - ubase) % NW + NW) % NW;
    if constexpr (!C::kRowPass) {
      if (!tile_switch(i)) return;
    }

    if constexpr (B == 1) {
      const float sg = sgs[0];
      const uint32_t sa = smem_u32(st);
      for (int u = u_first; u < rc.U; u += NW) {
        int bk, j0, ibase, cbase, nb;
        rc.unit(u, bk, j0, ibase, cbase, nb);
        const int copy = bk == 1 ? 1 : (bk == 2 ? 2 : 0);
        if (i != loaded_rec || copy != loaded_copy) {
          const uint32_t src = sa + so.xv + 256 * copy;
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float4 f = lds128f(src + 16 * q);
            xr[4 * q] = f.x; xr[4 * q + 1] = f.y; xr[4 * q + 2] = f.z; xr[4 * q + 3] = f.w;
          }
          loaded_rec = i;
          loaded_copy = copy;
        }
        const int j = j0 + lane;
        if (j < nb) {
          const uint32_t cp = sa + cbase;
          float d;
          if (bk == 0) {
            d = dot_b1(lds64(cp + 8 * j), xr, sg);
          } else if (bk == 1) {
            const uint4 a = lds128(cp + 16 * j);
            const uint32_t w[4] = {a.x, a.y, a.z, a.w};
            d = dot_magic<2>(w, xr, sg);
          } else if (bk == 2) {
            const uint4 a = lds128(cp + 32 * j), b2 = lds128(cp + 32 * j + 16);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b2.x, b2.y, b2.z, b2.w};
            d = dot_magic<4>(w, xr, sg);
          } else {
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 a = lds128(cp + 64 * j + 16 * q);
              w[4 * q] = a.x; w[4 * q + 1] = a.y; w[4 * q + 2] = a.z; w[4 * q + 3] = a.w;
            }
            d = dot_b8(w, xr, sg);
          }
          const int item = ibase + j;
          sts32f(sa + so.res + 4 * item, __half2float(__ushort_as_half((unsigned short)lds16(sa + rc.sc + 2 * item))) * d);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_done[s]);
      if (lag == 0) {
        if (!row_pass(i)) return;
      } else if (i >= 1) {
        if (!row_pass(i - 1)) return;
      }
      continue;
    } else if constexpr (B < 8) {
      // CUDA cores, B in {2, 4}: lane = group; activations of all batches broadcast from the stage.
      const float* xc = reinterpret_cast<const float*>(st + so.xv);
      for (int u = u_first; u < rc.U; u += NW) {
        int bk, j0, ibase, cbase, nb;
        rc.unit(u, bk, j0, ibase, cbase, nb);
        const int j = j0 + lane;
        if (j >= nb) continue;
        const int k = 1 << bk;
        const uint32_t* w = reinterpret_cast<const uint32_t*>(st + cbase + 8 * k * j);
        float acc[B];
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = 0.f;
        if (bk == 0) {
          const uint32_t w0 = w[0], w1 = w[1];
#pragma unroll 8
          for (int i2 = 0; i2 < 64; ++i2) {
            if ((i2 < 32 ? w0 : w1) & (1u << (i2 & 31))) {
#pragma unroll
              for (int b = 0; b < B; ++b) acc[b] += xc[i2 * B + b];
            }
          }
        } else {
#pragma unroll 4
          for (int i2 = 0; i2 < 64; ++i2) {
            const float qv = code_centered(w, k, i2);
#pragma unroll
            for (int b = 0; b < B; ++b) acc[b] = fmaf(qv, xc[i2 * B + b], acc[b]);
          }
        }
        const int item = ibase + j;
        const float sc = __half2float(reinterpret_cast<const __half*>(st + rc.sc)[item]);
        const int row = item_row(masks, pref, bk, item);
        // sum (q - 2^(k-1)) x + 1/2 sum x == sum (q - (2^k-1)/2) x; for k = 1 the first sum is sum_{q=1} x - S.
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float S = sgs[b];
          const float d = (bk == 0) ? acc[b] - 0.5f * S : acc[b] + 0.5f * S;
          ys[row * B + b] = fmaf(sc, d, ys[row * B + b]);
        }
      }
    } else {
      // Tensor cores, B in {8, 16}: lane = group, dequantized to bf16 2q-(2^k-1) in this warp's A tile; two
      // m16 tiles per unit through mma.sync m16n8k16 (bf16 in, fp32 accumulate), then s/2 per row.
      constexpr int NT = B >= 8 ? B / 8 : 1;
      __nv_bfloat16* As = reinterpret_cast<__nv_bfloat16*>(astage) + warp * 32 * kAStride;
      const uint32_t* xb = reinterpret_cast<const uint32_t*>(st + so.xraw);
      uint32_t bfr[4][NT][2];
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int nb2 = nt * 8 + (lane >> 2);
          bfr[ks][nt][0] = xb[nb2 * 32 + 8 * ks + (lane & 3)];
          bfr[ks][nt][1] = xb[nb2 * 32 + 8 * ks + 4 + (lane & 3)];
        }
      for (int u = u_first; u < rc.U; u += NW) {
        int bk, j0, ibase, cbase, nb;
        rc.unit(u, bk, j0, ibase, cbase, nb);
        const int k = 1 << bk;
        const int j = j0 + lane;
        const bool valid = j < nb;
        __nv_bfloat162* arow = reinterpret_cast<__nv_bfloat162*>(As + lane * kAStride);
        if (valid) {
          const uint32_t* w = reinterpret_cast<const uint32_t*>(st + cbase + 8 * k * j);
          const float off = float((1 << k) - 1);
          const uint32_t mask = (1u << k) - 1u;
#pragma unroll 8
          for (int i2 = 0; i2 < 64; i2 += 2) {
            const int b0 = k * i2, b1 = k * (i2 + 1);
            const uint32_t q0 = (w[b0 >> 5] >> (b0 & 31)) & mask;
            const uint32_t q1 = (w[b1 >> 5] >> (b1 & 31)) & mask;
            arow[i2 >> 1] = __floats2bfloat162_rn(2.f * float(q0) - off, 2.f * float(q1) - off);
          }
        } else {
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) arow[i2] = __floats2bfloat162_rn(0.f, 0.f);
        }
        __syncwarp();
        float scale_mine = 0.f;
        int row_mine = 0;
        if (valid) {
          scale_mine = 0.5f * __half2float(reinterpret_cast<const __half*>(st + rc.sc)[ibase + j]);
          row_mine = item_row(masks, pref, bk, ibase + j);
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
            uint32_t a0, a1, a2, a3;
            asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                         : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3) : "r"(smem_u32(As + r * kAStride + kk)));
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
            const int src = mt * 16 + (lane >> 2) + 8 * h;
            const float sc = __shfl_sync(0xFFFFFFFFu, scale_mine, src);
            const int row = __shfl_sync(0xFFFFFFFFu, row_mine, src);
            if (j0 + src < nb) {
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
    // shared accumulators: every warp is done with this record before any warp starts the next one
    if (!consumers_sync()) return;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_empty[s]);
  }
  if (lag == 1 && !row_pass(n - 1)) return;
  if (cur_t < 0 || !publish(cur_t)) return;
  for (int k = 0; k < npending; ++k)
    if (!reduce_shared(pending[k])) return;
}

// ------------------------------------------------------------------------------------------ launch plan
struct Plan {
  int grid, threads, NS, stage_bytes, stage_size, smem, ys_cap;
  uint64_t ws_bytes, status_off, counters_off;
};

inline int num_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int B>
inline bool make_plan_t(const vbq_desc& d, int sms, Plan& pl) {
  using C = Cfg<B>;
  pl.grid = sms < 1024 ? sms : 1024;  // owner bitmaps cover 1024 CTAs
  pl.threads = C::kThreads;
  pl.stage_bytes = align128i(int(d.max_record_bytes));
  const int R = int(d.R);
  pl.stage_size = StageOff(pl.stage_bytes, R, C::kXBytes, B, C::kRowPass).size();
  pl.ys_cap = R * B > pl.grid ? R * B : pl.grid;
  const int fixed = align128i(pl.ys_cap * 4) +
                    (B >= 8 ? align128i(C::kConsumers * 32 * kAStride * 2) : 0);
  int ns = (kSmemBudget - fixed) / pl.stage_size;
  if (ns > kMaxStages) ns = kMaxStages;
  if (ns < 1) return false;
  pl.NS = ns;
  pl.smem = fixed + ns * pl.stage_size;
  const uint64_t slots = uint64_t(pl.grid) + uint64_t(d.T);
  pl.counters_off = slots * uint64_t(R) * B * 4;
  pl.ws_bytes = (pl.counters_off + uint64_t(d.T) * 8 + 4 + 15) / 16 * 16;
  pl.status_off = pl.ws_bytes - 4;
  return true;
}

inline bool make_plan(const vbq_desc& d, int B, int sms, Plan& pl) {
  switch (B) {
    case 1: return make_plan_t<1>(d, sms, pl);
    case 2: return make_plan_t<2>(d, sms, pl);
    case 4: return make_plan_t<4>(d, sms, pl);
    case 8: return make_plan_t<8>(d, sms, pl);
    default: return make_plan_t<16>(d, sms, pl);
  }
}

inline bool desc_ok(const vbq_desc* d) {
  return d->version == 1 && d->N >= 1 && d->K >= 64 && d->K % 64 == 0 && d->G == d->K / 64 && d->R >= 16 &&
         d->R <= kMaxTileRows && d->R % 16 == 0 && d->T == (d->N + d->R - 1) / d->R && d->N <= INT32_MAX &&
         d->K <= INT32_MAX && d->dir_offset == 64 && d->rec_offset > d->dir_offset &&
         d->total_bytes > d->rec_offset && d->max_record_bytes >= 32 &&
         d->max_record_bytes <= d->total_bytes - d->rec_offset && d->max_record_bytes % 16 == 0 &&
         (d->total_bytes - d->rec_offset) % 16 == 0 && (d->total_bytes - d->rec_offset) / 16 <= 0xFFFFFFFFull;
}

template <int B>
int launch(const vbq_desc* d, const void* blob, const void* x, float* y, void* ws, uint64_t ws_bytes,
           cudaStream_t stream) {
  Plan pl;
  if (!make_plan_t<B>(*d, num_sms(), pl)) return VBQ_ERR_FORMAT;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15) || ws_bytes < pl.ws_bytes) return VBQ_ERR_WORKSPACE;
  Params p;
  const uint8_t* base = static_cast<const uint8_t*>(blob);
  p.dir = reinterpret_cast<const uint32_t*>(base + d->dir_offset);
  p.recs = base + d->rec_offset;
  p.x = static_cast<const uint16_t*>(x);
  p.y = y;
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.partial = reinterpret_cast<float*>(w);
  p.arrive = reinterpret_cast<unsigned*>(w + pl.counters_off);
  p.depart = p.arrive + d->T;
  p.status = reinterpret_cast<unsigned*>(w + pl.status_off);
  p.N = int(d->N); p.K = int(d->K); p.G = int(d->G); p.R = int(d->R); p.T = int(d->T);
  p.nrec = int(d->T * d->G);
  p.units_total = uint32_t((d->total_bytes - d->rec_offset) / 16);
  p.stage_bytes = pl.stage_bytes;
  p.stage_size = pl.stage_size;
  p.NS = pl.NS;
  p.ys_cap = pl.ys_cap;
  // Opt in to the dynamic shared memory once per device and size.
  static int opted[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& done = opted[dev & 63];
  if (pl.smem > done) {
    if (cudaFuncSetAttribute(vbq_kernel<B>, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem) != cudaSuccess)
      return VBQ_ERR_CUDA;
    done = pl.smem;
  }
  // Cooperative launch: all CTAs are co-resident, which the bounded cross-CTA wait of the split-K reduction
  // relies on.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(pl.grid));
  cfg.blockDim = dim3(unsigned(pl.threads));
  cfg.dynamicSmemBytes = size_t(pl.smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, vbq_kernel<B>, p) != cudaSuccess) return VBQ_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? VBQ_OK : VBQ_ERR_CUDA;
}

}  // namespace vbq

extern "C" {

int vbq_workspace_size(const vbq_desc* d, int B, uint64_t* out_bytes) {
  if (!d || !out_bytes) return VBQ_ERR_NULL;
  if (B != 1 && B != 2 && B != 4 && B != 8 && B != 16) return VBQ_ERR_BATCH;
  if (!vbq::desc_ok(d)) return VBQ_ERR_FORMAT;
  vbq::Plan pl;
  if (!vbq::make_plan(*d, B, vbq::num_sms(), pl)) return VBQ_ERR_FORMAT;
  *out_bytes = pl.ws_bytes;
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

// ------------------------------------------------------------------------------ allocation-free variant
// Scratch for vbq_gemm_skinny_noalloc: one fixed buffer per device, created when the library is loaded on that
// device and kept until the process exits. It replaces the caller-provided workspace of vbq_gemm_skinny.
namespace vbq {
constexpr uint64_t kStaticScratchBytes = 16ull << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device. In host code the array's name is only a host-side
// stand-in, so the address is looked up once per device with cudaGetSymbolAddress (that device current).
int static_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return VBQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return VBQ_ERR_CUDA;
    addr[dev] = ptr;
  }
  *out = addr[dev];
  return VBQ_OK;
}
}  // namespace vbq

extern "C" int vbq_gemm_skinny_noalloc(const vbq_desc* d, const void* blob_dev, const void* x_bf16, int B,
                                       float* y, void* stream) {
  if (!d || !blob_dev || !x_bf16 || !y) return VBQ_ERR_NULL;
  if (B != 1 && B != 2 && B != 4 && B != 8 && B != 16) return VBQ_ERR_BATCH;
  if (!vbq::desc_ok(d)) return VBQ_ERR_FORMAT;
  uint64_t need = 0;
  if (int st = vbq_workspace_size(d, B, &need)) return st;
  if (need > vbq::kStaticScratchBytes) return VBQ_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (int st = vbq::static_scratch(&scratch)) return st;
  // The buffer keeps the previous call's contents: clear the arrival counters and the status word, which the
  // kernel needs at zero. The partial-sum area is always written before it is read.
  vbq::Plan pl;
  if (!vbq::make_plan(*d, B, vbq::num_sms(), pl)) return VBQ_ERR_FORMAT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(static_cast<unsigned char*>(scratch) + pl.counters_off, 0,
                      size_t(need - pl.counters_off), st) != cudaSuccess)
    return VBQ_ERR_CUDA;
  return vbq_gemm_skinny(d, blob_dev, x_bf16, B, y, scratch, need, stream);
}
