// Device side of libvbq: fused dequantize-and-multiply GEMV and skinny GEMM over format-v1 VBQ blobs.
//
// What is computed (VBQ paper, "Variable Bit-width Quantization", section 3.1 and section 6, paragraph
// "Fused kernels over packed weights"): y[b][r] = sum_g s[r][g] * sum_i (q[r][64g+i] - (2^k-1)/2) * x[b][64g+i].
// The low-bit codes are expanded in registers. The dense matrix never exists in memory.
//
// Kernel structure (B200, sm_100a), one CTA per SM (details at the record-batch kernel below):
//  - The blob is one record per (row tile, group column), stored tile-major. Inside a record, the tile's groups
//    sit in four width buckets (1, 2, 4, 8 bits), each in ascending row order. CTA c owns the c-th share of the
//    records: equal counts in closed form, or equal estimated cost found in the directory when record sizes
//    differ much.
//  - The CTA streams its records in batches of up to seven records of one row tile into shared memory with
//    cp.async.bulk (the TMA engine, no multicast), waiting on mbarrier transaction counts bounded by a timer. A
//    meta job per record validates it and prepares its masks and activation side one batch ahead.
//  - All warps of the CTA split each batch's width-bucket units by estimated cost, so every unit runs a single
//    width. Batch 1, 2 (CUDA cores): 1- and 2-bit codes index nibble tables of partial sums of x, 4-bit codes go
//    through a magic-number bit-to-float expansion, 8-bit codes through byte permutes. Batch 4, 8, 16: mma.sync
//    bf16 tensor cores on exact small integers built from the codes in registers. Results land in item order,
//    and a row pass adds each record's results to the tile's rows in record order.
//  - Row tiles that several CTAs share are reduced without floating-point atomics: each CTA writes its partial
//    sums to the workspace and counts itself in, and the last to arrive adds every element over the owners in
//    CTA order. Results are bitwise deterministic, and no CTA ever waits for another.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <type_traits>
#include <mutex>

#include "vbq.h"

namespace vbq {

constexpr int kMaxTileRows = 1024;
constexpr int kEpiChunk = 32;          // SwiGLU epilogue: tiles counted in per round
constexpr int kSmemBudget = 227 * 1024 - 2048;  // dynamic shared memory; the rest is the static part
constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded mbarrier waits: 2 s
constexpr unsigned kSuspendNs = 20000;                  // a waiting thread sleeps (no issue slots) up to 20 us per poll
constexpr unsigned kStatusTimeout = 1u, kStatusOversize = 2u, kStatusRecord = 4u;

// Up to kMaxMats matrices with the same K and tile rows run as one sequence of records (and row tiles): matrix m
// holds global records [rec_start[m], rec_start[m+1]) and tiles [tile_start[m], tile_start[m+1]).
constexpr int kMaxMats = 4;
struct Params {
  const uint32_t* dir[kMaxMats];   // record directory of matrix m (16-byte units from recs[m]), T_m*G+1 entries
  const uint8_t* recs[kMaxMats];   // first record of matrix m
  float* y[kMaxMats];              // output of matrix m, [B][N_m]
  int N[kMaxMats];
  uint32_t units_total[kMaxMats];  // dir[m][T_m*G]: 16-byte units of matrix m's records
  int rec_start[kMaxMats + 1];
  int tile_start[kMaxMats + 1];
  int sym[kMaxMats];       // matrix m's widths >= 2 use Eq. 1's symmetric grid (format flag bit 0)
  int nmat;
  int swiglu;              // SwiGLU epilogue: matrices 0 (gate) and 1 (up) have the same rows; h = silu(y0) * y1
  uint16_t* h;             // bf16 bits, [B][N_0] (SwiGLU only)
  unsigned* pair;          // [T_0] row tiles of the gate/up pair already final; zero between calls (SwiGLU only)
  const uint16_t* x;       // bf16 bits, [B][K], shared by all matrices
  float* partial;          // [nCTA + T][B][R] partial sums of shared row tiles
  unsigned* arrive;        // [T] owners that have published their partial sums; zero between calls
  unsigned* status;        // device status word
  int K, G, R, T, nrec;    // T, nrec: all matrices
  int S;                   // batches in flight (record slots: NB x S)
  int stage_bytes;         // record capacity of one slot (multiple of 128)
  int stage_size;          // slot: record, then the column's bf16 activations [B][64]
  int NB;                  // records per batch
  int res_off, meta_off, row_off, dir_off;  // shared-memory offsets: item results, table blocks, row blocks, directory
  int res_rec, meta_rec;   // bytes per record: item results [R][B] f32, table block
  int res_sets;            // item-result sets: 2 (alternate batches) or 1
  int cost[5];             // job costs for the split of a batch among warps: units of 1, 2, 4, 8 bits; meta job
  int withhold;            // test hook: the record (global index) whose bulk copy is never issued, or -1
  int balanced;            // CTAs split the records by estimated cost (directory search) instead of by count
  unsigned long long base16[kMaxMats];  // start of matrix m's records in the byte sequence of all records, 16-B units
  unsigned long long rec_w16;           // cost of a record beyond its bytes, in 16-byte units
  unsigned long long total_w;           // cost of all records: 16-byte units + nrec * rec_w16
  unsigned long long wait_ns;  // limit of every mbarrier wait
};

// Element m of a kernel-parameter array through a select chain (a dynamic index would copy the array to local
// memory).
template <typename T>
__device__ __forceinline__ T pick(const T (&a)[kMaxMats], int m) {
  return m == 0 ? a[0] : m == 1 ? a[1] : m == 2 ? a[2] : a[3];
}
__device__ __forceinline__ int mat_of_tile(const Params& p, int t) {
  return (p.nmat > 1 && t >= p.tile_start[1]) + (p.nmat > 2 && t >= p.tile_start[2]) +
         (p.nmat > 3 && t >= p.tile_start[3]);
}
__device__ __forceinline__ int mat_of_rec(const Params& p, int j) {
  return (p.nmat > 1 && j >= p.rec_start[1]) + (p.nmat > 2 && j >= p.rec_start[2]) +
         (p.nmat > 3 && j >= p.rec_start[3]);
}
// Where tile t's outputs go: row r, batch b at y[b * ld + r]; Rt rows.
struct TileOut {
  float* y;
  int ld, Rt;
};
__device__ __forceinline__ TileOut tile_out(const Params& p, int t) {
  const int m = mat_of_tile(p, t);
  const int tl = t - (m == 0 ? 0 : m == 1 ? p.tile_start[1] : m == 2 ? p.tile_start[2] : p.tile_start[3]);
  const int N = pick(p.N, m);
  return TileOut{pick(p.y, m) + size_t(tl) * p.R, N, min(p.R, N - tl * p.R)};
}


__host__ __device__ constexpr int align16i(int v) { return (v + 15) & ~15; }
__host__ __device__ constexpr int align128i(int v) { return (v + 127) & ~127; }

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
// Wait for the phase with the given parity to complete. Gives up after limit_ns: sets the status word and the
// CTA's abort flag, after which every wait of the CTA returns at once and nothing more is written.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, unsigned* status, volatile int* abort,
                                          unsigned long long limit_ns) {
  if (*abort) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  for (unsigned it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort) return false;
      if (now_ns() - t0 > limit_ns) {
        *abort = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}
// Drain wait used after an abort: waits (bounded, ignoring the abort flag) for a bulk copy this CTA issued, so
// that no copy into its shared memory is still in flight when the CTA exits.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, unsigned parity, unsigned long long limit_ns) {
  const unsigned long long t0 = now_ns();
  while (!mbar_try_wait(bar, parity))
    if (now_ns() - t0 > limit_ns) return;
}
// Atomic add with acquire-release semantics at GPU scope; returns the old value.
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned* addr, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
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
// f(integral_constant<int, I>) for I = I0 .. N-1, unrolled at compile time (for immediates that must be constants)
template <int I, int N, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (I < N) {
    f(std::integral_constant<int, I>{});
    static_for<I + 1, N>(f);
  }
}
// ld.shared.f32 at a + OFF, the offset an immediate of the instruction
template <int OFF>
__device__ __forceinline__ float lds32f_off(uint32_t a) {
  float v;
  asm("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(a), "n"(OFF) : "memory");
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
__device__ __forceinline__ void sts64f(uint32_t a, float v0, float v1) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(v0), "f"(v1) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, const uint32_t (&v)[4]) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
               : "memory");
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
template <> struct Magic<1> { static constexpr int HI = 9; };
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

// Each returns sum_i (q_i - c) x_i for one 64-weight group; sg = sum_i x_i.
// 2- and 4-bit: xr holds x_i * 2^-shift(i). v - 2^23 = q * 2^shift exactly, so (v - 2^23) * xr_i = q * x_i.
// The grid offset is c = 2^(k-1) - corr: corr = 1/2 on the default grid, 1 on Eq. 1's symmetric grid.
template <int KB>
__device__ __forceinline__ float dot_magic(const uint32_t (&w)[2 * KB], const float (&xr)[64], float sg, float corr) {
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
  return ((acc0.x + acc0.y) + (acc1.x + acc1.y)) - (float(1 << (KB - 1)) - corr) * sg;
}

// 8-bit: a byte permute places q in the low mantissa byte of 2^23; subtracting 2^23 + 128 gives q - 128 exactly;
// q - c = (q - 128) + corr with corr = 128 - c.
__device__ __forceinline__ float dot_b8(const uint32_t (&w)[16], const float (&xr)[64], float sg, float corr) {
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
  return ((acc0.x + acc0.y) + (acc1.x + acc1.y)) + corr * sg;
}

// 2^e for a small integer e, exact in fp32.
__host__ __device__ constexpr float pow2f(int e) { return e >= 0 ? float(1u << e) : 1.0f / float(1u << -e); }

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Tensor-core A row of one KB-bit group: its 64 values 2(q_i - c) as bf16 at byte address arow, from the group's
// code words at byte address codes; off = 2c. Every value is an integer of magnitude at most 255, so every step
// is exact: the magic-number expansion gives q * 2^shift (as in the batch-1 loops), one packed FMA scales it by
// 2^(1 - shift) and subtracts 2c, and bf16 holds the result. 8-bit codes use the byte-permute form.
// ----------------------------------------------------------------------------------------- record view
// Offsets of the parts of a packed-format-v1 record with Rt rows and bucket counts n0..n3.
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

// CTA c owns records [lo(c), lo(c+1)) with lo(c) = floor(c * nrec / nCTA): records of one matrix have similar
// sizes, so equal record counts give nearly equal bytes. No memory is read to compute ownership.
// 32-bit arithmetic when (nCTA + 1) * (nrec + 1) fits, which covers every realistic matrix; 64-bit otherwise.
__device__ __forceinline__ bool small_ids(const Params& p) {
  return (unsigned long long)(gridDim.x + 1) * unsigned(p.nrec + 1) < (1ull << 32);
}
__device__ __forceinline__ int rec_lo(const Params& p, int c) {
  if (small_ids(p)) return int(unsigned(c) * unsigned(p.nrec) / gridDim.x);
  return int((long long)c * p.nrec / int(gridDim.x));
}
// Owner of record j: the largest c with lo(c) <= j.
__device__ __forceinline__ int owner(const Params& p, int j) {
  const long long c = small_ids(p) ? (long long)((unsigned(j + 1) * gridDim.x + p.nrec - 1) / unsigned(p.nrec)) - 1
                                   : ((long long)(j + 1) * gridDim.x + p.nrec - 1) / p.nrec - 1;
  return int(min(c, (long long)gridDim.x - 1));
}

// Split by cost (p.balanced, for matrices whose records differ much in size, such as an LM head whose frequent
// rows are wider, or a small last row tile). A record costs its bytes plus a fixed part (p.rec_w16, a few mean
// records: its meta job and row pass, and the rows' units whatever their width). With off(j) the cost of the
// records before j and T the total, CTA c owns the records j with c T <= n off(j) < (c + 1) T (n CTAs). So lo(c)
// is the first j with n off(j) >= c T, and the owner of record j is floor(n off(j) / T); a CTA can own nothing.
__device__ __forceinline__ unsigned long long rec_off16(const Params& p, int j) {   // j in [0, nrec]
  const int m = mat_of_rec(p, j);
  const int jl = j - (m == 0 ? 0 : m == 1 ? p.rec_start[1] : m == 2 ? p.rec_start[2] : p.rec_start[3]);
  return pick(p.base16, m) + __ldg(pick(p.dir, m) + jl) + (unsigned long long)j * p.rec_w16;
}
__device__ __forceinline__ int byte_owner(const Params& p, int j) {
  return int(rec_off16(p, j) * gridDim.x / p.total_w);
}
// lo(c) by a 128-way search of one warp (four probes per lane and round; the directory is read through L2).
__device__ int byte_lo(const Params& p, int c, int lane) {
  const unsigned long long tgt = (unsigned long long)c * p.total_w, n = gridDim.x;
  int lo = 0, hi = p.nrec;   // the answer is in [lo, hi]; off(nrec) = T satisfies every target
  while (lo < hi) {
    const int step = (hi - lo + 127) / 128;
    bool pr[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = lo + (4 * lane + q) * step;
      pr[q] = j >= hi || rec_off16(p, j) * n >= tgt;
    }
    unsigned first = 128;   // first probe (in probe order) that holds
#pragma unroll
    for (int q = 3; q >= 0; --q)
      if (pr[q]) first = 4 * lane + q;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) first = min(first, __shfl_xor_sync(0xFFFFFFFFu, first, off));
    if (first == 0) return lo;
    const int prev = lo + int(first - 1) * step;   // the last probe that fails
    hi = first == 128 ? hi : min(hi, lo + int(first) * step);
    lo = prev + 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------------------- end of a CTA
// Runs after every whole-tile output and every partial slot of this CTA is written (all threads, after a barrier).
//  - Tiles shared with other CTAs (only a CTA's first and last tile can be): one thread makes the CTA's slot writes
//    visible GPU-wide and counts the CTA in on the tile's arrival counter; the last owner to arrive adds all owners'
//    slots in an order fixed by the tile's shape and owner count, and resets the counter. No CTA waits for another.
//  - SwiGLU epilogue (p.swiglu): matrices 0 (gate) and 1 (up) have the same rows and tiles. Whoever writes a tile's
//    final y counts it in on the pair counter of its tile index; the second of the pair computes h = silu(gate) * up
//    for those rows from both final outputs, rounded once to bf16, and resets the counter.
template <int B, int kThreads>
__device__ void finish_cta(const Params& p, int L, int H, int* cta_flags, int* epi_tiles, int* epi_count) {
  const int tid = threadIdx.x, G = p.G, R = p.R;
  if (H <= L) return;
  extern __shared__ __align__(128) unsigned char smem_fin[];   // the kernel's dynamic shared memory, free by now
  int* own_list = reinterpret_cast<int*>(smem_fin);
  __shared__ int own_cnt[2];
  const int tfirst = L / G, tlast = (H - 1) / G;
  const bool part0 = !(L <= tfirst * G && H >= (tfirst + 1) * G);
  const bool part1 = tlast != tfirst && !(L <= tlast * G && H >= (tlast + 1) * G);
  // Owners of tile t, in CTA order. Split by count: with at least as many records as CTAs every CTA owns a
  // contiguous, non-empty record range, so the owners are first..last; with fewer records than CTAs each CTA owns
  // at most one record, so the owners are the owners of the tile's G records, one each. Split by bytes: the
  // distinct owners of the tile's records, listed by warp 0 (first tile) and warp 1 (last tile) in own_list.
  const bool dense = p.nrec >= int(gridDim.x), bal = p.balanced != 0;
  const int stride = int(gridDim.x) + 1;
  if (bal && (part0 || part1)) {
    __syncthreads();   // own_list reuses shared memory that the last row pass may still read
    const int w = tid >> 5, lane = tid & 31;
    if (w < 2 && (w == 0 ? part0 : part1)) {
      const int t = w == 0 ? tfirst : tlast, j0 = t * G, j1 = min(j0 + G, p.nrec);
      int cnt = 0, prev_q = -1;
      for (int jb = j0; jb < j1; jb += 32) {
        const int j = jb + lane;
        const int q = j < j1 ? byte_owner(p, j) : 0x7FFFFFFF;
        int up = __shfl_up_sync(0xFFFFFFFFu, q, 1);
        if (lane == 0) up = prev_q;
        const bool start = j < j1 && q != up;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, start);
        if (start) own_list[w * stride + cnt + __popc(m & ((1u << lane) - 1u))] = q;
        cnt += __popc(m);
        prev_q = __shfl_sync(0xFFFFFFFFu, q, 31);
      }
      if (lane == 0) own_cnt[w] = cnt;
    }
    __syncthreads();
  }
  // tile t is the first (index 0) or last (index 1) tile of this CTA
  auto tile_owners = [&](int t, int& first) -> int {
    if (bal) {
      first = t == tfirst ? 0 : 1;   // the list
      return own_cnt[first];
    }
    first = owner(p, t * G);
    return dense ? owner(p, t * G + G - 1) - first + 1 : G;
  };
  auto kth_owner = [&](int t, int first, int k) -> int {
    if (bal) return own_list[first * stride + k];
    return dense ? first + k : owner(p, t * G + k);
  };
  // Sums of all owners' partial slots of the tiles this CTA reduces (one or two) into y, each element over the
  // owners in CTA order (so the result does not depend on which CTA reduces). A slot holds [B][R] f32. The
  // elements of both tiles form one index space, so their loads overlap. Few elements: one element per thread and
  // step, 16 owners' loads in flight. Many: four rows of one batch row per 16-byte load (item f of a tile: batch
  // row f / nq, rows 4 (f % nq) ..), U items per thread and step, 8 owners' loads in flight each.
  auto reduce_tiles = [&](int ta, int tb, int ntiles) {
    // tile i in {0, 1} (selected by value: an indexed local array would live in local memory)
    int first0, first1 = 0;
    const int own0 = tile_owners(ta, first0), own1 = ntiles > 1 ? tile_owners(tb, first1) : 0;
    const TileOut y0 = tile_out(p, ta), y1 = tile_out(p, ntiles > 1 ? tb : ta);
    const int omax = max(own0, own1);
    auto slot_of = [&](bool sec, int o) {
      const int t = sec ? tb : ta;
      return p.partial + size_t(kth_owner(t, sec ? first1 : first0, o) + t) * R * B;
    };
    const int ne0 = y0.Rt * B, ne = ne0 + (ntiles > 1 ? y1.Rt * B : 0);
    if (ne <= 2 * kThreads) {
      constexpr int OC = 16;
      for (int e2 = tid; e2 < ne; e2 += kThreads) {
        const bool sec = e2 >= ne0;
        const int e = e2 - (sec ? ne0 : 0), Rt = sec ? y1.Rt : y0.Rt, own = sec ? own1 : own0;
        const int b = e / Rt, r = e - b * Rt;
        float v = 0.f;
        for (int o0 = 0; o0 < own; o0 += OC) {
          float part[OC];
#pragma unroll
          for (int q = 0; q < OC; ++q) part[q] = o0 + q < own ? __ldcg(slot_of(sec, o0 + q) + size_t(b) * R + r) : 0.f;
#pragma unroll
          for (int q = 0; q < OC; ++q)
            if (o0 + q < own) v += part[q];
        }
        (sec ? y1.y : y0.y)[size_t(b) * (sec ? y1.ld : y0.ld) + r] = v;
      }
      return;
    }
    constexpr int U = kThreads >= 512 ? 1 : 2, OC = 8;
    const int nq0 = (y0.Rt + 3) >> 2, nq1 = (y1.Rt + 3) >> 2;
    const int nf0 = nq0 * B, nf = nf0 + (ntiles > 1 ? nq1 * B : 0);
    auto add4 = [](float4& v, const float4& a) { v.x += a.x; v.y += a.y; v.z += a.z; v.w += a.w; };
    for (int f0 = tid; f0 < nf; f0 += U * kThreads) {
      float4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int o0 = 0; o0 < omax; o0 += OC) {
        float4 part[OC][U];
#pragma unroll
        for (int q = 0; q < OC; ++q)
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int f = f0 + u * kThreads;
            const bool sec = f >= nf0;
            const int fl = f - (sec ? nf0 : 0), nq = sec ? nq1 : nq0, b = fl / nq, r = 4 * (fl - b * nq);
            part[q][u] = (f < nf && o0 + q < (sec ? own1 : own0))
                             ? __ldcg(reinterpret_cast<const float4*>(slot_of(sec, o0 + q) + size_t(b) * R + r))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
        for (int q = 0; q < OC; ++q)
#pragma unroll
          for (int u = 0; u < U; ++u)
            if (o0 + q < (f0 + u * kThreads >= nf0 ? own1 : own0)) add4(v[u], part[q][u]);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int f = f0 + u * kThreads;
        if (f >= nf) continue;
        const bool sec = f >= nf0;
        const int fl = f - (sec ? nf0 : 0), nq = sec ? nq1 : nq0, b = fl / nq, r = 4 * (fl - b * nq);
        const int Rt = sec ? y1.Rt : y0.Rt;
        float* yr = (sec ? y1.y : y0.y) + size_t(b) * (sec ? y1.ld : y0.ld) + r;
        const float vv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (r + i < Rt) yr[i] = vv[i];
      }
    }
  };

  if (part0 || part1) {
    __syncthreads();
    // Thread 0 counts the CTA in on its first tile, thread 32 on its last, at the same time. Each atomic is
    // acq_rel at GPU scope: the release publishes the CTA's slot writes (ordered before it by the barrier), the
    // acquire makes the other owners' slots visible to the reduction that follows.
    if (tid == 0 || tid == 32) {
      const bool last = tid == 32;
      if (last ? part1 : part0) {
        const int t = last ? tlast : tfirst;
        int first;
        const int own = tile_owners(t, first);
        cta_flags[last] = atom_add_acq_rel(&p.arrive[t], 1u) == unsigned(own - 1);
      } else {
        cta_flags[last] = 0;
      }
    }
    __syncthreads();
    const int ntiles = cta_flags[0] + cta_flags[1];
    if (ntiles > 0) reduce_tiles(cta_flags[0] ? tfirst : tlast, tlast, ntiles);
    if (tid == 0) {
      if (cta_flags[0]) p.arrive[tfirst] = 0u;
      if (cta_flags[1]) p.arrive[tlast] = 0u;
    }
  } else if (tid == 0) {
    cta_flags[0] = cta_flags[1] = 0;
  }
  if (!p.swiglu) return;

  // SwiGLU epilogue. This CTA wrote the final y of its whole tiles and of the shared tiles it reduced.
  const int tiles_here = tlast - tfirst + 1;
  for (int c0 = 0; c0 < tiles_here; c0 += kEpiChunk) {
    __syncthreads();  // this CTA's y writes (and the previous chunk's epilogue) are done
    if (tid == 0) {
      int n = 0;
      for (int k = c0; k < min(tiles_here, c0 + kEpiChunk); ++k) {
        const int t = tfirst + k;
        const bool whole = L <= t * G && H >= (t + 1) * G;
        const bool reduced = (t == tfirst && part0 && cta_flags[0]) || (t == tlast && part1 && cta_flags[1]);
        if (!whole && !reduced) continue;
        const int m = mat_of_tile(p, t), tl = m == 0 ? t : t - p.tile_start[1];
        if (atom_add_acq_rel(&p.pair[tl], 1u) == 1u) epi_tiles[n++] = tl;
      }
      *epi_count = n;
    }
    __syncthreads();
    for (int k = 0; k < *epi_count; ++k) {
      const int tl = epi_tiles[k];
      const int N = p.N[0], Rt = min(R, N - tl * R);
      const size_t row0 = size_t(tl) * R;
      for (int e = tid; e < Rt * B; e += kThreads) {
        const int b = e / Rt, r = e - b * Rt;
        const size_t at = size_t(b) * N + row0 + r;
        const float g = __ldcg(p.y[0] + at), u = __ldcg(p.y[1] + at);
        const float silu = g / (1.f + expf(-g));
        p.h[at] = __bfloat16_as_ushort(__float2bfloat16_rn(silu * u));
      }
      if (tid == 0) p.pair[tl] = 0u;
    }
  }
}

// ===================================================================================== record-batch kernel
// Every batch B in {1, 2, 4, 8, 16}. One CTA per SM whose warps (16 at B = 1, 2; 12 at B = 4, 8, 16: as many as
// the registers of each batch size allow) work on the CTA's records together:
//  - The CTA's record range is cut into batches of up to NB records of one row tile. Records stream HBM ->
//    shared memory by cp.async.bulk (one copy per record plus one 128-byte copy per batch row of the column's
//    activations), S batches ahead, each record in its own slot with its own mbarrier.
//  - Each record gets a meta job one batch before its units run: validate it, build the width masks and item
//    starts per 32-row word, the group sums of x (and for B <= 2 the activation and nibble tables), and note where
//    its buckets lie.
//  - Per batch, the jobs are the width-bucket units of its records and the meta jobs of the next batch. Every warp
//    computes the same job list from the meta blocks and takes the jobs whose cost midpoint falls in its share of
//    the total, so the split is even to about one unit. A unit writes s * dot for each of its items (and batch
//    rows) into the record's result buffer: on CUDA cores for B <= 2, through mma.sync for B = 4, 8, 16.
//  - One CTA barrier per batch. Then each warp adds the results of its own 32-row words to its accumulators,
//    record by record in record order (row r takes the result of its item: the start of its bucket in its word
//    plus the rows of the same width before it), so every row is summed in a fixed order and results are bitwise
//    identical from run to run. The batch's slots are refilled right after the barrier.
//  - A finished tile goes to y when the CTA holds all its records, else to the CTA's partial slot; finish_cta then
//    reduces the tiles shared with neighbouring CTAs and runs the SwiGLU epilogue.
constexpr int kCudaCoreWarps = 16;      // warps per CTA at B = 1, 2
// smallest batch on the tensor-core units; at batch 4 the n8 mma tile is half used, and building the operands,
// not the mma, is the cost, so batch 4 gains from leaving its per-row CUDA-core loops
constexpr int kTensorCoreMinBatch = 4;
// floats per item in a record's result buffer: B, padded by 4 at B >= 8 so that the row pass's 16-byte loads of
// consecutive items (and the units' 8-byte stores) fall in distinct shared-memory banks
__host__ __device__ constexpr int res_stride(int B) { return B >= 8 ? B + 4 : B; }
constexpr int kCtasPerSM = 1;   // CTAs per SM in its grid
template <int B> struct KCfg {
  static constexpr bool kTC = B >= kTensorCoreMinBatch;             // tensor-core units
  static constexpr int kWarps = B <= 2 ? kCudaCoreWarps : 12;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kIPU = kTC ? 32 : 32 / B;                    // items per 4-, 8-bit unit
  static constexpr int kWordsPerWarp = (32 + kWarps - 1) / kWarps;  // row-pass words per warp (R <= 1024)
};
constexpr int kMaxNB = 7;        // records per batch: the 1 + 4 NB job segments of a batch fit in one warp
constexpr int kMaxSets = 4;      // batches in flight
constexpr int kDirCache = 512;   // directory entries cached in shared memory

// Per-record metadata, written by the record's meta job one batch before its units run, in two blocks.
// Table block (256-byte aligned; read only by the units, so two sets serve alternate batches). The tables exist
// for B <= 2 only, and each is built only when the record has rows of the widths that read it:
//  t1 [B][16][16] f32: 1-bit nibble tables; entry n of position p is the sum of x[4p + i] over the set bits i of n
//  t2 [B][32][16] f32: 2-bit nibble tables; entry n of position p is (n & 3) x[2p] + (n >> 2) x[2p + 1]
//  xt [2][B][64] f32:  x, and x * 2^-shift for the magic-number expansion of 4-bit codes
//  sg [B] f32:         group sums of x
//  fl [16] i32:        bad, scales offset, bucket counts n[4], bucket code offsets c[4], bucket item starts i[4]
// Row block (read by the row pass, which can run while the next batch's units write: three sets):
//  mk [4][32] u32:     width masks per 32-row word;  pf [4][32] u16: item index of the word's first row per width
//  wc [64] u32:        the record's width-code words
//  kind (i32):         0 mixed widths; 1 bad record (adds nothing); 2 + c every row has width code c, so the item
//                      index of a row is the row itself
struct MetaOff {
  int t1, t2, xt, sg, fl, size;      // table block
  int mk, pf, wc, kind, row_size;    // row block
  __host__ __device__ explicit MetaOff(int B) {
    const int tb = B >= kTensorCoreMinBatch ? 0 : B;   // the tensor-core path needs no activation tables
    t1 = 0;
    t2 = 1024 * tb;
    xt = t2 + 2048 * tb;
    sg = xt + 512 * tb;
    fl = sg + 4 * (B < 4 ? 4 : B);     // group sums of x, one per batch row
    size = (fl + 64 + 255) & ~255;
    mk = 0;
    pf = 512;
    wc = 768;
    kind = 1024;
    row_size = 1040;
  }
};

// The CTA's batches, in order: records [L, H) cut at row-tile boundaries, then into runs of at most NB records.
// Also tracks where batch's first record streams: slot s0 of the NS slots, its use u0 of that slot (mbarrier phase).
struct BatchIt {
  int rb, re, t, te, s0, u0;
  int H, G, NB, NS;
  __device__ void init(int L, int H_, int G_, int NB_, int NS_) {
    H = H_; G = G_; NB = NB_; NS = NS_;
    rb = L;
    t = L / G;
    te = min(H, (t + 1) * G);
    re = min(te, rb + NB);
    s0 = 0;
    u0 = 0;
  }
  __device__ bool valid() const { return rb < H; }
  __device__ void next() {
    s0 += re - rb;
    if (s0 >= NS) { s0 -= NS; ++u0; }
    rb = re;
    if (rb >= te) {
      ++t;
      te = min(H, te + G);
    }
    re = min(te, rb + NB);
  }
  // slot and mbarrier phase parity of record rb + pos
  __device__ void slot_of(int pos, int& slot, unsigned& parity) const {
    slot = s0 + pos;
    int u = u0;
    if (slot >= NS) { slot -= NS; ++u; }
    parity = unsigned(u) & 1u;
  }
};

// 1- and 2-bit groups against nibble tables of B batch rows at shared address tab (256-byte aligned, table b at
// tab + TB * b; entry n of position p at + 64 p + 4 n): one lookup per nibble. Each nibble times 4 is moved by one
// byte permute into the low byte of the table address. KB = 1: 16 positions of four 1-bit codes; KB = 2: 32
// positions of two 2-bit codes. Returns sum_i q_i x_i per row in d.
template <int KB, int B>
__device__ __forceinline__ void dot_lut(const uint32_t (&w)[2 * KB], uint32_t tab, float (&d)[B]) {
  constexpr int TB = KB == 1 ? 1024 : 2048;
  constexpr int NA = B == 1 ? 8 : 4;
  float a[B][NA];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int i = 0; i < NA; ++i) a[b][i] = 0.f;
  static_for<0, 2 * KB>([&](auto mc) {
    constexpr int m = decltype(mc)::value;                                        // word m: positions 8m .. 8m + 7
    const uint32_t e = (w[m] << 2) & 0x3C3C3C3Cu, o = (w[m] >> 2) & 0x3C3C3C3Cu;  // nibbles 2k / 2k+1, times 4
    static_for<0, 4>([&](auto kc) {
      constexpr int k = decltype(kc)::value;
      const uint32_t ae = __byte_perm(e, tab, 0x7650u + k), ao = __byte_perm(o, tab, 0x7650u + k);
      static_for<0, B>([&](auto bc) {
        constexpr int b = decltype(bc)::value;
        a[b][(2 * k) % NA] += lds32f_off<TB * b + 64 * (8 * m + 2 * k)>(ae);
        a[b][(2 * k + 1) % NA] += lds32f_off<TB * b + 64 * (8 * m + 2 * k + 1)>(ao);
      });
    });
  });
#pragma unroll
  for (int b = 0; b < B; ++b) {
    if constexpr (NA == 8) d[b] = ((a[b][0] + a[b][1]) + (a[b][2] + a[b][3])) + ((a[b][4] + a[b][5]) + (a[b][6] + a[b][7]));
    else d[b] = (a[b][0] + a[b][1]) + (a[b][2] + a[b][3]);
  }
}

// 1- or 2-bit units [lo, hi) of 32 items each (lane = item, all B batch rows): s * (sum q x - off * S_g) into
// res[item][b], off = 1/2 (1-bit) or 2 - corr (2-bit).
template <int KB, int B>
__device__ __forceinline__ void unit_range_lut(int n, int lo, int hi, int lane, uint32_t codes, uint32_t scales,
                                               uint32_t res, uint32_t tab, const float (&sg)[B], float off) {
  for (int u = lo; u < hi; ++u) {
    const int jj = 32 * u + lane;
    if (jj >= n) break;
    uint32_t w[2 * KB];
    if constexpr (KB == 1) {
      const uint2 v = lds64(codes + 8 * jj);
      w[0] = v.x; w[1] = v.y;
    } else {
      const uint4 v = lds128(codes + 16 * jj);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    }
    float d[B];
    dot_lut<KB, B>(w, tab, d);
    const float s = __half2float(__ushort_as_half((unsigned short)lds16(scales + 2 * jj)));
#pragma unroll
    for (int b = 0; b < B; ++b) sts32f(res + 4 * (jj * B + b), s * (d[b] - off * sg[b]));
  }
}

// 4- and 8-bit units [lo, hi) of 32 / B items each (lane = item * B + b): s * dot of the item's group with batch
// row b into res[item][b]. codes, scales and res are byte addresses of item 0 of the bucket.
template <int KB, int B>
__device__ __forceinline__ void unit_range(int n, int lo, int hi, int lane, uint32_t codes, uint32_t scales,
                                           uint32_t res, const float (&xr)[64], float sg, float corr) {
  constexpr int IPU = 32 / B;
  const int sub = lane / B, b = lane - sub * B;
  for (int u = lo; u < hi; ++u) {
    const int jj = IPU * u + sub;
    if (jj >= n) break;
    float d;
    if constexpr (KB == 4) {
      const uint4 a = lds128(codes + 32 * jj), c = lds128(codes + 32 * jj + 16);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
      d = dot_magic<4>(w, xr, sg, corr);
    } else {
      uint32_t w[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 a = lds128(codes + 64 * jj + 16 * q);
        w[4 * q] = a.x; w[4 * q + 1] = a.y; w[4 * q + 2] = a.z; w[4 * q + 3] = a.w;
      }
      d = dot_b8(w, xr, sg, corr);
    }
    sts32f(res + 4 * (jj * B + b), __half2float(__ushort_as_half((unsigned short)lds16(scales + 2 * jj))) * d);
  }
}

// Tensor-core A fragments (batch 4, 8, 16). Lane (g, t) = (lane / 4, lane % 4) of an mma.sync m16n8k16 holds, for
// each k-step ks, two bf16 pairs of A row g: logical columns 16 ks + 2t + {0, 1} and + {8, 9}. Logical columns
// map to codes so that lane t reads one contiguous run of its item's codes: 16t .. 16t + 15, as 8 bf16 pairs
// a[0..7], a[2 ks] and a[2 ks + 1] feeding k-step ks. The activations take the same map (tc_x_frags), so any
// pairing of codes into registers is allowed; each width takes its cheapest exact one:
//   1, 2 bits: pairs of adjacent codes (c_2r, c_2r+1), exact values q - c from a 16-entry nibble table;
//   4 bits:    (c_r, c_r+4) and (c_8+r, c_12+r), r < 4: the bf16 bits 0x4300 | q = 128 + q, minus 136: q - 8;
//   8 bits:    adjacent codes, q - 128 through fp32 (2^23 + q as bits, minus 2^23 + 128), then packed to bf16.
// Every value is a small integer or half-integer, exact in bf16; the grid offset left over in the 4- and 8-bit
// forms, (2^(k-1) - c) x group sum of x, seeds the accumulator.
template <int KB>
__device__ __forceinline__ void tc_a_frag(uint32_t addr, bool ok, uint32_t tab, uint32_t (&a)[8]) {
  if constexpr (KB == 1) {
    const uint32_t h = ok ? lds16(addr) : 0u;
    const uint32_t e = (h << 3) & 0x7878u, o = (h >> 1) & 0x7878u;   // nibbles times 8: codes 0-3, 8-11 / 4-7, 12-15
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint2 lo = lds64(__byte_perm(e, tab, 0x7650u + k)), hi = lds64(__byte_perm(o, tab, 0x7650u + k));
      a[4 * k] = lo.x; a[4 * k + 1] = lo.y; a[4 * k + 2] = hi.x; a[4 * k + 3] = hi.y;
    }
  } else if constexpr (KB == 2) {
    const uint32_t w = ok ? lds32(addr) : 0u;
    const uint32_t e = (w << 2) & 0x3C3C3C3Cu, o = (w >> 2) & 0x3C3C3C3Cu;   // nibbles times 4
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      a[2 * k] = lds32(__byte_perm(e, tab, 0x7650u + k));       // codes 4k, 4k + 1
      a[2 * k + 1] = lds32(__byte_perm(o, tab, 0x7650u + k));   // codes 4k + 2, 4k + 3
    }
  } else if constexpr (KB == 4) {
    uint2 w = make_uint2(0u, 0u);
    if (ok) w = lds64(addr);
    const __nv_bfloat162 m136 = __floats2bfloat162_rn(136.f, 136.f);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint32_t v = (((r < 4 ? w.x : w.y) >> (4 * (r & 3))) & 0x000F000Fu) | 0x43004300u;
      const __nv_bfloat162 d = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v), m136);
      a[r] = *reinterpret_cast<const uint32_t*>(&d);
    }
  } else {
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (ok) w = lds128(addr);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    const float2 neg = make_float2(-8388736.f, -8388736.f);   // -(2^23 + 128)
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint32_t x = ww[r >> 1], j = 2 * (r & 1);
      const float2 q = fadd2(make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7440u + j)),
                                         __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7441u + j))), neg);
      a[r] = bf16x2_bits(q.x, q.y);
    }
  }
}

// The activations of one group as mma B fragments in the code map of tc_a_frag: lane (g, t), batch row
// b = 8 nt + g, k-step ks: bfr[ks][nt][0] pairs with a[2 ks], bfr[ks][nt][1] with a[2 ks + 1]. xb: the staged
// bf16 activations [B][64] of the record's group. perm4: the 4-bit map, else adjacent pairs.
template <int B>
__device__ __forceinline__ void tc_x_frags(uint32_t xb, int lane, bool perm4, uint32_t (&bfr)[4][(B + 7) / 8][2]) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < (B + 7) / 8; ++nt) {
    if (nt * 8 + g >= B) {   // batch 4: columns 4..7 of the n8 tile are zero
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) bfr[ks][nt][0] = bfr[ks][nt][1] = 0u;
      continue;
    }
    const uint32_t row = xb + 128 * (nt * 8 + g) + 32 * t;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      if (perm4) {   // codes base, base + 4 | base + 1, base + 5 with base = 2 ks + 4 (ks / 2)
        const uint32_t base = 2 * ks + 4 * (ks >> 1);
        const uint32_t u = lds32(row + 2 * base), v = lds32(row + 2 * base + 8);
        bfr[ks][nt][0] = __byte_perm(u, v, 0x5410u);
        bfr[ks][nt][1] = __byte_perm(u, v, 0x7632u);
      } else {       // codes 4 ks, 4 ks + 1 | 4 ks + 2, 4 ks + 3
        const uint2 u = lds64(row + 8 * ks);
        bfr[ks][nt][0] = u.x;
        bfr[ks][nt][1] = u.y;
      }
    }
  }
}

// Tensor-core units [lo, hi) of one width bucket, 32 items each (B = 4, 8, 16): per 16-item m-tile, lane (g, t) builds
// the fragments of items 16 mt + g and + 8 from their codes, mma.sync m16n8k16 (bf16 in, fp32 accumulate, seeded
// with the grid-offset term init[nt]) against the activations bfr, and writes s times each result to res[item][b].
template <int B, int KB>
__device__ __forceinline__ void unit_range_tc(int n, int lo, int hi, int lane, uint32_t codes, uint32_t scales,
                                              uint32_t res, uint32_t tab, const float2 (&init)[(B + 7) / 8],
                                              const uint32_t (&bfr)[4][(B + 7) / 8][2]) {
  constexpr int NTL = (B + 7) / 8;
  const int g = lane >> 2, t = lane & 3;
  for (int u = lo; u < hi; ++u) {
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int i0 = 32 * u + 16 * mt + g, i1 = i0 + 8;
      const bool ok0 = i0 < n, ok1 = i1 < n;
      uint32_t a0[8], a1[8];
      tc_a_frag<KB>(codes + 8 * KB * i0 + 2 * KB * t, ok0, tab, a0);
      tc_a_frag<KB>(codes + 8 * KB * i1 + 2 * KB * t, ok1, tab, a1);
      float c4[NTL][4];
#pragma unroll
      for (int nt = 0; nt < NTL; ++nt) {
        c4[nt][0] = c4[nt][2] = init[nt].x;
        c4[nt][1] = c4[nt][3] = init[nt].y;
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int nt = 0; nt < NTL; ++nt)
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
              "{%0,%1,%2,%3};"
              : "+f"(c4[nt][0]), "+f"(c4[nt][1]), "+f"(c4[nt][2]), "+f"(c4[nt][3])
              : "r"(a0[2 * ks]), "r"(a1[2 * ks]), "r"(a0[2 * ks + 1]), "r"(a1[2 * ks + 1]), "r"(bfr[ks][nt][0]),
                "r"(bfr[ks][nt][1]));
      // c4[nt][0..1]: item i0, batch rows 8 nt + 2t + {0, 1}; c4[nt][2..3]: item i1
      const float s0 = ok0 ? __half2float(__ushort_as_half((unsigned short)lds16(scales + 2 * i0))) : 0.f;
      const float s1 = ok1 ? __half2float(__ushort_as_half((unsigned short)lds16(scales + 2 * i1))) : 0.f;
#pragma unroll
      for (int nt = 0; nt < NTL; ++nt) {
        const int b = nt * 8 + 2 * t;
        if (B % 8 != 0 && b >= B) continue;   // batch 4: only lanes t < 2 hold real columns
        if (ok0) sts64f(res + 4 * (i0 * res_stride(B) + b), s0 * c4[nt][0], s0 * c4[nt][1]);
        if (ok1) sts64f(res + 4 * (i1 * res_stride(B) + b), s1 * c4[nt][2], s1 * c4[nt][3]);
      }
    }
  }
}

// First job (of count jobs costing c each, in the segment starting at cost s0) whose cost midpoint reaches
// cut2 / (2 W): the smallest j >= 0 with W (2 s0 + c (2j + 1)) >= cut2, at most count. The quotient comes from a
// float division (all values are below 2^24), corrected to the exact integer.
__device__ __forceinline__ int first_job(int cut2, int s0, int c, int count, int W) {
  if (count <= 0) return 0;
  const int num = cut2 - (2 * s0 + c) * W;
  if (num <= 0) return 0;
  const int den = 2 * W * c;
  int j = __float2int_ru(__fdividef(float(num), float(den)));
  if (j * den < num) ++j;
  else if (j > 0 && (j - 1) * den >= num) --j;
  return min(count, j);
}

template <int B>
__global__ void __launch_bounds__(KCfg<B>::kThreads, 1) vbq_kernel(const __grid_constant__ Params params) {
  using C = KCfg<B>;
  constexpr int W = C::kWarps, IPU = C::kIPU, NWW = C::kWordsPerWarp;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint64_t bar_full[kMaxNB * kMaxSets];
  __shared__ int slot_bad[kMaxNB * kMaxSets];
  __shared__ volatile int cta_abort;
  __shared__ int cta_flags[2];
  __shared__ int epi_tiles[kEpiChunk];
  __shared__ int epi_count;
  __shared__ __align__(16) Params p;
  // tensor-core path: nibble tables of exact A values. [0, 32): 1-bit, 16 entries of four bf16 (bit_i(n) - 1/2);
  // [64, 80): 2-bit on the default grid, 16 entries of two bf16 (q - 3/2, q = n & 3 and n >> 2); [128, 144): 2-bit
  // on the symmetric grid (q - 1)
  __shared__ __align__(256) uint32_t tc_tab[192];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  static_assert(sizeof(Params) % 4 == 0 && sizeof(Params) / 4 <= C::kThreads, "parameter copy");
  if (tid < int(sizeof(Params) / 4))
    reinterpret_cast<uint32_t*>(&p)[tid] = reinterpret_cast<const uint32_t*>(&params)[tid];
  if (tid == 0) cta_abort = 0;
  if constexpr (C::kTC) {
    if (tid < 32) {   // 1-bit: entry tid / 2, bf16 pair (tid & 1)
      const int nib = tid >> 1, i0 = 2 * (tid & 1);
      tc_tab[tid] = bf16x2_bits(float((nib >> i0) & 1) - 0.5f, float((nib >> (i0 + 1)) & 1) - 0.5f);
    } else if (tid < 64) {   // 2-bit: default grid at [64, 80), symmetric grid at [128, 144)
      const int e = tid & 15;
      const bool sym = tid >= 48;
      const float c = sym ? 1.f : 1.5f;
      tc_tab[(sym ? 128 : 64) + e] = bf16x2_bits(float(e & 3) - c, float(e >> 2) - c);
    }
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int G = p.G, NB = p.NB, S = p.S, cta = blockIdx.x;
  __shared__ int lo_hi[2];
  if (p.balanced) {
    if (warp < 2) {
      const int v = byte_lo(p, cta + warp, lane);
      if (lane == 0) lo_hi[warp] = v;
    }
    __syncthreads();
  }
  const int L = p.balanced ? lo_hi[0] : rec_lo(p, cta), H = p.balanced ? lo_hi[1] : rec_lo(p, cta + 1);
  if (H <= L) return;  // nothing to read or write
  const MetaOff mo(B);
  const int NS = NB * S;

  // -- directory cache: entries (start, end) of records [dbase, dbase + kDirCache), in 16-byte units
  uint32_t* dlo = reinterpret_cast<uint32_t*>(smem + p.dir_off);
  uint32_t* dhi = dlo + kDirCache;
  int dbase = L;
  auto fill_dir = [&](int from) {
    for (int j = from + tid; j < min(H, from + kDirCache); j += C::kThreads) {
      const int m = mat_of_rec(p, j);
      const int jl = j - (m == 0 ? 0 : m == 1 ? p.rec_start[1] : m == 2 ? p.rec_start[2] : p.rec_start[3]);
      const uint32_t* dir = pick(p.dir, m);
      dlo[j - from] = __ldg(dir + jl);
      dhi[j - from] = __ldg(dir + jl + 1);
    }
  };
  fill_dir(L);
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&bar_full[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // Record j streams into slot (j - L) % NS; its use of that slot is number (j - L) / NS, which sets the mbarrier
  // phase parity (BatchIt tracks both). A batch is issued only when the batch S before it is done, and the S
  // batches from there hold at most NS records, so a slot's previous record is always finished.
  auto slot_ptr = [&](int slot) { return smem + slot * p.stage_size; };
  // metadata blocks from the first 256-byte boundary of their region (the nibble-table lookups put an index in
  // the low byte of a table address); the plan leaves 256 bytes of room for this
  const int meta0 = int(((smem_u32(smem + p.meta_off) + 255u) & ~255u) - smem_u32(smem));
  auto meta_ptr = [&](int tp, int pos) { return smem + meta0 + (tp * NB + pos) * p.meta_rec; };   // table block
  auto row_ptr = [&](int mp, int pos) { return smem + p.row_off + (mp * NB + pos) * MetaOff(B).row_size; };
  // result set of a batch: alternate sets when there are two, else the one set (and a barrier after each row pass)
  const bool two_sets = B < 8 || p.res_sets > 1;   // one set is planned only for batch 8, 16
  const uint32_t res0 = smem_u32(smem + p.res_off);
  const int res_rec = p.res_rec;
  auto res_addr = [=](int rp, int pos) { return res0 + uint32_t(((two_sets ? rp : 0) * NB + pos) * res_rec); };

  // Bulk copies of batch `it` (warp 0, one record per lane, at most NB <= 32): the records (with_rec) and the
  // activation rows (with_x) into their slots. The mbarrier of a slot expects both.
  auto issue = [&](const BatchIt& it, bool with_rec, bool with_x) {
    const int j = it.rb + lane;
    if (j >= it.re) return;
    int slot;
    unsigned parity;
    it.slot_of(lane, slot, parity);
    uint64_t* bar = &bar_full[slot];
    unsigned char* dst = slot_ptr(slot);
    if (with_rec) {
      const uint32_t a = dlo[j - dbase], b = dhi[j - dbase];
      const int m = mat_of_rec(p, j);
      const unsigned bytes = 16u * (b - a);
      if (b < a || b > pick(p.units_total, m) || bytes > unsigned(p.stage_bytes)) {  // not what was promised
        slot_bad[slot] = 1;
        atomicOr(p.status, kStatusOversize);
        mbar_arrive(bar);
        return;
      }
      slot_bad[slot] = 0;
      mbar_arrive_tx(bar, bytes + 128u * B);
      if (j != p.withhold) tma_bulk_load(dst, pick(p.recs, m) + 16ull * a, bytes, bar);
    }
    if (with_x && !slot_bad[slot] && j != p.withhold) {
      const int g = j - it.t * G;
#pragma unroll
      for (int bb = 0; bb < B; ++bb)
        tma_bulk_load(dst + p.stage_bytes + 128 * bb, p.x + size_t(bb) * p.K + size_t(g) * 64, 128u, bar);
    }
  };

  // Meta job of record pos of batch `it` (whole warp) into table set tp and row set mp: wait for the record,
  // validate it, write its metadata.
  auto meta_job = [&](const BatchIt& it, int pos, int tp, int mp) {
    int slot;
    unsigned parity;
    it.slot_of(pos, slot, parity);
    const unsigned char* st = slot_ptr(slot);
    const uint32_t sa = smem_u32(st);
    unsigned char* mb = meta_ptr(tp, pos);
    unsigned char* rb_ = row_ptr(mp, pos);
    bool ok = mbar_wait(&bar_full[slot], parity, p.status, &cta_abort, p.wait_ns);
    ok = __all_sync(0xFFFFFFFFu, ok) && !slot_bad[slot];
    const int Rt = tile_out(p, it.t).Rt;
    int n0 = 0, n1 = 0, n2 = 0, n3 = 0;
    if (ok) {
      const uint2 cnt = lds64(sa);
      n0 = cnt.x & 0xFFFF; n1 = cnt.x >> 16; n2 = cnt.y & 0xFFFF; n3 = cnt.y >> 16;
      const Rec rc(Rt, n0, n1, n2, n3);
      if (n0 + n1 + n2 + n3 != Rt || rc.c3 + 64 * n3 > p.stage_bytes) {
        if (lane == 0) atomicOr(p.status, kStatusRecord);
        ok = false;
      }
    }
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
    unsigned long long v = 0, pre = 0;
    if (ok) {
      // width masks and item starts per 32-row word (lane = word)
      const int nvalid = max(0, min(32, Rt - 32 * lane));
      if (nvalid > 0) {
        const uint2 v2 = lds64(sa + 8 + 8 * lane);
        v = (unsigned long long)v2.x | ((unsigned long long)v2.y << 32);
      }
      const uint32_t lo = even_bits(v), hi = even_bits(v >> 1);
      const uint32_t valid = nvalid >= 32 ? 0xFFFFFFFFu : ((1u << nvalid) - 1u);
      m0 = ~hi & ~lo & valid;
      m1 = ~hi & lo & valid;
      m2 = hi & ~lo & valid;
      m3 = hi & lo & valid;
      const unsigned long long mine = (unsigned long long)__popc(m0) | ((unsigned long long)__popc(m1) << 16) |
                                      ((unsigned long long)__popc(m2) << 32) | ((unsigned long long)__popc(m3) << 48);
      unsigned long long incl = mine;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += u;
      }
      pre = incl - mine;
      const unsigned long long tot = __shfl_sync(0xFFFFFFFFu, incl, 31);
      if (tot != ((unsigned long long)n0 | ((unsigned long long)n1 << 16) | ((unsigned long long)n2 << 32) |
                  ((unsigned long long)n3 << 48))) {
        if (lane == 0) atomicOr(p.status, kStatusRecord);
        ok = false;
      }
    }
    int* fl = reinterpret_cast<int*>(mb + mo.fl);
    if (ok) {
      uint32_t* mk = reinterpret_cast<uint32_t*>(rb_ + mo.mk);
      uint16_t* pf = reinterpret_cast<uint16_t*>(rb_ + mo.pf);
      uint32_t* wc = reinterpret_cast<uint32_t*>(rb_ + mo.wc);
      mk[lane] = m0; mk[32 + lane] = m1; mk[64 + lane] = m2; mk[96 + lane] = m3;
      pf[lane] = uint16_t(pre & 0xFFFFull);
      pf[32 + lane] = uint16_t(n0 + int((pre >> 16) & 0xFFFFull));
      pf[64 + lane] = uint16_t(n0 + n1 + int((pre >> 32) & 0xFFFFull));
      pf[96 + lane] = uint16_t(n0 + n1 + n2 + int(pre >> 48));
      wc[2 * lane] = uint32_t(v);
      wc[2 * lane + 1] = uint32_t(v >> 32);
      if constexpr (C::kTC) {
        // group sums of x per batch row: 32 / B lanes per row, each over 2B consecutive values
        constexpr int LPR = 32 / B, VPL = 64 / LPR;
        const uint32_t xa = smem_u32(st + p.stage_bytes) + 128 * (lane / LPR) + 2 * VPL * (lane % LPR);
        float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < VPL / 8; ++q) {
          const uint4 u = lds128(xa + 16 * q);
          const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            acc2 = fadd2(acc2, make_float2(__uint_as_float(uu[i] << 16), __uint_as_float(uu[i] & 0xFFFF0000u)));
        }
        float sgl = acc2.x + acc2.y;
#pragma unroll
        for (int off = 1; off < LPR; off <<= 1) sgl += __shfl_xor_sync(0xFFFFFFFFu, sgl, off);
        if (lane % LPR == 0) reinterpret_cast<float*>(mb + mo.sg)[lane / LPR] = sgl;
      } else {
      // activation tables [2][B][64]: x, x * 2^-shift (4-bit codes); group sums
      const uint16_t* xg = reinterpret_cast<const uint16_t*>(st + p.stage_bytes);
      float* xv = reinterpret_cast<float*>(mb + mo.xt);
      float* sgv = reinterpret_cast<float*>(mb + mo.sg);
      const float s4a = __uint_as_float(uint32_t(127 - code_shift<4>(lane)) << 23);
      const float s4b = __uint_as_float(uint32_t(127 - code_shift<4>(32 + lane)) << 23);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const float x0 = __uint_as_float(uint32_t(xg[b * 64 + lane]) << 16);
        const float x1 = __uint_as_float(uint32_t(xg[b * 64 + 32 + lane]) << 16);
        xv[b * 64 + lane] = x0;
        xv[b * 64 + 32 + lane] = x1;
        if (n2 > 0) {   // the 4-bit copy: only for a record with 4-bit rows
          xv[(B + b) * 64 + lane] = x0 * s4a;
          xv[(B + b) * 64 + 32 + lane] = x1 * s4b;
        }
        float sg = x0 + x1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sg += __shfl_xor_sync(0xFFFFFFFFu, sg, off);
        if (lane == 0) sgv[b] = sg;
      }
      __syncwarp();
      // nibble tables, each only for a record with rows of its width. 1-bit: lane = (position p, half h) builds
      // entries 8h .. 8h + 7 of position p. 2-bit: lane = position p (codes 2p, 2p + 1) builds its 16 entries.
      const uint32_t xa = smem_u32(mb + mo.xt);
      const int pp = lane >> 1, hh = lane & 1;
      const uint32_t t1a = smem_u32(mb + mo.t1) + 64 * pp + 32 * hh, t2a = smem_u32(mb + mo.t2) + 64 * lane;
#pragma unroll
      for (int b = 0; b < B; ++b) {
        if (n0 > 0) {
        const float4 q = lds128f(xa + 256 * b + 16 * pp);
        const float base = hh ? q.w : 0.f;
        const float e1 = base + q.x, e2 = base + q.y, e3 = e1 + q.y;
        const uint32_t lo4[4] = {__float_as_uint(base), __float_as_uint(e1), __float_as_uint(e2), __float_as_uint(e3)};
        const uint32_t hi4[4] = {__float_as_uint(base + q.z), __float_as_uint(e1 + q.z), __float_as_uint(e2 + q.z),
                                 __float_as_uint(e3 + q.z)};
        sts128(t1a + 1024 * b, lo4);
        sts128(t1a + 1024 * b + 16, hi4);
        }
        if (n1 == 0) continue;
        const uint2 xp = lds64(xa + 256 * b + 8 * lane);
        const float xa0 = __uint_as_float(xp.x), xb0 = __uint_as_float(xp.y);
#pragma unroll
        for (int qb = 0; qb < 4; ++qb) {
          const float hb = float(qb) * xb0;
          const uint32_t row[4] = {__float_as_uint(hb), __float_as_uint(fmaf(1.f, xa0, hb)),
                                   __float_as_uint(fmaf(2.f, xa0, hb)), __float_as_uint(fmaf(3.f, xa0, hb))};
          sts128(t2a + 2048 * b + 16 * qb, row);
        }
      }
      }
      if (lane == 0) {
        const Rec rc(Rt, n0, n1, n2, n3);
        fl[1] = rc.sc;
        fl[2] = n0; fl[3] = n1; fl[4] = n2; fl[5] = n3;
        fl[6] = rc.c0; fl[7] = rc.c1; fl[8] = rc.c2; fl[9] = rc.c3;
        fl[10] = 0; fl[11] = n0; fl[12] = n0 + n1; fl[13] = n0 + n1 + n2;
      }
    } else if (lane == 0) {
      fl[2] = fl[3] = fl[4] = fl[5] = 0;
    }
    if (lane == 0) {
      fl[0] = ok ? 0 : 1;
      // 1: bad record (adds nothing); 2 + c: every row has width code c (item index = row); 0: mixed widths
      const int uni = n0 == Rt ? 0 : n1 == Rt ? 1 : n2 == Rt ? 2 : n3 == Rt ? 3 : -1;
      *reinterpret_cast<int*>(rb_ + mo.kind) = !ok ? 1 : uni >= 0 ? 2 + uni : 0;
    }
  };

  // Jobs of batch `cur` (meta set mp, result set rp) for this warp: the units of its records, buckets in the order
  // 1, 2, 8, 4 bits, then the meta jobs of the next batch `nxt` (into meta set mpn). 1- and 2-bit units take 32
  // items (all batch rows per lane); 4- and 8-bit units 32 / B items.
  auto jobs = [&](const BatchIt& cur, const BatchIt& nxt, int rp, int mpn) {
    const int nrec = cur.re - cur.rb;
    // segment of this lane: 4 pos + q = record pos, bucket order q; lane 31 = the meta jobs
    int count = 0, cost = 0;
    if (lane == 31) {
      count = nxt.valid() ? nxt.re - nxt.rb : 0;
      cost = p.cost[4];
    } else if (lane < 4 * nrec) {
      const int pos = lane >> 2, q = lane & 3;
      const int k = q == 0 ? 0 : q == 1 ? 1 : q == 2 ? 3 : 2;
      const int* fl = reinterpret_cast<const int*>(meta_ptr(rp, pos) + mo.fl);
      const int nk = fl[2 + k];
      count = (k < 2 || C::kTC) ? (nk + 31) >> 5 : (nk + IPU - 1) / IPU;
      cost = p.cost[k];
    }
    const int tot = count * cost;
    int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += u;
    }
    const int s0 = incl - tot, total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    const int jlo = first_job(2 * total * warp, s0, max(cost, 1), count, W);
    const int jhi = first_job(2 * total * (warp + 1), s0, max(cost, 1), count, W);
    unsigned todo = __ballot_sync(0xFFFFFFFFu, jhi > jlo);
    float xr[C::kTC ? 1 : 64];
    int loaded = -1;
    const bool grid_sym = pick(p.sym, mat_of_tile(p, cur.t)) != 0;
    const float corr = grid_sym ? 1.f : 0.5f;
    uint32_t bfr[4][C::kTC ? (B + 7) / 8 : 1][2];   // tensor-core path: the record's activations as B fragments
    while (todo) {
      const int sgi = __ffs(todo) - 1;
      todo &= todo - 1;
      const int lo = __shfl_sync(0xFFFFFFFFu, jlo, sgi), hi = __shfl_sync(0xFFFFFFFFu, jhi, sgi);
      if (sgi == 31) {
        for (int jb = lo; jb < hi; ++jb) meta_job(nxt, jb, rp ^ 1, mpn);
        continue;
      }
      const int pos = sgi >> 2, q = sgi & 3;
      const int k = q == 0 ? 0 : q == 1 ? 1 : q == 2 ? 3 : 2;
      const unsigned char* mb = meta_ptr(rp, pos);
      const int* fl = reinterpret_cast<const int*>(mb + mo.fl);
      const int nk = fl[2 + k], cb = fl[6 + k], ib = fl[10 + k], sc = fl[1];
      int slot;
      unsigned parity;
      cur.slot_of(pos, slot, parity);
      const uint32_t sa = smem_u32(slot_ptr(slot));
      const uint32_t res = res_addr(rp, pos) + 4 * res_stride(B) * ib;
      const uint32_t sca = sa + sc + 2 * ib;
      if constexpr (C::kTC) {
        const int kind = pos * 2 + (k == 2 ? 1 : 0);   // the 4-bit code map differs from the others'
        if (loaded != kind) {
          tc_x_frags<B>(smem_u32(slot_ptr(slot) + p.stage_bytes), lane, k == 2, bfr);
          loaded = kind;
        }
        // accumulator seed: (2^(k-1) - c) sum x for 4 and 8 bits (1/2 on the default grid, 1 on the symmetric)
        float2 init[(B + 7) / 8];
        const float* sgv = reinterpret_cast<const float*>(mb + mo.sg);
        const float f = k < 2 ? 0.f : corr;
#pragma unroll
        for (int nt = 0; nt < (B + 7) / 8; ++nt) {
          const int b = nt * 8 + 2 * (lane & 3);
          const float2 sg2 = b < B ? *reinterpret_cast<const float2*>(sgv + b) : make_float2(0.f, 0.f);
          init[nt] = make_float2(f * sg2.x, f * sg2.y);
        }
        const uint32_t tb = smem_u32(tc_tab);
        if (k == 0) unit_range_tc<B, 1>(nk, lo, hi, lane, sa + cb, sca, res, tb, init, bfr);
        else if (k == 1) unit_range_tc<B, 2>(nk, lo, hi, lane, sa + cb, sca, res, tb + (grid_sym ? 512 : 256), init, bfr);
        else if (k == 2) unit_range_tc<B, 4>(nk, lo, hi, lane, sa + cb, sca, res, tb, init, bfr);
        else unit_range_tc<B, 8>(nk, lo, hi, lane, sa + cb, sca, res, tb, init, bfr);
      } else {
      if (k < 2) {
        float sgb[B];
#pragma unroll
        for (int b = 0; b < B; ++b) sgb[b] = reinterpret_cast<const float*>(mb + mo.sg)[b];
        if (k == 0) unit_range_lut<1, B>(nk, lo, hi, lane, sa + cb, sca, res, smem_u32(mb + mo.t1), sgb, 0.5f);
        else unit_range_lut<2, B>(nk, lo, hi, lane, sa + cb, sca, res, smem_u32(mb + mo.t2), sgb, 2.f - corr);
        continue;
      }
      const int tbl = k == 2 ? 1 : 0;
      const int b = lane % B;
      if (loaded != pos * 2 + tbl) {
        const uint32_t xa = smem_u32(mb + mo.xt) + 256 * (tbl * B + b);
#pragma unroll
        for (int qq = 0; qq < 16; ++qq) {
          const float4 f = lds128f(xa + 16 * qq);
          xr[4 * qq] = f.x; xr[4 * qq + 1] = f.y; xr[4 * qq + 2] = f.z; xr[4 * qq + 3] = f.w;
        }
        loaded = pos * 2 + tbl;
      }
      const float sg = reinterpret_cast<const float*>(mb + mo.sg)[b];
      if (k == 2) unit_range<4, B>(nk, lo, hi, lane, sa + cb, sca, res, xr, sg, corr);
      else unit_range<8, B>(nk, lo, hi, lane, sa + cb, sca, res, xr, sg, corr);
      }
    }
  };

  // -- prologue: the first S batches' records, then (once the kernel before this one has finished, under
  // programmatic dependent launch) their activations; the meta jobs of batch 0
  BatchIt cur, nxt, iss;
  cur.init(L, H, G, NB, NS);
  iss = cur;
  if (warp == 0)
    for (int n = 0; n < S && iss.valid(); ++n, iss.next()) issue(iss, true, false);
  else
    for (int n = 0; n < S && iss.valid(); ++n) iss.next();
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (warp == 0) {
    __syncwarp();
    BatchIt it = cur;
    for (; it.rb < iss.rb; it.next()) issue(it, false, true);
  }
  for (int pos = warp; pos < cur.re - cur.rb; pos += W) meta_job(cur, pos, 0, 0);
  // every thread leaves each barrier with the same verdict on the CTA's abort flag
  bool aborted = __syncthreads_or(cta_abort != 0) != 0;

  float acc[NWW][B];
#pragma unroll
  for (int ww = 0; ww < NWW; ++ww)
#pragma unroll
    for (int b = 0; b < B; ++b) acc[ww][b] = 0.f;
  int mp = 0, rp = 0;  // meta set (batch index % 3) and result set (batch index % 2) of the current batch
  // Row pass of batch bt (row set mp_, result set rp_): this warp's words, records in order. First every record's
  // item index for the row (independent loads, issued together), then the results added in record order. At a
  // tile end (tile_end: the next batch is in another tile, or there is none), this CTA's share of the tile goes to
  // y or to its partial slot.
  auto row_pass = [&](int t, int nrec, int mp_, int rp_, bool tile_end) {
    const TileOut to = tile_out(p, t);
    const int Rt = to.Rt;
#pragma unroll
    for (int ww = 0; ww < NWW; ++ww) {
      const int word = warp + ww * W, r = 32 * word + lane;
      if (32 * word >= Rt) continue;
      int item[kMaxNB];
#pragma unroll
      for (int pos = 0; pos < kMaxNB; ++pos) {
        item[pos] = -1;
        if (pos < nrec && r < Rt) {
          const unsigned char* rm = row_ptr(mp_, pos);
          const int kd = *reinterpret_cast<const int*>(rm + mo.kind);
          // the mixed-width item index, its loads issued alongside kind's (the meta job writes the masks of every
          // record, so they are valid for one-width records too)
          const uint32_t* mk = reinterpret_cast<const uint32_t*>(rm + mo.mk);
          const uint16_t* pf = reinterpret_cast<const uint16_t*>(rm + mo.pf);
          const uint32_t wcw = reinterpret_cast<const uint32_t*>(rm + mo.wc)[r >> 4];
          const int c = int(wcw >> (2 * (r & 15))) & 3;
          const int it = pf[c * 32 + word] + __popc(mk[c * 32 + word] & ((1u << lane) - 1u));
          item[pos] = kd >= 2 ? r : kd ? -1 : it;   // one width: the items are the rows; a bad record adds nothing
        }
      }
#pragma unroll
      for (int pos = 0; pos < kMaxNB; ++pos)
        if (item[pos] >= 0) {
          const uint32_t res = res_addr(rp_, pos) + 4 * (item[pos] * res_stride(B));
          if constexpr (B >= 4) {
#pragma unroll
            for (int b = 0; b < B; b += 4) {
              const float4 v = lds128f(res + 4 * b);
              acc[ww][b] += v.x; acc[ww][b + 1] += v.y; acc[ww][b + 2] += v.z; acc[ww][b + 3] += v.w;
            }
          } else {
#pragma unroll
            for (int b = 0; b < B; ++b) acc[ww][b] += lds32f(res + 4 * b);
          }
        }
    }
    if (!tile_end) return;
    const bool whole = L <= t * G && H >= (t + 1) * G;
    float* slot = p.partial + size_t(cta + t) * p.R * B;
#pragma unroll
    for (int ww = 0; ww < NWW; ++ww) {
      const int r = 32 * (warp + ww * W) + lane;
      if (r < Rt) {
#pragma unroll
        for (int b = 0; b < B; ++b) {
          if (whole) to.y[size_t(b) * to.ld + r] = acc[ww][b];
          else slot[b * p.R + r] = acc[ww][b];
        }
      }
#pragma unroll
      for (int b = 0; b < B; ++b) acc[ww][b] = 0.f;
    }
  };

  // At B >= 4 with two result sets, batch n's row pass runs after the warp's jobs of batch n + 1, before the
  // barrier that ends them: a warp that finishes its units early sums rows instead of waiting. (Batch n + 1's
  // units write the other result set; the row, result and table sets batch n's row pass reads are next written by
  // batch n + 2's and n + 3's meta jobs and units, which start after that barrier.) At B <= 2 the row pass is short
  // and follows the batch's own barrier (measured faster there). With one set, a second barrier guards the set.
  constexpr bool kDefer = B >= 4;
  int pt = 0, pn = 0, pmp = 0, prp = 0;   // the previous batch: tile, records, row and result sets
  bool have_prev = false;
  while (!aborted) {
    const bool live = cur.valid();   // one more round after the last batch, for its row pass
    int mpn = 0;
    if (live) {
      nxt = cur;
      nxt.next();
      mpn = mp == 2 ? 0 : mp + 1;
      jobs(cur, nxt, rp, mpn);
    }
    if (kDefer && two_sets && have_prev) row_pass(pt, pn, pmp, prp, !live || pt != cur.t);
    if (!live) break;
    aborted = __syncthreads_or(cta_abort != 0) != 0;
    if (aborted) break;
    // refill the slots of batch n with batch n + S (their records and activation rows)
    if (iss.valid()) {
      if (iss.re > dbase + kDirCache) {  // uniform: every thread takes this branch together
        dbase = iss.rb;
        fill_dir(iss.rb);
        __syncthreads();
      }
      if (warp == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(iss, true, true);
      }
      iss.next();
    }
    if (kDefer && two_sets) {
      pt = cur.t;
      pn = cur.re - cur.rb;
      pmp = mp;
      prp = rp;
      have_prev = true;
    } else {
      row_pass(cur.t, cur.re - cur.rb, mp, rp, !nxt.valid() || nxt.t != cur.t);
      if (!two_sets) __syncthreads();   // the next batch's units overwrite the one result set
    }
    cur = nxt;
    mp = mpn;
    rp ^= 1;
  }
  if (aborted) {
    // wait (bounded) for the copies still in flight before the CTA exits; publish nothing. Only the last use of
    // each slot can still be in flight: the last NS records issued, which end at iss.rb.
    if (warp == 0) {
      const int j = iss.rb - NS + lane;
      if (lane < NS && j >= L) mbar_drain(&bar_full[(j - L) % NS], ((j - L) / NS) & 1, p.wait_ns);
    }
    return;
  }
  finish_cta<B, C::kThreads>(p, L, H, cta_flags, epi_tiles, &epi_count);
}

// ------------------------------------------------------------------------------------------ launch plan
struct Plan {
  int grid, threads, S, stage_bytes, stage_size, res_off, smem;
  int NB, RS, meta_off, row_off, dir_off, res_rec, meta_rec;  // record-batch kernel
  uint64_t ws_bytes, status_off, counters_off;
};


inline int num_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// The matrices of one launch, seen as one record sequence.
struct Problem {
  int nmat;
  const vbq_desc* d[kMaxMats];
  int R, K, G;
  long long T, nrec;
  uint64_t max_record_bytes;
};

inline bool desc_ok(const vbq_desc* d) {
  return d->version == 1 && (d->flags & ~unsigned(VBQ_FLAG_GRID_SYMMETRIC)) == 0 && d->N >= 1 && d->K >= 64 && d->K % 64 == 0 && d->G == d->K / 64 && d->R >= 16 &&
         d->R <= kMaxTileRows && d->R % 16 == 0 && d->T == (d->N + d->R - 1) / d->R && d->N <= INT32_MAX &&
         d->K <= INT32_MAX && d->dir_offset == 64 && d->rec_offset > d->dir_offset &&
         d->total_bytes > d->rec_offset && d->max_record_bytes >= 32 &&
         d->max_record_bytes <= d->total_bytes - d->rec_offset && d->max_record_bytes % 16 == 0 &&
         (d->total_bytes - d->rec_offset) % 16 == 0 && (d->total_bytes - d->rec_offset) / 16 <= 0xFFFFFFFFull;
}

// Validates the descriptors of one launch: 1..kMaxMats consistent matrices with equal K (SHAPE) and equal tile
// rows (TILE), and record and tile counts that fit the kernel's 32-bit indices (FORMAT).
inline int make_problem(int nmat, const vbq_desc* const* d, Problem& pr) {
  if (!d) return VBQ_ERR_NULL;
  if (nmat < 1 || nmat > kMaxMats) return VBQ_ERR_SHAPE;
  pr.nmat = nmat;
  pr.T = pr.nrec = 0;
  pr.max_record_bytes = 0;
  for (int m = 0; m < nmat; ++m) {
    if (!d[m]) return VBQ_ERR_NULL;
    if (!desc_ok(d[m])) return VBQ_ERR_FORMAT;
    if (d[m]->K != d[0]->K) return VBQ_ERR_SHAPE;
    if (d[m]->R != d[0]->R) return VBQ_ERR_TILE;
    pr.d[m] = d[m];
    pr.T += d[m]->T;
    pr.nrec += d[m]->T * d[m]->G;
    if (d[m]->max_record_bytes > pr.max_record_bytes) pr.max_record_bytes = d[m]->max_record_bytes;
  }
  pr.R = int(d[0]->R);
  pr.K = int(d[0]->K);
  pr.G = int(d[0]->G);
  if (pr.nrec >= (1ll << 30) || pr.max_record_bytes > (1ull << 30)) return VBQ_ERR_FORMAT;
  return VBQ_OK;
}

// CTAs split the records by estimated cost when record sizes differ much: the largest record over 1.3 times the
// mean (an LM head whose frequent rows are wider, a small last tile); otherwise by count, which needs no directory
// search.
inline bool cost_split(const Problem& pr) {
  uint64_t units = 0;
  for (int m = 0; m < pr.nmat; ++m) units += (pr.d[m]->total_bytes - pr.d[m]->rec_offset) / 16;
  return double(pr.max_record_bytes) > 1.3 * 16.0 * double(units) / double(pr.nrec);
}

// Workspace: partial slots [nCTA + T][B][R] f32 of the row tiles that CTAs share, then an arrival counter and a
// SwiGLU pair counter per tile, then the status word.
inline void plan_workspace(const Problem& pr, int B, Plan& pl) {
  const uint64_t slots = uint64_t(pl.grid) + uint64_t(pr.T);
  pl.counters_off = slots * uint64_t(pr.R) * B * 4;
  pl.ws_bytes = (pl.counters_off + uint64_t(pr.T) * 8 + 4 + 15) / 16 * 16;
  pl.status_off = pl.ws_bytes - 4;
}

// Records per batch NB, batches in flight S and result sets RS: as many records per batch as fit (fewer batches
// cut the per-batch bookkeeping and barriers; measured faster at every batch size), then S = 3 when it fits (the
// meta jobs of a batch read records issued two batches earlier), else 2; at B >= 8 one result set (with a barrier
// after each row pass) before fewer records per batch.
template <int B>
inline bool make_plan_b(const Problem& pr, int sms, Plan& pl) {
  using C = KCfg<B>;
  pl.grid = sms * kCtasPerSM;
  pl.threads = C::kThreads;
  const int R = pr.R;
  pl.stage_bytes = align128i(int(pr.max_record_bytes));
  pl.stage_size = pl.stage_bytes + align128i(128 * B);
  pl.res_rec = align128i(R * res_stride(B) * 4);
  pl.meta_rec = MetaOff(B).size;
  const int dir_bytes = 8 * kDirCache;
  const int nb_want = kMaxNB;
  const MetaOff mo(B);
  auto need = [&](int NB, int S, int RS) {
    return (long long)S * NB * pl.stage_size + (long long)RS * NB * pl.res_rec + 256 + 2ll * NB * pl.meta_rec +
           3ll * NB * mo.row_size + dir_bytes;
  };
  // two result sets let the next batch's units start before every warp has finished this batch's row pass; at
  // B >= 8 (results of 48 or 80 bytes per row) a larger batch with one set measured faster than a smaller with two
  pl.NB = 0;
  for (int NB = nb_want; NB >= 1 && pl.NB == 0; --NB)
    for (int RS = 2; RS >= (B < 8 ? 2 : 1) && pl.NB == 0; --RS)
      for (int S = 3; S >= 2; --S)
        if (need(NB, S, RS) <= kSmemBudget) {
          pl.NB = NB;
          pl.S = S;
          pl.RS = RS;
          break;
        }
  if (pl.NB == 0) return false;
  pl.res_off = pl.S * pl.NB * pl.stage_size;
  pl.meta_off = pl.res_off + pl.RS * pl.NB * pl.res_rec;
  pl.row_off = pl.meta_off + 256 + 2 * pl.NB * pl.meta_rec;
  pl.dir_off = pl.row_off + 3 * pl.NB * mo.row_size;
  pl.smem = pl.dir_off + dir_bytes;
  plan_workspace(pr, B, pl);
  return true;
}

inline bool make_plan(const Problem& pr, int B, int sms, Plan& pl) {
  switch (B) {
    case 1: return make_plan_b<1>(pr, sms, pl);
    case 2: return make_plan_b<2>(pr, sms, pl);
    case 4: return make_plan_b<4>(pr, sms, pl);
    case 8: return make_plan_b<8>(pr, sms, pl);
    default: return make_plan_b<16>(pr, sms, pl);
  }
}

// Test hook (vbq_test_set_fault): a shorter limit for the kernels' bounded waits and one record whose bulk copy
// is never issued, so that a wait runs out. Off by default.
std::atomic<unsigned long long> g_test_wait_ns{0};
std::atomic<long long> g_test_withhold{-1};

template <int B>
int launch(const Problem& pr, const void* const* blobs, const void* x, float* const* ys, void* ws, uint64_t ws_bytes,
           unsigned flags, cudaStream_t stream, uint16_t* h = nullptr, unsigned* status = nullptr) {
  Plan pl;
  if (!make_plan_b<B>(pr, num_sms(), pl)) return VBQ_ERR_FORMAT;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15) || ws_bytes < pl.ws_bytes) return VBQ_ERR_WORKSPACE;
  Params p = {};
  p.nmat = pr.nmat;
  int tiles = 0, recs = 0;
  unsigned long long total16 = 0;
  for (int m = 0; m < kMaxMats; ++m) {
    p.tile_start[m] = tiles;
    p.rec_start[m] = recs;
    if (m >= pr.nmat) continue;
    const vbq_desc* d = pr.d[m];
    const uint8_t* base = static_cast<const uint8_t*>(blobs[m]);
    p.dir[m] = reinterpret_cast<const uint32_t*>(base + d->dir_offset);
    p.recs[m] = base + d->rec_offset;
    p.y[m] = ys[m];
    p.N[m] = int(d->N);
    p.sym[m] = (d->flags & VBQ_FLAG_GRID_SYMMETRIC) ? 1 : 0;
    p.units_total[m] = uint32_t((d->total_bytes - d->rec_offset) / 16);
    p.base16[m] = total16;
    total16 += p.units_total[m];
    tiles += int(d->T);
    recs += int(d->T * d->G);
  }
  p.tile_start[kMaxMats] = tiles;
  p.rec_start[kMaxMats] = recs;
  p.balanced = cost_split(pr) ? 1 : 0;
  // the fixed part of a record's cost, measured on LM heads: four mean records at batch 1 (the per-record work
  // dominates), two at larger batches (the units' share grows with B)
  p.rec_w16 = std::max<unsigned long long>(1, (B == 1 ? 4ull : 2ull) * total16 / unsigned(recs));
  p.total_w = total16 + p.rec_w16 * unsigned(recs);
  p.x = static_cast<const uint16_t*>(x);
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.partial = reinterpret_cast<float*>(w);
  p.arrive = reinterpret_cast<unsigned*>(w + pl.counters_off);
  p.pair = p.arrive + tiles;
  p.swiglu = h != nullptr;
  p.h = h;
  p.status = status ? status : reinterpret_cast<unsigned*>(w + pl.status_off);
  p.K = pr.K; p.G = pr.G; p.R = pr.R; p.T = tiles;
  p.nrec = recs;
  p.S = pl.S;
  p.stage_bytes = pl.stage_bytes;
  p.stage_size = pl.stage_size;
  p.res_off = pl.res_off;
  p.NB = pl.NB;
  p.meta_off = pl.meta_off;
  p.row_off = pl.row_off;
  p.dir_off = pl.dir_off;
  p.res_rec = pl.res_rec;
  p.meta_rec = pl.meta_rec;
  p.res_sets = pl.RS;
  // job costs (about the instructions a warp spends): units of 1-, 2-, 4-, 8-bit groups; a meta job
  // job costs, in scheduler cycles of one lane (integer and packed fp32 instructions take two, fp32 one):
  // 1- and 2-bit units (nibble tables, all batch rows), 4- and 8-bit units (magic-number expansion), a meta job
  // tensor-core batches: units of 32 items (fragment building dominates; mma.sync adds little per unit)
  if (!KCfg<B>::kTC) {
    p.cost[0] = 60 + 20 * B;
    p.cost[1] = 150 + 35 * B;
    p.cost[2] = 285;
    p.cost[3] = 275;
    p.cost[4] = 400 + 100 * B;
  } else {
    p.cost[0] = 110 + 4 * B;
    p.cost[1] = 150 + 4 * B;
    p.cost[2] = 190 + 4 * B;
    p.cost[3] = 260 + 4 * B;
    p.cost[4] = 500;
  }
  const unsigned long long wl = g_test_wait_ns.load();
  p.wait_ns = wl ? wl : kWaitNs;
  const long long wh = g_test_withhold.load();
  p.withhold = (wh >= 0 && wh < recs) ? int(wh) : -1;
  auto kern = vbq_kernel<B>;
  // Opt in to the dynamic shared memory once per device and size.
  static int opted[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& done = opted[dev & 63];
  if (pl.smem > done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem) != cudaSuccess)
      return VBQ_ERR_CUDA;
    done = pl.smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(pl.grid));
  cfg.blockDim = dim3(unsigned(pl.threads));
  cfg.dynamicSmemBytes = size_t(pl.smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (flags & VBQ_LAUNCH_OVERLAP) ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return VBQ_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? VBQ_OK : VBQ_ERR_CUDA;
}

inline bool batch_ok(int B) { return B == 1 || B == 2 || B == 4 || B == 8 || B == 16; }


}  // namespace vbq

extern "C" {

int vbq_workspace_size_multi(int nmat, const vbq_desc* const* d, int B, uint64_t* out_bytes) {
  if (!d || !out_bytes) return VBQ_ERR_NULL;
  if (!vbq::batch_ok(B)) return VBQ_ERR_BATCH;
  vbq::Problem pr;
  if (int st = vbq::make_problem(nmat, d, pr)) return st;
  vbq::Plan pl;
  if (!vbq::make_plan(pr, B, vbq::num_sms(), pl)) return VBQ_ERR_FORMAT;
  *out_bytes = pl.ws_bytes;
  return VBQ_OK;
}

int vbq_plan_info_get(int nmat, const vbq_desc* const* d, int B, int sm_count, vbq_plan_info* out) {
  if (!d || !out) return VBQ_ERR_NULL;
  if (!vbq::batch_ok(B)) return VBQ_ERR_BATCH;
  if (sm_count < 1 || sm_count > 4096) return VBQ_ERR_SHAPE;
  vbq::Problem pr;
  if (int st = vbq::make_problem(nmat, d, pr)) return st;
  vbq::Plan pl;
  if (!vbq::make_plan(pr, B, sm_count, pl)) return VBQ_ERR_FORMAT;
  out->grid = pl.grid;
  out->threads = pl.threads;
  out->records_per_batch = pl.NB;
  out->batches_in_flight = pl.S;
  out->result_sets = pl.RS;
  out->cost_split = vbq::cost_split(pr) ? 1 : 0;
  out->smem_bytes = uint32_t(pl.smem);
  out->workspace_bytes = pl.ws_bytes;
  return VBQ_OK;
}

int vbq_workspace_size(const vbq_desc* d, int B, uint64_t* out_bytes) {
  if (!d) return VBQ_ERR_NULL;
  return vbq_workspace_size_multi(1, &d, B, out_bytes);
}

int vbq_workspace_init(void* workspace, uint64_t workspace_bytes, void* stream) {
  if (!workspace) return VBQ_ERR_NULL;
  if (workspace_bytes == 0) return VBQ_OK;
  return cudaMemsetAsync(workspace, 0, size_t(workspace_bytes), static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? VBQ_OK : VBQ_ERR_CUDA;
}

int vbq_gemm_skinny_multi(int nmat, const vbq_desc* const* d, const void* const* blob_dev, const void* x_bf16,
                          int B, float* const* y, void* workspace, uint64_t workspace_bytes, unsigned flags,
                          void* stream) {
  if (!d || !blob_dev || !x_bf16 || !y) return VBQ_ERR_NULL;
  for (int m = 0; m < nmat && m < vbq::kMaxMats; ++m)
    if (!d[m] || !blob_dev[m] || !y[m]) return VBQ_ERR_NULL;
  if (!vbq::batch_ok(B)) return VBQ_ERR_BATCH;
  if (flags & ~unsigned(VBQ_LAUNCH_OVERLAP)) return VBQ_ERR_FLAGS;
  vbq::Problem pr;
  if (int st = vbq::make_problem(nmat, d, pr)) return st;
  if (reinterpret_cast<uintptr_t>(x_bf16) & 15) return VBQ_ERR_ALIGN;
  for (int m = 0; m < nmat; ++m)
    if ((reinterpret_cast<uintptr_t>(blob_dev[m]) & 15) || (reinterpret_cast<uintptr_t>(y[m]) & 3))
      return VBQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (B) {
    case 1: return vbq::launch<1>(pr, blob_dev, x_bf16, y, workspace, workspace_bytes, flags, st);
    case 2: return vbq::launch<2>(pr, blob_dev, x_bf16, y, workspace, workspace_bytes, flags, st);
    case 4: return vbq::launch<4>(pr, blob_dev, x_bf16, y, workspace, workspace_bytes, flags, st);
    case 8: return vbq::launch<8>(pr, blob_dev, x_bf16, y, workspace, workspace_bytes, flags, st);
    default: return vbq::launch<16>(pr, blob_dev, x_bf16, y, workspace, workspace_bytes, flags, st);
  }
}

int vbq_workspace_size_swiglu(const vbq_desc* gate, const vbq_desc* up, int B, uint64_t* out_bytes) {
  if (!gate || !up) return VBQ_ERR_NULL;
  if (gate->N != up->N) return VBQ_ERR_SHAPE;
  const vbq_desc* d[2] = {gate, up};
  return vbq_workspace_size_multi(2, d, B, out_bytes);
}

int vbq_gemm_swiglu(const vbq_desc* gate, const vbq_desc* up, const void* blob_gate, const void* blob_up,
                    const void* x_bf16, int B, float* y_gate, float* y_up, void* h_bf16, void* workspace,
                    uint64_t workspace_bytes, unsigned flags, void* stream) {
  if (!gate || !up || !blob_gate || !blob_up || !x_bf16 || !y_gate || !y_up || !h_bf16) return VBQ_ERR_NULL;
  if (!vbq::batch_ok(B)) return VBQ_ERR_BATCH;
  if (flags & ~unsigned(VBQ_LAUNCH_OVERLAP)) return VBQ_ERR_FLAGS;
  const vbq_desc* d[2] = {gate, up};
  vbq::Problem pr;
  if (int st = vbq::make_problem(2, d, pr)) return st;
  if (gate->N != up->N) return VBQ_ERR_SHAPE;
  const void* blobs[2] = {blob_gate, blob_up};
  float* ys[2] = {y_gate, y_up};
  if ((reinterpret_cast<uintptr_t>(x_bf16) & 15) || (reinterpret_cast<uintptr_t>(h_bf16) & 1)) return VBQ_ERR_ALIGN;
  for (int m = 0; m < 2; ++m)
    if ((reinterpret_cast<uintptr_t>(blobs[m]) & 15) || (reinterpret_cast<uintptr_t>(ys[m]) & 3)) return VBQ_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint16_t* h = static_cast<uint16_t*>(h_bf16);
  switch (B) {
    case 1: return vbq::launch<1>(pr, blobs, x_bf16, ys, workspace, workspace_bytes, flags, st, h);
    case 2: return vbq::launch<2>(pr, blobs, x_bf16, ys, workspace, workspace_bytes, flags, st, h);
    case 4: return vbq::launch<4>(pr, blobs, x_bf16, ys, workspace, workspace_bytes, flags, st, h);
    case 8: return vbq::launch<8>(pr, blobs, x_bf16, ys, workspace, workspace_bytes, flags, st, h);
    default: return vbq::launch<16>(pr, blobs, x_bf16, ys, workspace, workspace_bytes, flags, st, h);
  }
}

int vbq_gemm_skinny_ex(const vbq_desc* d, const void* blob_dev, const void* x_bf16, int B, float* y,
                       void* workspace, uint64_t workspace_bytes, unsigned flags, void* stream) {
  if (!d || !blob_dev || !x_bf16 || !y) return VBQ_ERR_NULL;
  return vbq_gemm_skinny_multi(1, &d, &blob_dev, x_bf16, B, &y, workspace, workspace_bytes, flags, stream);
}

int vbq_gemm_skinny(const vbq_desc* d, const void* blob_dev, const void* x_bf16, int B, float* y,
                    void* workspace, uint64_t workspace_bytes, void* stream) {
  return vbq_gemm_skinny_ex(d, blob_dev, x_bf16, B, y, workspace, workspace_bytes, 0u, stream);
}

int vbq_gemv(const vbq_desc* d, const void* blob_dev, const void* x_bf16, float* y, void* workspace,
             uint64_t workspace_bytes, void* stream) {
  return vbq_gemm_skinny(d, blob_dev, x_bf16, 1, y, workspace, workspace_bytes, stream);
}

int vbq_test_set_fault(uint64_t wait_limit_ns, int64_t withheld_record) {
  vbq::g_test_wait_ns.store(wait_limit_ns);
  vbq::g_test_withhold.store(withheld_record < 0 ? -1 : withheld_record);
  return VBQ_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------ allocation-free variant
// Scratch for vbq_gemm_skinny_noalloc: one fixed buffer per device, created when the library is loaded on that
// device and kept until the process exits. It replaces the caller-provided workspace of vbq_gemm_skinny: the
// split-K partial sums and the counters take its first 16 MiB - 256 bytes, and its last 256 bytes hold the status
// word, at a fixed place so that vbq_noalloc_status can read it.
namespace vbq {
constexpr uint64_t kStaticScratchBytes = 16ull << 20;  // 16 MiB
constexpr uint64_t kStaticStatusOff = kStaticScratchBytes - 256;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device. In host code the array's name is only a host-side
// stand-in, so the address is looked up once per device with cudaGetSymbolAddress (that device current) and
// kept; a device reset (cudaDeviceReset) would void it.
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
  if (!vbq::batch_ok(B)) return VBQ_ERR_BATCH;
  if (!vbq::desc_ok(d)) return VBQ_ERR_FORMAT;
  uint64_t need = 0;
  if (int st = vbq_workspace_size(d, B, &need)) return st;
  if (need > vbq::kStaticStatusOff) return VBQ_ERR_SCRATCH_LIMIT;
  if ((reinterpret_cast<uintptr_t>(x_bf16) & 15) || (reinterpret_cast<uintptr_t>(blob_dev) & 15) ||
      (reinterpret_cast<uintptr_t>(y) & 3))
    return VBQ_ERR_ALIGN;
  void* scratch = nullptr;
  if (int st = vbq::static_scratch(&scratch)) return st;
  unsigned char* base = static_cast<unsigned char*>(scratch);
  vbq::Problem pr;
  if (int st = vbq::make_problem(1, &d, pr)) return st;
  vbq::Plan pl;
  if (!vbq::make_plan(pr, B, vbq::num_sms(), pl)) return VBQ_ERR_FORMAT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The buffer keeps the previous call's contents: clear the arrival counters and the status word, which the
  // kernel needs at zero. The partial-sum area is always written before it is read.
  if (cudaMemsetAsync(base + pl.counters_off, 0, size_t(need - pl.counters_off), st) != cudaSuccess ||
      cudaMemsetAsync(base + vbq::kStaticStatusOff, 0, 4, st) != cudaSuccess)
    return VBQ_ERR_CUDA;
  unsigned* status = reinterpret_cast<unsigned*>(base + vbq::kStaticStatusOff);
  const void* blobs[1] = {blob_dev};
  float* ys[1] = {y};
  switch (B) {
    case 1: return vbq::launch<1>(pr, blobs, x_bf16, ys, base, need, 0u, st, nullptr, status);
    case 2: return vbq::launch<2>(pr, blobs, x_bf16, ys, base, need, 0u, st, nullptr, status);
    case 4: return vbq::launch<4>(pr, blobs, x_bf16, ys, base, need, 0u, st, nullptr, status);
    case 8: return vbq::launch<8>(pr, blobs, x_bf16, ys, base, need, 0u, st, nullptr, status);
    default: return vbq::launch<16>(pr, blobs, x_bf16, ys, base, need, 0u, st, nullptr, status);
  }
}

extern "C" int vbq_noalloc_status(uint32_t* status_host, void* stream) {
  if (!status_host) return VBQ_ERR_NULL;
  void* scratch = nullptr;
  if (int st = vbq::static_scratch(&scratch)) return st;
  return cudaMemcpyAsync(status_host, static_cast<unsigned char*>(scratch) + vbq::kStaticStatusOff, 4,
                         cudaMemcpyDeviceToHost, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? VBQ_OK : VBQ_ERR_CUDA;
}
