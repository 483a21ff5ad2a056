/*
 * VBQ oracle: a plain, slow, obviously correct CPU implementation of what the
 * VBQ fused dequantize-and-multiply path computes.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this file. The product path never does.
 * It shares no code with the CUDA library: it has its own packer, CRC, and
 * float decoders, written from the packed-format-v1 specification and from the IEEE
 * definitions.
 *
 * Method source: "Variable Bit-width Quantization: Learning Per-Group Precision
 * for 'Bigger-but-Smaller' Language Models", section 3.1 (contiguous groups of
 * 64 weights, one scale and one width from {1,2,4,8} per group) and section 6,
 * paragraph "Fused kernels over packed weights" (the kernel dequantizes each
 * group with its scale and accumulates the matrix-vector product).
 * The default value grid w = s*(q - (2^k-1)/2) with q in [0, 2^k) is this
 * project's reading: the paper's Eq. 1 uses a symmetric integer grid for k >= 2,
 * which a 2^k-level unsigned code cannot hold, while its 1-bit case (sign times a
 * per-group magnitude) is exactly +-s/2 here. Header flag bit 0 selects Eq. 1's
 * own grid for k >= 2 instead: w = s*(q - (2^(k-1)-1)), q in [0, 2^k - 2].
 *
 * Arithmetic is fp64. Every dequantized weight s*(q-c) is exact in fp64
 * (an 11-bit significand times a value with at most 9 significant bits), and
 * every bf16 activation is exact in fp64. The dot product is summed in index
 * order i = 0..K-1, with no blocking or reordering.
 *
 * Parity of the matvec and the dequant map is pinned by tests against exact
 * rational arithmetic, closed forms, and numpy/torch float decoders. Pack and
 * unpack are pinned by a hand-derived golden blob, a single-code bit-position
 * sweep, and round trips.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Status values. They are the same numbers as the C-ABI's documented codes,
 * defined here independently. */
enum {
  O_OK = 0, O_ERR_NULL = -1, O_ERR_SHAPE = -2, O_ERR_WIDTH = -3, O_ERR_CODE_RANGE = -4,
  O_ERR_BUFFER_TOO_SMALL = -5, O_ERR_BAD_MAGIC = -6, O_ERR_VERSION = -7, O_ERR_CRC = -8,
  O_ERR_BATCH = -9, O_ERR_ALIGN = -10, O_ERR_CUDA = -11, O_ERR_TILE = -12, O_ERR_FORMAT = -13,
  O_ERR_FLAGS = -16
};

/* Header flag bit 0: widths >= 2 use the paper's symmetric integer grid (Eq. 1, section 3.1):
 * w = s * (q - (2^(k-1) - 1)), q in [0, 2^k - 2]. 1-bit groups keep w = s * (q - 1/2) in both grids. */
#define O_FLAG_SYM 1u

/* Offset c of the value grid w = s * (q - c) for width k under header flags f. */
static double grid_offset(int k, unsigned f) {
  if ((f & O_FLAG_SYM) && k >= 2) return (double)((1 << (k - 1)) - 1);
  return ((double)((1 << k) - 1)) / 2.0;
}
static unsigned max_code(int k, unsigned f) {
  return ((f & O_FLAG_SYM) && k >= 2) ? (1u << k) - 2u : (1u << k) - 1u;
}

#define O_MAGIC 0x31514256u
#define O_VERSION 1u

/* ---------------------------------------------------------------- CRC-32 */
/* IEEE 802.3 CRC-32, bit by bit: reflected polynomial 0xEDB88320, initial
 * value and final XOR 0xFFFFFFFF. */
uint32_t vbqo_crc32(const uint8_t* p, uint64_t n) {
  uint32_t c = 0xFFFFFFFFu;
  for (uint64_t i = 0; i < n; ++i) {
    c ^= p[i];
    for (int b = 0; b < 8; ++b) c = (c & 1u) ? (c >> 1) ^ 0xEDB88320u : (c >> 1);
  }
  return c ^ 0xFFFFFFFFu;
}

/* ------------------------------------------------------- float decoders */
/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double vbqo_half_to_double(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  double v;
  if (e == 0) v = ldexp((double)m, -24);                 /* 2^-14 * m/2^10 */
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp(1.0 + (double)m / 1024.0, e - 15);
  return s ? -v : v;
}

/* bfloat16: the upper half of an IEEE binary32: 1 sign, 8 exponent bits (bias
 * 127), 7 fraction bits. */
double vbqo_bf16_to_double(uint16_t b) {
  int s = (b >> 15) & 1, e = (b >> 7) & 0xFF, m = b & 0x7F;
  double v;
  if (e == 0) v = ldexp((double)m, -133);                /* 2^-126 * m/2^7 */
  else if (e == 255) v = m ? NAN : INFINITY;
  else v = ldexp(1.0 + (double)m / 128.0, e - 127);
  return s ? -v : v;
}

/* ------------------------------------------------------------- helpers */
static uint64_t a16(uint64_t x) { return (x + 15u) & ~(uint64_t)15u; }
static void put16(uint8_t* p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void put32(uint8_t* p, uint32_t v) { for (int i = 0; i < 4; ++i) p[i] = (uint8_t)(v >> (8 * i)); }
static void put64(uint8_t* p, uint64_t v) { for (int i = 0; i < 8; ++i) p[i] = (uint8_t)(v >> (8 * i)); }
static uint16_t get16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t get32(const uint8_t* p) { uint32_t v = 0; for (int i = 3; i >= 0; --i) v = (v << 8) | p[i]; return v; }
static uint64_t get64(const uint8_t* p) { uint64_t v = 0; for (int i = 7; i >= 0; --i) v = (v << 8) | p[i]; return v; }

static int width_code(int k) { return k == 1 ? 0 : k == 2 ? 1 : k == 4 ? 2 : k == 8 ? 3 : -1; }

static int check_shape(int64_t N, int64_t K, int64_t R) {
  if (N < 1 || K < 64 || K % 64 != 0 || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return O_ERR_SHAPE;
  if (R < 16 || R > 1024 || R % 16 != 0) return O_ERR_TILE;
  return O_OK;
}

static int check_logical(int64_t N, int64_t K, const uint8_t* widths, const uint8_t* codes, unsigned f) {
  int64_t G = K / 64;
  for (int64_t i = 0; i < N * G; ++i)
    if (width_code(widths[i]) < 0) return O_ERR_WIDTH;
  if (codes) {
    for (int64_t r = 0; r < N; ++r)
      for (int64_t c = 0; c < K; ++c) {
        int k = widths[r * G + c / 64];
        if (codes[r * K + c] > max_code(k, f)) return O_ERR_CODE_RANGE;
      }
  }
  return O_OK;
}

/* Size in bytes of record (t, g) of packed format v1: counts, width codes, scales, then the
 * four code buckets, each part padded to 16 bytes. */
static uint64_t record_bytes(int64_t Rt, const int64_t cnt[4]) {
  uint64_t sz = a16(8 + 4 * (uint64_t)((Rt + 15) / 16));
  sz += a16(2 * (uint64_t)Rt);
  sz += a16(8 * (uint64_t)cnt[0]) + 16 * (uint64_t)cnt[1] + 32 * (uint64_t)cnt[2] + 64 * (uint64_t)cnt[3];
  return sz;
}

static void column_counts(int64_t N, int64_t G, int64_t r0, int64_t Rt, int64_t g,
                          const uint8_t* widths, int64_t cnt[4]) {
  (void)N;
  cnt[0] = cnt[1] = cnt[2] = cnt[3] = 0;
  for (int64_t j = 0; j < Rt; ++j) cnt[width_code(widths[(r0 + j) * G + g])]++;
}

int vbqo_packed_size(int64_t N, int64_t K, int64_t R, const uint8_t* widths, uint64_t* out_bytes) {
  if (!widths || !out_bytes) return O_ERR_NULL;
  int st = check_shape(N, K, R);
  if (st) return st;
  st = check_logical(N, K, widths, NULL, 0);
  if (st) return st;
  int64_t G = K / 64, T = (N + R - 1) / R;
  uint64_t rec = 0;
  for (int64_t t = 0; t < T; ++t) {
    int64_t r0 = t * R, Rt = (N - r0 < R) ? N - r0 : R;
    for (int64_t g = 0; g < G; ++g) {
      int64_t cnt[4];
      column_counts(N, G, r0, Rt, g, widths, cnt);
      rec += record_bytes(Rt, cnt);
    }
  }
  *out_bytes = 64 + a16(4 * (uint64_t)(T * G + 1)) + rec;
  return O_OK;
}

/* Pack logical (widths, scales, codes) into a canonical blob. Row-major logical
 * arrays: widths[N*G] in {1,2,4,8}, scales[N*G] fp16 bit patterns,
 * codes[N*K] with codes < 2^width. */
int vbqo_pack_ex(int64_t N, int64_t K, int64_t R, const uint8_t* widths, const uint16_t* scales,
                 const uint8_t* codes, unsigned flags, uint8_t* out, uint64_t cap, uint64_t* written) {
  if (!widths || !scales || !codes || !out) return O_ERR_NULL;
  if (flags & ~O_FLAG_SYM) return O_ERR_FLAGS;
  int st = check_shape(N, K, R);
  if (st) return st;
  st = check_logical(N, K, widths, codes, flags);
  if (st) return st;
  uint64_t total;
  st = vbqo_packed_size(N, K, R, widths, &total);
  if (st) return st;
  if (cap < total) return O_ERR_BUFFER_TOO_SMALL;
  memset(out, 0, total);

  int64_t G = K / 64, T = (N + R - 1) / R;
  uint64_t dir_off = 64, rec_off = 64 + a16(4 * (uint64_t)(T * G + 1));
  uint64_t pos = 0; /* bytes from rec_off */
  for (int64_t t = 0; t < T; ++t) {
    int64_t r0 = t * R, Rt = (N - r0 < R) ? N - r0 : R;
    for (int64_t g = 0; g < G; ++g) {
      put32(out + dir_off + 4 * (uint64_t)(t * G + g), (uint32_t)(pos / 16));
      uint8_t* rec = out + rec_off + pos;
      int64_t cnt[4];
      column_counts(N, G, r0, Rt, g, widths, cnt);
      for (int c = 0; c < 4; ++c) put16(rec + 2 * c, (uint16_t)cnt[c]);
      /* width codes, 16 rows per u32 word */
      for (int64_t j = 0; j < Rt; ++j) {
        uint32_t c = (uint32_t)width_code(widths[(r0 + j) * G + g]);
        uint8_t* wp = rec + 8 + 4 * (j / 16);
        put32(wp, get32(wp) | (c << (2 * (j % 16))));
      }
      uint64_t scale_off = a16(8 + 4 * (uint64_t)((Rt + 15) / 16));
      uint64_t code_off = scale_off + a16(2 * (uint64_t)Rt);
      /* items: bucket by bucket, rows ascending */
      int64_t item = 0;
      uint64_t cpos = code_off;
      for (int c = 0; c < 4; ++c) {
        int k = 1 << c;
        for (int64_t j = 0; j < Rt; ++j) {
          int64_t r = r0 + j;
          if (widths[r * G + g] != k) continue;
          put16(rec + scale_off + 2 * (uint64_t)item, scales[r * G + g]);
          uint8_t* gp = rec + cpos;
          for (int i = 0; i < 64; ++i) {
            uint32_t q = codes[r * K + 64 * g + i];
            for (int b = 0; b < k; ++b) {
              uint64_t bit = (uint64_t)k * i + b;
              if ((q >> b) & 1u) gp[bit / 8] |= (uint8_t)(1u << (bit % 8));
            }
          }
          cpos += 8 * (uint64_t)k;
          ++item;
        }
        if (c == 0) cpos = code_off + a16(8 * (uint64_t)cnt[0]);
      }
      pos += record_bytes(Rt, cnt);
    }
  }
  put32(out + dir_off + 4 * (uint64_t)(T * G), (uint32_t)(pos / 16));

  uint8_t* h = out;
  put32(h + 0, O_MAGIC);
  put16(h + 4, O_VERSION);
  put16(h + 6, (uint16_t)flags);
  put32(h + 8, (uint32_t)N);
  put32(h + 12, (uint32_t)K);
  put32(h + 16, (uint32_t)G);
  put32(h + 20, (uint32_t)R);
  put32(h + 24, (uint32_t)T);
  put32(h + 28, 0);
  put64(h + 32, dir_off);
  put64(h + 40, rec_off);
  put64(h + 48, total);
  put32(h + 56, vbqo_crc32(out + 64, total - 64));
  put32(h + 60, vbqo_crc32(out, 60));
  if (written) *written = total;
  return O_OK;
}

int vbqo_pack(int64_t N, int64_t K, int64_t R, const uint8_t* widths, const uint16_t* scales,
              const uint8_t* codes, uint8_t* out, uint64_t cap, uint64_t* written) {
  return vbqo_pack_ex(N, K, R, widths, scales, codes, 0u, out, cap, written);
}

/* Header check in the documented order: size, magic, version, header CRC,
 * field consistency, total size, body CRC. */
int vbqo_read_header_ex(const uint8_t* blob, uint64_t size, int64_t* N, int64_t* K, int64_t* R,
                        uint64_t* total, unsigned* flags) {
  if (!blob) return O_ERR_NULL;
  if (size < 64) return O_ERR_BUFFER_TOO_SMALL;
  if (get32(blob) != O_MAGIC) return O_ERR_BAD_MAGIC;
  if (get16(blob + 4) != O_VERSION) return O_ERR_VERSION;
  if (get32(blob + 60) != vbqo_crc32(blob, 60)) return O_ERR_CRC;
  int64_t n = get32(blob + 8), k = get32(blob + 12), g = get32(blob + 16), r = get32(blob + 20),
          t = get32(blob + 24);
  if ((get16(blob + 6) & ~O_FLAG_SYM) != 0 || get32(blob + 28) != 0) return O_ERR_FORMAT;
  if (check_shape(n, k, r) != O_OK) return O_ERR_FORMAT;
  if (g != k / 64 || t != (n + r - 1) / r) return O_ERR_FORMAT;
  uint64_t dir_off = get64(blob + 32), rec_off = get64(blob + 40), tot = get64(blob + 48);
  if (dir_off != 64 || rec_off != 64 + a16(4 * (uint64_t)(t * g + 1))) return O_ERR_FORMAT;
  if (tot < rec_off) return O_ERR_FORMAT;
  if (tot > size) return O_ERR_BUFFER_TOO_SMALL;
  if (get32(blob + 56) != vbqo_crc32(blob + 64, tot - 64)) return O_ERR_CRC;
  if (N) *N = n;
  if (K) *K = k;
  if (R) *R = r;
  if (total) *total = tot;
  if (flags) *flags = get16(blob + 6);
  return O_OK;
}

int vbqo_read_header(const uint8_t* blob, uint64_t size, int64_t* N, int64_t* K, int64_t* R,
                     uint64_t* total) {
  return vbqo_read_header_ex(blob, size, N, K, R, total, NULL);
}

/* Unpack a canonical blob to logical arrays; any non-canonical content is
 * O_ERR_FORMAT. Output arrays may be NULL to validate only. */
int vbqo_unpack(const uint8_t* blob, uint64_t size, uint8_t* widths, uint16_t* scales, uint8_t* codes) {
  int64_t N, K, R;
  uint64_t total;
  unsigned flags;
  int st = vbqo_read_header_ex(blob, size, &N, &K, &R, &total, &flags);
  if (st) return st;
  int64_t G = K / 64, T = (N + R - 1) / R;
  uint64_t dir_off = 64, rec_off = 64 + a16(4 * (uint64_t)(T * G + 1));
  for (uint64_t p = dir_off + 4 * (uint64_t)(T * G + 1); p < rec_off; ++p)
    if (blob[p]) return O_ERR_FORMAT;
  if (rec_off + 16 * (uint64_t)get32(blob + dir_off + 4 * (uint64_t)(T * G)) != total) return O_ERR_FORMAT;
  uint64_t expect = 0;
  uint8_t* wtmp = (uint8_t*)malloc((size_t)R);
  if (!wtmp) return O_ERR_NULL;
  for (int64_t t = 0; t < T; ++t) {
    int64_t r0 = t * R, Rt = (N - r0 < R) ? N - r0 : R;
    for (int64_t g = 0; g < G; ++g) {
      uint64_t start = 16 * (uint64_t)get32(blob + dir_off + 4 * (uint64_t)(t * G + g));
      if (start != expect) { free(wtmp); return O_ERR_FORMAT; }
      const uint8_t* rec = blob + rec_off + start;
      if (rec_off + start + a16(8 + 4 * (uint64_t)((Rt + 15) / 16)) > total) { free(wtmp); return O_ERR_FORMAT; }
      int64_t cnt[4], seen[4] = {0, 0, 0, 0};
      for (int c = 0; c < 4; ++c) cnt[c] = get16(rec + 2 * c);
      for (int64_t j = 0; j < Rt; ++j) {
        int c = (int)((get32(rec + 8 + 4 * (j / 16)) >> (2 * (j % 16))) & 3u);
        wtmp[j] = (uint8_t)c;
        seen[c]++;
      }
      if (seen[0] != cnt[0] || seen[1] != cnt[1] || seen[2] != cnt[2] || seen[3] != cnt[3]) {
        free(wtmp); return O_ERR_FORMAT;
      }
      uint64_t sz = record_bytes(Rt, cnt);
      if (rec_off + start + sz > total) { free(wtmp); return O_ERR_FORMAT; }
      uint64_t scale_off = a16(8 + 4 * (uint64_t)((Rt + 15) / 16));
      uint64_t code_off = scale_off + a16(2 * (uint64_t)Rt);
      /* every byte of the record that is not payload must be zero */
      uint8_t* used = (uint8_t*)calloc((size_t)sz, 1);
      if (!used) { free(wtmp); return O_ERR_NULL; }
      for (int b = 0; b < 8; ++b) used[b] = 1;
      for (int64_t j = 0; j < Rt; ++j) {
        uint64_t bit = 2 * (uint64_t)j;
        used[8 + bit / 8] |= (uint8_t)(3u << (bit % 8));
      }
      int64_t item = 0;
      uint64_t cpos = code_off;
      for (int c = 0; c < 4; ++c) {
        int k = 1 << c;
        for (int64_t j = 0; j < Rt; ++j) {
          if (wtmp[j] != c) continue;
          int64_t r = r0 + j;
          if (widths) widths[r * G + g] = (uint8_t)k;
          if (scales) scales[r * G + g] = get16(rec + scale_off + 2 * (uint64_t)item);
          used[scale_off + 2 * (uint64_t)item] = used[scale_off + 2 * (uint64_t)item + 1] = 0xFF;
          for (int i = 0; i < 64; ++i) {
            uint32_t q = 0;
            for (int b = 0; b < k; ++b) {
              uint64_t bit = (uint64_t)k * i + b;
              q |= (uint32_t)((rec[cpos + bit / 8] >> (bit % 8)) & 1u) << b;
            }
            if (q > max_code(k, flags)) { free(used); free(wtmp); return O_ERR_FORMAT; }
            if (codes) codes[r * K + 64 * g + i] = (uint8_t)q;
          }
          for (int b = 0; b < 8 * k; ++b) used[cpos + b] = 0xFF;
          cpos += 8 * (uint64_t)k;
          ++item;
        }
        if (c == 0) cpos = code_off + a16(8 * (uint64_t)cnt[0]);
      }
      /* width-code bytes: only the used bits may be set; other bytes fully zero */
      for (uint64_t b = 0; b < sz; ++b) {
        uint8_t mask = (b >= 8 && b < scale_off) ? used[b] : (used[b] ? 0xFF : 0x00);
        if (rec[b] & (uint8_t)~mask) { free(used); free(wtmp); return O_ERR_FORMAT; }
      }
      free(used);
      expect += sz;
    }
  }
  free(wtmp);
  if (rec_off + expect != total) return O_ERR_FORMAT;
  return O_OK;
}

/* fp64 dequantize-then-matvec. x_bf16[B*K] row-major (batch b at row b),
 * y[B*N] and bound[B*N] row-major. y[b][r] = sum_i w[r][i] x[b][i] summed in
 * order i = 0..K-1; bound[b][r] = sum_i |w[r][i]| |x[b][i]|. */
int vbqo_matvec_ex(int64_t N, int64_t K, int64_t B, const uint8_t* widths, const uint16_t* scales,
                   const uint8_t* codes, const uint16_t* x_bf16, unsigned flags, double* y, double* bound,
                   int nthreads) {
  if (!widths || !scales || !codes || !x_bf16 || !y) return O_ERR_NULL;
  if (N < 1 || K < 64 || K % 64 != 0) return O_ERR_SHAPE;
  if (B < 1) return O_ERR_BATCH;
  if (flags & ~O_FLAG_SYM) return O_ERR_FLAGS;
  int st = check_logical(N, K, widths, codes, flags);
  if (st) return st;
  int64_t G = K / 64;
  double* xd = (double*)malloc(sizeof(double) * (size_t)(B * K));
  if (!xd) return O_ERR_NULL;
  for (int64_t i = 0; i < B * K; ++i) xd[i] = vbqo_bf16_to_double(x_bf16[i]);
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
#endif
  for (int64_t r = 0; r < N; ++r) {
    for (int64_t b = 0; b < B; ++b) {
      double acc = 0.0, a = 0.0;
      for (int64_t i = 0; i < K; ++i) {
        int64_t g = i / 64;
        int k = widths[r * G + g];
        double s = vbqo_half_to_double(scales[r * G + g]);
        double c = grid_offset(k, flags);
        double w = s * ((double)codes[r * K + i] - c);
        acc += w * xd[b * K + i];
        a += fabs(w) * fabs(xd[b * K + i]);
      }
      y[b * N + r] = acc;
      if (bound) bound[b * N + r] = a;
    }
  }
  free(xd);
  (void)nthreads;
  return O_OK;
}

int vbqo_matvec(int64_t N, int64_t K, int64_t B, const uint8_t* widths, const uint16_t* scales,
                const uint8_t* codes, const uint16_t* x_bf16, double* y, double* bound, int nthreads) {
  return vbqo_matvec_ex(N, K, B, widths, scales, codes, x_bf16, 0u, y, bound, nthreads);
}

/* Dequantized dense matrix, w[N*K] in fp64 (same map as vbqo_matvec). */
int vbqo_dequant_ex(int64_t N, int64_t K, const uint8_t* widths, const uint16_t* scales,
                    const uint8_t* codes, unsigned flags, double* w) {
  if (!widths || !scales || !codes || !w) return O_ERR_NULL;
  if (N < 1 || K < 64 || K % 64 != 0) return O_ERR_SHAPE;
  if (flags & ~O_FLAG_SYM) return O_ERR_FLAGS;
  int st = check_logical(N, K, widths, codes, flags);
  if (st) return st;
  int64_t G = K / 64;
  for (int64_t r = 0; r < N; ++r)
    for (int64_t i = 0; i < K; ++i) {
      int k = widths[r * G + i / 64];
      double s = vbqo_half_to_double(scales[r * G + i / 64]);
      w[r * K + i] = s * ((double)codes[r * K + i] - grid_offset(k, flags));
    }
  return O_OK;
}

int vbqo_dequant(int64_t N, int64_t K, const uint8_t* widths, const uint16_t* scales,
                 const uint8_t* codes, double* w) {
  return vbqo_dequant_ex(N, K, widths, scales, codes, 0u, w);
}
