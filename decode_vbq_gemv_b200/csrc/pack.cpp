// Host side of libvbq: the packer, unpacker and blob validator of packed format v1.
//
// VBQ groups ("Variable Bit-width Quantization", section 3.1) are 64 contiguous weights along K of one output
// row, each with its own fp16 scale and a width from {1,2,4,8}. The packer is the export-time contract check
// of the paper's section 6 ("An export-time check validates this contract"): it rejects bad shapes, widths and
// codes before writing anything, and writes only canonical blobs (zero padding), so the same logical matrix
// always packs to the same bytes.
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <cmath>
#include <vector>

#include "vbq.h"

namespace {

constexpr uint32_t kMagic = 0x31514256u;  // "VBQ1"
constexpr uint32_t kVersion = 1;
// Directory entries count 16-byte units in 32 bits, so a blob's records span at most 2^32 - 1 units (64 GiB).
constexpr uint64_t kMaxRecordUnits = 0xFFFFFFFFull;
constexpr uint64_t kHeaderBytes = 64;

inline uint64_t align16(uint64_t v) { return (v + 15) / 16 * 16; }

// ---------------------------------------------------------------------------------------------- CRC-32
// IEEE 802.3 / zlib CRC-32 (reflected polynomial 0xEDB88320), one table lookup per byte.
struct CrcTable {
  uint32_t t[256];
  CrcTable() {
    for (uint32_t n = 0; n < 256; ++n) {
      uint32_t c = n;
      for (int k = 0; k < 8; ++k) c = (c >> 1) ^ (0xEDB88320u & (0u - (c & 1u)));
      t[n] = c;
    }
  }
};
const CrcTable& crc_table() {
  static const CrcTable table;
  return table;
}
uint32_t crc32(const uint8_t* p, uint64_t n) {
  const uint32_t* t = crc_table().t;
  uint32_t c = ~0u;
  for (uint64_t i = 0; i < n; ++i) c = t[(c ^ p[i]) & 0xFFu] ^ (c >> 8);
  return ~c;
}

// ------------------------------------------------------------------------------------ little-endian I/O
inline void st16(uint8_t* p, uint32_t v) { p[0] = uint8_t(v); p[1] = uint8_t(v >> 8); }
inline void st32(uint8_t* p, uint32_t v) { st16(p, v & 0xFFFFu); st16(p + 2, v >> 16); }
inline void st64(uint8_t* p, uint64_t v) { st32(p, uint32_t(v)); st32(p + 4, uint32_t(v >> 32)); }
inline uint32_t ld16(const uint8_t* p) { return uint32_t(p[0]) | (uint32_t(p[1]) << 8); }
inline uint32_t ld32(const uint8_t* p) { return ld16(p) | (ld16(p + 2) << 16); }
inline uint64_t ld64(const uint8_t* p) { return uint64_t(ld32(p)) | (uint64_t(ld32(p + 4)) << 32); }

// log2 of a valid width, or -1.
inline int wcode(uint8_t k) {
  switch (k) {
    case 1: return 0;
    case 2: return 1;
    case 4: return 2;
    case 8: return 3;
    default: return -1;
  }
}

int shape_status(int64_t N, int64_t K, int64_t R) {
  if (N < 1 || K < 64 || (K & 63) || N > INT32_MAX || K > INT32_MAX) return VBQ_ERR_SHAPE;
  if (R < 16 || R > 1024 || (R & 15)) return VBQ_ERR_TILE;
  return VBQ_OK;
}

// Geometry shared by the packer, the validator and the device launcher.
struct Geometry {
  int64_t N, K, G, R, T;
  uint64_t dir_off, rec_off;
  Geometry(int64_t n, int64_t k, int64_t r) : N(n), K(k), G(k / 64), R(r), T((n + r - 1) / r) {
    dir_off = kHeaderBytes;
    rec_off = kHeaderBytes + align16(4 * uint64_t(T * G + 1));
  }
  int64_t tile_rows(int64_t t) const { return (t + 1) * R <= N ? R : N - t * R; }
};

// Offsets inside one record with Rt rows and bucket counts n[4].
struct RecordLayout {
  uint64_t scales, codes, bucket[4], bytes;
  RecordLayout(int64_t Rt, const uint32_t n[4]) {
    scales = align16(8 + 4 * uint64_t((Rt + 15) / 16));
    codes = scales + align16(2 * uint64_t(Rt));
    bucket[0] = codes;
    bucket[1] = bucket[0] + align16(8 * uint64_t(n[0]));
    bucket[2] = bucket[1] + 16 * uint64_t(n[1]);
    bucket[3] = bucket[2] + 32 * uint64_t(n[2]);
    bytes = bucket[3] + 64 * uint64_t(n[3]);
  }
};

// Per-record bucket counts, record-major (t, g).
int record_counts(const Geometry& geo, const uint8_t* widths, std::vector<uint32_t>& counts) {
  counts.assign(size_t(geo.T * geo.G) * 4, 0u);
  for (int64_t r = 0; r < geo.N; ++r) {
    uint32_t* tile = &counts[size_t(r / geo.R) * geo.G * 4];
    const uint8_t* wr = widths + r * geo.G;
    for (int64_t g = 0; g < geo.G; ++g) {
      int c = wcode(wr[g]);
      if (c < 0) return VBQ_ERR_WIDTH;
      tile[g * 4 + c]++;
    }
  }
  return VBQ_OK;
}

void fill_desc(const Geometry& geo, uint64_t total, uint64_t max_rec, unsigned flags, vbq_desc* d) {
  d->version = kVersion;
  d->flags = flags;
  d->N = geo.N;
  d->K = geo.K;
  d->G = geo.G;
  d->R = geo.R;
  d->T = geo.T;
  d->dir_offset = geo.dir_off;
  d->rec_offset = geo.rec_off;
  d->total_bytes = total;
  d->max_record_bytes = max_rec;
}

// Writes one group's 64 k-bit codes as a little-endian bit string of 8k bytes (code i at bits [k*i, k*i+k)).
void put_group_codes(uint8_t* dst, const uint8_t* q, int k) {
  uint64_t words[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int i = 0; i < 64; ++i) {
    const unsigned bit = unsigned(k * i);
    words[bit >> 6] |= uint64_t(q[i]) << (bit & 63);
  }
  for (int w = 0; w < k; ++w) st64(dst + 8 * w, words[w]);
}

void get_group_codes(const uint8_t* src, uint8_t* q, int k) {
  const uint32_t mask = (1u << k) - 1u;
  for (int i = 0; i < 64; ++i) {
    const unsigned bit = unsigned(k * i);
    q[i] = uint8_t((ld64(src + 8 * (bit >> 6)) >> (bit & 63)) & mask);
  }
}

// Largest code of a k-bit group: 2^k - 1, or 2^k - 2 on the symmetric grid (header flag bit 0, k >= 2).
inline unsigned max_code(int k, unsigned flags) {
  return ((flags & VBQ_FLAG_GRID_SYMMETRIC) && k >= 2) ? (1u << k) - 2u : (1u << k) - 1u;
}

// IEEE binary16 bit pattern of a finite v >= 0, rounded to nearest, ties to even (values from 65520 up become
// infinity). The significand is scaled by a power of two (exact) and rounded with nearbyint, whose default
// rounding mode is to nearest even.
uint16_t half_bits_rne(double v) {
  if (v == 0.0) return 0;
  int e;
  std::frexp(v, &e);  // v = m * 2^e, m in [0.5, 1)
  if (e <= -14) {     // below 2^-14: subnormal step 2^-24 (a result of 1024 is the smallest normal)
    return uint16_t(std::nearbyint(std::ldexp(v, 24)));
  }
  double r = std::nearbyint(std::ldexp(v, 11 - e));  // 11 significant bits: r in [1024, 2048]
  int E = e - 1 + 15;
  if (r >= 2048.0) {
    r = 1024.0;
    ++E;
  }
  if (E >= 31) return 0x7C00u;
  return uint16_t((unsigned(E) << 10) | (unsigned(r) - 1024u));
}

double half_value(uint16_t h) {
  const int E = (h >> 10) & 31, M = h & 1023;
  const double mag = E == 0 ? std::ldexp(double(M), -24) : std::ldexp(double(M + 1024), E - 25);
  return (h & 0x8000u) ? -mag : mag;
}

}  // namespace

extern "C" {

const char* vbq_strerror(int status) {
  switch (status) {
    case VBQ_OK: return "ok";
    case VBQ_ERR_NULL: return "a required pointer is NULL";
    case VBQ_ERR_SHAPE: return "bad shape: need N >= 1 and K a positive multiple of 64";
    case VBQ_ERR_WIDTH: return "a group width is not 1, 2, 4 or 8";
    case VBQ_ERR_CODE_RANGE: return "a code does not fit its group width";
    case VBQ_ERR_BUFFER_TOO_SMALL: return "buffer too small";
    case VBQ_ERR_BAD_MAGIC: return "not a VBQ blob (bad magic)";
    case VBQ_ERR_VERSION: return "unsupported VBQ format version";
    case VBQ_ERR_CRC: return "CRC-32 mismatch";
    case VBQ_ERR_BATCH: return "batch must be 1, 2, 4, 8 or 16";
    case VBQ_ERR_ALIGN: return "misaligned device pointer";
    case VBQ_ERR_CUDA: return "CUDA error";
    case VBQ_ERR_TILE: return "tile rows must be a multiple of 16 in [16, 1024]";
    case VBQ_ERR_FORMAT: return "blob is not canonical VBQ format v1";
    case VBQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case VBQ_ERR_SCRATCH_LIMIT: return "problem needs more scratch than the 16 MiB fixed buffer of the allocation-free entry point";
    case VBQ_ERR_FLAGS: return "flags word has bits this entry point does not define";
    case VBQ_ERR_VALUE: return "a weight is not finite, or a group scale does not fit in fp16";
    default: return "unknown status";
  }
}

uint32_t vbq_version(void) { return (1u << 16) | 0u; }

int vbq_packed_size(int64_t N, int64_t K, int64_t R, const uint8_t* widths, uint64_t* out_bytes) {
  if (!widths || !out_bytes) return VBQ_ERR_NULL;
  if (int st = shape_status(N, K, R)) return st;
  Geometry geo(N, K, R);
  std::vector<uint32_t> counts;
  if (int st = record_counts(geo, widths, counts)) return st;
  uint64_t recs = 0;
  for (int64_t t = 0; t < geo.T; ++t)
    for (int64_t g = 0; g < geo.G; ++g) recs += RecordLayout(geo.tile_rows(t), &counts[size_t(t * geo.G + g) * 4]).bytes;
  if (recs / 16 > kMaxRecordUnits) return VBQ_ERR_SHAPE;
  *out_bytes = geo.rec_off + recs;
  return VBQ_OK;
}

int vbq_pack_ex(int64_t N, int64_t K, int64_t R, const uint8_t* widths, const uint16_t* scales,
                const uint8_t* codes, unsigned format_flags, void* out, uint64_t out_cap, vbq_desc* out_desc) {
  if (!widths || !scales || !codes || !out) return VBQ_ERR_NULL;
  if (format_flags & ~unsigned(VBQ_FLAG_GRID_SYMMETRIC)) return VBQ_ERR_FLAGS;
  if (int st = shape_status(N, K, R)) return st;
  Geometry geo(N, K, R);
  std::vector<uint32_t> counts;
  if (int st = record_counts(geo, widths, counts)) return st;
  // Code range check, row by row.
  for (int64_t r = 0; r < N; ++r)
    for (int64_t g = 0; g < geo.G; ++g) {
      const unsigned lim = max_code(widths[r * geo.G + g], format_flags);
      const uint8_t* q = codes + r * K + 64 * g;
      for (int i = 0; i < 64; ++i)
        if (q[i] > lim) return VBQ_ERR_CODE_RANGE;
    }
  std::vector<uint64_t> rec_start(size_t(geo.T * geo.G) + 1);
  uint64_t pos = 0;
  for (int64_t t = 0; t < geo.T; ++t)
    for (int64_t g = 0; g < geo.G; ++g) {
      rec_start[size_t(t * geo.G + g)] = pos;
      pos += RecordLayout(geo.tile_rows(t), &counts[size_t(t * geo.G + g) * 4]).bytes;
    }
  rec_start.back() = pos;
  if (pos / 16 > kMaxRecordUnits) return VBQ_ERR_SHAPE;  // directory entries would not fit in 32 bits
  uint64_t max_rec = 0;
  for (size_t i = 0; i + 1 < rec_start.size(); ++i) max_rec = std::max(max_rec, rec_start[i + 1] - rec_start[i]);
  const uint64_t total = geo.rec_off + pos;
  if (out_cap < total) return VBQ_ERR_BUFFER_TOO_SMALL;

  uint8_t* b = static_cast<uint8_t*>(out);
  std::memset(b, 0, size_t(total));
  for (size_t i = 0; i < rec_start.size(); ++i) st32(b + geo.dir_off + 4 * i, uint32_t(rec_start[i] / 16));

  std::vector<uint32_t> slot(size_t(geo.R));  // item index of each row in its record
  for (int64_t t = 0; t < geo.T; ++t) {
    const int64_t Rt = geo.tile_rows(t), r0 = t * geo.R;
    for (int64_t g = 0; g < geo.G; ++g) {
      const uint32_t* n = &counts[size_t(t * geo.G + g) * 4];
      const RecordLayout L(Rt, n);
      uint8_t* rec = b + geo.rec_off + rec_start[size_t(t * geo.G + g)];
      for (int c = 0; c < 4; ++c) st16(rec + 2 * c, n[c]);
      // Counting sort: item = bucket base + rank among earlier rows of the same width.
      uint32_t next[4] = {0, n[0], n[0] + n[1], n[0] + n[1] + n[2]};
      for (int64_t j = 0; j < Rt; ++j) {
        const int c = wcode(widths[(r0 + j) * geo.G + g]);
        rec[8 + j / 4] |= uint8_t(c << (2 * (j % 4)));
        slot[size_t(j)] = next[c]++;
      }
      const uint64_t item_base[4] = {0, n[0], n[0] + n[1], n[0] + n[1] + n[2]};
      for (int64_t j = 0; j < Rt; ++j) {
        const int64_t r = r0 + j;
        const int c = wcode(widths[r * geo.G + g]);
        const uint32_t item = slot[size_t(j)];
        st16(rec + L.scales + 2 * uint64_t(item), scales[r * geo.G + g]);
        put_group_codes(rec + L.bucket[c] + (uint64_t(item) - item_base[c]) * (8u << c), codes + r * K + 64 * g, 1 << c);
      }
    }
  }
  st32(b + 0, kMagic);
  st16(b + 4, kVersion);
  st16(b + 6, format_flags);
  st32(b + 8, uint32_t(N));
  st32(b + 12, uint32_t(K));
  st32(b + 16, uint32_t(geo.G));
  st32(b + 20, uint32_t(R));
  st32(b + 24, uint32_t(geo.T));
  st32(b + 28, 0);
  st64(b + 32, geo.dir_off);
  st64(b + 40, geo.rec_off);
  st64(b + 48, total);
  st32(b + 56, crc32(b + kHeaderBytes, total - kHeaderBytes));
  st32(b + 60, crc32(b, 60));
  if (out_desc) fill_desc(geo, total, max_rec, format_flags, out_desc);
  return VBQ_OK;
}

int vbq_pack(int64_t N, int64_t K, int64_t R, const uint8_t* widths, const uint16_t* scales,
             const uint8_t* codes, void* out, uint64_t out_cap, vbq_desc* out_desc) {
  return vbq_pack_ex(N, K, R, widths, scales, codes, 0u, out, out_cap, out_desc);
}

namespace {
// The logical arrays of an N x K matrix embedded in an N_pad x K_pad one: rows N.. and columns K.. are 1-bit
// groups with scale +0 (every weight exactly 0) and code 0.
struct Padded {
  std::vector<uint8_t> widths, codes;
  std::vector<uint16_t> scales;
};
int pad_status(int64_t N, int64_t K, int64_t N_pad, int64_t K_pad) {
  if (N_pad < N || K_pad < K || K_pad % 64 != 0 || N_pad < 1) return VBQ_ERR_SHAPE;
  if (N_pad > (int64_t(1) << 31) || K_pad > (int64_t(1) << 31)) return VBQ_ERR_SHAPE;
  return VBQ_OK;
}
void pad_logical(int64_t N, int64_t K, const uint8_t* widths, const uint16_t* scales, const uint8_t* codes,
                 int64_t N_pad, int64_t K_pad, Padded& out) {
  const int64_t G = K / 64, Gp = K_pad / 64;
  out.widths.assign(size_t(N_pad * Gp), uint8_t(1));
  if (scales) out.scales.assign(size_t(N_pad * Gp), uint16_t(0));
  if (codes) out.codes.assign(size_t(N_pad * K_pad), uint8_t(0));
  for (int64_t r = 0; r < N; ++r) {
    std::memcpy(&out.widths[size_t(r * Gp)], widths + r * G, size_t(G));
    if (scales) std::memcpy(&out.scales[size_t(r * Gp)], scales + r * G, size_t(G) * 2);
    if (codes) std::memcpy(&out.codes[size_t(r * K_pad)], codes + r * K, size_t(K));
  }
}
}  // namespace

int vbq_packed_size_padded(int64_t N, int64_t K, int64_t R, const uint8_t* widths, int64_t N_pad, int64_t K_pad,
                           uint64_t* out_bytes) {
  if (!widths || !out_bytes) return VBQ_ERR_NULL;
  if (int st = shape_status(N, K, R)) return st;
  if (int st = pad_status(N, K, N_pad, K_pad)) return st;
  Padded pd;
  pad_logical(N, K, widths, nullptr, nullptr, N_pad, K_pad, pd);
  return vbq_packed_size(N_pad, K_pad, R, pd.widths.data(), out_bytes);
}

int vbq_pack_padded(int64_t N, int64_t K, int64_t R, const uint8_t* widths, const uint16_t* scales,
                    const uint8_t* codes, int64_t N_pad, int64_t K_pad, unsigned format_flags, void* out,
                    uint64_t out_cap, vbq_desc* out_desc) {
  if (!widths || !scales || !codes || !out) return VBQ_ERR_NULL;
  if (int st = shape_status(N, K, R)) return st;
  if (int st = pad_status(N, K, N_pad, K_pad)) return st;
  Padded pd;
  pad_logical(N, K, widths, scales, codes, N_pad, K_pad, pd);
  return vbq_pack_ex(N_pad, K_pad, R, pd.widths.data(), pd.scales.data(), pd.codes.data(), format_flags, out,
                     out_cap, out_desc);
}

int vbq_describe(const void* blob_host, uint64_t blob_bytes, vbq_desc* out_desc) {
  if (!blob_host || !out_desc) return VBQ_ERR_NULL;
  const uint8_t* b = static_cast<const uint8_t*>(blob_host);
  if (blob_bytes < kHeaderBytes) return VBQ_ERR_BUFFER_TOO_SMALL;
  if (ld32(b) != kMagic) return VBQ_ERR_BAD_MAGIC;
  if (ld16(b + 4) != kVersion) return VBQ_ERR_VERSION;
  if (ld32(b + 60) != crc32(b, 60)) return VBQ_ERR_CRC;
  const int64_t N = ld32(b + 8), K = ld32(b + 12), G = ld32(b + 16), R = ld32(b + 20), T = ld32(b + 24);
  const unsigned flags = ld16(b + 6);
  if ((flags & ~unsigned(VBQ_FLAG_GRID_SYMMETRIC)) || ld32(b + 28) != 0 || shape_status(N, K, R) != VBQ_OK)
    return VBQ_ERR_FORMAT;
  const Geometry geo(N, K, R);
  if (G != geo.G || T != geo.T) return VBQ_ERR_FORMAT;
  const uint64_t total = ld64(b + 48);
  if (ld64(b + 32) != geo.dir_off || ld64(b + 40) != geo.rec_off || total < geo.rec_off) return VBQ_ERR_FORMAT;
  if (total > blob_bytes) return VBQ_ERR_BUFFER_TOO_SMALL;
  if (ld32(b + 56) != crc32(b + kHeaderBytes, total - kHeaderBytes)) return VBQ_ERR_CRC;
  // Directory: strictly increasing record starts that end exactly at total_bytes.
  const uint64_t nrec = uint64_t(geo.T * geo.G);
  if (geo.dir_off + 4 * (nrec + 1) > geo.rec_off) return VBQ_ERR_FORMAT;
  uint64_t max_rec = 0, prev = ld32(b + geo.dir_off);
  if (prev != 0) return VBQ_ERR_FORMAT;
  for (uint64_t i = 1; i <= nrec; ++i) {
    const uint64_t cur = ld32(b + geo.dir_off + 4 * i);
    if (cur <= prev) return VBQ_ERR_FORMAT;
    max_rec = std::max(max_rec, 16 * (cur - prev));
    prev = cur;
  }
  if (geo.rec_off + 16 * prev != total) return VBQ_ERR_FORMAT;
  fill_desc(geo, total, max_rec, flags, out_desc);
  return VBQ_OK;
}

int vbq_unpack(const void* blob_host, uint64_t blob_bytes, uint8_t* widths, uint16_t* scales, uint8_t* codes) {
  vbq_desc d;
  if (int st = vbq_describe(blob_host, blob_bytes, &d)) return st;
  const uint8_t* b = static_cast<const uint8_t*>(blob_host);
  const Geometry geo(d.N, d.K, d.R);
  const uint64_t nrec = uint64_t(geo.T * geo.G);
  // Directory: consecutive records, padding zero, last entry = end of the blob.
  for (uint64_t p = geo.dir_off + 4 * (nrec + 1); p < geo.rec_off; ++p)
    if (b[p]) return VBQ_ERR_FORMAT;
  if (geo.rec_off + 16 * uint64_t(ld32(b + geo.dir_off + 4 * nrec)) != d.total_bytes) return VBQ_ERR_FORMAT;

  std::vector<uint8_t> mask;  // allowed bits per record byte
  std::vector<uint32_t> row_of(size_t(geo.R));
  uint8_t q[64];
  uint64_t expect = 0;
  for (int64_t t = 0; t < geo.T; ++t) {
    const int64_t Rt = geo.tile_rows(t), r0 = t * geo.R;
    for (int64_t g = 0; g < geo.G; ++g) {
      const uint64_t start = 16 * uint64_t(ld32(b + geo.dir_off + 4 * uint64_t(t * geo.G + g)));
      if (start != expect) return VBQ_ERR_FORMAT;
      const uint8_t* rec = b + geo.rec_off + start;
      const uint64_t avail = d.total_bytes - (geo.rec_off + start);
      if (avail < 8 + uint64_t(Rt + 3) / 4) return VBQ_ERR_FORMAT;
      uint32_t n[4], seen[4] = {0, 0, 0, 0};
      for (int c = 0; c < 4; ++c) n[c] = ld16(rec + 2 * c);
      for (int64_t j = 0; j < Rt; ++j) seen[(rec[8 + j / 4] >> (2 * (j % 4))) & 3u]++;
      if (seen[0] != n[0] || seen[1] != n[1] || seen[2] != n[2] || seen[3] != n[3]) return VBQ_ERR_FORMAT;
      const RecordLayout L(Rt, n);
      if (L.bytes > avail) return VBQ_ERR_FORMAT;
      mask.assign(size_t(L.bytes), 0);
      for (int i = 0; i < 8; ++i) mask[size_t(i)] = 0xFF;
      for (int64_t j = 0; j < Rt; ++j) mask[size_t(8 + j / 4)] |= uint8_t(3u << (2 * (j % 4)));
      uint32_t next[4] = {0, n[0], n[0] + n[1], n[0] + n[1] + n[2]};
      const uint32_t item_base[4] = {0, n[0], n[0] + n[1], n[0] + n[1] + n[2]};
      for (int64_t j = 0; j < Rt; ++j) row_of[size_t(next[(rec[8 + j / 4] >> (2 * (j % 4))) & 3u]++)] = uint32_t(j);
      for (int c = 0; c < 4; ++c) {
        for (uint32_t it = item_base[c]; it < item_base[c] + n[c]; ++it) {
          const int64_t r = r0 + row_of[it];
          const uint64_t so = L.scales + 2 * uint64_t(it);
          const uint64_t co = L.bucket[c] + uint64_t(it - item_base[c]) * (8u << c);
          mask[size_t(so)] = mask[size_t(so + 1)] = 0xFF;
          std::memset(&mask[size_t(co)], 0xFF, size_t(8u << c));
          if (widths) widths[r * geo.G + g] = uint8_t(1u << c);
          if (scales) scales[r * geo.G + g] = uint16_t(ld16(rec + so));
          get_group_codes(rec + co, q, 1 << c);
          const unsigned lim = max_code(1 << c, d.flags);
          for (int i = 0; i < 64; ++i)
            if (q[i] > lim) return VBQ_ERR_FORMAT;
          if (codes) std::memcpy(codes + r * geo.K + 64 * g, q, 64);
        }
      }
      for (uint64_t i = 0; i < L.bytes; ++i)
        if (rec[i] & uint8_t(~mask[size_t(i)])) return VBQ_ERR_FORMAT;
      expect += L.bytes;
    }
  }
  if (geo.rec_off + expect != d.total_bytes) return VBQ_ERR_FORMAT;
  return VBQ_OK;
}

int vbq_quantize(int64_t N, int64_t K, const float* w, const uint8_t* widths, unsigned format_flags,
                 uint16_t* scales, uint8_t* codes) {
  if (!w || !widths || !scales || !codes) return VBQ_ERR_NULL;
  if (N < 1 || K < 64 || K % 64 != 0 || N > INT32_MAX || K > INT32_MAX) return VBQ_ERR_SHAPE;
  if (format_flags & ~unsigned(VBQ_FLAG_GRID_SYMMETRIC)) return VBQ_ERR_FLAGS;
  const bool sym = format_flags & VBQ_FLAG_GRID_SYMMETRIC;
  const int64_t G = K / 64;
  for (int64_t i = 0; i < N * G; ++i)
    if (wcode(widths[i]) < 0) return VBQ_ERR_WIDTH;
  for (int64_t i = 0; i < N * K; ++i)
    if (!std::isfinite(w[i])) return VBQ_ERR_VALUE;
  for (int64_t r = 0; r < N; ++r)
    for (int64_t g = 0; g < G; ++g) {
      const int k = widths[r * G + g];
      const float* wg = w + r * K + 64 * g;
      uint8_t* q = codes + r * K + 64 * g;
      double sum = 0.0, amax = 0.0;
      for (int i = 0; i < 64; ++i) {
        const double a = std::fabs(double(wg[i]));
        sum += a;
        amax = std::max(amax, a);
      }
      const double L = double((1 << (k - 1)) - 1), c = double((1 << k) - 1) / 2.0;
      const double ratio = k == 1 ? sum / 32.0 : (sym ? amax / L : amax / c);
      const uint16_t s16 = half_bits_rne(ratio);
      if (s16 == 0x7C00u) return VBQ_ERR_VALUE;
      scales[r * G + g] = s16;
      const double sd = half_value(s16);
      for (int i = 0; i < 64; ++i) {
        double v;
        if (k == 1) {
          v = wg[i] >= 0.f ? 1.0 : 0.0;
        } else if (sd == 0.0) {
          v = sym ? L : double(1 << (k - 1));
        } else if (sym) {
          v = std::min(std::max(std::round(double(wg[i]) / sd), -L), L) + L;
        } else {
          v = std::min(std::max(std::round(double(wg[i]) / sd + c), 0.0), double((1 << k) - 1));
        }
        q[i] = uint8_t(v);
      }
    }
  return VBQ_OK;
}

}  // extern "C"
