/*
 * vbq.h: C ABI of the VBQ mixed-bit GEMV / skinny-GEMM library (libvbq.so).
 *
 * VBQ ("Variable Bit-width Quantization: Learning Per-Group Precision for 'Bigger-but-Smaller' Language
 * Models") cuts each weight row into contiguous groups of 64 weights. Each group has its own scale and its
 * own width from {1,2,4,8} bits (section 3.1). At decode time, fused kernels read the packed low-bit bytes of
 * a group, expand them with the group scale in registers, and accumulate the matrix-vector product. The
 * dense FP16 matrix is never built (section 6, paragraph "Fused kernels over packed weights").
 *
 * The dequantized weight is w = s * (q - (2^k - 1)/2), with q in [0, 2^k). Format flag VBQ_FLAG_GRID_SYMMETRIC
 * puts widths k >= 2 on the paper's Eq. 1 integer grid instead: w = s * (q - (2^(k-1) - 1)), q in [0, 2^k - 2].
 * The byte layout is packed format v1: row tiles, one record per (tile, group column), and per-width
 * buckets inside each record.
 *
 * Conventions for every function:
 *  - The return value is a status: VBQ_OK (0) or a negative VBQ_ERR_* code. No function aborts, exits or
 *    prints.
 *  - The caller owns and allocates every buffer. No function allocates or frees host or device memory.
 *  - Logical host arrays are row-major: widths[N*G] (values 1,2,4,8), scales[N*G] (IEEE fp16 bit patterns),
 *    codes[N*K] (one byte per weight, q < 2^width), with G = K/64.
 *  - Device functions are asynchronous on the given CUDA stream (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream). They never synchronize. A launch failure is reported as VBQ_ERR_CUDA, read with
 *    cudaPeekAtLastError (the sticky error state is not cleared).
 */
#ifndef VBQ_H_
#define VBQ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vbq_status {
  VBQ_OK = 0,
  VBQ_ERR_NULL = -1,              /* a required pointer is NULL */
  VBQ_ERR_SHAPE = -2,             /* N < 1, K < 64, K % 64 != 0, N or K above 2^31 - 1, or (pack) records above
                                     64 GiB, which the 32-bit directory entries cannot address */
  VBQ_ERR_WIDTH = -3,             /* a width is not 1, 2, 4 or 8 */
  VBQ_ERR_CODE_RANGE = -4,        /* a code is >= 2^width (above 2^width - 2 for widths >= 2 on the symmetric grid) */
  VBQ_ERR_BUFFER_TOO_SMALL = -5,  /* output capacity or blob size too small */
  VBQ_ERR_BAD_MAGIC = -6,         /* blob does not start with "VBQ1" */
  VBQ_ERR_VERSION = -7,           /* unsupported format version */
  VBQ_ERR_CRC = -8,               /* header or body CRC-32 mismatch */
  VBQ_ERR_BATCH = -9,             /* batch B not in {1, 2, 4, 8, 16} */
  VBQ_ERR_ALIGN = -10,            /* a device pointer breaks its alignment rule */
  VBQ_ERR_CUDA = -11,             /* a CUDA runtime call or launch failed */
  VBQ_ERR_TILE = -12,             /* tile rows R not a multiple of 16 in [16, 1024] */
  VBQ_ERR_FORMAT = -13,           /* blob is not canonical format v1 (layout, padding, counts) */
  VBQ_ERR_WORKSPACE = -14,        /* workspace NULL, misaligned or smaller than vbq_workspace_size */
  VBQ_ERR_SCRATCH_LIMIT = -15,    /* vbq_gemm_skinny_noalloc: problem needs more than its 16 MiB fixed buffer */
  VBQ_ERR_FLAGS = -16,            /* unknown bits in a flags word (launch options or format flags) */
  VBQ_ERR_VALUE = -17             /* vbq_quantize: non-finite weight, or a group scale beyond fp16 */
} vbq_status;

/* Host-side description of a packed blob. It is filled by vbq_pack or vbq_describe and passed by pointer to
 * the device entry points, so the library never reads device memory from the host. */
typedef struct vbq_desc {
  uint32_t version;      /* format version (1) */
  uint32_t flags;        /* format flags of the blob header: 0 or VBQ_FLAG_GRID_SYMMETRIC */
  int64_t N;             /* output rows */
  int64_t K;             /* input columns, multiple of 64 */
  int64_t G;             /* K / 64 */
  int64_t R;             /* rows per tile */
  int64_t T;             /* ceil(N / R) tiles */
  uint64_t dir_offset;   /* byte offset of the record directory */
  uint64_t rec_offset;   /* byte offset of the first record */
  uint64_t total_bytes;  /* blob size in bytes */
  uint64_t max_record_bytes; /* largest record; sets the shared-memory staging size of the kernels */
} vbq_desc;

/* Static English text for a status code; never NULL. */
const char* vbq_strerror(int status);

/* Library version as (major << 16 | minor); the packed format it reads and writes is version 1. */
uint32_t vbq_version(void);

/* ---------------------------------------------------------------------------------------------- host */

/* Bytes of the canonical packed-format-v1 blob for this logical matrix. No passage of the VBQ paper defines it:
 * the paper fixes the group size and the width set, not a byte layout. R (tile rows) is a parameter of the
 * layout, so the size depends on it.
 * widths: [N*G] in {1,2,4,8}. R: tile rows. Errors: NULL, SHAPE, TILE, WIDTH. Thread-safe, pure. */
int vbq_packed_size(int64_t N, int64_t K, int64_t R, const uint8_t* widths, uint64_t* out_bytes);

/* Pack a logical matrix into a canonical format-v1 blob written to out[0 .. *size). This is the export-time
 * step of the VBQ paper's section 6 ("An export-time check validates this contract"): it validates every
 * width and code first and writes nothing on error.
 * Errors: NULL, SHAPE, TILE, WIDTH, CODE_RANGE, BUFFER_TOO_SMALL (out_cap < vbq_packed_size).
 * out_desc may be NULL. Thread-safe, pure. */
int vbq_pack(int64_t N, int64_t K, int64_t R, const uint8_t* widths, const uint16_t* scales,
             const uint8_t* codes, void* out, uint64_t out_cap, vbq_desc* out_desc);

/* Format flags of a blob (header field `flags`, vbq_desc.flags). */
#define VBQ_FLAG_GRID_SYMMETRIC 1u  /* widths >= 2 on the VBQ paper's Eq. 1 integer grid (section 3.1):
                                       w = s*(q - (2^(k-1)-1)), q in [0, 2^k - 2]; 1-bit groups unchanged */

/* vbq_pack with format flags (0 or VBQ_FLAG_GRID_SYMMETRIC); the codes are checked against the flagged grid
 * (CODE_RANGE). Errors: as vbq_pack, plus FLAGS. */
int vbq_pack_ex(int64_t N, int64_t K, int64_t R, const uint8_t* widths, const uint16_t* scales,
                const uint8_t* codes, unsigned format_flags, void* out, uint64_t out_cap, vbq_desc* out_desc);

/* Zero-padded packing (VBQ paper, section 6, "Granularity is deployment-friendly": MLP intermediate widths are
 * zero-padded to a multiple of 512, which changes nothing because silu(0) * 0 = 0). The N x K logical matrix is
 * packed as an N_pad x K_pad one whose extra rows and columns are 1-bit groups with scale +0 and code 0, so every
 * added weight is exactly 0: padded gate/up rows give h = silu(0) * 0 = 0, and padded down-projection columns
 * multiply those zeros. Nothing in this library's kernels needs K % 512; the padded form is offered for blobs
 * shared with kernels that do, and its cost is measured against the unpadded one.
 * Requires N_pad >= N, K_pad >= K, K_pad % 64 == 0 (SHAPE otherwise). Other errors: as vbq_pack_ex. Pure. */
int vbq_packed_size_padded(int64_t N, int64_t K, int64_t R, const uint8_t* widths, int64_t N_pad, int64_t K_pad,
                           uint64_t* out_bytes);
int vbq_pack_padded(int64_t N, int64_t K, int64_t R, const uint8_t* widths, const uint16_t* scales,
                    const uint8_t* codes, int64_t N_pad, int64_t K_pad, unsigned format_flags, void* out,
                    uint64_t out_cap, vbq_desc* out_desc);

/* Quantize float32 weights w[N*K] (row-major) to the logical arrays for given widths[N*G] (VBQ paper,
 * section 3.1), group by group (64 weights):
 *  - width 1: scale s = 2 * mean|w| (the grid points +-s/2 are +-mean|w|: sign times the mean magnitude), the
 *    mean being the index-order sum of |w| in fp64 divided by 64; code 1 where w >= 0, else 0.
 *  - width k >= 2 with VBQ_FLAG_GRID_SYMMETRIC (Eq. 1): L = 2^(k-1) - 1, s = max|w| / L,
 *    code = clamp(round(w / s), -L, L) + L.
 *  - width k >= 2 without it (the default grid): c = (2^k - 1)/2, s = max|w| / c,
 *    code = clamp(round(w / s + c), 0, 2^k - 1).
 * The scale is computed in fp64, rounded to fp16 (nearest even), and that rounded value is the s the codes
 * use; round() is to nearest, ties away from zero. A group whose rounded scale is 0 gets the code of the grid
 * point nearest 0 (L, or 2^(k-1)). Pack the result with vbq_pack_ex and the same flags.
 * Errors: NULL, SHAPE, WIDTH, FLAGS, VALUE (a non-finite weight, or a scale that rounds past fp16). Pure. */
int vbq_quantize(int64_t N, int64_t K, const float* w, const uint8_t* widths, unsigned format_flags,
                 uint16_t* scales, uint8_t* codes);

/* Validate a host copy of a blob and fill *out_desc (no passage of the VBQ paper: the blob's header and CRCs are
 * this library's). Checks, in order: size >= 64 (BUFFER_TOO_SMALL), magic
 * (BAD_MAGIC), version (VERSION), header CRC (CRC), header fields (FORMAT), total_bytes <= blob_bytes
 * (BUFFER_TOO_SMALL), body CRC (CRC). It does not walk the records; vbq_unpack does. */
int vbq_describe(const void* blob_host, uint64_t blob_bytes, vbq_desc* out_desc);

/* Unpack a canonical blob (host memory) back into logical arrays sized from its header (N*G, N*G, N*K); the
 * inverse of vbq_pack (no passage of the VBQ paper; the paper's kernels consume the packed form directly).
 * Performs every vbq_describe check, then checks each record: counts agree with the width codes, and every
 * padding byte and unused bit is zero (FORMAT). Any output pointer may be NULL to validate only. */
int vbq_unpack(const void* blob_host, uint64_t blob_bytes, uint8_t* widths, uint16_t* scales,
               uint8_t* codes);

/* -------------------------------------------------------------------------------------------- device */

/* Workspace bytes that vbq_gemv / vbq_gemm_skinny need for this matrix and batch on the CURRENT device (the
 * launch shape depends on its SM count). No passage of the VBQ paper: the workspace exists because the kernels
 * split the K dimension of a row tile among CTAs and reduce the partial sums without floating-point atomics. The workspace holds the partial sums of row tiles that several CTAs
 * share, one arrival counter per row tile, and, in its 4 bytes at offset (size - 4), a device status word: 0 after every
 * successful call; nonzero if a kernel gave up a bounded wait (bit 0), met a record larger than the staging
 * size its descriptor promised or a directory entry past the end of the records (bit 1), or met a record whose
 * bucket counts disagree with its tile or its width codes (bit 2). The outputs of such a call are not valid, and
 * the workspace must be zeroed again (vbq_workspace_init) before its next use.
 * Errors: NULL, BATCH, FORMAT (desc inconsistent). */
int vbq_workspace_size(const vbq_desc* d, int B, uint64_t* out_bytes);

/* The launch plan of a device call (no passage of the VBQ paper: it describes this library's kernels), computed
 * on the host without any CUDA call, for sm_count SMs: nmat descriptors as in vbq_gemm_skinny_multi (1 for
 * vbq_gemm_skinny), batch B.
 *   grid, threads:       CTAs (one per SM) and threads per CTA;
 *   records_per_batch:   records of one row tile handled between two CTA barriers (1..7);
 *   batches_in_flight:   record batches streamed ahead of the compute (2 or 3);
 *   result_sets:         item-result buffers (2: alternate batches; 1: a barrier after each row pass);
 *   cost_split:          1 when CTAs split the records by estimated cost (record sizes differ much), 0 by count;
 *   smem_bytes:          dynamic shared memory per CTA;
 *   workspace_bytes:     what vbq_workspace_size[_multi] returns on a GPU with sm_count SMs.
 * Errors: NULL, BATCH, SHAPE (nmat or sm_count out of range), TILE, FORMAT (no plan fits). Pure, thread-safe. */
typedef struct vbq_plan_info {
  int32_t grid, threads, records_per_batch, batches_in_flight, result_sets, cost_split;
  uint32_t smem_bytes;
  uint64_t workspace_bytes;
} vbq_plan_info;
int vbq_plan_info_get(int nmat, const vbq_desc* const* d, int B, int sm_count, vbq_plan_info* out);

/* Zero a workspace before its first use (cudaMemsetAsync on `stream`). Every kernel call leaves the arrival
 * counters at zero again, so one zeroing per workspace is enough. Errors: NULL, CUDA. */
int vbq_workspace_init(void* workspace, uint64_t workspace_bytes, void* stream);

/* y[N] = W x for one activation vector (batch 1): vbq_gemm_skinny with B = 1. This is the VBQ paper's fused
 * kernel (section 6, paragraph "Fused kernels over packed weights": the packed low-bit bytes of each group are
 * expanded with the group scale in registers and the matrix-vector product accumulated; the FP16 matrix is never
 * built), over the per-group widths and scales of section 3.1.
 * blob_dev: byte-identical device copy of the packed blob, 16-byte aligned (ALIGN).
 * x_bf16:   K bf16 values (device), 16-byte aligned (ALIGN).
 * y:        N fp32 values (device), 4-byte aligned; fully overwritten.
 * workspace: vbq_workspace_size(d, 1) device bytes, 16-byte aligned, zeroed once by vbq_workspace_init; it
 *           must not be shared by calls that can run at the same time.
 * Result per element: |y - y_exact| <= 1e-3 * sum_i |w_i||x_i| + 1e-6, with fp32 accumulation. Results are
 * bitwise identical from run to run (no floating-point atomics). */
int vbq_gemv(const vbq_desc* d, const void* blob_dev, const void* x_bf16, float* y, void* workspace,
             uint64_t workspace_bytes, void* stream);

/* Y[B][N] = X[B][K] W^T for B in {1, 2, 4, 8, 16} activation rows (skinny GEMM; decode with a small batch). The
 * same fused dequantize-and-multiply as vbq_gemv (VBQ paper, section 6, "Fused kernels over packed weights"),
 * applied to several activation rows at once; the paper decodes at batch 1, the small batches are this library's
 * extension.
 * x_bf16: B*K bf16 values, row-major (row b is activation b), 16-byte aligned. y: B*N fp32, row-major.
 * B <= 2 runs on CUDA cores; B = 4, 8 and 16 run the dequantized groups through tensor cores (bf16 operands
 * that hold exact small integers or half-integers: q - c, q - 8 or q - 128, fp32 accumulation seeded with the
 * leftover grid offset times the group's activation sum, the group scale applied in fp32).
 * Other arguments and guarantees as in vbq_gemv. Errors: NULL, BATCH, ALIGN, WORKSPACE, FORMAT, CUDA. */
int vbq_gemm_skinny(const vbq_desc* d, const void* blob_dev, const void* x_bf16, int B, float* y,
                    void* workspace, uint64_t workspace_bytes, void* stream);

/* Launch options of vbq_gemm_skinny_ex (bit flags). */
#define VBQ_LAUNCH_OVERLAP 1u

/* vbq_gemm_skinny with launch options (the VBQ paper has no counterpart; this is a deployment aid).
 * VBQ_LAUNCH_OVERLAP: programmatic dependent launch. The kernel may begin while the kernel before it on `stream`
 * is still running. Until that kernel has finished and its writes are visible, it reads only `blob_dev` (the
 * directory and the records it streams into shared memory); it reads x and touches y and the workspace only
 * afterwards. So a chain of launches (for example the projections of a decode step) overlaps each kernel's
 * weight streaming with the tail of the one before. Do not set it when the kernel just before this call on
 * `stream` writes the blob. Without the flag this is exactly vbq_gemm_skinny.
 * Errors: as vbq_gemm_skinny, plus FLAGS (unknown bits). */
int vbq_gemm_skinny_ex(const vbq_desc* d, const void* blob_dev, const void* x_bf16, int B, float* y,
                       void* workspace, uint64_t workspace_bytes, unsigned flags, void* stream);

/* Several matrices that share their input, in one launch: fused projections such as q/k/v or gate/up, which the
 * VBQ paper's deployment runs back to back on the same activation (the paper has no fused entry point; this
 * one is a deployment aid). Up to 4 matrices, all with the same K (SHAPE otherwise) and the same tile rows R
 * (TILE otherwise). Their records run as one sequence, so the launch's fixed costs are paid once and the
 * small matrices share the SMs with the large ones.
 * d[m], blob_dev[m]: descriptor and device blob of matrix m (blob 16-byte aligned).
 * x_bf16: B*K bf16 values, row-major, 16-byte aligned, shared by all matrices.
 * y[m]:   B*N_m fp32 values, row-major, 4-byte aligned; fully overwritten.
 * workspace: vbq_workspace_size_multi(nmat, d, B) device bytes, 16-byte aligned, zeroed once by
 *           vbq_workspace_init; not shared by calls that can run at the same time.
 * flags: as vbq_gemm_skinny_ex.
 * Each y[m] meets the tolerance of vbq_gemv and is bitwise identical from run to run. It need not be bitwise
 * equal to a separate launch of matrix m, whose split among CTAs (and so whose summation order) differs.
 * Errors: NULL, BATCH, FLAGS, SHAPE (nmat outside 1..4, or K differs), TILE (R differs), FORMAT, ALIGN,
 * WORKSPACE, CUDA. */
int vbq_workspace_size_multi(int nmat, const vbq_desc* const* d, int B, uint64_t* out_bytes);
int vbq_gemm_skinny_multi(int nmat, const vbq_desc* const* d, const void* const* blob_dev, const void* x_bf16,
                          int B, float* const* y, void* workspace, uint64_t workspace_bytes, unsigned flags,
                          void* stream);

/* Gated MLP input projections with the SwiGLU epilogue fused in (VBQ paper, section 4: the models are
 * LLaMA-style decoders with SwiGLU MLPs; the paper has no fused entry point, this is a deployment aid).
 * One launch computes y_gate = X W_gate^T and y_up = X W_up^T as vbq_gemm_skinny_multi does, and
 * h = silu(y_gate) * y_up with silu(g) = g / (1 + e^-g), rounded to bf16 (round to nearest even): the input
 * of the down projection. gate and up must have the same N (SHAPE), K (SHAPE) and tile rows (TILE).
 * h_bf16: B*N bf16 values, row-major, 2-byte aligned; y_gate, y_up as in vbq_gemm_skinny (also written).
 * workspace: vbq_workspace_size_swiglu(gate, up, B) bytes, zeroed once by vbq_workspace_init.
 * h meets |h - h_exact| <= P + 2^-8 (|h_exact| + P) + 1e-6 with P = 1.1 tol_g (|u| + tol_u) + |silu(g)| tol_u,
 * where tol_g, tol_u are the vbq_gemv tolerances of y_gate, y_up (1.1 bounds |silu'|); every output is bitwise
 * identical from run to run.
 * Errors: as vbq_gemm_skinny_multi. */
int vbq_workspace_size_swiglu(const vbq_desc* gate, const vbq_desc* up, int B, uint64_t* out_bytes);
int vbq_gemm_swiglu(const vbq_desc* gate, const vbq_desc* up, const void* blob_gate, const void* blob_up,
                    const void* x_bf16, int B, float* y_gate, float* y_up, void* h_bf16, void* workspace,
                    uint64_t workspace_bytes, unsigned flags, void* stream);

/* Allocation-free variant of vbq_gemm_skinny (the VBQ paper has no counterpart; this is a deployment aid).
 *
 * Some callers cannot allocate device memory at all. Examples: plug-in hosts that give the library only pointers
 * into their own pre-reserved pools, and serving loops that forbid cudaMalloc after start-up because it can
 * synchronize the device and fragment their pools. Those callers can neither hold a workspace nor size one.
 * This entry point takes the same inputs and outputs as vbq_gemm_skinny, but no workspace. Its scratch
 * (split-K partial sums, arrival counters, status word) lives in one fixed 16 MiB device buffer inside the
 * library. Every GPU that loads the library holds that buffer until the process exits.
 *
 * - Limit: problems whose vbq_workspace_size(d, B) exceeds 16 MiB - 256 bytes are rejected with
 *   VBQ_ERR_SCRATCH_LIMIT, and nothing is launched. With 1024-row tiles that covers any N at B <= 4, and N up to
 *   about 110K at B = 16. The buffer's last 256 bytes hold the status word.
 * - First call per device: it looks up the buffer's device address (cudaGetSymbolAddress, with that device
 *   current) and keeps it; a device reset voids it. Make this first call before any stream capture.
 * - Each call clears the counters and the status word with cudaMemsetAsync on `stream`, then launches the
 *   same kernel as vbq_gemm_skinny. It allocates nothing and frees nothing.
 * - All calls on a device share the one buffer, which keeps the last call's contents. Calls that can overlap
 *   on the GPU (different streams, different host threads) race on it: serialize them.
 * - Errors found on the device (a bounded wait that ran out, a record the kernel refused; the bits of the
 *   vbq_workspace_size status word) are not returned by this call, which only enqueues the work: read them with
 *   vbq_noalloc_status, enqueued on the same stream after the call and before the next noalloc call.
 * Errors: as vbq_gemm_skinny, plus SCRATCH_LIMIT; CUDA if the buffer's address cannot be obtained. */
int vbq_gemm_skinny_noalloc(const vbq_desc* d, const void* blob_dev, const void* x_bf16, int B, float* y,
                            void* stream);

/* Status word of the last vbq_gemm_skinny_noalloc call on the current device, as described for the workspace
 * status word under vbq_workspace_size (0: no device-side error). It enqueues one cudaMemcpyAsync of 4 bytes on
 * `stream` into *status_host; *status_host is valid once the stream has reached it (synchronize the stream or
 * an event recorded after this call). The next noalloc call clears the word. Errors: NULL, CUDA. */
int vbq_noalloc_status(uint32_t* status_host, void* stream);

/* Test hook of the failure-detection path (the VBQ paper has no counterpart). Sets, for every later launch in
 * this process: wait_limit_ns, the limit of the kernels' bounded mbarrier waits (0 restores the default of
 * 2 s); withheld_record, a record of each launch (its index in the launch's record sequence: records of matrix 0
 * first, tile-major) whose bulk copy is never issued, or -1 for none. A launch that withholds a record waits for
 * it until the limit, then sets bit 0 of its status word, publishes nothing and returns; its workspace must be
 * zeroed again before the next use. Not thread-safe against concurrent launches; meant for tests only.
 * Returns VBQ_OK. */
int vbq_test_set_fault(uint64_t wait_limit_ns, int64_t withheld_record);

#ifdef __cplusplus
}
#endif

#endif /* VBQ_H_ */
