/*
 * lbq.h -- C ABI of the low-bit weight-only GEMV/GEMM library for B200 (sm_100a).
 *
 * The library computes y = s * T(W)^T * (H x): bf16 activations times LLM weights
 * stored in one of three packed low-bit formats, dequantized on the fly inside
 * the kernels, accumulated in fp32 and written as bf16.
 *
 * Sources (web pages on extreme low-bit 27B inference):
 *   [tern]  pptc.cn, "8 GB card runs a ternary 27B" article: §1.2 (three states,
 *           log2 3 bits per weight; products become add / subtract / skip), §5.1
 *           (absmean ternarisation: s = mean|w|, t = clip(round(w/s), -1, 1)).
 *   [block] mhpq.cn, "27B in 5.9 GB" article: §2.1 (one shared scale per block of
 *           64 or 128 weights, weight = trit * scale), §2.2 (ternary matmul reduces
 *           to add / subtract / skip), §3.2 (fp16 scale per block).
 *   [sign]  neodrop.ai community round-up, part 2: a Q1_0 model whose weights are
 *           only +1 or -1, sped up by a dedicated matrix kernel.
 *   [rht]   feinterview.poetries.top, "27B in 12 GB laptop GPU" article, section
 *           "12 GB 装下 27B": random Hadamard rotation before low-bit coding
 *           (QuIP / QuIP# / QTIP lineage).
 *
 * Conventions shared by every call
 *   - A weight matrix is stored one output row per packed row: logical W is K x N
 *     (K = input features), stored [N][K] with K contiguous; y[n] = sum_k w[n][k] x[k].
 *   - Pointers are DEVICE pointers unless a comment says otherwise. The caller
 *     allocates and owns every buffer; the library never allocates, frees or
 *     synchronises. Calls enqueue on `stream` (a cudaStream_t passed as void*,
 *     NULL = legacy default stream) and return; results are valid once the
 *     stream reaches that point.
 *   - bf16 and fp16 values travel as their raw 16-bit patterns (uint16_t).
 *   - Every call validates its arguments on the host BEFORE any launch and
 *     returns a status; on any status other than LBQ_OK nothing was enqueued,
 *     except LBQ_ERR_CUDA from a failed launch (the launch error is cleared).
 *     No call aborts, exits or throws across the ABI.
 *   - Inputs must be finite; NaN/Inf inputs give unspecified (non-faulting) output.
 *
 * Packed formats (byte layouts are this library's; the pages fix only the number
 * system, the block size and the scale rule):
 *
 *   LBQ_TERN5 (ternary, [tern] + [block]): blocks of 128 weights, each 28 bytes:
 *     bytes 0..24  : five trits per byte, little-endian base 3 of d = t + 1:
 *                    byte j = sum_{i<5} d[5j+i] * 3^i    (weights 5j .. 5j+4)
 *     byte  25     : weights 125..127 in digits 0..2; digits 3 and 4 are zero
 *                    trits (d = 1), so the byte is d125 + 3 d126 + 9 d127 + 108
 *     bytes 26..27 : fp16 scale s16 of the block (little-endian bits)
 *     Every byte value is <= 242. Rows are padded to a 16-byte multiple
 *     (code_stride = round_up(28 * K/128, 16)); pad bytes are zero and never read
 *     for arithmetic. The scale lives inside the block so that every aligned
 *     32-bit word of a row belongs to exactly one block. `scales` is unused (NULL).
 *     Quantisation: s16 = fp16_rne(min(mean_k |w_k|, 65504)), mean taken in fp64;
 *     t = sign(w) if |w| > s16/2 else 0 (equal to clip(round_half_even(w/s16), -1, 1));
 *     t = 0 everywhere when s16 == 0. Dequantised weight = s16 * t.
 *
 *   LBQ_SIGN1 (1-bit, [sign]): codes [N][code_stride], code_stride = K/8 bytes;
 *     bit i of byte j is weight 8j+i, 1 -> +1, 0 -> -1, bit = (w >= 0).
 *     scales [N][scale_stride] fp16 with scale_stride = round_up(K/128, 8) (rows of
 *     scales padded with zeros to 16 bytes), s16 = fp16_rne(min(mean |w|, 65504))
 *     per 128 weights.
 *     Dequantised weight = s16 * (2 bit - 1).
 *
 *   LBQ_Q2RHT (2-bit, 4 levels, rotated input, [rht]): codes [N][K/4] bytes;
 *     weight 4j+i in bits 2i..2i+1 of byte j; code q in 0..3 means level q - 1.5.
 *     scales [N][K/32] fp16, s16 = fp16_rne(min(max|w| / 1.5, 65504)) per 32 weights
 *     (quotient in fp64); q = clip(floor(w/s16) + 2, 0, 3) (nearest level, ties up),
 *     q = 2 everywhere when s16 == 0. Dequantised weight = s16 * (q - 1.5).
 *     The weights are expressed in the rotated basis, so the product uses
 *     x' = H_512 D x / sqrt(512) (see lbq_hadamard) in place of x. K % 512 == 0.
 *
 * Storage order (all formats). The per-row byte strings above are stored with rows
 *   interleaved in groups of four, so that one 16-byte load brings the same 32-bit
 *   word of four rows. N is padded to a multiple of four with zero rows. In group g
 *   (rows 4g .. 4g+3) the group's codes take 4 * code_stride bytes starting at byte
 *   g * 4 * code_stride, and 32-bit word w of row 4g+q (its bytes 4w .. 4w+3) sits at
 *   bytes 16 w + 4 q of the group. Scales likewise: the group's 4 * scale_stride fp16
 *   start at element g * 4 * scale_stride, and scale e of row 4g+q is element 4 e + q
 *   of the group. Padding rows and padding words are zero bytes.
 *
 * Shape rules: K % 128 == 0 (LBQ_Q2RHT: K % 512 == 0), K >= 128, N >= 1, M >= 1;
 * a batch-1 product split over K (K > 512, or > 1024 for LBQ_SIGN1) has N <= 524288.
 * Alignment rules: codes, scales, x/X, W, D, out and workspace 16-byte aligned;
 * y/Y 2-byte aligned. Strides must be at least the packed row size; code strides a
 * multiple of 16 bytes, scale strides a multiple of 8 elements (16 bytes): the
 * kernels stream both with TMA.
 */
#ifndef LBQ_H
#define LBQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lbq_status {
  LBQ_OK = 0,
  LBQ_ERR_ARG = 1,        /* null pointer or bad enum/flag value            */
  LBQ_ERR_SHAPE = 2,      /* K, N, M or a stride violates the shape rules  */
  LBQ_ERR_ALIGN = 3,      /* a pointer violates the alignment rules        */
  LBQ_ERR_FORMAT = 4,     /* unknown packed format                         */
  LBQ_ERR_CUDA = 5,       /* a CUDA runtime call or launch failed          */
  LBQ_ERR_WORKSPACE = 6,  /* workspace missing or smaller than required    */
  LBQ_ERR_DEVICE_WAIT = 7 /* a bounded wait inside a kernel gave up        */
} lbq_status;

typedef enum lbq_format {
  LBQ_TERN5 = 1, /* ternary, 5 trits per byte, fp16 scale per 128, in-block     */
  LBQ_SIGN1 = 2, /* 1-bit sign, fp16 scale per 128, separate scale array       */
  LBQ_Q2RHT = 3  /* 2-bit 4-level, fp16 scale per 32, input rotated by RHT-512  */
} lbq_format;

/* A packed weight matrix (descriptor only; the buffers belong to the caller). */
typedef struct lbq_weights {
  int32_t fmt;           /* lbq_format                                            */
  int32_t reserved;      /* must be 0                                             */
  int64_t K;             /* input features (packed along a row)                   */
  int64_t N;             /* output features (rows)                                */
  const void* codes;     /* device, ceil(N/4) groups of 4*code_stride bytes        */
  const void* scales;    /* device, ceil(N/4) groups of 4*scale_stride fp16;       *
                          * NULL for LBQ_TERN5                                     */
  int64_t code_stride;   /* code bytes per row (a group holds four rows)           */
  int64_t scale_stride;  /* fp16 scales per row (0 for TERN5)                      */
} lbq_weights;

/* Human-readable name of a status. Never NULL. Host only. */
const char* lbq_status_string(lbq_status st);

/* The CUDA runtime error (a cudaError_t value) behind the last LBQ_ERR_CUDA that a
 * call returned on the calling host thread, or 0 if none has; and its text (never
 * NULL). Host only; no CUDA call is made. */
int32_t lbq_last_cuda_error(void);
const char* lbq_last_cuda_error_string(void);

/* Packed sizes for a K x N matrix in format `fmt` (host only, no CUDA call).
 * Any output pointer may be NULL. code_stride/scale_stride are the minimal
 * strides; with N4 = N rounded up to a multiple of four (the storage order groups
 * rows in fours), code_bytes = N4 * code_stride, scale_bytes = N4 * scale_stride * 2.
 * Errors: LBQ_ERR_FORMAT, LBQ_ERR_SHAPE. */
lbq_status lbq_packed_layout(int32_t fmt, int64_t K, int64_t N, int64_t* code_stride,
                             int64_t* scale_stride, size_t* code_bytes, size_t* scale_bytes);

/* Quantise and pack W (device fp32 [N][K], row-major, 16-byte aligned) into
 * `codes` (code_bytes) and `scales` (scale_bytes; NULL for TERN5) in the
 * group-of-four storage order, using the minimal strides of lbq_packed_layout;
 * padding rows and words are written as zeros. Rule per format: see the
 * header comment ([tern] §5.1 applied per block as in [block] §2.1; [sign]; [rht]).
 * Deterministic and bit-exact: the same W always gives the same bytes. Offline
 * step, not tuned for speed. */
lbq_status lbq_pack(int32_t fmt, const float* W, int64_t K, int64_t N, void* codes,
                    void* scales, void* stream);

/* Unpack codes to int8 values (t in {-1,0,1} for TERN5, 2b-1 in {-1,1} for SIGN1,
 * q in {0,1,2,3} for Q2RHT) into out [N][K] (device), and the block scales as fp32
 * into scales_out [N][K/blk] (device; blk = 128, or 32 for Q2RHT) when non-NULL.
 * A test hook for the bit-exact code check. */
lbq_status lbq_unpack(const lbq_weights* w, int8_t* out, float* scales_out, void* stream);

/* Random signs D[k] in {-1,+1}, k < K, for the Hadamard rotation ([rht]):
 * D[k] = -1 iff bit 63 of the (k+1)-th output of SplitMix64 seeded with `seed`
 * is set (Steele, Lea & Flood 2014; Vigna's public-domain reference generator).
 * D is a device int8 array of K elements. */
lbq_status lbq_rht_signs(uint64_t seed, int64_t K, int8_t* D, void* stream);

/* Block random Hadamard transform of M rows of bf16 activations ([rht]):
 * out[m][512c+i] = 2^-4.5 * sum_j (-1)^popcount(i&j) * D[512c+j] * x[m][512c+j].
 * x is [M][K] bf16 (row stride K), out is [M][K] fp32, K % 512 == 0.
 * One warp per (row, 512-block) computes the 9-stage butterfly in fp32: four stages
 * within each lane's 16 values in registers, five across lanes with warp shuffles.
 * (Output is fp32 only, and D is a device array only: the rotated activations feed
 * fp32 arithmetic, and the signs are made on the device from the seed.) */
lbq_status lbq_hadamard(const uint16_t* x, const int8_t* D, int64_t M, int64_t K,
                        float* out, void* stream);

/* Bytes of device workspace lbq_gemv / lbq_gemm need for this matrix and M
 * (0: none). The first 64 KB of a workspace hold arrival counters: they must be
 * zero when the workspace is first used, and every completed call leaves them zero
 * again, so one zero-fill at allocation serves any sequence of calls on matrices
 * of any shape. The rest is scratch. Calls sharing one workspace must not overlap
 * in time (use one workspace per stream). Returns 0 on bad arguments. */
size_t lbq_workspace_bytes(const lbq_weights* w, int64_t M);

/* Batch-1 product y = W_hat x (bf16 x [K] -> bf16 y [N]) with W_hat the dequantised
 * weights; for LBQ_Q2RHT the input is first rotated, y = W_hat (H D x / sqrt 512),
 * with D from lbq_rht_signs (NULL for other formats). fp32 accumulation; y is
 * rounded to bf16 once, at the end. Workspace as lbq_workspace_bytes(w, 1).
 * Ordering: the product starts early beside the previous kernel of the stream
 * (programmatic dependent launch) and touches x, y and the workspace only once that
 * kernel has finished, but it reads the packed weights at once. Weights written on
 * the same stream are therefore safe as long as the writing kernel does not itself
 * let its successor start early: lbq_pack, copies and ordinary kernels do not.
 * Errors: LBQ_ERR_ARG (nulls, D missing for Q2RHT), LBQ_ERR_SHAPE, LBQ_ERR_ALIGN,
 * LBQ_ERR_FORMAT, LBQ_ERR_WORKSPACE, LBQ_ERR_CUDA. */
lbq_status lbq_gemv(const lbq_weights* w, const uint16_t* x, const int8_t* D, uint16_t* y,
                    void* workspace, size_t workspace_bytes, void* stream);

/* lbq_gemv with an fp32 y [N] (4-byte aligned) in place of bf16: the same product,
 * without the final rounding, for partial products that are added up afterwards
 * (a layer whose input features are split over GPUs sums each GPU's partial y; a
 * residual add). Same arguments, workspace and errors as lbq_gemv. */
lbq_status lbq_gemv_f32(const lbq_weights* w, const uint16_t* x, const int8_t* D, float* y,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Batched product Y[m][n] = sum_k W_hat[n][k] X[m][k] for M rows of bf16 X
 * ([M][K], row stride K) into bf16 Y ([M][N], row stride N). Ternary weights:
 * up to 3 rows run as one batch-1 product per row (lbq_gemv's kernels, in stream
 * order), more rows dequantise weight tiles into tensor memory and run tcgen05
 * fp16 MMAs with fp32 accumulation. The activations are scaled into fp16 by an exact
 * power of two per row; a row whose values do not all convert exactly (its values
 * span more than about 2^31) is recomputed in fp32 on the CUDA cores, which is
 * slower but keeps the same accuracy. 1-bit and 2-bit weights: a CUDA-core kernel
 * in which each warp decodes a weight row's blocks once for up to 8 activation rows.
 * Same formats, D and workspace rules as lbq_gemv (workspace for this M, from
 * lbq_workspace_bytes). */
lbq_status lbq_gemm(const lbq_weights* w, const uint16_t* X, int64_t M, const int8_t* D,
                    uint16_t* Y, void* workspace, size_t workspace_bytes, void* stream);

/* Measurement hook: reads `bytes` of device memory at p once (16-byte loads that do
 * not allocate in L1, four CTAs per SM) and XORs the words read into *sink (device,
 * 4-byte aligned), so that nothing is skipped. Its rate is the ceiling a plain read
 * stream reaches on this GPU, the third denominator (after the nominal figure and
 * the measured copy rate) for the products' weight streams. Not part of the method.
 * Errors: LBQ_ERR_ARG (nulls), LBQ_ERR_SHAPE (bytes 0 or not a multiple of 16),
 * LBQ_ERR_ALIGN (p not 16-byte aligned), LBQ_ERR_CUDA. */
lbq_status lbq_read_probe(const void* p, size_t bytes, uint32_t* sink, void* stream);

/* Most products one launch of lbq_gemv_batch takes (longer lists, or lists of several
 * formats, run as several launches). */
#define LBQ_BATCH_MAX 256

/* One batch-1 product of a list: y = W_hat x (W_hat from w; D for LBQ_Q2RHT, else NULL). */
typedef struct lbq_product {
  lbq_weights w;
  const uint16_t* x;  /* device bf16 [K]                          */
  const int8_t* D;    /* device int8 [K] rotation signs, or NULL   */
  uint16_t* y;        /* device bf16 [N]                           */
} lbq_product;

/* Bytes of workspace lbq_gemv_batch needs for this list (0 on bad arguments): 64 KB
 * kept under the counter rule of lbq_workspace_bytes (zero when the workspace is first
 * used, zero again after every completed call; this call leaves them untouched), then
 * the piece sums of the products it splits along K (none for lists of many rows). */
size_t lbq_gemv_batch_workspace_bytes(const lbq_product* ps, int32_t n);

/* n independent batch-1 products, each within the bound lbq_gemv meets (the same
 * lookup arithmetic: [tern] §1.2, [block] §2.1-2.2, [sign], [rht]; its fp32 sums run
 * over the K-slices in slice order, so an output may differ from lbq_gemv's inside the
 * bound), computed by one launch per format present and LBQ_BATCH_MAX products of it,
 * in list order within a format. The list's products are laid end to end as 16-row
 * units of full K and cut into one range per SM, of equal cost (units plus table
 * builds): each CTA computes whole rows,
 * slice by slice, keeping running sums in shared memory, and no CTA waits for
 * another. A product too short in rows for that cut is split along K; its pieces'
 * fp32 sums go to the workspace and a second kernel adds them in piece order. Results
 * are deterministic. The products must be independent: no x or D of the list may
 * overlap any y of the list, and no two y may overlap (checked on the host:
 * LBQ_ERR_ARG). Products may use different formats and shapes. `ps` is host memory,
 * read during the call only (the list travels in the launch's parameters). Workspace
 * as lbq_gemv_batch_workspace_bytes; calls sharing one workspace must not overlap.
 * Errors: those of lbq_gemv for any product, LBQ_ERR_ARG (ps NULL, n < 1, overlap),
 * LBQ_ERR_WORKSPACE, LBQ_ERR_CUDA. */
lbq_status lbq_gemv_batch(const lbq_product* ps, int32_t n, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Most CTAs one launch of lbq_gemv_batch uses (one per SM, at most this many). */
#define LBQ_BATCH_MAX_CTAS 192

/* The schedule lbq_gemv_batch gives one launch's list when it runs `ctas` CTAs (it runs
 * one per SM): host only, no device work, for inspection and tests. The list must be
 * one launch's: one format, 1..LBQ_BATCH_MAX products, valid as for lbq_gemv_batch.
 * Work is counted in unit-slices (one 16-row unit of one K-slice: 512 weights, 1024 for
 * LBQ_SIGN1); product i has KS_i slices, NU_i = ceil(N_i / 16) units and starts at
 * c0_i = sum of KS_j * NU_j over j < i. Writes pieces[i] (host int32 [n]): the pieces
 * product i is split into along K (piece s holds slices [KS s / S, KS (s + 1) / S); 1:
 * whole rows on one CTA), bound (host int64 [ctas + 1]): CTA c computes the units
 * whose first unit-slice lies in [bound[c], bound[c + 1]) (unit u of piece s of product
 * i starts at c0_i + NU_i * j0 + u * (j1 - j0)), and *total, the list's unit-slices.
 * Errors: LBQ_ERR_ARG (NULL outputs, ctas < 1 or > LBQ_BATCH_MAX_CTAS, n > LBQ_BATCH_MAX,
 * mixed formats), and those of lbq_gemv_batch's checks. */
lbq_status lbq_gemv_batch_plan(const lbq_product* ps, int32_t n, int32_t ctas, int32_t* pieces,
                               int64_t* bound, int64_t* total);

/* Size of the scratch array that lbq_gemv_noalloc uses (4 MiB). */
#define LBQ_NOALLOC_SCRATCH_BYTES (4u << 20)

/* Reports whether a bounded wait inside one of the library's kernels gave up on the
 * current device since the last query, and clears that record. Every wait in the
 * kernels (on an mbarrier, for a TMA copy or a slot) is bounded by about 2 s; a
 * wait that runs out records a non-zero *code (3: shared-memory layout of the
 * batch-1 product, 4-9: tensor-core product stages, 10: the batch-1 product's
 * weight copies, 11: lbq_selftest_wait, 12: unused (lbq_gemv_batch has no waits),
 * 13: lbq_gemv_batch's shared-memory layout) and the kernel returns early with
 * incomplete outputs instead of hanging. Synchronises the device.
 * Returns LBQ_OK with *code = 0 when no wait gave up, LBQ_ERR_DEVICE_WAIT with the
 * code otherwise. Errors: LBQ_ERR_ARG (code NULL), LBQ_ERR_CUDA. */
lbq_status lbq_device_fault(uint32_t* code);

/* Test hook for the path above: enqueues a kernel whose one bounded wait (on an
 * mbarrier nothing arrives on, limited to 20 ms) runs out, records code 11 and
 * returns. The device stays usable; the next lbq_device_fault reports and clears it.
 * Errors: LBQ_ERR_CUDA. */
lbq_status lbq_selftest_wait(void* stream);

/* lbq_gemv without a workspace argument, for callers that cannot allocate device
 * memory: a host that reaches the library only through this C interface and has no
 * device allocator of its own, or one that must not call cudaMalloc once it is
 * running (cudaMalloc can synchronise the device, and a framework's memory pool
 * cannot account for memory taken behind its back). The pages have no counterpart
 * of this call; it only changes where the scratch memory comes from.
 *
 * Same arguments, result and errors as lbq_gemv, minus the workspace. The scratch
 * is one array of LBQ_NOALLOC_SCRATCH_BYTES compiled into the library: every GPU
 * that loads the library holds it until the process exits. A call whose product
 * needs more scratch than that (lbq_workspace_bytes(w, 1)) returns
 * LBQ_ERR_WORKSPACE and enqueues nothing; use lbq_gemv with your own workspace
 * then. The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 * library routine. It enqueues the product's kernels only: the product writes every
 * scratch value before reading it, and the array's arrival counters, which it never
 * writes, are zero from the moment the library is loaded, so there is nothing to
 * clear between calls.
 *
 * The first call on each device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream capture.
 * All calls on a device share the one array: calls that can overlap on the GPU
 * (different streams without ordering between them) race on it and give wrong
 * results. Order them on one stream, or use lbq_gemv with one workspace each. */
lbq_status lbq_gemv_noalloc(const lbq_weights* w, const uint16_t* x, const int8_t* D,
                            uint16_t* y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LBQ_H */
