/*
 * mxq.h -- C ABI of libmxq.so: block-scaled low-precision quantization of
 * training tensors on NVIDIA B200 (sm_100a).
 *
 *   MXFP8 rowwise: groups of 32 consecutive elements along the last dim share
 *   one power-of-two E8M0 scale; elements are FP8 E4M3.
 *   MXFP4 rowwise: the same power-of-two E8M0 scale per group of 32, with
 *   FP4 E2M1 elements packed two per byte.
 *   NVFP4 two-level: an fp32 global scale times per-16-element E4M3 block
 *   scales; elements are FP4 E2M1, packed two per byte.
 *
 * Sources (page title, section):
 *  - "PR #1935 完整报告 -- Use TransformerEngine for MXFP8 quantization",
 *    实现拆解 item 1 and 关键源码片段: `qweight, scale = mxfp8_quantize(weight)`,
 *    group size 32, rowwise only, rows zero-padded to a multiple of 32 and
 *    cropped back, compact non-swizzled (qweight, scale); the scale is stored
 *    as "<name>_scale_inv", a dequantisation multiplier. 实现拆解 item 4:
 *    grouped quantization of stacked expert weights (mxfp8_group_quantize).
 *  - "V4 mxfp4 #1372": power-of-two (float8_e8m0fnu) scales on Blackwell;
 *    E2M1 stored two per byte (float4_e2m1fn_x2, last dim N//2), with
 *    N % block_size == 0.
 *  - "Add FP8, NVFP4, and QARL training and export", review "What looked
 *    solid": NVFP4 two-level global + FP8-block scaling, the effective
 *    scale being the block scale times the global scale, zero blocks guarded.
 *  - "feat(training): MXFP8 混合精度训练落地", and the same xorl review,
 *    item 2: failures are visible, never a silent downgrade -- this library
 *    has no fallback path; every error is a status code.
 *
 * Conventions (all entry points):
 *  - Tensor pointers are DEVICE pointers owned by the caller (for example
 *    PyTorch tensors); host pointers appear only where stated. The library
 *    never allocates, frees or synchronizes, and keeps no state between
 *    calls (except the fixed scratch array of nvfp4_quantize_noalloc).
 *  - Work is enqueued on `stream` (NULL = the legacy default stream) and runs
 *    asynchronously; outputs are ready when the stream reaches that point.
 *  - Arguments are checked on the host before anything is enqueued. A call
 *    that returns anything other than MXQ_OK for an argument error has
 *    enqueued nothing. MXQ_ERR_CUDA reports a failed launch
 *    (cudaGetLastError after the launch); the CUDA error string is then
 *    available from mxq_last_cuda_error() on the calling thread.
 *  - Shapes are int64_t element counts, row-major; ld_x is the row stride of
 *    the input in elements (ld_x >= N). M == 0 is valid and does nothing
 *    (pointers may then be NULL).
 *  - Alignment: inputs and ld_x * element size must be multiples of 16 bytes;
 *    qweight / packed / outputs y must be 16-byte aligned; scale arrays have
 *    no alignment requirement. Otherwise MXQ_ERR_ALIGN.
 *  - Results are bit-exact functions of the input bits (no atomics on data,
 *    no order-dependent arithmetic): repeated calls give identical bytes.
 */
#ifndef MXQ_H_
#define MXQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA
 * include. */
typedef struct CUstream_st* mxq_stream_t;

typedef enum {
  MXQ_OK = 0,
  MXQ_ERR_NULL = 1,          /* a required pointer is NULL */
  MXQ_ERR_SHAPE = 2,         /* negative size, N not a multiple of the group
                                or block, ld_x < N, or a size limit exceeded */
  MXQ_ERR_DTYPE = 3,         /* unknown mxq_dtype */
  MXQ_ERR_ALIGN = 4,         /* pointer or row stride misaligned */
  MXQ_ERR_WORKSPACE = 5,     /* workspace NULL or smaller than required */
  MXQ_ERR_CUDA = 6,          /* a CUDA call or launch failed */
  MXQ_ERR_ARG = 7            /* inconsistent flags or arguments */
} mxq_status;

typedef enum { MXQ_BF16 = 0, MXQ_FP32 = 1 } mxq_dtype;

/* MX element formats (mx_fake_quantize). */
typedef enum { MXQ_FMT_MXFP8 = 0, MXQ_FMT_MXFP4 = 1 } mxq_mx_format;

#define MXQ_ABI_VERSION 2
#define MXQ_MXFP8_GROUP 32
#define MXQ_NVFP4_BLOCK 16
#define MXQ_GROUPED_MAX_EXPERTS 1024
#define MXQ_NVFP4_GLOBAL_GIVEN 1u
#define MXQ_NVFP4_MAX_SLICES 1024

/* Version of this ABI (MXQ_ABI_VERSION of the built library). */
int mxq_abi_version(void);

/* Static, human-readable name of a status code. */
const char* mxq_status_string(int status);

/* Message of the last CUDA error seen by this thread's calls ("" if none). */
const char* mxq_last_cuda_error(void);

/* ------------------------------------------------------------------ MXFP8 */

/* Bytes of the swizzled scale layout for an [M, S] scale (S = N/32):
 * ceil(M/128)*128 * ceil(S/4)*4. Returns -1 for negative sizes. */
int64_t mxq_swizzled_scale_bytes(int64_t M, int64_t S);

/* MXFP8 rowwise quantize ("PR #1935 完整报告 ...", 实现拆解 item 1).
 *  x        [M, N] bf16 or fp32 (dt), row stride ld_x elements.
 *  qweight  [M, N] uint8, E4M3 codes, row-major, compact.
 *  scale    [M, N/32] uint8, E8M0 biased exponents, row-major, compact:
 *           byte (r, j) covers row r, columns 32j .. 32j+31.
 *  scale_swz  NULL, or mxq_swizzled_scale_bytes(M, N/32) bytes that receive
 *           the same scales in the 128x4-tile layout read by block-scaled
 *           tensor-core MMA (tile (i, j) = rows 128i.., scale columns 4j..,
 *           at byte (i*ceil(S/4) + j)*512; entry (r, c) inside it at
 *           (r%32)*16 + ((r%128)/32)*4 + c%4; padding bytes are 0x00);
 *           N/32 > 2^27 - 4 with scale_swz is rejected (MXQ_ERR_SHAPE).
 * Per group: amax = max |x| over non-NaN elements; byte = 127 if amax == 0,
 * 254 if amax is infinite, else clamp(floor(log2 amax) - 8 + 127, 0, 254);
 * q = E4M3(x * 2^(127 - byte)) rounded to nearest even, |.| > 448 saturating
 * to 448, NaN -> 0x7F, zero results keeping the sign.
 * Rows need no padding: groups never cross rows, so the result equals the
 * pages' pad-to-32-rows-then-crop contract for any M.
 * Errors: NULL x/qweight/scale (M > 0), N % 32 != 0, ld_x < N, M*N/32 >=
 * 2^32, misalignment. */
mxq_status mxfp8_quantize(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                          uint8_t* qweight, uint8_t* scale, uint8_t* scale_swz,
                          mxq_stream_t stream);

/* MXFP8 dequantize: y[r, c] = decode_e4m3(q[r, c]) * 2^(scale[r, c/32] - 127)
 * ("_scale_inv" is the dequantisation multiplier, "PR #1935 完整报告 ...",
 * 关键源码片段). Computed exactly, then written as fp32 (exact; overflow to
 * inf only for scale byte 254) or bf16 (round to nearest even, subnormals
 * kept). NaN codes give 0x7FC0 / 0x7FC00000; scale byte 255 gives NaN.
 *  qweight [M, N] uint8, scale [M, N/32] uint8, y [M, N] of out_dt. */
mxq_status mxfp8_dequantize(const uint8_t* qweight, const uint8_t* scale, int64_t M,
                            int64_t N, void* y, int out_dt, mxq_stream_t stream);

/* Grouped MXFP8 quantize of a stack of E expert weights held in one tensor,
 * in one launch ("PR #1935 完整报告 ...", 实现拆解 item 4: grouped
 * quantization of stacked expert weights, mxfp8_group_quantize; "V4 mxfp4
 * #1372", description: MoE expert weights).
 *  x            [M_total, N] bf16 or fp32 (dt), contiguous rows; expert e
 *               owns rows [row_offsets[e], row_offsets[e+1]).
 *  row_offsets  DEVICE int64 [E + 1], 8-byte aligned, non-decreasing, with
 *               row_offsets[0] == 0 and row_offsets[E] == M_total (those two
 *               entries are taken as 0 and M_total, not read). Experts may be
 *               empty. 1 <= E <= MXQ_GROUPED_MAX_EXPERTS.
 *  qweight [M_total, N], scale [M_total, N/32]: compact, as for M_total rows.
 * Groups never cross rows, so every output byte equals what mxfp8_quantize
 * gives each expert on its own and what it gives the flattened [M_total, N]
 * tensor: the offsets do not change the compact outputs, and this call does
 * not read them (mxfp8_quantize_grouped_swizzled does). */
mxq_status mxfp8_quantize_grouped(const void* x, int dt, int32_t E, const int64_t* row_offsets,
                                  int64_t M_total, int64_t N, uint8_t* qweight, uint8_t* scale,
                                  mxq_stream_t stream);

/* mxfp8_quantize_grouped that also writes each expert's scales in its own
 * 128x4-tile swizzled layout (the layout described at mxfp8_quantize), as a
 * grouped block-scaled GEMM over the experts reads them: expert e's block is
 * mxq_swizzled_scale_bytes(M_e, N/32) bytes (its rows padded to a multiple
 * of 128, padding bytes 0x00) and starts where expert e-1's ends.
 *  scale_swz  device buffer of swz_bytes bytes, 16-byte aligned; it must hold
 *             the sum over the experts of mxq_swizzled_scale_bytes(M_e, N/32),
 *             which is at most mxq_grouped_swizzled_scale_bytes_max(E,
 *             M_total, N/32).
 * Two launches: the quantize of mxfp8_quantize_grouped, then a gather of each
 * expert's compact scales into its swizzled block, which reads row_offsets on
 * the device. Offsets that break the rules above are clamped into a
 * non-decreasing sequence from 0 to M_total, and no byte at or past
 * scale_swz + swz_bytes is written, whatever the offsets. N/32 > 2^27 - 4 is
 * rejected (MXQ_ERR_SHAPE). */
mxq_status mxfp8_quantize_grouped_swizzled(const void* x, int dt, int32_t E,
                                           const int64_t* row_offsets, int64_t M_total, int64_t N,
                                           uint8_t* qweight, uint8_t* scale, uint8_t* scale_swz,
                                           int64_t swz_bytes, mxq_stream_t stream);

/* Writes a compact [M, S] scale array in the 128x4-tile layout described at
 * mxfp8_quantize (rows padded to a multiple of 128 and columns to a multiple
 * of 4 with 0x00): the E8M0 scales of mxfp8_quantize / mxfp4_quantize
 * (S = N/32), or the E4M3 block scales of nvfp4_quantize (S = N/16), which
 * block-scaled tensor-core MMAs read in the same tiling. (The pages have no
 * such step; it lays out what the quantizers wrote.)
 *  scale      device [M, S] bytes, row-major, compact.
 *  scale_swz  device, 16-byte aligned, mxq_swizzled_scale_bytes(M, S) bytes.
 * M == 0 or S == 0 writes nothing; S > 2^27 - 4 is rejected (MXQ_ERR_SHAPE).
 * One launch. */
mxq_status mxq_swizzle_scales(const uint8_t* scale, int64_t M, int64_t S, uint8_t* scale_swz,
                              mxq_stream_t stream);

/* Upper bound of the per-expert swizzled scale bytes of E experts with
 * M_total rows in all (each expert adds at most 127 padding rows):
 * floor((M_total + 127 E) / 128) * 128 * ceil(S/4) * 4; -1 for negative
 * sizes. */
int64_t mxq_grouped_swizzled_scale_bytes_max(int32_t E, int64_t M_total, int64_t S);

/* Grouped MXFP8 quantize of E expert tensors that live in separate
 * allocations, in one launch.
 *  xs    HOST array of E device pointers; expert e is a contiguous
 *        [rows[e], N] tensor of dtype dt (16-byte aligned).
 *  rows  HOST array of E row counts (>= 0).
 *  qweight [sum rows, N] and scale [sum rows, N/32]: expert e's rows follow
 *        expert e-1's, as if the experts were stacked and quantized by
 *        mxfp8_quantize (identical bytes).
 * 1 <= E <= MXQ_GROUPED_MAX_EXPERTS (the pointers and per-expert tile counts
 * travel in the kernel's parameters). The host arrays are read during the
 * call only. */
mxq_status mxfp8_quantize_grouped_ptrs(int32_t E, const void* const* xs, const int64_t* rows,
                                       int64_t N, int dt, uint8_t* qweight, uint8_t* scale,
                                       mxq_stream_t stream);

/* MXFP8 columnwise quantize: groups of 32 consecutive ROWS of one column (the
 * layout a backward GEMM reads), i.e. the rowwise quantize of the transposed
 * tensor. Rows are zero-padded to a multiple of 32 and the result cropped
 * back ("PR #1935 完整报告 ...", 实现拆解 item 1); for columnwise groups the
 * zero padding takes part in the last group of every column.
 *  x          [M, N] bf16 or fp32, row stride ld_x elements; N % 16 == 0.
 *  qweight_t  [N, M] uint8 E4M3 codes (transposed, row-major): qweight_t[c, r]
 *             is the code of x[r, c].
 *  scale_t    [N, ceil(M/32)] uint8 E8M0 bytes.
 *  qweight, scale  both NULL, or the rowwise outputs of mxfp8_quantize
 *             ([M, N] and [M, N/32], compact; then N % 32 == 0): the fused
 *             mode produces both layouts from one read of x.
 * Per group the rule of mxfp8_quantize applies (amax over non-NaN elements,
 * E8M0 byte, E4M3 RNE with saturation). One launch; tiles of 128 rows x 256
 * bytes staged in shared memory. */
mxq_status mxfp8_quantize_columnwise(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                                     uint8_t* qweight_t, uint8_t* scale_t, uint8_t* qweight,
                                     uint8_t* scale, mxq_stream_t stream);

/* ------------------------------------------------------------------ MXFP4 */

/* MXFP4 rowwise quantize ("V4 mxfp4 #1372": E8M0 power-of-two scales per
 * group of 32, E2M1 elements stored as float4_e2m1fn_x2 with last dim N/2;
 * the QAT simulation mxfp4_simulate_qat(kv, 32) uses the same groups).
 * The rule of mxfp8_quantize with E2M1 in place of E4M3: byte = 127 if
 * amax == 0, 254 if amax is infinite, else clamp(floor(log2 amax) - 2 + 127,
 * 0, 254) (2 = exponent of E2M1's largest value, 6 = 1.5 * 2^2); the code is
 * E2M1(x * 2^(127 - byte)) rounded to nearest even, |.| > 6 saturating to 6,
 * NaN -> +6 (0x7), zero results keeping the sign.
 *  x        [M, N] bf16 or fp32 (dt), row stride ld_x elements; N % 32 == 0.
 *  packed   [M, N/2] uint8: element 2k in the low nibble, 2k+1 in the high.
 *  scale    [M, N/32] uint8 E8M0 bytes, compact.
 *  scale_swz  NULL, or mxq_swizzled_scale_bytes(M, N/32) bytes receiving the
 *           scales in the 128x4-tile layout described at mxfp8_quantize.
 * Errors as for mxfp8_quantize. */
mxq_status mxfp4_quantize(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                          uint8_t* packed, uint8_t* scale, uint8_t* scale_swz,
                          mxq_stream_t stream);

/* MXFP4 dequantize: y[r, c] = decode_e2m1(code) * 2^(scale[r, c/32] - 127),
 * exact in fp32 (overflow to inf only for scale bytes above 252), written as
 * fp32 or bf16 (round to nearest even). Scale byte 255 gives NaN (0x7FC0 /
 * 0x7FC00000). packed [M, N/2], scale [M, N/32], y [M, N] of out_dt. */
mxq_status mxfp4_dequantize(const uint8_t* packed, const uint8_t* scale, int64_t M, int64_t N,
                            void* y, int out_dt, mxq_stream_t stream);

/* Grouped MXFP4 quantize of a stacked tensor: arguments and rules as for
 * mxfp8_quantize_grouped, outputs packed [M_total, N/2] and scale
 * [M_total, N/32], identical to mxfp4_quantize of the stacked rows. */
mxq_status mxfp4_quantize_grouped(const void* x, int dt, int32_t E, const int64_t* row_offsets,
                                  int64_t M_total, int64_t N, uint8_t* packed, uint8_t* scale,
                                  mxq_stream_t stream);

/* mxfp4_quantize_grouped plus per-expert swizzled scales, as for
 * mxfp8_quantize_grouped_swizzled. */
mxq_status mxfp4_quantize_grouped_swizzled(const void* x, int dt, int32_t E,
                                           const int64_t* row_offsets, int64_t M_total, int64_t N,
                                           uint8_t* packed, uint8_t* scale, uint8_t* scale_swz,
                                           int64_t swz_bytes, mxq_stream_t stream);

/* Grouped MXFP4 quantize of E experts in separate allocations: arguments as
 * for mxfp8_quantize_grouped_ptrs, outputs packed [sum rows, N/2] and scale
 * [sum rows, N/32]. */
mxq_status mxfp4_quantize_grouped_ptrs(int32_t E, const void* const* xs, const int64_t* rows,
                                       int64_t N, int dt, uint8_t* packed, uint8_t* scale,
                                       mxq_stream_t stream);

/* ------------------------------------------------------- fake quantize */

/* Fused fake-quantize (QAT simulation: "V4 mxfp4 #1372", mxfp4_simulate_qat;
 * "PR #1935 完整报告 ...", the round trip through (qweight, scale)):
 * y = dequantize(quantize(x)) for fmt MXQ_FMT_MXFP8 or MXQ_FMT_MXFP4, in one
 * pass that reads x once and writes y once; the codes and scales are never
 * stored. Bytes of y are identical to mxfp8_/mxfp4_quantize followed by the
 * matching dequantize with out_dt.
 *  x  [M, N] bf16 or fp32 (dt), row stride ld_x; N % 32 == 0.
 *  y  [M, N] of out_dt, contiguous, 16-byte aligned; may not overlap x.
 * Errors: unknown fmt -> MXQ_ERR_ARG; otherwise as for mxfp8_quantize. */
mxq_status mx_fake_quantize(int fmt, const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                            void* y, int out_dt, mxq_stream_t stream);

/* ------------------------------------------------ block-scaled MXFP8 GEMM */

/* D = A * B^T on the tensor cores (tcgen05 kind::mxf8f6f4.block_scale), the
 * consumer of mxfp8_quantize's codes and swizzled scales:
 *   D[m, n] = sum_k decode(qa[m, k]) 2^(sa[m, k/32] - 127)
 *                 * decode(qb[n, k]) 2^(sb[n, k/32] - 127),
 * products exact, accumulated in fp32 in an order of the hardware's choosing.
 * (The pages quantize weights and activations for block-scaled GEMMs: "V4
 * mxfp4 #1372", description; "PR #1935 完整报告 ...", 功能与动机. This entry
 * point is the consumer that reads the swizzled scale layout.)
 *  qa      [M, K] uint8 E4M3 codes, row-major (mxfp8_quantize of A).
 *  sa_swz  mxq_swizzled_scale_bytes(M, K/32) bytes: A's scales in the
 *          128x4-tile layout (mxfp8_quantize's scale_swz).
 *  qb      [N, K] uint8 E4M3 codes, row-major (B as a linear layer's
 *          [out, in] weight), sb_swz its swizzled scales.
 *  d       [M, N] row-major, bf16 (RNE of the fp32 sum) or fp32 (out_dt).
 *  error_flag  NULL, or a device int32 that the kernel sets to a non-zero
 *          code if one of its waits gives up (after about one second); the
 *          result is then undefined. It is never cleared by the library.
 * K % 32 == 0, N % 16 == 0; all pointers 16-byte aligned. K == 0 writes
 * zeros. One launch of persistent CTAs (at most one per multiprocessor, 192
 * threads, about 220 KB of shared memory each): when M > 128 and N > 128,
 * clusters of two CTAs over 256 x 256 output tiles (the pair form of the
 * MMA); otherwise single CTAs over 128 x 256 tiles (128 x 128 when
 * N <= 128). */
mxq_status mxfp8_gemm(const uint8_t* qa, const uint8_t* sa_swz, const uint8_t* qb,
                      const uint8_t* sb_swz, int64_t M, int64_t N, int64_t K, void* d,
                      int out_dt, int32_t* error_flag, mxq_stream_t stream);

/* Self-check of the bounded barrier wait that lets mxfp8_gemm give up
 * instead of hanging (the wait behind error_flag), run on the device in one
 * single-thread launch: first a wait, limited to timeout_ns, on a
 * shared-memory barrier that nothing arrives on; then a wait on a barrier
 * whose phase the thread has just completed. Writes the device array result
 * (4 int64, 8-byte aligned):
 *   result[0]  1 if the first wait gave up, else 0 (expected 1);
 *   result[1]  1 if the second wait saw its phase complete, else 0 (1);
 *   result[2]  nanoseconds the first wait took, by %globaltimer;
 *   result[3]  0.
 * The wait polls with a 20 us suspend hint and reads %globaltimer every 16
 * polls, so the first wait ends within about timeout_ns + 0.7 ms.
 * 1000 <= timeout_ns <= 1000000000, else MXQ_ERR_ARG; result NULL ->
 * MXQ_ERR_NULL; result not 8-byte aligned -> MXQ_ERR_ALIGN. */
mxq_status mxq_check_bounded_wait(int64_t timeout_ns, int64_t* result, mxq_stream_t stream);

/* ------------------------------------------------------------------ NVFP4 */

/* Workspace bytes nvfp4_quantize / nvfp4_amax need (per-CTA partial maxima of
 * the tensor-amax pass); a constant independent of M and N. */
size_t mxq_nvfp4_workspace_bytes(int64_t M, int64_t N);

/* Tensor amax (max |x| over non-NaN elements, fp32) into *amax (device).
 * The pass-1 reduction of nvfp4_quantize on its own, for a tensor sharded
 * across ranks: all-reduce the per-rank amax with MAX, then pass it to
 * nvfp4_quantize as amax_in. */
mxq_status nvfp4_amax(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                      float* amax, void* workspace, size_t ws_bytes, mxq_stream_t stream);

/* NVFP4 two-level quantize ("Add FP8, NVFP4, and QARL training and export",
 * review; "V4 mxfp4 #1372", review), all arithmetic in fp32:
 *   g    = A / 2688 (A = tensor amax, 2688 = 448 * 6), written to
 *          *global_scale; or, with flags & MXQ_NVFP4_GLOBAL_GIVEN, read from
 *          *global_scale; or, with amax_in != NULL, A read from *amax_in;
 *   per block of 16: s_b = E4M3(amax_b / (6 g)) (RNE, saturating),
 *          eff = decode(s_b) * g, q_i = E2M1(x_i / eff) (correctly rounded
 *          quotient, then RNE, |.| > 6 -> 6, NaN -> +6), or a zero of x_i's
 *          sign when eff == 0 (zero-block guard); g == 0 gives s_b = 0.
 *  packed      [M, N/2] uint8: element 2k in the low nibble, 2k+1 high.
 *  block_scale [M, N/16] uint8 E4M3 codes.
 *  global_scale device fp32 scalar (out, or in with GLOBAL_GIVEN).
 *  amax_in     device fp32 scalar or NULL; must be NULL with GLOBAL_GIVEN.
 *  workspace   device, >= mxq_nvfp4_workspace_bytes; needed only when the
 *              tensor amax is computed here (no GLOBAL_GIVEN, no amax_in).
 * N % 16 != 0 -> MXQ_ERR_SHAPE. Non-finite inputs are outside the method's
 * contract: the same fp32 operations are applied to them. */
mxq_status nvfp4_quantize(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                          uint8_t* packed, uint8_t* block_scale, float* global_scale,
                          const float* amax_in, uint32_t flags, void* workspace,
                          size_t ws_bytes, mxq_stream_t stream);

/* nvfp4_quantize without a workspace argument, for callers that cannot
 * allocate device memory at the point where they quantize: code running
 * inside a serving engine or plugin whose device memory is planned up front,
 * or a C program with no device allocator of its own. (The pages have no
 * counterpart to this entry point; it is an interface convenience.)
 * Arguments, results and errors are those of nvfp4_quantize. The scratch of
 * the tensor-amax pass (2048 fp32 partial maxima, 8 KiB) lives in a fixed
 * array inside the library, which every GPU that loads the library holds
 * until the process exits; the call allocates nothing.
 *  - The first call on a device looks up that array's device address with the
 *    caller's current device (one cudaGetSymbolAddress) and keeps it, keyed
 *    by the id of the current CUDA context; make that first call before any
 *    stream capture. A call that finds another context current (after a
 *    cudaDeviceReset, say) looks the address up again, so make the first
 *    call after such a change before any capture too. stream must belong to
 *    the current device.
 *  - Every call on a device shares the one array, so calls whose work
 *    overlaps on the GPU (for example on two streams) race and give wrong
 *    results; serialize them. Nothing in the array needs to start at zero:
 *    each call writes every slot it reads.
 *  - A call whose scratch need (mxq_nvfp4_workspace_bytes(M, N)) exceeds the
 *    array is rejected with MXQ_ERR_WORKSPACE; today the need is 8 KiB for
 *    every M and N. */
mxq_status nvfp4_quantize_noalloc(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                                  uint8_t* packed, uint8_t* block_scale, float* global_scale,
                                  const float* amax_in, uint32_t flags, mxq_stream_t stream);

/* ------------------------------------------- NVFP4, one global scale per slice */

/* Workspace bytes of nvfp4_quantize_sliced / nvfp4_amax_sliced:
 * 4 * (2048 + n_slices); 0 for n_slices outside [1, MXQ_NVFP4_MAX_SLICES]. */
size_t mxq_nvfp4_sliced_workspace_bytes(int32_t n_slices);

/* NVFP4 quantize of x [M, N] cut into n_slices consecutive row ranges, each
 * with its own global scale ("Add FP8, NVFP4, and QARL training and export",
 * review: _nvfp4_block_quantize_per_slice, weight_scale_2 per expert;
 * non-blocking item 3: a fused gate/up weight takes one global scale per
 * half during QAT and one shared scale per expert at export). Each slice is
 * quantized exactly as nvfp4_quantize would quantize a tensor holding only
 * its rows: g_s = A_s / 2688 with A_s the slice's amax, then the block rule
 * of nvfp4_quantize with g_s. Typical slicings of a stacked expert weight
 * [E, R, N]: R rows per slice (one scale per expert), or R/2 (one scale per
 * gate / up half of a fused gate/up weight whose first R/2 rows are the
 * gate).
 *  slice_rows    HOST array of n_slices row counts (>= 0, summing to M), read
 *                during the call only; 1 <= n_slices <= MXQ_NVFP4_MAX_SLICES.
 *  packed, block_scale  as for nvfp4_quantize ([M, N/2], [M, N/16]).
 *  global_scales device fp32 [n_slices]: written (g_s; 0 for an empty slice),
 *                or read with flags & MXQ_NVFP4_GLOBAL_GIVEN.
 *  amax_in       NULL, or device fp32 [n_slices] slice amaxes (for example
 *                all-reduced across ranks): g_s = amax_in[s] / 2688.
 *  workspace     >= mxq_nvfp4_sliced_workspace_bytes(n_slices), when the
 *                slice amaxes are computed here.
 * M == 0 or N == 0 writes nothing. Errors as for nvfp4_quantize, and
 * MXQ_ERR_SHAPE for a bad slicing. Two launches (amax pass, block pass), or
 * one with GLOBAL_GIVEN or amax_in. */
mxq_status nvfp4_quantize_sliced(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                                 int32_t n_slices, const int64_t* slice_rows, uint8_t* packed,
                                 uint8_t* block_scale, float* global_scales,
                                 const float* amax_in, uint32_t flags, void* workspace,
                                 size_t ws_bytes, mxq_stream_t stream);

/* Slice amaxes (max |x| over each slice's non-NaN elements, 0 for an empty
 * slice) into device fp32 amax[n_slices]: the amax pass of
 * nvfp4_quantize_sliced on its own. */
mxq_status nvfp4_amax_sliced(const void* x, int dt, int64_t M, int64_t N, int64_t ld_x,
                             int32_t n_slices, const int64_t* slice_rows, float* amax,
                             void* workspace, size_t ws_bytes, mxq_stream_t stream);

/* NVFP4 dequantize ("Add FP8, NVFP4, and QARL training and export", review
 * "What looked solid": the effective scale is the block scale times the
 * global scale): eff = decode_e4m3(s_b) * g and y = decode_e2m1(q) * eff,
 * both fp32 products, written as fp32 or bf16 (RNE); NaN products (only from
 * a non-finite g) are written as the canonical NaN.
 *  packed [M, N/2], block_scale [M, N/16] as nvfp4_quantize writes them;
 *  global_scale device fp32 scalar; y [M, N] of out_dt, 16-byte aligned.
 * Errors: N % 16 != 0, NULL pointers (M > 0), misalignment. */
mxq_status nvfp4_dequantize(const uint8_t* packed, const uint8_t* block_scale,
                            const float* global_scale, int64_t M, int64_t N, void* y,
                            int out_dt, mxq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_H_ */
