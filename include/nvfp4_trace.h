/*
 * nvfp4_trace.h -- C ABI of libnvfp4trace.so: NVFP4 block quantization with
 * train/rollout rounding alignment (TRACE-style guidance), for sm_100a.
 *
 * Sources cited below (pages are named by title; none has numbered sections):
 *   [TRACE]  "TRACE explainer" -- blog.ontle.kr/blog/286
 *   [RLQ]    "Quantization in RL training" -- ai-systems-engineering.com/posts/rl-quantized-training
 *   [TML4]   "Thinking Machines Lab releases 4-bit training" -- metallab.ai/2026/11/thinking-machines-4bit-training
 *
 * ---------------------------------------------------------------------------
 * Number format (one definition for both the rollout and the train side, the
 * "same quantization convention on both engines" of [RLQ], shared-convention
 * paragraph):
 *
 *   * 16 consecutive values of a row share one scale ([TML4], paragraph on the
 *     forward/backward mismatch); 4 bits per code + 8 bits per 16 values =
 *     4.5 bits per value ([TRACE], guidance-volume paragraph; [TML4], format
 *     comparison table).
 *   * Code: E2M1, 4 bits = sign<<3 | m, magnitude index m in 0..7 selects
 *     G = {0, 0.5, 1, 1.5, 2, 3, 4, 6} (16 representable values, [TML4]).
 *   * Block scale: one E4M3 byte (OCP "fn": bias 7, max 448, no inf,
 *     min subnormal 2^-9).  Tensor scale: one FP32 decode multiplier s_t.
 *   * Decoded value = (G[m] * sb) * s_t with the sign applied: code times scale
 *     ([RLQ], "code 3 with scale 0.1 is 0.3, with scale 0.2 it is 0.6").
 *
 * Scale recipe (all FP32 ops IEEE round-to-nearest-even, no FMA, no FTZ):
 *   A    = max |x| over the tensor
 *   s_t  = A / 2688            (2688 = 6 * 448);  A == 0  ->  s_t = 1
 *   sb   = E4M3_RNE_satfinite((amax_block / 6) / s_t)
 *   inv  = 1 / (sb * s_t)      sb == 0  ->  every code of the block is sign<<3
 *   v    = x * inv;  m = RNE onto G of |v| (ties to even m; |v| > 6 -> 6);
 *   sign = sign bit of x.
 *
 * Storage layouts (row-major, caller-owned device buffers):
 *   x       [rows, cols]        BF16 bit patterns (uint16), cols % 16 == 0
 *   codes   [rows, cols/2]      bytes; element 2j in the low nibble of byte j
 *   scales  [rows, cols/16]     E4M3 bytes, block b covers elements 16b..16b+15
 *   hints   n*bits/8 bytes      read LSB first.  bits 4: element i at bit 4i.
 *                               bits 1, 2: block b (elements 16b..16b+15) owns
 *                               bits 16*bits*b ..; its element k takes field
 *                               2*(k%8) + k/8 (fields of k and k+8 adjacent)
 *   ws      NVFP4_WS_WORDS uint32 words of device scratch (see below)
 *
 * Conventions for every call:
 *   * Pointers are DEVICE pointers unless stated; the library never allocates,
 *     frees or keeps them.  Alignment (NVFP4_ERR_MISALIGNED otherwise): BF16
 *     inputs and y_out 32 bytes (one 16-value block is one 256-bit load),
 *     codes/scales/hints/ws 16 bytes, tensor scales 4, counters 8.  Any
 *     row-offset view of a [rows, cols] tensor keeps these (cols % 16 == 0).
 *   * `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it; they return once the kernels are enqueued.
 *   * Arguments are validated before anything is enqueued: a call that returns
 *     an error has written nothing.  Inputs are never modified.
 *   * n = rows * cols must be below 2^40 (NVFP4_ERR_SHAPE otherwise).
 *   * NVFP4_ERR_CUDA means a launch failed; cudaGetLastError() has been
 *     consumed, the stream's earlier work is unaffected.
 *   * Non-finite inputs are outside the contract: they never fault, the
 *     outputs are unspecified and bit NVFP4_WARN_NONFINITE is set in ws[1].
 */
#ifndef NVFP4_TRACE_H_
#define NVFP4_TRACE_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int nvfp4_status;

#define NVFP4_OK                0
#define NVFP4_ERR_INVALID_ARG   1   /* null pointer, negative size, bad flag */
#define NVFP4_ERR_MISALIGNED    2   /* a pointer breaks its alignment rule (see above) */
#define NVFP4_ERR_SHAPE         3   /* cols % 16 (RHT: % 32), rows % 16 (SR), size >= 2^40 */
#define NVFP4_ERR_CUDA          4   /* a kernel launch failed */
#define NVFP4_ERR_UNSUPPORTED   5   /* hint_bits not in {1, 2, 4} */
#define NVFP4_ERR_SCRATCH_LIMIT 6   /* batch above NVFP4_SR_NOALLOC_MAX_BATCH (no-allocation entry point) */

/* Scratch words written by the amax pass and read by the quantize pass:
 *   ws[0] = FP32 bits of A, ws[1] = warning bits, ws[2] = max |D| observed by
 *   nvfp4_gemm_quantize, ws[3] reserved;
 *   ws[4], ws[5] = the amax pass's arrival counter and running maximum, which
 *   must be ZERO before the first call that uses this ws (allocate it zeroed)
 *   and which every call leaves zero (the pass needs no clearing launch);
 *   ws[6..7] reserved (left zero). */
#define NVFP4_WS_WORDS          8
#define NVFP4_WARN_NONFINITE    1u  /* ws[1]: an input was Inf or NaN */
#define NVFP4_WARN_TIMEOUT      2u  /* ws[1]: a pipeline wait inside nvfp4_gemm_quantize gave
                                       up (outputs unspecified; the GPU stays usable) */

/* flags */
#define NVFP4_AMAX_PRECOMPUTED  1   /* ws[0] already holds A (e.g. from nvfp4_tensor_amax) */

/* stats8 indices (nvfp4_mismatch_stats). "pos" is the signed grid position
 * (s ? -m : m), so +0 and -0 are the same position. */
#define NVFP4_STAT_ELEMENTS      0  /* elements compared */
#define NVFP4_STAT_CODE_MISMATCH 1  /* pos_a != pos_b */
#define NVFP4_STAT_ADJACENT      2  /* |pos_a - pos_b| == 1 */
#define NVFP4_STAT_FAR           3  /* |pos_a - pos_b| >= 2 */
#define NVFP4_STAT_SUM_ABS_DELTA 4  /* sum of |pos_a - pos_b| */
#define NVFP4_STAT_SCALE_MISMATCH 5 /* 16-blocks whose E4M3 scale bytes differ */
#define NVFP4_STAT_VALUE_MISMATCH 6 /* decoded FP32 values differ (-0 == +0) */
#define NVFP4_STATS8_WORDS       8  /* word 7: left unchanged, except that bit 0 is set if a
                                       bounded wait of the counting pipeline gave up (never
                                       expected; the counters are then unspecified) */

/* stats4 indices (nvfp4_guided_requant) */
#define NVFP4_GSTAT_CONSULTED    0  /* off-grid and |v| < 6: the hint decided */
#define NVFP4_GSTAT_CHANGED      1  /* guided code != round-to-nearest code */
#define NVFP4_GSTAT_OUTSIDE      2  /* hint matched neither bracket end: RTN kept */
#define NVFP4_STATS4_WORDS       4  /* word 3 is reserved (left unchanged) */

/*
 * nvfp4_tensor_amax -- A = max |x| over n BF16 values.
 *   Defines the per-tensor scale's input ([TML4]: a shared scale needs the
 *   group maximum).  ws[0] receives the FP32 bit pattern of A (exact: the
 *   maximum of BF16 magnitudes is a BF16 value), ws[1] the warning bits, and
 *   ws[2], ws[3] are cleared.  One kernel launch: the CTA that finishes last
 *   publishes the result (ws[4], ws[5] must be zero on entry, see
 *   NVFP4_WS_WORDS).  n == 0 gives A = 0.
 */
nvfp4_status nvfp4_tensor_amax(const uint16_t* x_bf16, int64_t n, uint32_t* ws,
                               void* stream);

/*
 * nvfp4_quantize_rtn -- rollout-side round-to-nearest NVFP4 quantization, with
 * an optional fused hint emit.
 *   [TRACE], rounding-analogy paragraph: each engine rounds to the nearest
 *   cell; the compaction paragraph: the rollout ships only the low bits that
 *   tell adjacent cells apart.
 *   x [rows, cols] BF16 -> codes, scales, *tensor_scale = s_t.
 *   ws: scratch; unless flags has NVFP4_AMAX_PRECOMPUTED the call first runs
 *   the amax pass into it.
 *   hints: NULL for none (hint_bits ignored), else hint_bits in {1, 2, 4}:
 *   1 -> m & 1, 2 -> m & 3 (magnitude bits, no sign), 4 -> the full code.
 *   rows == 0 or cols == 0: writes *tensor_scale = 1 and nothing else.
 */
nvfp4_status nvfp4_quantize_rtn(const uint16_t* x_bf16, int64_t rows, int64_t cols,
                                uint32_t* ws, int flags,
                                uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                uint8_t* hints, int hint_bits, void* stream);

/*
 * nvfp4_emit_hint -- standalone compact hint from already-quantized codes.
 *   [TRACE], compaction paragraph (>99% of mismatches are one cell apart, so a
 *   few low bits of the code pick the rollout's cell).
 *   codes: n/2 bytes (n % 16 == 0) -> hints: ceil(n*hint_bits/8) bytes.
 */
nvfp4_status nvfp4_emit_hint(const uint8_t* codes, int64_t n, int hint_bits,
                             uint8_t* hints, void* stream);

/*
 * nvfp4_guided_requant -- train-side re-quantization that follows the
 * rollout's cell.
 *   [TRACE], prescription paragraph: near a boundary the train side takes the
 *   cell the rollout chose instead of the nearest one.
 *   The train tensor gets its own A, s_t, sb, inv and v exactly as in
 *   nvfp4_quantize_rtn.  With a = |v| and lo = #{g in G, g > 0, g <= a}:
 *     a >= 6            -> m = 7
 *     a == G[lo]        -> m = lo (no rounding decision, hint ignored)
 *     otherwise         -> hi = lo + 1;  m = lo if h == lo (mod 2^bits),
 *                          hi if h == hi (mod 2^bits), else round-to-nearest.
 *   hint_bits 1 or 2 compare magnitudes; the sign comes from x.  hint_bits 4
 *   compares signed grid positions (the bracket is the pair of signed grid
 *   points around v).  hints == NULL gives plain round-to-nearest.
 *   stats4: NULL, or NVFP4_STATS4_WORDS uint64 counters that are ADDED to
 *   (the caller zeroes them).
 */
nvfp4_status nvfp4_guided_requant(const uint16_t* x_train_bf16, int64_t rows, int64_t cols,
                                  const uint8_t* hints, int hint_bits,
                                  uint32_t* ws, int flags,
                                  uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                  uint64_t* stats4, void* stream);

/*
 * nvfp4_mismatch_stats -- train/rollout discrepancy counters between two NVFP4
 * tensors of the same shape.
 *   [TRACE]: the distance between the two paths is the quantity to shrink
 *   (opening and prescription paragraphs); most mismatches are one cell apart
 *   (compaction paragraph).
 *   ts_a, ts_b: device pointers to the two FP32 tensor scales.
 *   stats8: NVFP4_STATS8_WORDS uint64 counters that are ADDED to (the caller
 *   zeroes them); indices NVFP4_STAT_*.  Decoded values use
 *   (G[m] * sb) * s_t in FP32 (the first product is exact).
 */
nvfp4_status nvfp4_mismatch_stats(const uint8_t* codes_a, const uint8_t* scales_a,
                                  const float* ts_a,
                                  const uint8_t* codes_b, const uint8_t* scales_b,
                                  const float* ts_b,
                                  int64_t rows, int64_t cols, uint64_t* stats8,
                                  void* stream);

/*
 * nvfp4_guided_requant_stats -- nvfp4_guided_requant and nvfp4_mismatch_stats
 * against the rollout's tensor in one pass over the train tensor.
 *   [TRACE]: the train side follows the rollout's cells (prescription
 *   paragraph), and the train/rollout distance is what the method shrinks
 *   (opening and compaction paragraphs).  The counters compare the rollout's
 *   NVFP4 tensor (roll_codes, roll_scales, *roll_tensor_scale: side a) with
 *   the train codes this call produces (side b), counted while they are still
 *   in registers instead of being written and read back.
 *   Outputs, bit for bit: codes, scales, *tensor_scale and stats4 as
 *   nvfp4_guided_requant with the same arguments; stats8 (required, ADDED to,
 *   the caller zeroes it; word 7 unchanged) as nvfp4_mismatch_stats(roll_codes,
 *   roll_scales, roll_tensor_scale, codes, scales, tensor_scale, rows, cols,
 *   stats8) run afterwards.  roll_codes [rows, cols/2] and roll_scales
 *   [rows, cols/16] 16-byte aligned, roll_tensor_scale a device float.
 *   rows == 0 or cols == 0: writes *tensor_scale = 1 and nothing else.
 */
nvfp4_status nvfp4_guided_requant_stats(const uint16_t* x_train_bf16, int64_t rows, int64_t cols,
                                        const uint8_t* hints, int hint_bits,
                                        uint32_t* ws, int flags,
                                        uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                        uint64_t* stats4,
                                        const uint8_t* roll_codes, const uint8_t* roll_scales,
                                        const float* roll_tensor_scale, uint64_t* stats8,
                                        void* stream);

/*
 * nvfp4_sr_transpose_requant -- dequantize, transpose, stochastic-rounding
 * re-quantize, for a stack of `batch` independent [rows, cols] matrices.
 *   [TML4], forward/backward mismatch paragraph: transposing changes which 16
 *   values share a scale, so return to high precision, transpose, and
 *   re-quantize with stochastic rounding (2.25 -> 2 three times in four, 3
 *   once; the mean is kept).
 *   Per matrix e: y = (G[m] * sb) * s_t[e];  y^T is [cols, rows]; it gets its
 *   own A', s_t', sb', inv' by the recipe above; v = y * inv'; with a = |v|,
 *   a >= 6 -> 6; on-grid values stay; otherwise lo/hi bracket a and
 *     p = (a - G[lo]) / (G[hi] - G[lo]),
 *     r = Philox4x32-10(key = (seed lo32, seed hi32),
 *                       counter = (i lo32, i hi32, draw, 0)).x0,
 *     round up iff (r >> 8) < p * 2^24,
 *   i = row-major index of the element in the OUTPUT stack [batch, cols, rows].
 *   Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *   easy as 1, 2, 3", SC'11.
 *   codes [batch, rows, cols/2], scales [batch, rows, cols/16],
 *   tensor_scale [batch] -> codes_t [batch, cols, rows/2],
 *   scales_t [batch, cols, rows/16], tensor_scale_t [batch].
 *   ws: batch uint32 words of scratch (per-matrix amax of y), cleared here.
 *   rows % 16 == 0 and cols % 16 == 0 (NVFP4_ERR_SHAPE).
 */
nvfp4_status nvfp4_sr_transpose_requant(const uint8_t* codes, const uint8_t* scales,
                                        const float* tensor_scale,
                                        int64_t batch, int64_t rows, int64_t cols,
                                        uint64_t seed, uint32_t draw, uint32_t* ws,
                                        uint8_t* codes_t, uint8_t* scales_t,
                                        float* tensor_scale_t, void* stream);

/*
 * nvfp4_rht_quantize -- 32-point random Hadamard transform, then NVFP4
 * round-to-nearest quantization.
 *   [TML4], communication paragraph: a 32-dimensional random Hadamard
 *   transform precedes the low-bit combine payload.
 *   For each contiguous group of 32 values of a row:
 *     y = (H32 * (sigma (.) x)) * fl32(1/sqrt(32)),
 *   H32 the Sylvester Hadamard matrix H[i][j] = (-1)^popcount(i & j),
 *   sigma_j = (Philox4x32-10(key = (seed lo32, seed hi32),
 *                            counter = (j, 0, 0, 0)).x0 & 1) ? -1 : +1,
 *   one sign vector for the whole tensor.  Then A, s_t, sb, codes as in
 *   nvfp4_quantize_rtn on the FP32 y.  cols % 32 == 0 (NVFP4_ERR_SHAPE).
 *   y_out: NULL, or [rows, cols] FP32 receiving y (for verification).
 */
nvfp4_status nvfp4_rht_quantize(const uint16_t* x_bf16, int64_t rows, int64_t cols,
                                uint64_t sign_seed, uint32_t* ws,
                                uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                float* y_out, void* stream);

/*
 * nvfp4_sr_transpose_requant_noalloc -- nvfp4_sr_transpose_requant for callers
 * that cannot allocate device memory.  (The pages have no counterpart: this is
 * an interface variant, not a step of the method.)
 *   Who needs it: callers that may not call cudaMalloc at this point -- e.g. a
 *   rollout/serving engine that reserved nearly all HBM for its weight and
 *   KV-cache pools at start-up and forbids later allocations, or C code with no
 *   caching allocator that cannot afford the device synchronisation a
 *   cudaMalloc/cudaFree may cause mid-step.  They cannot supply `ws`.
 *   What it does: exactly what nvfp4_sr_transpose_requant does (same outputs,
 *   bit for bit), with the per-matrix scratch words taken from a fixed array of
 *   NVFP4_SR_NOALLOC_MAX_BATCH uint32 (16 KiB) inside the library.  Every GPU
 *   that loads the library holds that array until the process exits.  Inputs
 *   and outputs are still the caller's device buffers; nothing is allocated.
 *   Limit: batch > NVFP4_SR_NOALLOC_MAX_BATCH returns NVFP4_ERR_SCRATCH_LIMIT
 *   and enqueues nothing.
 *   Argument checks are those of nvfp4_sr_transpose_requant (same status for
 *   the same arguments, batch == 0 returns NVFP4_OK), then the limit below.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current -- call with the stream's
 *   device current) and caches it; make that first call before any stream
 *   capture.  The cached address is valid for that device's primary context
 *   only: after cudaDeviceReset (or any teardown of the primary context) the
 *   process must not call this entry point again.
 *   Sharing: all calls on a device share the one array; each call clears the
 *   words it uses on `stream` before its kernels read them, and the array keeps
 *   the last call's contents.  Calls whose work overlaps on the GPU (different
 *   streams without ordering between them) race on the array: order them.
 */
#define NVFP4_SR_NOALLOC_MAX_BATCH 4096
nvfp4_status nvfp4_sr_transpose_requant_noalloc(const uint8_t* codes, const uint8_t* scales,
                                                const float* tensor_scale,
                                                int64_t batch, int64_t rows, int64_t cols,
                                                uint64_t seed, uint32_t draw,
                                                uint8_t* codes_t, uint8_t* scales_t,
                                                float* tensor_scale_t, void* stream);

/* ======================================================================
 * Hint transport: the guidance leaves the GPU.
 * ====================================================================== */

/*
 * nvfp4_hint_pack -- gather the hint streams of several tensors (the layers
 * that ship guidance) into one contiguous device staging buffer, then copy it
 * to host memory.
 *   [TRACE], guidance-volume paragraph: the guidance of every step leaves the
 *   GPU (to host memory or storage), and its volume and that transfer are the
 *   cost of naive alignment; compaction paragraph: only the back half of the
 *   layers ship guidance, as a few low bits per code (the hint streams of
 *   nvfp4_quantize_rtn / nvfp4_emit_hint; no further compaction here).
 *   srcs, sizes: HOST arrays of `count` device pointers and byte counts (any
 *   size >= 0; a non-empty stream 16-byte aligned).  staging: device buffer
 *   of nvfp4_hint_pack_size(sizes, count) bytes, 16-byte aligned: stream i
 *   occupies bytes off_i .. off_i + sizes[i] - 1 with off_i = the sum over
 *   j < i of sizes[j] rounded up to a multiple of 16; the bytes up to the next
 *   multiple of 16 are written as 0.  One gather kernel per 128 streams.
 *   host_dst: NULL (staging only), or host memory of the same size that
 *   receives the staging buffer by one cudaMemcpyAsync on `stream` after the
 *   gather (page-locked memory keeps the call asynchronous; pageable memory
 *   makes the copy synchronous with the host).  Total size below 2^40
 *   (NVFP4_ERR_SHAPE).  count == 0 or all sizes 0: nothing is enqueued.
 */
nvfp4_status nvfp4_hint_pack(const uint8_t* const* srcs, const int64_t* sizes, int64_t count,
                             uint8_t* staging, uint8_t* host_dst, void* stream);

/* Staging size in bytes for nvfp4_hint_pack (sum of sizes rounded up to 16
 * each), or -1 for a negative count or size, a NULL `sizes` with count > 0,
 * or a total of 2^40 or more.  Host-only; touches no device. */
int64_t nvfp4_hint_pack_size(const int64_t* sizes, int64_t count);

/* ======================================================================
 * KV-cache layout: one FP32 scale per row.
 * ====================================================================== */

/*
 * nvfp4_quantize_rtn_rows / nvfp4_guided_requant_rows -- the rollout and
 * train quantizers for a KV cache [tokens x heads, head_dim].
 *   [TRACE], hyper-parameter table: the rollout keeps the KV cache in FP4 as
 *   well.  A cache entry is written one token at a time, so no tensor-wide
 *   amax exists when it is quantized: every row (one token's vector for one
 *   head) is its own tensor, with its own FP32 scale s_row = amax_row / 2688
 *   (1 for an all-zero row) and 16-value blocks along head_dim, quantized
 *   exactly as nvfp4_quantize_rtn / nvfp4_guided_requant quantize a
 *   one-row tensor (same rounding, hints and guidance rules).
 *   x_bf16 [rows, cols], cols = head_dim in {16, 32, 64, 128, 256, 512}
 *   (NVFP4_ERR_SHAPE otherwise); codes [rows, cols/2], scales [rows, cols/16],
 *   row_scales [rows] floats; hints laid out as for the tensor calls (the
 *   hints of row r start at byte r * cols * bits / 8).  No scratch: the row
 *   amax is reduced inside the kernel.  stats4 as in nvfp4_guided_requant
 *   (added to).  Non-finite inputs: outputs unspecified (there is no warning
 *   word on this path).
 */
nvfp4_status nvfp4_quantize_rtn_rows(const uint16_t* x_bf16, int64_t rows, int64_t cols,
                                     uint8_t* codes, uint8_t* scales, float* row_scales,
                                     uint8_t* hints, int hint_bits, void* stream);
nvfp4_status nvfp4_guided_requant_rows(const uint16_t* x_bf16, int64_t rows, int64_t cols,
                                       const uint8_t* hints, int hint_bits, uint8_t* codes,
                                       uint8_t* scales, float* row_scales, uint64_t* stats4,
                                       void* stream);

/* ======================================================================
 * Alternatives to nvfp4_sr_transpose_requant that [TML4] weighs
 * (forward/backward mismatch paragraph and format table).
 * ====================================================================== */

#define NVFP4_SCALES_BLOCK16  0   /* one scale per 16 consecutive values of a row */
#define NVFP4_SCALES_TILE16   1   /* one scale per 16 x 16 tile */

/*
 * nvfp4_quantize_tile16 -- NVFP4 with one E4M3 scale per 16 x 16 tile.
 *   [TML4], forward/backward mismatch paragraph: NVIDIA's proposal enlarges
 *   the group that shares a scale to a 256-value tile, which a transpose maps
 *   onto itself (so no re-quantization is needed after transposing), at the
 *   price of one large value flattening the rest of its tile.
 *   Recipe as nvfp4_quantize_rtn with the block amax replaced by the tile
 *   amax: sb = RNE_E4M3_satfinite((amax_tile / 6) / s_t), inv = 1/(sb * s_t),
 *   codes round-to-nearest, sign from x.
 *   x_bf16 [rows, cols], rows % 16 == cols % 16 == 0 (NVFP4_ERR_SHAPE).
 *   codes [rows, cols/2] (same layout as blocks), tile_scales [rows/16,
 *   cols/16] row-major E4M3 bytes, tensor_scale: 1 float.  ws and flags as in
 *   nvfp4_quantize_rtn.
 */
nvfp4_status nvfp4_quantize_tile16(const uint16_t* x_bf16, int64_t rows, int64_t cols,
                                   uint32_t* ws, int flags, uint8_t* codes,
                                   uint8_t* tile_scales, float* tensor_scale, void* stream);

/*
 * nvfp4_transpose_tile16 -- transpose a stack of tile-scaled NVFP4 matrices
 * without re-rounding: code (r, c) moves to (c, r), tile scale (i, j) to
 * (j, i); each matrix keeps its tensor scale (the caller reuses it).  The
 * result equals nvfp4_quantize_tile16 of the transposed input, bit for bit.
 *   codes [batch, rows, cols/2], tile_scales [batch, rows/16, cols/16] ->
 *   codes_t [batch, cols, rows/2], tile_scales_t [batch, cols/16, rows/16].
 *   rows % 16 == cols % 16 == 0, batch <= 65535 (NVFP4_ERR_SHAPE).
 */
nvfp4_status nvfp4_transpose_tile16(const uint8_t* codes, const uint8_t* tile_scales,
                                    int64_t batch, int64_t rows, int64_t cols,
                                    uint8_t* codes_t, uint8_t* tile_scales_t, void* stream);

/*
 * mxfp8_sr_transpose_requant -- dequantize a stack of NVFP4 matrices,
 * transpose, and re-quantize to MXFP8 with stochastic rounding.
 *   [TML4]: the backward runs in MXFP8 with stochastic rounding after the
 *   dequantize -> transpose step; MXFP8 costs 8.25 bits per value (format
 *   table): 8-bit E4M3 elements and one 8-bit E8M0 scale per 32 values.
 *   Per matrix e: y = (G[m] * sb) * s_t[e] as in nvfp4_sr_transpose_requant,
 *   y^T is [cols, rows]; each 32 consecutive values of a row of y^T share
 *   2^x, x = floor(log2(amax_32)) - 8 clamped to [-127, 127] (-127 for an
 *   all-zero block; OCP MX: 8 is the exponent of E4M3's top binade), stored
 *   as the byte x + 127.  v = y * 2^-x; with a = |v|: a >= 448 -> 448; lo =
 *   the largest E4M3 value <= a, hi the next one;
 *     round up iff (r >> 8) < ((a - lo) / (hi - lo)) * 2^24,
 *   r the same Philox4x32-10 word as in nvfp4_sr_transpose_requant (counter
 *   = row-major index i in the OUTPUT stack [batch, cols, rows], draw).
 *   Element byte = sign(y) << 7 | E4M3 bits of the magnitude.
 *   codes [batch, rows, cols/2], scales [batch, rows, cols/16],
 *   tensor_scale [batch] -> q_t [batch, cols, rows] bytes,
 *   e8_t [batch, cols, rows/32] bytes.  rows % 32 == 0, cols % 16 == 0,
 *   batch <= 65535 (NVFP4_ERR_SHAPE).  No scratch: every scale is per block.
 */
nvfp4_status mxfp8_sr_transpose_requant(const uint8_t* codes, const uint8_t* scales,
                                        const float* tensor_scale,
                                        int64_t batch, int64_t rows, int64_t cols,
                                        uint64_t seed, uint32_t draw,
                                        uint8_t* q_t, uint8_t* e8_t, void* stream);

/*
 * nvfp4_dequantize -- NVFP4 -> FP32: value = sign * ((G[m] * sb) * s_t) in
 * FP32 (the first product is exact).  [RLQ]: a decoded value is the code's
 * value times the scale.
 *   scale_layout NVFP4_SCALES_BLOCK16: scales [rows, cols/16];
 *   NVFP4_SCALES_TILE16: scales [rows/16, cols/16] (rows % 16 == 0).
 *   tensor_scale: device pointer to 1 float.  out [rows, cols] FP32, 32-byte
 *   aligned.  cols % 16 == 0.
 */
nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales,
                              const float* tensor_scale, int64_t rows, int64_t cols,
                              int scale_layout, float* out, void* stream);

/*
 * mxfp8_dequantize -- MXFP8 -> FP32: E4M3 value of q[i] times
 * 2^(e8[i / 32] - 127), one FP32 multiply (infinite if it overflows).
 *   n % 32 == 0; q, e8 16-byte aligned, out 32-byte aligned.
 */
nvfp4_status mxfp8_dequantize(const uint8_t* q, const uint8_t* e8, int64_t n, float* out,
                              void* stream);

/* ======================================================================
 * Rollout producer: NVFP4 GEMM on the tensor cores with a quantizing epilogue.
 * ====================================================================== */

/*
 * nvfp4_scales_to_mma -- row-layout block scales -> the layout the block-
 * scaled tensor-core MMA of sm_100 reads (NVIDIA PTX ISA, tcgen05 block
 * scaling; cuBLAS documentation, 1D block scaling factors layout).
 *   scales [rows, sf_cols] bytes (sf_cols = cols / 16 of the NVFP4 tensor).
 *   scales_mma: ceil(rows / 128) * ceil(sf_cols / 4) tiles of 512 bytes; tile
 *   (rt, kt) at byte (rt * ceil(sf_cols / 4) + kt) * 512 holds rows
 *   128 rt .. 128 rt + 127 and scale columns 4 kt .. 4 kt + 3, the scale of
 *   (row r, column c) at (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4; padding
 *   (rows past `rows`, columns past `sf_cols`) is written as 0.  scales_mma
 *   16-byte aligned.  Any rows, sf_cols >= 0.
 */
nvfp4_status nvfp4_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t sf_cols,
                                 uint8_t* scales_mma, void* stream);

/*
 * nvfp4_gemm_quantize -- D = s_a s_b (A B^T) on the tensor cores, quantized
 * to NVFP4 in the epilogue, with the rollout hints of D.
 *   [TML4], configuration paragraph and format table: the MoE forward GEMMs
 *   (pre-training and rollout sampling) run in NVFP4, and what they produce
 *   is sent on in NVFP4; [TRACE] (problem statement): the rollout records a
 *   few low bits of each code for the trainer.  This is the producer of those
 *   codes fused into the GEMM, so D never round-trips through HBM.
 *   A: a_codes [m, k/2] (element 2j in the low nibble), a_scales_mma its block
 *   scales in the MMA layout of nvfp4_scales_to_mma (rows m, sf_cols k/16),
 *   a_tensor_scale 1 float (device); B likewise with n rows ([n, k]: the
 *   weight of y = x W^T).
 *   Product: the block-scaled MMA's FP32 accumulation of the exact products
 *   (G_a sa)(G_b sb), then one FP32 multiply by fl(s_a * s_b).  The order and
 *   internal precision of the accumulation are the hardware's: D is not
 *   bit-reproducible against a CPU sum, its quantization of D is (same rules
 *   as nvfp4_quantize_rtn applied to FP32 D).
 *   Output tensor scale: one pass cannot know max |D| before quantizing, so
 *   ws[0] must hold the FP32 bits of the amax A_out to use (the previous
 *   step's, or a calibration); s_t = A_out / 2688 goes to tensor_scale, and
 *   blocks above 6 * 448 * s_t saturate to scale 448 / code 7.  The call
 *   clears ws[1..3], records the observed max |D| (FP32 bits) in ws[2] for the
 *   next call, and sets NVFP4_WARN_TIMEOUT in ws[1] if a pipeline wait gave up.
 *   Outputs: codes [m, n/2], scales [m, n/16] (row layout), scales_mma
 *   (nullable: the same scales in the MMA layout, ready for the next GEMM),
 *   hints (nullable; hint_bits 1, 2 or 4, laid out as nvfp4_emit_hint's),
 *   d_out (nullable: FP32 D [m, n], for checking).
 *   Shapes: m % 128 == 0, n % 128 == 0, k % 256 == 0 and k > 0
 *   (NVFP4_ERR_SHAPE); m or n == 0 only writes tensor_scale.  codes, hints and
 *   d_out 32-byte aligned (each thread writes a whole 32-byte row segment),
 *   every other pointer 16 (tensor scales 4).  Runs on sm_100 only.
 */
nvfp4_status nvfp4_gemm_quantize(const uint8_t* a_codes, const uint8_t* a_scales_mma,
                                 const float* a_tensor_scale, const uint8_t* b_codes,
                                 const uint8_t* b_scales_mma, const float* b_tensor_scale,
                                 int64_t m, int64_t n, int64_t k, uint32_t* ws, uint8_t* codes,
                                 uint8_t* scales, uint8_t* scales_mma, float* tensor_scale,
                                 uint8_t* hints, int hint_bits, float* d_out, void* stream);

/*
 * nvfp4_moe_gemm_quantize -- nvfp4_gemm_quantize over the experts of an MoE
 * layer: the routed tokens, grouped by expert, times each expert's weight,
 * one launch for all experts.
 *   [TML4], configuration paragraph: the MoE layers' forward runs in NVFP4,
 *   and tokens reach the experts in NVFP4 (communication paragraph).  The
 *   all-to-all that delivers them is not part of this call: A arrives
 *   grouped, expert e owning rows expert_rows[e] .. expert_rows[e + 1] - 1.
 *   expert_rows: device int32 [experts + 1], non-decreasing, expert_rows[0] =
 *   0, expert_rows[experts] <= m, every entry a multiple of 128 (pad each
 *   expert's tokens to 128 rows); an entry breaking that gives wrong rows,
 *   never an out-of-bounds read (every 128-row tile takes the weight of the
 *   expert owning its first row).  Rows expert_rows[experts] .. m - 1 are not
 *   computed and their outputs are left unchanged, so m may be the capacity
 *   of a grouping the GPU produced (nvfp4_moe_route) without the host
 *   reading its size back.
 *   w_codes [experts, n, k/2] and w_scales_mma (each expert's scales in the
 *   MMA layout, concatenated, i.e. the MMA layout of [experts * n, k/16]);
 *   w_tensor_scales [experts] floats (device).  D rows follow A's rows, row r
 *   of expert e being s_a s_w[e] (A_r . W_e^T); everything else (one output
 *   tensor scale from ws[0], hints, both scale layouts, ws[2], warnings,
 *   shapes, alignment) as nvfp4_gemm_quantize, expert_rows 4-byte aligned.
 *   1 <= experts <= 65536 (NVFP4_ERR_INVALID_ARG).
 */
nvfp4_status nvfp4_moe_gemm_quantize(const uint8_t* a_codes, const uint8_t* a_scales_mma,
                                     const float* a_tensor_scale, const uint8_t* w_codes,
                                     const uint8_t* w_scales_mma, const float* w_tensor_scales,
                                     const int32_t* expert_rows, int64_t experts, int64_t m,
                                     int64_t n, int64_t k, uint32_t* ws, uint8_t* codes,
                                     uint8_t* scales, uint8_t* scales_mma, float* tensor_scale,
                                     uint8_t* hints, int hint_bits, float* d_out, void* stream);

/*
 * nvfp4_moe_route -- group the routed tokens by expert, on the GPU.
 *   [TML4], communication paragraph: tokens are sent to the experts in NVFP4;
 *   the expert GEMM (nvfp4_moe_gemm_quantize) reads each expert's rows as one
 *   contiguous group padded to a multiple of 128 rows.  The pages give no
 *   layout; this is the reading taken: the assignments a = token * top_k +
 *   slot (topk_ids [tokens, top_k] int32, device) are grouped by expert id,
 *   in increasing a within an expert (a stable counting sort: every call
 *   gives the same rows); an id outside 0 .. experts - 1 drops its
 *   assignment.
 *   Outputs (device int32): expert_rows [experts + 1] (group offsets, each a
 *   multiple of 128, expert_rows[0] = 0); row_src [m_cap] (the assignment each
 *   grouped row holds, -1 for a padding row and for every row from
 *   expert_rows[experts] on); assign_row [tokens * top_k] (the row of each
 *   assignment, -1 if dropped).  m_cap >= nvfp4_moe_rows_cap(tokens * top_k,
 *   experts), the largest grouping possible (NVFP4_ERR_SHAPE otherwise).
 *   ws: nvfp4_moe_route_ws_words(tokens * top_k, experts) int32 words of
 *   device scratch, 16-byte aligned (no initial value needed).
 *   1 <= experts <= 1024, top_k >= 1, tokens * top_k < 2^31 - 2^17.
 */
nvfp4_status nvfp4_moe_route(const int32_t* topk_ids, int64_t tokens, int64_t top_k,
                             int64_t experts, int32_t* ws, int32_t* expert_rows,
                             int32_t* row_src, int64_t m_cap, int32_t* assign_row, void* stream);

/* Largest number of grouped rows for `assignments` over `experts` experts:
 * (assignments + 127 * experts) rounded down to a multiple of 128, or -1 for
 * arguments nvfp4_moe_route rejects.  Host-only. */
int64_t nvfp4_moe_rows_cap(int64_t assignments, int64_t experts);
/* Scratch words of nvfp4_moe_route (experts * (ceil(assignments / 2048) + 1),
 * at least one chunk), or -1.  Host-only. */
int64_t nvfp4_moe_route_ws_words(int64_t assignments, int64_t experts);

/*
 * nvfp4_moe_gather -- the routed tokens' NVFP4 rows in the grouped layout of
 * nvfp4_moe_gemm_quantize's A operand.
 *   codes [tokens, k/2] and scales [tokens, k/16] (row layout, as the
 *   quantizers write them) of the tokens; row_src [m_cap] from
 *   nvfp4_moe_route (any value outside 0 .. tokens * top_k - 1 is a padding
 *   row); grouped row r holds token row_src[r] / top_k.
 *   -> a_codes [m_cap, k/2] and a_scales_mma (the tensor-core layout of
 *   [m_cap, k/16], nvfp4_scales_to_mma's); padding rows are zero codes with
 *   zero scales (their products are 0).  k % 64 == 0, m_cap % 128 == 0
 *   (NVFP4_ERR_SHAPE); codes, scales, a_codes, a_scales_mma 16-byte aligned.
 */
nvfp4_status nvfp4_moe_gather(const uint8_t* codes, const uint8_t* scales, int64_t tokens,
                              int64_t k, const int32_t* row_src, int64_t m_cap, int64_t top_k,
                              uint8_t* a_codes, uint8_t* a_scales_mma, void* stream);

/*
 * nvfp4_wait_selftest -- failure detection of the producer pipeline, without
 * a fault: runs the bounded mbarrier wait that nvfp4_gemm_quantize uses on a
 * barrier that nothing completes.  After about 2 s the wait gives up and
 * NVFP4_WARN_TIMEOUT is set in ws[1] (the call clears ws[1] first); the
 * kernel returns normally and the context stays usable.  ws: NVFP4_WS_WORDS
 * words, 16-byte aligned.
 */
nvfp4_status nvfp4_wait_selftest(uint32_t* ws, void* stream);

/*
 * nvfp4_measure_mul_wide -- measurement helper (the pages have no
 * counterpart; not a step of the method): the issue rate of the
 * 32 x 32 -> 64-bit integer multiply that Philox4x32-10 spends 20 of per
 * random word, which bounds nvfp4_sr_transpose_requant and
 * mxfp8_sr_transpose_requant.  `ctas` CTAs of 1024 threads (one per SM when
 * ctas = the SM count), each thread running 8 independent multiply chains for
 * `iters` iterations; cycles[i] receives CTA i's SM clock cycles for its loop
 * (uint64, device).  Multiplies per clock per SM = 1024 * 8 * iters /
 * cycles[i].  sink: ctas uint32 words the kernel may write (keeps the work
 * from being optimised away).
 */
nvfp4_status nvfp4_measure_mul_wide(int64_t ctas, int64_t iters, uint64_t* cycles, uint32_t* sink,
                                    void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* nvfp4_status_string(nvfp4_status status);

/*
 * nvfp4_last_cuda_error -- the cudaError_t value (as int) behind the most
 * recent NVFP4_ERR_CUDA returned on the calling host thread; 0 if no call on
 * this thread has returned NVFP4_ERR_CUDA.  Not reset by later successful
 * calls.  nvfp4_last_cuda_error_string: the CUDA runtime's text for it
 * ("no error" for 0; static string, never NULL).
 */
int nvfp4_last_cuda_error(void);
const char* nvfp4_last_cuda_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_TRACE_H_ */
