/*
 * nvfp4_oracle.c -- plain, slow, scalar CPU oracle for NVFP4 quantization with
 * train/rollout rounding alignment.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check of the
 * package entry module and the CPU-baseline leg of bench.py may load this.
 * It shares no code, header, table or constant generator with the CUDA path.
 *
 * Compile with  gcc -O2 -ffp-contract=off -fno-fast-math  so that every float
 * operation below is one IEEE binary32 operation rounded to nearest-even (no
 * fused multiply-add, no flush-to-zero).  Rounding decisions onto the E2M1
 * grid and the E4M3 scale set are taken by exhaustive search over all
 * candidates, in double precision where every distance that can tie is exact.
 *
 * Pages followed (named by title):
 *   [TRACE] "TRACE explainer" (blog.ontle.kr/blog/286)
 *   [RLQ]   "Quantization in RL training" (ai-systems-engineering.com)
 *   [TML4]  "Thinking Machines Lab releases 4-bit training" (metallab.ai)
 * Numeric format: E2M1 codes, 16-value blocks with an E4M3 block scale and an
 * FP32 tensor scale; the scale recipe and every reading the pages leave open
 * are listed with the function that applies them.
 *
 * Parity pins: every function here is pinned by the tests under tests/
 * (test_oracle_*.py) against library casts, brute force, closed forms and the
 * pages' worked examples.  The per-tensor scale constants (2688 = 6 * 448) and
 * the order of the two block-scale divisions are readings, not pinned values.
 * oracle_scales_to_mma: parity unpinned on the CPU beyond its structure (the
 * byte positions are the tensor core's operand format, not the pages'); the
 * GPU tests pin it through the tensor core, whose GEMM must match
 * oracle_gemm_nvfp4.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Element format: E2M1 magnitudes.  [TML4] format comparison: 4 bits give 16
 * representable values (8 magnitudes x sign). */
static const double GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_value(int m) { return GRID[m & 7]; }

/* Round a >= 0 to the nearest grid magnitude, ties to the even index (the
 * IEEE rule: even index = zero mantissa bit), values above 6 saturate to 6.
 * Exhaustive search over the eight candidates. */
int oracle_e2m1_rne(float a)
{
    if (a != a) return 0;          /* NaN: outside the contract */
    if (a >= 6.0f) return 7;       /* saturation (includes +inf) */
    int best = 0;
    double bestd = fabs((double)a - GRID[0]);
    for (int m = 1; m < 8; ++m) {
        double d = fabs((double)a - GRID[m]);
        if (d < bestd || (d == bestd && (m % 2) == 0)) {
            best = m;
            bestd = d;
        }
    }
    return best;
}

/* ------------------------------------------------------------------------ */
/* Block-scale format: E4M3 "fn" (bias 7, no infinities, 0x7F = NaN). */
double oracle_e4m3_value(int byte)
{
    int e = (byte >> 3) & 15, mant = byte & 7;
    double mag = (e == 0) ? ldexp((double)mant, -9) : ldexp((double)(8 + mant), e - 10);
    return (byte & 0x80) ? -mag : mag;
}

/* Round f >= 0 to the nearest finite non-negative E4M3 value, ties to the
 * even byte (even mantissa), saturating at 448.  Exhaustive search over the
 * 127 finite non-negative encodings 0x00..0x7E. */
int oracle_e4m3_rne_satfinite(float f)
{
    if (f != f) return 0x7F;       /* NaN: outside the contract */
    if (f >= 448.0f) return 0x7E;  /* satfinite (includes +inf) */
    int best = 0;
    double bestd = fabs((double)f - oracle_e4m3_value(0));
    for (int b = 1; b <= 0x7E; ++b) {
        double d = fabs((double)f - oracle_e4m3_value(b));
        if (d < bestd || (d == bestd && (b % 2) == 0)) {
            best = b;
            bestd = d;
        }
    }
    return best;
}

/* ------------------------------------------------------------------------ */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static int sign_of(float f) { return signbit(f) ? 1 : 0; }

static int nibble_get(const uint8_t* p, int64_t i) { return (p[i >> 1] >> ((i & 1) * 4)) & 15; }

static void nibble_put(uint8_t* p, int64_t i, int v)
{
    int sh = (int)(i & 1) * 4;
    p[i >> 1] = (uint8_t)((p[i >> 1] & ~(15 << sh)) | ((v & 15) << sh));
}

/* ------------------------------------------------------------------------ */
/* Step 1: tensor amax.  A shared scale is fitted to the largest magnitude of
 * what it covers ([TML4], forward/backward mismatch paragraph: one large value
 * sets the scale for the rest).  Exact: the result is one of the inputs. */
float oracle_amax_f32(const float* y, int64_t n)
{
    float A = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(y[i]);
        if (a > A) A = a;
    }
    return A;
}

float oracle_amax_bf16(const uint16_t* x, int64_t n)
{
    float A = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(oracle_bf16_to_f32(x[i]));
        if (a > A) A = a;
    }
    return A;
}

/* Step 2: scales.  Tensor decode multiplier s_t = A / (6 * 448) so that the
 * largest magnitude lands on the top of both formats; A == 0 -> 1.
 * Block scale sb = E4M3((amax_block / 6) / s_t): two rounded divisions in that
 * order.  Decoded value = code value * scale ([RLQ], code 3 x scale 0.1). */
float oracle_tensor_scale(float A) { return (A == 0.0f) ? 1.0f : A / 2688.0f; }

int oracle_block_scale(float amax_block, float s_t)
{
    float q = amax_block / 6.0f;
    float sbf = q / s_t;
    return oracle_e4m3_rne_satfinite(sbf);
}

/* Step 3: the per-element scaled value v = x * (1 / (sb * s_t)), three
 * rounded FP32 operations in that order.  When s_t lies deep in the subnormal
 * range, 1 / (sb * s_t) overflows to +inf: every nonzero x then scales to
 * +-inf and saturates, and x = +-0 keeps magnitude 0 (0 * inf would be a
 * NaN; zero sits on the grid).  Callers skip the product for x == 0. */
static float scaled_value(float x, float sbv, float s_t)
{
    float denom = sbv * s_t;
    float inv = 1.0f / denom;
    return x * inv;
}

/* Round-to-nearest NVFP4 quantization of an FP32 tensor whose amax A is given
 * ([TRACE], rounding-analogy paragraph: each engine rounds to the nearest
 * cell).  codes: rows*cols/2 bytes, scales: rows*cols/16 bytes. */
void oracle_quantize_f32(const float* y, int64_t rows, int64_t cols, float A,
                         uint8_t* codes, uint8_t* scales, float* tensor_scale)
{
    float s_t = oracle_tensor_scale(A);
    *tensor_scale = s_t;
    int64_t nblk = cols / 16;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            const float* blk = y + r * cols + b * 16;
            float amax_b = 0.0f;
            for (int k = 0; k < 16; ++k)
                if (fabsf(blk[k]) > amax_b) amax_b = fabsf(blk[k]);
            int sb = oracle_block_scale(amax_b, s_t);
            scales[r * nblk + b] = (uint8_t)sb;
            float sbv = (float)oracle_e4m3_value(sb);
            for (int k = 0; k < 16; ++k) {
                int m = 0;
                if (sbv != 0.0f && blk[k] != 0.0f)
                    m = oracle_e2m1_rne(fabsf(scaled_value(blk[k], sbv, s_t)));
                nibble_put(codes, r * cols + b * 16 + k, (sign_of(blk[k]) << 3) | m);
            }
        }
    }
}

static float* bf16_rows_to_f32(const uint16_t* x, int64_t n)
{
    float* y = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    for (int64_t i = 0; i < n; ++i) y[i] = oracle_bf16_to_f32(x[i]);
    return y;
}

/* Step 4: compact hint ([TRACE], compaction paragraph).  bits 1 -> m & 1
 * (the E2M1 mantissa bit, enough to tell two adjacent cells apart), 2 ->
 * m & 3, 4 -> the whole code (the uncompacted guidance).
 *
 * Layout (the page fixes only that a few low bits are sent, not their order):
 * the hint stream is read LSB first, byte by byte.  With 4 bits, element i
 * takes bits 4i .. 4i+3, like the codes.  With 1 or 2 bits, each 16-element
 * block owns 16*bits consecutive bits, and inside the block element k takes
 * field 2*(k mod 8) + (k div 8): the fields of elements k and k + 8 sit next
 * to each other.  (A reader holding the block's codes as two words of 8
 * nibbles then finds the hint of nibble k of either word at bit 4k of one
 * 32-bit word, shifted by 0 or 2, or at bit 2k of a 16-bit word, shifted by 0
 * or 1.) */
static int64_t hint_pos(int64_t i, int bits)
{
    if (bits == 4) return i * 4;
    int64_t blk = i / 16;
    int k = (int)(i % 16);
    return blk * 16 * bits + (int64_t)bits * (2 * (k % 8) + k / 8);
}

void oracle_emit_hint(const uint8_t* codes, int64_t n, int bits, uint8_t* hints)
{
    int64_t nbytes = (n * bits + 7) / 8;
    memset(hints, 0, (size_t)nbytes);
    for (int64_t i = 0; i < n; ++i) {
        int code = nibble_get(codes, i);
        int h = (bits == 4) ? code : ((code & 7) & ((1 << bits) - 1));
        int64_t pos = hint_pos(i, bits);
        hints[pos >> 3] |= (uint8_t)(h << (pos & 7));
    }
}

static int hint_get(const uint8_t* hints, int64_t i, int bits)
{
    int64_t pos = hint_pos(i, bits);
    return (hints[pos >> 3] >> (pos & 7)) & ((1 << bits) - 1);
}

/* Rollout side: round-to-nearest codes of a BF16 tensor, plus its hints. */
void oracle_quantize_rtn_bf16(const uint16_t* x, int64_t rows, int64_t cols, float A,
                              uint8_t* codes, uint8_t* scales, float* tensor_scale,
                              uint8_t* hints, int hint_bits)
{
    float* y = bf16_rows_to_f32(x, rows * cols);
    oracle_quantize_f32(y, rows, cols, A, codes, scales, tensor_scale);
    free(y);
    if (hints) oracle_emit_hint(codes, rows * cols, hint_bits, hints);
}

/* Step 5: guided re-quantization on the train side ([TRACE], prescription
 * paragraph: near a boundary take the cell the rollout chose, not the nearest
 * one).  The train tensor derives its own scales (only cells are aligned).
 * For off-grid |v| < 6 the two candidate cells are the grid points that
 * bracket |v|: lo = the largest grid index with G[lo] <= |v|, hi = lo + 1.
 * hint_bits 1/2 compare magnitude indices modulo 2^bits; hint_bits 4 compares
 * signed grid positions.  No match -> round-to-nearest.  stats4 (may be NULL)
 * is added to: [consulted, changed, outside-bracket, reserved]. */
void oracle_guided_bf16(const uint16_t* x, int64_t rows, int64_t cols, float A,
                        const uint8_t* hints, int hint_bits,
                        uint8_t* codes, uint8_t* scales, float* tensor_scale,
                        uint64_t* stats4)
{
    float s_t = oracle_tensor_scale(A);
    *tensor_scale = s_t;
    int64_t nblk = cols / 16;
    uint64_t consulted = 0, changed = 0, outside = 0;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            float blk[16];
            for (int k = 0; k < 16; ++k) blk[k] = oracle_bf16_to_f32(x[r * cols + b * 16 + k]);
            float amax_b = 0.0f;
            for (int k = 0; k < 16; ++k)
                if (fabsf(blk[k]) > amax_b) amax_b = fabsf(blk[k]);
            int sb = oracle_block_scale(amax_b, s_t);
            scales[r * nblk + b] = (uint8_t)sb;
            float sbv = (float)oracle_e4m3_value(sb);
            for (int k = 0; k < 16; ++k) {
                int64_t i = r * cols + b * 16 + k;
                int sgn = sign_of(blk[k]);
                int m = 0;
                if (sbv != 0.0f && blk[k] != 0.0f) {
                    float a = fabsf(scaled_value(blk[k], sbv, s_t));
                    int m_rtn = oracle_e2m1_rne(a);
                    m = m_rtn;
                    if (hints != NULL && a < 6.0f) {
                        int lo = 0;
                        for (int g = 1; g < 8; ++g)
                            if (GRID[g] <= (double)a) lo = g;
                        if ((double)a != GRID[lo]) {
                            int hi = lo + 1;
                            int h = hint_get(hints, i, hint_bits);
                            int take_lo, take_hi;
                            consulted++;
                            if (hint_bits == 4) {
                                int pos_h = (h & 8) ? -(h & 7) : (h & 7);
                                int pos_lo = sgn ? -lo : lo;
                                int pos_hi = sgn ? -hi : hi;
                                take_lo = (pos_h == pos_lo);
                                take_hi = (pos_h == pos_hi);
                            } else {
                                int mask = (1 << hint_bits) - 1;
                                take_lo = ((h & mask) == (lo & mask));
                                take_hi = ((h & mask) == (hi & mask));
                            }
                            if (take_lo) m = lo;
                            else if (take_hi) m = hi;
                            else outside++;
                            if (m != m_rtn) changed++;
                        }
                    }
                }
                nibble_put(codes, i, (sgn << 3) | m);
            }
        }
    }
    if (stats4) {
        stats4[0] += consulted;
        stats4[1] += changed;
        stats4[2] += outside;
    }
}

/* KV-cache layout ([TRACE], hyper-parameter table: the rollout keeps the KV
 * cache in FP4 as well).  Reading: a cache entry is written one token at a
 * time, so no tensor-wide amax exists when it is quantized; each row of the
 * [tokens x heads, head_dim] cache (one token's vector for one head) is its
 * own tensor, with its own FP32 scale amax_row / 2688 and blocks of 16 along
 * head_dim.  So these are the tensor quantizers applied row by row; the hints
 * of row r start at byte r * cols * bits / 8 of the stream (blocks never
 * straddle rows).  row_scales: one float per row. */
void oracle_quantize_rtn_rows_bf16(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* codes,
                                   uint8_t* scales, float* row_scales, uint8_t* hints,
                                   int hint_bits)
{
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* xr = x + r * cols;
        float A = oracle_amax_bf16(xr, cols);
        oracle_quantize_rtn_bf16(xr, 1, cols, A, codes + r * cols / 2, scales + r * cols / 16,
                                 row_scales + r, hints ? hints + r * cols * hint_bits / 8 : NULL,
                                 hint_bits);
    }
}

void oracle_guided_rows_bf16(const uint16_t* x, int64_t rows, int64_t cols, const uint8_t* hints,
                             int hint_bits, uint8_t* codes, uint8_t* scales, float* row_scales,
                             uint64_t* stats4)
{
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* xr = x + r * cols;
        float A = oracle_amax_bf16(xr, cols);
        oracle_guided_bf16(xr, 1, cols, A, hints ? hints + r * cols * hint_bits / 8 : NULL, hint_bits,
                           codes + r * cols / 2, scales + r * cols / 16, row_scales + r, stats4);
    }
}

/* Decoded value of element i: sign * ((G[m] * sb) * s_t) in FP32; the first
 * product is exact (2 x 4 significant bits).  [RLQ], shared-convention
 * paragraph: a code means code value times scale (code 3 with scale 0.1 is
 * 0.3, with scale 0.2 it is 0.6). */
float oracle_dequant_one(int code, int scale_byte, float s_t)
{
    float sbv = (float)oracle_e4m3_value(scale_byte);
    float val = ((float)GRID[code & 7] * sbv) * s_t;
    return (code & 8) ? -val : val;
}

void oracle_dequant(const uint8_t* codes, const uint8_t* scales, float s_t, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_dequant_one(nibble_get(codes, i), scales[i / 16], s_t);
}

/* Step 6: mismatch counters between two NVFP4 tensors ([TRACE]: the
 * train/rollout distance is the quantity to shrink; most mismatches are one
 * cell apart).  Positions are signed grid indices (s ? -m : m); decoded values
 * are compared in FP32 (-0 equals +0).  stats8 is added to. */
void oracle_mismatch_stats(const uint8_t* codes_a, const uint8_t* scales_a, float ts_a,
                           const uint8_t* codes_b, const uint8_t* scales_b, float ts_b,
                           int64_t rows, int64_t cols, uint64_t* stats8)
{
    int64_t n = rows * cols;
    for (int64_t i = 0; i < n; ++i) {
        int ca = nibble_get(codes_a, i), cb = nibble_get(codes_b, i);
        int pa = (ca & 8) ? -(ca & 7) : (ca & 7);
        int pb = (cb & 8) ? -(cb & 7) : (cb & 7);
        int d = abs(pa - pb);
        stats8[0] += 1;
        if (d != 0) stats8[1] += 1;
        if (d == 1) stats8[2] += 1;
        if (d >= 2) stats8[3] += 1;
        stats8[4] += (uint64_t)d;
        float ya = oracle_dequant_one(ca, scales_a[i / 16], ts_a);
        float yb = oracle_dequant_one(cb, scales_b[i / 16], ts_b);
        if (ya != yb) stats8[6] += 1;
    }
    for (int64_t b = 0; b < n / 16; ++b)
        if (scales_a[b] != scales_b[b]) stats8[5] += 1;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10, from its published definition (Salmon, Moraes, Dror, Shaw,
 * "Parallel random numbers: as easy as 1, 2, 3", SC'11): ten rounds of two
 * 32x32->64 multiplications with multipliers 0xD2511F53 and 0xCD9E8D57, the
 * key bumped by the Weyl constants 0x9E3779B9 / 0xBB67AE85 between rounds. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Stochastic rounding of a magnitude a = |v| onto the grid with the random
 * word r ([TML4]: 2.25 becomes 2 three times in four and 3 once, so the mean
 * is kept).  p = (a - G[lo]) / (G[hi] - G[lo]); round up iff
 * (r >> 8) < p * 2^24.  On-grid values stay, a >= 6 gives 6. */
int oracle_sr_magnitude(float a, uint32_t r)
{
    if (a != a) return 0;
    if (a >= 6.0f) return 7;
    int lo = 0;
    for (int g = 1; g < 8; ++g)
        if (GRID[g] <= (double)a) lo = g;
    if ((double)a == GRID[lo]) return lo;
    int hi = lo + 1;
    double p = ((double)a - GRID[lo]) / (GRID[hi] - GRID[lo]);
    return ((double)(r >> 8) < p * 16777216.0) ? hi : lo;
}

void oracle_sr_transpose_requant_from(const uint8_t* codes, const uint8_t* scales,
                                      const float* tensor_scale, int64_t first, int64_t batch,
                                      int64_t rows, int64_t cols, uint64_t seed, uint32_t draw,
                                      uint8_t* codes_t, uint8_t* scales_t, float* tensor_scale_t);

/* Step 7: dequantize -> transpose -> stochastic re-quantize, per matrix of a
 * stack ([TML4], forward/backward mismatch paragraph).  Each matrix e is its
 * own tensor (own A', s_t').  The random word of output element i (row-major
 * in the [batch, cols, rows] output stack) is Philox4x32-10 with key
 * (seed lo32, seed hi32) and counter (i lo32, i hi32, draw, 0), word x0. */
void oracle_sr_transpose_requant(const uint8_t* codes, const uint8_t* scales,
                                 const float* tensor_scale, int64_t batch, int64_t rows,
                                 int64_t cols, uint64_t seed, uint32_t draw,
                                 uint8_t* codes_t, uint8_t* scales_t, float* tensor_scale_t)
{
    oracle_sr_transpose_requant_from(codes, scales, tensor_scale, 0, batch, rows, cols, seed, draw,
                                     codes_t, scales_t, tensor_scale_t);
}

/* The same for matrices first .. first+batch-1 of a larger stack whose data
 * starts at the given pointers (the counter keeps the whole stack's index). */
void oracle_sr_transpose_requant_from(const uint8_t* codes, const uint8_t* scales,
                                      const float* tensor_scale, int64_t first, int64_t batch,
                                      int64_t rows, int64_t cols, uint64_t seed, uint32_t draw,
                                      uint8_t* codes_t, uint8_t* scales_t, float* tensor_scale_t)
{
    int64_t n = rows * cols;
    float* y = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    float* yt = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (int64_t e = 0; e < batch; ++e) {
        const uint8_t* ce = codes + e * n / 2;
        const uint8_t* se = scales + e * n / 16;
        oracle_dequant(ce, se, tensor_scale[e], n, y);
        /* transpose [rows, cols] -> [cols, rows] */
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < cols; ++c) yt[c * rows + r] = y[r * cols + c];
        float A = oracle_amax_f32(yt, n);
        float s_t = oracle_tensor_scale(A);
        tensor_scale_t[e] = s_t;
        uint8_t* cte = codes_t + e * n / 2;
        uint8_t* ste = scales_t + e * n / 16;
        int64_t nblk = rows / 16;
        for (int64_t c = 0; c < cols; ++c) {
            for (int64_t b = 0; b < nblk; ++b) {
                const float* blk = yt + c * rows + b * 16;
                float amax_b = 0.0f;
                for (int k = 0; k < 16; ++k)
                    if (fabsf(blk[k]) > amax_b) amax_b = fabsf(blk[k]);
                int sb = oracle_block_scale(amax_b, s_t);
                ste[c * nblk + b] = (uint8_t)sb;
                float sbv = (float)oracle_e4m3_value(sb);
                for (int k = 0; k < 16; ++k) {
                    int64_t local = c * rows + b * 16 + k;
                    int64_t gi = (first + e) * n + local;
                    int m = 0;
                    if (sbv != 0.0f && blk[k] != 0.0f) {
                        uint32_t ctr[4] = {(uint32_t)gi, (uint32_t)((uint64_t)gi >> 32), draw, 0u};
                        uint32_t out[4];
                        oracle_philox4x32_10(ctr, key, out);
                        m = oracle_sr_magnitude(fabsf(scaled_value(blk[k], sbv, s_t)), out[0]);
                    }
                    nibble_put(cte, local, (sign_of(blk[k]) << 3) | m);
                }
            }
        }
    }
    free(y);
    free(yt);
}

/* ------------------------------------------------------------------------ */
/* Alternative to step 7, A: 16x16-tile scaling ([TML4], forward/backward
 * mismatch paragraph: NVIDIA's proposal enlarges the group sharing a scale to a
 * 16 x 16 tile of 256 values, which a transpose maps onto itself, at the price
 * of one large value flattening the rest of its tile).  Reading: the tile
 * scale follows the same recipe as the 16-value block scale (E4M3 of
 * (amax_tile / 6) / s_t with the FP32 tensor scale s_t = A / 2688), codes are
 * round-to-nearest as in step 3.  Layout: codes [rows, cols/2] as for blocks,
 * tile scales [rows/16, cols/16] row-major; rows % 16 == cols % 16 == 0. */
void oracle_quantize_tile16_bf16(const uint16_t* x, int64_t rows, int64_t cols, float A,
                                 uint8_t* codes, uint8_t* tscales, float* tensor_scale)
{
    float s_t = oracle_tensor_scale(A);
    *tensor_scale = s_t;
    int64_t tr = rows / 16, tc = cols / 16;
    for (int64_t ti = 0; ti < tr; ++ti) {
        for (int64_t tj = 0; tj < tc; ++tj) {
            float amax_t = 0.0f;
            for (int64_t r = 16 * ti; r < 16 * ti + 16; ++r)
                for (int64_t c = 16 * tj; c < 16 * tj + 16; ++c) {
                    float a = fabsf(oracle_bf16_to_f32(x[r * cols + c]));
                    if (a > amax_t) amax_t = a;
                }
            int sb = oracle_block_scale(amax_t, s_t);
            tscales[ti * tc + tj] = (uint8_t)sb;
            float sbv = (float)oracle_e4m3_value(sb);
            for (int64_t r = 16 * ti; r < 16 * ti + 16; ++r)
                for (int64_t c = 16 * tj; c < 16 * tj + 16; ++c) {
                    float xv = oracle_bf16_to_f32(x[r * cols + c]);
                    int m = 0;
                    if (sbv != 0.0f && xv != 0.0f) m = oracle_e2m1_rne(fabsf(scaled_value(xv, sbv, s_t)));
                    nibble_put(codes, r * cols + c, (sign_of(xv) << 3) | m);
                }
        }
    }
}

/* Transpose of tile-scaled matrices: code (r, c) moves to (c, r) and tile
 * scale (ti, tj) to (tj, ti); the tensor scale is unchanged.  Nothing is
 * re-rounded: the result is the tile quantization of the transposed input. */
void oracle_transpose_tile16(const uint8_t* codes, const uint8_t* tscales, int64_t batch,
                             int64_t rows, int64_t cols, uint8_t* codes_t, uint8_t* tscales_t)
{
    int64_t n = rows * cols, tr = rows / 16, tc = cols / 16;
    for (int64_t e = 0; e < batch; ++e) {
        const uint8_t* ce = codes + e * n / 2;
        uint8_t* cte = codes_t + e * n / 2;
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < cols; ++c) nibble_put(cte, c * rows + r, nibble_get(ce, r * cols + c));
        for (int64_t ti = 0; ti < tr; ++ti)
            for (int64_t tj = 0; tj < tc; ++tj)
                tscales_t[e * tr * tc + tj * tr + ti] = tscales[e * tr * tc + ti * tc + tj];
    }
}

/* Decoded values of a tile-scaled matrix (same per-element rule as blocks). */
void oracle_dequant_tile16(const uint8_t* codes, const uint8_t* tscales, float s_t, int64_t rows,
                           int64_t cols, float* out)
{
    int64_t tc = cols / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            out[r * cols + c] = oracle_dequant_one(nibble_get(codes, r * cols + c),
                                                   tscales[(r / 16) * tc + c / 16], s_t);
}

/* ------------------------------------------------------------------------ */
/* Alternative to step 7, B: the backward in MXFP8 with stochastic rounding
 * ([TML4]: the backward runs in MXFP8 with stochastic rounding after the
 * dequantize -> transpose step; MXFP8 costs 8.25 bits per value, i.e. 8-bit
 * elements and one 8-bit scale per 32 values).  Readings (OCP MX): elements
 * E4M3 "fn", one E8M0 scale 2^e per 32 consecutive values along the new rows,
 * e = floor(log2(amax_32)) - 8 (8 = exponent of the largest E4M3 binade),
 * clamped to [-127, 127], e = -127 for an all-zero block; byte = e + 127.
 * Element: v = y * 2^-e, stochastic rounding of |v| onto the E4M3 values with
 * the same rule and random word as step 7 (the same Philox counter: the
 * element's row-major index in the [batch, cols, rows] output stack),
 * saturating at 448; sign from y. */
int oracle_e8m0_exponent(float amax)
{
    if (!(amax > 0.0f)) return -127;
    int ex;
    frexp((double)amax, &ex);   /* amax = f * 2^ex, f in [0.5, 1) */
    int e = (ex - 1) - 8;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* Stochastic rounding of a >= 0 onto the non-negative E4M3 values (a byte
 * 0x00..0x7E): lo = the largest value <= a (exhaustive search), hi the next
 * one; p = (a - lo) / (hi - lo); round up iff (r >> 8) < p * 2^24.  Values on
 * the grid stay, a >= 448 gives 448. */
int oracle_e4m3_sr(float a, uint32_t r)
{
    if (a != a) return 0x7F;
    if (a >= 448.0f) return 0x7E;
    int lo = 0;
    for (int b = 1; b <= 0x7E; ++b)
        if (oracle_e4m3_value(b) <= (double)a) lo = b;
    double vlo = oracle_e4m3_value(lo);
    if ((double)a == vlo) return lo;
    double vhi = oracle_e4m3_value(lo + 1);
    double p = ((double)a - vlo) / (vhi - vlo);
    return ((double)(r >> 8) < p * 16777216.0) ? lo + 1 : lo;
}

/* codes/scales/tensor_scale: a stack of NVFP4 matrices [batch, rows, cols]
 * (16-value blocks along cols).  Output: E4M3 bytes [batch, cols, rows] and
 * E8M0 bytes [batch, cols, rows / 32]. */
void oracle_mxfp8_sr_transpose_requant_from(const uint8_t* codes, const uint8_t* scales,
                                            const float* tensor_scale, int64_t first,
                                            int64_t batch, int64_t rows, int64_t cols,
                                            uint64_t seed, uint32_t draw, uint8_t* q_t,
                                            uint8_t* e8_t);

void oracle_mxfp8_sr_transpose_requant(const uint8_t* codes, const uint8_t* scales,
                                       const float* tensor_scale, int64_t batch, int64_t rows,
                                       int64_t cols, uint64_t seed, uint32_t draw, uint8_t* q_t,
                                       uint8_t* e8_t)
{
    oracle_mxfp8_sr_transpose_requant_from(codes, scales, tensor_scale, 0, batch, rows, cols, seed,
                                           draw, q_t, e8_t);
}

/* The same for matrices first .. first+batch-1 of a larger stack whose data
 * starts at the given pointers (the counter keeps the whole stack's index). */
void oracle_mxfp8_sr_transpose_requant_from(const uint8_t* codes, const uint8_t* scales,
                                            const float* tensor_scale, int64_t first,
                                            int64_t batch, int64_t rows, int64_t cols,
                                            uint64_t seed, uint32_t draw, uint8_t* q_t,
                                            uint8_t* e8_t)
{
    int64_t n = rows * cols;
    float* y = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    float* yt = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    int64_t nb = rows / 32;
    for (int64_t e = 0; e < batch; ++e) {
        oracle_dequant(codes + e * n / 2, scales + e * n / 16, tensor_scale[e], n, y);
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < cols; ++c) yt[c * rows + r] = y[r * cols + c];
        for (int64_t c = 0; c < cols; ++c) {
            for (int64_t b = 0; b < nb; ++b) {
                const float* blk = yt + c * rows + b * 32;
                float amax_b = oracle_amax_f32(blk, 32);
                int ex = oracle_e8m0_exponent(amax_b);
                e8_t[e * cols * nb + c * nb + b] = (uint8_t)(ex + 127);
                float down = ldexpf(1.0f, -ex);  /* exact: 2^-127 .. 2^127 are floats */
                for (int k = 0; k < 32; ++k) {
                    int64_t local = c * rows + b * 32 + k;
                    int64_t gi = (first + e) * n + local;
                    uint32_t ctr[4] = {(uint32_t)gi, (uint32_t)((uint64_t)gi >> 32), draw, 0u};
                    uint32_t out[4];
                    oracle_philox4x32_10(ctr, key, out);
                    float v = blk[k] * down;
                    q_t[e * n + local] =
                        (uint8_t)((sign_of(blk[k]) << 7) | oracle_e4m3_sr(fabsf(v), out[0]));
                }
            }
        }
    }
    free(y);
    free(yt);
}

/* Decoded MXFP8 values, blocks of 32 consecutive elements: E4M3 value times
 * 2^(byte - 127), one FP32 multiply (exact unless it overflows). */
void oracle_mxfp8_dequant(const uint8_t* q, const uint8_t* e8, int64_t n, float* out)
{
    for (int64_t i = 0; i < n; ++i) {
        float v = (float)oracle_e4m3_value(q[i]);
        out[i] = v * ldexpf(1.0f, (int)e8[i / 32] - 127);
    }
}

/* ------------------------------------------------------------------------ */
/* Step 8: 32-point random Hadamard transform ([TML4], communication
 * paragraph).  Signs: sigma_j = -1 iff bit 0 of Philox4x32-10(key = (seed lo32,
 * seed hi32), counter = (j, 0, 0, 0)).x0 is set.  The transform is the plain
 * matrix product with the Sylvester matrix H[j][k] = (-1)^popcount(j & k),
 * in double precision, scaled by 1/sqrt(32). */
void oracle_rht_signs(uint64_t seed, int* sigma32)
{
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (uint32_t j = 0; j < 32; ++j) {
        uint32_t ctr[4] = {j, 0u, 0u, 0u}, out[4];
        oracle_philox4x32_10(ctr, key, out);
        sigma32[j] = (out[0] & 1u) ? -1 : 1;
    }
}

static int popcount_u32(uint32_t v)
{
    int c = 0;
    while (v) {
        c += (int)(v & 1u);
        v >>= 1;
    }
    return c;
}

void oracle_rht32_f64(const uint16_t* x, int64_t rows, int64_t cols, uint64_t seed, double* y)
{
    int sigma[32];
    oracle_rht_signs(seed, sigma);
    double norm = 1.0 / sqrt(32.0);
    int64_t n = rows * cols;
    for (int64_t g = 0; g < n; g += 32) {
        for (int j = 0; j < 32; ++j) {
            double s = 0.0;
            for (int k = 0; k < 32; ++k) {
                double h = (popcount_u32((uint32_t)(j & k)) % 2) ? -1.0 : 1.0;
                s += h * (double)sigma[k] * (double)oracle_bf16_to_f32(x[g + k]);
            }
            y[g + j] = s * norm;
        }
    }
}

/* RHT then round-to-nearest quantization of the FP32-rounded transform. */
void oracle_rht_quantize(const uint16_t* x, int64_t rows, int64_t cols, uint64_t seed,
                         uint8_t* codes, uint8_t* scales, float* tensor_scale, float* y_f32)
{
    int64_t n = rows * cols;
    double* yd = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    oracle_rht32_f64(x, rows, cols, seed, yd);
    for (int64_t i = 0; i < n; ++i) y_f32[i] = (float)yd[i];
    free(yd);
    float A = oracle_amax_f32(y_f32, n);
    oracle_quantize_f32(y_f32, rows, cols, A, codes, scales, tensor_scale);
}

/* ------------------------------------------------------------------------ */
/* Rollout producer ([TML4], configuration paragraph and format table: the MoE
 * forward GEMMs of pre-training and of rollout sampling run in NVFP4).
 *
 * D[i][j] = sum_k dec(A)[i][k] * dec(B)[j][k] for A [m, k] and B [n, k], both
 * NVFP4 with 16-element blocks along k, dec = code value * E4M3(scale) * s_t.
 * The sum is taken without s_t (each term G_a * sa * G_b * sb is a multiple
 * of 2^-20 below 2^23 and has at most 12 significant bits) in long double,
 * whose 64-bit mantissa holds every partial sum exactly for k <= 2^16; the
 * exact sum is then multiplied once by s_a * s_b and rounded to double.
 * dabs receives the same with |term|, the scale of any accumulation error. */
void oracle_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, float a_ts,
                       const uint8_t* b_codes, const uint8_t* b_scales, float b_ts,
                       int64_t m, int64_t n, int64_t k, double* d, double* dabs)
{
    int64_t kb = k / 16;
    long double st = (long double)a_ts * (long double)b_ts;
    for (int64_t i = 0; i < m; ++i) {
        for (int64_t j = 0; j < n; ++j) {
            long double s = 0.0L, sa = 0.0L;
            for (int64_t e = 0; e < k; ++e) {
                int ca = nibble_get(a_codes, i * k + e), cb = nibble_get(b_codes, j * k + e);
                long double va = (long double)GRID[ca & 7] *
                                 (long double)oracle_e4m3_value(a_scales[i * kb + e / 16]);
                long double vb = (long double)GRID[cb & 7] *
                                 (long double)oracle_e4m3_value(b_scales[j * kb + e / 16]);
                long double t = va * vb;
                sa += t;
                s += ((ca >> 3) ^ (cb >> 3)) ? -t : t;
            }
            d[i * n + j] = (double)(s * st);
            dabs[i * n + j] = (double)(sa * fabsl(st));
        }
    }
}

/* Scale-factor layout read by the block-scaled tensor-core MMA of sm_100
 * (NVIDIA PTX ISA, tcgen05 block scaling; cuBLAS documentation, 1D block
 * scaling factors layout).  The [rows, sf_cols] scale matrix (sf_cols =
 * cols / 16) is cut into tiles of 128 rows x 4 scale columns, 512 bytes each,
 * tile (rt, kt) at byte (rt * ceil(sf_cols / 4) + kt) * 512; inside a tile the
 * scale of row r, column c sits at (r % 32) * 16 + (r / 32) * 4 + c.  Rows
 * padded to 128 and columns to 4 hold zero. */
void oracle_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t sf_cols, uint8_t* out)
{
    int64_t row_tiles = (rows + 127) / 128, col_tiles = (sf_cols + 3) / 4;
    memset(out, 0, (size_t)(row_tiles * col_tiles * 512));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < sf_cols; ++c) {
            int64_t tile = (r / 128) * col_tiles + c / 4;
            int64_t rr = r % 128;
            out[tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + c % 4] = scales[r * sf_cols + c];
        }
    }
}
