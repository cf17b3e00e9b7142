/*
 * nvfp4pt oracle -- plain, slow, single-threaded CPU reference of the NVFP4
 * per-token quantization cast and its running-absmax bookkeeping.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this code. The product path (the CUDA
 * library) never calls it, and the two share no source: no header, no table,
 * no helper.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC.
 * Every floating-point step below is ONE IEEE-754 binary32 operation, rounded
 * to nearest-even (x86-64 SSE arithmetic; no FMA contraction, no flush-to-zero).
 *
 * What it follows:
 *  - TransformerEngine PR #3045 "Add NVFP4 per-token quantization recipe",
 *    Description: one outer amax per row (length M) for the rowwise data and one
 *    per column (length K) for the columnwise data, in place of the single
 *    per-tensor amax of the default NVFP4 recipe.
 *  - The same page, Changes: a vector-amax stage, then an encode stage that makes
 *    E2M1 codes with E4M3 scales per 16-element block; the opt-in 2D weight
 *    cast uses 16x16 blocks emitted in the per-token layout.
 *  - Model-Optimizer PR #2598 (GPTQ fused update), review thread on the FP8 block
 *    scale: the weight quantizer's block scale is (amax/6) * 448 / (gA/6), and
 *    algebraically equal orderings round to different E4M3 codes, so the fp32
 *    operation order is part of the definition. Here 448/(gA/6) = 2688/gA is the
 *    per-row "s_enc" and the block scale is RN(RN(block_amax/6) * s_enc).
 *  - TransformerEngine PR #3296 "[PTQ] Store FP32 global scaling factors",
 *    Description: New AbsMax = Max(Old AbsMax * Decay, Observed AbsMax); with
 *    per-token scaling the observed value is the row amaxes max-reduced to a scalar.
 *  - TransformerEngine PR #3244 (row-wise pre-quantized grouped GEMM input),
 *    review: "compact" scales means the unswizzled row-major layout.
 *  - TransformerEngine PR #3045, Changes and Greptile summary: the per-token GEMM
 *    over NVFP4 operands, rescaled by the per-row and per-column outer-amax
 *    vectors in its epilogue (oracle_gemm_per_token, with its reading).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - s_enc = 1 when amax == 0; an overflowing 2688/amax (amax below ~7.9e-36)
 *    is clamped to FLT_MAX, and so is an overflowing s_enc/float(sf), so that
 *    0 * enc never makes a NaN.
 *  - E4M3 is e4m3fn (max 448, no infinity), saturating; E2M1 saturates at 6.
 *  - Rounding a negative value to zero keeps its sign: E2M1 code 0x8.
 *  - Two codes per byte, element 2j in the low nibble.
 *  - Columnwise = the rowwise cast of X^T using the column amax; stored [K, M/2].
 *  - NaN and infinity in X are outside the contract.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#define OR_ROWWISE 1
#define OR_COLWISE 2

/* ------------------------------------------------------------------ values */

/* The eight non-negative E2M1 magnitudes, indexed by the 3-bit code. */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Value of a non-negative e4m3fn code 0..126 (4 exponent bits, bias 7,
 * 3 mantissa bits; exponent field 0 is subnormal: m * 2^-9). */
static double e4m3_magnitude(int code)
{
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    if (e == 0) return (double)m * ldexp(1.0, -9);
    return (1.0 + (double)m / 8.0) * ldexp(1.0, e - 7);
}

float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16; /* bf16 is the top half of a binary32 */
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round-to-nearest-even, saturating, to e4m3fn. Scans all 127 finite
 * non-negative values; on an exact tie the code with an even last bit wins.
 * Comparisons are in double, where every value and midpoint is exact. */
uint8_t oracle_e4m3(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a > 448.0) return sign | 0x7E; /* satfinite: clamp to 448 */
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(e4m3_magnitude(c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return sign | (uint8_t)best;
}

float oracle_e4m3_decode(uint8_t code)
{
    double v = e4m3_magnitude(code & 0x7F);
    return (float)((code & 0x80) ? -v : v);
}

/* Round-to-nearest-even, saturating, to E2M1. Returns a 4-bit code:
 * bit 3 = sign (set iff signbit(y), so -0.0 and small negatives give 0x8),
 * bits 0-2 index kE2M1. */
uint8_t oracle_e2m1(float y)
{
    uint8_t sign = signbit(y) ? 0x8 : 0x0;
    double a = fabs((double)y);
    if (a > 6.0) return sign | 0x7;
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double d = fabs(kE2M1[c] - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return sign | (uint8_t)best;
}

float oracle_e2m1_decode(uint8_t code)
{
    double v = kE2M1[code & 0x7];
    return (float)((code & 0x8) ? -v : v);
}

/* ------------------------------------------------------------ block steps */

/* Outer encode scale of one row (or column): s_enc = 2688 / amax. */
float oracle_s_enc(float amax)
{
    if (amax == 0.0f) return 1.0f;
    float s = 2688.0f / amax;
    if (s > FLT_MAX) s = FLT_MAX; /* reading: clamp the overflow */
    return s;
}

/* The scale argument of one 16-element block: RN(RN(block_amax / 6) * s_enc). */
float oracle_block_scale_arg(float block_amax, float s_enc)
{
    float t = block_amax / 6.0f;
    float u = t * s_enc;
    return u;
}

/* Per-element multiplier of a block with scale code sf. */
float oracle_block_enc(uint8_t sf, float s_enc)
{
    if (sf == 0) return 0.0f;
    float e = s_enc / oracle_e4m3_decode(sf);
    if (e > FLT_MAX) e = FLT_MAX; /* reading: clamp the overflow */
    return e;
}

/* Encode 16 values v[0..15] with multiplier enc into 8 bytes (low nibble first). */
static void encode16(const float* v, float enc, uint8_t* out8)
{
    for (int j = 0; j < 8; ++j) {
        float y0 = v[2 * j] * enc;
        float y1 = v[2 * j + 1] * enc;
        out8[j] = (uint8_t)(oracle_e2m1(y0) | (oracle_e2m1(y1) << 4));
    }
}

/* One 1D block: 16 values with the row's (or column's) s_enc. */
static void quantize_block_1d(const float* v, float s_enc, uint8_t* codes8, uint8_t* sf_out)
{
    float ba = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(v[i]);
        if (a > ba) ba = a;
    }
    uint8_t sf = oracle_e4m3(oracle_block_scale_arg(ba, s_enc));
    encode16(v, oracle_block_enc(sf, s_enc), codes8);
    *sf_out = sf;
}

/* ------------------------------------------------------------ amax vectors */

static float absf_at(const uint16_t* x, int64_t K, int64_t r, int64_t c)
{
    return fabsf(oracle_bf16_to_f32(x[r * K + c]));
}

/* amax_row[m] = max_k |x[m,k]| */
void oracle_amax_rows(const uint16_t* x, int64_t M, int64_t K, float* amax_row)
{
    for (int64_t r = 0; r < M; ++r) {
        float m = 0.0f;
        for (int64_t c = 0; c < K; ++c) {
            float a = absf_at(x, K, r, c);
            if (a > m) m = a;
        }
        amax_row[r] = m;
    }
}

/* amax over rows [r0, r1) of each column: out[k] = max_{r0<=m<r1} |x[m,k]| */
void oracle_amax_cols(const uint16_t* x, int64_t K, int64_t r0, int64_t r1, float* out)
{
    for (int64_t c = 0; c < K; ++c) out[c] = 0.0f;
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t c = 0; c < K; ++c) {
            float a = absf_at(x, K, r, c);
            if (a > out[c]) out[c] = a;
        }
}

/* -------------------------------------------------------------- the casts */

/* Rowwise cast of rows [r0, r1): codes [.., K/2], scales [.., K/16]. */
static void cast_rows(const uint16_t* x, int64_t K, int64_t r0, int64_t r1, const float* amax_row,
                      uint8_t* q_row, uint8_t* sf_row)
{
    float v[16];
    for (int64_t r = r0; r < r1; ++r) {
        float s_enc = oracle_s_enc(amax_row[r]);
        for (int64_t b = 0; b < K / 16; ++b) {
            for (int i = 0; i < 16; ++i) v[i] = oracle_bf16_to_f32(x[r * K + 16 * b + i]);
            quantize_block_1d(v, s_enc, q_row + r * (K / 2) + 8 * b, sf_row + r * (K / 16) + b);
        }
    }
}

/* Columnwise cast of the row range [r0, r0+m) (one token group): the rowwise cast
 * of its transpose. Codes [K, m/2], scales [K, m/16], both starting at the given
 * pointers; amax_col has K entries for this range. */
static void cast_cols(const uint16_t* x, int64_t K, int64_t r0, int64_t m, const float* amax_col,
                      uint8_t* q_col, uint8_t* sf_col)
{
    float v[16];
    for (int64_t c = 0; c < K; ++c) {
        float s_enc = oracle_s_enc(amax_col[c]);
        for (int64_t b = 0; b < m / 16; ++b) {
            for (int i = 0; i < 16; ++i) v[i] = oracle_bf16_to_f32(x[(r0 + 16 * b + i) * K + c]);
            quantize_block_1d(v, s_enc, q_col + c * (m / 2) + 8 * b, sf_col + c * (m / 16) + b);
        }
    }
}

/* New AbsMax = Max(Old AbsMax * Decay, Observed AbsMax). */
static float absmax_step(float old, float decay, float observed)
{
    float d = old * decay;
    return (d > observed) ? d : observed;
}

void oracle_update_absmax(float* buf, const float* amax_vec, int64_t n, float decay)
{
    float obs = 0.0f;
    for (int64_t i = 0; i < n; ++i)
        if (amax_vec[i] > obs) obs = amax_vec[i];
    *buf = absmax_step(*buf, decay, obs);
}

static int shape_ok(int64_t M, int64_t K)
{
    return M > 0 && K > 0 && M % 16 == 0 && K % 16 == 0;
}

/* Ungrouped per-token cast. Returns 0 on success, -1 on a bad shape.
 * flags: 1 = rowwise, 2 = columnwise. amax_row is always written (it is the
 * observed value of the absmax update); absmax_buf may be NULL. */
int oracle_quantize(const uint16_t* x, int64_t M, int64_t K, int flags,
                    uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                    uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                    float* absmax_buf, float decay)
{
    if (!shape_ok(M, K)) return -1;
    oracle_amax_rows(x, M, K, amax_row);
    if (flags & OR_ROWWISE) cast_rows(x, K, 0, M, amax_row, q_row, sf_row);
    if (flags & OR_COLWISE) {
        oracle_amax_cols(x, K, 0, M, amax_col);
        cast_cols(x, K, 0, M, amax_col, q_col, sf_col);
    }
    if (absmax_buf) oracle_update_absmax(absmax_buf, amax_row, M, decay);
    return 0;
}

/* Grouped (MoE) cast: token groups are the row ranges [offsets[g], offsets[g+1]).
 * Rowwise outputs and amax_row are those of the ungrouped cast. The columnwise
 * direction is cast per group with amax_col[g*K + k] over the group's rows;
 * group g's codes are [K, m_g/2] at byte K*offsets[g]/2 of q_col and its scales
 * [K, m_g/16] at byte K*offsets[g]/16 of sf_col. absmax_bufs (NULL or [G]) gets
 * the update with the group's observed max (0 for an empty group).
 * Returns 0, or -1 on bad shape/offsets. */
int oracle_quantize_grouped(const uint16_t* x, int64_t M, int64_t K, const int64_t* offsets, int G,
                            int flags, uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                            uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                            float* absmax_bufs, float decay)
{
    if (!shape_ok(M, K) || G < 1) return -1;
    if (offsets[0] != 0 || offsets[G] != M) return -1;
    for (int g = 0; g < G; ++g)
        if (offsets[g + 1] < offsets[g] || offsets[g] % 16 != 0) return -1;
    oracle_amax_rows(x, M, K, amax_row);
    if (flags & OR_ROWWISE) cast_rows(x, K, 0, M, amax_row, q_row, sf_row);
    for (int g = 0; g < G; ++g) {
        int64_t r0 = offsets[g], m = offsets[g + 1] - offsets[g];
        if (flags & OR_COLWISE) {
            float* ac = amax_col + (int64_t)g * K;
            oracle_amax_cols(x, K, r0, r0 + m, ac);
            cast_cols(x, K, r0, m, ac, q_col + K * r0 / 2, sf_col + K * r0 / 16);
        }
        if (absmax_bufs) {
            float obs = 0.0f;
            for (int64_t r = r0; r < r0 + m; ++r)
                if (amax_row[r] > obs) obs = amax_row[r];
            absmax_bufs[g] = absmax_step(absmax_bufs[g], decay, obs);
        }
    }
    return 0;
}

/* 2D weight cast (16x16 blocks emitted in the per-token layout). Each row keeps
 * its own s_enc from amax_row; the 16 rows of a band share one E4M3 scale per
 * 16-column block: sf = e4m3(max over the band's rows of the 1D scale argument);
 * each row encodes with its own enc = s_enc[r] / float(sf). The shared scale is
 * written to all 16 rows of the band in sf_row [N, K/16]. Returns 0 or -1. */
int oracle_quantize_weight_2d(const uint16_t* w, int64_t N, int64_t K,
                              uint8_t* q_row, uint8_t* sf_row, float* amax_row)
{
    if (!shape_ok(N, K)) return -1;
    oracle_amax_rows(w, N, K, amax_row);
    float v[16];
    for (int64_t band = 0; band < N / 16; ++band) {
        for (int64_t b = 0; b < K / 16; ++b) {
            float umax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                int64_t r = 16 * band + i;
                float s_enc = oracle_s_enc(amax_row[r]);
                float ba = 0.0f;
                for (int j = 0; j < 16; ++j) {
                    float a = absf_at(w, K, r, 16 * b + j);
                    if (a > ba) ba = a;
                }
                float u = oracle_block_scale_arg(ba, s_enc);
                if (u > umax) umax = u;
            }
            uint8_t sf = oracle_e4m3(umax);
            for (int i = 0; i < 16; ++i) {
                int64_t r = 16 * band + i;
                float s_enc = oracle_s_enc(amax_row[r]);
                for (int j = 0; j < 16; ++j) v[j] = oracle_bf16_to_f32(w[r * K + 16 * b + j]);
                encode16(v, oracle_block_enc(sf, s_enc), q_row + r * (K / 2) + 8 * b);
                sf_row[r * (K / 16) + b] = sf;
            }
        }
    }
    return 0;
}

/* --------------------------------------------------------- dequantization */

/* Nearest bf16 to a finite binary32 f, ties to the even significand: the two bf16
 * neighbours of |f| (its truncation and the next magnitude up) are compared in
 * double, where both distances are exact. */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    const uint16_t lo = (uint16_t)(u >> 16);   /* truncation toward zero, same sign */
    if ((u & 0xFFFFu) == 0) return lo;         /* exactly representable */
    const uint16_t hi = (uint16_t)(lo + 1);    /* next magnitude away from zero */
    const double a = fabs((double)f);
    const double dl = a - fabs((double)oracle_bf16_to_f32(lo));
    /* Above the largest finite bf16 the next magnitude is infinity; IEEE 754's rounding
     * to nearest treats it as 2^128 (the next step were the exponent range unbounded),
     * so from halfway to 2^128 upwards the result is infinity. */
    const double up = ((hi & 0x7FFFu) == 0x7F80u) ? ldexp(1.0, 128) : fabs((double)oracle_bf16_to_f32(hi));
    const double dh = up - a;
    if (dl < dh) return lo;
    if (dh < dl) return hi;
    return (lo & 1) ? hi : lo;
}

/* Dequantization of rowwise-layout NVFP4 data, the inverse of the cast (the pages
 * store fp32 "scale_inv" factors beside the block scales, TransformerEngine PR #3296;
 * PR #3244's flow dequantizes rowwise data before requantizing it columnwise). The
 * reading taken: with the decode scale S_dec = RN(amax / 2688) of the row,
 *     x'[r][16b + j] = bf16_rn( RN( (val(q) * float(sf[r][b])) * S_dec ) ),
 * where val(q) * float(sf) is exact in binary32 (at most 2 + 4 significant bits).
 * q: [M, K/2] (element 2j in the low nibble), sf: [M, K/16], amax: [M]; out: bf16
 * [M, K]. The columnwise data [K, M/2], [K, M/16], [K] give X^T the same way. */
int oracle_dequantize_rows(const uint8_t* q, const uint8_t* sf, const float* amax, int64_t M, int64_t K,
                           uint16_t* out)
{
    if (!shape_ok(M, K)) return -1;
    for (int64_t r = 0; r < M; ++r) {
        const float sdec = amax[r] / 2688.0f;
        for (int64_t b = 0; b < K / 16; ++b) {
            const float s = oracle_e4m3_decode(sf[r * (K / 16) + b]);
            for (int j = 0; j < 16; ++j) {
                const uint8_t byte = q[r * (K / 2) + 8 * b + j / 2];
                const uint8_t code = (j & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
                const float t = oracle_e2m1_decode(code) * s; /* exact */
                const float y = t * sdec;
                out[r * K + 16 * b + j] = oracle_f32_to_bf16(y);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------- per-token GEMM */

/* 2 * val(code) for an E2M1 code (integer: -12..12; -0 gives 0). */
static int64_t e2m1_twice(uint8_t code)
{
    static const int64_t kTwice[8] = {0, 1, 2, 3, 4, 6, 8, 12};
    const int64_t v = kTwice[code & 7];
    return (code & 8) ? -v : v;
}

/* 2^9 * float(sf) for a non-negative finite e4m3fn code 0..126 (an integer:
 * subnormals are m * 2^-9, normals (8 + m) * 2^(e - 10) with e >= 1); -1 for any
 * other code. */
static int64_t e4m3_times_512(uint8_t code)
{
    if (code > 0x7E) return -1;
    return (int64_t)ldexp(e4m3_magnitude(code), 9);
}

/* The per-token NVFP4 GEMM (TransformerEngine PR #3045, Changes and the Greptile
 * summary: a GEMM over the per-token NVFP4 operands that applies the per-row and
 * per-column outer-amax vectors in its epilogue; the call takes each operand's
 * codes, block scales and amax vector and returns an M x N output). The reading
 * taken: both operands are K-major rowwise-layout NVFP4 data,
 *     A: codes [M, K/2], scales [M, K/16], amax [M];  B: [N, K/2], [N, K/16], [N],
 * and, with S_dec(a) = RN(a / 2688) the binary32 decode scale of the dequantization,
 *     D[m][n] = S_dec(amax_a[m]) * S_dec(amax_b[n])
 *               * sum_k val(qa[m][k]) sf_a[m][k/16] val(qb[n][k]) sf_b[n][k/16].
 * Every term is a whole multiple of 2^-20 (val is a multiple of 1/2, sf of 2^-9),
 * so the sum is taken exactly in integers in units of 2^-20 and rounded once to
 * double; the product of the two decode scales (exact in double) then multiplies
 * it with one more rounding, the same for D(A, B) and D(B, A)^T. abs_out (optional) gets
 * the same expression over the terms' magnitudes: the scale of the rounding error
 * of any binary32 evaluation. Returns -1 for a bad shape, -2 for a scale code that
 * is not a non-negative finite e4m3fn value. */
int oracle_gemm_per_token(const uint8_t* qa, const uint8_t* sfa, const float* amax_a, int64_t M,
                          const uint8_t* qb, const uint8_t* sfb, const float* amax_b, int64_t N,
                          int64_t K, double* out, double* abs_out)
{
    if (M < 1 || N < 1 || K < 16 || K % 16) return -1;
    for (int64_t i = 0; i < M * (K / 16); ++i)
        if (e4m3_times_512(sfa[i]) < 0) return -2;
    for (int64_t i = 0; i < N * (K / 16); ++i)
        if (e4m3_times_512(sfb[i]) < 0) return -2;
    for (int64_t m = 0; m < M; ++m) {
        const double sa = (double)(amax_a[m] / 2688.0f);
        for (int64_t n = 0; n < N; ++n) {
            const double scale = sa * (double)(amax_b[n] / 2688.0f);   /* exact: 24 + 24 bits */
            __int128 acc = 0, acc_abs = 0;
            for (int64_t k = 0; k < K; ++k) {
                const uint8_t ba = qa[m * (K / 2) + k / 2], bb = qb[n * (K / 2) + k / 2];
                const uint8_t ca = (k & 1) ? (uint8_t)(ba >> 4) : (uint8_t)(ba & 0xF);
                const uint8_t cb = (k & 1) ? (uint8_t)(bb >> 4) : (uint8_t)(bb & 0xF);
                const int64_t t = e2m1_twice(ca) * e2m1_twice(cb) * e4m3_times_512(sfa[m * (K / 16) + k / 16]) *
                                  e4m3_times_512(sfb[n * (K / 16) + k / 16]);   /* |t| < 2^43 */
                acc += t;
                acc_abs += t < 0 ? -t : t;
            }
            out[m * N + n] = ldexp((double)acc, -20) * scale;
            if (abs_out) abs_out[m * N + n] = ldexp((double)acc_abs, -20) * fabs(scale);
        }
    }
    return 0;
}

/* ------------------------------------------------ array forms (for sweeps) */

void oracle_e4m3_array(const float* v, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3(v[i]);
}

void oracle_e2m1_array(const float* y, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1(y[i]);
}

void oracle_f32_to_bf16_array(const float* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(v[i]);
}

/* ------------------------------------- columnwise options: RHT and SR */

/* TransformerEngine PR #3045, Changes: an opt-in random Hadamard transform (RHT) and
 * opt-in stochastic rounding (SR) on the per-token path, off by default; its review:
 * the row direction never uses RHT. The pages fix neither the transform size, the
 * signs, the evaluation order nor the random numbers. The readings taken (each listed
 * in the design notes):
 *  - RHT acts on each columnwise 16-element block (16 consecutive rows of one column
 *    inside a token group): v' = (1/4) H16 S v, H16 the Sylvester Hadamard matrix
 *    (H[i][j] = (-1)^popcount(i & j)), S = diag(s_j), s_j = -1 where bit j of a
 *    caller-given 16-bit mask is set. Orthogonal: (1/4 H16)^2 = I. Evaluated as the
 *    radix-2 butterfly in four stages (pairs i, i+h for h = 1, 2, 4, 8: sum and
 *    difference, each one binary32 rounding), then the exact multiply by 1/4.
 *  - The columnwise cast then runs on v' exactly as on x: the column amax is the
 *    max |v'| over the group's rows, and the block steps are unchanged.
 *  - SR replaces the final E2M1 rounding: with a = |y| < 6, lo <= a < hi the
 *    neighbouring E2M1 values and f = (a - lo) / (hi - lo) (exact), a 32-bit random
 *    word r rounds up iff r < ceil(f * 2^32), so up with probability f up to 2^-32;
 *    a >= 6 saturates to 6; the sign bit is y's.
 *  - The random word of columnwise element (row m, column k) is output m % 4 of
 *    Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) with counter
 *    (m / 4, k, lo32(offset), hi32(offset)) and key (lo32(seed), hi32(seed)). */

/* Philox4x32 with 10 rounds: each round maps the counter (c0, c1, c2, c3) with the key
 * (k0, k1) to (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)) with the
 * multipliers M0 = 0xD2511F53, M1 = 0xCD9E8D57; between rounds the key grows by the
 * Weyl constants (0x9E3779B9, 0xBB67AE85). */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n1 = (uint32_t)p1;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        const uint32_t n3 = (uint32_t)p0;
        c0 = n0;
        c1 = n1;
        c2 = n2;
        c3 = n3;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* The random word of columnwise element (row m, column k). */
uint32_t oracle_sr_word(int64_t m, int64_t k, uint64_t seed, uint64_t offset)
{
    const uint32_t ctr[4] = {(uint32_t)(m >> 2), (uint32_t)k, (uint32_t)offset, (uint32_t)(offset >> 32)};
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    return out[m & 3];
}

/* v' = (1/4) H16 S v by the four butterfly stages (see above). */
void oracle_rht16(const float* v, uint32_t signs, float* out)
{
    float w[16];
    for (int j = 0; j < 16; ++j) w[j] = ((signs >> j) & 1u) ? -v[j] : v[j];
    for (int h = 1; h < 16; h <<= 1)
        for (int i = 0; i < 16; ++i)
            if ((i & h) == 0) {
                const float a = w[i], b = w[i + h];
                w[i] = a + b;
                w[i + h] = a - b;
            }
    for (int j = 0; j < 16; ++j) out[j] = w[j] * 0.25f;
}

/* Stochastic rounding of y to E2M1 with the random word r (see above). */
uint8_t oracle_e2m1_sr(float y, uint32_t r)
{
    const uint8_t sign = signbit(y) ? 0x8 : 0x0;
    const double a = fabs((double)y);
    if (a >= 6.0) return sign | 0x7;
    int c = 0;
    while (c < 7 && kE2M1[c + 1] <= a) ++c;
    const double f = (a - kE2M1[c]) / (kE2M1[c + 1] - kE2M1[c]);   /* exact */
    const uint64_t t = (uint64_t)ceil(ldexp(f, 32));
    return sign | (uint8_t)((uint64_t)r < t ? c + 1 : c);
}

/* The columnwise direction of the grouped cast with the options: rht (0/1) with the
 * sign mask, sr (0/1) with seed and offset. Outputs and layouts as in
 * oracle_quantize_grouped (amax_col [G, K] of the transformed values when rht).
 * col_base: the index of x's first column in the full matrix (x may be a column
 * slice of it), which the random words use. Returns 0, or -1 on bad shape/offsets. */
int oracle_quantize_colwise_opts(const uint16_t* x, int64_t M, int64_t K, int64_t col_base, const int64_t* offsets,
                                 int G, int rht, uint32_t rht_signs, int sr, uint64_t seed, uint64_t offset,
                                 uint8_t* q_col, uint8_t* sf_col, float* amax_col)
{
    if (!shape_ok(M, K) || G < 1) return -1;
    if (offsets[0] != 0 || offsets[G] != M) return -1;
    for (int g = 0; g < G; ++g)
        if (offsets[g + 1] < offsets[g] || offsets[g] % 16 != 0) return -1;
    float v[16], y[16];
    for (int g = 0; g < G; ++g) {
        const int64_t r0 = offsets[g], m = offsets[g + 1] - offsets[g];
        uint8_t* qg = q_col + K * r0 / 2;
        uint8_t* sg = sf_col + K * r0 / 16;
        for (int64_t c = 0; c < K; ++c) {
            /* the column's amax over the group, of the (transformed) values */
            float amax = 0.0f;
            for (int64_t b = 0; b < m / 16; ++b) {
                for (int i = 0; i < 16; ++i) v[i] = oracle_bf16_to_f32(x[(r0 + 16 * b + i) * K + c]);
                if (rht) oracle_rht16(v, rht_signs, v);
                for (int i = 0; i < 16; ++i)
                    if (fabsf(v[i]) > amax) amax = fabsf(v[i]);
            }
            amax_col[(int64_t)g * K + c] = amax;
            const float s_enc = oracle_s_enc(amax);
            for (int64_t b = 0; b < m / 16; ++b) {
                for (int i = 0; i < 16; ++i) v[i] = oracle_bf16_to_f32(x[(r0 + 16 * b + i) * K + c]);
                if (rht) oracle_rht16(v, rht_signs, v);
                float ba = 0.0f;
                for (int i = 0; i < 16; ++i)
                    if (fabsf(v[i]) > ba) ba = fabsf(v[i]);
                const uint8_t sf = oracle_e4m3(oracle_block_scale_arg(ba, s_enc));
                const float enc = oracle_block_enc(sf, s_enc);
                uint8_t codes[16];
                for (int i = 0; i < 16; ++i) {
                    y[i] = v[i] * enc;
                    codes[i] = sr ? oracle_e2m1_sr(y[i], oracle_sr_word(r0 + 16 * b + i, col_base + c, seed, offset))
                                  : oracle_e2m1(y[i]);
                }
                for (int j = 0; j < 8; ++j)
                    qg[c * (m / 2) + 8 * b + j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
                sg[c * (m / 16) + b] = sf;
            }
        }
    }
    return 0;
}
