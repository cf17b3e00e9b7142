// Device steps of the columnwise options of the cast (TransformerEngine PR #3045,
// Changes: opt-in RHT / SR on the per-token path, off by default; its review: the row
// direction never uses RHT). The pages fix neither the transform nor the random
// numbers; the readings taken:
//   - RHT: each columnwise 16-element block v (16 consecutive rows of one column in a
//     token group) becomes v' = (1/4) H16 S v, H16 the Sylvester Hadamard matrix
//     (entry (i, j) = (-1)^popcount(i & j)) and S the diagonal of signs given by a
//     16-bit mask (bit j set: -1). Evaluated as the radix-2 butterfly in four stages
//     (pairs i, i + h for h = 1, 2, 4, 8: sum and difference, one binary32 rounding
//     each), then the exact multiply by 1/4. The column amax is then max |v'|.
//   - SR: the E2M1 rounding of y = RN(v' * enc) becomes stochastic: with a = |y| < 6
//     between the E2M1 neighbours lo <= a < hi and f = (a - lo) / (hi - lo) (exact),
//     a 32-bit random word r rounds up iff r < ceil(f * 2^32); a >= 6 gives 6; the
//     sign bit is y's.
//   - r of element (row m, column k) is word m % 4 of Philox4x32-10 (Salmon, Moraes,
//     Dror, Shaw, SC'11) at counter (m / 4, k, lo32(offset), hi32(offset)) with key
//     (lo32(seed), hi32(seed)).
#pragma once

#include "nvfp4pt_device.cuh"

namespace nvfp4pt {

// Philox4x32 with 10 rounds. A round maps (c0, c1, c2, c3) with key (k0, k1) to
// (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)), M0 = 0xD2511F53,
// M1 = 0xCD9E8D57; the key grows by (0x9E3779B9, 0xBB67AE85) between rounds.
__device__ __forceinline__ uint4 philox10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                                          uint32_t k1)
{
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t hi0 = __umulhi(0xD2511F53u, c0), lo0 = 0xD2511F53u * c0;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2), lo1 = 0xCD9E8D57u * c2;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
    }
    return make_uint4(c0, c1, c2, c3);
}

// v' = (1/4) H16 S v in place (four butterfly stages, then the exact 1/4).
__device__ __forceinline__ void rht16(float (&f)[16], uint32_t signs)
{
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if ((signs >> j) & 1u) f[j] = -f[j];
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if ((i & h) == 0) {
                const float a = f[i], b = f[i + h];
                f[i] = __fadd_rn(a, b);
                f[i + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) f[j] = __fmul_rn(f[j], 0.25f);
}

// Stochastic E2M1 code of y with the random word r (4 bits: sign in bit 3), without
// branches: for a = |y| < 6 the grid point lo at or below a, the gap to the next one and
// lo's code come from a's bits --
//   a >= 1 (biased exponent e = 127, 128, 129): lo = a with its significand cut to one
//          bit, gap = 2^(e - 128), code 2 (e - 127) + 2 + (the significand's top bit);
//   a < 1: lo = 0 or 0.5 (codes 0, 1), gap = 0.5 --
// then f = (a - lo) / gap (exact: a - lo is exact and the gap a power of two) and the
// code steps up iff r < ceil(f * 2^32).
__device__ __forceinline__ uint32_t e2m1_sr(float y, uint32_t r)
{
    const uint32_t yb = __float_as_uint(y);
    const uint32_t sign = (yb >> 28) & 8u;
    const uint32_t ab = yb & 0x7FFFFFFFu;
    const bool big = ab >= 0x3F800000u;                                  // a >= 1
    const bool half = ab >= 0x3F000000u;                                 // a >= 0.5
    const uint32_t lo_b = big ? (ab & 0xFFC00000u) : (half ? 0x3F000000u : 0u);
    const uint32_t gap_b = big ? ((ab & 0x7F800000u) - 0x00800000u) : 0x3F000000u;
    const uint32_t c = big ? 2u * ((ab >> 23) - 127u) + 2u + ((ab >> 22) & 1u) : (half ? 1u : 0u);
    const float f = __fmul_rn(__fsub_rn(__uint_as_float(ab), __uint_as_float(lo_b)),
                              __uint_as_float(0x7F000000u - gap_b));   // times 1 / gap
    const uint32_t t = __float2uint_ru(__fmul_rn(f, 4294967296.0f));   // ceil(f * 2^32) < 2^32
    const uint32_t code = ab >= 0x40C00000u ? 7u : (r < t ? c + 1u : c);   // a >= 6 saturates
    return sign | code;
}

// The block steps with IEEE divisions (the block amax of transformed values is any
// binary32 number): sf = e4m3(RN(RN(ba / 6) * s)), enc = sf ? RN(s / float(sf)) : 0,
// enc clamped to FLT_MAX.
__device__ __forceinline__ void block_scale_ieee(float ba, float s, uint32_t& sf, float& enc)
{
    const float u = __fmul_rn(__fdiv_rn(ba, 6.0f), s);
    sf = e4m3x2(u, 0.0f) & 0xFFu;
    float d, unused;
    e4m3x2_decode(sf, d, unused);
    enc = sf ? fminf(__fdiv_rn(s, d), FLT_MAX) : 0.0f;
}

}  // namespace nvfp4pt
