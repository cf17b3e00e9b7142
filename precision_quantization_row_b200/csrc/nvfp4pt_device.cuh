// Device building blocks of the NVFP4 per-token cast for sm_100a.
//
// Everything here is one binary32 IEEE operation per step (the library is built
// with -fmad=false, -prec-div=true, -ftz=false, and the arithmetic below uses the
// explicitly rounded intrinsics), so that the codes are bit-identical to the
// definition in include/nvfp4pt.h.
#pragma once

#include <cfloat>
#include <cstdint>
#include <cuda.h>

namespace nvfp4pt {

constexpr int kTile = 128;        // tile edge (rows and columns) of both passes
constexpr int kThreads = 256;     // threads per CTA of both passes
constexpr int kStages = 3;        // TMA stages of the encode pass
constexpr int kBoxBytes = kTile * 64 * 2;     // one 128 x 64 bf16 TMA box (16 KB)
constexpr int kStageBytes = 2 * kBoxBytes;    // a 128 x 128 bf16 tile (32 KB)
constexpr int kMaxGroups = 1024;
constexpr uint32_t kErrTmaTimeout = 1u;
constexpr uint32_t kErrDrainTimeout = 2u;
constexpr uint32_t kWaitLimit = 1u << 22;     // try_wait rounds before giving up (~seconds)

// ------------------------------------------------------------------ geometry
//
// Both passes of the tile path walk the same sequence of 128 x 128 tiles: for each token group g
// (one group when ungrouped), its rows split into 128-row bands (the last band of a
// group may be shorter, a multiple of 16), each band into ceil(cols/128) column
// tiles. Tile t is band t / ntc, column tile t % ntc. CTA c of both passes owns the
// same contiguous tile range; pass 2 walks it backwards so it starts on the tiles
// pass 1 touched last (still in L2).

struct Geometry {
    int64_t rows;
    int64_t cols;
    int64_t total_tiles;
    int32_t ntc;          // column tiles per band
    int32_t num_groups;
    int32_t num_ctas;     // CTAs of the launch
    int32_t interleave;   // CTAs sharing one tile range (1 or 2), each taking every
                          // interleave-th tile of it
};

template <int MAXG>
struct Groups {
    int32_t band_start[MAXG + 1];  // bands before group g (non-decreasing)
    int32_t row_off[MAXG + 1];     // first row of group g; row_off[G] = rows
};

struct TileInfo {
    int64_t band;   // global band index
    int64_t r0;     // first row of the tile
    int64_t c0;     // first column of the tile
    int32_t g;      // token group
    int32_t nr;     // valid rows (multiple of 16, 16..128)
    int32_t nc;     // valid columns (multiple of 16, 16..128)
    int32_t goff;   // first row of the group
    int32_t grows;  // rows of the group
};

template <int MAXG>
__device__ __forceinline__ TileInfo tile_info(const Geometry& geo, const Groups<MAXG>& grp, int64_t t)
{
    TileInfo ti;
    ti.band = t / geo.ntc;
    const int32_t ct = (int32_t)(t - ti.band * geo.ntc);
    int g = 0;
    if (MAXG > 1) {
        int lo = 0, hi = geo.num_groups;  // band_start[lo] <= band < band_start[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if ((int64_t)grp.band_start[mid] <= ti.band) lo = mid; else hi = mid;
        }
        g = lo;
    }
    ti.g = g;
    ti.goff = grp.row_off[g];
    ti.grows = grp.row_off[g + 1] - grp.row_off[g];
    const int64_t local_band = ti.band - grp.band_start[g];
    ti.r0 = (int64_t)ti.goff + local_band * kTile;
    const int64_t rem_r = (int64_t)grp.row_off[g + 1] - ti.r0;
    ti.nr = (int32_t)(rem_r < kTile ? rem_r : kTile);
    ti.c0 = (int64_t)ct * kTile;
    const int64_t rem_c = geo.cols - ti.c0;
    ti.nc = (int32_t)(rem_c < kTile ? rem_c : kTile);
    return ti;
}

// Walks tiles backwards from a start tile in steps of `step` tiles, keeping (band,
// column tile) and the band's group facts up to date without dividing per tile.
template <int MAXG>
struct TileWalker {
    int64_t band;
    int32_t ct;
    TileInfo ti;

    __device__ __forceinline__ void locate(const Geometry& geo, const Groups<MAXG>& grp)
    {
        int g = 0;
        if (MAXG > 1) {
            int lo = 0, hi = geo.num_groups;
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if ((int64_t)grp.band_start[mid] <= band) lo = mid; else hi = mid;
            }
            g = lo;
        }
        ti.band = band;
        ti.g = g;
        ti.goff = grp.row_off[g];
        ti.grows = grp.row_off[g + 1] - grp.row_off[g];
        ti.r0 = (int64_t)ti.goff + (band - grp.band_start[g]) * kTile;
        const int64_t rem_r = (int64_t)grp.row_off[g + 1] - ti.r0;
        ti.nr = (int32_t)(rem_r < kTile ? rem_r : kTile);
    }
    __device__ __forceinline__ void set_cols(const Geometry& geo)
    {
        ti.c0 = (int64_t)ct * kTile;
        const int64_t rem_c = geo.cols - ti.c0;
        ti.nc = (int32_t)(rem_c < kTile ? rem_c : kTile);
    }
    __device__ __forceinline__ void start(const Geometry& geo, const Groups<MAXG>& grp, int64_t t)
    {
        band = t / geo.ntc;
        ct = (int32_t)(t - band * geo.ntc);
        locate(geo, grp);
        set_cols(geo);
    }
    __device__ __forceinline__ void back(const Geometry& geo, const Groups<MAXG>& grp, int32_t step)
    {
        ct -= step;
        if (ct < 0) {
            do { ct += geo.ntc; --band; } while (ct < 0);
            locate(geo, grp);
        }
        set_cols(geo);
    }
};

// Tile range [t0, t1) of a CTA when every CTA owns its own range (interleave 1).
__device__ __forceinline__ void cta_tile_range(const Geometry& geo, int cta, int64_t& t0, int64_t& t1)
{
    t0 = (geo.total_tiles * cta) / geo.num_ctas;
    t1 = (geo.total_tiles * (cta + 1)) / geo.num_ctas;
}

// The encode pass walks its range backwards; with interleave il, CTAs il*k .. il*k+il-1
// share range k (ranges are cut as for num_ctas / il CTAs) and CTA il*k+j takes tiles
// t1-1-j, t1-1-j-il, ... . Returns the count n; the i-th tile is last - i * step.
__device__ __forceinline__ int64_t cta_reverse_tiles(const Geometry& geo, int cta, int64_t& last, int64_t& step)
{
    const int il = geo.interleave;
    const int ranges = geo.num_ctas / il;
    const int k = cta / il, j = cta - k * il;
    const int64_t t0 = (geo.total_tiles * k) / ranges;
    const int64_t t1 = (geo.total_tiles * (k + 1)) / ranges;
    last = t1 - 1 - j;
    step = il;
    return last < t0 ? 0 : (last - t0) / il + 1;
}

// ----------------------------------------------------- programmatic launch
// The passes are chained with programmatic dependent launch: a dependent grid may
// start while its predecessor drains, and must wait before touching its results.

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// --------------------------------------------------------------- bf16 words
// A 32-bit word holds two bf16 values: element 2j in the low half, 2j+1 in the high.

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Per-half max of magnitudes. The sign bits of the result are not meaningful (they
// are the xor of the inputs' signs); callers clear them with & 0x7FFF7FFF.
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Larger of the two magnitudes held in w, as binary32 (exact: bf16 -> fp32).
__device__ __forceinline__ float absmax_of_pair(uint32_t w)
{
    const uint32_t lo = w & 0x7FFFu;
    const uint32_t hi = (w >> 16) & 0x7FFFu;
    return __uint_as_float((lo > hi ? lo : hi) << 16);
}

// -------------------------------------------------------------- conversions

// Byte of two E2M1 codes, round-to-nearest-even, saturating: `lo` -> bits 0-3,
// `hi` -> bits 4-7 (zero-extended to 32 bits). The hardware conversion puts its
// first source operand in the high nibble.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 q;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q, %2, %1;\n\t"
        "cvt.u32.u8 %0, q;\n\t}"
        : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

// (y0, y1) = (RN(x0 * e), RN(x1 * e)) with one packed two-lane binary32 multiply.
__device__ __forceinline__ void mul2(float& y0, float& y1, float x0, float x1, float e)
{
    unsigned long long a, b, d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(x0), "f"(x1));
    asm("mov.b64 %0, {%1, %1};" : "=l"(b) : "f"(e));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(d));
}

// Two E4M3 (e4m3fn) codes, round-to-nearest-even, saturating: `lo` -> bits 0-7,
// `hi` -> bits 8-15.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(lo), "f"(hi));
    return r;
}

// Exact value of the two E4M3 codes in the low 16 bits of `codes` (bits 0-7 -> lo).
__device__ __forceinline__ void e4m3x2_decode(uint32_t codes, float& lo, float& hi)
{
    uint32_t h2;
    const uint16_t c = (uint16_t)codes;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.f32.f16 %0, l;\n\t"
        "cvt.f32.f16 %1, h;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(h2));
}

// ------------------------------------------------------------ block arithmetic

// RN(b / 6) for every finite non-negative bf16 value b, in three operations:
// q0 = RN(b * r), the exact remainder b - 6*q0 by one fused multiply-add, then one
// correction step q0 + rem * r (the correction of Markstein's method, with the
// reciprocal r = RN(1/6) fixed in advance). The result equals the IEEE quotient for
// all 32640 such inputs; the library's probe entry checks that on the device.
__device__ __forceinline__ float div6(float b)
{
    const float r = 0x1.555556p-3f;  // RN(1/6)
    const float q0 = __fmul_rn(b, r);
    const float rem = __fmaf_rn(-q0, 6.0f, b);
    return __fmaf_rn(rem, r, q0);
}

// s_enc = 2688 / amax, 1 when amax == 0, clamped to FLT_MAX instead of overflowing.
__device__ __forceinline__ float s_enc_of(float amax)
{
    if (amax == 0.0f) return 1.0f;
    return fminf(__fdiv_rn(2688.0f, amax), FLT_MAX);
}

// Reciprocal table of the E4M3 significands: tab[f] = bits of RN(1 / (1 + f/8)),
// f = 0..7. Each CTA keeps it in shared memory (8 words, one bank each).
__device__ __forceinline__ void init_rcp_table(uint32_t* tab)
{
    if (threadIdx.x < 8) tab[threadIdx.x] = __float_as_uint(__fdiv_rn(1.0f, 1.0f + 0.125f * (float)threadIdx.x));
}

// RN(s / d) for s a positive normal binary32 and d a positive E4M3 value (as exact
// binary32). d has a 4-bit significand, so y = RN(1/d) is a table entry scaled by d's
// power of two (exactly); then q0 = RN(s * y), the exact remainder r = s - q0*d by one
// fused multiply-add, and one correction q0 + r*y -- the correction step of Markstein's
// division (IBM J. Res. Dev. 34(1), 1990). It equals the IEEE quotient for every E4M3
// divisor and every s tried (all significands of 20 binades from 2^-117 up to 2^127,
// and FLT_MAX); the probe entry compares it with the IEEE division on the device.
// An overflowing quotient comes out as +inf or NaN; the caller clamps it.
__device__ __forceinline__ float div_by_e4m3(float s, float d, const uint32_t* tab)
{
    const uint32_t db = __float_as_uint(d);
    const float y = __uint_as_float(tab[(db >> 20) & 7u] + 0x3F800000u - (db & 0x7F800000u));
    const float q0 = __fmul_rn(s, y);
    const float r = __fmaf_rn(-q0, d, s);
    return __fmaf_rn(r, y, q0);
}

// enc = s_enc / float(sf), 0 when sf == 0, clamped to FLT_MAX (fminf also maps the NaN
// of an overflowed quotient to FLT_MAX).
__device__ __forceinline__ float enc_of(uint32_t sf_code, float d, float s, const uint32_t* tab)
{
    return (sf_code & 0xFFu) ? fminf(div_by_e4m3(s, d, tab), FLT_MAX) : 0.0f;
}

// Scale codes and multipliers of two blocks with block amaxes b0, b1 and outer
// scales s0, s1. sf01 receives the two codes (block 0 in bits 0-7).
__device__ __forceinline__ void block_pair_scales(float b0, float b1, float s0, float s1,
                                                  uint32_t& sf01, float& e0, float& e1, const uint32_t* tab)
{
    const float u0 = __fmul_rn(div6(b0), s0);
    const float u1 = __fmul_rn(div6(b1), s1);
    sf01 = e4m3x2(u0, u1);
    float d0, d1;
    e4m3x2_decode(sf01, d0, d1);
    e0 = enc_of(sf01, d0, s0, tab);
    e1 = enc_of(sf01 >> 8, d1, s1, tab);
}

// ------------------------------------------------- packed two-lane binary32
// One 64-bit register holds two binary32 lanes (lo, hi); the f32x2 instructions
// round each lane exactly as the scalar instruction would.

__device__ __forceinline__ unsigned long long pack2(float lo, float hi)
{
    unsigned long long v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
    return v;
}

__device__ __forceinline__ void unpack2(unsigned long long v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ unsigned long long mul_f32x2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// a * b + c per lane, one rounding
__device__ __forceinline__ unsigned long long fma_f32x2(unsigned long long a, unsigned long long b,
                                                        unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// block_pair_scales with the two blocks in the lanes of packed instructions. Same
// arithmetic step for step: RN(b/6) by div6's three operations (the remainder as
// fma(q0, -6, b), equal to fma(-q0, 6, b)), times s, the E4M3 codes, and the quotient
// s / d by div_by_e4m3's correction step written on the negated reciprocal -y:
// q0n = s*(-y) = -RN(s*y), r = fma(q0n, d, s) = RN(s - q0*d), and
// fma(r, -y, q0n) = -RN(q0 + r*y), negated back where it is clamped.
__device__ __forceinline__ void block_pair_scales_x2(float b0, float b1, float s0, float s1, uint32_t& sf01,
                                                     float& e0, float& e1, const uint32_t* tab)
{
    const unsigned long long r6 = pack2(0x1.555556p-3f, 0x1.555556p-3f);   // RN(1/6)
    const unsigned long long b = pack2(b0, b1);
    const unsigned long long q0 = mul_f32x2(b, r6);
    const unsigned long long rem = fma_f32x2(q0, pack2(-6.0f, -6.0f), b);
    const unsigned long long q1 = fma_f32x2(rem, r6, q0);
    const unsigned long long s = pack2(s0, s1);
    float u0, u1;
    unpack2(mul_f32x2(q1, s), u0, u1);
    sf01 = e4m3x2(u0, u1);
    float d0, d1;
    e4m3x2_decode(sf01, d0, d1);
    const uint32_t db0 = __float_as_uint(d0), db1 = __float_as_uint(d1);
    // -RN(1/d): the table entry with d's power of two taken out and the sign set
    const float ny0 = __uint_as_float(tab[(db0 >> 20) & 7u] + 0xBF800000u - (db0 & 0x7F800000u));
    const float ny1 = __uint_as_float(tab[(db1 >> 20) & 7u] + 0xBF800000u - (db1 & 0x7F800000u));
    const unsigned long long ny = pack2(ny0, ny1);
    const unsigned long long q0n = mul_f32x2(s, ny);
    const unsigned long long r = fma_f32x2(q0n, pack2(d0, d1), s);
    float qn0, qn1;
    unpack2(fma_f32x2(r, ny, q0n), qn0, qn1);
    e0 = (sf01 & 0xFFu) ? fminf(-qn0, FLT_MAX) : 0.0f;
    e1 = (sf01 & 0xFF00u) ? fminf(-qn1, FLT_MAX) : 0.0f;
}

// Codes of four scaled pairs (y[2i], y[2i+1]) -> one word, y[j] in bits 4j..4j+3.
__device__ __forceinline__ uint32_t e2m1x8_packed(const float (&y)[8])
{
    uint32_t r;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(r) : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
    return r;
}

// Codes of the 8 elements held in 4 bf16 words with one multiplier: one word,
// element i in bits 4i..4i+3.
__device__ __forceinline__ uint32_t encode8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float e)
{
    float y[8];
    mul2(y[0], y[1], bf16_lo(w0), bf16_hi(w0), e);
    mul2(y[2], y[3], bf16_lo(w1), bf16_hi(w1), e);
    mul2(y[4], y[5], bf16_lo(w2), bf16_hi(w2), e);
    mul2(y[6], y[7], bf16_lo(w3), bf16_hi(w3), e);
    return e2m1x8_packed(y);
}

// Codes of one column over 8 consecutive rows, the column being the low (hi=false) or
// high (hi=true) half of the words x[0..7] (row i in x[i]): one word, row i in bits 4i.
template <bool HI>
__device__ __forceinline__ uint32_t encode8_col(const uint32_t* x, float e)
{
    auto v = [&](int i) { return HI ? bf16_hi(x[i]) : bf16_lo(x[i]); };
    float y[8];
    mul2(y[0], y[1], v(0), v(1), e);
    mul2(y[2], y[3], v(2), v(3), e);
    mul2(y[4], y[5], v(4), v(5), e);
    mul2(y[6], y[7], v(6), v(7), e);
    return e2m1x8_packed(y);
}

// ---------------------------------------------------------------- memory ops

__device__ __forceinline__ uint4 ldg_stream(const void* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// 8 bytes through the read-only path, not kept in L1.
__device__ __forceinline__ uint2 ldg_stream64(const void* p)
{
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// 32 bytes (one 16-element bf16 block) through the read-only path, not kept in L1.
__device__ __forceinline__ void ldg256_stream(const void* p, uint32_t (&v)[8])
{
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "l"(p));
}

// Stores of outputs that nothing in the cast reads again, marked evict-first in L2 so
// that they do not push out the lines of x that the column pass is about to read.
__device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void stg16_ef(uint8_t* p, uint4 v, uint64_t pol)   // 16-byte aligned
{
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(pol) : "memory");
}
__device__ __forceinline__ void stg32_ef(uint8_t* p, uint4 a, uint4 b, uint64_t pol)   // 32-byte aligned
{
    asm volatile("st.global.L2::cache_hint.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8}, %9;"
                 :: "l"(p), "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void stg8_ef(uint8_t* p, uint32_t a, uint32_t b, uint64_t pol)   // 8-byte aligned
{
    asm volatile("st.global.L2::cache_hint.v2.u32 [%0], {%1, %2}, %3;" :: "l"(p), "r"(a), "r"(b), "l"(pol) : "memory");
}
__device__ __forceinline__ void stg1_ef(uint8_t* p, uint32_t v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.u8 [%0], %1, %2;" :: "l"(p), "r"(v), "l"(pol) : "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// 16 bytes to global memory that is at least 8-byte aligned.
__device__ __forceinline__ void stg16(uint8_t* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    if ((reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
        asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" :: "l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
    } else {
        asm volatile("st.global.v2.u32 [%0], {%1, %2};" :: "l"(p), "r"(a), "r"(b) : "memory");
        asm volatile("st.global.v2.u32 [%0], {%1, %2};" :: "l"(p + 8), "r"(c), "r"(d) : "memory");
    }
}

// 32 bytes to a 32-byte aligned address in one store.
__device__ __forceinline__ void stg32(uint8_t* p, uint4 a, uint4 b)
{
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :: "l"(p), "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

__device__ __forceinline__ void stg8(uint8_t* p, uint32_t a, uint32_t b)
{
    asm volatile("st.global.v2.u32 [%0], {%1, %2};" :: "l"(p), "r"(a), "r"(b) : "memory");
}

// n (<= 4) bytes of v, low byte first, at any alignment.
__device__ __forceinline__ void stg_bytes(uint8_t* p, uint32_t v, int n)
{
    if (n == 4 && (reinterpret_cast<uintptr_t>(p) & 3u) == 0) {
        *reinterpret_cast<uint32_t*>(p) = v;
    } else if (n == 2 && (reinterpret_cast<uintptr_t>(p) & 1u) == 0) {
        *reinterpret_cast<uint16_t*>(p) = (uint16_t)v;
    } else {
        for (int i = 0; i < n; ++i) p[i] = (uint8_t)(v >> (8 * i));
    }
}

// Non-negative binary32 maxima are combined as their bit patterns (order-preserving
// for non-negative values); the targets start at +0.
__device__ __forceinline__ void red_max_f32(float* p, uint32_t bits)
{
    atomicMax(reinterpret_cast<unsigned int*>(p), bits);
}

// Lane-wise atomic max of 8 non-negative bf16 values (four bf16x2 words) into 16-byte
// aligned global memory: one reduction operation instead of eight.
__device__ __forceinline__ void red_max_bf16x8(uint32_t* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("red.global.max.noftz.v4.bf16x2 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// ------------------------------------------------------------ mbarrier + TMA

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Wait for phase `parity` of the barrier to complete, giving up after kWaitLimit
// rounds (each try_wait round may itself suspend the thread for a while).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
    for (uint32_t i = 0; i < kWaitLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// One 2D tiled TMA load (box = the tensor map's box) into shared memory, completing
// on `bar`. x is the column (innermost) coordinate, a multiple of 64 elements.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];"
                 :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" :: "l"(map) : "memory");
}

// Byte offset, inside a 128-row x 128-byte box loaded with 128-byte swizzling, of the
// 16-byte chunk `chunk` of row `row`: the chunk index is xor-ed with row % 8.
__device__ __forceinline__ uint32_t swz128(int row, int chunk)
{
    return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

}  // namespace nvfp4pt
