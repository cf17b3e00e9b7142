// Columnwise requantization of rowwise NVFP4 data: the columnwise cast of
// X' = dequantize(q, sf, amax), the per-token form of the "dequantize, then requantize
// columnwise only" flow of TransformerEngine PR #3244 (Description and flowchart).
// Two kernels follow the zeroing kernel, chained by programmatic dependent launch:
//   rq_colmax  one read of the rowwise codes and scales: the rows' decode scales
//              S_dec = RN(amax / 2688), the bf16 column maxima of X' per token group
//              (8-wide bf16 atomics) and each group's observed maximum;
//   rq_colenc  a second read (the rowwise data are 9/16 byte per element, so most of it
//              comes back from L2) that rebuilds X' in registers, 32 rows x 64 columns
//              per warp step, and writes the columnwise codes, block scales and fp32
//              column amaxes; its CTA 0 applies the decayed absmax update.
// Element values: X'[r][c] = bf16(RN(RN(val(q) * sf) * S_dec[r])). val(q) * sf has at
// most six significant bits and lies in [2^-10, 2688] (or is zero), so binary16 holds it
// exactly: the E2M1 pair conversion to f16x2 and one f16x2 multiply give two products
// exactly, then two widenings, one packed binary32 multiply by S_dec and one packed bf16
// rounding give the element pair. The cast of X' is the per-token cast's own arithmetic.
#pragma once

#include "nvfp4pt_device.cuh"

namespace nvfp4pt {

constexpr int kRqThreads = 256;
constexpr int kRqWarps = kRqThreads / 32;
constexpr int kRqChunkCols = 256;   // rq_colmax: columns of a warp's chunk (8 per lane)
constexpr int kRqSliceRows = 16;    // rq_colmax: rows of a slice (a token group holds whole slices)
constexpr int kRqStripCols = 64;    // rq_colenc: columns of a strip (8 per lane, 8 lanes)
constexpr int kRqStepRows = 32;     // rq_colenc: rows of a step (8 per lane, 4 lanes)

template <int MAXG>
struct RqParams {
    const uint8_t* q;      // rowwise codes [rows, cols/2], element 2j in the low nibble
    const uint8_t* sf;     // rowwise block scales [rows, cols/16]
    const float* amax;     // row amaxes [rows]
    float* dscale;         // [rows] decode scales: written by rq_colmax, read by rq_colenc
    uint16_t* colmax;      // [G, cols] bf16 column maxima of X' (zeroed before rq_colmax)
    float* obs;            // [G] observed maxima (zeroed), or null
    uint8_t* q_col;        // group g: [cols, m_g/2] at byte cols*offsets[g]/2
    uint8_t* sf_col;       // group g: [cols, m_g/16] at byte cols*offsets[g]/16
    float* amax_col;       // [G, cols] (zeroed: empty groups keep 0)
    float* absmax;         // [nbuf] running buffers, or null
    float decay;
    int32_t nbuf;
    int64_t rows;
    int64_t cols;
    int64_t chunks;        // rq_colmax: ceil(cols / 256)
    int64_t slices;        // rq_colmax: rows / 16
    int32_t strips;        // rq_colenc: ceil(cols / 64)
    int32_t num_groups;
    int32_t row_off[MAXG + 1];    // first row of each group
    int32_t step_off[MAXG + 1];   // first 32-row step of each group (a group's steps start at its first row)
    // rq_tile only (rows a multiple of 256 wide)
    CUtensorMap tm_q;             // codes: uint8 [rows, cols/2], boxes 128 x 64
    CUtensorMap tm_sf;            // scales: uint8 [rows, cols/16], boxes 16 x 64
    CUtensorMap tm_amax;          // row amaxes: fp32 [1, rows], boxes of 64
    uint32_t* err;                // device error word (a copy that never lands)
    int32_t tstep_off[MAXG + 1];  // first 64-row step of each group
};

// The last group g with row_off[g] <= row: the group holding the row, empty groups skipped.
template <int MAXG>
__device__ __forceinline__ int rq_group_of_row(const RqParams<MAXG>& p, int64_t row)
{
    if (MAXG == 1) return 0;
    int lo = 0, hi = p.num_groups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.row_off[mid] <= row) lo = mid; else hi = mid;
    }
    return lo;
}

// The last group g with step_off[g] <= k: the group holding step k, empty groups skipped.
template <int MAXG>
__device__ __forceinline__ int rq_group_of_step(const RqParams<MAXG>& p, int64_t k)
{
    if (MAXG == 1) return 0;
    int lo = 0, hi = p.num_groups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.step_off[mid] <= k) lo = mid; else hi = mid;
    }
    return lo;
}

// A warp's share [u, u_end) of n units, n split as evenly as the warps allow.
__device__ __forceinline__ void rq_warp_share(int64_t n, int64_t& u, int64_t& u_end)
{
    const int64_t nw = (int64_t)gridDim.x * kRqWarps;
    const int64_t w = (int64_t)blockIdx.x * kRqWarps + (threadIdx.x >> 5);
    const int64_t base = n / nw, rem = n % nw;
    u = w * base + (w < rem ? w : rem);
    u_end = u + base + (w < rem ? 1 : 0);
}

// X' of the eight elements of one code word (element i in bits 4i..4i+3) with block
// scale code sfc and decode scale m: four bf16x2 words, element 2j in the low half of word j.
__device__ __forceinline__ void rq_dequant8(uint32_t codes, uint32_t sfc, float m, uint32_t (&w)[4])
{
    uint32_t s2;   // (sf, sf) as f16x2
    const uint16_t sc2 = (uint16_t)(sfc * 0x0101u);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s2) : "h"(sc2));
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(codes));
    const unsigned long long mm = pack2(m, m);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t t;
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(t) : "r"(h[j]), "r"(s2));   // val * sf: exact
        float lo, hi;
        asm("{\n\t.reg .b16 l, h;\n\t"
            "mov.b32 {l, h}, %2;\n\t"
            "cvt.f32.f16 %0, l;\n\t"
            "cvt.f32.f16 %1, h;\n\t}"
            : "=f"(lo), "=f"(hi) : "r"(t));
        float y0, y1;
        unpack2(mul_f32x2(pack2(lo, hi), mm), y0, y1);
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w[j]) : "f"(y1), "f"(y0));
    }
}

__device__ __forceinline__ void stg4_ef(uint8_t* p, uint32_t v, uint64_t pol)   // 4-byte aligned
{
    asm volatile("st.global.L2::cache_hint.u32 [%0], %1, %2;" :: "l"(p), "r"(v), "l"(pol) : "memory");
}

// ------------------------------------------------------------------ rq_colmax
// Units are (256-column chunk, 16-row slice) pairs in chunk-major order; each warp takes
// a contiguous run of them and keeps its lanes' eight column maxima in registers until
// the chunk or the token group changes, then raises colmax (one 16-byte atomic per lane)
// and the group's observed maximum (one atomic per warp).
template <int MAXG>
__global__ void __launch_bounds__(kRqThreads, 3) rq_colmax(const __grid_constant__ RqParams<MAXG> p)
{
    // rq_colenc may launch early: it waits for this grid before it reads what this grid writes.
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    int64_t u, u_end;
    rq_warp_share(p.slices * p.chunks, u, u_end);
    if (u >= u_end) return;

    const int64_t cols = p.cols;
    const int64_t half = cols / 2, sfr = cols / 16;
    int64_t ch = u / p.slices;
    int64_t s = u - ch * p.slices;
    int g = rq_group_of_row(p, s * kRqSliceRows);
    bool waited = false;
    uint32_t acc[4] = {0u, 0u, 0u, 0u};
    for (;;) {
        const int64_t c = ch * kRqChunkCols + 8 * lane;   // this lane's first column
        const bool cok = c < cols;
        const int64_t r0 = s * kRqSliceRows;
        // lane i < 16: the decode scale of row r0 + i (the first chunk's warp keeps it)
        float dl = 0.0f;
        if (lane < kRqSliceRows) {
            dl = __fdiv_rn(__ldg(p.amax + r0 + lane), 2688.0f);
            if (ch == 0) p.dscale[r0 + lane] = dl;
        }
        uint32_t cw[kRqSliceRows], sb[kRqSliceRows];
        const uint8_t* qp = p.q + r0 * half + c / 2;
        const uint8_t* sp = p.sf + r0 * sfr + c / 16;
#pragma unroll
        for (int i = 0; i < kRqSliceRows; ++i) {
            cw[i] = cok ? __ldg(reinterpret_cast<const uint32_t*>(qp + i * half)) : 0u;
            sb[i] = cok ? (uint32_t)__ldg(sp + i * sfr) : 0u;
        }
#pragma unroll
        for (int i = 0; i < kRqSliceRows; ++i) {
            const float m = __shfl_sync(0xFFFFFFFFu, dl, i);
            uint32_t x[4];
            rq_dequant8(cw[i], sb[i], m, x);
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = absmax2(acc[j], x[j]);
        }

        // the next unit; the maxima go out at the end of the run, of a chunk or of a group
        ++u;
        const bool last = u >= u_end;
        int64_t nch = ch, ns = s + 1;
        if (ns == p.slices) {
            ++nch;
            ns = 0;
        }
        int ng = nch == ch ? g : 0;
        if (MAXG > 1 && !last)
            while (ng + 1 < p.num_groups && p.row_off[ng + 1] <= ns * kRqSliceRows) ++ng;
        if (last || nch != ch || ng != g) {
            if (!waited) {   // colmax and obs were zeroed by the kernel before this one
                griddep_wait();
                waited = true;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] &= 0x7FFF7FFFu;
            if (cok)
                red_max_bf16x8(reinterpret_cast<uint32_t*>(p.colmax + (int64_t)g * cols + c), acc[0], acc[1],
                               acc[2], acc[3]);
            if (p.obs) {
                uint32_t mx = 0u;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    mx = max(mx, acc[j] & 0xFFFFu);
                    mx = max(mx, acc[j] >> 16);
                }
                mx = __reduce_max_sync(0xFFFFFFFFu, mx << 16);   // binary32 bits of the bf16 maximum
                if (lane == 0 && mx) red_max_f32(p.obs + g, mx);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = 0u;
        }
        if (last) break;
        ch = nch;
        s = ns;
        g = ng;
    }
}

// ------------------------------------------------------------------ rq_colenc
// Units are (64-column strip, 32-row step) pairs in strip-major order, the steps of each
// token group starting at its first row; each warp takes a contiguous run. Lane
// (cg, rh) = (lane & 7, lane >> 3) holds columns 8cg..8cg+7 of rows 8rh..8rh+7 of the
// step, so lanes rh = 2b and 2b + 1 together hold the 16-row block b of each column:
// they combine their halves of the block amax with one shuffle, each finds the block
// scales of four of the eight columns, and they trade the multipliers.
struct RqStep {
    int32_t g;       // token group
    int32_t strip;
    int64_t k;       // step index within the strip (over all groups)
    int64_t row0;    // first row of the step
    int32_t nrows;   // rows of the step in its group: 16 or 32
};

template <int MAXG>
__global__ void __launch_bounds__(kRqThreads, 2) rq_colenc(const __grid_constant__ RqParams<MAXG> p)
{
    // The next call's zeroing kernel may take this grid's place early; it waits for it.
    griddep_launch_dependents();
    __shared__ uint32_t rcp_tab[8];
    init_rcp_table(rcp_tab);

    const int lane = threadIdx.x & 31;
    const int cg = lane & 7;
    const int rh = lane >> 3;
    const int odd = rh & 1;
    const int64_t cols = p.cols;
    const int64_t half = cols / 2, sfr = cols / 16;
    const int64_t steps = p.step_off[p.num_groups];   // steps of one strip
    int64_t u, u_end;
    rq_warp_share(steps * p.strips, u, u_end);

    auto locate = [&](RqStep& st, int32_t strip, int64_t k, int g) {
        st.g = g;
        st.strip = strip;
        st.k = k;
        st.row0 = p.row_off[g] + (k - p.step_off[g]) * kRqStepRows;
        const int64_t left = p.row_off[g + 1] - st.row0;
        st.nrows = left < kRqStepRows ? (int32_t)left : kRqStepRows;
    };
    // the step after st in strip-major order
    auto advance = [&](const RqStep& st, RqStep& nx) {
        int32_t strip = st.strip;
        int64_t k = st.k + 1;
        int g = st.g;
        if (k == steps) {
            ++strip;
            k = 0;
            g = 0;
        }
        if (MAXG > 1)
            while (g + 1 < p.num_groups && p.step_off[g + 1] <= k) ++g;
        locate(nx, strip, k, g);
    };

    uint32_t cw[8], sb[8];
    float4 d0, d1;
    auto load_codes = [&](const RqStep& st) {
        const int64_t c = (int64_t)st.strip * kRqStripCols + 8 * cg;
        const bool ok = c < cols && 8 * rh < st.nrows;
        const int64_t row = st.row0 + 8 * rh;
        const uint8_t* qp = p.q + row * half + c / 2;
        const uint8_t* sp = p.sf + row * sfr + c / 16;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            cw[i] = ok ? __ldg(reinterpret_cast<const uint32_t*>(qp + i * half)) : 0u;
            sb[i] = ok ? (uint32_t)__ldg(sp + i * sfr) : 0u;
        }
    };
    auto load_dscale = [&](const RqStep& st) {
        const bool ok = 8 * rh < st.nrows;
        const float4* dp = reinterpret_cast<const float4*>(p.dscale + st.row0 + 8 * rh);
        d0 = ok ? dp[0] : make_float4(0.f, 0.f, 0.f, 0.f);
        d1 = ok ? dp[1] : make_float4(0.f, 0.f, 0.f, 0.f);
    };

    RqStep cur;
    if (u < u_end) {
        const int32_t strip = (int32_t)(u / steps);
        const int64_t k = u - (int64_t)strip * steps;
        locate(cur, strip, k, rq_group_of_step(p, k));
        load_codes(cur);   // the rowwise data are read-only for the whole chain
    }

    griddep_wait();
    if (blockIdx.x == 0 && p.absmax) {
        for (int i = threadIdx.x; i < p.nbuf; i += kRqThreads) {
            const float d = __fmul_rn(p.absmax[i], p.decay);
            const float o = p.obs[i];
            p.absmax[i] = d > o ? d : o;
        }
    }
    __syncthreads();   // rcp_tab
    if (u >= u_end) return;
    load_dscale(cur);

    const uint64_t pol_out = l2_evict_first();
    int sc_g = -1, sc_strip = -1;   // (group, strip) whose outer scales sc holds
    float sc[8];
    for (;;) {
        const int64_t c = (int64_t)cur.strip * kRqStripCols + 8 * cg;   // this lane's first column
        const bool cok = c < cols;
        const bool rok = 8 * rh < cur.nrows;
        if (cur.g != sc_g || cur.strip != sc_strip) {
            // outer scales of the lane's eight columns: lane (cg, rh) finds those of columns
            // 2rh and 2rh + 1, the four lanes of cg share them
            sc_g = cur.g;
            sc_strip = cur.strip;
            const uint16_t* cm = p.colmax + (int64_t)cur.g * cols + c;
            const uint32_t a2 = cok ? __ldg(reinterpret_cast<const uint32_t*>(cm) + rh) : 0u;
            const float s_lo = s_enc_of(bf16_lo(a2)), s_hi = s_enc_of(bf16_hi(a2));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                sc[2 * j] = __shfl_sync(0xFFFFFFFFu, s_lo, cg + 8 * j);
                sc[2 * j + 1] = __shfl_sync(0xFFFFFFFFu, s_hi, cg + 8 * j);
            }
            // the group's first step writes the fp32 column amaxes
            if (cok && cur.k == p.step_off[cur.g]) {
                float* ac = p.amax_col + (int64_t)cur.g * cols + c + 2 * rh;
                *reinterpret_cast<float2*>(ac) = make_float2(bf16_lo(a2), bf16_hi(a2));
            }
        }

        // X' of this lane's 8 x 8 elements: x[i][j] = columns 2j, 2j+1 of row 8rh + i
        uint32_t x[8][4];
        {
            const float dm[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) rq_dequant8(cw[i], sb[i], dm[i], x[i]);
        }

        // prefetch the next step
        RqStep nxt = cur;
        const bool more = u + 1 < u_end;
        if (more) {
            advance(cur, nxt);
            load_codes(nxt);
            load_dscale(nxt);
        }

        // block amaxes: this lane's 8 rows, then the partner's 8 (lane ^ 8)
        uint32_t bm[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t t0 = absmax2(x[0][j], x[1][j]);
            const uint32_t t1 = absmax2(x[2][j], x[3][j]);
            uint32_t t2 = absmax2(x[4][j], x[5][j]);
            const uint32_t t3 = absmax2(x[6][j], x[7][j]);
            t0 = absmax2(t0, t1);
            t2 = absmax2(t2, t3);
            t0 = absmax2(t0, t2);
            bm[j] = absmax2(t0, __shfl_xor_sync(0xFFFFFFFFu, t0, 8)) & 0x7FFF7FFFu;
        }
        // block scales: the even lane of a pair takes columns 0-3, the odd one 4-7
        const uint32_t bA = odd ? bm[2] : bm[0], bB = odd ? bm[3] : bm[1];
        const float sA0 = odd ? sc[4] : sc[0], sA1 = odd ? sc[5] : sc[1];
        const float sB0 = odd ? sc[6] : sc[2], sB1 = odd ? sc[7] : sc[3];
        uint32_t sfA, sfB;
        float em[4];
        block_pair_scales_x2(bf16_lo(bA), bf16_hi(bA), sA0, sA1, sfA, em[0], em[1], rcp_tab);
        block_pair_scales_x2(bf16_lo(bB), bf16_hi(bB), sB0, sB1, sfB, em[2], em[3], rcp_tab);
        float ep[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) ep[j] = __shfl_xor_sync(0xFFFFFFFFu, em[j], 8);
        float e[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            e[j] = odd ? ep[j] : em[j];
            e[4 + j] = odd ? em[j] : ep[j];
        }

        if (cok && rok) {
            const int64_t goff = p.row_off[cur.g];
            const int64_t grows = p.row_off[cur.g + 1] - goff;
            const int64_t lrow = cur.row0 - goff + 8 * rh;   // the lane's first row in its group
            uint8_t* qc = p.q_col + cols * goff / 2 + c * (grows / 2) + lrow / 2;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t xs[8] = {x[0][j], x[1][j], x[2][j], x[3][j], x[4][j], x[5][j], x[6][j], x[7][j]};
                stg4_ef(qc + (2 * j) * (grows / 2), encode8_col<false>(xs, e[2 * j]), pol_out);
                stg4_ef(qc + (2 * j + 1) * (grows / 2), encode8_col<true>(xs, e[2 * j + 1]), pol_out);
            }
            // the block's scale bytes of the four columns this lane scaled
            uint8_t* sc_out = p.sf_col + cols * goff / 16 + (c + 4 * odd) * (grows / 16) + lrow / 16;
            const uint32_t sf4 = sfA | (sfB << 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) stg1_ef(sc_out + j * (grows / 16), (sf4 >> (8 * j)) & 0xFFu, pol_out);
        }
        if (!more) break;
        cur = nxt;
        ++u;
    }
}


// ------------------------------------------------------------------ rq_tile
// Both requantization passes again for rows a multiple of 256 wide (each row's scales
// are then whole 16-byte pieces, as TMA needs): a CTA walks tiles of 256 columns x 64
// rows down the matrix, TMA copies stay kRtStages tiles ahead of the warps (the codes,
// the scales and the 64 rows' amaxes), and the warps read shared memory only; each lane
// decodes whole 32-bit words of codes (eight elements of one block of its row).
// ENC = false keeps column maxima (rq_colmax's job): warp w takes rows 8w .. 8w+7 of a
// tile and lane l columns 8l .. 8l+7. ENC = true encodes (rq_colenc's job): warp w takes
// the 16-row block w & 3 and the 128-column half w >> 2, and lanes l and l + 16 take the
// half's columns 8l .. 8l+7, rows 0-7 and 8-15 of the block; the pair joins its block
// maxima by one shuffle, each lane finds the block scales of four of the columns, and the
// pair swaps codes so that each lane leaves four whole 8-byte column segments and their
// scale bytes in a staging tile. After the CTA's barrier each thread writes one column's
// 32 code bytes and 4 scale bytes. Units are (256-column chunk, 64-row step) pairs in
// chunk-major order, the steps of each token group starting at its first row; each CTA
// takes a contiguous run and walks it with a cursor.
constexpr int kRtThreads = 256;
constexpr int kRtCols = 256;
constexpr int kRtRows = 64;
constexpr int kRtStages = 4;
constexpr int kRtCodeBytes = kRtRows * kRtCols / 2;                           // 8192
constexpr int kRtScaleBytes = kRtRows * kRtCols / 16;                         // 1024
constexpr int kRtStageBytes = kRtCodeBytes + kRtScaleBytes + kRtRows * 4;    // + the amaxes: 9472
constexpr int kRtOutCodes = 4 * kRtCols * 8;                                  // [row block][column] 8 bytes
constexpr int kRtOutBytes = kRtOutCodes + 4 * kRtCols;                        // + [row block][column] scale bytes
constexpr int kSmemRqTile = kRtStages * kRtStageBytes + 2 * kRtOutBytes + 128;   // ENC
constexpr int kSmemRqTileMax = kRtStages * kRtStageBytes + 128;                  // !ENC: no staging
constexpr int kRtCtasMax = 4;   // !ENC CTAs per SM (56 registers, 38 KB)
constexpr int kRtCtasEnc = 2;   // ENC CTAs per SM (about 100 registers)

struct RtUnit {
    int64_t chunk;
    int64_t row0;     // first row of the step
    int32_t nrows;    // rows of the step in its group: 16, 32, 48 or 64
    int32_t g;
    bool first;       // the group's first step
};

// A CTA's units are consecutive: a cursor walks them without a division per unit.
struct RtCursor {
    int64_t chunk;
    int64_t k;   // step within the chunk
    int g;       // the group holding step k (empty groups skipped)
};

template <int MAXG>
__device__ __forceinline__ void rt_seek(const RqParams<MAXG>& p, int64_t u, int64_t steps, RtCursor& c)
{
    c.chunk = u / steps;
    c.k = u - c.chunk * steps;
    c.g = 0;
    if (MAXG > 1) {
        int lo = 0, hi = p.num_groups;   // the last group whose first step is <= k
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.tstep_off[mid] <= c.k) lo = mid; else hi = mid;
        }
        c.g = lo;
    }
}

template <int MAXG>
__device__ __forceinline__ void rt_next(const RqParams<MAXG>& p, int64_t steps, RtCursor& c)
{
    if (++c.k == steps) {
        c.k = 0;
        ++c.chunk;
        c.g = 0;
    }
    if (MAXG > 1)
        while (c.g + 1 < p.num_groups && p.tstep_off[c.g + 1] <= c.k) ++c.g;
}

template <int MAXG>
__device__ __forceinline__ RtUnit rt_unit(const RqParams<MAXG>& p, const RtCursor& c)
{
    RtUnit t;
    t.chunk = c.chunk;
    t.g = c.g;
    t.row0 = p.row_off[c.g] + (c.k - p.tstep_off[c.g]) * kRtRows;
    const int64_t left = p.row_off[c.g + 1] - t.row0;
    t.nrows = left < kRtRows ? (int32_t)left : kRtRows;
    t.first = c.k == p.tstep_off[c.g];
    return t;
}

// X' of four elements (codes: 4 nibbles, element i in bits 4i..4i+3) with block scale s2
// (the scale as f16x2, both halves) and decode scale m: two bf16x2 words.
__device__ __forceinline__ void rq_dequant4(uint32_t codes, uint32_t s2, float m, uint32_t& w0, uint32_t& w1)
{
    uint32_t h0, h1;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t}"
        : "=r"(h0), "=r"(h1) : "r"(codes));
    const unsigned long long mm = pack2(m, m);
    uint32_t w[2];
    const uint32_t h[2] = {h0, h1};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        uint32_t t;
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(t) : "r"(h[j]), "r"(s2));   // val * sf: exact
        float lo, hi;
        asm("{\n\t.reg .b16 l, h;\n\t"
            "mov.b32 {l, h}, %2;\n\t"
            "cvt.f32.f16 %0, l;\n\t"
            "cvt.f32.f16 %1, h;\n\t}"
            : "=f"(lo), "=f"(hi) : "r"(t));
        float y0, y1;
        unpack2(mul_f32x2(pack2(lo, hi), mm), y0, y1);
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w[j]) : "f"(y1), "f"(y0));
    }
    w0 = w[0];
    w1 = w[1];
}

template <int MAXG, bool ENC>
__global__ void __launch_bounds__(kRtThreads, ENC ? kRtCtasEnc : kRtCtasMax) rq_tile(const __grid_constant__ RqParams<MAXG> p)
{
    // The kernel after this one may launch early: it waits for this grid itself.
    griddep_launch_dependents();
    extern __shared__ uint8_t rt_raw[];
    __shared__ __align__(8) uint64_t bars[kRtStages];
    __shared__ uint32_t rcp_tab[8];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rt_raw) + 127) & ~uintptr_t(127));
    const uint32_t stage0 = smem_u32(smem);
    const uint32_t bar0 = smem_u32(bars);
    uint8_t* ostage = smem + kRtStages * kRtStageBytes;

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int rb = warp & 3;       // 16-row block of the tile
    const int half = warp >> 2;    // 128-column half of the tile
    const int64_t cols = p.cols;
    const int64_t steps = p.tstep_off[p.num_groups];
    const int64_t total = (cols / kRtCols) * steps;
    const int64_t per = total / gridDim.x, rem = total % gridDim.x;
    const int64_t u0 = (int64_t)blockIdx.x * per + ((int64_t)blockIdx.x < rem ? blockIdx.x : rem);
    const int64_t n = per + ((int64_t)blockIdx.x < rem ? 1 : 0);

    if (ENC) init_rcp_table(rcp_tab);
    if (tid == 0) {
        for (int s = 0; s < kRtStages; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
        prefetch_tensormap(&p.tm_q);
        prefetch_tensormap(&p.tm_sf);
        prefetch_tensormap(&p.tm_amax);
    }
    __syncthreads();
    RtCursor pc;   // thread 0: the next unit to copy
    if (tid == 0 && n > 0) rt_seek(p, u0, steps, pc);
    auto issue = [&](int64_t i) {   // unit u0 + i (the cursor's) into stage i % kRtStages (thread 0)
        const RtUnit t = rt_unit(p, pc);
        rt_next(p, steps, pc);
        const int s = (int)(i % kRtStages);
        const uint32_t bar = bar0 + 8 * s, dst = stage0 + s * kRtStageBytes;
        mbar_arrive_expect_tx(bar, kRtStageBytes);
        tma_load_2d(dst, &p.tm_q, (int32_t)(t.chunk * (kRtCols / 2)), (int32_t)t.row0, bar);
        tma_load_2d(dst + kRtCodeBytes, &p.tm_sf, (int32_t)(t.chunk * (kRtCols / 16)), (int32_t)t.row0, bar);
        tma_load_2d(dst + kRtCodeBytes + kRtScaleBytes, &p.tm_amax, (int32_t)t.row0, 0, bar);
    };
    // the rowwise data are read-only for the whole chain: copy before the wait
    if (tid == 0)
        for (int64_t i = 0; i < n && i < kRtStages; ++i) issue(i);

    griddep_wait();
    if (ENC && blockIdx.x == 0 && p.absmax) {
        for (int i = tid; i < p.nbuf; i += kRtThreads) {
            const float d = __fmul_rn(p.absmax[i], p.decay);
            const float o = p.obs[i];
            p.absmax[i] = d > o ? d : o;
        }
    }
    if (n <= 0) return;   // no barrier follows for a CTA without units

    // !ENC: warp w takes rows 8w .. 8w+7 of the step, lane l columns 8l .. 8l+7 of the chunk.
    // ENC: warp (rb, half) takes the 16-row block rb and the 128-column half; lanes l and
    // l + 16 share columns half*128 + 8(l & 15) .. +7, rows 0-7 and 8-15 of the block.
    const int pl = lane & 15;
    const int sub = lane >> 4;
    const int cl = ENC ? half * 128 + 8 * pl : 8 * lane;   // this lane's first column in the chunk
    uint32_t acc[4] = {0u, 0u, 0u, 0u};     // !ENC: column maxima since the last flush
    int64_t acc_chunk = -1;
    int acc_g = -1;
    float sc[8];                            // ENC: outer scales of the lane's columns
#pragma unroll
    for (int j = 0; j < 8; ++j) sc[j] = 0.f;
    int64_t sc_chunk = -1;
    int sc_g = -1;

    // !ENC: raise colmax and obs with the maxima kept since the last flush
    auto flush = [&]() {
        if (acc_chunk < 0) return;
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] &= 0x7FFF7FFFu;
        if (acc[0] | acc[1] | acc[2] | acc[3])
            red_max_bf16x8(reinterpret_cast<uint32_t*>(p.colmax + (int64_t)acc_g * cols + acc_chunk * kRtCols + cl),
                           acc[0], acc[1], acc[2], acc[3]);
        if (p.obs) {
            uint32_t mx = 0u;
#pragma unroll
            for (int j = 0; j < 4; ++j) mx = max(mx, max(acc[j] & 0xFFFFu, acc[j] >> 16));
            mx = __reduce_max_sync(0xFFFFFFFFu, mx << 16);
            if (lane == 0 && mx) red_max_f32(p.obs + acc_g, mx);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = 0u;
    };

    RtCursor cc;
    rt_seek(p, u0, steps, cc);
    for (int64_t i = 0; i < n; ++i, rt_next(p, steps, cc)) {
        const int s = (int)(i % kRtStages);
        const RtUnit t = rt_unit(p, cc);
        const bool ok = mbar_wait_bounded(bar0 + 8 * s, (uint32_t)((i / kRtStages) & 1));
        const uint8_t* st = smem + s * kRtStageBytes;
        const bool rok = ok && (ENC ? 16 * rb : 8 * warp) < t.nrows;
        uint8_t* os = ostage + (i & 1) * kRtOutBytes;

        if (!ENC && (t.chunk != acc_chunk || t.g != acc_g)) {
            flush();
            acc_chunk = t.chunk;
            acc_g = t.g;
        }
        if (ENC && (t.chunk != sc_chunk || t.g != sc_g)) {
            // outer scales of the lane's eight columns, from the group's column maxima
            sc_chunk = t.chunk;
            sc_g = t.g;
            const int64_t c = t.chunk * kRtCols + cl;
            const uint4 a = *reinterpret_cast<const uint4*>(p.colmax + (int64_t)t.g * cols + c);
            const float a8[8] = {bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y),
                                 bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w)};
#pragma unroll
            for (int j = 0; j < 8; ++j) sc[j] = s_enc_of(a8[j]);
            if (t.first && rb == 0 && sub == 0) {
                float4* d = reinterpret_cast<float4*>(p.amax_col + (int64_t)t.g * cols + c);
                d[0] = make_float4(a8[0], a8[1], a8[2], a8[3]);
                d[1] = make_float4(a8[4], a8[5], a8[6], a8[7]);
            }
        }

        if (rok) {
            const float* amax_st = reinterpret_cast<const float*>(st + kRtCodeBytes + kRtScaleBytes);
            if (!ENC) {
                // decode scales of the warp's 8 rows: lane r finds row r's, the warp shares them
                const float dl = __fdiv_rn(amax_st[8 * warp + (lane & 7)], 2688.0f);
                const uint8_t* cq = st + (8 * warp) * (kRtCols / 2) + 4 * lane;
                const uint8_t* cs = st + kRtCodeBytes + (8 * warp) * (kRtCols / 16) + (lane >> 1);
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const uint32_t codes = *reinterpret_cast<const uint32_t*>(cq + r * (kRtCols / 2));
                    uint32_t x[4];
                    rq_dequant8(codes, cs[r * (kRtCols / 16)], __shfl_sync(0xFFFFFFFFu, dl, r), x);
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[j] = absmax2(acc[j], x[j]);
                }
            } else {
                // decode scales of the block's 16 rows: lanes r and r + 16 find row r's
                const float dl = __fdiv_rn(amax_st[16 * rb + pl], 2688.0f);
                const int r0 = 16 * rb + 8 * sub;   // the lane's first row in the step
                const uint8_t* cq = st + r0 * (kRtCols / 2) + half * 64 + 4 * pl;
                const uint8_t* cs = st + kRtCodeBytes + r0 * (kRtCols / 16) + half * 8 + (pl >> 1);
                uint32_t x[8][4];   // the lane's row r: columns 2j, 2j+1 in word j
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const uint32_t codes = *reinterpret_cast<const uint32_t*>(cq + r * (kRtCols / 2));
                    rq_dequant8(codes, cs[r * (kRtCols / 16)], __shfl_sync(0xFFFFFFFFu, dl, 8 * sub + r), x[r]);
                }
                // block maxima of the eight columns over the block's 16 rows (both lanes)
                uint32_t bm[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t m = absmax2(absmax2(absmax2(x[0][j], x[1][j]), absmax2(x[2][j], x[3][j])),
                                               absmax2(absmax2(x[4][j], x[5][j]), absmax2(x[6][j], x[7][j])));
                    bm[j] = absmax2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16)) & 0x7FFF7FFFu;
                }
                // each lane of the pair finds the scales of four columns (4 * sub ..), and
                // the pair swaps the encode scales
                const uint32_t ba = sub ? bm[2] : bm[0], bb = sub ? bm[3] : bm[1];
                uint32_t sf01, sf23;
                float eo[4];
                block_pair_scales_x2(bf16_lo(ba), bf16_hi(ba), sub ? sc[4] : sc[0], sub ? sc[5] : sc[1], sf01, eo[0],
                                     eo[1], rcp_tab);
                block_pair_scales_x2(bf16_lo(bb), bf16_hi(bb), sub ? sc[6] : sc[2], sub ? sc[7] : sc[3], sf23, eo[2],
                                     eo[3], rcp_tab);
                float e[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float ep = __shfl_xor_sync(0xFFFFFFFFu, eo[k], 16);
                    e[k] = sub ? ep : eo[k];
                    e[4 + k] = sub ? eo[k] : ep;
                }
                uint32_t q[8];   // column k of the lane's eight: the codes of the lane's eight rows
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t c8[8] = {x[0][j], x[1][j], x[2][j], x[3][j], x[4][j], x[5][j], x[6][j], x[7][j]};
                    q[2 * j] = encode8_col<false>(c8, e[2 * j]);
                    q[2 * j + 1] = encode8_col<true>(c8, e[2 * j + 1]);
                }
                // the lane stages columns 4 * sub .. 4 * sub + 3 whole: rows 0-7 and 8-15
                uint32_t lo[4], hi[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t keep = sub ? q[4 + k] : q[k];
                    const uint32_t recv = __shfl_xor_sync(0xFFFFFFFFu, sub ? q[k] : q[4 + k], 16);
                    lo[k] = sub ? recv : keep;
                    hi[k] = sub ? keep : recv;
                }
                const int oc0 = cl + 4 * sub;
                uint4* oc = reinterpret_cast<uint4*>(os + rb * (kRtCols * 8) + oc0 * 8);
                oc[0] = make_uint4(lo[0], hi[0], lo[1], hi[1]);
                oc[1] = make_uint4(lo[2], hi[2], lo[3], hi[3]);
                *reinterpret_cast<uint32_t*>(os + kRtOutCodes + rb * kRtCols + oc0) = sf01 | (sf23 << 16);
            }
        }

        // every warp is done with stage s and has staged its output
        if (__syncthreads_or(!ok)) {
            // give up: record the error, let the copies in flight land (bounded), leave
            if (tid == 0) {
                atomicOr(p.err, kErrTmaTimeout);
                for (int64_t k = i; k < n && k < i + kRtStages; ++k)
                    if (!mbar_wait_bounded(bar0 + 8 * (int)(k % kRtStages), (uint32_t)((k / kRtStages) & 1)))
                        atomicOr(p.err, kErrDrainTimeout);
            }
            __syncthreads();
            return;
        }
        if (tid == 0 && i + kRtStages < n) issue(i + kRtStages);

        if (ENC) {
            // thread tid writes column tid of the chunk: its code bytes and scale bytes of
            // the step's row blocks
            const int nb = t.nrows / 16;
            const int64_t goff = p.row_off[t.g];
            const int64_t grows = p.row_off[t.g + 1] - goff;
            const int64_t lrow = t.row0 - goff;
            const int64_t c = t.chunk * kRtCols + tid;
            uint8_t* qd = p.q_col + cols * goff / 2 + c * (grows / 2) + lrow / 2;
            uint8_t* sd = p.sf_col + cols * goff / 16 + c * (grows / 16) + lrow / 16;
            const uint64_t pol = l2_evict_first();
            uint2 w[4];
            uint32_t sfw = 0u;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                w[b] = *reinterpret_cast<const uint2*>(os + b * (kRtCols * 8) + tid * 8);
                sfw |= (uint32_t)os[kRtOutCodes + b * kRtCols + tid] << (8 * b);
            }
            const uintptr_t qa = reinterpret_cast<uintptr_t>(qd);
            if (nb == 4 && (qa & 31u) == 0) {
                stg32_ef(qd, make_uint4(w[0].x, w[0].y, w[1].x, w[1].y), make_uint4(w[2].x, w[2].y, w[3].x, w[3].y),
                         pol);
            } else if (nb == 4 && (qa & 15u) == 0) {
                stg16_ef(qd, make_uint4(w[0].x, w[0].y, w[1].x, w[1].y), pol);
                stg16_ef(qd + 16, make_uint4(w[2].x, w[2].y, w[3].x, w[3].y), pol);
            } else {
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    if (b < nb) stg8_ef(qd + 8 * b, w[b].x, w[b].y, pol);
            }
            if (nb == 4 && (reinterpret_cast<uintptr_t>(sd) & 3u) == 0) {
                stg4_ef(sd, sfw, pol);
            } else {
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    if (b < nb) stg1_ef(sd + b, (sfw >> (8 * b)) & 0xFFu, pol);
            }
        }
    }
    if (!ENC) flush();
}

}  // namespace nvfp4pt
