// The 16x16 weight cast (sm_100a) in one sweep of the weight: per-row outer amax and
// s_enc, one E4M3 scale per 16x16 block (the largest of the block's 16 per-row scale
// arguments RN(RN(ba/6) * s_enc)), each row encoded with its own RN(s_enc / sf), rowwise
// outputs only (TransformerEngine PR #3045, "transposition-invariant 16x16 cast emitted
// in per-token layout").
//
// Why one kernel: a row's s_enc needs only that row, so a CTA that takes a band of 16
// whole rows (at most 256 KB of bf16) can find its row amaxes and then encode the band.
// The first read brings the band from HBM; the second finds it in L2 (the grid holds
// one band per CTA at a time, a few tens of MB). HBM then moves the weight once and the
// outputs once, where a separate amax pass would read the weight twice.
//
// Layout of the work: thread j of the CTA owns the 16-column block j of every band
// (rows up to 16 x 512 = 8192 elements wide); it keeps its 16 per-row block maxima
// between the reads, so the block scale needs no exchange between threads. Row amaxes
// are joined over the CTA (warp reduction, then shared memory). Loads go four rows at a
// time, two groups in flight.
#pragma once

#include "nvfp4pt_device.cuh"

namespace nvfp4pt {

constexpr int kW2dMaxThreads = 512;   // 16-column blocks per row at most (rows <= 8192 wide)
constexpr int kW2dRows = 16;          // rows of a band

struct W2dParams {
    const uint16_t* w;    // bf16 [rows, cols]
    int64_t bands;        // rows / 16
    int64_t cols;
    int32_t nbc;          // 16-column blocks per row: cols / 16 <= the CTA's threads
    float* amax_row;      // [rows]
    uint8_t* q_row;       // [rows, cols / 2]
    uint8_t* sf_row;      // [rows, cols / 16]
    uint32_t* err;        // the workspace error word: cleared (no wait here can fail)
};

__global__ void __launch_bounds__(kW2dMaxThreads, 1) w2d_band(const __grid_constant__ W2dParams p)
{
    griddep_launch_dependents();
    __shared__ uint32_t part[kW2dRows][kW2dMaxThreads / 32];   // [row][warp] partial amax bits
    __shared__ float srow[kW2dRows];                              // s_enc of the band's rows
    __shared__ uint32_t rcp_tab[8];
    init_rcp_table(rcp_tab);   // first read after the band's barriers

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int nwarps = (int)(blockDim.x >> 5);
    const bool act = tid < p.nbc;
    const int64_t cols = p.cols;
    const uint64_t pol = l2_evict_first();

    // outputs of the previous call on the stream may still be in flight
    griddep_wait();
    if (blockIdx.x == 0 && tid == 0 && p.err) *p.err = 0u;

    for (int64_t band = blockIdx.x; band < p.bands; band += gridDim.x) {
        const uint16_t* src = p.w + band * kW2dRows * cols + 16 * (int64_t)tid;
        auto load4 = [&](uint32_t (&v)[4][8], int r0) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (act) {
                    ldg256_stream(src + (int64_t)(r0 + k) * cols, v[k]);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[k][i] = 0u;
                }
            }
        };

        // first read: the block maximum of each of the 16 rows (bf16 magnitude bits)
        uint32_t bm[kW2dRows];
        auto max4 = [&](const uint32_t (&v)[4][8], int r0) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t* x = v[k];
                uint32_t m = absmax2(absmax2(absmax2(x[0], x[1]), absmax2(x[2], x[3])),
                                     absmax2(absmax2(x[4], x[5]), absmax2(x[6], x[7])));
                m &= 0x7FFF7FFFu;
                bm[r0 + k] = (m & 0xFFFFu) > (m >> 16) ? (m & 0xFFFFu) : (m >> 16);
            }
        };
        {
            uint32_t a[4][8], b[4][8];
            load4(a, 0);
            load4(b, 4);
            max4(a, 0);
            load4(a, 8);
            max4(b, 4);
            load4(b, 12);
            max4(a, 8);
            max4(b, 12);
        }
#pragma unroll
        for (int i = 0; i < kW2dRows; ++i) {
            const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, bm[i]);
            if (lane == 0) part[i][warp] = m;
        }
        __syncthreads();
        if (tid < kW2dRows) {
            uint32_t m = 0u;
            for (int w = 0; w < nwarps; ++w) m = part[tid][w] > m ? part[tid][w] : m;
            const float a = __uint_as_float(m << 16);
            p.amax_row[band * kW2dRows + tid] = a;
            srow[tid] = s_enc_of(a);
        }
        __syncthreads();

        // the block's scale: the largest per-row argument; each row's multiplier
        float e[kW2dRows];
        uint32_t sf = 0u;
        {
            float u = 0.0f;
#pragma unroll
            for (int i = 0; i < kW2dRows; ++i) u = fmaxf(u, __fmul_rn(div6(__uint_as_float(bm[i] << 16)), srow[i]));
            sf = e4m3x2(u, u) & 0xFFu;
            float d, d_unused;
            e4m3x2_decode(sf, d, d_unused);
#pragma unroll
            for (int i = 0; i < kW2dRows; ++i) e[i] = enc_of(sf, d, srow[i], rcp_tab);
        }

        // second read (from L2): the codes of each row, and the block's scale byte
        const int64_t row0 = band * kW2dRows;
        auto enc4 = [&](const uint32_t (&v)[4][8], int r0) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (!act) continue;
                const int64_t row = row0 + r0 + k;
                const uint32_t* x = v[k];
                const uint32_t q0 = encode8(x[0], x[1], x[2], x[3], e[r0 + k]);
                const uint32_t q1 = encode8(x[4], x[5], x[6], x[7], e[r0 + k]);
                stg8_ef(p.q_row + row * (cols / 2) + 8 * (int64_t)tid, q0, q1, pol);
                stg1_ef(p.sf_row + row * (cols / 16) + tid, sf, pol);
            }
        };
        {
            uint32_t a[4][8], b[4][8];
            load4(a, 0);
            load4(b, 4);
            enc4(a, 0);
            load4(a, 8);
            enc4(b, 4);
            load4(b, 12);
            enc4(a, 8);
            enc4(b, 12);
        }
    }
}

}  // namespace nvfp4pt
