// Row pass of the NVFP4 per-token cast (sm_100a): one read of x gives the per-row
// amax, the complete rowwise encode (codes + E4M3 scales) and the per-column amax
// (per token group). The columnwise encode follows in the column pass (colpass).
//
// Why here: a row's outer amax needs only that row, so a CTA that holds whole rows
// can encode them as soon as its own reduction ends, from registers. That moves
// half of the encode arithmetic into the pass that is otherwise only streaming,
// leaving each of the two passes bound by HBM alone.
//
// Layout of the work: a "sweep" is `rps` whole rows covered once by the CTA's 512
// threads (tpr threads per row, a multiple of 32, each holding BT 16-element blocks
// of its row); a "batch" is S sweeps. A CTA prefetches the next batch (one 256-bit
// load per block) while it reduces and encodes the current one. A batch has S * rps
// rows, a divisor of 16, so it never straddles a token group (group offsets are
// multiples of 16).
//
// Order of the batches: with one token group the CTAs take batches c, c + num_ctas,
// ... so that the grid sweeps x from top to bottom as one front, and the bottom of x
// is what L2 holds when the column pass starts there. With several groups a CTA owns
// a contiguous run of batches instead, so that its column partials change group (and
// go out to amax_col) about once per group rather than once per batch.
#pragma once

#include "nvfp4pt_device.cuh"

namespace nvfp4pt {

constexpr int kRowThreads = 512;   // one CTA per SM: 128 registers per thread

template <int MAXG>
struct RowParams {
    int64_t rows;
    int64_t cols;
    int64_t num_batches;
    int32_t bpr;         // 16-element blocks per row
    int32_t tpr;         // threads per row (multiple of 32, <= 512)
    int32_t rps;         // rows per sweep (power of two, <= 16)
    int32_t num_ctas;
    int32_t num_groups;
    int32_t do_row;      // write rowwise codes and scales
    int32_t strided;     // batches c, c + num_ctas, ... (else a contiguous run per CTA)
    const uint16_t* x;
    float* amax_row;     // [rows], written directly (not accumulated)
    uint8_t* q_row;
    uint8_t* sf_row;
    float* amax_col;     // [G, cols] accumulated with atomic max, or null (used when colmax is null)
    uint32_t* colmax;    // [G, cols] bf16 column maxima accumulated with 8-wide atomic max, or null
    float* obs;          // [G] accumulated with atomic max, or null
    int32_t row_off[MAXG + 1];
};

template <int MAXG>
__device__ __forceinline__ int group_of_row(const RowParams<MAXG>& p, int64_t row)
{
    if (MAXG == 1) return 0;
    int lo = 0, hi = p.num_groups;  // row_off[lo] <= row < row_off[hi]; empty groups skipped
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)p.row_off[mid] <= row) lo = mid; else hi = mid;
    }
    return lo;
}

// Encode two blocks (8 bf16 words each) with block amaxes ba, bb (binary32) and outer
// scales sa, sb: two words of codes per block and the two scale bytes (a in bits 0-7).
__device__ __forceinline__ void encode_block_pair(const uint32_t (&a)[8], const uint32_t (&b)[8], float ba, float bb,
                                                  float sa, float sb, uint32_t& qa0, uint32_t& qa1, uint32_t& qb0,
                                                  uint32_t& qb1, uint32_t& sf, const uint32_t* tab)
{
    float ea, eb;
    block_pair_scales(ba, bb, sa, sb, sf, ea, eb, tab);
    qa0 = encode8(a[0], a[1], a[2], a[3], ea);
    qa1 = encode8(a[4], a[5], a[6], a[7], ea);
    qb0 = encode8(b[0], b[1], b[2], b[3], eb);
    qb1 = encode8(b[4], b[5], b[6], b[7], eb);
}

template <int MAXG, int BT, int S>
__global__ void __launch_bounds__(kRowThreads, 1) rowpass(const __grid_constant__ RowParams<MAXG> p)
{
    griddep_launch_dependents();
    __shared__ uint32_t part[S * 16][kRowThreads / 32];   // [row of batch][warp of row] partial amax bits
    __shared__ float srow[S * 16];            // outer scale of each row of the batch
    __shared__ uint32_t rcp_tab[8];           // E4M3 significand reciprocals
    init_rcp_table(rcp_tab);                  // first read after the batch barriers

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int rsw = tid / p.tpr;              // row within the sweep
    const int tj = tid - rsw * p.tpr;         // position within the row
    const bool active = rsw < p.rps;
    const int wpr = p.tpr >> 5;               // warps per row
    const int rows_per_batch = S * p.rps;
    const int64_t cols = p.cols;

    const int64_t nb = p.num_batches;
    int64_t b0, bstep, nbat;   // this CTA's batches: b0 + k * bstep, k < nbat
    if (p.strided) {
        b0 = blockIdx.x;
        bstep = p.num_ctas;
        nbat = b0 < nb ? (nb - 1 - b0) / bstep + 1 : 0;
    } else {
        b0 = (nb * blockIdx.x) / p.num_ctas;
        bstep = 1;
        nbat = (nb * (blockIdx.x + 1)) / p.num_ctas - b0;
    }
    if (nbat <= 0) return;

    bool valid[BT];
    int bj[BT];
#pragma unroll
    for (int b = 0; b < BT; ++b) {
        bj[b] = tj + p.tpr * b;
        valid[b] = active && bj[b] < p.bpr;
    }

    uint32_t va[S][BT][8];
    uint32_t vb[S][BT][8];
    const uint64_t pol_out = l2_evict_first();   // row outputs: not read again
    auto load = [&](int64_t batch, uint32_t (&v)[S][BT][8]) {
        const int64_t r0 = batch * rows_per_batch;
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const int64_t row = r0 + s * p.rps + rsw;
#pragma unroll
            for (int b = 0; b < BT; ++b) {
                if (valid[b]) {
                    ldg256_stream(p.x + row * cols + 16 * (int64_t)bj[b], v[s][b]);
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) v[s][b][k] = 0u;
                }
            }
        }
    };

    uint32_t colacc[BT][8];
#pragma unroll
    for (int b = 0; b < BT; ++b)
#pragma unroll
        for (int k = 0; k < 8; ++k) colacc[b][k] = 0u;
    uint32_t obsacc = 0u;   // lanes 0 of the row-reducing warps
    bool waited = false;

    auto flush = [&](int g) {
        if (!waited) { griddep_wait(); waited = true; }
        if (p.colmax) {
#pragma unroll
            for (int b = 0; b < BT; ++b) {
                if (!valid[b]) continue;
                uint32_t* dst = p.colmax + ((int64_t)g * cols + 16 * (int64_t)bj[b]) / 2;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t w0 = colacc[b][4 * h] & 0x7FFF7FFFu, w1 = colacc[b][4 * h + 1] & 0x7FFF7FFFu;
                    const uint32_t w2 = colacc[b][4 * h + 2] & 0x7FFF7FFFu, w3 = colacc[b][4 * h + 3] & 0x7FFF7FFFu;
                    if (w0 | w1 | w2 | w3) red_max_bf16x8(dst + 4 * h, w0, w1, w2, w3);
                }
#pragma unroll
                for (int k = 0; k < 8; ++k) colacc[b][k] = 0u;
            }
        } else if (p.amax_col) {
#pragma unroll
            for (int b = 0; b < BT; ++b) {
                if (!valid[b]) continue;
                float* dst = p.amax_col + (int64_t)g * cols + 16 * (int64_t)bj[b];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t w = colacc[b][k] & 0x7FFF7FFFu;
                    if (w & 0xFFFFu) red_max_f32(dst + 2 * k, w << 16);
                    if (w >> 16) red_max_f32(dst + 2 * k + 1, w & 0xFFFF0000u);
                    colacc[b][k] = 0u;
                }
            }
        }
        if (p.obs && obsacc) red_max_f32(p.obs + g, obsacc << 16);
        obsacc = 0u;
    };

    int g_cur = group_of_row(p, b0 * rows_per_batch);
    auto process = [&](int64_t batch, bool more, uint32_t (&cur)[S][BT][8], uint32_t (&nxt)[S][BT][8]) {
        if (more) load(batch + bstep, nxt);
        const int64_t r0 = batch * rows_per_batch;

        // block amaxes (kept for the encode), row partials (one per warp and row),
        // column partials
        uint32_t bmax[S][BT];
#pragma unroll
        for (int s = 0; s < S; ++s) {
            uint32_t m = 0u;
#pragma unroll
            for (int b = 0; b < BT; ++b) {
                const uint32_t* v = cur[s][b];
                bmax[s][b] = absmax2(absmax2(absmax2(v[0], v[1]), absmax2(v[2], v[3])),
                                     absmax2(absmax2(v[4], v[5]), absmax2(v[6], v[7])));
                m = absmax2(m, bmax[s][b]);
#pragma unroll
                for (int k = 0; k < 8; ++k) colacc[b][k] = absmax2(colacc[b][k], v[k]);
            }
            m &= 0x7FFF7FFFu;
            m = (m & 0xFFFFu) > (m >> 16) ? (m & 0xFFFFu) : (m >> 16);
            m = __reduce_max_sync(0xFFFFFFFFu, m);
            if (lane == 0 && active) part[s * p.rps + rsw][warp - rsw * wpr] = m;
        }
        __syncthreads();
        // one warp per row of the batch finishes its amax and outer scale
        if (warp < rows_per_batch) {
            uint32_t m = lane < wpr ? part[warp][lane] : 0u;
            m = __reduce_max_sync(0xFFFFFFFFu, m);
            if (lane == 0) {
                const float a = __uint_as_float(m << 16);
                if (p.amax_row) p.amax_row[r0 + warp] = a;
                srow[warp] = s_enc_of(a);
                obsacc = m > obsacc ? m : obsacc;
            }
        }
        __syncthreads();

        if (p.do_row) {
            float sv[S];
#pragma unroll
            for (int s = 0; s < S; ++s) sv[s] = srow[s * p.rps + rsw];
            // blocks in pairs: (s, b) enumerated s-major
#pragma unroll
            for (int i = 0; i < S * BT; i += 2) {
                const int sa = i / BT, ba = i % BT;
                const int sb = (i + 1 < S * BT) ? (i + 1) / BT : sa;
                const int bb = (i + 1 < S * BT) ? (i + 1) % BT : ba;
                uint32_t qa0, qa1, qb0, qb1, sf;
                encode_block_pair(cur[sa][ba], cur[sb][bb], absmax_of_pair(bmax[sa][ba]), absmax_of_pair(bmax[sb][bb]),
                                  sv[sa], sv[sb], qa0, qa1, qb0, qb1, sf, rcp_tab);
                if (valid[ba]) {
                    const int64_t row = r0 + sa * p.rps + rsw;
                    stg8_ef(p.q_row + row * (cols / 2) + 8 * (int64_t)bj[ba], qa0, qa1, pol_out);
                    stg1_ef(p.sf_row + row * (cols / 16) + bj[ba], sf & 0xFFu, pol_out);
                }
                if (i + 1 < S * BT && valid[bb]) {
                    const int64_t row = r0 + sb * p.rps + rsw;
                    stg8_ef(p.q_row + row * (cols / 2) + 8 * (int64_t)bj[bb], qb0, qb1, pol_out);
                    stg1_ef(p.sf_row + row * (cols / 16) + bj[bb], (sf >> 8) & 0xFFu, pol_out);
                }
            }
        }

        // the column partials belong to the batch's token group
        const int g_next = more ? group_of_row(p, (batch + bstep) * rows_per_batch) : -1;
        if (g_next != g_cur) {
            flush(g_cur);
            g_cur = g_next;
        }
    };

    // the next batch loads into vb while va is reduced and encoded, then moves over
    load(b0, va);
    for (int64_t k = 0; k < nbat; ++k) {
        process(b0 + k * bstep, k + 1 < nbat, va, vb);
#pragma unroll
        for (int s = 0; s < S; ++s)
#pragma unroll
            for (int b = 0; b < BT; ++b)
#pragma unroll
                for (int i = 0; i < 8; ++i) va[s][b][i] = vb[s][b][i];
    }
}

}  // namespace nvfp4pt
