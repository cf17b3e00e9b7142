// Kernels of the NVFP4 per-token cast (sm_100a) shared by every route, and the tile
// path (the 16x16 weight cast and rows wider than 16384 elements; the 1D casts of
// narrower rows run the row pass and the column pass of nvfp4pt_rowpass.cuh and
// nvfp4pt_colpass.cuh instead).
//
//   pass0_zero   zeroes the amax outputs and the per-call scratch (the maxima are
//                accumulated with atomic max on non-negative float or bf16 bits).
//   pass1_amax   the vector-amax stage of TransformerEngine PR #3045 (its "K1"): one
//                read of x gives the per-row amax, the per-column amax (per token
//                group when grouped) and the observed maximum of the running buffer.
//   pass2_encode the encode stage ("K2"): 128 x 128 tiles staged by TMA into shared
//                memory; rowwise codes/scales and transposed columnwise codes/scales
//                come from the same tile; the first CTA also applies the decayed
//                absmax update of PR #3296.
//   update_absmax_kernel  the buffer step alone.
#pragma once

#include "nvfp4pt_device.cuh"

namespace nvfp4pt {

// ===================================================================== pass 0

struct ZeroParams {
    float4* ptr[4];
    int64_t n4[4];     // float4 count of each range
    uint32_t* err;     // error word to clear (may be null)
};

// Launched as a programmatic dependent of whatever precedes the cast on the stream: it
// waits for that grid (and its memory) before anything else, and only then lets the
// cast's next kernel start, which reads x without waiting itself.
__global__ void __launch_bounds__(kThreads) pass0_zero(const __grid_constant__ ZeroParams p)
{
    griddep_wait();
    griddep_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float4* d = p.ptr[k];
        if (!d) continue;
        for (int64_t i = i0; i < p.n4[k]; i += stride) d[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (i0 == 0 && p.err) *p.err = 0u;
}

// ===================================================================== pass 1

template <int MAXG>
struct P1Params {
    Geometry geo;
    const uint16_t* x;
    float* amax_row;   // [rows] or null
    float* amax_col;   // [G, cols] or null
    float* obs;        // [G] observed maxima, or null
    Groups<MAXG> grp;
};

// Thread layout over a 128 x 128 tile (128 rows of 256 bytes): lane & 15 picks the
// 16-byte chunk (8 columns) of a row, and each warp covers 2 rows per instruction
// (512 contiguous bytes); a thread reads rows rs, rs+16, ..., rs+112.
template <int MAXG, bool DO_COL>
__global__ void __launch_bounds__(kThreads, 2) pass1_amax(const __grid_constant__ P1Params<MAXG> p)
{
    griddep_launch_dependents();
    __shared__ uint32_t colpart[2][8][64];   // [buffer][warp][column pair]

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int j = lane & 15;
    const int rs = 2 * warp + (lane >> 4);
    const int64_t cols = p.geo.cols;

    int64_t t0, t1;
    cta_tile_range(p.geo, blockIdx.x, t0, t1);
    if (t0 >= t1) return;

    bool waited = false;
    uint32_t rowacc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) rowacc[i] = 0u;

    TileInfo cur = tile_info(p.geo, p.grp, t0);
    TileInfo nxt = cur;
    uint4 vn[8];
    auto load_tile = [&](const TileInfo& ti, uint4* v) {
        const bool cok = 8 * j < ti.nc;
        const uint16_t* base = p.x + (ti.r0 + rs) * cols + ti.c0 + 8 * j;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (cok && rs + 16 * i < ti.nr) v[i] = ldg_stream(base + (int64_t)16 * i * cols);
            else v[i] = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    // Row amaxes of the band held in rowacc go out once per band segment.
    auto flush_rows = [&](const TileInfo& ti) {
        if (!waited) { griddep_wait(); waited = true; }
        uint32_t bandmax = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w = rowacc[i] & 0x7FFF7FFFu;
            uint32_t m = (w & 0xFFFFu) > (w >> 16) ? (w & 0xFFFFu) : (w >> 16);
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) {
                const uint32_t q = __shfl_xor_sync(0xFFFFFFFFu, m, o);
                m = q > m ? q : m;
            }
            if (rs + 16 * i < ti.nr) bandmax = m > bandmax ? m : bandmax;
            if (j == 0 && p.amax_row && rs + 16 * i < ti.nr) red_max_f32(p.amax_row + ti.r0 + rs + 16 * i, m << 16);
            rowacc[i] = 0u;
        }
        bandmax = __reduce_max_sync(0xFFFFFFFFu, bandmax);
        if (lane == 0 && p.obs && bandmax) red_max_f32(p.obs + ti.g, bandmax << 16);
    };

    load_tile(cur, vn);
    int buf = 0;
    for (int64_t t = t0; t < t1; ++t) {
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = vn[i];
        cur = nxt;
        if (t + 1 < t1) {
            nxt = tile_info(p.geo, p.grp, t + 1);
            load_tile(nxt, vn);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
            rowacc[i] = absmax2(rowacc[i], absmax2(absmax2(v[i].x, v[i].y), absmax2(v[i].z, v[i].w)));
        if (DO_COL) {
            uint32_t c0 = v[0].x, c1 = v[0].y, c2 = v[0].z, c3 = v[0].w;
#pragma unroll
            for (int i = 1; i < 8; ++i) {
                c0 = absmax2(c0, v[i].x); c1 = absmax2(c1, v[i].y);
                c2 = absmax2(c2, v[i].z); c3 = absmax2(c3, v[i].w);
            }
            c0 = absmax2(c0, __shfl_xor_sync(0xFFFFFFFFu, c0, 16));
            c1 = absmax2(c1, __shfl_xor_sync(0xFFFFFFFFu, c1, 16));
            c2 = absmax2(c2, __shfl_xor_sync(0xFFFFFFFFu, c2, 16));
            c3 = absmax2(c3, __shfl_xor_sync(0xFFFFFFFFu, c3, 16));
            if (lane < 16) *reinterpret_cast<uint4*>(&colpart[buf][warp][4 * j]) = make_uint4(c0, c1, c2, c3);
            __syncthreads();
            if (tid < kTile) {
                uint32_t m = colpart[buf][0][tid >> 1];
#pragma unroll
                for (int w8 = 1; w8 < 8; ++w8) m = absmax2(m, colpart[buf][w8][tid >> 1]);
                const uint32_t bits = (tid & 1) ? (m & 0x7FFF0000u) : ((m & 0x7FFFu) << 16);
                if (!waited) { griddep_wait(); waited = true; }
                if (tid < cur.nc && bits) red_max_f32(p.amax_col + (int64_t)cur.g * cols + cur.c0 + tid, bits);
            }
            buf ^= 1;
        }
        const bool band_ends = (t + 1 == t1) || (nxt.band != cur.band);
        if (band_ends) flush_rows(cur);
    }
}

// ===================================================================== pass 2

template <int MAXG>
struct P2Params {
    CUtensorMap tmap;        // x as [rows, cols] bf16, 128 x 64 boxes, 128-byte swizzle
    Geometry geo;
    const float* amax_row;   // [rows]
    const float* amax_col;   // [G, cols] or null
    uint8_t* q_row;
    uint8_t* sf_row;
    uint8_t* q_col;
    uint8_t* sf_col;
    float* absmax;           // [nbuf] running buffers, or null
    const float* obs;        // [nbuf] observed maxima (from pass 1)
    uint32_t* err;           // device error word
    float decay;
    int32_t nbuf;
    int32_t flags;           // 1 rowwise, 2 columnwise
    int32_t pad_;
    Groups<MAXG> grp;
};

// staging of one tile's columnwise outputs: codes [128 columns][64 B], scales [128][8 B]
constexpr int kColCodeBytes = kTile * 64;
constexpr int kColScaleBytes = kTile * 8;
constexpr int kSmemPass2 = kStages * kStageBytes + kColCodeBytes + kColScaleBytes + 2 * kTile * 4 + kStages * 8 + 1024;

// Rowwise encode of one half-row (64 columns = 4 blocks) of the tile in `box`.
// Thread: row r of the tile, half h. W2D: the 16 rows of a band (16 consecutive
// lanes) share one scale per block (the largest of their 1D scale arguments).
template <bool W2D>
__device__ __forceinline__ void encode_rows(uint32_t box, int r, float s, uint32_t out[8], uint32_t& sf4,
                                            const uint32_t* tab)
{
    uint32_t w[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 q = lds128(box + swz128(r, c));
        w[4 * c] = q.x; w[4 * c + 1] = q.y; w[4 * c + 2] = q.z; w[4 * c + 3] = q.w;
    }
    float ba[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t* x = w + 8 * b;
        const uint32_t m = absmax2(absmax2(absmax2(x[0], x[1]), absmax2(x[2], x[3])),
                                   absmax2(absmax2(x[4], x[5]), absmax2(x[6], x[7])));
        ba[b] = absmax_of_pair(m);
    }
    float e[4];
    uint32_t sf01, sf23;
    if (!W2D) {
        block_pair_scales(ba[0], ba[1], s, s, sf01, e[0], e[1], tab);
        block_pair_scales(ba[2], ba[3], s, s, sf23, e[2], e[3], tab);
    } else {
        float u[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            u[b] = __fmul_rn(div6(ba[b]), s);
#pragma unroll
            for (int o = 1; o <= 8; o <<= 1) u[b] = fmaxf(u[b], __shfl_xor_sync(0xFFFFFFFFu, u[b], o));
        }
        sf01 = e4m3x2(u[0], u[1]);
        sf23 = e4m3x2(u[2], u[3]);
        float d0, d1, d2, d3;
        e4m3x2_decode(sf01, d0, d1);
        e4m3x2_decode(sf23, d2, d3);
        e[0] = enc_of(sf01, d0, s, tab);
        e[1] = enc_of(sf01 >> 8, d1, s, tab);
        e[2] = enc_of(sf23, d2, s, tab);
        e[3] = enc_of(sf23 >> 8, d3, s, tab);
    }
    sf4 = (sf01 & 0xFFFFu) | (sf23 << 16);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t* x = w + 8 * b;
        out[2 * b] = encode8(x[0], x[1], x[2], x[3], e[b]);
        out[2 * b + 1] = encode8(x[4], x[5], x[6], x[7], e[b]);
    }
}

// Columnwise encode of a column pair (2p, 2p+1) over 32 rows (2 blocks) of the tile.
// v[i] holds row 32*hb+i of both columns (low half = column 2p).
__device__ __forceinline__ void encode_cols(uint32_t box, int p, int hb, float s0, float s1,
                                            uint32_t out0[4], uint32_t out1[4], uint32_t& sf, const uint32_t* tab)
{
    uint32_t v[32];
    const int chunk = (p & 31) >> 2;
    const uint32_t sub = (uint32_t)(p & 3) * 4u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int row = 32 * hb + i;
        v[i] = lds32(box + swz128(row, chunk) + sub);
    }
    uint32_t m[2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        const uint32_t* x = v + 16 * b;
        uint32_t a0 = absmax2(absmax2(x[0], x[1]), absmax2(x[2], x[3]));
        uint32_t a1 = absmax2(absmax2(x[4], x[5]), absmax2(x[6], x[7]));
        uint32_t a2 = absmax2(absmax2(x[8], x[9]), absmax2(x[10], x[11]));
        uint32_t a3 = absmax2(absmax2(x[12], x[13]), absmax2(x[14], x[15]));
        m[b] = absmax2(absmax2(a0, a1), absmax2(a2, a3)) & 0x7FFF7FFFu;
    }
    // block amaxes: [block][column]
    const float b00 = __uint_as_float(m[0] << 16), b01 = __uint_as_float(m[0] & 0xFFFF0000u);
    const float b10 = __uint_as_float(m[1] << 16), b11 = __uint_as_float(m[1] & 0xFFFF0000u);
    uint32_t sfc0, sfc1;   // column 0: blocks 0,1 ; column 1: blocks 0,1
    float e00, e10, e01, e11;
    block_pair_scales(b00, b10, s0, s0, sfc0, e00, e10, tab);
    block_pair_scales(b01, b11, s1, s1, sfc1, e01, e11, tab);
    sf = (sfc0 & 0xFFFFu) | (sfc1 << 16);
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        const uint32_t* x = v + 16 * b;
        const float ea = b ? e10 : e00;
        const float eb = b ? e11 : e01;
        // column 2p: low halves of rows 16b..16b+15, two per byte (row 2j low nibble)
        out0[2 * b] = encode8_col<false>(x, ea);
        out0[2 * b + 1] = encode8_col<false>(x + 8, ea);
        out1[2 * b] = encode8_col<true>(x, eb);
        out1[2 * b + 1] = encode8_col<true>(x + 8, eb);
    }
}

template <int MAXG, bool W2D>
__global__ void __launch_bounds__(kThreads, 2) pass2_encode(const __grid_constant__ P2Params<MAXG> p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ccode = smem + kStages * kStageBytes;           // staged column codes
    uint8_t* cscale = ccode + kColCodeBytes;                  // staged column scales
    float* srow = reinterpret_cast<float*>(cscale + kColScaleBytes);
    float* scol = srow + kTile;
    uint64_t* bars = reinterpret_cast<uint64_t*>(scol + kTile);
    const uint32_t stage0 = smem_u32(smem);
    const uint32_t bar0 = smem_u32(bars);
    __shared__ uint32_t rcp_tab[8];
    init_rcp_table(rcp_tab);

    const int tid = threadIdx.x;
    const int64_t cols = p.geo.cols;
    const bool do_row = (p.flags & 1) != 0;
    const bool do_col = !W2D && (p.flags & 2) != 0;

    int64_t last, step;
    const int64_t n = (do_row || do_col) ? cta_reverse_tiles(p.geo, blockIdx.x, last, step) : 0;

    if (tid == 0) {
        prefetch_tensormap(&p.tmap);
        for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // Tiles go backwards: the k-th tile of this CTA is last - k * step. Thread 0 walks
    // the issued tiles (kStages ahead of the encoded ones) with its own walker.
    TileWalker<MAXG> iw;
    int64_t issued = 0;
    auto issue_next = [&]() {
        if (issued > 0) iw.back(p.geo, p.grp, (int32_t)step);
        const int s = (int)(issued % kStages);
        const uint32_t bar = bar0 + 8 * s;
        const uint32_t dst = stage0 + s * kStageBytes;
        mbar_arrive_expect_tx(bar, kStageBytes);
        tma_load_2d(dst, &p.tmap, (int32_t)iw.ti.c0, (int32_t)iw.ti.r0, bar);
        tma_load_2d(dst + kBoxBytes, &p.tmap, (int32_t)iw.ti.c0 + 64, (int32_t)iw.ti.r0, bar);
        ++issued;
    };
    // x is read-only for the whole chain, so the first tiles load before pass 1 ends.
    if (tid == 0 && n > 0) {
        iw.start(p.geo, p.grp, last);
        for (int64_t k = 0; k < n && k < kStages; ++k) issue_next();
    }

    griddep_wait();
    if (blockIdx.x == 0 && p.absmax) {
        for (int g = tid; g < p.nbuf; g += kThreads) {
            const float d = __fmul_rn(p.absmax[g], p.decay);
            const float o = p.obs[g];
            p.absmax[g] = d > o ? d : o;
        }
    }
    if (n <= 0) return;

    // amax of the rows (threads 0..127) or columns (128..255) of a tile
    auto fetch_amax = [&](const TileInfo& ti) -> float {
        if (tid < kTile) {
            return (do_row && tid < ti.nr) ? p.amax_row[ti.r0 + tid] : 0.0f;
        }
        const int c = tid - kTile;
        return (do_col && c < ti.nc) ? p.amax_col[(int64_t)ti.g * cols + ti.c0 + c] : 0.0f;
    };

    TileWalker<MAXG> w;
    w.start(p.geo, p.grp, last);
    float a_next = fetch_amax(w.ti);
    int s = 0;
    uint32_t parity = 0;
    for (int64_t k = 0; k < n; ++k) {
        const TileInfo cur = w.ti;
        // outer scales of this tile's rows and columns
        const float sv = s_enc_of(a_next);
        if (tid < kTile) srow[tid] = sv; else scol[tid - kTile] = sv;
        if (k + 1 < n) {
            w.back(p.geo, p.grp, (int32_t)step);
            a_next = fetch_amax(w.ti);
        }
        __syncthreads();

        const bool ok = mbar_wait_bounded(bar0 + 8 * s, parity);
        const uint32_t stage = stage0 + s * kStageBytes;
        if (ok) {
            if (do_row) {
                const int r = tid & (kTile - 1);
                const int h = tid >> 7;
                uint32_t out[8], sf4;
                encode_rows<W2D>(stage + h * kBoxBytes, r, srow[r], out, sf4, rcp_tab);
                const int nb = min(4, max(0, (cur.nc - 64 * h) / 16));
                if (r < cur.nr && nb > 0) {
                    const int64_t row = cur.r0 + r;
                    uint8_t* q = p.q_row + row * (cols / 2) + cur.c0 / 2 + 32 * h;
                    uint8_t* sfp = p.sf_row + row * (cols / 16) + cur.c0 / 16 + 4 * h;
                    if (nb == 4) {
                        stg16(q, out[0], out[1], out[2], out[3]);
                        stg16(q + 16, out[4], out[5], out[6], out[7]);
                    } else {
                        for (int b = 0; b < nb; ++b) stg8(q + 8 * b, out[2 * b], out[2 * b + 1]);
                    }
                    stg_bytes(sfp, sf4, nb);
                }
            }
            if (do_col) {
                const int pc = tid & 63;   // column pair
                const int hb = tid >> 6;   // 32-row quarter
                uint32_t o0[4], o1[4], sf;
                encode_cols(stage + (pc >> 5) * kBoxBytes, pc, hb, scol[2 * pc], scol[2 * pc + 1], o0, o1, sf,
                            rcp_tab);
                // stage: column c's 64 code bytes hold 16-byte chunk q at slot q ^ ((c >> 1) & 3)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int col = 2 * pc + c;
                    const uint32_t* o = c ? o1 : o0;
                    *reinterpret_cast<uint4*>(ccode + col * 64 + 16 * (hb ^ ((col >> 1) & 3))) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint16_t*>(cscale + col * 8 + 2 * hb) = (uint16_t)(c ? (sf >> 16) : sf);
                }
            }
        }
        const int failed = __syncthreads_or(!ok);
        if (!failed && do_col) {
            // write-back from the staging area: 64 contiguous code bytes and 8 scale bytes
            // per column of the tile
            const int64_t lrow = cur.r0 - cur.goff;            // first row inside the group
            const int64_t qstride = cur.grows / 2, sstride = cur.grows / 16;
            uint8_t* qtile = p.q_col + cols * (int64_t)cur.goff / 2 + lrow / 2 + cur.c0 * qstride;
            uint8_t* stile = p.sf_col + cols * (int64_t)cur.goff / 16 + lrow / 16 + cur.c0 * sstride;
            const bool full = cur.nr == kTile && cur.nc == kTile;
            if (full && ((reinterpret_cast<uintptr_t>(qtile) | (uintptr_t)qstride) & 31u) == 0) {
                // one 32-byte half-column per thread
                const int col = tid >> 1, h = tid & 1, sw = (col >> 1) & 3;
                const uint8_t* src = ccode + col * 64;
                const uint4 a = *reinterpret_cast<const uint4*>(src + 16 * ((2 * h) ^ sw));
                const uint4 b = *reinterpret_cast<const uint4*>(src + 16 * ((2 * h + 1) ^ sw));
                stg32(qtile + (int64_t)col * qstride + 32 * h, a, b);
            } else {
                const int qbytes = cur.nr / 2;                  // code bytes of this tile per column
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int i = tid + kThreads * j;
                    const int col = i >> 2, q = i & 3;
                    if (col < cur.nc && 16 * q < qbytes) {
                        const uint4 v = *reinterpret_cast<const uint4*>(ccode + col * 64 + 16 * (q ^ ((col >> 1) & 3)));
                        uint8_t* dst = qtile + (int64_t)col * qstride + 16 * q;
                        if (16 * q + 16 <= qbytes) stg16(dst, v.x, v.y, v.z, v.w);
                        else stg8(dst, v.x, v.y);
                    }
                }
            }
            if (tid < cur.nc) {
                const uint2 v = *reinterpret_cast<const uint2*>(cscale + tid * 8);
                uint8_t* dst = stile + (int64_t)tid * sstride;
                const int nb = cur.nr / 16;
                if (nb == 8 && ((reinterpret_cast<uintptr_t>(stile) | (uintptr_t)sstride) & 7u) == 0) {
                    stg8(dst, v.x, v.y);
                } else {
                    stg_bytes(dst, v.x, nb < 4 ? nb : 4);
                    if (nb > 4) stg_bytes(dst + 4, v.y, nb - 4);
                }
            }
        }
        if (failed) {
            // Give up: record the error, let every copy this CTA issued land (bounded),
            // then leave. Stages k .. k+kStages-1 may still have copies in flight.
            if (tid == 0) {
                atomicOr(p.err, kErrTmaTimeout);
                for (int64_t kk = k; kk < n && kk < k + kStages; ++kk) {
                    const int ss = (int)(kk % kStages);
                    if (!mbar_wait_bounded(bar0 + 8 * ss, (uint32_t)((kk / kStages) & 1)))
                        atomicOr(p.err, kErrDrainTimeout);
                }
            }
            __syncthreads();
            return;
        }
        if (tid == 0 && k + kStages < n) issue_next();
        if (++s == kStages) { s = 0; parity ^= 1u; }
    }
}

// ================================================================ absmax alone

__global__ void __launch_bounds__(1024) update_absmax_kernel(float* buf, const float* v, int64_t n, float decay)
{
    __shared__ float part[32];
    float m = 0.0f;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, v[i]);
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0f;
        for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (threadIdx.x == 0) {
            const float d = __fmul_rn(*buf, decay);
            *buf = d > m ? d : m;
        }
    }
}

}  // namespace nvfp4pt
