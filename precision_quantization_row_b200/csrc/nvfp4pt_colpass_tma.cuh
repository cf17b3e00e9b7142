// Column pass fed by TMA: the columnwise encode of colpass (plain mode) with each warp's
// 64-row x 32-column steps copied by cp.async.bulk.tensor into a ring of kTcStages
// shared-memory slots, kTcStages - 1 steps ahead of the step being encoded, instead of
// the register double buffer of colpass. The walk over tasks, the staging of codes and
// scale bytes and the stores are colpass's.
//
// Why: colpass waits on its own global loads (one step in flight per warp); here the
// copy engine keeps four steps per warp in flight and the warps' loads become shared-
// memory reads. 8 warps per CTA with 4 slots of 4 KB each measured faster than 12 warps
// with 3 slots and than colpass on the 16384 x 8192 activation.
#pragma once

#include "nvfp4pt_colpass.cuh"

namespace nvfp4pt {

constexpr int kTcWarps = 8;
constexpr int kTcThreads = 32 * kTcWarps;
constexpr int kTcStages = 4;
constexpr int kTcStepBytes = kStepRows * kTaskCols * 2;                     // 64 rows x 64 bytes
constexpr int kTcWarpBytes = kTcStages * kTcStepBytes + kColStageBytes;     // ring, then staging
constexpr int kSmemColTma = kTcWarps * kTcWarpBytes + 128;                  // + room to align to 128

// Orders this thread's generic-proxy reads of shared memory before later async-proxy
// (TMA) writes to it.
__device__ __forceinline__ void fence_proxy_async_shared()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int MAXG>
struct ColTmaParams {
    CUtensorMap tmap;    // x as bf16 [rows, cols], boxes of 32 columns x 64 rows, zeros outside
    ColParams<MAXG> c;
};

// A position of a warp's walk: a task and a step of it.
struct ColPos {
    ColTask ct;
    int rt, strip, g, step;
    int64_t k;   // tasks done before this one
};

template <int MAXG>
__global__ void __launch_bounds__(kTcThreads, 1) colpass_tma(const __grid_constant__ ColTmaParams<MAXG> tp)
{
    const ColParams<MAXG>& p = tp.c;
    // The next cast's zeroing kernel may take this grid's place early; it waits for it.
    griddep_launch_dependents();
    extern __shared__ __align__(128) uint8_t tc_smem[];
    __shared__ __align__(8) uint64_t tc_full[kTcWarps][kTcStages];
    __shared__ uint32_t rcp_tab[8];
    init_rcp_table(rcp_tab);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int quad = lane & 7;         // columns 4 quad .. 4 quad + 3 of the task
    const int blk = lane >> 3;         // 16-row block of the step this lane encodes
    const int64_t cols = p.cols;

    // this warp's tasks: first, first - wstride, ... >= t0 (as in colpass)
    const int64_t wstride = p.strided ? (int64_t)p.num_ctas * kTcWarps : kTcWarps;
    const int64_t t0 = p.strided ? 0 : (p.num_tasks * blockIdx.x) / p.num_ctas;
    const int64_t first = p.strided ? p.num_tasks - 1 - ((int64_t)blockIdx.x * kTcWarps + warp)
                                    : (p.num_tasks * (blockIdx.x + 1)) / p.num_ctas - 1 - warp;
    const int64_t ntask = first < t0 ? 0 : (first - t0) / wstride + 1;
    const int32_t back_rt = (int32_t)(wstride / p.strips), back_strip = (int32_t)(wstride % p.strips);

    auto locate = [&](ColPos& q) {
        if (MAXG > 1) {
            while (q.g > 0 && q.rt < p.task_off[q.g]) --q.g;
        }
        ColTask& ct = q.ct;
        ct.g = q.g;
        ct.goff = p.row_off[q.g];
        ct.grows = p.row_off[q.g + 1] - ct.goff;
        int tr = p.task_rows;
        if (MAXG == 1 && p.small_tasks > 0) {
            tr = q.rt < p.small_tasks ? kHalfRows : kTaskRows;
            ct.row0 = q.rt < p.small_tasks ? q.rt * kHalfRows
                                           : p.small_tasks * kHalfRows + (q.rt - p.small_tasks) * kTaskRows;
        } else {
            ct.row0 = ct.goff + (q.rt - p.task_off[q.g]) * p.task_rows;
        }
        const int left = ct.goff + ct.grows - ct.row0;
        ct.nrows = left >= tr ? tr : left;
        ct.c0 = q.strip * kTaskCols;
    };
    auto start = [&](ColPos& q) {
        q.k = 0;
        q.rt = (int)(first / p.strips);
        q.strip = (int)(first - (int64_t)q.rt * p.strips);
        q.g = (MAXG > 1) ? group_of_task(p, q.rt) : 0;
        locate(q);
        q.step = (q.ct.nrows - 1) / kStepRows;   // steps go backwards
    };
    // the next position of the walk; false after the last
    auto advance = [&](ColPos& q) -> bool {
        if (q.step > 0) {
            --q.step;
            return true;
        }
        if (q.k + 1 >= ntask) return false;
        ++q.k;
        q.strip -= back_strip;
        q.rt -= back_rt;
        if (q.strip < 0) {
            q.strip += p.strips;
            --q.rt;
        }
        locate(q);
        q.step = (q.ct.nrows - 1) / kStepRows;
        return true;
    };

    uint8_t* const aligned = tc_smem + ((128u - (smem_u32(tc_smem) & 127u)) & 127u);
    uint8_t* wbase = aligned + warp * kTcWarpBytes;
    uint8_t* xc = wbase + kTcStages * kTcStepBytes;   // staging: codes of a 256-row half
    uint8_t* xs = xc + kTaskCols * 128;                // then the task's scale bytes
    const uint32_t ring = smem_u32(wbase);
    const uint32_t bar0 = smem_u32(&tc_full[warp][0]);
    if (lane == 0) {
        for (int i = 0; i < kTcStages; ++i) mbar_init(bar0 + 8 * i, 1);
        fence_mbar_init();
    }
    __syncwarp();

    ColPos cur, pre;   // the step being encoded, the next step to copy
    int64_t n_issued = 0;
    bool pre_ok = ntask > 0;
    if (pre_ok) {
        start(cur);
        pre = cur;
    }
    auto issue = [&]() {
        if (!pre_ok) return;
        const int slot = (int)(n_issued % kTcStages);
        if (lane == 0) {
            const uint32_t b = bar0 + 8 * slot;
            mbar_arrive_expect_tx(b, kTcStepBytes);
            tma_load_2d(ring + slot * kTcStepBytes, &tp.tmap, pre.ct.c0, pre.ct.row0 + kStepRows * pre.step, b);
        }
        ++n_issued;
        pre_ok = advance(pre);
    };
    // x is read-only for the whole cast: the first steps copy before the row pass ends
    for (int i = 0; i < kTcStages; ++i) issue();

    griddep_wait();
    if (blockIdx.x == 0 && p.absmax) {
        for (int i = tid; i < p.nbuf; i += kTcThreads) {
            const float d = __fmul_rn(p.absmax[i], p.decay);
            const float o = p.obs[i];
            p.absmax[i] = d > o ? d : o;
        }
    }
    __syncthreads();   // rcp_tab
    if (ntask == 0) return;

    // amax of column 4q + j of a task for lane 4q + j
    auto load_amax = [&](const ColTask& ct) -> float {
        const int c = ct.c0 + 4 * quad + blk;
        if (c >= cols) return 0.0f;
        const int64_t i = (int64_t)ct.g * cols + c;
        return p.colmax ? __uint_as_float((uint32_t)p.colmax[i] << 16) : p.amax_col[i];
    };
    // the fp32 amax_col of (group, strip) comes from the warp holding the group's first row task
    auto publish_amax = [&](const ColTask& ct, float a) {
        const int c = ct.c0 + 4 * quad + blk;
        if (p.colmax && ct.row0 == ct.goff && c < cols) p.amax_col[(int64_t)ct.g * cols + c] = a;
    };
    float sc[4];
    auto outer_scales = [&](float a) {
        const float mine = s_enc_of(a);
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[j] = __shfl_sync(0xFFFFFFFFu, mine, (j << 3) | quad);
    };
    {
        const float a = load_amax(cur.ct);
        publish_amax(cur.ct, a);
        outer_scales(a);
    }

    // staging slots as in colpass
    uint8_t* xq = xc + 512 * quad + 8 * (blk & 1);
    uint8_t* xsq = xs + 128 * quad + blk;
    const int gq = (4 * (quad & 1)) ^ (quad & 6);
    const uint64_t pol_out = l2_evict_first();
    const uint32_t rot = 4u * (uint32_t)blk;   // this lane reads its block's rows rotated by blk

    for (int64_t n = 0;; ++n) {
        const int slot = (int)(n % kTcStages);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(bar0 + 8 * slot, (uint32_t)((n / kTcStages) & 1)))) {
            if (lane == 0) atomicOr(p.err, kErrTmaTimeout);
            break;
        }
        const ColTask& ct = cur.ct;
        const int step = cur.step;
        // rows 16 blk + ((i + blk) & 15) of the step, 8 bytes at column 4 quad: the four
        // row blocks of one load instruction then fall on different banks
        uint32_t v[16][2];
        const bool ok = kStepRows * step + 16 * blk < ct.nrows;
        const uint32_t sbase = ring + slot * kTcStepBytes + 64u * 16u * (uint32_t)blk + 8u * (uint32_t)quad;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            uint32_t a, b;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                         : "=r"(a), "=r"(b) : "r"(sbase + 64u * (uint32_t)((i + blk) & 15)));
            v[i][0] = ok ? a : 0u;
            v[i][1] = ok ? b : 0u;
        }
        fence_proxy_async_shared();
        __syncwarp();
        issue();   // the slot just read takes the step kTcStages ahead

        // block amax of the four columns over this lane's 16 rows (in any order)
        uint32_t m[2];
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            uint32_t t[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) t[i] = absmax2(v[i][w], v[i + 8][w]);
#pragma unroll
            for (int i = 0; i < 4; ++i) t[i] = absmax2(t[i], t[i + 4]);
            t[0] = absmax2(t[0], t[2]);
            t[1] = absmax2(t[1], t[3]);
            m[w] = absmax2(t[0], t[1]) & 0x7FFF7FFFu;
        }
        uint32_t sf01, sf23;
        float e[4];
        block_pair_scales_x2(bf16_lo(m[0]), bf16_hi(m[0]), sc[0], sc[1], sf01, e[0], e[1], rcp_tab);
        block_pair_scales_x2(bf16_lo(m[1]), bf16_hi(m[1]), sc[2], sc[3], sf23, e[2], e[3], rcp_tab);

        const int hg = (2 * (step & 3) + (blk >> 1)) ^ gq;
        uint8_t* xsb = xsq + 4 * (step ^ quad);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int w = j >> 1;
            const uint32_t lo = (j & 1) ? encode8_strided<true>(v, 0, w, e[j]) : encode8_strided<false>(v, 0, w, e[j]);
            const uint32_t hi = (j & 1) ? encode8_strided<true>(v, 8, w, e[j]) : encode8_strided<false>(v, 8, w, e[j]);
            // nibble i holds row (i + blk) & 15: rotate the 64-bit word left by 4 blk
            const uint32_t nlo = __funnelshift_l(hi, lo, rot), nhi = __funnelshift_l(lo, hi, rot);
            *reinterpret_cast<uint2*>(xq + 128 * j + 16 * (hg ^ j)) = make_uint2(nlo, nhi);
            xsb[32 * j] = (uint8_t)(((j < 2) ? sf01 : sf23) >> (8 * (j & 1)));
        }

        if ((step & 3) == 0) {
            // a 256-row half done: its codes leave staging (the half starts at row 64 step)
            __syncwarp();
            const int nblk = min(16, ct.nrows / 16 - 4 * step);
            const int lrow = ct.row0 - ct.goff + kStepRows * step;
            const int64_t gqo = cols * ct.goff / 2 + lrow / 2;
            const int64_t cstride = ct.grows / 2;
            const bool wide = p.q_col_32 && (ct.grows & 63) == 0;
            if (wide) {
                const int kk = lane & 7;
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int cl = 4 * it + (lane >> 3);
                    const int c = ct.c0 + cl;
                    if (c < cols && 2 * kk < nblk) {
                        const uint4 a = *reinterpret_cast<const uint4*>(xc + stage_off(cl, 2 * kk));
                        stg16_ef(p.q_col + gqo + (int64_t)c * cstride + 16 * kk, a, pol_out);
                    }
                }
            } else if (ct.c0 + lane < cols) {
                uint8_t* q = p.q_col + gqo + (int64_t)(ct.c0 + lane) * cstride;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (i < nblk) {
                        const uint2 a = *reinterpret_cast<const uint2*>(xc + stage_off(lane, i));
                        stg8_ef(q + 8 * i, a.x, a.y, pol_out);
                    }
                }
            }
            __syncwarp();
        }
        if (step == 0) {
            // task done: lane j writes column j's block scales
            const int nblk = ct.nrows / 16;
            const int lrow = ct.row0 - ct.goff;
            const int c = ct.c0 + lane;
            if (c < cols) {
                uint8_t* sf = p.sf_col + cols * ct.goff / 16 + (int64_t)c * (ct.grows / 16) + lrow / 16;
                uint4 s0 = *reinterpret_cast<const uint4*>(xs + 32 * lane);
                uint4 s1 = *reinterpret_cast<const uint4*>(xs + 32 * lane + 16);
                unswizzle_words(s0, s1, lane >> 2);
                const uintptr_t al = reinterpret_cast<uintptr_t>(sf);
                if (nblk == 32 && (al & 31u) == 0) {
                    stg32_ef(sf, s0, s1, pol_out);
                } else if (nblk == 32 && (al & 15u) == 0) {
                    stg16_ef(sf, s0, pol_out);
                    stg16_ef(sf + 16, s1, pol_out);
                } else if (nblk == 16 && (al & 15u) == 0) {
                    stg16_ef(sf, s0, pol_out);
                } else {
                    const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (4 * i < nblk) stg_bytes(sf + 4 * i, sw[i], min(4, nblk - 4 * i));
                }
            }
            __syncwarp();
        }
        const int64_t k_before = cur.k;
        if (!advance(cur)) break;
        if (cur.k != k_before) {
            const float a = load_amax(cur.ct);
            publish_amax(cur.ct, a);
            outer_scales(a);
        }
    }
    // copies still in flight land before the CTA's shared memory goes away
    for (int64_t n = n_issued - kTcStages > 0 ? n_issued - kTcStages : 0; n < n_issued; ++n) {
        const int slot = (int)(n % kTcStages);
        if (!mbar_wait_bounded(bar0 + 8 * slot, (uint32_t)((n / kTcStages) & 1)) && lane == 0)
            atomicOr(p.err, kErrDrainTimeout);
    }
}

}  // namespace nvfp4pt
