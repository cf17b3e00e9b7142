// Column pass of the NVFP4 per-token cast (sm_100a): the columnwise encode (codes and
// E4M3 scales of X^T) once the row pass has left the per-column amax of every token
// group in amax_col. It reads x once more, straight into registers: no shared-memory
// tiles of x, no block barriers in the loop.
//
// Layout of the work: a "task" is up to 512 rows x 32 columns of one token group,
// given to one warp and taken in "steps" of 64 rows. In a step, lane l = q + 8s holds
// the 16 rows 16s..16s+15 of the step's columns 4q..4q+3 (one 8-byte load per row, so
// eight consecutive lanes read one row's 64 bytes), encodes its four 16-row blocks and
// parks codes and scales in the warp's staging area. After each 256 rows (a "half")
// the warp writes their codes: up to 128 code bytes per column (one whole L2 line),
// eight lanes to a line so that each store instruction covers four lines. After the
// task's last step it writes 32 scale bytes per column (one whole 32-byte sector).
// Whole lines and sectors matter: column outputs are strided by the group's row count,
// and lines or sectors written in parts, far apart in time, go back to DRAM in parts
// (a half-written sector costs a read of the sector before its write).
//
// Tasks are numbered row-task-major over all groups and walked backwards, each warp
// prefetching the next step's rows into a second register buffer. With one token group the grid's warps take tasks
// T-1-w, T-1-w-W, ... (W warps in all): the grid sweeps x from the bottom up as one
// front and starts on the rows that the row pass, sweeping downwards, read last and
// left in L2. With several groups CTA c owns a contiguous run of tasks, warp w taking
// every 16th from its end, which lines up with the contiguous runs of the row pass.
#pragma once

#include "nvfp4pt_device.cuh"
#include "nvfp4pt_xform.cuh"

namespace nvfp4pt {

constexpr int kColThreads = 512;   // one CTA per SM: 128 registers per thread
constexpr int kColWarps = kColThreads / 32;
constexpr int kStepRows = 64;      // rows of a step: four 16-row blocks
constexpr int kTaskRows = 512;     // rows of a task: up to eight steps (256 when tasks would be few)
constexpr int kHalfRows = 256;     // rows whose codes are staged and written at once
constexpr int kTaskCols = 32;      // columns of a task: 8 quads x 4
constexpr int kColStageBytes = kTaskCols * (128 + 32);      // per warp: codes of a half, scales of a task
constexpr int kSmemColPass = kColWarps * kColStageBytes;    // dynamic shared memory

template <int MAXG>
struct ColParams {
    int64_t cols;
    int64_t num_tasks;   // row tasks x strips
    int32_t task_rows;   // rows of a task: kTaskRows, or kHalfRows when that leaves warps idle
    int32_t small_tasks; // one token group: the first small_tasks row tasks have kHalfRows rows
    int32_t strips;      // ceil(cols / 32)
    int32_t num_ctas;
    int32_t num_groups;
    int32_t nbuf;        // running buffers to update (0: none)
    float decay;
    int32_t q_col_32;    // q_col is 32-byte aligned: full column segments go in one store
    int32_t strided;     // one front over the whole grid (else a contiguous run per CTA)
    int32_t back_rt;     // a warp's next task is wstride tasks back:
    int32_t back_strip;  //   wstride = back_rt * strips + back_strip, back_strip < strips
    const uint16_t* x;
    float* amax_col;         // [G, cols] fp32: final when the row pass has ended, or (when colmax is
                             //   set) written here from colmax
    const uint16_t* colmax;  // [G, cols] bf16 column maxima left by the row pass, or null
    uint8_t* q_col;
    uint8_t* sf_col;
    float* absmax;           // [nbuf] running amax buffers, or null
    const float* obs;        // [G] amax observed by the row pass
    uint32_t* err;           // device error word (colpass_tma: a copy that never landed)
    // columnwise options (nvfp4pt_xform.cuh): the Hadamard transform with its sign mask,
    // stochastic rounding with its Philox key and counter offset
    int32_t rht;
    uint32_t rht_signs;
    int32_t sr;
    uint32_t sr_key0, sr_key1, sr_off0, sr_off1;
    int32_t row_off[MAXG + 1];    // first row of each group
    int32_t task_off[MAXG + 1];   // first row task of each group
};

// What the column pass does with its tasks: the plain columnwise encode, the encode
// with the columnwise options (the values of each block transformed and/or rounded
// stochastically), or a sweep that only finds the column amax of the transformed values
// (atomic max on the float bits into amax_col, which starts at zero).
enum ColMode { kColPlain = 0, kColOpts = 1, kColXformAmax = 2 };

// Codes of 8 consecutive rows of one column with one multiplier; the column is the
// low (HI = false) or high half of the bf16 words v[r0 .. r0+7][w]. Row i -> bits 4i.
template <bool HI>
__device__ __forceinline__ uint32_t encode8_strided(const uint32_t (&v)[16][2], int r0, int w, float e)
{
    auto val = [&](int i) { return HI ? bf16_hi(v[r0 + i][w]) : bf16_lo(v[r0 + i][w]); };
    float y[8];
    mul2(y[0], y[1], val(0), val(1), e);
    mul2(y[2], y[3], val(2), val(3), e);
    mul2(y[4], y[5], val(4), val(5), e);
    mul2(y[6], y[7], val(6), val(7), e);
    return e2m1x8_packed(y);
}

// Where a task sits: its group, first row, row count and first column.
struct ColTask {
    int32_t g;        // token group
    int32_t row0;
    int32_t goff;
    int32_t grows;
    int32_t c0;
    int32_t nrows;    // 16..512, a multiple of 16
};

// Undo the staging order of a column's 32 scale bytes: position p of the row (p = 0..7
// over the words of s0, s1) holds word p ^ x of the column.
__device__ __forceinline__ void unswizzle_words(uint4& s0, uint4& s1, int x)
{
    uint32_t w[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int b = 1; b < 8; b <<= 1) {
        if (x & b) {
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                if ((p & b) == 0) {
                    const uint32_t t = w[p];
                    w[p] = w[p | b];
                    w[p | b] = t;
                }
            }
        }
    }
    s0 = make_uint4(w[0], w[1], w[2], w[3]);
    s1 = make_uint4(w[4], w[5], w[6], w[7]);
}

// Staging slot of 8-byte chunk k (16 rows) of column c: 16-byte chunk (k >> 1) ^ g(c)
// of the column's 128-byte row. g keeps both the lanes' 8-byte stores of a step and
// the column reads of the write-out free of bank conflicts.
__device__ __forceinline__ int stage_off(int c, int k)
{
    const int g = (c & 7) ^ ((c >> 2) & 6);
    return c * 128 + 16 * ((k >> 1) ^ g) + 8 * (k & 1);
}

template <int MAXG>
__device__ __forceinline__ int group_of_task(const ColParams<MAXG>& p, int rt)
{
    if (MAXG == 1) return 0;
    int lo = 0, hi = p.num_groups;  // task_off[lo] <= rt < task_off[hi]; empty groups skipped
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.task_off[mid] <= rt) lo = mid; else hi = mid;
    }
    return lo;
}

// MODE: ColMode.
template <int MAXG, int MODE = kColPlain>
__global__ void __launch_bounds__(kColThreads, 1) colpass(const __grid_constant__ ColParams<MAXG> p)
{
    // per warp: codes [column][16 chunks of 8 bytes] (swizzled), then scales [column][32]
    // The next cast's zeroing kernel may take its place early; it waits for this grid.
    griddep_launch_dependents();
    extern __shared__ __align__(16) uint8_t col_stage[];
    __shared__ uint32_t rcp_tab[8];
    init_rcp_table(rcp_tab);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int quad = lane & 7;         // columns 4 quad .. 4 quad + 3 of the task
    const int blk = lane >> 3;         // 16-row block of the step this lane loads
    const int64_t cols = p.cols;

    // this warp's tasks: first, first - wstride, ... >= t0
    int64_t t0, first, wstride;
    if (p.strided) {
        t0 = 0;
        wstride = (int64_t)p.num_ctas * kColWarps;
        first = p.num_tasks - 1 - ((int64_t)blockIdx.x * kColWarps + warp);
    } else {
        t0 = (p.num_tasks * blockIdx.x) / p.num_ctas;
        wstride = kColWarps;
        first = (p.num_tasks * (blockIdx.x + 1)) / p.num_ctas - 1 - warp;
    }
    const int64_t ntask = first < t0 ? 0 : (first - t0) / wstride + 1;

    // The current task is row task rt, column strip `strip`, of group g; the walk only
    // goes backwards, wstride tasks at a time.
    int g = 0, rt = 0, strip = 0;
    auto locate = [&](ColTask& ct) {
        if (MAXG > 1) {
            while (g > 0 && rt < p.task_off[g]) --g;
        }
        ct.g = g;
        ct.goff = p.row_off[g];
        ct.grows = p.row_off[g + 1] - ct.goff;
        int tr = p.task_rows;
        if (MAXG == 1 && p.small_tasks > 0) {
            // the top rows (walked last) in 256-row tasks, the rest in 512-row tasks
            tr = rt < p.small_tasks ? kHalfRows : kTaskRows;
            ct.row0 = rt < p.small_tasks ? rt * kHalfRows : p.small_tasks * kHalfRows + (rt - p.small_tasks) * kTaskRows;
        } else {
            ct.row0 = ct.goff + (rt - p.task_off[g]) * p.task_rows;
        }
        const int left = ct.goff + ct.grows - ct.row0;
        ct.nrows = left >= tr ? tr : left;
        ct.c0 = strip * kTaskCols;
    };
    auto step_back = [&]() {
        strip -= p.back_strip;
        rt -= p.back_rt;
        if (strip < 0) { strip += p.strips; --rt; }
    };

    uint32_t va[16][2], vb[16][2];
    // rows row0 + 16 * blk .. + 15 of columns c0 + 4 * quad .. + 3, zero where the
    // block or the columns lie outside the task
    const uint32_t row_bytes = (uint32_t)cols * 2u;
    auto load = [&](const ColTask& ct, int step, uint32_t (&v)[16][2]) {
        const int c = ct.c0 + 4 * quad;
        const int r = kStepRows * step + 16 * blk;
        const bool ok = r < ct.nrows && c < cols;
        const uint8_t* src = reinterpret_cast<const uint8_t*>(p.x + (int64_t)(ct.row0 + r) * cols + c);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (ok) {
                const uint2 w = ldg_stream64(src);
                v[i][0] = w.x;
                v[i][1] = w.y;
            } else {
                v[i][0] = 0u;
                v[i][1] = 0u;
            }
            src += row_bytes;
        }
    };
    // amax of column 4q + j of a task for lane 4q + j (g is the task's group)
    auto load_amax = [&](const ColTask& ct) -> float {
        const int c = ct.c0 + 4 * quad + blk;
        if (c >= cols) return 0.0f;
        const int64_t i = (int64_t)g * cols + c;
        return p.colmax ? __uint_as_float((uint32_t)p.colmax[i] << 16) : p.amax_col[i];
    };
    // With colmax, the fp32 amax_col output of (group, strip) comes from the warp that
    // takes the group's first row task there: lane l holds column c0 + 4 quad + blk's amax.
    auto publish_amax = [&](const ColTask& ct, float a) {
        const int c = ct.c0 + 4 * quad + blk;
        if (p.colmax && ct.row0 == ct.goff && c < cols) p.amax_col[(int64_t)g * cols + c] = a;
    };
    // outer scales of the quad's four columns: each lane finds one, the quad shares them
    auto outer_scales = [&](float a, float (&sc)[4]) {
        const float mine = s_enc_of(a);
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[j] = __shfl_sync(0xFFFFFFFFu, mine, (j << 3) | quad);
    };

    ColTask cur;
    int step = 0;
    if (ntask > 0) {
        rt = (int)(first / p.strips);
        strip = (int)(first - (int64_t)rt * p.strips);
        if (MAXG > 1) g = group_of_task(p, rt);
        locate(cur);
        step = (cur.nrows - 1) / kStepRows;   // steps go backwards too
        load(cur, step, va);   // x is read-only for the whole chain: load before the row pass ends
    }

    griddep_wait();
    if (MODE != kColXformAmax && blockIdx.x == 0 && p.absmax) {
        for (int i = tid; i < p.nbuf; i += kColThreads) {
            const float d = __fmul_rn(p.absmax[i], p.decay);
            const float o = p.obs[i];
            p.absmax[i] = d > o ? d : o;
        }
    }
    __syncthreads();   // rcp_tab
    if (ntask == 0) return;

    uint8_t* xc = col_stage + warp * kColStageBytes;
    uint8_t* xs = xc + kTaskCols * 128;
    // This lane's slots: column 4q+j, block kb = 4*(step & 3) + blk of the current half
    // goes to stage_off(4q+j, kb) = xq + 128j + 16*(hg ^ j), hg = (kb >> 1) ^ G(q), where
    // g(4q+j) = j ^ G(q) with G(q) = 4(q & 1) ^ (q & 6); its scale byte (block
    // 4*step + blk of the task) to column 4q+j's 32-byte row at word (step ^ q), byte
    // blk: the scale stores of a step then fall on eight different banks.
    uint8_t* xq = xc + 512 * quad + 8 * (blk & 1);
    uint8_t* xsq = xs + 128 * quad + blk;
    const int gq = (4 * (quad & 1)) ^ (quad & 6);
    const uint64_t pol_out = l2_evict_first();
    float xamax[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // kColXformAmax: this lane's column maxima of the task
    float sc[4];
    {
        const float a = load_amax(cur);
        publish_amax(cur, a);
        outer_scales(a, sc);
    }

    int64_t k = 0;   // tasks finished
    // One step on the rows in `v` while the next step's rows load into `vn`; the
    // loop alternates the two buffers. Returns false after the last step.
    auto run_step = [&](uint32_t (&v)[16][2], uint32_t (&vn)[16][2]) -> bool {
        // prefetch the next step: of this task, or the last step of the next task
        ColTask nxt = cur;
        int nstep = step - 1;
        float a_nxt = 0.0f;
        const bool more = step > 0 || k + 1 < ntask;
        if (step == 0 && more) {
            step_back();
            locate(nxt);
            nstep = (nxt.nrows - 1) / kStepRows;
            a_nxt = load_amax(nxt);
        }
        if (more) load(nxt, nstep, vn);


        if constexpr (MODE == kColPlain) {
            // block amax of the four columns over this lane's 16 rows
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

            // codes and scales of this lane's block of each column -> staging
            const int hg = (2 * (step & 3) + (blk >> 1)) ^ gq;
            uint8_t* xsb = xsq + 4 * (step ^ quad);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int w = j >> 1;
                const uint32_t lo = (j & 1) ? encode8_strided<true>(v, 0, w, e[j]) : encode8_strided<false>(v, 0, w, e[j]);
                const uint32_t hi = (j & 1) ? encode8_strided<true>(v, 8, w, e[j]) : encode8_strided<false>(v, 8, w, e[j]);
                *reinterpret_cast<uint2*>(xq + 128 * j + 16 * (hg ^ j)) = make_uint2(lo, hi);
                xsb[32 * j] = (uint8_t)(((j < 2) ? sf01 : sf23) >> (8 * (j & 1)));
            }
        } else {
            // one column at a time: its 16 values as binary32, the transform, the block
            // steps with IEEE divisions, codes by nearest or stochastic rounding
            const int hg = (2 * (step & 3) + (blk >> 1)) ^ gq;
            uint8_t* xsb = xsq + 4 * (step ^ quad);
            const int64_t m0 = (int64_t)cur.row0 + kStepRows * step + 16 * blk;   // first row of the block
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float f[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) f[i] = (j & 1) ? bf16_hi(v[i][j >> 1]) : bf16_lo(v[i][j >> 1]);
                if (p.rht) rht16(f, p.rht_signs);
                float ba = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; ++i) ba = fmaxf(ba, fabsf(f[i]));
                if constexpr (MODE == kColXformAmax) {
                    xamax[j] = fmaxf(xamax[j], ba);
                } else {
                    uint32_t sf;
                    float e;
                    block_scale_ieee(ba, sc[j], sf, e);
                    float y[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(f[i], e);
                    uint32_t lo = 0u, hi = 0u;
                    if (p.sr) {
                        const uint32_t col = (uint32_t)(cur.c0 + 4 * quad + j);
#pragma unroll
                        for (int t4 = 0; t4 < 4; ++t4) {
                            const uint4 r = philox10((uint32_t)((m0 >> 2) + t4), col, p.sr_off0, p.sr_off1,
                                                     p.sr_key0, p.sr_key1);
                            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int i = 4 * t4 + u;
                                const uint32_t code = e2m1_sr(y[i], rw[u]);
                                if (i < 8) lo |= code << (4 * i); else hi |= code << (4 * (i - 8));
                            }
                        }
                    } else {
                        float ylo[8], yhi[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            ylo[i] = y[i];
                            yhi[i] = y[i + 8];
                        }
                        lo = e2m1x8_packed(ylo);
                        hi = e2m1x8_packed(yhi);
                    }
                    *reinterpret_cast<uint2*>(xq + 128 * j + 16 * (hg ^ j)) = make_uint2(lo, hi);
                    xsb[32 * j] = (uint8_t)sf;
                }
            }
        }

        if (MODE != kColXformAmax && (step & 3) == 0) {
            // a half done: write its codes out of staging (the half's rows start at
            // 64 * step of the task)
            __syncwarp();
            const int nblk = min(16, cur.nrows / 16 - 4 * step);
            const int lrow = cur.row0 - cur.goff + kStepRows * step;
            const int64_t gq = cols * cur.goff / 2 + lrow / 2;    // column 0's code bytes, then
            const int64_t cstride = cur.grows / 2;                //   one column every cstride
            const bool wide = p.q_col_32 && (cur.grows & 63) == 0;
            if (wide) {
                // 32-byte aligned, nblk a multiple of 4: 8 lanes per column, 16 bytes
                // each, so one store covers four columns' whole segments
                const int k = lane & 7;
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int cl = 4 * it + (lane >> 3);
                    const int c = cur.c0 + cl;
                    if (c < cols && 2 * k < nblk) {
                        const uint4 a = *reinterpret_cast<const uint4*>(xc + stage_off(cl, 2 * k));
                        stg16_ef(p.q_col + gq + (int64_t)c * cstride + 16 * k, a, pol_out);
                    }
                }
            } else if (cur.c0 + lane < cols) {
                // lane j: column j's codes
                uint8_t* q = p.q_col + gq + (int64_t)(cur.c0 + lane) * cstride;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (i < nblk) {
                        const uint2 a = *reinterpret_cast<const uint2*>(xc + stage_off(lane, i));
                        stg8_ef(q + 8 * i, a.x, a.y, pol_out);
                    }
                }
            }
            __syncwarp();   // staging is written again by the next step
        }
        if (step == 0) {
            if constexpr (MODE == kColXformAmax) {
                // task done: the four lanes of each column quad combine their maxima and
                // one of them raises the task's group's amax_col entries (the walk's g
                // already names the next task's group)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float a = fmaxf(xamax[j], __shfl_xor_sync(0xFFFFFFFFu, xamax[j], 8));
                    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 16));
                    const int c = cur.c0 + 4 * quad + j;
                    if (blk == 0 && c < cols && a > 0.0f)
                        red_max_f32(p.amax_col + (int64_t)cur.g * cols + c, __float_as_uint(a));
                    xamax[j] = 0.0f;
                }
            } else {
                // task done: lane j writes column j's block scales, one whole 32-byte sector
                // per column when the task has 512 rows
                const int nblk = cur.nrows / 16;
                const int lrow = cur.row0 - cur.goff;
                const int c = cur.c0 + lane;
                if (c < cols) {
                    uint8_t* sf = p.sf_col + cols * cur.goff / 16 + (int64_t)c * (cur.grows / 16) + lrow / 16;
                    // the row's word at position w ^ (lane >> 2) is the column's word w
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
            }
            __syncwarp();
            ++k;
            if (more) {
                cur = nxt;
                publish_amax(cur, a_nxt);
                outer_scales(a_nxt, sc);
            }
        }
        step = nstep;
        return more;
    };
    while (run_step(va, vb) && run_step(vb, va)) {
    }
}

}  // namespace nvfp4pt
