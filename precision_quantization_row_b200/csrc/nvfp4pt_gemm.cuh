// Per-token NVFP4 GEMM on the 5th-generation tensor cores (sm_100a):
//
//   D[m, n] = S_dec(a_m) * S_dec(b_n) * sum_k val(qA[m,k]) sf_A[m, k/16] val(qB[n,k]) sf_B[n, k/16]
//
// with S_dec = RN(amax / 2688), the decode scale of the per-token cast. Both operands are
// the cast's rowwise NVFP4 data (K-major: codes [rows, K/2], compact E4M3 block scales
// [rows, K/16], one outer amax per row); the TN, NN and NT products of a layer all take
// this one form, each operand being the rowwise data of a matrix or of its transpose
// (TransformerEngine PR #3045 "Add NVFP4 per-token quantization recipe": a GEMM that
// rescales with the per-row and per-column outer-amax vectors inside its epilogue).
//
// First gemm_sf_prep writes each operand's block scales into the workspace in the
// layout of the scale copy into tensor memory (one contiguous 2048-byte piece per
// 128-row block and 256-element K step). Then a persistent CTA per SM takes 128 x 256
// tiles of D in turn:
//   warp 0       TMA producer: per 256-element K step, the A and B code tiles (128-byte
//                rows, 128-byte swizzle) and the A and B scale pieces (bulk copies),
//                four stages deep, running ahead into the next tile.
//   warp 1       allocates tensor memory; lane 0 issues the scale copies into tensor
//                memory (tcgen05.cp) and the four block-scaled MMAs of the step
//                (tcgen05.mma kind::mxf4nvf4, 16-element E4M3 scale vectors).
//   warps 2..9   epilogue: each drains 32 rows x 128 columns of the fp32 accumulator
//                into registers (tcgen05.ld) and frees it, so the next tile's MMAs run
//                while it multiplies by S_dec(a_m) and S_dec(b_n) and stores D.
// Every wait on an mbarrier is bounded; a wait that gives up sets the error word and
// the warp skips the rest of its work (after its copies in flight have landed).
#pragma once

#include "nvfp4pt_device.cuh"

namespace nvfp4pt {

constexpr int kGemmBM = 128;           // rows of A per tile (the MMA's M)
constexpr int kGemmBN = 256;           // rows of B per tile (the MMA's N)
constexpr int kGemmBK = 256;           // K elements per pipeline stage: one 128-byte row of codes
constexpr int kGemmStages = 4;
constexpr int kGemmEpiWarps = 8;       // two per 32-lane group of tensor memory, 128 columns each
constexpr int kGemmThreads = 32 * (2 + kGemmEpiWarps);
constexpr int kGemmTmemCols = 512;     // accumulator 256 columns + scale factors 48

// shared memory of one stage (offsets from the 1024-aligned stage base)
constexpr int kGsA = 0;                               // A codes  128 x 128 B
constexpr int kGsB = kGsA + kGemmBM * 128;            // B codes  256 x 128 B
constexpr int kGsSfa = kGsB + kGemmBN * 128;          // A scales: one 2048-byte piece in copy layout
constexpr int kGsSfb = kGsSfa + kGemmBM * 16;         // B scales: two pieces
constexpr int kGemmStageBytes = kGsSfb + kGemmBN * 16;
constexpr int kGemmTxBytes = kGemmStageBytes;         // bytes the copies bring per stage
constexpr int kGemmSfPiece = 2048;                     // scales of 128 rows x one 256-element K step
constexpr int kGemmSmem = kGemmStages * kGemmStageBytes + 1024;   // + room to align the stages to 1024

// tensor memory columns (lane field 0)
constexpr uint32_t kTmAcc = 0;      // 256 fp32 columns
constexpr uint32_t kTmSfa = 256;    // 4 per MMA K step: A row 32c + i of a step in lane i, column c
constexpr uint32_t kTmSfb = 272;    // 8 per MMA K step: B row 32c + i of a step in lane i, column c

struct GemmParams {
    CUtensorMap tmA;     // codes of A: uint8 [M, K/2], box 128 x 128, 128-byte swizzle
    CUtensorMap tmB;     // codes of B: uint8 [N, K/2], box 128 x 256, 128-byte swizzle
    int64_t m, n, k;
    const uint8_t* sfa_pre;   // A's scales in copy layout: [ceil(M/128)][K/256] pieces
    const uint8_t* sfb_pre;   // B's scales in copy layout: [2 ceil(N/256)][K/256] pieces
    const float* amax_a;
    const float* amax_b;
    float* d;            // [M, N] fp32
    uint32_t* err;
    int32_t m_tiles;     // tiles along M
    int32_t n_tiles;     // tiles along N; tile t as gemm_tile maps it, CTA c takes c, c + grid, ...
};

// Block-scaled MMA instruction descriptor: E2M1 A and B (K-major), E4M3 scales, fp32
// accumulator, M = 128, N = 256, dense K = 64 per instruction.
__host__ __device__ constexpr uint32_t gemm_idesc()
{
    return (1u << 7)                        // A format: E2M1
           | (1u << 10)                     // B format: E2M1
           | ((uint32_t)(kGemmBN >> 3) << 17)
           | (0u << 23)                     // scale format: E4M3
           | ((uint32_t)(kGemmBM >> 4) << 24);
}

// Shared-memory matrix descriptor of a K-major operand tile with 128-byte rows and the
// 128-byte swizzle: groups of 8 rows 1024 bytes apart; the tile base is 1024-aligned,
// and a K offset inside the 128-byte row is added to the start address.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4)          // start address
           | ((uint64_t)1 << 16)                        // leading byte offset (unused here)
           | ((uint64_t)(1024 >> 4) << 32)              // stride byte offset: 8 rows
           | ((uint64_t)1 << 46)                        // descriptor version
           | ((uint64_t)2 << 61);                       // 128-byte swizzle
}

// Descriptor of a 32-row x 16-byte block of scale factors (no swizzle; 8-row groups of
// 128 contiguous bytes, 128 bytes apart), the source of one tcgen05.cp.32x128b.
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(128 >> 4) << 32) |
           ((uint64_t)1 << 46);
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// The 32 x 16-byte scale block at `sdesc` into tensor memory at `taddr`: lane i of each
// of the four 32-lane groups receives row i (four 32-bit columns).
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_fp4_block16(uint32_t tacc, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t tsfa, uint32_t tsfb, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                 ::"r"(tacc), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
                 : "memory");
}

// Arrive once on the mbarrier when every tcgen05 operation this thread issued before has
// completed.
__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 lanes: lane i gets row (base lane + i);
// the registers are valid after tmem_wait_ld().
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                   "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                   "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                   "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
                   "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }


// One contiguous copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from
// global into shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// An operand's block scales ([rows, K/16]: 16 bytes per row and 256-element K step) in the
// layout of tcgen05.cp.32x128b.warpx4: for each 128-row block and K step a 2048-byte piece
// whose 512-byte part kb holds, in its 16-byte line i, the kb-th 4-byte scale word of the
// block's rows i, i + 32, i + 64, i + 96. Rows from `rows` up to `padded_rows` get zero
// scales. Thread u takes row u / ksteps, K step u % ksteps (the reads are contiguous).
__global__ void __launch_bounds__(256) gemm_sf_prep(const uint8_t* sf, int64_t rows, int64_t padded_rows,
                                                    int64_t ksteps, uint8_t* pre)
{
    const int64_t total = padded_rows * ksteps;
    for (int64_t u = (int64_t)blockIdx.x * 256 + threadIdx.x; u < total; u += (int64_t)gridDim.x * 256) {
        const int64_t r = u / ksteps, ks = u - r * ksteps;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < rows) v = __ldg(reinterpret_cast<const uint4*>(sf + r * (ksteps * 16) + ks * 16));
        uint8_t* dst = pre + ((r >> 7) * ksteps + ks) * kGemmSfPiece + (r & 31) * 16 + ((r >> 5) & 3) * 4;
        *reinterpret_cast<uint32_t*>(dst) = v.x;
        *reinterpret_cast<uint32_t*>(dst + 512) = v.y;
        *reinterpret_cast<uint32_t*>(dst + 1024) = v.z;
        *reinterpret_cast<uint32_t*>(dst + 1536) = v.w;
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Tile t -> its first row of A and of B: groups of kGemmGroupM row blocks are walked
// column-major (all tiles of the group's first column of B, then the next), so that the
// CTAs running at one time share few slices of A and B.
constexpr int kGemmGroupM = 8;
__device__ __forceinline__ void gemm_tile(int64_t t, int32_t m_tiles, int32_t n_tiles, int32_t& m0, int32_t& n0)
{
    const int64_t per = (int64_t)kGemmGroupM * n_tiles;
    const int64_t g = t / per;
    const int64_t first = g * kGemmGroupM;
    const int64_t gm = m_tiles - first < kGemmGroupM ? m_tiles - first : kGemmGroupM;
    const int64_t r = t - g * per;
    m0 = (int32_t)((first + r % gm) * kGemmBM);
    n0 = (int32_t)((r / gm) * kGemmBN);
}

__device__ __forceinline__ void gemm_fail(uint32_t* err, uint32_t code)
{
    atomicOr(err, code);
}

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_per_token_kernel(const __grid_constant__ GemmParams p)
{
    extern __shared__ __align__(1024) uint8_t gemm_smem_raw[];
    // full[S], empty[S], acc_full, acc_empty
    __shared__ __align__(8) uint64_t bar_mem[2 * kGemmStages + 2];
    __shared__ uint32_t tmem_slot_mem;
    const uint32_t smem0 = (smem_u32(gemm_smem_raw) + 1023u) & ~1023u;
    const uint32_t full0 = smem_u32(bar_mem), empty0 = full0 + 8 * kGemmStages;
    const uint32_t acc_full = full0 + 16 * kGemmStages, acc_empty = acc_full + 8;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ksteps = (int)(p.k / kGemmBK);
    const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kGemmEpiWarps);
        fence_mbar_init();
        prefetch_tensormap(&p.tmA);
        prefetch_tensormap(&p.tmB);
    }
    if (warp == 1) tmem_alloc(smem_u32(&tmem_slot_mem), kGemmTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(&tmem_slot_mem);

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int64_t it = 0;   // K steps issued over all tiles
            bool ok = true;
            for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                int32_t m0, n0;
                gemm_tile(t, p.m_tiles, p.n_tiles, m0, n0);
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = (int)(it % kGemmStages);
                    const uint32_t ph = (uint32_t)((it / kGemmStages) & 1);
                    if (it >= kGemmStages && !mbar_wait_bounded(empty0 + 8 * s, ph ^ 1u)) {
                        gemm_fail(p.err, kErrTmaTimeout);
                        ok = false;
                        break;
                    }
                    const uint32_t st = smem0 + s * kGemmStageBytes;
                    const uint32_t fb = full0 + 8 * s;
                    mbar_arrive_expect_tx(fb, kGemmTxBytes);
                    tma_load_2d(st + kGsA, &p.tmA, ks * 128, m0, fb);
                    tma_load_2d(st + kGsB, &p.tmB, ks * 128, n0, fb);
                    const int64_t pa = ((int64_t)(m0 / 128) * ksteps + ks) * kGemmSfPiece;
                    bulk_load(st + kGsSfa, p.sfa_pre + pa, kGemmSfPiece, fb);
                    for (int h = 0; h < kGemmBN / 128; ++h) {
                        const int64_t pb = ((int64_t)(n0 / 128 + h) * ksteps + ks) * kGemmSfPiece;
                        bulk_load(st + kGsSfb + kGemmSfPiece * h, p.sfb_pre + pb, kGemmSfPiece, fb);
                    }
                }
            }
            // copies must not land in freed shared memory: wait for the last ones issued
            for (int64_t j = it - kGemmStages > 0 ? it - kGemmStages : 0; j < it; ++j) {
                const int s = (int)(j % kGemmStages);
                if (!mbar_wait_bounded(full0 + 8 * s, (uint32_t)((j / kGemmStages) & 1)))
                    gemm_fail(p.err, kErrDrainTimeout);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        const uint32_t idesc = gemm_idesc();
        int64_t it = 0;
        int j = 0;    // tiles of this CTA so far
        bool ok = true;
        for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
            // the epilogue has drained the previous tile's accumulator
            if (j > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait_bounded(acc_empty, (uint32_t)((j - 1) & 1)))) {
                if (lane == 0) gemm_fail(p.err, kErrTmaTimeout);
                break;
            }
            tc_fence_after();
            for (int ks = 0; ks < ksteps; ++ks, ++it) {
                const int s = (int)(it % kGemmStages);
                const uint32_t ph = (uint32_t)((it / kGemmStages) & 1);
                // the whole warp leaves together if any lane's wait gave up
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(full0 + 8 * s, ph))) {
                    if (lane == 0) gemm_fail(p.err, kErrTmaTimeout);
                    ok = false;
                    break;
                }
                const uint32_t st = smem0 + s * kGemmStageBytes;
                if (lane == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        tmem_cp_sf(tbase + kTmSfa + 4 * kb, smem_desc_sf(st + kGsSfa + 512 * kb));
#pragma unroll
                        for (int h = 0; h < kGemmBN / 128; ++h)
                            tmem_cp_sf(tbase + kTmSfb + 8 * kb + 4 * h,
                                       smem_desc_sf(st + kGsSfb + 2048 * h + 512 * kb));
                    }
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        // K step kb of the stage: 64 codes = 32 bytes into each 128-byte row
                        const uint64_t ad = smem_desc_sw128(st + kGsA + 32 * kb);
                        const uint64_t bd = smem_desc_sw128(st + kGsB + 32 * kb);
                        mma_fp4_block16(tbase + kTmAcc, ad, bd, idesc, tbase + kTmSfa + 4 * kb,
                                        tbase + kTmSfb + 8 * kb, (ks > 0 || kb > 0) ? 1u : 0u);
                    }
                    tc_commit(empty0 + 8 * s);   // the stage's shared memory is free once these finish
                }
                __syncwarp();
            }
            if (lane == 0) tc_commit(acc_full);   // the tile's accumulator is complete
        }
    } else {
        // ------------------------------------------------------------- epilogue
        const int q = warp & 3;                  // this warp's 32-lane group of tensor memory
        const int half = (warp - 2) >> 2;        // and its 128 columns of the tile
        int j = 0;
        for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
            int32_t tm0, tn0;
            gemm_tile(t, p.m_tiles, p.n_tiles, tm0, tn0);
            const int64_t m0 = tm0, n0 = (int64_t)tn0 + 128 * half;
            const int64_t row = m0 + 32 * q + lane;
            // the column decode scales S_dec(b_n) of this warp's 128 columns, 4 per lane
            float sdec[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t n = n0 + 4 * lane + u;
                sdec[u] = n < p.n ? __fdiv_rn(__ldg(p.amax_b + n), 2688.0f) : 0.0f;
            }
            const float sa = row < p.m ? __fdiv_rn(__ldg(p.amax_a + row), 2688.0f) : 0.0f;
            const bool ok = mbar_wait_bounded(acc_full, (uint32_t)(j & 1));
            if (!ok) gemm_fail(p.err, kErrTmaTimeout);
            tc_fence_after();
            // tcgen05.ld is warp-collective: the warp reads the accumulator only if every lane may
            if (!__all_sync(0xFFFFFFFFu, ok && *reinterpret_cast<volatile uint32_t*>(p.err) == 0)) break;
            uint32_t v[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld32_nowait(tbase + ((uint32_t)(32 * q) << 16) + kTmAcc + (uint32_t)(128 * half + 32 * c), v[c]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);   // the MMA warp may overwrite the accumulator
            // every lane takes part in the shuffles; lanes past the last row store nothing
            float* dst = p.d + row * p.n + n0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const int col = 32 * c + 4 * j4;       // column of the warp's 128
                    float o[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float sb = __shfl_sync(0xFFFFFFFFu, sdec[u], col >> 2);
                        o[u] = __fmul_rn(__fmul_rn(__uint_as_float(v[c][4 * j4 + u]), sa), sb);
                    }
                    if (row < p.m && n0 + col < p.n)
                        *reinterpret_cast<float4*>(dst + col) = make_float4(o[0], o[1], o[2], o[3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kGemmTmemCols);
    }
}

}  // namespace nvfp4pt
