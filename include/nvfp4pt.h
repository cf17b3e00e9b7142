/*
 * nvfp4pt.h -- C ABI of the B200 (sm_100a) NVFP4 per-token quantization cast.
 *
 * The cast (TransformerEngine PR #3045 "Add NVFP4 per-token quantization recipe",
 * Description): where the default NVFP4 recipe keeps one outer amax per tensor,
 * the per-token recipe keeps one per row (length M) for the rowwise data and one
 * per column (length K) for the columnwise data. With
 *     s_enc = 2688 / amax        (binary32, round-to-nearest-even; 1 when amax == 0)
 * each 16-element block gets an E4M3 scale
 *     sf    = e4m3_rn_satfinite( RN( RN(block_amax / 6) * s_enc ) )
 * (the order of the weight quantizer's (amax/6) * 448 / (gA/6), Model-Optimizer
 * PR #2598, review thread on the FP8 block scale: other orders round to other codes),
 *     enc   = sf == 0 ? 0 : RN(s_enc / float(sf))
 * and each element becomes q = e2m1_rn_satfinite(RN(x * enc)), two codes per byte,
 * element 2j in the low nibble. Readings where the pages are silent: s_enc and enc
 * are clamped to FLT_MAX instead of overflowing; a negative value that rounds to
 * zero keeps its sign (code 0x8); NaN/inf inputs are outside the contract.
 *
 * Layouts ("compact" = unswizzled, TransformerEngine PR #3244, review):
 *   x         bf16 row-major [rows, cols], leading dimension = cols.
 *   q_row     uint8 [rows, cols/2]      codes of row r, block b at bytes 8b..8b+7.
 *   sf_row    uint8 [rows, cols/16]     E4M3 scale of each 16-element row block.
 *   amax_row  fp32  [rows]
 *   q_col     uint8 [cols, rows/2]      the rowwise cast of x^T ("stored transposed").
 *   sf_col    uint8 [cols, rows/16]
 *   amax_col  fp32  [cols]              (grouped: [num_groups, cols])
 *
 * Conventions shared by every call:
 *   - All array pointers are device pointers owned by the caller; the library keeps
 *     no pointer after the call returns and allocates no device memory.
 *   - Calls are asynchronous: the work is ordered on `stream` (0 = legacy default
 *     stream), and outputs are valid once the stream reaches that point.
 *   - rows and cols are > 0, multiples of 16, and at most 2^30; each pointer that is
 *     used is non-NULL and 16-byte aligned. Violations are reported by the return
 *     value BEFORE anything is launched; nothing is written then.
 *   - A launch or CUDA API failure returns NVFP4PT_ERR_CUDA.
 *   - Calls on one stream may reuse the same workspace; concurrent calls on
 *     different streams need different workspaces.
 *   - The library is for sm_100 (B200) devices only (NVFP4 is a Blackwell format;
 *     PR #3045 gates its path to SM100 the same way): NVFP4PT_ERR_ARCH elsewhere.
 */
#ifndef NVFP4PT_H
#define NVFP4PT_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define NVFP4PT_API __attribute__((visibility("default")))
#else
#define NVFP4PT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4PT_OK = 0,
    NVFP4PT_ERR_NULL = 1,      /* a pointer that the flags require is NULL              */
    NVFP4PT_ERR_SHAPE = 2,     /* rows/cols not in (0, 2^30] or not multiples of 16      */
    NVFP4PT_ERR_ALIGN = 3,     /* a pointer is not 16-byte aligned                      */
    NVFP4PT_ERR_GROUPS = 4,    /* num_groups outside [1, 1024], or offsets not 0 = o[0] <=
                                  o[1] <= ... <= o[G] = rows with every o[g] % 16 == 0   */
    NVFP4PT_ERR_ARCH = 5,      /* the current device is not compute capability 10.0     */
    NVFP4PT_ERR_CUDA = 6,      /* a CUDA call or a kernel launch failed                 */
    NVFP4PT_ERR_FLAGS = 7,     /* flags is not a non-empty subset of ROWWISE|COLWISE    */
    NVFP4PT_ERR_DEVICE = 8     /* a kernel reported a device-side error (see below)     */
} nvfp4pt_status;

/* Output selection. The same meaning, and the same default in the bindings
 * (both directions), in every call: PR #3045's review found split APIs whose
 * columnwise defaults disagreed. */
enum { NVFP4PT_ROWWISE = 1, NVFP4PT_COLWISE = 2 };

/* Maximum number of token groups of nvfp4pt_quantize_grouped. */
#define NVFP4PT_MAX_GROUPS 1024

/* A constant, human-readable name of a status code. Never NULL. */
NVFP4PT_API const char* nvfp4pt_status_string(nvfp4pt_status status);

/* Bytes of device workspace a call with these sizes needs (num_groups = 1 for the
 * ungrouped and weight calls): about num_groups * cols * 2 bytes plus a few hundred.
 * The workspace holds per-call scratch (a device error word, the observed maxima of
 * the absmax update, and the column maxima as bf16 while the columnwise cast runs);
 * it needs no initialisation and its contents after a call are unspecified except for
 * the error word. */
NVFP4PT_API size_t nvfp4pt_workspace_bytes(int64_t rows, int64_t cols, int num_groups);

/*
 * nvfp4pt_quantize -- per-token cast of x[rows, cols] (PR #3045, Description and
 * Changes; the composite "vector amax, then encode" of its sequence diagram).
 *
 * flags      NVFP4PT_ROWWISE and/or NVFP4PT_COLWISE.
 * q_row, sf_row, amax_row   rowwise outputs (required iff ROWWISE, else ignored).
 * q_col, sf_col, amax_col   columnwise outputs (required iff COLWISE, else ignored).
 * absmax_buf NULL, or one fp32 running buffer, updated in place with
 *            New = max(RN(Old * decay), Observed), Observed = max |x| = max(amax_row)
 *            (TransformerEngine PR #3296 "[PTQ] Store FP32 global scaling factors",
 *            Description: decay 0 keeps the latest value, decay 1 the all-time max;
 *            with per-token scales the row amaxes are max-reduced to a scalar).
 * workspace  nvfp4pt_workspace_bytes(rows, cols, 1) bytes of device memory.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_quantize(const void* x_bf16, int64_t rows, int64_t cols, int flags,
                                uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                                uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                                float* absmax_buf, float decay,
                                void* workspace, cudaStream_t stream);

/*
 * nvfp4pt_quantize_grouped -- the cast of MoE token groups in one pass each
 * (PR #3045, Important Files: the grouped per-token quantize helper that splits
 * tokens per expert; its per-group metadata goes up in one batch). Group g is the
 * row range [offsets_host[g], offsets_host[g+1]); empty groups are allowed (the
 * page's helper rejects them; unbalanced routing produces them).
 *
 * offsets_host  HOST array of num_groups+1 row offsets (read during the call only).
 * Rowwise outputs and amax_row are exactly those of nvfp4pt_quantize.
 * amax_col   fp32 [num_groups, cols]: column amax over the group's rows (0 for an
 *            empty group).
 * q_col      group g's codes are [cols, m_g/2] starting at byte cols*offsets[g]/2.
 * sf_col     group g's scales are [cols, m_g/16] starting at byte cols*offsets[g]/16.
 * absmax_bufs NULL, or fp32 [num_groups]: one running buffer per group (one per
 *            grouped GEMM, PR #3296 Important Files), Observed = max over the group's
 *            rows (0 for an empty group, which then only decays).
 * workspace  nvfp4pt_workspace_bytes(rows, cols, num_groups) bytes.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_quantize_grouped(const void* x_bf16, int64_t rows, int64_t cols,
                                        const int64_t* offsets_host, int num_groups, int flags,
                                        uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                                        uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                                        float* absmax_bufs, float decay,
                                        void* workspace, cudaStream_t stream);

/*
 * Columnwise options of nvfp4pt_quantize_grouped_opts (TransformerEngine PR #3045,
 * Changes: opt-in RHT / SR on the per-token path, off by default; its review: the row
 * direction never uses RHT). The pages fix neither the transform nor the random
 * numbers; the readings taken:
 *   NVFP4PT_COL_RHT  each columnwise 16-element block v (16 consecutive rows of a column
 *                    inside a token group) is replaced by v' = (1/4) H16 S v before the
 *                    columnwise cast: H16 the Sylvester Hadamard matrix (entry (i, j) =
 *                    (-1)^popcount(i & j)), S the diagonal of signs with -1 where bit j of
 *                    rht_signs is set. It is evaluated as four radix-2 butterfly stages
 *                    (pairs i, i + h, h = 1, 2, 4, 8: sum and difference, one binary32
 *                    rounding each), then the exact multiply by 1/4. amax_col is then
 *                    max |v'| over the group's rows; the block steps are unchanged.
 *   NVFP4PT_COL_SR   the columnwise E2M1 rounding of y = RN(v * enc) is stochastic: with
 *                    a = |y| < 6 between the E2M1 neighbours lo <= a < hi and the exact
 *                    fraction f = (a - lo) / (hi - lo), the random word r rounds up iff
 *                    r < ceil(f * 2^32); a >= 6 gives 6; the sign is y's. The word of
 *                    element (row m, column k) is output m % 4 of Philox4x32-10 (Salmon
 *                    et al., SC'11) at counter (m / 4, k, lo32(sr_offset), hi32(sr_offset))
 *                    with key (lo32(sr_seed), hi32(sr_seed)).
 * The rowwise direction and the running buffers are those of the call without options.
 */
enum { NVFP4PT_COL_RHT = 1, NVFP4PT_COL_SR = 2 };
typedef struct nvfp4pt_colwise_options {
    int flags;              /* NVFP4PT_COL_RHT and/or NVFP4PT_COL_SR; 0: none     */
    uint32_t rht_signs;     /* bits 0..15: the sign mask S                        */
    uint64_t sr_seed;       /* Philox key                                         */
    uint64_t sr_offset;     /* Philox counter words 2-3 (e.g. the training step)  */
} nvfp4pt_colwise_options;

/*
 * nvfp4pt_quantize_grouped_opts -- nvfp4pt_quantize_grouped with columnwise options
 * (NULL or flags 0: exactly nvfp4pt_quantize_grouped). One token group (offsets {0,
 * rows}) gives the ungrouped cast's outputs. With options the columnwise direction
 * needs rows of at most 16384 elements (cols <= 16384), else NVFP4PT_ERR_SHAPE; flags
 * outside NVFP4PT_COL_RHT | NVFP4PT_COL_SR give NVFP4PT_ERR_FLAGS. Workspace as in
 * nvfp4pt_quantize_grouped. With NVFP4PT_COL_RHT the call launches one more kernel
 * (the sweep that finds the column amax of the transformed values).
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_quantize_grouped_opts(const void* x_bf16, int64_t rows, int64_t cols,
                                                         const int64_t* offsets_host, int num_groups, int flags,
                                                         uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                                                         uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                                                         float* absmax_bufs, float decay,
                                                         const nvfp4pt_colwise_options* opts, void* workspace,
                                                         cudaStream_t stream);

/*
 * nvfp4pt_quantize_weight_2d -- the opt-in 2D weight cast (PR #3045, Changes:
 * "transposition-invariant 16x16 cast emitted in per-token layout").
 * Each row keeps its own s_enc from amax_row; the 16 rows of a band share one E4M3
 * scale per 16-column block, sf = e4m3(max over the band's rows of
 * RN(RN(block_amax/6) * s_enc[row])), which equals the largest of the 16 rowwise
 * 1D scales; each row encodes with enc = RN(s_enc[row] / float(sf)). The shared
 * scale is written to all 16 rows of the band: sf_row is [rows, cols/16] as in the
 * 1D cast. Weights are kept rowwise only (PR #3296, Description).
 * workspace  nvfp4pt_workspace_bytes(rows, cols, 1) bytes.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_quantize_weight_2d(const void* w_bf16, int64_t rows, int64_t cols,
                                          uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                                          void* workspace, cudaStream_t stream);

/*
 * nvfp4pt_dequantize -- rowwise-layout NVFP4 data back to bf16. The pages keep fp32
 * "scale_inv" factors beside the block scales (PR #3296, title and Description) and
 * dequantize rowwise data before requantizing it (PR #3244, flowchart: "Dequantize",
 * then "Columnwise-only requantize"); the exact formula is not printed. Reading taken:
 * with the decode scale S_dec = RN(amax[r] / 2688) of row r,
 *     out[r][16b + j] = bf16_rn( RN( (val(q) * float(sf[r][b])) * S_dec ) ),
 * val(q) * float(sf) being exact in binary32. An amax of 0 gives signed zeros.
 *
 * q        uint8 [rows, cols/2]  codes, element 2j in the low nibble of byte j.
 * sf       uint8 [rows, cols/16] E4M3 block scales.
 * amax     fp32  [rows]          the rows' amax (as the cast wrote it).
 * out_bf16 bf16  [rows, cols]    written in full.
 * Columnwise data (q_col [cols, rows/2], sf_col [cols, rows/16], amax_col [cols])
 * passed with rows and cols swapped give X^T. Same conventions as the casts (device
 * pointers, 16-byte alignment, sizes multiples of 16, asynchronous on `stream`); no
 * workspace.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_dequantize(const uint8_t* q, const uint8_t* sf, const float* amax,
                                              int64_t rows, int64_t cols, void* out_bf16, cudaStream_t stream);

/* Workspace bytes of nvfp4pt_requantize_colwise: the rows' fp32 decode scales (rows * 4,
 * rounded up to 256) plus nvfp4pt_workspace_bytes(rows, cols, num_groups). */
NVFP4PT_API size_t nvfp4pt_requantize_workspace_bytes(int64_t rows, int64_t cols, int num_groups);

/*
 * nvfp4pt_requantize_colwise -- columnwise NVFP4 data made from rowwise NVFP4 data
 * (the per-token NVFP4 analog of PR #3244's "dequant + requant with col-wise to save
 * for backward", Description and flowchart): the columnwise cast, per token group,
 * of X' = nvfp4pt_dequantize(q_row, sf_row, amax_row).
 *
 * offsets_host  NULL (one group: outputs as nvfp4pt_quantize's columnwise ones) or
 *               num_groups+1 host row offsets as in nvfp4pt_quantize_grouped.
 * q_col, sf_col, amax_col, absmax_bufs, decay: as in nvfp4pt_quantize_grouped's
 *               columnwise direction (absmax_bufs NULL or [groups]; Observed = the
 *               group's max |x'|).
 * workspace     nvfp4pt_requantize_workspace_bytes(rows, cols, groups) bytes.
 * Errors as in nvfp4pt_quantize_grouped, reported before anything is launched.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_requantize_colwise(const uint8_t* q_row, const uint8_t* sf_row,
                                                      const float* amax_row, int64_t rows, int64_t cols,
                                                      const int64_t* offsets_host, int num_groups,
                                                      uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                                                      float* absmax_bufs, float decay, void* workspace,
                                                      cudaStream_t stream);

/* Bytes of the workspace of nvfp4pt_gemm_per_token for an m x n x k product: the device
 * error word, then both operands' block scales rearranged into the layout of the copy
 * into tensor memory (about (m + n) * k / 16 bytes). */
NVFP4PT_API size_t nvfp4pt_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k);

/*
 * nvfp4pt_gemm_per_token -- the GEMM of two per-token NVFP4 operands, rescaled in its
 * epilogue by the per-row and per-column outer-amax vectors (TransformerEngine PR #3045
 * "Add NVFP4 per-token quantization recipe", Description: a CUTLASS GEMM that rescales
 * with the per-row/per-col outer-amax vectors inside the epilogue; Greptile summary: the
 * TN forward, NN data-gradient and NT weight-gradient products). The page prints no
 * formula; the reading taken, with the decode scale S_dec(amax) = RN(amax / 2688) of the
 * dequantization:
 *     acc[m][n] = sum_k val(qa[m][k]) * float(sfa[m][k/16]) * val(qb[n][k]) * float(sfb[n][k/16])
 *     d[m][n]   = RN( RN(acc[m][n] * S_dec(amax_a[m])) * S_dec(amax_b[n]) )
 * Each 16-element block product is exact in binary32; acc is the tensor cores' fp32
 * accumulation of them (block-scaled MMAs of 64 elements, summed in K order), so d
 * differs from the exact value by a few fp32 roundings of the partial sums.
 * Both operands are K-major rowwise data as nvfp4pt_quantize writes it (the rowwise
 * data of a matrix, or the columnwise data of its transpose), so all three products are
 * this one call:
 *   qa, sfa, amax_a  uint8 [m, k/2] codes, uint8 [m, k/16] E4M3 scales, fp32 [m] amax
 *   qb, sfb, amax_b  uint8 [n, k/2], uint8 [n, k/16], fp32 [n]
 *   d                fp32 [m, n] row-major, written in full
 *   workspace        nvfp4pt_gemm_workspace_bytes(m, n, k) bytes; holds the error word that
 *                    nvfp4pt_workspace_error reads (a wait inside the kernel that gave up)
 *                    and, written by the call, the block scales in tensor-memory copy layout
 * Block scales must be non-negative finite E4M3 codes (0x00..0x7E), as the cast writes.
 * m and n are multiples of 16, k a multiple of 256 (a row of block scales is then a
 * whole number of 16-byte units, as the tensor-memory-access copies require), all at
 * most 2^30; pointers 16-byte aligned. Errors as in the casts, before any launch.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_gemm_per_token(const uint8_t* qa, const uint8_t* sfa, const float* amax_a,
                                                  int64_t m, const uint8_t* qb, const uint8_t* sfb,
                                                  const float* amax_b, int64_t n, int64_t k, float* d,
                                                  void* workspace, cudaStream_t stream);

/*
 * nvfp4pt_update_absmax -- the running-buffer step alone (PR #3296, Description):
 * *absmax_buf = max(RN(*absmax_buf * decay), max_i amax_vec[i]); n may be 0
 * (Observed = 0). Both pointers are device pointers; amax_vec holds n non-negative
 * fp32 values. No workspace; n <= 2^40.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_update_absmax(float* absmax_buf, const float* amax_vec, int64_t n,
                                     float decay, cudaStream_t stream);

/*
 * nvfp4pt_quantize_grouped_noalloc -- nvfp4pt_quantize_grouped for callers that cannot
 * allocate device memory (no counterpart in the cast's description: it exists for
 * callers whose code must not allocate -- inside an allocator or memory-pool callback,
 * under a fixed memory budget, or with no workspace to hand over).
 *
 * Same arguments and results as nvfp4pt_quantize_grouped, without the workspace: the
 * scratch lives in a static device array of NVFP4PT_NOALLOC_SCRATCH_BYTES inside the
 * library, which every GPU that loads the library holds until the process exits. The
 * call allocates nothing (no cudaMalloc, no allocating library routine).
 *   - num_groups above NVFP4PT_NOALLOC_MAX_GROUPS (what the array holds) returns
 *     NVFP4PT_ERR_GROUPS before anything is launched.
 *   - Argument errors are reported exactly as nvfp4pt_quantize_grouped reports them,
 *     before any CUDA call (no device is touched for a rejected call).
 *   - The first call on a device looks up the array's device address (with that device
 *     current), and so does the first call after the device's context was replaced
 *     (cudaDeviceReset); make those calls before any stream capture.
 *   - Every call shares the array and clears what it accumulates at its start; calls
 *     that overlap on the GPU (different streams, or different host threads) race on it.
 *   - The device error word sits in the library's array, where no caller can read it:
 *     a bounded wait that gives up inside a kernel (only the TMA tile path, taken for
 *     rows wider than 16384 elements, has such waits) is not reported by this entry;
 *     the outputs of such a call are then incomplete. Callers that need that report use
 *     nvfp4pt_quantize_grouped with a workspace and nvfp4pt_workspace_error.
 */
#define NVFP4PT_NOALLOC_SCRATCH_BYTES 1024
#define NVFP4PT_NOALLOC_MAX_GROUPS 252
NVFP4PT_API nvfp4pt_status nvfp4pt_quantize_grouped_noalloc(const void* x_bf16, int64_t rows, int64_t cols,
                                        const int64_t* offsets_host, int num_groups, int flags,
                                        uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                                        uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                                        float* absmax_bufs, float decay, cudaStream_t stream);

/*
 * nvfp4pt_workspace_error -- read the device error word the last call on this
 * workspace left (0 = none). Synchronises `stream`. A nonzero word means a kernel
 * gave up a bounded wait (a TMA copy that never arrived) and skipped the rest of its
 * work; outputs of that call are then incomplete. Returns NVFP4PT_ERR_DEVICE if the
 * word is nonzero, NVFP4PT_OK otherwise (the word is stored in *word if non-NULL).
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_workspace_error(const void* workspace, uint32_t* word, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4PT_H */
