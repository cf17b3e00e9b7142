// Host side of the C ABI declared in include/nvfp4pt.h and nvfp4pt_timing.h: argument
// checks, the workspace layout, and the launches on the caller's stream (zero -> amax
// pass -> encode pass, chained with programmatic dependent launch): the row pass and
// the column pass for rows up to 16384 elements (also from NVFP4 rowwise data, for the
// requantization), else the TMA tile path; the dequantization kernel.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "nvfp4pt.h"
#include "nvfp4pt_timing.h"
#include "nvfp4pt_internal.h"
#include "nvfp4pt_kernels.cuh"
#include "nvfp4pt_rowpass.cuh"
#include "nvfp4pt_w2d.cuh"
#include "nvfp4pt_colpass.cuh"
#include "nvfp4pt_colpass_tma.cuh"
#include "nvfp4pt_dequant.cuh"
#include "nvfp4pt_requant.cuh"

using namespace nvfp4pt;

namespace {

constexpr int64_t kMaxDim = int64_t(1) << 30;
constexpr int kMaxDevices = 64;

struct DeviceState {
    bool ready = false;
    int sm_count = 0;
    int major = 0;
    int minor = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

template <typename T>
bool aligned16(const T* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device facts and one-time kernel attributes. Only called after all pure
// argument checks have passed.
nvfp4pt_status device_state(DeviceState** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4PT_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4PT_ERR_CUDA;
        if (d.major == 10 && d.minor == 0) {
            const void* encoders[] = {(const void*)pass2_encode<1, false>, (const void*)pass2_encode<1, true>,
                                      (const void*)pass2_encode<kMaxGroups, false>};
            for (const void* f : encoders) {
                if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPass2) != cudaSuccess ||
                    cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
                    return NVFP4PT_ERR_CUDA;
            }
            const void* colpasses[] = {(const void*)colpass<1>, (const void*)colpass<kMaxGroups>,
                                       (const void*)colpass<1, kColOpts>, (const void*)colpass<kMaxGroups, kColOpts>};
            for (const void* f : colpasses) {
                if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemColPass) != cudaSuccess)
                    return NVFP4PT_ERR_CUDA;
            }
            const void* tcols[] = {(const void*)colpass_tma<1>, (const void*)colpass_tma<kMaxGroups>};
            for (const void* f : tcols) {
                if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemColTma) != cudaSuccess ||
                    cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
                    return NVFP4PT_ERR_CUDA;
            }
            // the one-group row passes use a few KB of shared memory: the rest of the SM's
            // on-chip memory is theirs as L1
            const void* rps[] = {(const void*)rowpass<1, 1, 4>, (const void*)rowpass<1, 2, 2>, (const void*)rowpass<1, 1, 2>,
                                 (const void*)rowpass<1, 1, 1>};
            for (const void* f : rps)
                if (cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, 0) != cudaSuccess)
                    return NVFP4PT_ERR_CUDA;
            const void* rq_tiles[] = {(const void*)rq_tile<1, false>, (const void*)rq_tile<1, true>,
                                      (const void*)rq_tile<kMaxGroups, false>, (const void*)rq_tile<kMaxGroups, true>};
            for (const void* f : rq_tiles) {
                if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemRqTile) != cudaSuccess)
                    return NVFP4PT_ERR_CUDA;
            }
            if (!g_encode) {
                cudaDriverEntryPointQueryResult q;
                void* fn = nullptr;
                if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                    q != cudaDriverEntryPointSuccess || !fn)
                    return NVFP4PT_ERR_CUDA;
                g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
            }
        }
        d.ready = true;
    }
    if (d.major != 10 || d.minor != 0) return NVFP4PT_ERR_ARCH;
    *out = &d;
    return NVFP4PT_OK;
}

nvfp4pt_status check_shape(int64_t rows, int64_t cols)
{
    if (rows <= 0 || cols <= 0 || rows > kMaxDim || cols > kMaxDim || rows % 16 || cols % 16)
        return NVFP4PT_ERR_SHAPE;
    return NVFP4PT_OK;
}

// x as a 2D bf16 tensor [rows, cols]; 128-row x 64-column boxes (128 bytes wide, the
// span of the 128-byte swizzle); out-of-range elements read as zero.
nvfp4pt_status encode_map(CUtensorMap* map, const void* x, int64_t rows, int64_t cols)
{
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kTile};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
}

// uint8 matrix [rows, width] (row stride `width` bytes, a multiple of 16) in boxes of
// box_w bytes x box_rows rows, no swizzle; out-of-range bytes read as zero.
nvfp4pt_status encode_u8_map(CUtensorMap* map, const void* base, int64_t rows, int64_t width, int box_w, int box_rows)
{
    cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)width};
    cuuint32_t box[2] = {(cuuint32_t)box_w, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
}

// fp32 vector [n] as a one-row matrix [1, n], in boxes of `box` elements; out-of-range
// elements read as zero.
nvfp4pt_status encode_f32_vector_map(CUtensorMap* map, const float* base, int64_t n, int box)
{
    cuuint64_t dims[2] = {(cuuint64_t)n, 1};
    cuuint64_t strides[1] = {(cuuint64_t)((n * 4 + 15) & ~int64_t(15))};
    cuuint32_t boxd[2] = {(cuuint32_t)box, 1};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
                                boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
}

// Workspace layout: the error word at 0, the observed maxima (one float per group) at
// 16, then -- in a full workspace -- the row pass's bf16 column maxima [G, cols].
int64_t pad4(int64_t n) { return (n + 3) & ~int64_t(3); }
int64_t align256(int64_t n) { return (n + 255) & ~int64_t(255); }
int64_t ws_small_bytes(int64_t groups) { return align256(16 + 4 * pad4(groups)); }
uint32_t* ws_err(void* ws) { return reinterpret_cast<uint32_t*>(ws); }
float* ws_obs(void* ws) { return reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 16); }
uint16_t* ws_colmax(void* ws, int64_t groups)
{
    return reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + ws_small_bytes(groups));
}

template <typename Kernel, typename Params>
cudaError_t launch(Kernel kernel, int grid, int smem, cudaStream_t stream, const Params& p, bool pdl,
                   int threads = kThreads)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

cudaError_t launch_zero(cudaStream_t stream, const ZeroParams& z)
{
    int64_t total = 0;
    for (int k = 0; k < 4; ++k) total += z.ptr[k] ? z.n4[k] : 0;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(148, (total + kThreads - 1) / kThreads));
    return launch(pass0_zero, grid, 0, stream, z, true);
}

// The geometry and group tables of a call (offsets already validated).
template <int MAXG>
void fill_geometry(Geometry& geo, Groups<MAXG>& grp, int64_t rows, int64_t cols, const int64_t* off, int G,
                   int num_ctas_max, int interleave)
{
    geo.rows = rows;
    geo.cols = cols;
    geo.ntc = (int32_t)((cols + kTile - 1) / kTile);
    geo.num_groups = G;
    int64_t bands = 0;
    for (int g = 0; g < G; ++g) {
        grp.band_start[g] = (int32_t)bands;
        grp.row_off[g] = (int32_t)off[g];
        bands += (off[g + 1] - off[g] + kTile - 1) / kTile;
    }
    grp.band_start[G] = (int32_t)bands;
    grp.row_off[G] = (int32_t)off[G];
    geo.total_tiles = bands * geo.ntc;
    const int64_t ranges = std::max<int64_t>(1, std::min<int64_t>(geo.total_tiles, num_ctas_max / interleave));
    geo.interleave = interleave;
    geo.num_ctas = (int32_t)(ranges * interleave);
}

// Shape of the row pass for `cols` columns (cols <= kRowPassMaxCols): blocks per thread
// and row (bt), threads per row (tpr), rows per sweep (rps) and sweeps per batch (S).
constexpr int64_t kRowPassMaxCols = 16384;
struct RowShape {
    int bpr, bt, tpr, rps, S;
};
RowShape row_shape(int64_t cols)
{
    RowShape r;
    r.bpr = (int)(cols / 16);
    r.bt = (r.bpr + kRowThreads - 1) / kRowThreads;
    const int per = (r.bpr + r.bt - 1) / r.bt;
    r.tpr = (per + 31) / 32 * 32;
    r.rps = 1;
    while (r.rps * 2 <= 16 && r.rps * 2 * r.tpr <= kRowThreads) r.rps *= 2;
    r.S = r.bt == 2 ? 2 : std::min(4, 16 / r.rps);
    return r;
}

// One token group, 512-row column tasks: how many of the top row tasks (an even number)
// to cut into 256-row tasks so that the grid-strided walk (warp w takes tasks T-1-w,
// T-1-w-W, ..., so the top rows come last) leaves no warp much more work than the mean.
// Takes the count whose largest per-warp work (in 256-row units) is least, the fewest
// small tasks on ties. The last shape asked for is remembered.
int32_t balanced_small_tasks(int64_t rows, int64_t strips, int64_t warps)
{
    static std::mutex mu;
    static int64_t key[3] = {-1, -1, -1};
    static int32_t val = 0;
    std::lock_guard<std::mutex> lock(mu);
    if (key[0] == rows && key[1] == strips && key[2] == warps) return val;
    int64_t best_units = INT64_MAX;
    int32_t best = 0;
    for (int64_t st = 0; st <= rows / kHalfRows; st += 2) {
        const int64_t big = (rows - st * kHalfRows + kTaskRows - 1) / kTaskRows;
        const int64_t T = (st + big) * strips, S = st * strips;   // tasks; the first S are small
        int64_t worst = 0;
        for (int64_t w = 0; w < warps && w < T; ++w) {
            const int64_t n = (T - 1 - w) / warps + 1;        // warp w's tasks: T-1-w-k*warps, k < n
            const int64_t kfirst = (T - 1 - w >= S) ? (T - 1 - w - S) / warps + 1 : 0;   // first small one
            const int64_t units = 2 * n - (n > kfirst ? n - kfirst : 0);
            worst = units > worst ? units : worst;
        }
        if (worst < best_units) {
            best_units = worst;
            best = (int32_t)st;
        }
    }
    key[0] = rows;
    key[1] = strips;
    key[2] = warps;
    val = best;
    return val;
}

template <int MAXG>
cudaError_t launch_rowpass(const RowShape& rs, const RowParams<MAXG>& rp, cudaStream_t stream)
{
    const int grid = rp.num_ctas;
    if (rs.bt == 2) return launch(rowpass<MAXG, 2, 2>, grid, 0, stream, rp, true, kRowThreads);
    if (rs.S == 4) return launch(rowpass<MAXG, 1, 4>, grid, 0, stream, rp, true, kRowThreads);
    if (rs.S == 2) return launch(rowpass<MAXG, 1, 2>, grid, 0, stream, rp, true, kRowThreads);
    return launch(rowpass<MAXG, 1, 1>, grid, 0, stream, rp, true, kRowThreads);
}

// The columnwise options of a call (nvfp4pt_colwise_options), as the kernels take them.
struct ColOptions {
    bool rht;
    uint32_t rht_signs;
    bool sr;
    uint64_t seed;
    uint64_t offset;
};

template <int MAXG>
nvfp4pt_status run_cast(const void* x, int64_t rows, int64_t cols, const int64_t* off, int G, int flags,
                        uint8_t* q_row, uint8_t* sf_row, float* amax_row, uint8_t* q_col, uint8_t* sf_col,
                        float* amax_col, float* absmax, float decay, bool w2d, void* ws, cudaStream_t stream,
                        void* const* events = nullptr, bool full_ws = true, const ColOptions* co = nullptr)
{
    // events[0] before the first launch, events[i] after the i-th (measurement hook)
    auto mark = [&](int i) -> bool {
        return !events || cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream) == cudaSuccess;
    };
    DeviceState* dev = nullptr;
    nvfp4pt_status st = device_state(&dev);
    if (st != NVFP4PT_OK) return st;

    const bool do_row = (flags & NVFP4PT_ROWWISE) != 0;
    const bool do_col = (flags & NVFP4PT_COLWISE) != 0;
    // The 1D cast of rows up to kRowPassMaxCols wide encodes rows in the amax pass.
    const bool row_pass = !w2d && cols <= kRowPassMaxCols;
    // bf16 column maxima in the workspace (8 columns per atomic), else fp32 atomics
    // With the transform the column amax is of the transformed values: a sweep of its
    // own accumulates it in amax_col, and the row pass takes no column maxima.
    const bool opts = do_col && co && (co->rht || co->sr);
    const bool xf_amax = opts && co->rht;
    uint16_t* colmax = (row_pass && do_col && full_ws && !xf_amax) ? ws_colmax(ws, G) : nullptr;

    ZeroParams z;
    std::memset(&z, 0, sizeof z);
    if (do_row && !row_pass) { z.ptr[0] = reinterpret_cast<float4*>(amax_row); z.n4[0] = rows / 4; }
    if (do_col) { z.ptr[1] = reinterpret_cast<float4*>(amax_col); z.n4[1] = (int64_t)G * cols / 4; }
    if (absmax) { z.ptr[2] = reinterpret_cast<float4*>(ws_obs(ws)); z.n4[2] = pad4(G) / 4; }
    if (colmax) { z.ptr[3] = reinterpret_cast<float4*>(colmax); z.n4[3] = (int64_t)G * cols * 2 / 16; }
    z.err = ws_err(ws);
    if (!mark(0) || launch_zero(stream, z) != cudaSuccess || !mark(1)) return NVFP4PT_ERR_CUDA;

    cudaError_t e;
    if (row_pass) {
        const RowShape rs = row_shape(cols);
        RowParams<MAXG> rp;
        std::memset(&rp, 0, sizeof rp);
        rp.rows = rows;
        rp.cols = cols;
        rp.num_batches = rows / (rs.S * rs.rps);
        rp.bpr = rs.bpr;
        rp.tpr = rs.tpr;
        rp.rps = rs.rps;
        rp.num_ctas = (int32_t)std::min<int64_t>(rp.num_batches, dev->sm_count);
        rp.num_groups = G;
        rp.do_row = do_row;
        rp.strided = G == 1;
        rp.x = static_cast<const uint16_t*>(x);
        rp.amax_row = do_row ? amax_row : nullptr;
        rp.q_row = q_row;
        rp.sf_row = sf_row;
        rp.amax_col = (do_col && !colmax && !xf_amax) ? amax_col : nullptr;
        rp.colmax = reinterpret_cast<uint32_t*>(colmax);
        rp.obs = absmax ? ws_obs(ws) : nullptr;
        for (int g = 0; g <= G; ++g) rp.row_off[g] = (int32_t)off[g];
        e = launch_rowpass<MAXG>(rs, rp, stream);
        if (e != cudaSuccess || !mark(2)) return NVFP4PT_ERR_CUDA;

        // Column pass: 256-row tasks per group (the last one ragged) x 32-column strips.
        // With nothing to encode it runs the running-buffer update alone (one CTA).
        ColParams<MAXG> cp;
        std::memset(&cp, 0, sizeof cp);
        // 512-row tasks (whole 32-byte sectors of column scales) unless that leaves fewer
        // than two tasks per warp of the grid; then 256-row tasks
        const int64_t strips = (cols + kTaskCols - 1) / kTaskCols;
        auto count_tasks = [&](int32_t tr) {
            int64_t t = 0;
            for (int g = 0; g < G; ++g) t += (off[g + 1] - off[g] + tr - 1) / tr;
            return t;
        };
        // The plain encode of one token group with at least four 512-row tasks per warp runs
        // colpass_tma (kTcWarps warps per CTA); smaller or grouped casts and the options
        // run colpass, whose 16 warps per CTA even out fewer tasks.
        const int64_t tasks512 = count_tasks(kTaskRows) * strips;
        const bool tma_col = !opts && MAXG == 1 && tasks512 >= 4 * (int64_t)dev->sm_count * kTcWarps;
        const int64_t cw = tma_col ? kTcWarps : kColWarps;
        cp.task_rows = tasks512 >= 2 * (int64_t)dev->sm_count * cw ? kTaskRows : kHalfRows;
        int32_t tasks = 0;
        for (int g = 0; g < G; ++g) {
            cp.row_off[g] = (int32_t)off[g];
            cp.task_off[g] = tasks;
            tasks += (int32_t)((off[g + 1] - off[g] + cp.task_rows - 1) / cp.task_rows);
        }
        if (MAXG == 1 && cp.task_rows == kTaskRows) {
            // cut the top row tasks in two where that evens out the warps' work (the
            // one-group kernel reads small_tasks; the grouped one keeps one task height)
            const int64_t warps =
                std::max<int64_t>(1, std::min<int64_t>(dev->sm_count, (tasks * strips + cw - 1) / cw)) * cw;
            cp.small_tasks = balanced_small_tasks(rows, strips, warps);
            tasks = cp.small_tasks + (int32_t)((rows - (int64_t)cp.small_tasks * kHalfRows + kTaskRows - 1) / kTaskRows);
        }
        cp.row_off[G] = (int32_t)off[G];
        cp.task_off[G] = tasks;
        cp.cols = cols;
        cp.strips = (int32_t)((cols + kTaskCols - 1) / kTaskCols);
        cp.num_tasks = do_col ? (int64_t)tasks * cp.strips : 0;
        cp.num_ctas = (int32_t)std::max<int64_t>(
            1, std::min<int64_t>(dev->sm_count, (cp.num_tasks + kColWarps - 1) / kColWarps));
        cp.num_groups = G;
        cp.nbuf = absmax ? G : 0;
        cp.decay = decay;
        cp.q_col_32 = (reinterpret_cast<uintptr_t>(q_col) & 31u) == 0;
        cp.strided = G == 1;
        const int64_t wstride = cp.strided ? (int64_t)cp.num_ctas * kColWarps : kColWarps;
        cp.back_rt = (int32_t)(wstride / cp.strips);
        cp.back_strip = (int32_t)(wstride % cp.strips);
        cp.x = static_cast<const uint16_t*>(x);
        cp.amax_col = amax_col;
        cp.colmax = colmax;
        cp.q_col = q_col;
        cp.sf_col = sf_col;
        cp.absmax = absmax;
        cp.obs = ws_obs(ws);
        cp.err = ws_err(ws);
        if (tma_col) {
            // steps copied by TMA (boxes of 32 columns x 64 rows of x)
            ColTmaParams<MAXG> tp;
            std::memset(&tp, 0, sizeof tp);
            tp.c = cp;
            tp.c.num_ctas = (int32_t)std::max<int64_t>(
                1, std::min<int64_t>(dev->sm_count, (cp.num_tasks + kTcWarps - 1) / kTcWarps));
            cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
            cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
            cuuint32_t box[2] = {(cuuint32_t)kTaskCols, (cuuint32_t)kStepRows};
            cuuint32_t estr[2] = {1, 1};
            if (g_encode(&tp.tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return NVFP4PT_ERR_CUDA;
            e = launch(colpass_tma<MAXG>, tp.c.num_ctas, kSmemColTma, stream, tp, true, kTcThreads);
            return e == cudaSuccess && mark(3) ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
        }
        if (opts) {
            cp.rht = co->rht;
            cp.rht_signs = co->rht_signs & 0xFFFFu;
            cp.sr = co->sr;
            cp.sr_key0 = (uint32_t)co->seed;
            cp.sr_key1 = (uint32_t)(co->seed >> 32);
            cp.sr_off0 = (uint32_t)co->offset;
            cp.sr_off1 = (uint32_t)(co->offset >> 32);
            if (xf_amax) {
                ColParams<MAXG> ap = cp;
                ap.absmax = nullptr;
                ap.nbuf = 0;
                if (launch(colpass<MAXG, kColXformAmax>, ap.num_ctas, 0, stream, ap, true, kColThreads) !=
                    cudaSuccess)
                    return NVFP4PT_ERR_CUDA;
            }
            e = launch(colpass<MAXG, kColOpts>, cp.num_ctas, kSmemColPass, stream, cp, true, kColThreads);
            return e == cudaSuccess ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
        }
        e = launch(colpass<MAXG>, cp.num_ctas, kSmemColPass, stream, cp, true, kColThreads);
        return e == cudaSuccess && mark(3) ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
    }

    P2Params<MAXG> p2;
    std::memset(&p2, 0, sizeof p2);
    if ((st = encode_map(&p2.tmap, x, rows, cols)) != NVFP4PT_OK) return st;
    fill_geometry<MAXG>(p2.geo, p2.grp, rows, cols, off, G, 2 * dev->sm_count, 1);
    p2.amax_row = amax_row;
    p2.amax_col = amax_col;
    p2.q_row = q_row;
    p2.sf_row = sf_row;
    p2.q_col = q_col;
    p2.sf_col = sf_col;
    p2.absmax = absmax;
    p2.obs = ws_obs(ws);
    p2.err = ws_err(ws);
    p2.decay = decay;
    p2.nbuf = absmax ? G : 0;
    p2.flags = flags;

    P1Params<MAXG> p1;
    std::memset(&p1, 0, sizeof p1);
    fill_geometry<MAXG>(p1.geo, p1.grp, rows, cols, off, G, 2 * dev->sm_count, 1);
    p1.x = static_cast<const uint16_t*>(x);
    p1.amax_row = do_row ? amax_row : nullptr;
    p1.amax_col = do_col ? amax_col : nullptr;
    p1.obs = absmax ? ws_obs(ws) : nullptr;
    if (do_col) e = launch(pass1_amax<MAXG, true>, p1.geo.num_ctas, 0, stream, p1, true, kThreads);
    else e = launch(pass1_amax<MAXG, false>, p1.geo.num_ctas, 0, stream, p1, true, kThreads);
    if (e != cudaSuccess || !mark(2)) return NVFP4PT_ERR_CUDA;
    if (w2d) e = launch(pass2_encode<MAXG, true>, p2.geo.num_ctas, kSmemPass2, stream, p2, true, kThreads);
    else e = launch(pass2_encode<MAXG, false>, p2.geo.num_ctas, kSmemPass2, stream, p2, true, kThreads);
    return e == cudaSuccess && mark(3) ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
}

cudaError_t launch_dequant(const uint8_t* q, const uint8_t* sf, const float* amax, int64_t rows, int64_t cols,
                           uint16_t* out, int sm_count, cudaStream_t stream)
{
    DequantParams d;
    d.q = q;
    d.sf = sf;
    d.amax = amax;
    d.out = out;
    d.rows = rows;
    d.cols = cols;
    d.out32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    // two blocks per thread when rows hold an even number of blocks (a pair never spans
    // two rows); the grid covers every unit once, up to 128 CTAs per SM
    const bool pairs = (cols / 16) % 2 == 0;
    d.units = rows * (cols / 16) / (pairs ? 2 : 1);
    const int grid = (int)std::min<int64_t>((d.units + 255) / 256, 128 * (int64_t)sm_count);
    if (pairs) dequant_rows_kernel<2><<<grid, 256, 0, stream>>>(d);
    else dequant_rows_kernel<1><<<grid, 256, 0, stream>>>(d);
    return cudaGetLastError();
}

// Requantization scratch ahead of the cast's workspace: the rows' decode scales.
int64_t requant_scratch_bytes(int64_t rows) { return align256(rows * 4); }

// The columnwise requantization (nvfp4pt_requant.cuh): zeroing, rq_colmax, rq_colenc,
// chained by programmatic dependent launch. ws is a full cast workspace (error word,
// observed maxima, bf16 column maxima [G, cols]).
template <int MAXG>
nvfp4pt_status run_requant(const uint8_t* q, const uint8_t* sf, const float* amax, int64_t rows, int64_t cols,
                           const int64_t* off, int G, uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                           float* absmax, float decay, float* dscale, void* ws, cudaStream_t stream)
{
    DeviceState* dev = nullptr;
    const nvfp4pt_status st = device_state(&dev);
    if (st != NVFP4PT_OK) return st;
    uint16_t* colmax = ws_colmax(ws, G);
    ZeroParams z;
    std::memset(&z, 0, sizeof z);
    z.ptr[1] = reinterpret_cast<float4*>(amax_col);
    z.n4[1] = (int64_t)G * cols / 4;
    if (absmax) {
        z.ptr[2] = reinterpret_cast<float4*>(ws_obs(ws));
        z.n4[2] = pad4(G) / 4;
    }
    z.ptr[3] = reinterpret_cast<float4*>(colmax);
    z.n4[3] = (int64_t)G * cols * 2 / 16;
    z.err = ws_err(ws);
    if (launch_zero(stream, z) != cudaSuccess) return NVFP4PT_ERR_CUDA;

    RqParams<MAXG> p;
    std::memset(&p, 0, sizeof p);
    p.q = q;
    p.sf = sf;
    p.amax = amax;
    p.dscale = dscale;
    p.colmax = colmax;
    p.obs = absmax ? ws_obs(ws) : nullptr;
    p.q_col = q_col;
    p.sf_col = sf_col;
    p.amax_col = amax_col;
    p.absmax = absmax;
    p.decay = decay;
    p.nbuf = absmax ? G : 0;
    p.rows = rows;
    p.cols = cols;
    p.chunks = (cols + kRqChunkCols - 1) / kRqChunkCols;
    p.slices = rows / kRqSliceRows;
    p.strips = (int32_t)((cols + kRqStripCols - 1) / kRqStripCols);
    p.num_groups = G;
    int64_t steps = 0;
    for (int g = 0; g < G; ++g) {
        p.row_off[g] = (int32_t)off[g];
        p.step_off[g] = (int32_t)steps;
        steps += (off[g + 1] - off[g] + kRqStepRows - 1) / kRqStepRows;
    }
    p.row_off[G] = (int32_t)rows;
    p.step_off[G] = (int32_t)steps;
    const int64_t sms = dev->sm_count;
    if (cols % kRtCols == 0) {
        // whole 256-column tiles: the TMA-fed kernels
        int64_t tsteps = 0;
        for (int g = 0; g < G; ++g) {
            p.tstep_off[g] = (int32_t)tsteps;
            tsteps += (off[g + 1] - off[g] + kRtRows - 1) / kRtRows;
        }
        p.tstep_off[G] = (int32_t)tsteps;
        p.err = ws_err(ws);
        if (encode_u8_map(&p.tm_q, q, rows, cols / 2, kRtCols / 2, kRtRows) != NVFP4PT_OK ||
            encode_u8_map(&p.tm_sf, sf, rows, cols / 16, kRtCols / 16, kRtRows) != NVFP4PT_OK ||
            encode_f32_vector_map(&p.tm_amax, amax, rows, kRtRows) != NVFP4PT_OK)
            return NVFP4PT_ERR_CUDA;
        const int64_t units = (cols / kRtCols) * tsteps;
        const int grid1 = (int)std::min<int64_t>(units, kRtCtasMax * sms);
        const int grid2 = (int)std::min<int64_t>(units, kRtCtasEnc * sms);
        if (launch(rq_tile<MAXG, false>, grid1, kSmemRqTileMax, stream, p, true, kRtThreads) != cudaSuccess ||
            launch(rq_tile<MAXG, true>, grid2, kSmemRqTile, stream, p, true, kRtThreads) != cudaSuccess)
            return NVFP4PT_ERR_CUDA;
        return NVFP4PT_OK;
    }
    const int64_t warps1 = p.slices * p.chunks, warps2 = steps * p.strips;
    const int grid1 = (int)std::min<int64_t>((warps1 + kRqWarps - 1) / kRqWarps, 3 * sms);
    const int grid2 = (int)std::min<int64_t>((warps2 + kRqWarps - 1) / kRqWarps, 2 * sms);
    if (launch(rq_colmax<MAXG>, grid1, 0, stream, p, true, kRqThreads) != cudaSuccess ||
        launch(rq_colenc<MAXG>, grid2, 0, stream, p, true, kRqThreads) != cudaSuccess)
        return NVFP4PT_ERR_CUDA;
    return NVFP4PT_OK;
}

}  // namespace

extern "C" {

const char* nvfp4pt_status_string(nvfp4pt_status s)
{
    switch (s) {
    case NVFP4PT_OK: return "ok";
    case NVFP4PT_ERR_NULL: return "a required pointer is NULL";
    case NVFP4PT_ERR_SHAPE: return "rows and cols must be in (0, 2^30] and multiples of 16";
    case NVFP4PT_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case NVFP4PT_ERR_GROUPS: return "invalid token groups (count or offsets)";
    case NVFP4PT_ERR_ARCH: return "the current device is not sm_100 (B200)";
    case NVFP4PT_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case NVFP4PT_ERR_FLAGS: return "flags must be a non-empty subset of ROWWISE|COLWISE";
    case NVFP4PT_ERR_DEVICE: return "a kernel reported a device-side error";
    }
    return "unknown status";
}

size_t nvfp4pt_workspace_bytes(int64_t rows, int64_t cols, int num_groups)
{
    (void)rows;
    const int64_t g = num_groups < 1 ? 1 : num_groups;
    const int64_t c = cols < 0 ? 0 : cols;
    return (size_t)(ws_small_bytes(g) + align256(g * c * 2));
}

nvfp4pt_status nvfp4pt_quantize(const void* x, int64_t rows, int64_t cols, int flags, uint8_t* q_row,
                                uint8_t* sf_row, float* amax_row, uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                                float* absmax_buf, float decay, void* workspace, cudaStream_t stream)
{
    return nvfp4pt_quantize_timed(x, rows, cols, flags, q_row, sf_row, amax_row, q_col, sf_col, amax_col, absmax_buf,
                                  decay, workspace, stream, nullptr);
}

nvfp4pt_status nvfp4pt_quantize_timed(const void* x, int64_t rows, int64_t cols, int flags, uint8_t* q_row,
                                      uint8_t* sf_row, float* amax_row, uint8_t* q_col, uint8_t* sf_col,
                                      float* amax_col, float* absmax_buf, float decay, void* workspace,
                                      cudaStream_t stream, void* const* events)
{
    const bool do_row = (flags & NVFP4PT_ROWWISE) != 0;
    const bool do_col = (flags & NVFP4PT_COLWISE) != 0;
    if (!x || !workspace || (do_row && (!q_row || !sf_row || !amax_row)) ||
        (do_col && (!q_col || !sf_col || !amax_col)))
        return NVFP4PT_ERR_NULL;
    nvfp4pt_status st = check_shape(rows, cols);
    if (st != NVFP4PT_OK) return st;
    if (flags & ~(NVFP4PT_ROWWISE | NVFP4PT_COLWISE) || !(do_row || do_col)) return NVFP4PT_ERR_FLAGS;
    if (!aligned16(x) || !aligned16(static_cast<uint8_t*>(workspace)) || (absmax_buf && !aligned16(absmax_buf)) ||
        (do_row && (!aligned16(q_row) || !aligned16(sf_row) || !aligned16(amax_row))) ||
        (do_col && (!aligned16(q_col) || !aligned16(sf_col) || !aligned16(amax_col))))
        return NVFP4PT_ERR_ALIGN;
    const int64_t off[2] = {0, rows};
    return run_cast<1>(x, rows, cols, off, 1, flags, q_row, sf_row, amax_row, q_col, sf_col, amax_col, absmax_buf,
                       decay, false, workspace, stream, events);
}

nvfp4pt_status nvfp4pt_quantize_grouped(const void* x, int64_t rows, int64_t cols, const int64_t* offsets,
                                        int num_groups, int flags, uint8_t* q_row, uint8_t* sf_row,
                                        float* amax_row, uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                                        float* absmax_bufs, float decay, void* workspace, cudaStream_t stream)
{
    return nvfp4pt::quantize_grouped_ws(x, rows, cols, offsets, num_groups, flags, q_row, sf_row, amax_row, q_col,
                                        sf_col, amax_col, absmax_bufs, decay, workspace, stream, true);
}

}  // extern "C"

namespace nvfp4pt {

size_t small_workspace_bytes(int num_groups) { return (size_t)ws_small_bytes(num_groups < 1 ? 1 : num_groups); }

nvfp4pt_status check_grouped_args(const void* x, int64_t rows, int64_t cols, const int64_t* offsets, int num_groups,
                                  int flags, const uint8_t* q_row, const uint8_t* sf_row, const float* amax_row,
                                  const uint8_t* q_col, const uint8_t* sf_col, const float* amax_col,
                                  const float* absmax_bufs, const void* workspace, bool need_workspace)
{
    const bool do_row = (flags & NVFP4PT_ROWWISE) != 0;
    const bool do_col = (flags & NVFP4PT_COLWISE) != 0;
    if (!x || (need_workspace && !workspace) || !offsets || (do_row && (!q_row || !sf_row || !amax_row)) ||
        (do_col && (!q_col || !sf_col || !amax_col)))
        return NVFP4PT_ERR_NULL;
    nvfp4pt_status st = check_shape(rows, cols);
    if (st != NVFP4PT_OK) return st;
    if (flags & ~(NVFP4PT_ROWWISE | NVFP4PT_COLWISE) || !(do_row || do_col)) return NVFP4PT_ERR_FLAGS;
    if (!aligned16(x) || (need_workspace && !aligned16(static_cast<const uint8_t*>(workspace))) ||
        (absmax_bufs && !aligned16(absmax_bufs)) ||
        (do_row && (!aligned16(q_row) || !aligned16(sf_row) || !aligned16(amax_row))) ||
        (do_col && (!aligned16(q_col) || !aligned16(sf_col) || !aligned16(amax_col))))
        return NVFP4PT_ERR_ALIGN;
    if (num_groups < 1 || num_groups > NVFP4PT_MAX_GROUPS || offsets[0] != 0 || offsets[num_groups] != rows)
        return NVFP4PT_ERR_GROUPS;
    for (int g = 0; g < num_groups; ++g)
        if (offsets[g + 1] < offsets[g] || offsets[g] % 16) return NVFP4PT_ERR_GROUPS;
    return NVFP4PT_OK;
}

nvfp4pt_status check_device()
{
    DeviceState* dev = nullptr;
    return device_state(&dev);
}

nvfp4pt_status quantize_grouped_ws(const void* x, int64_t rows, int64_t cols, const int64_t* offsets,
                                   int num_groups, int flags, uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                                   uint8_t* q_col, uint8_t* sf_col, float* amax_col, float* absmax_bufs, float decay,
                                   void* workspace, cudaStream_t stream, bool full_ws)
{
    const nvfp4pt_status st = check_grouped_args(x, rows, cols, offsets, num_groups, flags, q_row, sf_row, amax_row,
                                                 q_col, sf_col, amax_col, absmax_bufs, workspace, true);
    if (st != NVFP4PT_OK) return st;
    return run_cast<kMaxGroups>(x, rows, cols, offsets, num_groups, flags, q_row, sf_row, amax_row, q_col, sf_col,
                                amax_col, absmax_bufs, decay, false, workspace, stream, nullptr, full_ws);
}

}  // namespace nvfp4pt

extern "C" {

nvfp4pt_status nvfp4pt_quantize_grouped_opts(const void* x, int64_t rows, int64_t cols, const int64_t* offsets,
                                             int num_groups, int flags, uint8_t* q_row, uint8_t* sf_row,
                                             float* amax_row, uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                                             float* absmax_bufs, float decay, const nvfp4pt_colwise_options* opts,
                                             void* workspace, cudaStream_t stream)
{
    nvfp4pt_status st = nvfp4pt::check_grouped_args(x, rows, cols, offsets, num_groups, flags, q_row, sf_row,
                                                    amax_row, q_col, sf_col, amax_col, absmax_bufs, workspace, true);
    if (st != NVFP4PT_OK) return st;
    ColOptions co = {};
    if (opts) {
        if (opts->flags & ~(NVFP4PT_COL_RHT | NVFP4PT_COL_SR)) return NVFP4PT_ERR_FLAGS;
        co.rht = (opts->flags & NVFP4PT_COL_RHT) != 0;
        co.sr = (opts->flags & NVFP4PT_COL_SR) != 0;
        co.rht_signs = opts->rht_signs;
        co.seed = opts->sr_seed;
        co.offset = opts->sr_offset;
        if ((co.rht || co.sr) && (flags & NVFP4PT_COLWISE) && cols > kRowPassMaxCols) return NVFP4PT_ERR_SHAPE;
    }
    return run_cast<kMaxGroups>(x, rows, cols, offsets, num_groups, flags, q_row, sf_row, amax_row, q_col, sf_col,
                                amax_col, absmax_bufs, decay, false, workspace, stream, nullptr, true, &co);
}

nvfp4pt_status nvfp4pt_quantize_weight_2d(const void* w, int64_t rows, int64_t cols, uint8_t* q_row,
                                          uint8_t* sf_row, float* amax_row, void* workspace, cudaStream_t stream)
{
    if (!w || !workspace || !q_row || !sf_row || !amax_row) return NVFP4PT_ERR_NULL;
    nvfp4pt_status st = check_shape(rows, cols);
    if (st != NVFP4PT_OK) return st;
    if (!aligned16(w) || !aligned16(static_cast<uint8_t*>(workspace)) || !aligned16(q_row) || !aligned16(sf_row) ||
        !aligned16(amax_row))
        return NVFP4PT_ERR_ALIGN;
    if (cols <= 16 * kW2dMaxThreads) {
        // one sweep: a CTA per 16-row band at a time, a thread per 16-column block
        DeviceState* dev = nullptr;
        if ((st = device_state(&dev)) != NVFP4PT_OK) return st;
        W2dParams p;
        std::memset(&p, 0, sizeof p);
        p.w = static_cast<const uint16_t*>(w);
        p.bands = rows / kW2dRows;
        p.cols = cols;
        p.nbc = (int32_t)(cols / 16);
        p.amax_row = amax_row;
        p.q_row = q_row;
        p.sf_row = sf_row;
        p.err = ws_err(workspace);
        const int threads = std::min(kW2dMaxThreads, (p.nbc + 31) / 32 * 32);
        const int grid = (int)std::min<int64_t>(p.bands, (int64_t)dev->sm_count * (kW2dMaxThreads / threads));
        return launch(w2d_band, grid, 0, stream, p, true, threads) == cudaSuccess ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
    }
    const int64_t off[2] = {0, rows};
    return run_cast<1>(w, rows, cols, off, 1, NVFP4PT_ROWWISE, q_row, sf_row, amax_row, nullptr, nullptr, nullptr,
                       nullptr, 0.0f, true, workspace, stream);
}

nvfp4pt_status nvfp4pt_update_absmax(float* buf, const float* v, int64_t n, float decay, cudaStream_t stream)
{
    if (!buf || (n > 0 && !v)) return NVFP4PT_ERR_NULL;
    if (n < 0 || n > (int64_t(1) << 40)) return NVFP4PT_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(buf) & 3u) || (reinterpret_cast<uintptr_t>(v) & 3u)) return NVFP4PT_ERR_ALIGN;
    DeviceState* dev = nullptr;
    nvfp4pt_status st = device_state(&dev);
    if (st != NVFP4PT_OK) return st;
    update_absmax_kernel<<<1, 1024, 0, stream>>>(buf, v, n, decay);
    return cudaGetLastError() == cudaSuccess ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
}

nvfp4pt_status nvfp4pt_workspace_error(const void* workspace, uint32_t* word, cudaStream_t stream)
{
    if (!workspace) return NVFP4PT_ERR_NULL;
    uint32_t w = 0;
    if (cudaMemcpyAsync(&w, workspace, sizeof w, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return NVFP4PT_ERR_CUDA;
    if (word) *word = w;
    return w ? NVFP4PT_ERR_DEVICE : NVFP4PT_OK;
}

nvfp4pt_status nvfp4pt_dequantize(const uint8_t* q, const uint8_t* sf, const float* amax, int64_t rows, int64_t cols,
                                  void* out_bf16, cudaStream_t stream)
{
    if (!q || !sf || !amax || !out_bf16) return NVFP4PT_ERR_NULL;
    nvfp4pt_status st = check_shape(rows, cols);
    if (st != NVFP4PT_OK) return st;
    if (!aligned16(q) || !aligned16(sf) || !aligned16(amax) || !aligned16(out_bf16)) return NVFP4PT_ERR_ALIGN;
    DeviceState* dev = nullptr;
    if ((st = device_state(&dev)) != NVFP4PT_OK) return st;
    return launch_dequant(q, sf, amax, rows, cols, static_cast<uint16_t*>(out_bf16), dev->sm_count, stream) ==
                   cudaSuccess
               ? NVFP4PT_OK
               : NVFP4PT_ERR_CUDA;
}

size_t nvfp4pt_requantize_workspace_bytes(int64_t rows, int64_t cols, int num_groups)
{
    return (size_t)requant_scratch_bytes(rows < 0 ? 0 : rows) + nvfp4pt_workspace_bytes(rows, cols, num_groups);
}

nvfp4pt_status nvfp4pt_requantize_colwise(const uint8_t* q_row, const uint8_t* sf_row, const float* amax_row,
                                          int64_t rows, int64_t cols, const int64_t* offsets_host, int num_groups,
                                          uint8_t* q_col, uint8_t* sf_col, float* amax_col, float* absmax_bufs,
                                          float decay, void* workspace, cudaStream_t stream)
{
    if (!q_row || !sf_row || !amax_row || !q_col || !sf_col || !amax_col || !workspace) return NVFP4PT_ERR_NULL;
    nvfp4pt_status st = check_shape(rows, cols);
    if (st != NVFP4PT_OK) return st;
    if (!aligned16(q_row) || !aligned16(sf_row) || !aligned16(amax_row) || !aligned16(q_col) || !aligned16(sf_col) ||
        !aligned16(amax_col) || !aligned16(static_cast<uint8_t*>(workspace)) || (absmax_bufs && !aligned16(absmax_bufs)))
        return NVFP4PT_ERR_ALIGN;
    const int64_t one[2] = {0, rows};
    const int64_t* off = offsets_host ? offsets_host : one;
    const int G = offsets_host ? num_groups : 1;
    if (G < 1 || G > NVFP4PT_MAX_GROUPS || off[0] != 0 || off[G] != rows) return NVFP4PT_ERR_GROUPS;
    for (int g = 0; g < G; ++g)
        if (off[g + 1] < off[g] || off[g] % 16) return NVFP4PT_ERR_GROUPS;
    DeviceState* dev = nullptr;
    if ((st = device_state(&dev)) != NVFP4PT_OK) return st;
    float* dscale = static_cast<float*>(workspace);
    void* ws = static_cast<uint8_t*>(workspace) + requant_scratch_bytes(rows);
    if (G == 1)
        return run_requant<1>(q_row, sf_row, amax_row, rows, cols, off, 1, q_col, sf_col, amax_col, absmax_bufs,
                              decay, dscale, ws, stream);
    return run_requant<kMaxGroups>(q_row, sf_row, amax_row, rows, cols, off, G, q_col, sf_col, amax_col,
                                   absmax_bufs, decay, dscale, ws, stream);
}

}  // extern "C"
