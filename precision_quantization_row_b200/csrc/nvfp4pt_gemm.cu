// Host side of nvfp4pt_gemm_per_token (include/nvfp4pt.h): argument checks, the scale
// rearrangement into the workspace, the TMA descriptors of the codes and the launch of
// the tcgen05 kernel.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "nvfp4pt.h"
#include "nvfp4pt_internal.h"
#include "nvfp4pt_gemm.cuh"

using namespace nvfp4pt;

namespace {

constexpr int64_t kMaxDim = int64_t(1) << 30;
constexpr int kMaxDevices = 64;

std::mutex g_mu;
bool g_ready[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

int dev_index()
{
    int dev = 0;
    return cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices ? dev : 0;
}
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The kernel's shared-memory size and the tensor-map encoder, once per device.
nvfp4pt_status gemm_setup()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4PT_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_encode) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return NVFP4PT_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    if (!g_ready[dev]) {
        if (cudaFuncSetAttribute(gemm_per_token_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem) !=
                cudaSuccess ||
            cudaDeviceGetAttribute(&g_sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || g_sms[dev] < 1)
            return NVFP4PT_ERR_CUDA;
        g_ready[dev] = true;
    }
    return NVFP4PT_OK;
}

// A uint8 matrix [rows, row_bytes] (row_bytes a multiple of 16) read in boxes of
// box_rows x box_bytes; rows beyond the matrix read as zero.
nvfp4pt_status byte_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes, uint32_t box_bytes,
                        uint32_t box_rows, CUtensorMapSwizzle swizzle)
{
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_bytes, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
}

int64_t align256(int64_t n) { return (n + 255) & ~int64_t(255); }

// Workspace: the error word, then A's and B's block scales in copy layout (A's rows padded
// to whole 128-row blocks, B's to whole 256-row tiles).
int64_t sfa_pre_bytes(int64_t m, int64_t k) { return align256((m + kGemmBM - 1) / kGemmBM * kGemmBM * (k / 16)); }
int64_t sfb_pre_bytes(int64_t n, int64_t k) { return align256((n + kGemmBN - 1) / kGemmBN * kGemmBN * (k / 16)); }
}  // namespace

extern "C" {
size_t nvfp4pt_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k)
{
    if (m < 0 || n < 0 || k < 0 || m > kMaxDim || n > kMaxDim || k > kMaxDim) return 256;
    return (size_t)(256 + sfa_pre_bytes(m, k) + sfb_pre_bytes(n, k));
}

nvfp4pt_status nvfp4pt_gemm_per_token(const uint8_t* qa, const uint8_t* sfa, const float* amax_a, int64_t m,
                                      const uint8_t* qb, const uint8_t* sfb, const float* amax_b, int64_t n,
                                      int64_t k, float* d, void* workspace, cudaStream_t stream)
{
    if (!qa || !sfa || !amax_a || !qb || !sfb || !amax_b || !d || !workspace) return NVFP4PT_ERR_NULL;
    if (m <= 0 || n <= 0 || k <= 0 || m > kMaxDim || n > kMaxDim || k > kMaxDim || m % 16 || n % 16 ||
        k % kGemmBK || ((m + kGemmBM - 1) / kGemmBM) * ((n + kGemmBN - 1) / kGemmBN) > 0x7FFFFFFF)
        return NVFP4PT_ERR_SHAPE;
    if (!aligned16(qa) || !aligned16(sfa) || !aligned16(amax_a) || !aligned16(qb) || !aligned16(sfb) ||
        !aligned16(amax_b) || !aligned16(d) || !aligned16(workspace))
        return NVFP4PT_ERR_ALIGN;
    nvfp4pt_status st = check_device();
    if (st != NVFP4PT_OK) return st;
    if ((st = gemm_setup()) != NVFP4PT_OK) return st;

    GemmParams p;
    std::memset(&p, 0, sizeof p);
    if ((st = byte_map(&p.tmA, qa, m, k / 2, 128, kGemmBM, CU_TENSOR_MAP_SWIZZLE_128B)) != NVFP4PT_OK ||
        (st = byte_map(&p.tmB, qb, n, k / 2, 128, kGemmBN, CU_TENSOR_MAP_SWIZZLE_128B)) != NVFP4PT_OK)
        return st;
    p.m = m;
    p.n = n;
    p.k = k;
    p.amax_a = amax_a;
    p.amax_b = amax_b;
    p.d = d;
    p.err = static_cast<uint32_t*>(workspace);
    uint8_t* sfa_pre = static_cast<uint8_t*>(workspace) + 256;
    uint8_t* sfb_pre = sfa_pre + sfa_pre_bytes(m, k);
    p.sfa_pre = sfa_pre;
    p.sfb_pre = sfb_pre;
    if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), stream) != cudaSuccess) return NVFP4PT_ERR_CUDA;
    p.m_tiles = (int32_t)((m + kGemmBM - 1) / kGemmBM);
    p.n_tiles = (int32_t)((n + kGemmBN - 1) / kGemmBN);
    const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;
    const int sms = g_sms[dev_index()];
    // the scales in copy layout, then one persistent CTA per SM (or per tile, when there
    // are fewer tiles)
    const int64_t ks = k / kGemmBK;
    const int64_t ma = (int64_t)p.m_tiles * kGemmBM, nb = (int64_t)p.n_tiles * kGemmBN;
    const int ga = (int)std::max<int64_t>(1, std::min<int64_t>((ma * ks + 255) / 256, 8 * (int64_t)sms));
    const int gb = (int)std::max<int64_t>(1, std::min<int64_t>((nb * ks + 255) / 256, 8 * (int64_t)sms));
    gemm_sf_prep<<<ga, 256, 0, stream>>>(sfa, m, ma, ks, sfa_pre);
    gemm_sf_prep<<<gb, 256, 0, stream>>>(sfb, n, nb, ks, sfb_pre);
    const int grid = (int)std::min<int64_t>(tiles, sms);
    gemm_per_token_kernel<<<grid, kGemmThreads, kGemmSmem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
}

}  // extern "C"
