// nvfp4pt_quantize_grouped_noalloc: the grouped cast with its scratch in a static
// device array, for callers that cannot allocate device memory themselves -- code
// that runs where the allocator is off limits (inside a custom allocator or a memory
// pool's callback, a stream-ordered region that must not allocate, an embedding with
// a fixed memory budget), or that simply has no workspace to hand over.
//
// The cast's scratch (an error word and one observed maximum per token group) lives
// in g_scratch below instead of a caller-provided workspace; the kernels and the
// launch sequence are those of nvfp4pt_quantize_grouped, with the column maxima
// accumulated in amax_col itself (fp32 atomic max) for want of workspace room.
#include <mutex>

#include "nvfp4pt.h"
#include "nvfp4pt_internal.h"

namespace {

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_scratch[NVFP4PT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device. Host code must not hand the
// symbol itself to a kernel (on the host it is only a stand-in); the address is looked
// up once per device, with that device current, on its first call.
nvfp4pt_status scratch_address(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4PT_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return NVFP4PT_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return NVFP4PT_OK;
}

}  // namespace

extern "C" nvfp4pt_status nvfp4pt_quantize_grouped_noalloc(
    const void* x_bf16, int64_t rows, int64_t cols, const int64_t* offsets_host, int num_groups, int flags,
    uint8_t* q_row, uint8_t* sf_row, float* amax_row, uint8_t* q_col, uint8_t* sf_col, float* amax_col,
    float* absmax_bufs, float decay, cudaStream_t stream)
{
    if (num_groups < 1 || num_groups > NVFP4PT_NOALLOC_MAX_GROUPS ||
        nvfp4pt::small_workspace_bytes(num_groups) > NVFP4PT_NOALLOC_SCRATCH_BYTES)
        return NVFP4PT_ERR_GROUPS;
    void* scratch = nullptr;
    const nvfp4pt_status st = scratch_address(&scratch);
    if (st != NVFP4PT_OK) return st;
    // The cast clears the scratch it accumulates into at the start of every call. The
    // scratch has no room for the bf16 column maxima of a full workspace, so the column
    // maxima accumulate in amax_col by fp32 atomic max instead.
    return nvfp4pt::quantize_grouped_ws(x_bf16, rows, cols, offsets_host, num_groups, flags, q_row, sf_row,
                                        amax_row, q_col, sf_col, amax_col, absmax_bufs, decay, scratch, stream,
                                        false);
}
