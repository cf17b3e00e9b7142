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
#include <cudaTypedefs.h>

#include <mutex>

#include "nvfp4pt.h"
#include "nvfp4pt_internal.h"

namespace {

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_scratch[NVFP4PT_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// The looked-up address of g_scratch on one device, valid for the context it was
// looked up in (a device reset makes a new context, where the array may sit elsewhere).
struct ScratchSlot {
    unsigned long long ctx_id = 0;   // 0: not looked up yet
    void* addr = nullptr;
};

std::mutex g_mu;
ScratchSlot g_slot[kMaxDevices];
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;

// A process-unique id of the current device's context (CUDA 12's context ids are
// never reused), 0 if it cannot be had.
unsigned long long current_context_id()
{
    if (!g_ctx_current || !g_ctx_id) {
        cudaDriverEntryPointQueryResult q1, q2;
        void* f1 = nullptr;
        void* f2 = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || !f1 ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess || !f2)
            return 0;
        g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
        g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
    }
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx || g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of g_scratch on the current device. Host code must not hand the
// symbol itself to a kernel (on the host it is only a stand-in); the address is looked
// up with the device current, on the device's first call and again whenever the
// device's context has changed since (after a device reset).
nvfp4pt_status scratch_address(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4PT_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long id = current_context_id();
    if (id == 0) return NVFP4PT_ERR_CUDA;
    ScratchSlot& s = g_slot[dev];
    if (s.ctx_id != id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();   // leave no error pending for the caller's next check
            return NVFP4PT_ERR_CUDA;
        }
        s.addr = p;
        s.ctx_id = id;
    }
    *out = s.addr;
    return NVFP4PT_OK;
}

}  // namespace

extern "C" nvfp4pt_status nvfp4pt_quantize_grouped_noalloc(
    const void* x_bf16, int64_t rows, int64_t cols, const int64_t* offsets_host, int num_groups, int flags,
    uint8_t* q_row, uint8_t* sf_row, float* amax_row, uint8_t* q_col, uint8_t* sf_col, float* amax_col,
    float* absmax_bufs, float decay, cudaStream_t stream)
{
    // The same host-side checks, in the same order, as nvfp4pt_quantize_grouped, then
    // the limit of the static array, then the device; only then the address lookup.
    nvfp4pt_status st = nvfp4pt::check_grouped_args(x_bf16, rows, cols, offsets_host, num_groups, flags, q_row,
                                                    sf_row, amax_row, q_col, sf_col, amax_col, absmax_bufs, nullptr,
                                                    false);
    if (st != NVFP4PT_OK) return st;
    if (num_groups > NVFP4PT_NOALLOC_MAX_GROUPS ||
        nvfp4pt::small_workspace_bytes(num_groups) > NVFP4PT_NOALLOC_SCRATCH_BYTES)
        return NVFP4PT_ERR_GROUPS;
    if ((st = nvfp4pt::check_device()) != NVFP4PT_OK) return st;
    void* scratch = nullptr;
    if ((st = scratch_address(&scratch)) != NVFP4PT_OK) return st;
    // The cast clears the scratch it accumulates into at the start of every call. The
    // scratch has no room for the bf16 column maxima of a full workspace, so the column
    // maxima accumulate in amax_col by fp32 atomic max instead.
    return nvfp4pt::quantize_grouped_ws(x_bf16, rows, cols, offsets_host, num_groups, flags, q_row, sf_row,
                                        amax_row, q_col, sf_col, amax_col, absmax_bufs, decay, scratch, stream,
                                        false);
}
