// Diagnostic kernels (nvfp4pt_probe.h, a test-only library): the cast's device conversions run
// over whole input domains so the tests can compare them with the CPU definition.
#include "nvfp4pt_probe.h"
#include "nvfp4pt_device.cuh"

using namespace nvfp4pt;

namespace {

constexpr uint32_t kChunk = 4096;

__device__ __forceinline__ uint32_t probe_code(int which, uint32_t bits)
{
    const float f = __uint_as_float(bits);
    return which == 0 ? (e2m1x2(f, 0.0f) & 0xFu) : (e4m3x2(f, 0.0f) & 0xFFu);
}

// Ranges: [0, 0x7F800000] and [0x80000000, 0xFF800000], each 0x7F800001 patterns.
__global__ void transitions_kernel(int which, uint32_t* out, uint32_t cap, uint32_t* count)
{
    const uint64_t per_range = 0x7F800001ull;
    const uint64_t chunks_per_range = (per_range + kChunk - 1) / kChunk;
    const uint64_t total_chunks = 2 * chunks_per_range;
    for (uint64_t c = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total_chunks;
         c += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t range = c / chunks_per_range;
        const uint64_t first = (c % chunks_per_range) * kChunk;
        const uint64_t last = first + kChunk < per_range ? first + kChunk : per_range;
        const uint32_t base = range ? 0x80000000u : 0u;
        uint32_t prev = first == 0 ? 0xFFFFFFFFu : probe_code(which, base + (uint32_t)(first - 1));
        for (uint64_t i = first; i < last; ++i) {
            const uint32_t bits = base + (uint32_t)i;
            const uint32_t code = probe_code(which, bits);
            if (code != prev) {
                const uint32_t slot = atomicAdd(count, 1u);
                if (slot < cap) {
                    out[2 * (uint64_t)slot] = bits;
                    out[2 * (uint64_t)slot + 1] = code;
                }
            }
            prev = code;
        }
    }
}

__global__ void pairs_kernel(const float* in, int64_t n, uint32_t* out)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float lo = in[2 * i], hi = in[2 * i + 1];
        out[i] = (e2m1x2(lo, hi) & 0xFFu) | (e4m3x2(lo, hi) << 16);
    }
}

__global__ void decode_kernel(float* out)
{
    const uint32_t c = threadIdx.x;
    float lo, hi;
    e4m3x2_decode(c, lo, hi);
    out[c] = lo;
    e4m3x2_decode(c << 8, lo, hi);
    out[256 + c] = hi;
}

__global__ void div6_kernel(float* out)
{
    const uint32_t h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h < 0x7F80u) out[h] = div6(__uint_as_float(h << 16));
}

// For every positive E4M3 divisor and every s with exponent field in [e_lo, e_hi]:
// count where the division used by the cast differs from the IEEE division.
__global__ void e4m3_div_kernel(int e_lo, int e_hi, unsigned long long* mismatches)
{
    __shared__ uint32_t tab[8];
    init_rcp_table(tab);
    __syncthreads();
    const uint64_t per = 1ull << 23;
    const uint64_t total = (uint64_t)(e_hi - e_lo + 1) * per;
    unsigned long long bad = 0;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (uint64_t)gridDim.x * blockDim.x) {
        const uint32_t bits = ((uint32_t)(e_lo + i / per) << 23) | (uint32_t)(i % per);
        const float s = __uint_as_float(bits);
        for (uint32_t c = 1; c <= 0x7E; c += 2) {
            float d0, d1;
            e4m3x2_decode(c | ((c + 1) << 8), d0, d1);
            const float ref0 = fminf(__fdiv_rn(s, d0), FLT_MAX);
            const float ref1 = fminf(__fdiv_rn(s, d1), FLT_MAX);
            const float got0 = fminf(div_by_e4m3(s, d0, tab), FLT_MAX);
            const float got1 = fminf(div_by_e4m3(s, d1, tab), FLT_MAX);
            bad += (__float_as_uint(ref0) != __float_as_uint(got0)) + (__float_as_uint(ref1) != __float_as_uint(got1));
        }
    }
    if (bad) atomicAdd(mismatches, bad);
}

// Both forms of the block-scale step on the same (b0, b1, s0, s1); counts the codes and
// multipliers that differ. Thread (e, m) takes s0 = 2^e-binade significand m and s1 a
// second significand of the same binade; b0 runs over all bf16 magnitudes, b1 the
// other way round. The first thread also takes s = FLT_MAX and s = 1.
__device__ unsigned long long pair_scales_diff(float s0, float s1, const uint32_t* tab)
{
    unsigned long long bad = 0;
    for (uint32_t h = 0; h < 0x7F80u; ++h) {
        const float b0 = __uint_as_float(h << 16);
        const float b1 = __uint_as_float((0x7F7Fu - h) << 16);
        uint32_t sfa, sfb;
        float ea0, ea1, eb0, eb1;
        block_pair_scales(b0, b1, s0, s1, sfa, ea0, ea1, tab);
        block_pair_scales_x2(b0, b1, s0, s1, sfb, eb0, eb1, tab);
        bad += ((sfa & 0xFFFFu) != (sfb & 0xFFFFu)) + (__float_as_uint(ea0) != __float_as_uint(eb0)) +
               (__float_as_uint(ea1) != __float_as_uint(eb1));
    }
    return bad;
}

__global__ void pair_scales_kernel(int e_lo, int e_hi, uint32_t stride, unsigned long long* mismatches)
{
    __shared__ uint32_t tab[8];
    init_rcp_table(tab);
    __syncthreads();
    const uint64_t per = ((1u << 23) - 1) / stride + 1;   // significands 0, stride, ... < 2^23
    const uint64_t total = (uint64_t)(e_hi - e_lo + 1) * per;
    unsigned long long bad = 0;
    const uint64_t t0 = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (uint64_t i = t0; i < total; i += (uint64_t)gridDim.x * blockDim.x) {
        const uint32_t e = (uint32_t)(e_lo + i / per);
        const uint32_t m = (uint32_t)(i % per) * stride;
        const float s0 = __uint_as_float((e << 23) | m);
        const float s1 = __uint_as_float((e << 23) | ((m * 2654435761u) & 0x7FFFFFu));
        bad += pair_scales_diff(s0, s1, tab);
    }
    if (t0 == 0) bad += pair_scales_diff(FLT_MAX, 1.0f, tab) + pair_scales_diff(1.0f, FLT_MAX, tab);
    if (bad) atomicAdd(mismatches, bad);
}

nvfp4pt_status arch_ok()
{
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return NVFP4PT_ERR_CUDA;
    return (major == 10 && minor == 0) ? NVFP4PT_OK : NVFP4PT_ERR_ARCH;
}

nvfp4pt_status last()
{
    return cudaGetLastError() == cudaSuccess ? NVFP4PT_OK : NVFP4PT_ERR_CUDA;
}

}  // namespace

extern "C" {

nvfp4pt_status nvfp4pt_probe_transitions(int which, uint32_t* out, uint32_t capacity, uint32_t* count,
                                         cudaStream_t stream)
{
    if (!out || !count) return NVFP4PT_ERR_NULL;
    if (which != 0 && which != 1) return NVFP4PT_ERR_FLAGS;
    nvfp4pt_status st = arch_ok();
    if (st != NVFP4PT_OK) return st;
    if (cudaMemsetAsync(count, 0, sizeof(uint32_t), stream) != cudaSuccess) return NVFP4PT_ERR_CUDA;
    transitions_kernel<<<148 * 8, 256, 0, stream>>>(which, out, capacity, count);
    return last();
}

nvfp4pt_status nvfp4pt_probe_pairs(const float* in, int64_t n, uint32_t* out, cudaStream_t stream)
{
    if (!in || !out) return NVFP4PT_ERR_NULL;
    if (n <= 0) return NVFP4PT_ERR_SHAPE;
    nvfp4pt_status st = arch_ok();
    if (st != NVFP4PT_OK) return st;
    const int64_t blocks = (n + 255) / 256;
    pairs_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(in, n, out);
    return last();
}

nvfp4pt_status nvfp4pt_probe_e4m3_decode(float* out, cudaStream_t stream)
{
    if (!out) return NVFP4PT_ERR_NULL;
    nvfp4pt_status st = arch_ok();
    if (st != NVFP4PT_OK) return st;
    decode_kernel<<<1, 256, 0, stream>>>(out);
    return last();
}

nvfp4pt_status nvfp4pt_probe_e4m3_div(int exp_lo, int exp_hi, unsigned long long* mismatches, cudaStream_t stream)
{
    if (!mismatches) return NVFP4PT_ERR_NULL;
    if (exp_lo < 1 || exp_hi > 254 || exp_lo > exp_hi) return NVFP4PT_ERR_SHAPE;
    nvfp4pt_status st = arch_ok();
    if (st != NVFP4PT_OK) return st;
    if (cudaMemsetAsync(mismatches, 0, sizeof(unsigned long long), stream) != cudaSuccess) return NVFP4PT_ERR_CUDA;
    e4m3_div_kernel<<<148 * 8, 256, 0, stream>>>(exp_lo, exp_hi, mismatches);
    return last();
}

nvfp4pt_status nvfp4pt_probe_pair_scales(int exp_lo, int exp_hi, unsigned int stride, unsigned long long* mismatches,
                                         cudaStream_t stream)
{
    if (!mismatches) return NVFP4PT_ERR_NULL;
    if (exp_lo < 1 || exp_hi > 254 || exp_lo > exp_hi || stride < 1) return NVFP4PT_ERR_SHAPE;
    nvfp4pt_status st = arch_ok();
    if (st != NVFP4PT_OK) return st;
    if (cudaMemsetAsync(mismatches, 0, sizeof(unsigned long long), stream) != cudaSuccess) return NVFP4PT_ERR_CUDA;
    pair_scales_kernel<<<148 * 4, 256, 0, stream>>>(exp_lo, exp_hi, (uint32_t)stride, mismatches);
    return last();
}

nvfp4pt_status nvfp4pt_probe_div6(float* out, cudaStream_t stream)
{
    if (!out) return NVFP4PT_ERR_NULL;
    nvfp4pt_status st = arch_ok();
    if (st != NVFP4PT_OK) return st;
    div6_kernel<<<(0x7F80 + 255) / 256, 256, 0, stream>>>(out);
    return last();
}

}  // extern "C"
