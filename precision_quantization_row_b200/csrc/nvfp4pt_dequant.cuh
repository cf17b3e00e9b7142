// Dequantization of rowwise-layout NVFP4 data (sm_100a): codes [rows, cols/2], E4M3
// block scales [rows, cols/16] and row amaxes [rows] back to bf16 [rows, cols]:
//     x' = bf16_rn( RN( (val(q) * float(sf)) * RN(amax / 2688) ) ),
// the inverse of the cast with the decode scale amax/2688 (the "scale_inv" factor
// the TransformerEngine pages store beside the block scales). val(q) * float(sf) is
// exact in binary32. Columnwise data ([cols, rows/2], ...) give X^T the same way.
//
// Each thread takes one unit of one or two blocks of a row (two when a row holds an even
// number of blocks): 8 or 16 code bytes and the units' scale bytes in, 32 bytes out per
// block, the row's decode scale recomputed per unit. The grid covers every unit once
// up to 128 CTAs per SM and strides beyond that; the short life of each thread keeps
// loads of many units in flight. HBM-bound: 0.5625 B read and 2 B written per element.
#pragma once

#include "nvfp4pt_device.cuh"

namespace nvfp4pt {

struct DequantParams {
    const uint8_t* q;
    const uint8_t* sf;
    const float* amax;
    uint16_t* out;
    int64_t rows;
    int64_t cols;
    int64_t units;    // rows * cols / (16 * blocks per unit)
    int32_t out32;    // out is 32-byte aligned: one store per block
};

// The E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 are bf16 values: high bytes
// 00 3F 3F 3F 40 40 40 40, low bytes 00 00 80 C0 00 40 80 C0. One byte permute per
// table picks the bytes of four codes at once (selector nibble = the code's 3-bit
// magnitude index); the sign goes to bit 15.
__device__ __forceinline__ void e2m1x4_to_bf16(uint32_t codes4, uint32_t& w01, uint32_t& w23)
{
    const uint32_t sel = codes4 & 0x7777u;   // nibble i: magnitude index of element i
    const uint32_t hi = __byte_perm(0x3F3F3F00u, 0x40404040u, sel);   // high byte of element i -> byte i
    const uint32_t lo = __byte_perm(0xC0800000u, 0xC0804000u, sel);   // low byte of element i -> byte i
    // element i's bf16 = hi byte i : lo byte i; elements 0,1 -> w01 (0 in the low half)
    w01 = __byte_perm(lo, hi, 0x5140);
    w23 = __byte_perm(lo, hi, 0x7362);
    // signs: code bit 3 of element i -> bit 15 of its half
    const uint32_t s = codes4 & 0x8888u;
    w01 |= ((s & 0x8u) << 12) | ((s & 0x80u) << 24);
    w23 |= ((s & 0x800u) << 4) | ((s & 0x8000u) << 16);
}

// (bf16(RN(a.lo * m)), bf16(RN(a.hi * m))) for the two exact products in a (binary32
// pair) and the decode scale m, as one bf16x2 word (first element in the low half).
__device__ __forceinline__ uint32_t scale_to_bf16x2(float t0, float t1, float m)
{
    float y0, y1;
    mul2(y0, y1, t0, t1, m);
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y1), "f"(y0));
    return r;
}

// Dequantized values of four consecutive elements (codes4: 4 nibbles, element 0 in the
// low nibble) with block scale s (the decoded E4M3 value) and decode scale m, as two
// bf16x2 words (elements 0,1 and 2,3; first element in the low half).
__device__ __forceinline__ void dequant4(uint32_t codes4, float s, float m, uint32_t& w01, uint32_t& w23)
{
    uint32_t b01, b23;
    e2m1x4_to_bf16(codes4, b01, b23);
    float t0, t1, t2, t3;
    mul2(t0, t1, bf16_lo(b01), bf16_hi(b01), s);   // val * float(sf): exact
    mul2(t2, t3, bf16_lo(b23), bf16_hi(b23), s);
    w01 = scale_to_bf16x2(t0, t1, m);
    w23 = scale_to_bf16x2(t2, t3, m);
}

// One 16-element block (8 code bytes c8, scale code sfc, decode scale m) as the eight
// bf16x2 words a 32-byte load of the same block of x would give.
__device__ __forceinline__ void dequant16(uint2 c8, uint32_t sfc, float m, uint32_t (&w)[8])
{
    float s, s_unused;
    e4m3x2_decode(sfc & 0xFFu, s, s_unused);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const uint32_t word = (h < 2) ? c8.x : c8.y;
        dequant4((word >> (16 * (h & 1))) & 0xFFFFu, s, m, w[2 * h], w[2 * h + 1]);
    }
}

// The 32 output bytes of one block.
__device__ __forceinline__ void store_block(uint16_t* dst, const uint32_t (&w)[8], bool out32)
{
    uint8_t* d = reinterpret_cast<uint8_t*>(dst);
    if (out32) {
        stg32(d, make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]));
    } else {
        *reinterpret_cast<uint4*>(d) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(d + 16) = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

// BPT blocks (1 or 2) per unit; units are numbered row-major, so unit u starts at
// block BPT * u of the flat [rows, cols / 16] block grid.
template <int BPT>
__global__ void __launch_bounds__(256, 8) dequant_rows_kernel(const __grid_constant__ DequantParams p)
{
    const int64_t upr = p.cols / (16 * BPT);   // units per row
    const int64_t stride = (int64_t)gridDim.x * 256;
    for (int64_t u = (int64_t)blockIdx.x * 256 + threadIdx.x; u < p.units; u += stride) {
        const float m = __fdiv_rn(__ldg(p.amax + u / upr), 2688.0f);   // decode scale of the row
        uint32_t w[8];
        if constexpr (BPT == 2) {
            const uint4 c = __ldg(reinterpret_cast<const uint4*>(p.q + 16 * u));   // element 2i low nibble
            const uint32_t s = __ldg(reinterpret_cast<const uint16_t*>(p.sf) + u);
            dequant16(make_uint2(c.x, c.y), s & 0xFFu, m, w);
            store_block(p.out + 32 * u, w, p.out32);
            dequant16(make_uint2(c.z, c.w), s >> 8, m, w);
            store_block(p.out + 32 * u + 16, w, p.out32);
        } else {
            const uint2 c = __ldg(reinterpret_cast<const uint2*>(p.q + 8 * u));
            dequant16(c, __ldg(p.sf + u), m, w);
            store_block(p.out + 16 * u, w, p.out32);
        }
    }
}

}  // namespace nvfp4pt
