/*
 * nvfp4pt_probe.h -- diagnostic entry points of the test-only libnvfp4pt_probe.so
 * (built apart from libnvfp4pt.so, which exports only the cast).
 *
 * They run the exact device functions the cast kernels use (the hardware E2M1/E4M3
 * conversions, the E4M3 decode and the correctly rounded division by 6) over whole
 * input domains, so the tests can compare them with the CPU definition of the
 * formats. They are not part of the cast; like the cast they need an sm_100 device.
 * All array pointers are device pointers; calls are asynchronous on `stream`.
 */
#ifndef NVFP4PT_PROBE_H
#define NVFP4PT_PROBE_H

#include <stdint.h>
#include "nvfp4pt.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Sweep every binary32 bit pattern of [0x00000000, 0x7F800000] (+0 .. +inf) and of
 * [0x80000000, 0xFF800000] (-0 .. -inf) through one device conversion and record
 * where its result changes: for `which` = 0 the E2M1 code (4 bits, as the cast stores
 * it), for `which` = 1 the E4M3 code (8 bits). Each record is two uint32 words
 * (bit pattern, code) at out[2*i], out[2*i+1], i < min(*count, capacity), in no
 * particular order; a record is made at the first pattern of each range and wherever
 * the code differs from the previous pattern's. *count (device, zeroed here) receives
 * the number of records; more than `capacity` means the list was cut.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_probe_transitions(int which, uint32_t* out, uint32_t capacity, uint32_t* count,
                                         cudaStream_t stream);

/*
 * For i < n: the device conversions of the pair (lo = in[2i], hi = in[2i+1]) as the
 * cast packs them: out[i] = e2m1 byte (bits 0-7: lo code in bits 0-3, hi code in 4-7)
 * | e4m3 pair (bits 16-31: lo code in bits 16-23, hi code in bits 24-31).
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_probe_pairs(const float* in, int64_t n, uint32_t* out, cudaStream_t stream);

/*
 * Device decode of every E4M3 code c (0..255): out[c] with c in the low byte of a
 * code pair, out[256 + c] with c in the high byte.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_probe_e4m3_decode(float* out, cudaStream_t stream);

/*
 * The device's division by 6 of the block amax for every non-negative finite bf16
 * value: out[h] = (bf16 bits h as binary32) / 6 for h in [0, 0x7F80).
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_probe_div6(float* out, cudaStream_t stream);

/*
 * The division the cast uses for enc = s_enc / float(sf) against the IEEE division,
 * both clamped to FLT_MAX: for every positive E4M3 divisor and every binary32 s whose
 * exponent field lies in [exp_lo, exp_hi] (1..254), *mismatches (device, zeroed here)
 * receives the number of results that differ in any bit.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_probe_e4m3_div(int exp_lo, int exp_hi, unsigned long long* mismatches,
                                                  cudaStream_t stream);

/*
 * The block-scale step (sf = E4M3(RN(b/6) * s), enc = s / float(sf)) as the cast's
 * packed two-lane form computes it, against its scalar form, which the tests pin to
 * the oracle: for every non-negative finite bf16 block amax b and every `stride`-th
 * significand of s in each binade whose exponent field lies in [exp_lo, exp_hi]
 * (1..254), plus s = FLT_MAX and s = 1, *mismatches (device, zeroed here) receives
 * the number of scale codes or multipliers that differ in any bit. stride >= 1.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_probe_pair_scales(int exp_lo, int exp_hi, unsigned int stride,
                                                     unsigned long long* mismatches, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4PT_PROBE_H */
