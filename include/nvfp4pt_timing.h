/*
 * nvfp4pt_timing.h -- measurement hook of the NVFP4 per-token cast library.
 *
 * The pages describe no such call: it exists so that a benchmark can time each
 * kernel of the cast with CUDA events on the stream the kernels run on.
 */
#ifndef NVFP4PT_TIMING_H
#define NVFP4PT_TIMING_H

#include "nvfp4pt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Kernel launches of one nvfp4pt_quantize call, and events taken by the timed form. */
#define NVFP4PT_CAST_LAUNCHES 3
#define NVFP4PT_TIMED_EVENTS (NVFP4PT_CAST_LAUNCHES + 1)

/*
 * nvfp4pt_quantize_timed -- nvfp4pt_quantize (same arguments, checks, outputs and
 * error returns) with a CUDA event recorded on `stream` before the first kernel
 * launch (events[0]) and after each launch i (events[i], i = 1..3). The launches are,
 * in order: zeroing of the accumulators; the amax pass (the row pass, which also
 * writes the rowwise outputs, for rows up to 16384 elements); the encode pass (the
 * column pass).
 *
 * events  NULL (the call is then exactly nvfp4pt_quantize) or an array of
 *         NVFP4PT_TIMED_EVENTS cudaEvent_t handles created by the caller on the
 *         current device; the library only records them. Recording an event between
 *         two launches keeps the second from starting before the first ends, so the
 *         times are those of each kernel alone.
 * Nothing is recorded when the call returns an error before launching.
 */
NVFP4PT_API nvfp4pt_status nvfp4pt_quantize_timed(const void* x_bf16, int64_t rows, int64_t cols, int flags,
                                                  uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                                                  uint8_t* q_col, uint8_t* sf_col, float* amax_col,
                                                  float* absmax_buf, float decay, void* workspace,
                                                  cudaStream_t stream, void* const* events);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4PT_TIMING_H */
