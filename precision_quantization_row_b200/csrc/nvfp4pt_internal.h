// Library-internal entry points shared between the library's translation units (not
// exported: the library is built with hidden visibility).
#pragma once

#include "nvfp4pt.h"

namespace nvfp4pt {

// Workspace bytes of a call whose workspace holds only the error word and the
// observed maxima (the column maxima then go to amax_col by fp32 atomics).
size_t small_workspace_bytes(int num_groups);

// The host-side argument checks of nvfp4pt_quantize_grouped, in its order (NULL,
// shape, flags, alignment, token groups); no CUDA call. need_workspace = false skips
// the workspace pointer (the entry without allocation has none).
nvfp4pt_status check_grouped_args(const void* x, int64_t rows, int64_t cols, const int64_t* offsets, int num_groups,
                                  int flags, const uint8_t* q_row, const uint8_t* sf_row, const float* amax_row,
                                  const uint8_t* q_col, const uint8_t* sf_col, const float* amax_col,
                                  const float* absmax_bufs, const void* workspace, bool need_workspace);

// NVFP4PT_OK when the current device is an sm_100 device (its one-time kernel
// attributes then set), else NVFP4PT_ERR_ARCH or NVFP4PT_ERR_CUDA.
nvfp4pt_status check_device();

// nvfp4pt_quantize_grouped; full_ws = false for a workspace of small_workspace_bytes.
nvfp4pt_status quantize_grouped_ws(const void* x, int64_t rows, int64_t cols, const int64_t* offsets,
                                   int num_groups, int flags, uint8_t* q_row, uint8_t* sf_row, float* amax_row,
                                   uint8_t* q_col, uint8_t* sf_col, float* amax_col, float* absmax_bufs, float decay,
                                   void* workspace, cudaStream_t stream, bool full_ws);

}  // namespace nvfp4pt
