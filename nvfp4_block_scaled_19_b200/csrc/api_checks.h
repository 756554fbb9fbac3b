// Checks shared by the C-ABI entry points (api.cu, noalloc.cu), so every
// entry point refuses a bad call in the same way and before any device work.
#pragma once

#include <cstdint>

#include "nvfp4.h"

namespace nvfp4 {

// Arguments of a quantize call: rows >= 0, cols > 0 with cols % 16 == 0,
// rows * cols <= 2^40, a non-NULL scale (or workspace) pointer, x / q / sf
// non-NULL unless rows == 0, and all three 16-byte aligned.
nvfp4_status check_quantize_args(const void *x, int64_t rows, int64_t cols, const void *scale,
                                 const uint8_t *q, const uint8_t *sf);

// The current device, if it can run this library's sm_100a kernels
// (compute capability 10.0); its SM count in *num_sms.
nvfp4_status current_device(int *num_sms);

}  // namespace nvfp4
