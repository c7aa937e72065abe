// qk_fp8.h -- FP8 block-scaled linear / shared-expert launches with a choice
// of scale tile (qk_fp8.cu): blk = 128 (128x128 tiles) or 32 (32x32 tiles).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "qk.h"

namespace qk {
qk_status fp8_linear_launch_blk(const void* x, int M, int K, const uint8_t* w, const uint8_t* ws, int N,
                                void* y, int y_bf16, int blk, cudaStream_t st);
qk_status fp8_ffn_launch_blk(const void* x, int M, int H, int I, const uint8_t* wg, const uint8_t* sg,
                             const uint8_t* wu, const uint8_t* su, const uint8_t* wd, const uint8_t* sd,
                             float* y, void* ws, int blk, cudaStream_t st);
}  // namespace qk
