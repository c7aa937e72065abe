// qk_convert_nv.h -- the NVFP4 -> MXFP4 scale conversion (qk_convert_nv.cu):
// its per-block rule, and the host launch.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "qk.h"

#ifdef __CUDACC__
#include <cuda_fp16.h>
#include <cuda_fp8.h>

namespace qk {
// e4m3 code -> double, exact (NaN stays NaN).  Host and device.
__host__ __device__ inline double nv_e4m3_to_double(uint8_t c) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return (double)__half2float(__half(h));
}

// e8m0 code of one 32-block from its half scales a = e4m3(s0) * scale_2 and
// b = e4m3(s1) * scale_2 (exact doubles).  Sets `inexact` when the block does
// not convert exactly, `nan` (code 255) for a non-finite scale.  Host and
// device: a CPU test checks it against the oracle over every code pair.
__host__ __device__ inline uint32_t nv_block_code(double a, double b, bool& inexact, bool& nan) {
  if (!isfinite(a) || !isfinite(b)) {
    nan = true;
    return 255u;
  }
  int ex;
  if (a == b && a > 0.0) {
    const double f = frexp(a, &ex);  // a = f * 2^ex, f in [0.5, 1)
    if (f == 0.5 && ex - 1 >= -127 && ex - 1 <= 127) return (uint32_t)(ex - 1 + 127);
  }
  inexact = true;
  const double v = fmax(fabs(a), fabs(b));
  if (v == 0.0) return 0u;
  const double f = frexp(v, &ex);    // v = (2 f) * 2^(ex - 1)
  int p = (2.0 * f < 1.4142135623730951) ? ex - 1 : ex;  // sqrt 2 to double precision
  p = p < -127 ? -127 : (p > 127 ? 127 : p);
  return (uint32_t)(p + 127);
}
}  // namespace qk
#endif

namespace qk {
qk_status convert_nv_launch(const uint8_t* e4m3, const float* scale_2, int E, int N, int K, uint8_t* e8m0,
                            unsigned long long* n_inexact, cudaStream_t st);
}  // namespace qk
