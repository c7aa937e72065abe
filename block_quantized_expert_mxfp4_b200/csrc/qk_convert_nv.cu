// qk_convert_nv.cu -- quant_convert_nvfp4_to_mxfp4: scale-only NVFP4 -> MXFP4.
//
// "DeepSeek-v4-Flash-REAP-K180-NVFP4", "NVFP4: lossless MXFP4->NVFP4
// conversion" defines both formats (NVFP4: an e4m3 scale per 16 and an fp32
// scale_2 per expert; MXFP4: an e8m0 scale 2^(c-127) per 32) and the forward
// direction; this is the reverse, for the blocks where it is exact.  A
// 32-block's half scales e4m3(s0) * scale_2 and e4m3(s1) * scale_2 (exact in
// fp64: at most 4 + 24 significant bits) convert exactly when they are equal
// and a power of two 2^p, -127 <= p <= 127: code p + 127.  Any other block is
// counted once in n_inexact and takes the code whose power of two is nearest
// in log2 to the larger magnitude (mantissa below sqrt 2 -> 2^p, else
// 2^(p+1), clamped to 0 .. 254; 0 for two zero scales).  A NaN e4m3 code or a
// non-finite product writes code 255 and records QK_ERR_NAN_SCALE.  Nibbles
// are not read or written.
//
// Pure HBM traffic (2 bytes in, 1 byte out per block): one thread per block,
// grid-stride over all experts' blocks.
#include <algorithm>

#include "qk_common.cuh"
#include "qk_convert_nv.h"

namespace qk {

constexpr int kNvThreads = 256;

__global__ void __launch_bounds__(kNvThreads)
    k_convert_nv(const uint8_t* __restrict__ e4m3, const float* __restrict__ scale_2, int64_t per,
                 int64_t total, uint8_t* __restrict__ e8m0, unsigned long long* __restrict__ n_inexact) {
  __shared__ unsigned s_cnt[kNvThreads / 32];
  unsigned cnt = 0;
  bool nan = false;
  for (int64_t i = (int64_t)blockIdx.x * kNvThreads + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * kNvThreads) {
    const double s2 = (double)__ldg(scale_2 + i / per);
    const double a = nv_e4m3_to_double(__ldg(e4m3 + 2 * i)) * s2;
    const double b = nv_e4m3_to_double(__ldg(e4m3 + 2 * i + 1)) * s2;
    bool inexact = false;
    e8m0[i] = (uint8_t)nv_block_code(a, b, inexact, nan);
    cnt += inexact ? 1u : 0u;
  }
  if (nan) set_status(QK_ERR_NAN_SCALE);
#pragma unroll
  for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) s_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long tot = 0;
    for (int w = 0; w < kNvThreads / 32; ++w) tot += s_cnt[w];
    if (tot) atomicAdd(n_inexact, tot);
  }
}

qk_status convert_nv_launch(const uint8_t* e4m3, const float* scale_2, int E, int N, int K, uint8_t* e8m0,
                            unsigned long long* n_inexact, cudaStream_t st) {
  if (cudaMemsetAsync(n_inexact, 0, sizeof(unsigned long long), st) != cudaSuccess) return QK_ERR_CUDA;
  const int64_t per = (int64_t)N * (K / 32), total = per * E;
  if (total == 0) return QK_OK;
  const int64_t want = (total + kNvThreads - 1) / kNvThreads;
  const int grid = (int)std::min<int64_t>(want, (int64_t)num_sms() * 8);
  k_convert_nv<<<grid, kNvThreads, 0, st>>>(e4m3, scale_2, per, total, e8m0, n_inexact);
  return cudaGetLastError() == cudaSuccess ? QK_OK : QK_ERR_CUDA;
}

}  // namespace qk
