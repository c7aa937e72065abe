// qk_convert.cu -- quant_convert_mxfp4_to_nvfp4: scale-only MXFP4 -> NVFP4.
//
// "DeepSeek-v4-Flash-REAP-K180-NVFP4", "NVFP4: lossless MXFP4->NVFP4
// conversion": the e2m1 nibbles stay as they are; the e8m0 scale of each
// 32-block becomes two e4m3 scales (one per 16) and each expert gets an fp32
// scale_2.  Lossless requires e4m3(s) * scale_2 = 2^(c-127), so scale_2 is a
// power of two; it is anchored at the expert's largest code c_max:
//   scale_2 = 2^(c_max - 135),   s = e4m3 code of 2^(c - c_max + 8).
// e4m3 holds 2^-9 .. 2^8 exactly; 2^-10 rounds (to nearest even) to 0 and
// smaller values flush to 0 -- those blocks are counted in n_inexact.
//
// One thread-block cluster of kParts CTAs per expert: each CTA reduces the max
// code of its slice, the cluster combines the maxima through distributed
// shared memory, then each CTA maps its slice (re-read from L2) to e4m3.
#include <cooperative_groups.h>

#include "qk_device.cuh"
#include "qk_internal.h"

namespace cg = cooperative_groups;

namespace qk {

constexpr int kParts = 8;  // CTAs per expert (cluster size)
constexpr int kConvThreads = 512;

// e4m3 code of 2^d for d <= 8 (d < -10 and d = -10 round to 0).
__device__ __forceinline__ uint32_t e4m3_pow2_code(int d) {
  if (d >= -6) return (uint32_t)(d + 7) << 3;  // normal: exponent field d+7, mantissa 0
  if (d >= -9) return 1u << (d + 9);           // subnormal: (m/8) * 2^-6 = 2^d -> m = 2^(d+9)
  return 0u;
}

__device__ __forceinline__ uint32_t map_code(uint32_t c, int cmax, unsigned& inexact, bool& nan) {
  if (c == 255u) {
    nan = true;
    return 0x7Fu;
  }
  const int d = (int)c - cmax + 8;
  inexact += (d < -9);
  return e4m3_pow2_code(d);
}

__global__ void __cluster_dims__(kParts, 1, 1) __launch_bounds__(kConvThreads)
    k_convert(const uint8_t* __restrict__ e8m0, int64_t per, uint8_t* __restrict__ e4m3,
              float* __restrict__ scale_2, unsigned long long* __restrict__ n_inexact) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ int s_max;
  __shared__ int s_warp[kConvThreads / 32];
  __shared__ unsigned s_cnt[kConvThreads / 32];
  const int part = (int)cluster.block_rank();
  const int64_t e = blockIdx.x / kParts;
  const uint8_t* src = e8m0 + e * per;
  uint8_t* dst = e4m3 + e * per * 2;
  // slice [c0, c1) of this expert's codes, 16-aligned when `per` is
  const bool vec = (per % 16) == 0;
  const int64_t chunk = vec ? ((per / 16 + kParts - 1) / kParts) * 16 : (per + kParts - 1) / kParts;
  const int64_t c0 = min(per, chunk * part), c1 = min(per, c0 + chunk);

  int m = 0;
  if (vec) {
    for (int64_t i = c0 + 16 * (int64_t)threadIdx.x; i < c1; i += 16 * (int64_t)blockDim.x) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(src + i));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int c = (w[j] >> (8 * b)) & 0xFF;
          if (c != 255) m = max(m, c);
        }
    }
  } else {
    for (int64_t i = c0 + threadIdx.x; i < c1; i += blockDim.x) {
      const int c = src[i];
      if (c != 255) m = max(m, c);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    int mm = 0;
    for (int i = 0; i < kConvThreads / 32; ++i) mm = max(mm, s_warp[i]);
    s_max = mm;
  }
  cluster.sync();
  int cmax = 0;
  for (int r = 0; r < kParts; ++r) cmax = max(cmax, *cluster.map_shared_rank(&s_max, r));
  cluster.sync();  // no CTA leaves while a peer may still read its s_max

  if (part == 0 && threadIdx.x == 0) {
    const int ex = cmax - 135;  // >= -135: exact even as an fp32 subnormal
    scale_2[e] = ex >= -126 ? __uint_as_float((uint32_t)(ex + 127) << 23)
                            : __uint_as_float(1u << (ex + 149));
  }
  unsigned inexact = 0;
  bool nan = false;
  if (vec) {
    for (int64_t i = c0 + 16 * (int64_t)threadIdx.x; i < c1; i += 16 * (int64_t)blockDim.x) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(src + i));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      uint32_t o[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          const uint32_t s0 = map_code((w[j] >> (8 * b)) & 0xFF, cmax, inexact, nan);
          const uint32_t s1 = map_code((w[j] >> (8 * (b + 2))) & 0xFF, cmax, inexact, nan);
          lo |= (s0 | (s0 << 8)) << (16 * b);
          hi |= (s1 | (s1 << 8)) << (16 * b);
        }
        o[2 * j] = lo;
        o[2 * j + 1] = hi;
      }
      uint4* d = reinterpret_cast<uint4*>(dst + 2 * i);
      d[0] = make_uint4(o[0], o[1], o[2], o[3]);
      d[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  } else {
    for (int64_t i = c0 + threadIdx.x; i < c1; i += blockDim.x) {
      const uint32_t s = map_code(src[i], cmax, inexact, nan);
      dst[2 * i] = (uint8_t)s;
      dst[2 * i + 1] = (uint8_t)s;
    }
  }
  if (nan) set_status(QK_ERR_NAN_SCALE);
#pragma unroll
  for (int o = 16; o; o >>= 1) inexact += __shfl_xor_sync(0xffffffffu, inexact, o);
  if ((threadIdx.x & 31) == 0) s_cnt[threadIdx.x >> 5] = inexact;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long tot = 0;
    for (int i = 0; i < kConvThreads / 32; ++i) tot += s_cnt[i];
    if (tot) atomicAdd(n_inexact, tot);
  }
}

qk_status convert_launch(const uint8_t* e8m0, int E, int N, int K, uint8_t* e4m3, float* scale_2,
                         unsigned long long* n_inexact, cudaStream_t st) {
  if (cudaMemsetAsync(n_inexact, 0, sizeof(unsigned long long), st) != cudaSuccess)
    return QK_ERR_CUDA;
  if (E == 0) return QK_OK;
  const int64_t per = (int64_t)N * (K / 32);
  k_convert<<<E * kParts, kConvThreads, 0, st>>>(e8m0, per, e4m3, scale_2, n_inexact);
  return cudaGetLastError() == cudaSuccess ? QK_OK : QK_ERR_CUDA;
}

}  // namespace qk
