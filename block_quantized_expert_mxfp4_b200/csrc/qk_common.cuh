// qk_common.cuh -- helpers shared by the tensor-core GEMV kernels: activation
// staging into f16 shared rows with a per-row power-of-two shift, block
// reductions, cross-warp fragment reduction, and the bounded-wait abort path.
#pragma once

#include <cuda_bf16.h>

#include "qk_device.cuh"
#include "qk_internal.h"

namespace qk {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kTileN = 8;  // token columns per m16n8k16 MMA

// ---------------------------------------------------------- small helpers --
__device__ __forceinline__ float pow2f(int s) {  // 2^s, |s| <= 126
  return __uint_as_float((uint32_t)(127 + s) << 23);
}

__device__ __forceinline__ int clamp_shift(int s) { return max(-100, min(100, s)); }

// Block-wide max of up to kTileN values per thread; result in out[j] (smem).
__device__ inline void block_max8(float (&v)[kTileN], float* red /*[kWarps][kTileN]*/, float* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int j = 0; j < kTileN; ++j) {
    float m = v[j];
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp * kTileN + j] = m;
  }
  __syncthreads();
  if (threadIdx.x < kTileN) {
    float m = 0.f;
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w * kTileN + threadIdx.x]);
    out[threadIdx.x] = m;
  }
  __syncthreads();
}

// Stage `nt` activation rows (bf16 [.][K] at rows[j]) into f16 smem rows,
// scaled by 2^-shift[j]; shift[j] chosen from the row's absmax.
__device__ inline void stage_bf16_rows(const uint16_t* __restrict__ x, const int* rows, int nt, int K,
                                __half* dst, int dst_stride, int* shift, float* red, float* tmp) {
  float v[kTileN];
  const int chunks = K / 8;
#pragma unroll
  for (int j = 0; j < kTileN; ++j) {
    v[j] = 0.f;
    if (j < nt) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)rows[j] * K);
      for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
        const uint4 q = __ldg(src + c);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float a = bf16_bits_to_f32(w[i] & 0xFFFFu), b = bf16_bits_to_f32(w[i] >> 16);
          if (!(finite_bits(a) && finite_bits(b))) set_status(QK_ERR_NONFINITE);
          v[j] = fmaxf(v[j], fabsf(a));
          v[j] = fmaxf(v[j], fabsf(b));
        }
      }
    }
  }
  block_max8(v, red, tmp);
  if (threadIdx.x < kTileN) shift[threadIdx.x] = clamp_shift(f16_shift_for(tmp[threadIdx.x]));
  __syncthreads();
  for (int j = 0; j < nt; ++j) {
    const float sc = pow2f(-shift[j]);
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)rows[j] * K);
    uint4* d = reinterpret_cast<uint4*>(dst + (size_t)j * dst_stride);
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      const uint4 q = __ldg(src + c);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = pack_f16x2(bf16_bits_to_f32(w[i] & 0xFFFFu) * sc, bf16_bits_to_f32(w[i] >> 16) * sc);
      d[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  __syncthreads();
}

// Stage `nt` fp32 rows h[rows[j]][K] into f16 smem rows, scaled by
// 2^-shift[j] with shift from amax[j] (already reduced).
__device__ inline void stage_f32_rows(const float* __restrict__ h, const int* rows, int nt, int K,
                               const float* amax, __half* dst, int dst_stride, int* shift) {
  if (threadIdx.x < kTileN) shift[threadIdx.x] = clamp_shift(f16_shift_for(amax[threadIdx.x]));
  __syncthreads();
  const int chunks = K / 8;
  for (int i = threadIdx.x; i < nt * chunks; i += blockDim.x) {
    const int j = i / chunks, c = i - j * chunks;
    const float sc = pow2f(-shift[j]);
    const float4* src = reinterpret_cast<const float4*>(h + (size_t)rows[j] * K) + 2 * c;
    const float4 a = __ldcg(src), b = __ldcg(src + 1);
    uint4 o;
    o.x = pack_f16x2(a.x * sc, a.y * sc);
    o.y = pack_f16x2(a.z * sc, a.w * sc);
    o.z = pack_f16x2(b.x * sc, b.y * sc);
    o.w = pack_f16x2(b.z * sc, b.w * sc);
    reinterpret_cast<uint4*>(dst + (size_t)j * dst_stride)[c] = o;
  }
  __syncthreads();
}

// Sum the 8 warps' fragments into warp 0's registers.
__device__ __forceinline__ bool reduce_warps(float (&acc)[4], float* red, int warp, int lane) {
  reinterpret_cast<float4*>(red)[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  __syncthreads();
  if (warp != 0) return false;
  float4 s = reinterpret_cast<float4*>(red)[lane];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) {
    const float4 v = reinterpret_cast<float4*>(red)[w * 32 + lane];
    s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
  }
  acc[0] = s.x; acc[1] = s.y; acc[2] = s.z; acc[3] = s.w;
  return true;
}

// Abort path after a bounded wait ran out: record it, drain the copies this
// CTA still has in flight (bounded), and let the caller return.
__device__ inline void drain_stages(uint64_t* full, int from, int to, int S) {
  if (threadIdx.x == 0) {
    set_status(QK_ERR_TIMEOUT);
    for (int j = from; j < to; ++j) mbar_wait_bounded(&full[j % S], (j / S) & 1, kDrainLimitNs);
  }
  __syncthreads();
}

// ------------------------------------------------------------- host side --
inline int device_attr(cudaDeviceAttr attr) {
  int dev = 0, v = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&v, attr, dev);
  return v;
}

inline int num_sms() { return device_attr(cudaDevAttrMultiProcessorCount); }
inline int max_smem_optin() { return device_attr(cudaDevAttrMaxSharedMemoryPerBlockOptin); }

// Launch kernel<<<grid, block, smem, st>>>(args...), optionally as a
// programmatic dependent launch of the previous kernel on the stream, with
// the shared-memory attribute set once per kernel and device (smem_attr).
template <typename... KArgs, typename... Args>
inline qk_status launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                           bool pdl, Args&&... args) {
  if (!smem_attr(reinterpret_cast<const void*>(kernel), smem)) return QK_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess && smem > 48 * 1024) {  // the attribute may have been cleared (device reset)
    (void)cudaGetLastError();
    smem_attr_forget(reinterpret_cast<const void*>(kernel));
    if (!smem_attr(reinterpret_cast<const void*>(kernel), smem)) return QK_ERR_CUDA;
    e = cudaLaunchKernelEx(&cfg, kernel, args...);
  }
  return e == cudaSuccess ? QK_OK : QK_ERR_CUDA;
}

// Launch `kernel<<<grid, kThreads, smem, st>>>(args)` (see launch_ex).
template <typename Kern, typename Args>
inline qk_status launch_k(Kern kernel, size_t smem, int grid, const Args& args, cudaStream_t st,
                          bool pdl) {
  return launch_ex(kernel, dim3(grid), dim3(kThreads), smem, st, pdl, args);
}

}  // namespace qk
