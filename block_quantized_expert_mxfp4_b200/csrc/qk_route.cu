// qk_route.cu -- moe_route_topk: softmax top-k router with renormalised weights.
//
// DeepSeek-V4-Flash routes each token to 6 of 256 experts
// ("DeepSeek-V4-Flash-W4A16-FP8", base-model table).  The selection is made on
// the logits (softmax is monotonic, so the top-k probabilities are the top-k
// logits); equal logits go to the lower expert id.  The renormalised weights
// depend only on the selected logits:
//   w_s = exp(l_s - l_max) / sum_{s'} exp(l_{s'} - l_max).
// One warp per token; the token's logits are staged in shared memory and a
// selected entry is overwritten with NaN (never chosen again).
#include <math.h>

#include "qk_common.cuh"

namespace qk {

constexpr int kRouteWarps = 4;

__global__ void __launch_bounds__(kRouteWarps * 32) k_route(const float* __restrict__ logits, int T,
                                                            int E, int k, int32_t* __restrict__ ids,
                                                            float* __restrict__ w) {
  extern __shared__ float srow[];
  // the expert FFN launched next may start its own prologue now; it waits
  // for this grid's completion before it reads ids and w
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouteWarps + warp;
  if (t >= T) return;
  float* v = srow + (size_t)warp * E;
  for (int i = lane; i < E; i += 32) v[i] = logits[(size_t)t * E + i];
  __syncwarp();
  // lane s keeps slot s (top_k <= 32): no local-memory arrays
  float my_v = -INFINITY;
  int my_i = 0;
  float lmax = -INFINITY;
  for (int s = 0; s < k; ++s) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = lane; i < E; i += 32) {
      const float x = v[i];
      if (x > bv || (x == bv && i < bi)) {
        bv = x;
        bi = i;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    // every lane holds the same (bv, bi); bi is a valid index unless all were NaN
    if (bi >= E) bi = 0;
    if (lane == 0) v[bi] = NAN;
    __syncwarp();
    if (s == 0) lmax = bv;
    if (lane == s) {
      my_v = bv;
      my_i = bi;
    }
  }
  if (!(lmax > -INFINITY) || !isfinite(lmax)) {
    if (lane == 0) set_status(QK_ERR_INVALID_ARG);
  }
  const float ex = lane < k ? expf(my_v - lmax) : 0.f;
  float z = ex;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (lane < k) {
    ids[(size_t)t * k + lane] = my_i;
    w[(size_t)t * k + lane] = ex / z;
  }
}

qk_status route_topk_launch(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                            cudaStream_t st) {
  const int grid = (T + kRouteWarps - 1) / kRouteWarps;
  const size_t smem = (size_t)kRouteWarps * E * sizeof(float);
  return launch_ex(k_route, dim3(grid), dim3(kRouteWarps * 32), smem, st, false, logits, T, E, k, ids, w);
}

}  // namespace qk
