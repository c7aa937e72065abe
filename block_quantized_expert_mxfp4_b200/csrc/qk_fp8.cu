// qk_fp8.cu -- FP8 E4M3 linear layers with one UE8M0 scale per 128x128 tile
// (or per 32x32 tile).
//
// "DeepSeek-V4-Flash-IQ2XXS-Q2K-FP8-120GB-target", component table: dense
// linears are FP8 E4M3, block-128, UE8M0 scales; "DeepSeek-V4-Flash-W4A16-FP8"
// stores attention as FP8_BLOCK 128x128.  Used here for the shared expert
// (a SwiGLU FFN that is added to the routed output) and as a plain linear.
//
// Same structure as the decode kernels: a work unit is a 16-row weight tile
// over the full reduction length, copied by the bulk-copy engine into padded
// shared rows; eight warps split the reduction in 128-wide scale chunks.
// e4m3 -> f16 is exact (hardware e4m3x2 -> f16x2), products run on the
// tensor cores (m16n8k16, fp32 accumulate), and the tile scale 2^(s-127)
// multiplies each chunk's fp32 partial.  With 32x32 tiles ("DeepSeek-V4.1-Flash
// mixed-Q2 GGUF (IQ2_XXS gate/up + Q2_K down)", "Recipe": DeepSeek-V4.1 stores
// its FP8 dense weights with 32x32 E8M0 block scales, V4 with 128x128) each
// 32-wide step of a chunk is scaled by its own tile's code; a 16-row unit
// lies in one 32-row tile.
#include <algorithm>

#include "qk_common.cuh"
#include "qk_fp8.h"

namespace qk {

enum Fp8Mode { kLinear = 0, kGateUp = 1, kDownAcc = 2 };

struct Fp8Args {
  const uint16_t* x;      // bf16 [M][K] (kLinear, kGateUp)
  const float* hin;       // fp32 [M][K] (kDownAcc)
  const float* hmax_in;   // [M][K/8]    (kDownAcc)
  const uint8_t* wa;      // rows 0..7 of a unit (all 16 rows unless kGateUp)
  const uint8_t* sa;
  const uint8_t* wb;      // kGateUp: rows 8..15 (up projection)
  const uint8_t* sb;
  int M, K, N, kb;        // N output rows, kb = ceil(K/blk) scale columns
  int blk;                // scale tile edge: 128 or 32
  void* y;                // kLinear: [M][N] fp32/bf16; kDownAcc: fp32 [M][N] (+=)
  int y_bf16;
  float* hout;            // kGateUp: [M][N]
  float* hmax_out;        // kGateUp: [M][N/8]
  int stages, rows_act;
};

struct Fp8Head {
  alignas(8) uint64_t full[kMaxStages];
  alignas(16) float red[kWarps * 32 * 4];  // read and written as float4
  float mx_red[kWarps * kTileN];
  float mx_out[kTileN];
  int shift[kTileN];
  int rows[kTileN];
};
constexpr int kFp8Head = (int)((sizeof(Fp8Head) + 127) / 128 * 128);

__host__ __device__ inline int fp8_row(int K) { return K + 16; }            // bytes per smem row
__host__ __device__ inline int fp8_stage(int K) { return 16 * fp8_row(K); }  // bytes per stage
__host__ __device__ inline int fp8_act_stride(int K) { return K + 16; }      // halves per act row

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) k_fp8(const Fp8Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  Fp8Head& S = *reinterpret_cast<Fp8Head*>(smem);
  __half* act = reinterpret_cast<__half*>(smem + kFp8Head);
  uint8_t* stages = smem + kFp8Head + (size_t)a.rows_act * fp8_act_stride(a.K) * 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nstage = a.stages;
  const int rows_per_unit = MODE == kGateUp ? 8 : 16;
  const int U = a.N / rows_per_unit;
  const int u0 = (int)((int64_t)U * blockIdx.x / gridDim.x);
  const int u1 = (int)((int64_t)U * (blockIdx.x + 1) / gridDim.x);
  const int n = u1 - u0;
  if (MODE == kGateUp) pdl_launch_dependents();
  if (n <= 0) {
    if (MODE == kDownAcc) pdl_wait();
    return;
  }
  const int RS = fp8_row(a.K);
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int i) {
    const int u = u0 + i, s = i % nstage;
    uint8_t* st = stages + (size_t)s * fp8_stage(a.K);
    mbar_arrive_expect_tx(&S.full[s], 16u * a.K);
    const int64_t r0 = (int64_t)u * rows_per_unit;
#pragma unroll 1
    for (int j = 0; j < 16; ++j) {
      const uint8_t* src = (MODE == kGateUp) ? (j < 8 ? a.wa + (r0 + j) * a.K : a.wb + (r0 + j - 8) * a.K)
                                             : a.wa + (r0 + j) * a.K;
      bulk_g2s_evict_first(st + j * RS, src, a.K, &S.full[s], pol);
    }
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < nstage; ++s) mbar_init(&S.full[s], 1);
    fence_mbar_init();
    for (int i = 0; i < min(n, nstage); ++i) issue(i);
  }
  __syncthreads();
  if (MODE == kDownAcc) pdl_wait();  // h / hmax come from the gate/up kernel

  const int ntiles = (a.M + kTileN - 1) / kTileN;
  const bool stage_once = (ntiles == 1);
  auto stage_tile = [&](int tile) {
    const int nt = min(kTileN, a.M - tile * kTileN);
    if (threadIdx.x < kTileN) S.rows[threadIdx.x] = tile * kTileN + min((int)threadIdx.x, nt - 1);
    __syncthreads();
    if (MODE == kDownAcc) {
      float v[kTileN];
      const int R = a.K / 8;
#pragma unroll
      for (int j = 0; j < kTileN; ++j) {
        v[j] = 0.f;
        if (j < nt)
          for (int q = threadIdx.x; q < R; q += blockDim.x)
            v[j] = fmaxf(v[j], __ldcg(a.hmax_in + (size_t)S.rows[j] * R + q));
      }
      block_max8(v, S.mx_red, S.mx_out);
      stage_f32_rows(a.hin, S.rows, nt, a.K, S.mx_out, act, fp8_act_stride(a.K), S.shift);
    } else {
      stage_bf16_rows(a.x, S.rows, nt, a.K, act, fp8_act_stride(a.K), S.shift, S.mx_red, S.mx_out);
    }
  };
  if (stage_once) stage_tile(0);

  const int nk = a.K / 128;
  const int c0 = warp * nk / kWarps, c1 = (warp + 1) * nk / kWarps;
  const int mj = lane >> 3, mr = lane & 7;
  const unsigned long long limit = g_wait_limit_ns;
  bool bad = false;
  for (int i = 0; i < n; ++i) {
    const int u = u0 + i, s = i % nstage;
    const uint8_t* st = stages + (size_t)s * fp8_stage(a.K);
    const bool ready = mbar_wait_bounded(&S.full[s], (i / nstage) & 1, limit);
    if (__syncthreads_or(!ready)) {
      drain_stages(S.full, i, min(n, i + nstage), nstage);
      return;
    }
    const int64_t r0 = (int64_t)u * rows_per_unit;
    const uint8_t* sa_row = a.sa + (r0 / a.blk) * a.kb;
    const uint8_t* sb_row = MODE == kGateUp ? a.sb + (r0 / a.blk) * a.kb : sa_row;
    for (int tile = 0; tile < ntiles; ++tile) {
      const int nt = min(kTileN, a.M - tile * kTileN);
      if (!stage_once) stage_tile(tile);
      const __half* xrow = act + min(g, a.rows_act - 1) * fp8_act_stride(a.K) + 4 * t;
      const uint8_t* lrow = st + ((mj & 1) * 8 + mr) * RS + (mj >> 1) * 16;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c = c0; c < c1 && a.blk == 32; ++c) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {  // one 32x32 scale tile per step
          float d[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t wa0, wb0, wa1, wb1;
          ldmatrix_x4(wa0, wb0, wa1, wb1, lrow + c * 128 + jj * 32);
          const uint2 x0 = *reinterpret_cast<const uint2*>(xrow + c * 128 + jj * 32);
          const uint2 x1 = *reinterpret_cast<const uint2*>(xrow + c * 128 + jj * 32 + 16);
          mma_f16_16816(d, e4m3x2_to_f16x2<0>(wa0), e4m3x2_to_f16x2<0>(wb0),
                        e4m3x2_to_f16x2<1>(wa0), e4m3x2_to_f16x2<1>(wb0), x0.x, x0.y);
          mma_f16_16816(d, e4m3x2_to_f16x2<0>(wa1), e4m3x2_to_f16x2<0>(wb1),
                        e4m3x2_to_f16x2<1>(wa1), e4m3x2_to_f16x2<1>(wb1), x1.x, x1.y);
          const uint32_t ca = __ldg(sa_row + 4 * c + jj), cb = __ldg(sb_row + 4 * c + jj);
          bad |= (ca == 255u) | (cb == 255u);
          const float fa = e8m0_to_f32(ca), fb = e8m0_to_f32(cb);
          acc[0] = fmaf(d[0], fa, acc[0]);
          acc[1] = fmaf(d[1], fa, acc[1]);
          acc[2] = fmaf(d[2], fb, acc[2]);
          acc[3] = fmaf(d[3], fb, acc[3]);
        }
      }
      for (int c = c0; c < c1 && a.blk == 128; ++c) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          uint32_t wa0, wb0, wa1, wb1;
          ldmatrix_x4(wa0, wb0, wa1, wb1, lrow + c * 128 + jj * 32);
          const uint2 x0 = *reinterpret_cast<const uint2*>(xrow + c * 128 + jj * 32);
          const uint2 x1 = *reinterpret_cast<const uint2*>(xrow + c * 128 + jj * 32 + 16);
          mma_f16_16816(d, e4m3x2_to_f16x2<0>(wa0), e4m3x2_to_f16x2<0>(wb0),
                        e4m3x2_to_f16x2<1>(wa0), e4m3x2_to_f16x2<1>(wb0), x0.x, x0.y);
          mma_f16_16816(d, e4m3x2_to_f16x2<0>(wa1), e4m3x2_to_f16x2<0>(wb1),
                        e4m3x2_to_f16x2<1>(wa1), e4m3x2_to_f16x2<1>(wb1), x1.x, x1.y);
        }
        const uint32_t ca = __ldg(sa_row + c), cb = __ldg(sb_row + c);
        bad |= (ca == 255u) | (cb == 255u);
        const float fa = e8m0_to_f32(ca), fb = e8m0_to_f32(cb);
        acc[0] = fmaf(d[0], fa, acc[0]);
        acc[1] = fmaf(d[1], fa, acc[1]);
        acc[2] = fmaf(d[2], fb, acc[2]);
        acc[3] = fmaf(d[3], fb, acc[3]);
      }
      if (reduce_warps(acc, S.red, warp, lane)) {
        if (MODE == kGateUp) {
          float hm[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int col = 2 * t + j;
            hm[j] = 0.f;
            if (col < nt) {
              const float sx = pow2f(S.shift[col]);
              const float hv = silu_mul(acc[j] * sx, acc[2 + j] * sx);
              const int m = tile * kTileN + col;
              a.hout[(size_t)m * a.N + r0 + g] = hv;
              hm[j] = fabsf(hv);
            }
          }
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) hm[j] = fmaxf(hm[j], __shfl_xor_sync(0xffffffffu, hm[j], o));
          if (g == 0)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int col = 2 * t + j;
              if (col < nt) a.hmax_out[(size_t)(tile * kTileN + col) * (a.N / 8) + u] = hm[j];
            }
        } else {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int col = 2 * t + j;
            if (col < nt) {
              const float sx = pow2f(S.shift[col]);
              const size_t o = (size_t)(tile * kTileN + col) * a.N + r0 + g;
              if (MODE == kDownAcc) {
                float* y = reinterpret_cast<float*>(a.y);
                y[o] += acc[j] * sx;
                y[o + 8] += acc[2 + j] * sx;
              } else if (a.y_bf16) {
                __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(a.y);
                y[o] = __float2bfloat16_rn(acc[j] * sx);
                y[o + 8] = __float2bfloat16_rn(acc[2 + j] * sx);
              } else {
                float* y = reinterpret_cast<float*>(a.y);
                y[o] = acc[j] * sx;
                y[o + 8] = acc[2 + j] * sx;
              }
            }
          }
        }
      }
      __syncthreads();
    }
    if (threadIdx.x == 0 && i + nstage < n) issue(i + nstage);
  }
  if (bad) set_status(QK_ERR_NAN_SCALE);
}

static int fp8_plan(int K, int rows_act, size_t budget, size_t& smem) {
  const size_t fixed = kFp8Head + (size_t)rows_act * fp8_act_stride(K) * 2;
  const size_t cap = std::min(budget, (size_t)max_smem_optin());
  int s = kMaxStages;
  while (s > 2 && fixed + (size_t)s * fp8_stage(K) > cap) --s;
  smem = fixed + (size_t)s * fp8_stage(K);
  return smem <= (size_t)max_smem_optin() ? s : 0;
}

template <int MODE>
static qk_status fp8_go(Fp8Args& a, int units, size_t budget, cudaStream_t st, bool pdl) {
  size_t smem = 0;
  a.rows_act = std::min(a.M, kTileN);
  a.stages = fp8_plan(a.K, a.rows_act, budget, smem);
  if (!a.stages) return QK_ERR_UNSUPPORTED;
  const int grid = std::max(1, std::min(num_sms(), units));
  return launch_k(k_fp8<MODE>, smem, grid, a, st, pdl);
}

qk_status fp8_linear_launch(const void* x, int M, int K, const uint8_t* w, const uint8_t* ws, int N,
                            void* y, int y_bf16, cudaStream_t st) {
  return fp8_linear_launch_blk(x, M, K, w, ws, N, y, y_bf16, 128, st);
}

qk_status fp8_linear_launch_blk(const void* x, int M, int K, const uint8_t* w, const uint8_t* ws, int N,
                                void* y, int y_bf16, int blk, cudaStream_t st) {
  Fp8Args a = {};
  a.x = static_cast<const uint16_t*>(x);
  a.wa = w;
  a.sa = ws;
  a.M = M;
  a.K = K;
  a.N = N;
  a.blk = blk;
  a.kb = (K + blk - 1) / blk;
  a.y = y;
  a.y_bf16 = y_bf16;
  return fp8_go<kLinear>(a, N / 16, 200 * 1024, st, false);
}

// From this many rows the shared expert runs on the block-scaled grouped
// GEMMs (tcgen05, e4m3 weights as stored): there the weights are read once
// per 64 (gate/up) or 40 (down) rows of tokens, while this file's kernel is
// shaped for a handful of rows.
constexpr int kFp8BigM = 128;

static bool fp8_big_shape(int M, int H, int I) { return M >= kFp8BigM && H % 512 == 0 && I % 512 == 0; }

static bool fp8_big_eligible(int M, int H, int I, const uint8_t* sg, const uint8_t* su, const uint8_t* sd) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return fp8_big_shape(M, H, I) && al(sg) && al(su) && al(sd);
}

size_t fp8_ffn_workspace_bytes(int M, int H, int I) {
  const size_t small = align256((size_t)M * I * 4) + align256((size_t)M * (I / 8) * 4);
  return fp8_big_shape(M, H, I) ? std::max(small, fp8_group_workspace_bytes(M, H, I)) : small;
}

qk_status fp8_ffn_launch(const void* x, int M, int H, int I, const uint8_t* wg, const uint8_t* sg,
                         const uint8_t* wu, const uint8_t* su, const uint8_t* wd, const uint8_t* sd,
                         float* y, void* ws, cudaStream_t st) {
  return fp8_ffn_launch_blk(x, M, H, I, wg, sg, wu, su, wd, sd, y, ws, 128, st);
}

qk_status fp8_ffn_launch_blk(const void* x, int M, int H, int I, const uint8_t* wg, const uint8_t* sg,
                             const uint8_t* wu, const uint8_t* su, const uint8_t* wd, const uint8_t* sd,
                             float* y, void* ws, int blk, cudaStream_t st) {
  if (fp8_big_eligible(M, H, I, sg, su, sd))
    return fp8_group_forward(x, M, H, I, wg, sg, wu, su, wd, sd, blk, y, ws, st);
  float* h = static_cast<float*>(ws);
  float* hmax = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + align256((size_t)M * I * 4));
  Fp8Args a = {};
  a.x = static_cast<const uint16_t*>(x);
  a.wa = wg;
  a.sa = sg;
  a.wb = wu;
  a.sb = su;
  a.M = M;
  a.K = H;
  a.N = I;
  a.blk = blk;
  a.kb = (H + blk - 1) / blk;
  a.hout = h;
  a.hmax_out = hmax;
  qk_status rc = fp8_go<kGateUp>(a, I / 8, 132 * 1024, st, false);
  if (rc != QK_OK) return rc;
  Fp8Args b = {};
  b.hin = h;
  b.hmax_in = hmax;
  b.wa = wd;
  b.sa = sd;
  b.M = M;
  b.K = I;
  b.N = H;
  b.blk = blk;
  b.kb = (I + blk - 1) / blk;
  b.y = y;
  return fp8_go<kDownAcc>(b, H / 16, 92 * 1024, st, true);
}

}  // namespace qk
