// qk_group.cu -- grouped (prefill) path of moe_expert_forward.
//
// For token counts where every routed expert sees many tokens, weights are
// read once per group of tokens instead of once per token tile: the
// (token, slot) pairs are grouped by expert ("DeepSeekv4 Flash for 1x Spark
// [REAP25]", "What's actually different": one grouped GEMM per projection),
// and each projection runs as a grouped GEMM on the 5th-generation tensor
// cores.
//
//   k_grp_count / k_grp_scan / k_grp_scatter
//       counting sort of the pairs by expert; x rows gathered into expert
//       order as f16 scaled by a power of two per row (row maximum in
//       [2^14, 2^15)); the list of token tiles (<= 256 rows of one expert).
//   k_ggemm<gate/up>  per (token tile, 64 gate + 64 up weight rows):
//       D[128 x n] = A . B^T on tcgen05 (kind::f16, fp32 accumulator in TMEM);
//       A = the weight rows dequantized on chip to f16 (interleaved gate/up
//       rows), B = the token tile; epilogue h = silu(g) * u (fp32).
//   k_grp_h16         h rows -> f16 with a power-of-two shift per row.
//   k_ggemm<down>     per (token tile, 128 down rows): d (fp32).
//   k_grp_combine     y[t] = sum_s w[t][s] d[pair(t, s)] in slot order.
//
// Dequantization to f16.  NVFP4: e2m1 x e4m3 is exact in f16 and scale_2 is
// applied in the epilogue.  MXFP4: each weight row is scaled relative to
// its largest e8m0 code c_ref, A = e2m1 * 2^(c - c_ref + 8) (exact in f16 for
// c >= c_ref - 31; smaller blocks lose low bits or flush to 0), and the
// epilogue multiplies the row by 2^(c_ref - 135).
#include <cuda.h>

#include <algorithm>

#include "qk_actq.cuh"
#include "qk_common.cuh"
#include "qk_group.cuh"
#include "qk_tmap.h"

namespace qk {

constexpr int kGM = 128;        // weight rows per tile (tcgen05 M)
constexpr int kGK = 64;         // reduction per stage (one 128-byte f16 row)
constexpr int kGRS = 3;         // packed-weight stages (16 KB: four reduction steps of 128 rows)
constexpr int kGRK = 4;         // reduction steps per packed-weight stage
constexpr int kGAS = 3;         // f16 weight-tile stages (16 KB)
constexpr int kGBS = 3;         // token-tile stages (32 KB: 256 / n reduction steps of n tokens)
constexpr int kGDW = 8;         // dequant / epilogue warps
constexpr int kGEW = 4;         // epilogue warps (one per TMEM lane quadrant)
constexpr int kGThreads = (3 + kGDW + kGEW) * 32;  // weight producer, MMA, token producer, dequant, epilogue
constexpr int kGNBox = 4;       // token-box heights 32, 64, 128, 256

}  // namespace qk

namespace qk {

// ------------------------------------------------------- grouping kernels --
__global__ void k_grp_count(const int32_t* __restrict__ ids, int P, int E, int* __restrict__ counts) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= P) return;
  const int e = ids[p];
  if (e < 0 || e >= E) {
    set_status(QK_ERR_INVALID_ARG);
    return;
  }
  atomicAdd(&counts[e], 1);
}

// One block: exclusive scans of the per-expert pair counts and token-tile
// counts; writes the token-tile list.
// One block: the tile list L of tiles of at most tn rows (with `mx`, also
// each tile's expert extent and each expert's first tile); `first` also
// writes the experts' first sorted rows and resets the scatter cursors.
__global__ void __launch_bounds__(kScanThreads) k_grp_scan(GroupWs W, TileList L, int E, int tn, int mx,
                                                            int first) {
  __shared__ int s_pairs[kScanThreads / 32], s_tiles[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (E + kScanThreads - 1) / kScanThreads;
  const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
  int np = 0, nt = 0;
  for (int e = e0; e < e1; ++e) {
    const int c = W.counts[e];
    np += c;
    nt += (c + tn - 1) / tn;
  }
  int ip = np, it = nt;  // inclusive scans within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, ip, o), b = __shfl_up_sync(0xffffffffu, it, o);
    if (lane >= o) {
      ip += a;
      it += b;
    }
  }
  if (lane == 31) {
    s_pairs[warp] = ip;
    s_tiles[warp] = it;
  }
  __syncthreads();
  if (warp == 0) {
    int a = s_pairs[lane], b = s_tiles[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, a, o), y = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) {
        a += x;
        b += y;
      }
    }
    s_pairs[lane] = a;
    s_tiles[lane] = b;
  }
  __syncthreads();
  int row = ip - np + (warp ? s_pairs[warp - 1] : 0);
  int tile = it - nt + (warp ? s_tiles[warp - 1] : 0);
  for (int e = e0; e < e1; ++e) {
    const int c = W.counts[e];
    const int t0 = tile, cnt = (c + tn - 1) / tn;
    if (first) {
      W.offsets[e] = row;
      W.fill[e] = 0;
    }
    if (mx) L.exp_tile0[e] = t0;
    for (int r = 0; r < c; r += tn, ++tile) {
      L.tile_e[tile] = e;
      L.tile_row0[tile] = row + r;
      L.tile_n[tile] = min(tn, c - r);
      if (mx) {
        L.tile_first[tile] = t0;
        L.tile_cnt[tile] = cnt;
      }
    }
    row += c;
  }
  if (tid == kScanThreads - 1) {
    if (first) W.offsets[E] = row;
    *L.n_tiles = tile;
  }
}

// One block per token: the row maximum, then the row in f16 (scaled by
// 2^-shift) at the sorted position of each of the token's pairs.
__device__ __forceinline__ int block_shift(float m, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return clamp_shift(f16_shift_for(r));
}

__global__ void __launch_bounds__(kRowThreads) k_grp_scatter(GroupWs W, const uint16_t* __restrict__ x,
                                                             const int32_t* __restrict__ ids, int k, int E,
                                                             int H) {
  __shared__ float red[kRowThreads / 32];
  __shared__ int pos[8];
  const int t = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  const int nv = H / 8;
  float m = 0.f;
  bool fin = true;
  for (int j = threadIdx.x; j < nv; j += kRowThreads) {
    const uint4 v = __ldg(src + j);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float a = bf16_bits_to_f32(wv[q] & 0xFFFFu), b = bf16_bits_to_f32(wv[q] >> 16);
      fin &= finite_bits(a) && finite_bits(b);
      m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
    }
  }
  if (!fin) set_status(QK_ERR_NONFINITE);
  const int shift = block_shift(m, red);
  if (threadIdx.x < k) {
    const int p = t * k + threadIdx.x;
    const int e = ids[p];
    int r = -1;
    if (e >= 0 && e < E) {
      r = W.offsets[e] + atomicAdd(&W.fill[e], 1);
      W.xshift[r] = shift;
    }
    W.inv[p] = r;
    pos[threadIdx.x] = r;
  }
  __syncthreads();
  const float sc = pow2f(-shift);
  for (int j = threadIdx.x; j < nv; j += kRowThreads) {
    const uint4 v = __ldg(src + j);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      o[q] = pack_f16x2(bf16_bits_to_f32(wv[q] & 0xFFFFu) * sc, bf16_bits_to_f32(wv[q] >> 16) * sc);
    for (int s = 0; s < k; ++s)
      if (pos[s] >= 0) reinterpret_cast<uint4*>(W.xperm + (size_t)pos[s] * H)[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// One block per sorted row: h (fp32) -> f16 with its own power-of-two shift.
__global__ void __launch_bounds__(kRowThreads) k_grp_h16(GroupWs W, int E, int I) {
  __shared__ float red[kRowThreads / 32];
  const int r = blockIdx.x;
  if (r >= W.offsets[E]) return;  // block-uniform
  const float4* src = reinterpret_cast<const float4*>(W.hperm + (size_t)r * I);
  const int nv = I / 4;
  float m = 0.f;
  bool fin = true;
  for (int j = threadIdx.x; j < nv; j += kRowThreads) {
    const float4 v = __ldcg(src + j);
    fin &= finite_bits(v.x) && finite_bits(v.y) && finite_bits(v.z) && finite_bits(v.w);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  if (!fin) set_status(QK_ERR_NONFINITE);
  const int shift = block_shift(m, red);
  if (threadIdx.x == 0) W.hshift[r] = shift;
  const float sc = pow2f(-shift);
  for (int j = threadIdx.x; j < nv; j += kRowThreads) {
    const float4 v = __ldcg(src + j);
    reinterpret_cast<uint2*>(W.h16 + (size_t)r * I)[j] =
        make_uint2(pack_f16x2(v.x * sc, v.y * sc), pack_f16x2(v.z * sc, v.w * sc));
  }
}

// One block per token: y[t] = sum_s w[t][s] d[pair (t, s)], slots in order.
__global__ void __launch_bounds__(256) k_grp_combine(GroupWs W, const float* __restrict__ w, int k, int H,
                                                     void* y, int y_bf16, int accumulate) {
  const int t = blockIdx.x;
  int pos[8];
  float ws[8];
  for (int s = 0; s < k; ++s) {
    pos[s] = W.inv[t * k + s];
    ws[s] = w[t * k + s];
  }
  for (int j = threadIdx.x; j < H / 4; j += blockDim.x) {
    // y added to (accumulate: the shared expert's output joins the routed one)
    float4 acc = accumulate ? reinterpret_cast<const float4*>(reinterpret_cast<const float*>(y) + (size_t)t * H)[j]
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < k; ++s) {
      if (pos[s] < 0) continue;
      const float4 d = __ldcg(reinterpret_cast<const float4*>(W.dperm + (size_t)pos[s] * H) + j);
      acc.x = fmaf(ws[s], d.x, acc.x);
      acc.y = fmaf(ws[s], d.y, acc.y);
      acc.z = fmaf(ws[s], d.z, acc.z);
      acc.w = fmaf(ws[s], d.w, acc.w);
    }
    if (!(finite_bits(acc.x) && finite_bits(acc.y) && finite_bits(acc.z) && finite_bits(acc.w)))
      set_status(QK_ERR_NONFINITE);
    if (y_bf16) {
      __nv_bfloat16* yb = reinterpret_cast<__nv_bfloat16*>(y) + (size_t)t * H + 4 * j;
      yb[0] = __float2bfloat16_rn(acc.x);
      yb[1] = __float2bfloat16_rn(acc.y);
      yb[2] = __float2bfloat16_rn(acc.z);
      yb[3] = __float2bfloat16_rn(acc.w);
    } else {
      reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + (size_t)t * H)[j] = acc;
    }
  }
}

}  // namespace qk

namespace qk {

// ------------------------------------------------------ the grouped GEMM --
struct GemmArgs {
  GroupWs W;
  qk_weight A, B;      // gate/up phase: gate, up; down phase: down, down
  int E, K;            // experts, reduction length
  int rows_per_e;      // weight rows of one expert (gate/up: inter; down: hidden)
  int MB;              // weight-row tiles per expert (gate/up: inter/64; down: hidden/128)
  int out_ld;          // output row length (gate/up: inter; down: hidden)
  int sc_stride;       // bytes per row of the staged tile scales (row length + 4: rows on distinct banks)
  alignas(64) CUtensorMap tqa, tqb;    // packed rows, 2-D bytes {K/2, rows}, box {128, 64}, 128B swizzle
  alignas(64) CUtensorMap tb[kGNBox];  // token rows, f16 {K, P}, box {64, 32 << i}, 128-byte swizzle
};

struct GHead {
  alignas(8) uint64_t rfull[kGRS];   // packed weight rows landed (TMA)
  alignas(8) uint64_t rempty[kGRS];  // packed rows consumed (dequant warps)
  alignas(8) uint64_t afull[kGAS];   // f16 weight tile written (dequant warps)
  alignas(8) uint64_t aempty[kGAS];  // f16 weight tile's MMAs completed
  alignas(8) uint64_t bfull[kGBS];   // token rows landed (TMA)
  alignas(8) uint64_t bempty[kGBS];  // token stage's MMAs completed
  alignas(8) uint64_t acc_full[2];   // accumulator buffer complete (by tile parity)
  alignas(8) uint64_t acc_empty[2];  // accumulator buffer read out
  alignas(8) uint64_t drained;       // every MMA of the block completed (exit)
  alignas(8) uint64_t cref_full[4];  // the tile's per-row reference codes written (tile % 4)
  uint32_t tmem;
  int abort;                         // a wait ran out: every role stops
  uint8_t cref[4][kGM];              // per tile row (tile % 4): largest e8m0 code of the row
};

constexpr int kGStageA = kGM * kGK * 2;   // 16 KB f16 weight tile
constexpr int kGStageB = kGN * kGK * 2;   // 32 KB of token rows
constexpr int kGStageR = kGM * kGK / 2 * kGRK;  // 16 KB packed weight rows (two 64-row boxes)
constexpr int kGTmemCols = 2 * kGN;  // two accumulator buffers

__host__ __device__ inline int g_smem_bytes(int sc_stride) {
  return 1024 + kGAS * kGStageA + kGBS * kGStageB + kGRS * kGStageR + kGM * sc_stride + (int)sizeof(GHead);
}

__device__ __forceinline__ int box_index(int n) { return n <= 32 ? 0 : n <= 64 ? 1 : n <= 128 ? 2 : 3; }

// f16x2 broadcast of 2^e (0 below the smallest f16 subnormal).
__device__ __forceinline__ uint32_t f16x2_pow2(int e) {
  uint32_t b = 0;
  if (e >= -14) b = (uint32_t)(e + 15) << 10;
  else if (e >= -24) b = 1u << (e + 24);
  return b | (b << 16);
}

template <int FA, int FB, bool GATEUP>
__global__ void __launch_bounds__(kGThreads, 1) k_ggemm(const __grid_constant__ GemmArgs G) {
  extern __shared__ __align__(16) uint8_t smem_raw[];  // rounded up to 1024 below, at run time
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sA = base;                      // kGAS f16 weight tiles (1024-aligned)
  uint8_t* sB = sA + kGAS * kGStageA;      // kGBS token stages
  uint8_t* sR = sB + kGBS * kGStageB;      // kGRS packed-row stages
  uint8_t* sS = sR + kGRS * kGStageR;      // the tile's scale rows
  GHead& S = *reinterpret_cast<GHead*>(sS + kGM * G.sc_stride);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const GroupWs& W = G.W;
  const int MB = G.MB, nks = G.K / kGK;
  const unsigned long long limit = g_wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGRS; ++s) {
      mbar_init(&S.rfull[s], 1);
      mbar_init(&S.rempty[s], kGDW);
    }
    for (int s = 0; s < kGAS; ++s) {
      mbar_init(&S.afull[s], kGDW);
      mbar_init(&S.aempty[s], 1);
    }
    for (int s = 0; s < kGBS; ++s) {
      mbar_init(&S.bfull[s], 1);
      mbar_init(&S.bempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.acc_full[b], 1);
      mbar_init(&S.acc_empty[b], kGEW);
    }
    mbar_init(&S.drained, 1);
    for (int b = 0; b < 4; ++b) mbar_init(&S.cref_full[b], kGDW);
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&S.tmem, kGTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem;
  const int n_tiles = *W.L1.n_tiles * MB;
  // Bounded wait; the first one that runs out stops every role of the block.
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*reinterpret_cast<volatile int*>(&S.abort)) return false;
    if (mbar_wait_bounded(bar, parity, limit)) return true;
    set_status(QK_ERR_TIMEOUT);
    *reinterpret_cast<volatile int*>(&S.abort) = 1;
    return false;
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile int*>(&S.abort) != 0; };

  if (warp == 0 || warp == 2) {
    // ----------------------------------------------------------- producers --
    // warp 0: packed weight rows, kGRK reduction steps per stage (one 8 KB box
    // per 64-row half); warp 2: token rows, 32 KB per stage (256 / n steps of
    // an n-row tile).
    if (warp == 0 && lane == 0) {
      const uint64_t pw = policy_evict_first();
      int n = 0;
      for (int t = blockIdx.x; t < n_tiles && !aborted(); t += gridDim.x) {
        const int f = t / MB, mb = t - f * MB;
        const int wrow = W.L1.tile_e[f] * G.rows_per_e + (GATEUP ? mb * 64 : mb * 128);
        for (int k0 = 0; k0 < nks; k0 += kGRK, ++n) {
          const int s = n % kGRS;
          if (n >= kGRS && !wait(&S.rempty[s], (uint32_t)((n / kGRS - 1) & 1))) break;
          mbar_arrive_expect_tx(&S.rfull[s], (uint32_t)kGStageR);
          uint8_t* r = sR + s * kGStageR;
          tma_load_2d(r, &G.tqa, k0 * (kGK / 2), wrow, &S.rfull[s], pw);
          tma_load_2d(r + kGStageR / 2, GATEUP ? &G.tqb : &G.tqa, k0 * (kGK / 2), GATEUP ? wrow : wrow + 64,
                      &S.rfull[s], pw);
        }
      }
      for (int q = n > kGRS ? n - kGRS : 0; q < n; ++q)  // nothing may still be landing at exit
        if (!mbar_wait_bounded(&S.rfull[q % kGRS], (uint32_t)((q / kGRS) & 1), kDrainLimitNs)) break;
    } else if (warp == 2 && lane == 0) {
      const uint64_t px = policy_evict_last();
      int n = 0;
      for (int t = blockIdx.x; t < n_tiles && !aborted(); t += gridDim.x) {
        const int f = t / MB;
        const int row0 = W.L1.tile_row0[f], bi = box_index(W.L1.tile_n[f]);
        const int nbox = 32 << bi, kpb = kGN / nbox;  // reduction steps per token stage
        for (int k0 = 0; k0 < nks; k0 += kpb, ++n) {
          const int s = n % kGBS, nsub = min(kpb, nks - k0);
          if (n >= kGBS && !wait(&S.bempty[s], (uint32_t)((n / kGBS - 1) & 1))) break;
          mbar_arrive_expect_tx(&S.bfull[s], (uint32_t)(nsub * nbox * kGK * 2));
          for (int j = 0; j < nsub; ++j)
            tma_load_2d(sB + s * kGStageB + j * nbox * kGK * 2, &G.tb[bi], (k0 + j) * kGK, row0, &S.bfull[s], px);
        }
      }
      for (int q = n > kGBS ? n - kGBS : 0; q < n; ++q)
        if (!mbar_wait_bounded(&S.bfull[q % kGBS], (uint32_t)((q / kGBS) & 1), kDrainLimitNs)) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA --
    if (lane == 0) {
      int na = 0, nb = 0, i = 0;
      for (int t = blockIdx.x; t < n_tiles && !aborted(); t += gridDim.x, ++i) {
        const int f = t / MB;
        const int nbox = 32 << box_index(W.L1.tile_n[f]), kpb = kGN / nbox;
        const uint32_t idesc = umma_idesc_f16(kGM, nbox);
        const int ab = i & 1;  // accumulator buffer
        if (i >= 2 && !wait(&S.acc_empty[ab], (uint32_t)((i / 2 - 1) & 1))) break;
        tc_fence_after();
        const uint32_t tacc = tmem + (uint32_t)(ab * kGN);
        for (int k0 = 0; k0 < nks && !aborted(); k0 += kpb, ++nb) {
          const int sb = nb % kGBS, nsub = min(kpb, nks - k0);
          if (!wait(&S.bfull[sb], (uint32_t)((nb / kGBS) & 1))) break;
          for (int j = 0; j < nsub; ++j, ++na) {
            const int sa = na % kGAS;
            if (!wait(&S.afull[sa], (uint32_t)((na / kGAS) & 1))) break;
            tc_fence_after();
            const uint64_t da = umma_desc_k_sw128(sA + sa * kGStageA);
            const uint64_t db = umma_desc_k_sw128(sB + sb * kGStageB + j * nbox * kGK * 2);
#pragma unroll
            for (int kk = 0; kk < kGK / 16; ++kk)  // 16 elements = 32 bytes = 2 descriptor units
              umma_f16(tacc, da + 2 * kk, db + 2 * kk, idesc, (k0 + j + kk) != 0 ? 1u : 0u);
            umma_commit(&S.aempty[sa]);
          }
          umma_commit(&S.bempty[sb]);
        }
        if (aborted()) break;
        umma_commit(&S.acc_full[ab]);
      }
      // every MMA issued here completes before the accumulator is freed
      umma_commit(&S.drained);
      mbar_wait_bounded(&S.drained, 0, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp < 3 + kGDW) {
    // ------------------------------------------------------------ dequant --
    const int dt = threadIdx.x - 96;  // 0 .. 255
    const int r = dt >> 1, hh = dt & 1;
    // GATEUP: tile row r = gate row r/2 (even r) or up row r/2 (odd r)
    const bool rowB = GATEUP && (r & 1);
    const int fr = rowB ? FB : FA;
    const qk_weight& WR = rowB ? G.B : G.A;
    const int wr_in_tile = GATEUP ? (r >> 1) : r;
    const int sc_len = fr == QK_FMT_MXFP4 ? G.K / 32 : G.K / 16;
    // NaN scale codes: e8m0 0xFF; e4m3 0x7F and 0xFF (the sign bit set first).
    const uint32_t nan_or = fr == QK_FMT_MXFP4 ? 0u : 0x80808080u;
    // The next tile's scale rows are loaded into registers while this tile is
    // dequantized (two threads per row, 16-byte pieces).
    constexpr int kScV = 8;
    const int nvq = sc_len % 32 == 0 ? sc_len / 32 : 0;
    const bool vec = nvq > 0 && nvq <= kScV;
    auto scale_row = [&](int tt) {
      const int f = tt / MB, mb = tt - f * MB;
      const int wrow = W.L1.tile_e[f] * G.rows_per_e + (GATEUP ? mb * 64 : mb * 128) + wr_in_tile;
      return WR.scales + (size_t)wrow * sc_len;
    };
    uint4 pre[kScV];
    auto prefetch = [&](int tt) {
      if (!vec || tt >= n_tiles) return;
      const uint8_t* g = scale_row(tt) + hh * 16;
#pragma unroll
      for (int q = 0; q < kScV; ++q)
        if (q < nvq) pre[q] = __ldg(reinterpret_cast<const uint4*>(g + q * 32));
    };
    prefetch(blockIdx.x);
    int n = 0, nr = 0, i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      // ---- the tile's scale rows, and (MXFP4) their largest code
      uint8_t* srow = sS + r * G.sc_stride;
      uint32_t m4 = 0, ff = 0;  // byte-wise maxima; any NaN code
      if (vec) {
#pragma unroll
        for (int q = 0; q < kScV; ++q) {
          if (q >= nvq) break;
          const uint4 v = pre[q];
          uint32_t* d = reinterpret_cast<uint32_t*>(srow + hh * 16 + q * 32);  // 4-byte aligned rows
          d[0] = v.x;
          d[1] = v.y;
          d[2] = v.z;
          d[3] = v.w;
          m4 = __vmaxu4(m4, __vmaxu4(__vmaxu4(v.x, v.y), __vmaxu4(v.z, v.w)));
          ff |= __vcmpeq4(v.x | nan_or, 0xFFFFFFFFu) | __vcmpeq4(v.y | nan_or, 0xFFFFFFFFu) |
                __vcmpeq4(v.z | nan_or, 0xFFFFFFFFu) | __vcmpeq4(v.w | nan_or, 0xFFFFFFFFu);
        }
        prefetch(t + gridDim.x);
      } else {
        const uint8_t* gsrc = scale_row(t);
        for (int b = hh; b < sc_len; b += 2) {
          const uint32_t c = gsrc[b];
          srow[b] = (uint8_t)c;
          m4 = max(m4, c);
          ff |= (c | (nan_or & 0x80u)) == 255u ? 1u : 0u;
        }
      }
      int cmax = (int)max(max(m4 & 0xFFu, (m4 >> 8) & 0xFFu), max((m4 >> 16) & 0xFFu, m4 >> 24));
      if (ff) set_status(QK_ERR_NAN_SCALE);
      cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));  // the row's two halves
      const int cref = fr == QK_FMT_MXFP4 ? min(cmax, 254) : 0;  // MXFP4 rows: relative to the row's max
      if (hh == 0) S.cref[i & 3][r] = (uint8_t)cref;
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&S.cref_full[i & 3]);
      // ---- dequantize every reduction step of the tile.  Packed stage layout:
      // two boxes of 64 rows x 128 bytes (kGRK steps), 128-byte swizzle.
      // GATEUP: box 0 = the gate rows, box 1 = the up rows; else rows 0-63, 64-127.
      const int brow = GATEUP ? (r >> 1) : (r & 63);
      const int bofs = (GATEUP ? (rowB ? 1 : 0) : (r >> 6)) * (kGStageR / 2) + brow * 128;
      bool ok = true;
      for (int ks = 0; ks < nks; ++ks, ++n) {
        const int sub = ks % kGRK, s = nr % kGRS, sa = n % kGAS;
        if (sub == 0 && !__all_sync(0xffffffffu, wait(&S.rfull[s], (uint32_t)((nr / kGRS) & 1)))) {
          ok = false;
          break;
        }
        const uint8_t* raw = sR + s * kGStageR + bofs + (((sub * 2 + hh) ^ (brow & 7)) << 4);
        const uint4 q = *reinterpret_cast<const uint4*>(raw);
        if (sub == kGRK - 1 || ks == nks - 1) {  // the stage's packed rows are all in registers
          __syncwarp();
          if (lane == 0) mbar_arrive_one(&S.rempty[s]);
          ++nr;
        }
        if (n >= kGAS && !__all_sync(0xffffffffu, wait(&S.aempty[sa], (uint32_t)((n / kGAS - 1) & 1)))) {
          ok = false;
          break;
        }
        const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
        uint32_t h2[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          h2[4 * j + 0] = e2m1x2_to_f16x2<0>(qw[j]);
          h2[4 * j + 1] = e2m1x2_to_f16x2<1>(qw[j]);
          h2[4 * j + 2] = e2m1x2_to_f16x2<2>(qw[j]);
          h2[4 * j + 3] = e2m1x2_to_f16x2<3>(qw[j]);
        }
        if (fr == QK_FMT_MXFP4) {  // one 32-block: e2m1 * 2^(c - cref + 8)
          const int c = srow[ks * 2 + hh];
          const uint32_t sc = f16x2_pow2(c - cref + 8);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            uint32_t d;
            asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(h2[j]), "r"(sc));
            h2[j] = d;
          }
        } else {  // two 16-blocks: e2m1 * e4m3
          const uint32_t c2 = (uint32_t)srow[ks * 4 + 2 * hh] | ((uint32_t)srow[ks * 4 + 2 * hh + 1] << 8);
          const uint32_t s01 = e4m3x2_to_f16x2<0>(c2);
          const uint32_t s0 = __byte_perm(s01, s01, 0x1010), s1 = __byte_perm(s01, s01, 0x3232);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            uint32_t d;
            asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(h2[j]), "r"(j < 8 ? s0 : s1));
            h2[j] = d;
          }
        }
        uint8_t* arow = sA + sa * kGStageA + r * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = 4 * hh + j;
          *reinterpret_cast<uint4*>(arow + ((c ^ (r & 7)) << 4)) =
              make_uint4(h2[4 * j], h2[4 * j + 1], h2[4 * j + 2], h2[4 * j + 3]);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_one(&S.afull[sa]);
      }
      if (!ok) break;
    }
  } else {
    // ----------------------------------------------------------- epilogue --
    // TMEM -> registers -> h (gate/up: SwiGLU of the interleaved gate/up rows)
    // or d (down), overlapping the next tile's dequantization and MMAs.
    const int quad = warp & 3;         // TMEM lanes 32 quad .. 32 quad + 31
    const int feat = quad * 32 + lane;  // tile row of this thread
    const bool frow_b = GATEUP && (feat & 1);
    const int frow_fmt = frow_b ? FB : FA;
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int f = t / MB, mb = t - f * MB;
      const int e = W.L1.tile_e[f], row0 = W.L1.tile_row0[f], nrow = W.L1.tile_n[f];
      const int ab = i & 1;
      if (!__all_sync(0xffffffffu, wait(&S.acc_full[ab], (uint32_t)((i / 2) & 1)) &&
                                       wait(&S.cref_full[i & 3], (uint32_t)((i / 4) & 1))))
        break;
      tc_fence_after();
      const int nbox = 32 << box_index(nrow);
      // MXFP4 rows were scaled by 2^(135 - cref) on chip; NVFP4 rows carry scale_2
      const float post = frow_fmt == QK_FMT_MXFP4 ? ldexpf(1.f, S.cref[i & 3][feat] - 135)
                                                  : (frow_b ? G.B.scale_2[e] : G.A.scale_2[e]);
      const int* rshift = GATEUP ? W.xshift : W.hshift;
      for (int c0 = 0; c0 < nbox && c0 < nrow; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + (uint32_t)(ab * kGN) + ((uint32_t)(quad * 32) << 16) + (uint32_t)c0, v);
        // the 32 columns' row shifts, one load per lane, broadcast by shuffles
        const int sh_l = c0 + lane < nrow ? rshift[row0 + c0 + lane] : 0;
        if (GATEUP) {
          // lane pair (gate, up) of one feature: the even lane finishes column
          // j, the odd lane column j + 1, after swapping one value each
          const bool odd = lane & 1;
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float a0 = __uint_as_float(v[j]) * post, a1 = __uint_as_float(v[j + 1]) * post;
            const float give = odd ? a0 : a1;  // even lane sends its column j+1, odd lane its column j
            const float got = __shfl_xor_sync(0xffffffffu, give, 1);
            const float g = odd ? got : a0, u = odd ? a1 : got;  // even: (g_j, u_j); odd: (g_j+1, u_j+1)
            const int col = c0 + j + (odd ? 1 : 0);
            const float sx = pow2f(__shfl_sync(0xffffffffu, sh_l, j + (odd ? 1 : 0)));
            if (col < nrow) {
              const float gs = g * sx;
              W.hperm[(size_t)(row0 + col) * G.out_ld + mb * 64 + (feat >> 1)] =
                  __fdividef(gs, 1.0f + __expf(-gs)) * (u * sx);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float sx = pow2f(__shfl_sync(0xffffffffu, sh_l, j));
            const int col = c0 + j;
            if (col < nrow)
              W.dperm[(size_t)(row0 + col) * G.out_ld + mb * 128 + feat] = __uint_as_float(v[j]) * post * sx;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&S.acc_empty[ab]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_free(tmem, kGTmemCols);
  }
}

}  // namespace qk

namespace qk {

// ================================================================= host ==
struct GWsLayout {
  size_t counts, n_tiles1, n_tiles2, n_flush, zero_end, offsets, fill, inv, dperm;
  size_t t1[5], t2[5], exp1, exp2;  // tile_e, tile_row0, tile_n, tile_first, tile_cnt
  size_t xshift, hshift, xperm, hperm, h16;
  size_t rtile2, xt, sfx, gu, ht, sfh, fac1, fac2, total;
};

enum { kWsF16 = 0, kWsMx = 1, kWsNv = 2 };

// Workspace of the grouped path: the f16 buffers, the MXFP4 block-scaled
// ones, or (NVFP4 layers in QK_ACT_MXFP4) those with twice the token scale
// atoms and the per-row factors.
static GWsLayout g_layout(int T, int k, int E, int H, int I, int kind) {
  const bool mx = kind != kWsF16;
  const size_t sf_mul = kind == kWsNv ? 2 : 1;
  const size_t P = (size_t)T * k;
  const size_t F1 = (size_t)g_max_tiles((int)P, E, mx ? kXTok1 : kGN), F2 = (size_t)g_max_tiles((int)P, E, kXTok2);
  GWsLayout L = {};
  size_t o = 0;
  L.counts = o; o += (size_t)E * 4;          // zeroed on every call: counts .. n_flush
  L.n_tiles1 = o; o += 8;
  L.n_tiles2 = o; o += 8;
  L.n_flush = o; o += 8;
  L.zero_end = o;
  o = align256(o);
  L.offsets = o; o += align256((size_t)(E + 1) * 4);
  L.fill = o; o += align256((size_t)E * 4);
  L.inv = o; o += align256(P * 4);
  L.dperm = o; o += align256(P * H * 4);
  for (int i = 0; i < (mx ? 5 : 3); ++i) { L.t1[i] = o; o += align256(F1 * 4); }
  if (mx) {
    for (int i = 0; i < 5; ++i) { L.t2[i] = o; o += align256(F2 * 4); }
    L.exp1 = o; o += align256((size_t)E * 4);
    L.exp2 = o; o += align256((size_t)E * 4);
    L.rtile2 = o; o += align256(P * 4);
    L.xt = o; o += align256(F1 * (H / kXK) * kXBlock);
    L.sfx = o; o += align256(F1 * (H / kXK) * kSfAtom * sf_mul);
    L.gu = o; o += align256(P * 2 * I * 4);
    L.ht = o; o += align256(F2 * (I / kXK) * kXBlock);
    L.sfh = o; o += align256(F2 * (I / kXK) * kSfAtom * sf_mul);
    if (kind == kWsNv) {
      L.fac1 = o; o += align256(P * 4);
      L.fac2 = o; o += align256(P * 4);
    }
  } else {
    L.xshift = o; o += align256(P * 4);
    L.hshift = o; o += align256(P * 4);
    L.xperm = o; o += align256(P * H * 2);
    L.hperm = o; o += align256(P * I * 4);
    L.h16 = o; o += align256(P * I * 2);
  }
  L.total = o;
  return L;
}

static bool g_mx(const qk_moe_layer* L) { return gmx_eligible(L->gate, L->up, L->down, L->hidden, L->inter); }

size_t group_workspace_bytes(const qk_moe_layer* L, int T, int k) {
  return g_layout(T, k, L->gate.n_experts, L->hidden, L->inter, g_mx(L) ? kWsMx : kWsF16).total;
}

size_t group_workspace_bytes_act(const qk_moe_layer* L, int T, int k, int act_quant) {
  if (act_quant != QK_ACT_MXFP4 && act_quant != QK_ACT_E4M3) return 0;
  if (g_mx(L)) return g_layout(T, k, L->gate.n_experts, L->hidden, L->inter, kWsMx).total;
  if (act_quant == QK_ACT_MXFP4 && gmx_nv_eligible(L->gate, L->up, L->down, L->hidden, L->inter))
    return g_layout(T, k, L->gate.n_experts, L->hidden, L->inter, kWsNv).total;
  return 0;
}

static TileList g_list(uint8_t* p, const size_t (&t)[5], size_t exp, size_t n_tiles, bool mx) {
  TileList L = {};
  L.tile_e = reinterpret_cast<int*>(p + t[0]);
  L.tile_row0 = reinterpret_cast<int*>(p + t[1]);
  L.tile_n = reinterpret_cast<int*>(p + t[2]);
  if (mx) {
    L.tile_first = reinterpret_cast<int*>(p + t[3]);
    L.tile_cnt = reinterpret_cast<int*>(p + t[4]);
    L.exp_tile0 = reinterpret_cast<int*>(p + exp);
  }
  L.n_tiles = reinterpret_cast<int*>(p + n_tiles);
  return L;
}

static GroupWs g_carve(void* ws, int T, int k, int E, int H, int I, int kind) {
  const bool mx = kind != kWsF16;
  const GWsLayout L = g_layout(T, k, E, H, I, kind);
  uint8_t* p = static_cast<uint8_t*>(ws);
  GroupWs W = {};
  W.counts = reinterpret_cast<int*>(p + L.counts);
  W.n_flush = reinterpret_cast<unsigned long long*>(p + L.n_flush);
  W.zero_bytes = L.zero_end - L.counts;
  W.offsets = reinterpret_cast<int*>(p + L.offsets);
  W.fill = reinterpret_cast<int*>(p + L.fill);
  W.inv = reinterpret_cast<int*>(p + L.inv);
  W.dperm = reinterpret_cast<float*>(p + L.dperm);
  W.L1 = g_list(p, L.t1, L.exp1, L.n_tiles1, mx);
  if (mx) {
    W.L2 = g_list(p, L.t2, L.exp2, L.n_tiles2, true);
    W.rtile2 = reinterpret_cast<int*>(p + L.rtile2);
    W.xt = p + L.xt;
    W.sfx = p + L.sfx;
    W.gu = reinterpret_cast<float*>(p + L.gu);
    W.ht = p + L.ht;
    W.sfh = p + L.sfh;
    if (kind == kWsNv) {
      W.fac1 = reinterpret_cast<float*>(p + L.fac1);
      W.fac2 = reinterpret_cast<float*>(p + L.fac2);
    }
  } else {
    W.xshift = reinterpret_cast<int*>(p + L.xshift);
    W.hshift = reinterpret_cast<int*>(p + L.hshift);
    W.xperm = reinterpret_cast<__half*>(p + L.xperm);
    W.hperm = reinterpret_cast<float*>(p + L.hperm);
    W.h16 = reinterpret_cast<__half*>(p + L.h16);
  }
  return W;
}

// Packed rows [rows][K/2] bytes, boxes {128 bytes = kGRK reduction steps, 64 rows}, 128-byte swizzle.
static bool g_map_packed(CUtensorMap* m, const uint8_t* q, int64_t rows, int K) {
  const uint64_t dims[2] = {(uint64_t)K / 2, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)K / 2};
  const uint32_t box[2] = {(uint32_t)(kGK / 2 * kGRK), 64};
  return tmap_get(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Token rows [P][K] f16, boxes {64 elements, 32 << i rows}, 128-byte swizzle.
static bool g_map_tokens(CUtensorMap (&m)[kGNBox], const __half* x, int64_t P, int K) {
  const uint64_t dims[2] = {(uint64_t)K, (uint64_t)P};
  const uint64_t strides[1] = {(uint64_t)K * 2};
  for (int i = 0; i < kGNBox; ++i) {
    const uint32_t box[2] = {(uint32_t)kGK, (uint32_t)(32 << i)};
    if (!tmap_get(&m[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  }
  return true;
}

template <int FA, int FB, bool GATEUP>
static qk_status g_launch(const GemmArgs& A, cudaStream_t st) {
  const int smem = g_smem_bytes(A.sc_stride);
  if (smem > max_smem_optin()) return QK_ERR_UNSUPPORTED;
  return launch_ex(k_ggemm<FA, FB, GATEUP>, dim3(num_sms()), dim3(kGThreads), (size_t)smem, st, false, A);
}

template <bool GATEUP>
static qk_status g_dispatch(const GemmArgs& A, cudaStream_t st) {
  constexpr int MX = QK_FMT_MXFP4, NV = QK_FMT_NVFP4;
  const int fa = A.A.fmt, fb = A.B.fmt;
  if (fa == MX && fb == MX) return g_launch<MX, MX, GATEUP>(A, st);
  if (fa == MX) return g_launch<MX, NV, GATEUP>(A, st);
  if (fb == MX) return g_launch<NV, MX, GATEUP>(A, st);
  return g_launch<NV, NV, GATEUP>(A, st);
}

qk_status group_forward(const DecodeArgs& a, void* workspace, cudaStream_t st) {
  return group_forward_act(a, QK_ACT_NONE, workspace, st);
}

// act_quant other than QK_ACT_NONE runs only on the block-scaled kernels (the
// caller checks eligibility).
qk_status group_forward_act(const DecodeArgs& a, int act_quant, void* workspace, cudaStream_t st) {
  const int T = a.T, k = a.k, E = a.E, H = a.H, I = a.I, P = a.P;
  const bool nv = act_quant == QK_ACT_MXFP4 && gmx_nv_eligible(a.gate, a.up, a.down, H, I);
  const bool mx = gmx_eligible(a.gate, a.up, a.down, H, I) || nv;  // the block-scaled grouped kernels
  if (act_quant != QK_ACT_NONE && !mx) return QK_ERR_UNSUPPORTED;
  GroupWs W = g_carve(workspace, T, k, E, H, I, nv ? kWsNv : mx ? kWsMx : kWsF16);
  if (cudaMemsetAsync(W.counts, 0, W.zero_bytes, st) != cudaSuccess) return QK_ERR_CUDA;
  k_grp_count<<<(P + 255) / 256, 256, 0, st>>>(a.ids, P, E, W.counts);
  k_grp_scan<<<1, kScanThreads, 0, st>>>(W, W.L1, E, mx ? gmx_tok1(act_quant) : kGN, mx ? 1 : 0, 1);
  if (mx) k_grp_scan<<<1, kScanThreads, 0, st>>>(W, W.L2, E, gmx_tok2(act_quant), 1, 0);
  if (cudaGetLastError() != cudaSuccess) return QK_ERR_CUDA;
  if (mx) {
    const qk_status rc = gmx_forward_act(a, W, act_quant, st);
    if (rc != QK_OK) return rc;
    k_grp_combine<<<T, 256, 0, st>>>(W, a.w, k, H, a.y, a.y_bf16, 0);
    return cudaGetLastError() == cudaSuccess ? QK_OK : QK_ERR_CUDA;
  }
  k_grp_scatter<<<T, kRowThreads, 0, st>>>(W, a.x, a.ids, k, E, H);
  if (cudaGetLastError() != cudaSuccess) return QK_ERR_CUDA;

  GemmArgs g1 = {};
  g1.W = W;
  g1.A = a.gate;
  g1.B = a.up;
  g1.E = E;
  g1.K = H;
  g1.rows_per_e = I;
  g1.MB = I / 64;
  g1.out_ld = I;
  g1.sc_stride = ((a.gate.fmt == QK_FMT_NVFP4 || a.up.fmt == QK_FMT_NVFP4) ? H / 16 : H / 32) + 4;
  if (!g_map_packed(&g1.tqa, a.gate.q, (int64_t)E * I, H) || !g_map_packed(&g1.tqb, a.up.q, (int64_t)E * I, H) ||
      !g_map_tokens(g1.tb, W.xperm, P, H))
    return QK_ERR_CUDA;
  qk_status rc = g_dispatch<true>(g1, st);
  if (rc != QK_OK) return rc;

  k_grp_h16<<<P, kRowThreads, 0, st>>>(W, E, I);
  GemmArgs g2 = {};
  g2.W = W;
  g2.A = a.down;
  g2.B = a.down;
  g2.E = E;
  g2.K = I;
  g2.rows_per_e = H;
  g2.MB = H / 128;
  g2.out_ld = H;
  g2.sc_stride = (a.down.fmt == QK_FMT_NVFP4 ? I / 16 : I / 32) + 4;
  if (!g_map_packed(&g2.tqa, a.down.q, (int64_t)E * H, I) || !g_map_tokens(g2.tb, W.h16, P, I)) return QK_ERR_CUDA;
  g2.tqb = g2.tqa;
  rc = g_dispatch<false>(g2, st);
  if (rc != QK_OK) return rc;
  k_grp_combine<<<T, 256, 0, st>>>(W, a.w, k, H, a.y, a.y_bf16, 0);
  return cudaGetLastError() == cudaSuccess ? QK_OK : QK_ERR_CUDA;
}

// ------------------------------------------------ FP8 shared expert, large M --
// Every token routed to the one (shared) expert with weight 1.
__global__ void k_fp8_route_all(int32_t* ids, float* w, int M) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < M; i += gridDim.x * blockDim.x) {
    ids[i] = 0;
    w[i] = 1.0f;
  }
}

size_t fp8_group_workspace_bytes(int M, int H, int I) {
  return g_layout(M, 1, 1, H, I, kWsMx).total + 2 * align256((size_t)M * 4);
}

qk_status fp8_group_forward(const void* x, int M, int H, int I, const uint8_t* wg, const uint8_t* sg,
                            const uint8_t* wu, const uint8_t* su, const uint8_t* wd, const uint8_t* sd, int blk,
                            float* y, void* workspace, cudaStream_t st) {
  const size_t base = g_layout(M, 1, 1, H, I, kWsMx).total;
  int32_t* ids = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + base);
  float* w = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + base + align256((size_t)M * 4));
  GroupWs W = g_carve(workspace, M, 1, 1, H, I, kWsMx);
  if (cudaMemsetAsync(W.counts, 0, W.zero_bytes, st) != cudaSuccess) return QK_ERR_CUDA;
  k_fp8_route_all<<<(M + 255) / 256, 256, 0, st>>>(ids, w, M);
  k_grp_count<<<(M + 255) / 256, 256, 0, st>>>(ids, M, 1, W.counts);
  k_grp_scan<<<1, kScanThreads, 0, st>>>(W, W.L1, 1, kXTok1, 1, 1);
  k_grp_scan<<<1, kScanThreads, 0, st>>>(W, W.L2, 1, kXTok2, 1, 0);
  if (cudaGetLastError() != cudaSuccess) return QK_ERR_CUDA;
  const qk_status rc = gmx_fp8_ffn(W, static_cast<const uint16_t*>(x), ids, M, H, I, wg, sg, wu, su, wd, sd, blk, st);
  if (rc != QK_OK) return rc;
  k_grp_combine<<<M, 256, 0, st>>>(W, w, 1, H, y, 0, 1);
  return cudaGetLastError() == cudaSuccess ? QK_OK : QK_ERR_CUDA;
}

}  // namespace qk
