// qk_decode.cu -- decode path of moe_expert_forward (a few tokens per call).
//
// The routed-expert FFN of a DeepSeek-V4-Flash-style MoE layer
// ("DeepSeek-V4-Flash-W4A16-FP8", base-model table: hidden 4096, 256 routed
// experts, top-6) with MXFP4 / NVFP4 expert weights
// ("DeepSeek-v4-Flash-REAP-K180-NVFP4", "NVFP4: lossless MXFP4->NVFP4
// conversion"; gate+up carry ~2/3 of the expert bytes, "Why this mix?").
//
// Two kernels, chained with programmatic dependent launch:
//   k_gateup  h[p][n]  = silu(g) * u, g/u = gate/up row n of expert e(p) . x[t(p)]
//   k_down    part[p][m] = down row m of expert e(p) . h[p];  y[t] = sum_s w * part
// Work unit: k_gateup = 8 output rows (8 gate + 8 up weight rows = one 16-row
// MMA tile), k_down = 16 output rows, both over the full reduction length.
// The unit's packed rows are copied by the bulk-copy (TMA) engine into padded
// shared-memory rows, a ring of stages deep.  Eight warps split the reduction
// dimension; each forms m16n8k16 A fragments with ldmatrix and the hardware
// e2m1x2 -> f16x2 conversion (exact), multiplies with f16 activations on the
// tensor cores (fp32 accumulate) and applies the block scale in fp32:
//   MXFP4: once per 32-block on the fp32 partial (2^(c-127), exact)
//   NVFP4: the e4m3 scale is folded into the f16 A fragment (e2m1*e4m3 is
//          exact in f16), scale_2 at the end.
// Activations enter the MMA as f16 scaled by a power of two per token (x) or
// per pair (h) so that the largest magnitude sits in [2^14, 2^15).
//
// Token columns: the N=8 side of the MMA holds up to 8 tokens routed to the
// unit's expert; more tokens are processed in further 8-column tiles.
#include <algorithm>

#include "qk_common.cuh"

namespace qk {


// --------------------------------------------------------------- routing --
// Per-CTA routing tables built in shared memory from the ids (P <= kMaxPairs
// <= blockDim, one pair per thread).  Active experts ascend by id; the pairs
// of one expert ascend by pair index (= token-major order).
struct Route {
  int n_active;
  int16_t act_expert[kMaxPairs];    // active experts, ascending id
  int16_t act_cnt[kMaxPairs];       // pairs per active expert
  int16_t act_off[kMaxPairs + 1];   // pair-list offsets per active expert
  int16_t pair_list[kMaxPairs];     // pair indices, grouped by expert
  int16_t tmp_e[kMaxPairs];
  int8_t tmp_first[kMaxPairs];
};

__device__ void build_route(const int32_t* __restrict__ ids, int P, int E, Route& R) {
  const int p = threadIdx.x;
  int e = -1;
  if (p < P) {
    e = ids[p];
    if (e < 0 || e >= E) {
      set_status(QK_ERR_INVALID_ARG);
      e = -1;
    }
    R.tmp_e[p] = (int16_t)e;
  }
  __syncthreads();
  int first = (e >= 0);
  for (int q = 0; q < p && first && p < P; ++q) first = (R.tmp_e[q] != e);
  if (p < P) R.tmp_first[p] = (int8_t)first;
  const int n_active = __syncthreads_count(first);
  int slot = 0, rank = 0, total = 0;
  if (e >= 0) {
    for (int q = 0; q < P; ++q) {
      const int eq = R.tmp_e[q];
      slot += (R.tmp_first[q] && eq >= 0 && eq < e);
      rank += (q < p && eq == e);
      total += (eq == e);
    }
    if (first) {
      R.act_expert[slot] = (int16_t)e;
      R.act_cnt[slot] = (int16_t)total;
    }
  }
  if (p == 0) R.n_active = n_active;
  __syncthreads();
  if (p <= n_active) {
    int off = 0;
    for (int a = 0; a < p; ++a) off += R.act_cnt[a];
    R.act_off[p] = (int16_t)off;
  }
  __syncthreads();
  if (e >= 0) R.pair_list[R.act_off[slot] + rank] = (int16_t)p;
  __syncthreads();
}

// Decoded scale for the fragment rows of one 32-block.
//  MX: fp32 2^(c-127), applied to the fp32 partial.
//  NV: f16x2 broadcast of the e4m3 scale of this thread's 16-half, applied to A.
template <int FMT>
struct BlockScale;

template <>
struct BlockScale<QK_FMT_MXFP4> {
  float f;
  __device__ __forceinline__ void load(const uint8_t* row_scales, int blk, int /*t*/, bool& bad) {
    const uint32_t c = row_scales[blk];
    bad |= (c == 255u);
    f = e8m0_to_f32(c);
  }
};

template <>
struct BlockScale<QK_FMT_NVFP4> {
  uint32_t h2;
  __device__ __forceinline__ void load(const uint8_t* row_scales, int blk, int t, bool& bad) {
    const uint32_t c = row_scales[2 * blk + (t >> 1)];
    bad |= ((c & 0x7Fu) == 0x7Fu);
    const uint32_t h = e4m3x2_to_f16x2<0>(c) & 0xFFFFu;
    h2 = h | (h << 16);
  }
};

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// One 32-block of a 16-row tile against one 8-column activation tile.
// wa: A word of rows g (rows 0..7 of the tile), wb: rows g+8.  xb: the
// thread's 8 f16 activations (4 regs).  acc rows g -> acc[0..1], g+8 -> acc[2..3].
template <int FA, int FB>
__device__ __forceinline__ void block_mma(float (&acc)[4], uint32_t wa, uint32_t wb,
                                          const uint4& xb, const BlockScale<FA>& sa,
                                          const BlockScale<FB>& sb) {
  uint32_t a0 = e2m1x2_to_f16x2<0>(wa), a1 = e2m1x2_to_f16x2<0>(wb);
  uint32_t a2 = e2m1x2_to_f16x2<1>(wa), a3 = e2m1x2_to_f16x2<1>(wb);
  uint32_t c0 = e2m1x2_to_f16x2<2>(wa), c1 = e2m1x2_to_f16x2<2>(wb);
  uint32_t c2 = e2m1x2_to_f16x2<3>(wa), c3 = e2m1x2_to_f16x2<3>(wb);
  if constexpr (FA == QK_FMT_NVFP4) {
    a0 = hmul2(a0, sa.h2); a2 = hmul2(a2, sa.h2); c0 = hmul2(c0, sa.h2); c2 = hmul2(c2, sa.h2);
  }
  if constexpr (FB == QK_FMT_NVFP4) {
    a1 = hmul2(a1, sb.h2); a3 = hmul2(a3, sb.h2); c1 = hmul2(c1, sb.h2); c3 = hmul2(c3, sb.h2);
  }
  if constexpr (FA == QK_FMT_NVFP4 && FB == QK_FMT_NVFP4) {
    mma_f16_16816(acc, a0, a1, a2, a3, xb.x, xb.y);
    mma_f16_16816(acc, c0, c1, c2, c3, xb.z, xb.w);
  } else {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    mma_f16_16816(d, a0, a1, a2, a3, xb.x, xb.y);
    mma_f16_16816(d, c0, c1, c2, c3, xb.z, xb.w);
    if constexpr (FA == QK_FMT_MXFP4) {
      acc[0] = fmaf(d[0], sa.f, acc[0]);
      acc[1] = fmaf(d[1], sa.f, acc[1]);
    } else {
      acc[0] += d[0];
      acc[1] += d[1];
    }
    if constexpr (FB == QK_FMT_MXFP4) {
      acc[2] = fmaf(d[2], sb.f, acc[2]);
      acc[3] = fmaf(d[3], sb.f, acc[3]);
    } else {
      acc[2] += d[2];
      acc[3] += d[3];
    }
  }
}

template <int FMT>
__host__ __device__ constexpr int scale_bytes_per_row(int K) {
  return FMT == QK_FMT_MXFP4 ? K / 32 : K / 16;
}

// Shared-memory geometry of one kernel instantiation (host and device agree).
struct Geo {
  int K;           // reduction length (bytes of a packed row = K/2)
  int nib_row;     // padded bytes per smem nibble row
  int sca, scb;    // scale bytes per row, rows 0..7 and 8..15
  int stage;       // bytes per stage
  int act_stride;  // halves per activation row in smem
};

__host__ __device__ inline Geo make_geo(int K, int fa, int fb) {
  Geo g;
  g.K = K;
  g.nib_row = K / 2 + 16;
  g.sca = fa == QK_FMT_MXFP4 ? K / 32 : K / 16;
  g.scb = fb == QK_FMT_MXFP4 ? K / 32 : K / 16;
  g.stage = (16 * g.nib_row + 8 * g.sca + 8 * g.scb + 127) / 128 * 128;
  g.act_stride = K + 32;  // 2K+64 bytes: conflict-free 16-B fragment loads
  return g;
}

// Fixed shared-memory header (routing, barriers, reduction buffers).
struct SmemHead {
  Route R;
  alignas(8) uint64_t full[kMaxStages];
  alignas(16) float red[kWarps * 32 * 4];  // read and written as float4
  float mx_red[kWarps * kTileN];
  float mx_out[kTileN];
  int shift[kTileN];
  int rows[kTileN];
  int flag;
};

constexpr int kHeadBytes = (int)((sizeof(SmemHead) + 127) / 128 * 128);

// Issue the bulk copies of one unit: 16 nibble rows + the two scale slabs.
// rows 0..7 come from (qa, sa) rows ra0.., rows 8..15 from (qb, sb) rows rb0..
__device__ __forceinline__ void issue_unit(uint8_t* stage, uint64_t* bar, const Geo& G,
                                           const uint8_t* qa, const uint8_t* sa, int64_t ra0,
                                           const uint8_t* qb, const uint8_t* sb, int64_t rb0,
                                           uint64_t pol) {
  const int rb = G.K / 2;
  mbar_arrive_expect_tx(bar, 16u * rb + 8u * G.sca + 8u * G.scb);
#pragma unroll 1
  for (int i = 0; i < 8; ++i) {
    bulk_g2s_evict_first(stage + i * G.nib_row, qa + (ra0 + i) * rb, rb, bar, pol);
    bulk_g2s_evict_first(stage + (8 + i) * G.nib_row, qb + (rb0 + i) * rb, rb, bar, pol);
  }
  uint8_t* sc = stage + 16 * G.nib_row;
  bulk_g2s_evict_first(sc, sa + ra0 * G.sca, 8 * G.sca, bar, pol);
  bulk_g2s_evict_first(sc + 8 * G.sca, sb + rb0 * G.scb, 8 * G.scb, bar, pol);
}

// Warp's share of one unit: 16 tile rows x its block range, one token tile.
template <int FA, int FB>
__device__ __forceinline__ void unit_mma(float (&acc)[4], const uint8_t* stage, const Geo& G,
                                         const __half* act, int rows_act, int warp, int lane,
                                         bool& bad) {
  const int g = lane >> 2, t = lane & 3;
  const int nb = G.K / 32;
  const int b0 = warp * nb / kWarps, b1 = (warp + 1) * nb / kWarps;
  const uint8_t* sc_a = stage + 16 * G.nib_row + g * G.sca;
  const uint8_t* sc_b = stage + 16 * G.nib_row + 8 * G.sca + g * G.scb;
  // token columns past the staged rows read a staged row (their results are unused)
  const __half* xrow = act + min(g, rows_act - 1) * G.act_stride + 8 * t;
  // ldmatrix row address: matrix j = lane>>3 (0: rows 0-7 blk b, 1: rows 8-15
  // blk b, 2: rows 0-7 blk b+1, 3: rows 8-15 blk b+1), row lane&7.
  const int mj = lane >> 3, mr = lane & 7;
  const uint8_t* lrow = stage + ((mj & 1) * 8 + mr) * G.nib_row + (mj >> 1) * 16;
  int b = b0;
  for (; b + 1 < b1; b += 2) {
    uint32_t wa0, wb0, wa1, wb1;
    ldmatrix_x4(wa0, wb0, wa1, wb1, lrow + b * 16);
    BlockScale<FA> sa0, sa1;
    BlockScale<FB> sb0, sb1;
    sa0.load(sc_a, b, t, bad);
    sb0.load(sc_b, b, t, bad);
    sa1.load(sc_a, b + 1, t, bad);
    sb1.load(sc_b, b + 1, t, bad);
    const uint4 x0 = *reinterpret_cast<const uint4*>(xrow + b * 32);
    const uint4 x1 = *reinterpret_cast<const uint4*>(xrow + (b + 1) * 32);
    block_mma<FA, FB>(acc, wa0, wb0, x0, sa0, sb0);
    block_mma<FA, FB>(acc, wa1, wb1, x1, sa1, sb1);
  }
  if (b < b1) {
    uint32_t wa0, wb0;
    ldmatrix_x2(wa0, wb0, lrow + b * 16);
    BlockScale<FA> sa0;
    BlockScale<FB> sb0;
    sa0.load(sc_a, b, t, bad);
    sb0.load(sc_b, b, t, bad);
    const uint4 x0 = *reinterpret_cast<const uint4*>(xrow + b * 32);
    block_mma<FA, FB>(acc, wa0, wb0, x0, sa0, sb0);
  }
}

// =================================================================== k1 ==
template <int FG, int FU>
__global__ void __launch_bounds__(kThreads, 1) k_gateup(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  SmemHead& S = *reinterpret_cast<SmemHead*>(smem);
  const Geo G = make_geo(a.H, FG, FU);
  __half* act = reinterpret_cast<__half*>(smem + kHeadBytes);
  uint8_t* stages = smem + kHeadBytes + (size_t)a.rows_act * G.act_stride * 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nstage = a.stages;
  const int tn = a.rows_act;  // token columns per tile = staged activation rows (<= 8)

  pdl_launch_dependents();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < a.n_counters; i += blockDim.x) a.counters[i] = 0;

  build_route(a.ids, a.P, a.E, S.R);
  const int R1 = a.I / 8;
  const int U = S.R.n_active * R1;
  const int u0 = (int)((int64_t)U * blockIdx.x / gridDim.x);
  const int u1 = (int)((int64_t)U * (blockIdx.x + 1) / gridDim.x);
  const int n = u1 - u0;
  if (n <= 0) return;

  const uint64_t pol = policy_evict_first();
  auto issue = [&](int i) {
    const int u = u0 + i, s = i % nstage;
    const int e = S.R.act_expert[u / R1];
    const int64_t row0 = (int64_t)e * a.I + (int64_t)(u % R1) * 8;
    issue_unit(stages + (size_t)s * G.stage, &S.full[s], G, a.gate.q, a.gate.scales, row0, a.up.q,
               a.up.scales, row0, pol);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < nstage; ++s) mbar_init(&S.full[s], 1);
    fence_mbar_init();
    for (int i = 0; i < min(n, nstage); ++i) issue(i);
  }
  __syncthreads();

  bool bad = false;
  int cur_a = -1;
  const unsigned long long limit = g_wait_limit_ns;
  for (int i = 0; i < n; ++i) {
    const int u = u0 + i, s = i % nstage;
    const int as = u / R1, r = u % R1;
    const int e = S.R.act_expert[as];
    const int p0 = S.R.act_off[as], np = S.R.act_off[as + 1] - p0;
    const uint8_t* st = stages + (size_t)s * G.stage;
    const bool ready = mbar_wait_bounded(&S.full[s], (i / nstage) & 1, limit);
    if (__syncthreads_or(!ready)) {
      drain_stages(S.full, i, min(n, i + nstage), nstage);
      return;
    }
    for (int tile = 0; tile * tn < np; ++tile) {
      const int nt = min(tn, np - tile * tn);
      if (as != cur_a || np > tn) {
        if (threadIdx.x < kTileN)
          S.rows[threadIdx.x] =
              threadIdx.x < nt ? S.R.pair_list[p0 + tile * tn + threadIdx.x] / a.k : 0;
        __syncthreads();
        stage_bf16_rows(a.x, S.rows, nt, a.H, act, G.act_stride, S.shift, S.mx_red, S.mx_out);
        cur_a = as;
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      unit_mma<FG, FU>(acc, st, G, act, a.rows_act, warp, lane, bad);
      if (reduce_warps(acc, S.red, warp, lane)) {
        const int g = lane >> 2, t = lane & 3;
        const float s2g = FG == QK_FMT_NVFP4 ? a.gate.scale_2[e] : 1.f;
        const float s2u = FU == QK_FMT_NVFP4 ? a.up.scale_2[e] : 1.f;
        float hm[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int col = 2 * t + j;
          hm[j] = 0.f;
          if (col < nt) {
            const float sx = pow2f(S.shift[col]);
            const float gv = acc[j] * sx * s2g, uv = acc[2 + j] * sx * s2u;
            const float hv = silu_mul(gv, uv);
            const int p = S.R.pair_list[p0 + tile * tn + col];
            a.h[(size_t)p * a.I + r * 8 + g] = hv;
            hm[j] = fabsf(hv);
          }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) hm[j] = fmaxf(hm[j], __shfl_xor_sync(0xffffffffu, hm[j], o));
        }
        if (g == 0) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int col = 2 * t + j;
            if (col < nt) a.hmax[(size_t)S.R.pair_list[p0 + tile * tn + col] * R1 + r] = hm[j];
          }
        }
      }
      __syncthreads();
    }
    if (threadIdx.x == 0 && i + nstage < n) issue(i + nstage);
  }
  if (bad) set_status(QK_ERR_NAN_SCALE);
}

// =================================================================== k2 ==
template <int FD>
__global__ void __launch_bounds__(kThreads, 1) k_down(const DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  SmemHead& S = *reinterpret_cast<SmemHead*>(smem);
  const Geo G = make_geo(a.I, FD, FD);
  __half* act = reinterpret_cast<__half*>(smem + kHeadBytes);
  uint8_t* stages = smem + kHeadBytes + (size_t)a.rows_act * G.act_stride * 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nstage = a.stages;
  const int tn = a.rows_act;  // token columns per tile = staged activation rows (<= 8)

  build_route(a.ids, a.P, a.E, S.R);
  const int R1 = a.I / 8, R2 = a.H / 16;
  const int U = S.R.n_active * R2;
  const int u0 = (int)((int64_t)U * blockIdx.x / gridDim.x);
  const int u1 = (int)((int64_t)U * (blockIdx.x + 1) / gridDim.x);
  const int n = u1 - u0;
  if (n <= 0) {
    pdl_wait();
    return;
  }
  const uint64_t pol = policy_evict_first();
  auto issue = [&](int i) {
    const int u = u0 + i, s = i % nstage;
    const int e = S.R.act_expert[u / R2];
    const int64_t row0 = (int64_t)e * a.H + (int64_t)(u % R2) * 16;
    issue_unit(stages + (size_t)s * G.stage, &S.full[s], G, a.down.q, a.down.scales, row0, a.down.q,
               a.down.scales, row0 + 8, pol);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < nstage; ++s) mbar_init(&S.full[s], 1);
    fence_mbar_init();
    for (int i = 0; i < min(n, nstage); ++i) issue(i);  // weights do not depend on k_gateup
  }
  __syncthreads();
  pdl_wait();  // h, hmax and the counters are written by k_gateup

  bool bad = false;
  int cur_a = -1;
  const unsigned long long limit = g_wait_limit_ns;
  for (int i = 0; i < n; ++i) {
    const int u = u0 + i, s = i % nstage;
    const int as = u / R2, r = u % R2;
    const int e = S.R.act_expert[as];
    const int p0 = S.R.act_off[as], np = S.R.act_off[as + 1] - p0;
    const uint8_t* st = stages + (size_t)s * G.stage;
    const bool ready = mbar_wait_bounded(&S.full[s], (i / nstage) & 1, limit);
    if (__syncthreads_or(!ready)) {
      drain_stages(S.full, i, min(n, i + nstage), nstage);
      return;
    }
    for (int tile = 0; tile * tn < np; ++tile) {
      const int nt = min(tn, np - tile * tn);
      if (as != cur_a || np > tn) {
        // pair rows and their absmax over all of h (from k_gateup's per-tile maxima)
        float v[kTileN];
#pragma unroll
        for (int j = 0; j < kTileN; ++j) {
          v[j] = 0.f;
          if (j < nt) {
            const int p = S.R.pair_list[p0 + tile * tn + j];
            for (int q = threadIdx.x; q < R1; q += blockDim.x) v[j] = fmaxf(v[j], __ldcg(a.hmax + (size_t)p * R1 + q));
          }
        }
        if (threadIdx.x < kTileN)
          S.rows[threadIdx.x] = threadIdx.x < nt ? S.R.pair_list[p0 + tile * tn + threadIdx.x] : 0;
        block_max8(v, S.mx_red, S.mx_out);
        stage_f32_rows(a.h, S.rows, nt, a.I, S.mx_out, act, G.act_stride, S.shift);
        cur_a = as;
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      unit_mma<FD, FD>(acc, st, G, act, a.rows_act, warp, lane, bad);
      if (reduce_warps(acc, S.red, warp, lane)) {
        const int g = lane >> 2, t = lane & 3;
        const float s2 = FD == QK_FMT_NVFP4 ? a.down.scale_2[e] : 1.f;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int col = 2 * t + j;
          if (col < nt) {
            const float sh = pow2f(S.shift[col]) * s2;
            const int p = S.rows[col];
            float* pr = a.part + (size_t)p * a.H + r * 16;
            pr[g] = acc[j] * sh;
            pr[g + 8] = acc[2 + j] * sh;
          }
        }
      }
      __syncthreads();
    }
    // last expert to finish row tile r combines it, in slot order
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) S.flag = (atomicAdd(&a.counters[r], 1) == S.R.n_active - 1);
    __syncthreads();
    if (S.flag) {
      __threadfence();
      for (int idx = threadIdx.x; idx < a.T * 16; idx += blockDim.x) {
        const int tok = idx >> 4, m = r * 16 + (idx & 15);
        float yv = 0.f;
        for (int sl = 0; sl < a.k; ++sl) {
          const int p = tok * a.k + sl;
          const int ep = a.ids[p];
          if (ep < 0 || ep >= a.E) continue;
          yv = fmaf(a.w[p], __ldcg(a.part + (size_t)p * a.H + m), yv);
        }
        if (a.y_bf16)
          reinterpret_cast<__nv_bfloat16*>(a.y)[(size_t)tok * a.H + m] = __float2bfloat16_rn(yv);
        else
          reinterpret_cast<float*>(a.y)[(size_t)tok * a.H + m] = yv;
      }
    }
    if (threadIdx.x == 0 && i + nstage < n) issue(i + nstage);
  }
  if (bad) set_status(QK_ERR_NAN_SCALE);
}

// ================================================================= host ==
// Deepest ring (2..kMaxStages) that fits `budget` bytes of shared memory.
static int plan_stages(const Geo& G, int rows_act, size_t budget, size_t& smem) {
  const size_t fixed = kHeadBytes + (size_t)rows_act * G.act_stride * 2;
  const size_t cap = std::min(budget, (size_t)max_smem_optin());
  int s = kMaxStages;
  while (s > 2 && fixed + (size_t)s * G.stage > cap) --s;
  smem = fixed + (size_t)s * G.stage;
  return (smem <= (size_t)max_smem_optin()) ? s : 0;
}

// Budgets chosen so one k_gateup CTA and one k_down CTA fit on an SM together
// (228 KB): the dependent down kernel starts streaming its weights while the
// gate/up kernel drains.
constexpr size_t kBudgetGateUp = 132 * 1024;
constexpr size_t kBudgetDown = 92 * 1024;

template <int FG, int FU>
static qk_status launch_gateup(DecodeArgs& args, int grid, cudaStream_t st) {
  size_t smem = 0;
  const int s = plan_stages(make_geo(args.H, FG, FU), args.rows_act, kBudgetGateUp, smem);
  if (!s) return QK_ERR_UNSUPPORTED;
  args.stages = s;
  return launch_k(k_gateup<FG, FU>, smem, grid, args, st, false);
}

template <int FD>
static qk_status launch_down(DecodeArgs& args, int grid, cudaStream_t st) {
  size_t smem = 0;
  const int s = plan_stages(make_geo(args.I, FD, FD), args.rows_act, kBudgetDown, smem);
  if (!s) return QK_ERR_UNSUPPORTED;
  args.stages = s;
  return launch_k(k_down<FD>, smem, grid, args, st, true);
}

qk_status decode_forward(DecodeArgs args, cudaStream_t st) {
  const int sms = num_sms();
  args.rows_act = std::min(args.T, kTileN);
  const int amax = std::min(args.E, args.P);
  const int grid1 = std::max(1, std::min(sms, amax * (args.I / 8)));
  const int grid2 = std::max(1, std::min(sms, amax * (args.H / 16)));
  const int fg = args.gate.fmt, fu = args.up.fmt, fd = args.down.fmt;
  qk_status rc;
  if (fg == QK_FMT_MXFP4 && fu == QK_FMT_MXFP4) rc = launch_gateup<QK_FMT_MXFP4, QK_FMT_MXFP4>(args, grid1, st);
  else if (fg == QK_FMT_MXFP4) rc = launch_gateup<QK_FMT_MXFP4, QK_FMT_NVFP4>(args, grid1, st);
  else if (fu == QK_FMT_MXFP4) rc = launch_gateup<QK_FMT_NVFP4, QK_FMT_MXFP4>(args, grid1, st);
  else rc = launch_gateup<QK_FMT_NVFP4, QK_FMT_NVFP4>(args, grid1, st);
  if (rc != QK_OK) return rc;
  return fd == QK_FMT_MXFP4 ? launch_down<QK_FMT_MXFP4>(args, grid2, st)
                            : launch_down<QK_FMT_NVFP4>(args, grid2, st);
}

size_t decode_workspace_bytes(int T, int k, int H, int I) {
  const size_t P = (size_t)T * k;
  return align256(P * I * 4) + align256(P * (I / 8) * 4) + align256(P * H * 4) +
         align256((size_t)(H / 16) * 4);
}

void decode_carve(DecodeArgs& a, void* ws) {
  const size_t P = (size_t)a.P;
  uint8_t* p = static_cast<uint8_t*>(ws);
  a.h = reinterpret_cast<float*>(p);
  p += align256(P * a.I * 4);
  a.hmax = reinterpret_cast<float*>(p);
  p += align256(P * (a.I / 8) * 4);
  a.part = reinterpret_cast<float*>(p);
  p += align256(P * a.H * 4);
  a.counters = reinterpret_cast<int*>(p);
  a.n_counters = a.H / 16;
}

}  // namespace qk
