// qk_dmx.cu -- decode path for MXFP4 layers on the block-scaled tensor cores.
//
// At decode sizes (a few tokens, top-k experts each) the expert projections
// are weight-streaming matrix-vector products ("DeepSeek-v4-Flash-REAP-K180-
// NVFP4", "Why this mix?": gate+up carry about 2/3 of the expert bytes).  Here
// the e2m1 weights and their e8m0 scales go from HBM to the tensor core as
// stored (tcgen05.mma kind::mxf8f6f4.block_scale, B operand), and the few
// activation rows are the A operand, written as e4m3 terms with per-32
// scales: x (bf16) as two terms (exact), h (fp32) as three (relative error
// below 2^-12).  No weight element passes through a register.
//
// Work unit = (virtual expert of <= 8 pairs, 128 weight rows, 1024 elements
// of K): 8 reduction steps of 4 MMAs (M = 128 lanes, of which the first
// terms x pairs carry data; N = 128 weight rows; K = 32).  Units are split
// evenly and contiguously over two CTAs per SM: the per-instruction cost of
// tcgen05 issue, not the tensor pipe, bounds one CTA, and two issue in
// parallel (each holds 256 TMEM columns and ~112 KB of shared memory).
//
//   k_dmx<gate/up>  A = x terms; partial sums of each unit (per K chunk) to
//                   pg, no reduction across units.
//   k_dmx<down>     (programmatic dependent launch) A = h terms, built from
//                   the gate/up partials summed in chunk order, SwiGLU, and
//                   the split; partial sums to pd.
//   k_dmx_y         (programmatic dependent launch) one warp per (token,
//                   128 output rows): y in slot order from pd
//                   (deterministic).
//
// Warp roles (8 warps): weight TMA (16 x 4-bit -> 16-byte slots, box 128
// codes x 128 rows, 3 stages), MMA issuer, weight-scale formatter (16 bytes
// of 4 rows per lane per 4 steps, loaded a chunk ahead, written as
// tensor-memory scale atoms), epilogue (TMEM lanes 0-31: adds a pair's terms
// with shuffles), and 4 A builders (4 threads per 32-element block; one unit
// ahead, double-buffered).  One accumulator: the next unit's MMAs wait for
// the epilogue to read it.  Every wait is bounded.
#include <cuda.h>
#include <cuda_fp8.h>

#include "qk_common.cuh"
#include "qk_group.cuh"
#include "qk_route_table.cuh"
#include "qk_tmap.h"

namespace qk {

constexpr int kDN = 128;                 // weight rows per unit (MMA N)
constexpr int kDSteps = 8;               // reduction steps per unit
constexpr int kDKc = kDSteps * kXK;      // 1024 elements of K per unit
constexpr int kDWS = 3;                  // weight stages
constexpr int kDStageW = kDN * kXK;      // 16 KB (unpacked), 8 KB of packed weights
constexpr int kDRows = 24;               // A rows per step block (terms x pairs <= 24)
constexpr int kDABlock = kDRows * kXK;   // 3 KB
constexpr int kDAUnit = kDSteps * kDABlock;  // 24 KB per unit
constexpr int kDThreads = 8 * 32;    // warp 0 weights, 1 MMA, 2 weight scales, 4 epilogue, 3 and 5-7 A builders
constexpr int kDBuild = 4;           // A builder warps
constexpr int kDTmemCols = 256;          // one 128-column accumulator; scales from 128

struct DmxArgs {
  qk_weight A, B;        // gate/up phase: gate, up; down phase: down, down
  const uint16_t* x;     // bf16 [T][H]
  const int32_t* ids;    // [T][k]
  const float* w;        // [T][k]
  void* y;               // [T][H] fp32 or bf16
  float* pg;             // [P sorted][2 I / 128][H / 1024][128] gate/up partial sums
  float* pd;             // [P sorted][H / 128][I / 1024][128] down partial sums
  int T, k, E, H, I, P, y_bf16;
  alignas(64) CUtensorMap ta, tb;  // packed weights, 16 x 4-bit -> 16-byte slots, box {128, 128}, 128B swizzle
};

struct DmxHead {
  alignas(8) uint64_t wfull[kDWS];
  alignas(8) uint64_t wempty[kDWS];
  alignas(8) uint64_t afull[2];      // a unit's A blocks and scale atoms built
  alignas(8) uint64_t aempty[2];
  alignas(8) uint64_t sfull[2];      // four steps' weight scale atoms written
  alignas(8) uint64_t sempty[2];
  alignas(8) uint64_t acc_full[2];   // [0]: the accumulator holds a finished unit
  alignas(8) uint64_t acc_empty[2];  // [0]: the epilogue has read it ([1] unused)
  alignas(8) uint64_t drained;
  alignas(8) uint64_t epi_done;      // the epilogue warp has left its loop (TMEM reads done)
  uint32_t tmem;
  int abort;
};

constexpr int kDSmem = 1024 + 2 * kDAUnit + 2 * kDSteps * kSfAtom + kDWS * kDStageW + 2 * 4 * kSfAtom +
                       (((int)sizeof(Route) + 15) & ~15) + 256;
static_assert(sizeof(DmxHead) <= 256, "head");

// The A builders: 4 warps, 4 threads per 32-element block (8 elements each;
// the block's largest magnitude by two shuffles).  One e4m3 term of the 8
// values of this thread: codes in q (byte i = element i), the residual in v.
__device__ __forceinline__ int dsplit8(float (&v)[8], uint32_t (&q)[2]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const int ef = (int)((__float_as_uint(m) >> 23) & 0xFFu);
  const int c = min(max(ef - 7, 0), 254);  // the block maximum / 2^(c-127) in [128, 256)
  const float up = __uint_as_float((uint32_t)(254 - c) << 23);
  const float dn = c >= 1 ? __uint_as_float((uint32_t)c << 23) : __uint_as_float(0x00400000u);
#pragma unroll
  for (int i = 0; i < 8; i += 4) {
    const __nv_fp8x2_storage_t a =
        __nv_cvt_float2_to_fp8x2(make_float2(v[i] * up, v[i + 1] * up), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t b =
        __nv_cvt_float2_to_fp8x2(make_float2(v[i + 2] * up, v[i + 3] * up), __NV_SATFINITE, __NV_E4M3);
    q[i / 4] = (uint32_t)a | ((uint32_t)b << 16);
    const float2 da = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(a, __NV_E4M3)));
    const float2 db = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(b, __NV_E4M3)));
    v[i] -= da.x * dn;
    v[i + 1] -= da.y * dn;
    v[i + 2] -= db.x * dn;
    v[i + 3] -= db.y * dn;
  }
  return c;
}

// Quarter qq (8 codes) of block kb of A row m in a step block, and (qq = 0)
// the block's scale byte in the step's atom.
__device__ __forceinline__ void dput8(uint8_t* blk, uint8_t* atom, int m, int kb, int qq, const uint32_t (&q)[2],
                                      int c) {
  uint8_t* row = blk + m * kXK;
  *reinterpret_cast<uint2*>(row + (((2 * kb + (qq >> 1)) ^ (m & 7)) << 4) + 8 * (qq & 1)) = make_uint2(q[0], q[1]);
  if (qq == 0) atom[(m & 31) * 16 + (m >> 5) * 4 + kb] = (uint8_t)c;
}

// Gate/up A rows of one unit: pair j of the virtual expert -> rows 2 j, 2 j + 1
// (x split in two terms), 32-element block b (0..31) of the unit's K chunk.
// bt: builder thread (0..127).
__device__ __forceinline__ void build_x(const DmxArgs& G, const Route& R, int v, int kc, uint8_t* ablk,
                                        uint8_t* aatom, int bt) {
  const int n = R.v_n[v], p0 = R.v_p0[v], qq = bt & 3;
  for (int it = bt >> 2; it < n * (kDKc / 32); it += kDBuild * 8) {
    const int j = it / (kDKc / 32), b = it % (kDKc / 32);
    const int t = R.pair_list[p0 + j] / G.k;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(G.x + (size_t)t * G.H + (size_t)kc * kDKc + b * 32 + qq * 8));
    const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
    float v8[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v8[2 * i] = bf16_bits_to_f32(wd[i] & 0xFFFFu);
      v8[2 * i + 1] = bf16_bits_to_f32(wd[i] >> 16);
    }
    bool fin = true;
#pragma unroll
    for (int i = 0; i < 8; ++i) fin &= finite_bits(v8[i]);
    if (!fin) set_status(QK_ERR_NONFINITE);  // an inf or NaN in x
    const int s = b >> 2, kb = b & 3;
    uint32_t q[2];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      const int c = dsplit8(v8, q);
      dput8(ablk + s * kDABlock, aatom + s * kSfAtom, 2 * j + tt, kb, qq, q, c);
    }
  }
}

// Down A rows of one unit: pair j -> rows 3 j .. 3 j + 2, h = silu(g) * u with
// g and u the gate/up partial sums added in chunk order.
__device__ __forceinline__ void build_h(const DmxArgs& G, const Route& R, int v, int kc, uint8_t* ablk,
                                        uint8_t* aatom, int bt) {
  const int n = R.v_n[v], p0 = R.v_p0[v], qq = bt & 3;
  const int NB1 = 2 * G.I / kDN, CH1 = G.H / kDKc;
  for (int it = bt >> 2; it < n * (kDKc / 32); it += kDBuild * 8) {
    const int j = it / (kDKc / 32), b = it % (kDKc / 32);
    const int k0 = kc * kDKc + b * 32 + qq * 8;  // first element of I of this thread
    const int gb = k0 / kDN, off = k0 % kDN;
    const float* pg = G.pg + (size_t)(p0 + j) * NB1 * CH1 * kDN;
    float g[8], u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) g[i] = u[i] = 0.f;
    for (int c = 0; c < CH1; ++c) {
      const float4* gs = reinterpret_cast<const float4*>(pg + ((size_t)gb * CH1 + c) * kDN + off);
      const float4* us = reinterpret_cast<const float4*>(pg + ((size_t)(NB1 / 2 + gb) * CH1 + c) * kDN + off);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float4 a = __ldcg(gs + q), d = __ldcg(us + q);
        g[4 * q] += a.x;
        g[4 * q + 1] += a.y;
        g[4 * q + 2] += a.z;
        g[4 * q + 3] += a.w;
        u[4 * q] += d.x;
        u[4 * q + 1] += d.y;
        u[4 * q + 2] += d.z;
        u[4 * q + 3] += d.w;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) g[i] = __fdividef(g[i], 1.0f + __expf(-g[i])) * u[i];
    bool fin = true;
#pragma unroll
    for (int i = 0; i < 8; ++i) fin &= finite_bits(g[i]);
    if (!fin) set_status(QK_ERR_NONFINITE);  // h beyond fp32 (or from non-finite inputs)
    const int s = b >> 2, kb = b & 3;
    uint32_t q[2];
#pragma unroll
    for (int tt = 0; tt < 3; ++tt) {
      const int c = dsplit8(g, q);
      dput8(ablk + s * kDABlock, aatom + s * kSfAtom, 3 * j + tt, kb, qq, q, c);
    }
  }
}

}  // namespace qk

namespace qk {

template <bool GATEUP>
__global__ void __launch_bounds__(kDThreads, 2) k_dmx(const __grid_constant__ DmxArgs G) {
  constexpr int NT = GATEUP ? 2 : 3;  // terms per pair
  extern __shared__ __align__(16) uint8_t smem_raw[];  // rounded up to 1024 below, at run time
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  // A blocks first: the MMA reads 128 rows (16 KB) from each 3-KB step block,
  // so the rows past a block's 24 fall on later blocks or the weight ring.
  uint8_t* sA = base;                                // 2 units x 8 steps x 3 KB
  uint8_t* sW = sA + 2 * kDAUnit;                    // kDWS x 16 KB
  uint8_t* sAa = sW + kDWS * kDStageW;               // 2 units x 8 steps x 512 B A scale atoms
  uint8_t* sWa = sAa + 2 * kDSteps * kSfAtom;        // 2 slots x 4 steps x 512 B weight scale atoms
  Route& R = *reinterpret_cast<Route*>(sWa + 2 * 4 * kSfAtom);
  DmxHead& S = *reinterpret_cast<DmxHead*>(reinterpret_cast<uint8_t*>(&R) + ((sizeof(Route) + 15) & ~(size_t)15));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned long long limit = g_wait_limit_ns;
  const int K = GATEUP ? G.H : G.I;
  const int NB = GATEUP ? 2 * G.I / kDN : G.H / kDN;  // weight blocks per expert
  const int CH = K / kDKc;                             // K chunks

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDWS; ++s) {
      mbar_init(&S.wfull[s], 1);
      mbar_init(&S.wempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&S.afull[s], kDBuild);
      mbar_init(&S.aempty[s], 1);
      mbar_init(&S.sfull[s], 1);
      mbar_init(&S.sempty[s], 1);
      mbar_init(&S.acc_full[s], 1);
      mbar_init(&S.acc_empty[s], 1);
    }
    mbar_init(&S.drained, 1);
    mbar_init(&S.epi_done, 1);
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&S.tmem, kDTmemCols);
  // The ids may come from the kernel launched just before (router); the down
  // kernel's ids were complete before the gate/up kernel it follows started.
  if (GATEUP) pdl_wait();
  build_route(G.ids, G.P, G.E, R);  // ends with __syncthreads
  pdl_launch_dependents();  // the next kernel (down, then k_dmx_y) may start its prologue
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem;
  const int U = R.n_v * NB * CH;
  const int u0 = (int)((long long)blockIdx.x * U / gridDim.x), u1 = (int)((long long)(blockIdx.x + 1) * U / gridDim.x);
  auto unit = [&](int u, int& v, int& nb, int& c) {
    c = u % CH;
    nb = (u / CH) % NB;
    v = u / (CH * NB);
  };
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(&S.abort)) return false;
    if (mbar_wait_bounded(bar, parity, limit)) return true;
    set_status(QK_ERR_TIMEOUT);
    *reinterpret_cast<volatile int*>(&S.abort) = 1;
    return false;
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile int*>(&S.abort) != 0; };
  auto wrow_of = [&](int v, int nb, const void*& map) {
    const int e = R.v_expert[v];
    if (GATEUP && nb >= NB / 2) {
      map = &G.tb;
      return e * G.I + (nb - NB / 2) * kDN;
    }
    map = &G.ta;
    return e * (GATEUP ? G.I : G.H) + nb * kDN;
  };

  if (warp == 0) {
    // ----------------------------------------------------- weight tiles --
    if (lane == 0) {
      const uint64_t pw = policy_evict_first();
      int q = 0;
      bool ok = true;
      for (int u = u0; u < u1 && ok && !aborted(); ++u) {
        int v, nb, c;
        unit(u, v, nb, c);
        const void* m;
        const int y = wrow_of(v, nb, m);
        for (int st = 0; st < kDSteps; ++st, ++q) {
          const int s = q % kDWS;
          if (q >= kDWS && !wait(&S.wempty[s], (uint32_t)((q / kDWS - 1) & 1))) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&S.wfull[s], (uint32_t)kDStageW / 2);  // counted in packed (4-bit) bytes
          tma_load_2d(sW + s * kDStageW, m, (c * kDSteps + st) * kXK, y, &S.wfull[s], pw);
        }
      }
      for (int r = q > kDWS ? q - kDWS : 0; r < q; ++r)  // nothing may still be landing at exit
        if (!mbar_wait_bounded(&S.wfull[r % kDWS], (uint32_t)((r / kDWS) & 1), kDrainLimitNs)) break;
    }
    __syncwarp();
  } else if (warp == 2) {
    // ----------------------------------------------------- weight scales --
    // Per 4 steps: 16 bytes of each of the unit's 128 rows (4 per lane),
    // loaded one chunk ahead.
    const int srow = K / 32;
    auto load = [&](int n, uint4 (&r)[4]) {  // chunk n of this CTA
      int v, nb, c;
      unit(u0 + n / 2, v, nb, c);
      const void* m;
      const int r0 = wrow_of(v, nb, m);
      const uint8_t* sc = (GATEUP && nb >= NB / 2) ? G.B.scales : G.A.scales;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        r[j] = __ldg(reinterpret_cast<const uint4*>(sc + (size_t)(r0 + 32 * j + lane) * srow + (2 * c + (n & 1)) * 16));
    };
    const int nch = 2 * (u1 - u0);
    uint4 cur[4], nxt[4];
    if (nch > 0) load(0, nxt);
    for (int n = 0; n < nch; ++n) {
#pragma unroll
      for (int j = 0; j < 4; ++j) cur[j] = nxt[j];
      if (n + 1 < nch) load(n + 1, nxt);
      uint32_t ff = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        ff |= __vcmpeq4(cur[j].x, 0xFFFFFFFFu) | __vcmpeq4(cur[j].y, 0xFFFFFFFFu) | __vcmpeq4(cur[j].z, 0xFFFFFFFFu) |
              __vcmpeq4(cur[j].w, 0xFFFFFFFFu);
      if (ff) set_status(QK_ERR_NAN_SCALE);
      const int s = n & 1;
      if (n >= 2 && !__all_sync(0xffffffffu, wait(&S.sempty[s], (uint32_t)((n / 2 - 1) & 1)))) break;
      uint8_t* d = sWa + s * 4 * kSfAtom + lane * 16;
      *reinterpret_cast<uint4*>(d) = make_uint4(cur[0].x, cur[1].x, cur[2].x, cur[3].x);
      *reinterpret_cast<uint4*>(d + kSfAtom) = make_uint4(cur[0].y, cur[1].y, cur[2].y, cur[3].y);
      *reinterpret_cast<uint4*>(d + 2 * kSfAtom) = make_uint4(cur[0].z, cur[1].z, cur[2].z, cur[3].z);
      *reinterpret_cast<uint4*>(d + 3 * kSfAtom) = make_uint4(cur[0].w, cur[1].w, cur[2].w, cur[3].w);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&S.sfull[s]);
    }
  } else if (warp == 3 || warp >= 5) {
    // -------------------------------------------------------- A builders --
    const int bt = (warp == 3 ? 0 : warp - 4) * 32 + lane;
    if (!GATEUP) pdl_wait();  // the gate/up partial sums
    int i = 0;
    for (int u = u0; u < u1; ++u, ++i) {
      int v, nb, c;
      unit(u, v, nb, c);
      const int b = i & 1;
      if (i >= 2 && !__all_sync(0xffffffffu, wait(&S.aempty[b], (uint32_t)((i / 2 - 1) & 1)))) break;
      if (GATEUP)
        build_x(G, R, v, c, sA + b * kDAUnit, sAa + b * kDSteps * kSfAtom, bt);
      else
        build_h(G, R, v, c, sA + b * kDAUnit, sAa + b * kDSteps * kSfAtom, bt);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&S.afull[b]);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t t_sfa = tmem + kDN, t_sfb = t_sfa + 4;
      const uint32_t idesc = umma_idesc_mx(128, kDN, 0, 5);  // A e4m3 (activation terms), B e2m1 (weights)
      int q = 0, ns = 0, i = 0;
      for (int u = u0; u < u1 && !aborted(); ++u, ++i) {
        const int ab = i & 1;
        if (i >= 1 && !wait(&S.acc_empty[0], (uint32_t)((i - 1) & 1))) break;
        if (!wait(&S.afull[ab], (uint32_t)((i / 2) & 1))) break;
        tc_fence_after();
        bool ok = true;
        for (int st = 0; st < kDSteps; ++st, ++q) {
          const int sw = q % kDWS, sc = ns & 1, h = st & 3;
          if (!wait(&S.wfull[sw], (uint32_t)((q / kDWS) & 1)) || (h == 0 && !wait(&S.sfull[sc], (uint32_t)((ns / 2) & 1)))) {
            ok = false;
            break;
          }
          tc_fence_after();
          utccp_32x128b_x4(t_sfa, umma_desc_sf(sAa + (ab * kDSteps + st) * kSfAtom));
          utccp_32x128b_x4(t_sfb, umma_desc_sf(sWa + (sc * 4 + h) * kSfAtom));
          const uint64_t da = umma_desc_k_sw128(sA + ab * kDAUnit + st * kDABlock);
          const uint64_t db = umma_desc_k_sw128(sW + sw * kDStageW);
#pragma unroll
          for (int kb = 0; kb < kXK / 32; ++kb)
            umma_mx(tmem, da + 2 * kb, db + 2 * kb, umma_idesc_sf_ids(idesc, kb, kb),
                    t_sfa | ((uint32_t)kb << 30), t_sfb | ((uint32_t)kb << 30), (st | kb) != 0 ? 1u : 0u);
          umma_commit(&S.wempty[sw]);
          if (h == 3) {
            umma_commit(&S.sempty[sc]);
            ++ns;
          }
        }
        if (!ok) break;
        umma_commit(&S.aempty[ab]);
        umma_commit(&S.acc_full[0]);
      }
      umma_commit(&S.drained);  // every MMA issued here completes before the accumulator is freed
      mbar_wait_bounded(&S.drained, 0, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp == 4) {
    // ---------------------------------------------------------- epilogue --
    // TMEM lanes 0-31: lane NT j + t = term t of pair j.  The pair's sum goes
    // to the unit's partial row (sorted pair position, weight block, chunk).
    float* part = GATEUP ? G.pg : G.pd;
    int i = 0;
    for (int u = u0; u < u1; ++u, ++i) {
      int v, nb, c;
      unit(u, v, nb, c);
      const int n = R.v_n[v], p0 = R.v_p0[v];
      if (!__all_sync(0xffffffffu, wait(&S.acc_full[0], (uint32_t)(i & 1)))) break;
      tc_fence_after();
      const int j = lane / NT;
      const bool st = lane % NT == 0 && j < n;
      float* dst = part + (((size_t)(p0 + (st ? j : 0)) * NB + nb) * CH + c) * kDN;
#pragma unroll 1
      for (int ch = 0; ch < kDN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(tmem + (uint32_t)(ch * 32), r);
        if (ch == kDN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_one(&S.acc_empty[0]);
        }
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const float a = __uint_as_float(r[jj]);
          float s = a + __shfl_down_sync(0xffffffffu, a, 1);
          if (NT == 3) s += __shfl_down_sync(0xffffffffu, a, 2);
          r[jj] = __float_as_uint(s);
        }
        if (st) {
          float4* o = reinterpret_cast<float4*>(dst + ch * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            o[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                               __uint_as_float(r[4 * q + 3]));
        }
      }
    }
  }
  if (warp == 4) {  // the epilogue's TMEM reads are done (also on an early exit)
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_one(&S.epi_done);
  }
  __syncthreads();
  if (warp == 1) {
    // (a CTA barrier after long single-lane loops is not relied on alone)
    mbar_wait_bounded(&S.epi_done, 0, kDrainLimitNs);
    tc_fence_after();
    tmem_free(tmem, kDTmemCols);
  }
}

// y[t][block nb] = sum over slots s in order of w[t][s] * (sum over K chunks
// in order of the down partial sums): one warp per (token, 128-row output
// block), 32 lanes x 4 rows; all the (slot, chunk) loads in flight at once.
// Launched after the down kernel (programmatic dependent launch): the
// routing table is built while the down kernel runs; griddepcontrol.wait
// returns when its partial sums are complete and visible.
constexpr int kDyWarps = 8;
__global__ void __launch_bounds__(kDyWarps * 32) k_dmx_y(const __grid_constant__ DmxArgs G) {
  __shared__ Route R;
  build_route(G.ids, G.P, G.E, R);  // ends with __syncthreads
  pdl_wait();
  const int lane = threadIdx.x & 31, nb = blockIdx.x, t = blockIdx.y * kDyWarps + (threadIdx.x >> 5);
  if (t >= G.T) return;
  const int NB = G.H / kDN, CH = G.I / kDKc;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (CH <= 4) {
    float4 x4[8][4];
    float wt[8];
    bool on[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      on[s] = false;
      if (s < G.k) {
        const int p = t * G.k + s, pv = R.pair_v[p];
        if (pv >= 0) {
          on[s] = true;
          wt[s] = __ldg(G.w + p);
          const float4* src =
              reinterpret_cast<const float4*>(G.pd + (size_t)(R.v_p0[pv] + R.pair_j[p]) * NB * CH * kDN) +
              (size_t)nb * CH * (kDN / 4) + lane;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            if (cc < CH) x4[s][cc] = __ldcg(src + cc * (kDN / 4));
        }
      }
    }
#pragma unroll
    for (int s = 0; s < 8; ++s)
      if (on[s]) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          if (cc < CH) {
            d[0] += x4[s][cc].x;
            d[1] += x4[s][cc].y;
            d[2] += x4[s][cc].z;
            d[3] += x4[s][cc].w;
          }
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = fmaf(wt[s], d[q], acc[q]);
      }
  } else {
    for (int s = 0; s < G.k; ++s) {
      const int p = t * G.k + s, pv = R.pair_v[p];
      if (pv < 0) continue;
      const int sp = R.v_p0[pv] + R.pair_j[p];
      const float wt = G.w[p];
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      for (int cc = 0; cc < CH; ++cc) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(G.pd + (((size_t)sp * NB + nb) * CH + cc) * kDN) + lane);
        d[0] += v.x;
        d[1] += v.y;
        d[2] += v.z;
        d[3] += v.w;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = fmaf(wt, d[q], acc[q]);
    }
  }
  if (!(finite_bits(acc[0]) && finite_bits(acc[1]) && finite_bits(acc[2]) && finite_bits(acc[3])))
    set_status(QK_ERR_NONFINITE);
  const size_t o = (size_t)t * G.H + nb * kDN + lane * 4;
  if (G.y_bf16) {
    __nv_bfloat16* yb = reinterpret_cast<__nv_bfloat16*>(G.y) + o;
#pragma unroll
    for (int q = 0; q < 4; ++q) yb[q] = __float2bfloat16_rn(acc[q]);
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(G.y) + o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
}

}  // namespace qk

namespace qk {

// ================================================================= host ==
bool dmx_eligible(const qk_weight& gate, const qk_weight& up, const qk_weight& down, int H, int I) {
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (gate.fmt != QK_FMT_MXFP4 || up.fmt != QK_FMT_MXFP4 || down.fmt != QK_FMT_MXFP4) return false;
  if (H % kDKc != 0 || I % kDKc != 0) return false;
  return al(gate.q, 32) && al(up.q, 32) && al(down.q, 32) && al(gate.scales, 16) && al(up.scales, 16) &&
         al(down.scales, 16);
}

struct DmxWs {
  size_t pg, pd, total;
};
static DmxWs dmx_layout(int T, int k, int H, int I) {
  const size_t P = (size_t)T * k;
  DmxWs L;
  size_t o = 0;
  L.pg = o; o += align256(P * (2 * I / kDN) * (H / kDKc) * kDN * 4);
  L.pd = o; o += align256(P * (H / kDN) * (I / kDKc) * kDN * 4);
  L.total = o;
  return L;
}
size_t dmx_workspace_bytes(int T, int k, int H, int I) { return dmx_layout(T, k, H, I).total; }

static bool d_map_weights(CUtensorMap* m, const uint8_t* q, int64_t rows, int K) {
  const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)K / 2};
  const uint32_t box[2] = {(uint32_t)kXK, (uint32_t)kDN};
  return tmap_get(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

template <bool GATEUP>
static qk_status d_launch(const DmxArgs& A, cudaStream_t st) {
  if (kDSmem > max_smem_optin()) return QK_ERR_UNSUPPORTED;
  return launch_ex(k_dmx<GATEUP>, dim3(2 * num_sms()), dim3(kDThreads), (size_t)kDSmem, st, true, A);
}

qk_status dmx_forward(const DecodeArgs& a, void* workspace, cudaStream_t st) {
  const DmxWs L = dmx_layout(a.T, a.k, a.H, a.I);
  uint8_t* p = static_cast<uint8_t*>(workspace);
  DmxArgs g = {};
  g.x = a.x;
  g.ids = a.ids;
  g.w = a.w;
  g.y = a.y;
  g.pg = reinterpret_cast<float*>(p + L.pg);
  g.pd = reinterpret_cast<float*>(p + L.pd);
  g.T = a.T;
  g.k = a.k;
  g.E = a.E;
  g.H = a.H;
  g.I = a.I;
  g.P = a.P;
  g.y_bf16 = a.y_bf16;
  g.A = a.gate;
  g.B = a.up;
  if (!d_map_weights(&g.ta, a.gate.q, (int64_t)a.E * a.I, a.H) ||
      !d_map_weights(&g.tb, a.up.q, (int64_t)a.E * a.I, a.H))
    return QK_ERR_CUDA;
  qk_status rc = d_launch<true>(g, st);
  if (rc != QK_OK) return rc;
  g.A = a.down;
  g.B = a.down;
  if (!d_map_weights(&g.ta, a.down.q, (int64_t)a.E * a.H, a.I)) return QK_ERR_CUDA;
  g.tb = g.ta;
  rc = d_launch<false>(g, st);
  if (rc != QK_OK) return rc;
  return launch_ex(k_dmx_y, dim3(a.H / kDN, (a.T + kDyWarps - 1) / kDyWarps), dim3(kDyWarps * 32), 0, st, true, g);
}

}  // namespace qk
