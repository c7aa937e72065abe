// qk_gmx.cu -- MXFP4 grouped path on the block-scaled tensor cores.
//
// The pages store MXFP4 experts as e2m1 codes with one e8m0 scale per 32
// weights ("DeepSeek-v4-Flash-REAP-K180-NVFP4", "NVFP4: lossless MXFP4->NVFP4
// conversion") and run the expert projections as one grouped GEMM per
// projection ("DeepSeekv4 Flash for 1x Spark [REAP25]", "What's actually
// different").  sm_100a multiplies that format directly: tcgen05.mma
// kind::mxf8f6f4.block_scale takes e2m1 A with a ue8m0 scale per 32 elements
// of K, e4m3 B with its own per-32 scales, and accumulates in fp32.  The
// weights go from HBM to the tensor core unchanged (TMA expands each 8-byte
// group of 16 codes into the 16-byte slot the tensor core reads); nothing is
// dequantized in registers.
//
// Activations are bf16 (and h is fp32), so each is written as a sum of e4m3
// terms with per-32 scales:  v = t0 2^(c0-127) + t1 2^(c1-127) [+ t2 ...],
// t_i = RN_e4m3(residual / 2^(c_i-127)), c_i chosen so the block's largest
// residual maps into [128, 256).  A bf16 value has 8 significant bits and
// each e4m3 term takes 4, and the first residual of a bf16 value needs at most
// 4 bits, so two terms reproduce x exactly (except for values within the e4m3
// subnormal range of their block, below 2^-13 of its largest element).  h is
// fp32: three terms keep its relative error below 2^-12.  Each term is one
// more MMA on the same weight tile.
//
//   k_gmx_xsplit  per token: x -> 2 e4m3 terms at the sorted row of each of
//                 its pairs, scales in the tensor-memory atom layout per tile.
//   k_gmx<gate/up>  per (expert, 128 gate or 128 up rows, token tile of
//                 <= 80 rows): gate and up outputs (fp32) to gu.
//   k_gmx_hsplit  per sorted row: h = silu(gate) * up -> 3 e4m3 terms.
//   k_gmx<down>   per (expert, 128 down rows, token tile): d (fp32).
//
// The terms of a token tile are stacked along N: one MMA takes B = [t0 rows;
// t1 rows (; t2 rows)] (N' = terms x box rows <= 240) and the epilogue adds
// the terms' accumulator columns.  This keeps the instruction count per
// reduction step at four MMAs whatever the number of terms.
//
// Scale-factor atom (the layout tcgen05.cp 32x128b.warpx4 copies into tensor
// memory): 512 bytes for 128 rows x 4 blocks of 32 along K; row r, block b at
// byte (r % 32) * 16 + (r / 32) * 4 + b.  A token tile's B rows span two atoms
// per reduction step (rows 0-127, 128-255).
#include <cuda.h>
#include <cuda_fp8.h>

#include "qk_common.cuh"
#include "qk_group.cuh"
#include "qk_tmap.h"

namespace qk {

// ------------------------------------------------------------ term split --
// One e4m3 term of the 32 values v (one scale block): returns the ue8m0 code
// c, writes the 32 codes (byte i = element i) to q and leaves the residual
// v - t * 2^(c-127) in v (exact in fp32).
__device__ __forceinline__ int split_term(float (&v)[32], uint32_t (&q)[8]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
  const int ef = (int)((__float_as_uint(m) >> 23) & 0xFFu);  // biased exponent of the block maximum
  const int c = min(max(ef - 7, 0), 254);                     // m / 2^(c-127) in [128, 256)
  const float up = __uint_as_float((uint32_t)(254 - c) << 23);  // 2^(127-c)
  const float dn = c >= 1 ? __uint_as_float((uint32_t)c << 23) : __uint_as_float(0x00400000u);  // 2^(c-127)
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const __nv_fp8x2_storage_t a = __nv_cvt_float2_to_fp8x2(make_float2(v[i] * up, v[i + 1] * up), __NV_SATFINITE, __NV_E4M3);
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

// Token rows of tile f's B operand (the TMA box height): 32, 64 or 80.
__host__ __device__ __forceinline__ int xbox_rows(int n) { return n <= 32 ? 32 : n <= 64 ? 64 : kXN; }

// Byte of the scale of B row rb (term * box rows + token row), reduction
// step `stage` (of ns), block b4 (0-3) of tile f: [F][ns][2 atoms][512].
__device__ __forceinline__ size_t sf_atom_byte(int f, int stage, int ns, int rb, int b4) {
  const int r = rb & 127;
  return (((size_t)f * ns + stage) * 2 + (rb >> 7)) * kSfAtom + (size_t)((r & 31) * 16 + (r >> 5) * 4 + b4);
}

// One block per token: its pairs' sorted rows (counting-sort scatter), then
// x split into two e4m3 terms per 32-block, written at each of those rows.
__global__ void __launch_bounds__(kRowThreads) k_gmx_xsplit(GroupWs W, const uint16_t* __restrict__ x,
                                                            const int32_t* __restrict__ ids, int k, int E, int H,
                                                            int P) {
  __shared__ int pos[8], fj[8], fbox[8];
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    const int p = t * k + threadIdx.x;
    const int e = ids[p];
    int r = -1, tj = 0;
    if (e >= 0 && e < E) {
      const int o = W.offsets[e];
      r = o + atomicAdd(&W.fill[e], 1);
      const int rel = r - o;
      tj = ((W.exp_tile0[e] + rel / kXN) << 8) | (rel % kXN);
      W.rtile[r] = tj;
    } else {
      set_status(QK_ERR_INVALID_ARG);
    }
    W.inv[p] = r;
    pos[threadIdx.x] = r;
    fj[threadIdx.x] = tj;
    fbox[threadIdx.x] = r >= 0 ? xbox_rows(W.tile_n[tj >> 8]) : 0;
  }
  __syncthreads();
  const int nb = H / 32, ns = H / kXK;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  for (int b = threadIdx.x; b < nb; b += kRowThreads) {
    float v[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = __ldg(src + b * 4 + q);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[q * 8 + 2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        v[q * 8 + 2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
      }
    }
    uint32_t q0[8], q1[8];
    const int c0 = split_term(v, q0);
    const int c1 = split_term(v, q1);
    for (int s = 0; s < k; ++s) {
      const int r = pos[s];
      if (r < 0) continue;
      uint4* d0 = reinterpret_cast<uint4*>(W.xq + (size_t)r * H + b * 32);
      uint4* d1 = reinterpret_cast<uint4*>(W.xq + (size_t)P * H + (size_t)r * H + b * 32);
      d0[0] = make_uint4(q0[0], q0[1], q0[2], q0[3]);
      d0[1] = make_uint4(q0[4], q0[5], q0[6], q0[7]);
      d1[0] = make_uint4(q1[0], q1[1], q1[2], q1[3]);
      d1[1] = make_uint4(q1[4], q1[5], q1[6], q1[7]);
      const int f = fj[s] >> 8, j = fj[s] & 255;
      W.sfx[sf_atom_byte(f, b >> 2, ns, j, b & 3)] = (uint8_t)c0;
      W.sfx[sf_atom_byte(f, b >> 2, ns, fbox[s] + j, b & 3)] = (uint8_t)c1;
    }
  }
}

// One block per sorted row: h = silu(gate) * up in fp32, split into three
// e4m3 terms per 32-block.
__global__ void __launch_bounds__(kRowThreads) k_gmx_hsplit(GroupWs W, int E, int I, int P) {
  const int r = blockIdx.x;
  if (r >= W.offsets[E]) return;  // block-uniform
  const int tj = W.rtile[r], f = tj >> 8, j = tj & 255, nb_rows = xbox_rows(W.tile_n[f]);
  const float4* g4 = reinterpret_cast<const float4*>(W.gu + (size_t)r * 2 * I);
  const float4* u4 = g4 + I / 4;
  const int nb = I / 32, ns = I / kXK;
  for (int b = threadIdx.x; b < nb; b += kRowThreads) {
    float v[32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 g = __ldcg(g4 + b * 8 + q), u = __ldcg(u4 + b * 8 + q);
      v[4 * q + 0] = __fdividef(g.x, 1.0f + __expf(-g.x)) * u.x;
      v[4 * q + 1] = __fdividef(g.y, 1.0f + __expf(-g.y)) * u.y;
      v[4 * q + 2] = __fdividef(g.z, 1.0f + __expf(-g.z)) * u.z;
      v[4 * q + 3] = __fdividef(g.w, 1.0f + __expf(-g.w)) * u.w;
    }
#pragma unroll
    for (int term = 0; term < 3; ++term) {
      uint32_t q[8];
      const int c = split_term(v, q);
      uint4* d = reinterpret_cast<uint4*>(W.hq + (size_t)term * P * I + (size_t)r * I + b * 32);
      d[0] = make_uint4(q[0], q[1], q[2], q[3]);
      d[1] = make_uint4(q[4], q[5], q[6], q[7]);
      W.sfh[sf_atom_byte(f, b >> 2, ns, term * nb_rows + j, b & 3)] = (uint8_t)c;
    }
  }
}

}  // namespace qk

namespace qk {

// ---------------------------------------------------------- grouped GEMM --
constexpr int kXM = 128;          // weight rows per tile (tcgen05 M)
constexpr int kXNBox = 3;         // token-box heights 32, 64, 80
constexpr int kXThreads = 8 * 32; // warp 0 weights, 1 MMA, 2 tokens, 3 weight scales, 4-7 epilogue
constexpr int kXStageA = kXM * kXK;    // 16 KB: 128 rows x 128 codes, one code per byte position
constexpr int kXAS = 6;                // weight stages
constexpr int kXSS = 2;                // weight-scale chunk slots (4 atoms = 4 reduction steps each)
constexpr int kXAccCols = 256;         // accumulator buffer stride (two buffers)
constexpr int kXSfaCol = 496;          // weight scales: 4 columns; token scales: 8 columns after them
constexpr int kXTmemCols = 512;

// A token stage holds 128 / n' of the tile's reduction steps, n' = 32 << i
// (one step of the stacked terms of an 80-row tile).
template <int NT>
struct GmxCfg {
  static constexpr int BS = NT == 2 ? 3 : 2;            // token stages
  static constexpr int kStageB = NT * 4 * 32 * kXK;     // NT x 16 KB
  static constexpr int kSfbStage = 4 * 2 * kSfAtom;     // up to four steps x two atoms
  static constexpr int kSmem = 1024 + kXAS * kXStageA + BS * kStageB + kXSS * 4 * kSfAtom + BS * kSfbStage + 256;
};
__host__ __device__ constexpr int xkpb(int bi) { return bi == 0 ? 4 : bi == 1 ? 2 : 1; }  // steps per token stage

struct GmxArgs {
  GroupWs W;
  const uint8_t* sf_a;   // e8m0 scales [E * rows][K / 32] of the gate (or down) rows
  const uint8_t* sf_b;   // e8m0 scales of the up rows (gate/up phase)
  const uint8_t* sfb;    // [F][K / 128][2][512] scale atoms of the stacked token terms
  float* out;            // gate/up: gu [P][2 I]; down: dperm [P][H]
  int K, rows_per_e, MB, MBA, out_ld, F;  // MBA: weight blocks taken from ta / sf_a (the rest: tb / sf_b)
  alignas(64) CUtensorMap ta, tb;     // packed weights, 16 x 4-bit -> 16-byte slots, box {128, 128}, 128B swizzle
  alignas(64) CUtensorMap tx[kXNBox]; // token terms {128, P, NT, K / 128}, box {128, n, NT, kpb}, 128B swizzle
};

struct GmxHead {
  alignas(8) uint64_t afull[kXAS];   // weight tile landed (TMA)
  alignas(8) uint64_t aempty[kXAS];  // its MMAs completed
  alignas(8) uint64_t sfull[kXSS];   // four weight scale atoms written (scale warp)
  alignas(8) uint64_t sempty[kXSS];
  alignas(8) uint64_t bfull[4];      // token terms and their scale atoms landed
  alignas(8) uint64_t bempty[4];
  alignas(8) uint64_t acc_full[2];
  alignas(8) uint64_t acc_empty[2];
  alignas(8) uint64_t drained;
  uint32_t tmem;
  int abort;
};

__device__ __forceinline__ int xbox_index(int n) { return n <= 32 ? 0 : n <= 64 ? 1 : 2; }

__device__ __forceinline__ uint64_t policy_evict_last_x() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Work tile t: the tiles of one expert are ordered weight block major, so
// consecutive blocks share a weight block (read from HBM once, then from L2)
// and differ in their token tile.
__device__ __forceinline__ void gmx_tile(const GroupWs& W, int MB, int t, int& f, int& mb) {
  const int f0 = t / MB;
  const int first = W.tile_first[f0], cnt = W.tile_cnt[f0];
  const int u = t - first * MB;
  mb = u / cnt;
  f = first + (u - mb * cnt);
}

template <bool GATEUP, int NT>
__global__ void __launch_bounds__(kXThreads, 1) k_gmx(const __grid_constant__ GmxArgs G) {
  constexpr int BS = GmxCfg<NT>::BS, SB = GmxCfg<NT>::kStageB, SFB = GmxCfg<NT>::kSfbStage;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sA = base;                          // kXAS weight stages
  uint8_t* sB = sA + kXAS * kXStageA;          // BS token stages
  uint8_t* sSa = sB + BS * SB;                 // kXSS x 4 weight scale atoms
  uint8_t* sSb = sSa + kXSS * 4 * kSfAtom;     // BS token scale stages
  GmxHead& S = *reinterpret_cast<GmxHead*>(sSb + BS * SFB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const GroupWs& W = G.W;
  const int MB = G.MB, KS = G.K / kXK;
  const unsigned long long limit = g_wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kXAS; ++s) {
      mbar_init(&S.afull[s], 1);
      mbar_init(&S.aempty[s], 1);
    }
    for (int s = 0; s < kXSS; ++s) {
      mbar_init(&S.sfull[s], 1);
      mbar_init(&S.sempty[s], 1);
    }
    for (int s = 0; s < BS; ++s) {
      mbar_init(&S.bfull[s], 1);
      mbar_init(&S.bempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.acc_full[b], 1);
      mbar_init(&S.acc_empty[b], 4);
    }
    mbar_init(&S.drained, 1);
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&S.tmem, kXTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem;
  const int n_tiles = *W.n_tiles * MB;
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*reinterpret_cast<volatile int*>(&S.abort)) return false;
    if (mbar_wait_bounded(bar, parity, limit)) return true;
    set_status(QK_ERR_TIMEOUT);
    if (atomicExch(&S.abort, 1) == 0 && lane == 0)
      printf("k_gmx<%d> timeout: block %d warp %d barrier byte %d parity %u tiles %d\n", GATEUP ? 1 : 0,
             (int)blockIdx.x, warp, (int)((uint8_t*)bar - (uint8_t*)&S), parity, n_tiles);
    return false;
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile int*>(&S.abort) != 0; };

  if (warp == 0) {
    // ----------------------------------------------------- weight tiles --
    if (lane == 0) {
      const uint64_t pw = policy_evict_normal();
      int n = 0;
      for (int t = blockIdx.x; t < n_tiles && !aborted(); t += gridDim.x) {
        int f, mb;
        gmx_tile(W, MB, t, f, mb);
        const bool b = mb >= G.MBA;
        const int wrow = W.tile_e[f] * G.rows_per_e + (b ? mb - G.MBA : mb) * kXM;
        for (int ks = 0; ks < KS; ++ks, ++n) {
          const int s = n % kXAS;
          if (n >= kXAS && !wait(&S.aempty[s], (uint32_t)((n / kXAS - 1) & 1))) break;
          mbar_arrive_expect_tx(&S.afull[s], (uint32_t)kXStageA / 2);  // counted in packed (4-bit) bytes
          tma_load_2d(sA + s * kXStageA, b ? &G.tb : &G.ta, ks * kXK, wrow, &S.afull[s], pw);
        }
      }
      for (int q = n > kXAS ? n - kXAS : 0; q < n; ++q)  // nothing may still be landing at exit
        if (!mbar_wait_bounded(&S.afull[q % kXAS], (uint32_t)((q / kXAS) & 1), kDrainLimitNs)) break;
    }
    __syncwarp();
  } else if (warp == 3) {
    // ----------------------------------------------------- weight scales --
    // Four reduction steps at a time: every lane loads 16 bytes (4 steps x 4
    // blocks) of four of the tile's rows, one chunk ahead, and writes the
    // four steps' atoms; one proxy fence and one arrival per chunk.
    const int srow = G.K / 32;  // scale bytes per weight row
    auto rows_of = [&](int t, const uint8_t* (&p)[4]) {
      int f, mb;
      gmx_tile(W, MB, t, f, mb);
      const bool b = mb >= G.MBA;
      const uint8_t* sc = b ? G.sf_b : G.sf_a;
      const size_t r0 = (size_t)W.tile_e[f] * G.rows_per_e + (b ? mb - G.MBA : mb) * kXM;
#pragma unroll
      for (int j = 0; j < 4; ++j) p[j] = sc + (r0 + 32 * j + lane) * srow;
    };
    uint4 cur[4], nxt[4];
    const uint8_t* rp[4];
    if ((int)blockIdx.x < n_tiles) {
      rows_of(blockIdx.x, rp);
#pragma unroll
      for (int j = 0; j < 4; ++j) nxt[j] = __ldg(reinterpret_cast<const uint4*>(rp[j]));
    }
    int n = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      for (int c = 0; c < KS / 4; ++c, ++n) {
#pragma unroll
        for (int j = 0; j < 4; ++j) cur[j] = nxt[j];
        const int tn = c + 1 < KS / 4 ? t : t + (int)gridDim.x;
        if (tn < n_tiles) {
          if (tn != t) rows_of(tn, rp);
          const int chunk = tn == t ? c + 1 : 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) nxt[j] = __ldg(reinterpret_cast<const uint4*>(rp[j] + chunk * 16));
        }
        uint32_t ff = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          ff |= __vcmpeq4(cur[j].x, 0xFFFFFFFFu) | __vcmpeq4(cur[j].y, 0xFFFFFFFFu) |
                __vcmpeq4(cur[j].z, 0xFFFFFFFFu) | __vcmpeq4(cur[j].w, 0xFFFFFFFFu);
        if (ff) set_status(QK_ERR_NAN_SCALE);
        const int s = n % kXSS;
        if (n >= kXSS && !__all_sync(0xffffffffu, wait(&S.sempty[s], (uint32_t)((n / kXSS - 1) & 1)))) {
          ok = false;
          break;
        }
        uint8_t* d = sSa + s * 4 * kSfAtom + lane * 16;
        *reinterpret_cast<uint4*>(d) = make_uint4(cur[0].x, cur[1].x, cur[2].x, cur[3].x);
        *reinterpret_cast<uint4*>(d + kSfAtom) = make_uint4(cur[0].y, cur[1].y, cur[2].y, cur[3].y);
        *reinterpret_cast<uint4*>(d + 2 * kSfAtom) = make_uint4(cur[0].z, cur[1].z, cur[2].z, cur[3].z);
        *reinterpret_cast<uint4*>(d + 3 * kSfAtom) = make_uint4(cur[0].w, cur[1].w, cur[2].w, cur[3].w);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_one(&S.sfull[s]);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------- token terms --
    // One stage = kpb reduction steps of the tile's stacked terms (one 4-D
    // TMA box) and their scale atoms (one bulk copy: contiguous per tile).
    if (lane == 0) {
      const uint64_t px = policy_evict_last_x();
      int n = 0;
      for (int t = blockIdx.x; t < n_tiles && !aborted(); t += gridDim.x) {
        int f, mb;
        gmx_tile(W, MB, t, f, mb);
        const int row0 = W.tile_row0[f], bi = xbox_index(W.tile_n[f]), kpb = xkpb(bi);
        const int nb_rows = bi == 2 ? kXN : 32 << bi;
        const uint32_t bytes = (uint32_t)(kpb * (NT * nb_rows * kXK + 2 * kSfAtom));
        for (int k0 = 0; k0 < KS; k0 += kpb, ++n) {
          const int s = n % BS;
          if (n >= BS && !wait(&S.bempty[s], (uint32_t)((n / BS - 1) & 1))) break;
          mbar_arrive_expect_tx(&S.bfull[s], bytes);
          tma_load_4d(sB + s * SB, &G.tx[bi], 0, row0, 0, k0, &S.bfull[s], px);
          bulk_g2s(sSb + s * SFB, G.sfb + ((size_t)f * KS + k0) * 2 * kSfAtom, (uint32_t)(kpb * 2 * kSfAtom),
                   &S.bfull[s]);
        }
      }
      for (int q = n > BS ? n - BS : 0; q < n; ++q)
        if (!mbar_wait_bounded(&S.bfull[q % BS], (uint32_t)((q / BS) & 1), kDrainLimitNs)) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t t_sfa = tmem + kXSfaCol, t_sfb = t_sfa + 4;
      int na = 0, nb = 0, nc = 0, i = 0;
      for (int t = blockIdx.x; t < n_tiles && !aborted(); t += gridDim.x, ++i) {
        int f, mb;
        gmx_tile(W, MB, t, f, mb);
        const int bi = xbox_index(W.tile_n[f]), kpb = xkpb(bi);
        const int nb_rows = bi == 2 ? kXN : 32 << bi, ncols = NT * nb_rows;  // MMA N
        const uint32_t idesc = umma_idesc_mx(kXM, ncols, 5, 0);
        const int ab = i & 1;
        if (i >= 2 && !wait(&S.acc_empty[ab], (uint32_t)((i / 2 - 1) & 1))) break;
        tc_fence_after();
        const uint32_t tacc = tmem + (uint32_t)(ab * kXAccCols);
        bool ok = true;
        for (int ks = 0; ks < KS; ++ks, ++na) {
          const int sa = na % kXAS, sb = nb % BS, sc = nc % kXSS, j = ks & (kpb - 1), q = ks & 3;
          if (!wait(&S.afull[sa], (uint32_t)((na / kXAS) & 1)) ||
              (j == 0 && !wait(&S.bfull[sb], (uint32_t)((nb / BS) & 1))) ||
              (q == 0 && !wait(&S.sfull[sc], (uint32_t)((nc / kXSS) & 1)))) {
            ok = false;
            break;
          }
          tc_fence_after();
          utccp_32x128b_x4(t_sfa, umma_desc_sf(sSa + (sc * 4 + q) * kSfAtom));
          const uint8_t* sfb = sSb + sb * SFB + j * 2 * kSfAtom;
          utccp_32x128b_x4(t_sfb, umma_desc_sf(sfb));
          if (ncols > 128) utccp_32x128b_x4(t_sfb + 4, umma_desc_sf(sfb + kSfAtom));
          const uint64_t da = umma_desc_k_sw128(sA + sa * kXStageA);
          const uint64_t db = umma_desc_k_sw128(sB + sb * SB + j * ncols * kXK);
#pragma unroll
          for (int kb = 0; kb < kXK / 32; ++kb)
            umma_mx(tacc, da + 2 * kb, db + 2 * kb, umma_idesc_sf_ids(idesc, kb, kb), t_sfa | ((uint32_t)kb << 30),
                    t_sfb | ((uint32_t)kb << 30), (ks | kb) != 0 ? 1u : 0u);
          umma_commit(&S.aempty[sa]);
          if (j == kpb - 1) {
            umma_commit(&S.bempty[sb]);
            ++nb;
          }
          if (q == 3) {
            umma_commit(&S.sempty[sc]);
            ++nc;
          }
        }
        if (!ok) break;
        umma_commit(&S.acc_full[ab]);
      }
      umma_commit(&S.drained);  // every MMA issued here completes before the accumulator is freed
      mbar_wait_bounded(&S.drained, 0, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------- epilogue --
    // Accumulator column tt * n + j holds term tt of token row j.
    const int quad = warp & 3, feat = quad * 32 + lane;
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      int f, mb;
      gmx_tile(W, MB, t, f, mb);
      const int row0 = W.tile_row0[f], nrow = W.tile_n[f];
      const int bi = xbox_index(nrow), nb_rows = bi == 2 ? kXN : 32 << bi;
      const int ab = i & 1;
      if (!__all_sync(0xffffffffu, wait(&S.acc_full[ab], (uint32_t)((i / 2) & 1)))) break;
      tc_fence_after();
      float* out = G.out + (size_t)row0 * G.out_ld + mb * kXM + feat;
      const uint32_t tq = tmem + (uint32_t)(ab * kXAccCols) + ((uint32_t)(quad * 32) << 16);
      for (int c0 = 0; c0 < nrow; c0 += 32) {
        uint32_t v[32], w[32];
        tmem_ld32(tq + (uint32_t)c0, v);
#pragma unroll
        for (int tt = 1; tt < NT; ++tt) {
          tmem_ld32(tq + (uint32_t)(tt * nb_rows + c0), w);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) v[jj] = __float_as_uint(__uint_as_float(v[jj]) + __uint_as_float(w[jj]));
        }
#pragma unroll
        for (int jj = 0; jj < 32; ++jj)
          if (c0 + jj < nrow) out[(size_t)(c0 + jj) * G.out_ld] = __uint_as_float(v[jj]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&S.acc_empty[ab]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_free(tmem, kXTmemCols);
  }
}

}  // namespace qk

namespace qk {

// ================================================================= host ==
bool gmx_eligible(const qk_weight& gate, const qk_weight& up, const qk_weight& down, int H, int I) {
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (gate.fmt != QK_FMT_MXFP4 || up.fmt != QK_FMT_MXFP4 || down.fmt != QK_FMT_MXFP4) return false;
  if (H % 512 != 0 || I % 512 != 0) return false;  // 16-byte scale chunks per row (4 stages of 128)
  return al(gate.q, 32) && al(up.q, 32) && al(down.q, 32) && al(gate.scales, 16) && al(up.scales, 16) &&
         al(down.scales, 16);
}

// Packed e2m1 rows [rows][K / 2]: 16 codes (8 bytes) per 16-byte slot in
// shared memory, boxes {128 codes, 128 rows}, 128-byte swizzle.  A box reads
// 64 bytes of each row; 256-byte L2 promotion brings the row's next three
// steps into L2 with the first.
static bool x_map_weights(CUtensorMap* m, const uint8_t* q, int64_t rows, int K) {
  const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)K / 2};
  const uint32_t box[2] = {(uint32_t)kXK, (uint32_t)kXM};
  return tmap_get(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// The NT term arrays [NT][P][K] e4m3 viewed as {128 (within a reduction
// step), P rows, NT terms, K / 128 steps}; box {128, n, NT, kpb}: per step the
// terms' n rows stacked (the MMA's B rows), 128-byte swizzle.
static bool x_map_terms(CUtensorMap (&m)[kXNBox], const uint8_t* q, int NT, int64_t P, int K) {
  const uint64_t dims[4] = {(uint64_t)kXK, (uint64_t)P, (uint64_t)NT, (uint64_t)K / kXK};
  const uint64_t strides[3] = {(uint64_t)K, (uint64_t)P * K, (uint64_t)kXK};
  for (int i = 0; i < kXNBox; ++i) {
    const uint32_t box[4] = {(uint32_t)kXK, (uint32_t)(i == 2 ? kXN : 32 << i), (uint32_t)NT, (uint32_t)xkpb(i)};
    if (!tmap_get(&m[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  }
  return true;
}

template <bool GATEUP, int NT>
static qk_status x_launch(const GmxArgs& A, cudaStream_t st) {
  auto kern = k_gmx<GATEUP, NT>;
  constexpr int smem = GmxCfg<NT>::kSmem;
  static_assert(sizeof(GmxHead) <= 256, "head");
  if (smem > max_smem_optin()) return QK_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return QK_ERR_CUDA;
  kern<<<num_sms(), kXThreads, smem, st>>>(A);
  return cudaGetLastError() == cudaSuccess ? QK_OK : QK_ERR_CUDA;
}

qk_status gmx_forward(const DecodeArgs& a, const GroupWs& W, cudaStream_t st) {
  const int T = a.T, k = a.k, E = a.E, H = a.H, I = a.I, P = a.P;
  const int F = P / kXN + E + 1;  // token tiles at most (the workspace holds this many)
  k_gmx_xsplit<<<T, kRowThreads, 0, st>>>(W, a.x, a.ids, k, E, H, P);
  if (cudaGetLastError() != cudaSuccess) return QK_ERR_CUDA;

  GmxArgs g1 = {};
  g1.W = W;
  g1.sf_a = a.gate.scales;
  g1.sf_b = a.up.scales;
  g1.sfb = W.sfx;
  g1.out = W.gu;
  g1.K = H;
  g1.rows_per_e = I;
  g1.MB = 2 * I / kXM;  // gate blocks, then up blocks
  g1.MBA = I / kXM;
  g1.out_ld = 2 * I;
  g1.F = F;
  if (!x_map_weights(&g1.ta, a.gate.q, (int64_t)E * I, H) || !x_map_weights(&g1.tb, a.up.q, (int64_t)E * I, H) ||
      !x_map_terms(g1.tx, W.xq, 2, P, H))
    return QK_ERR_CUDA;
  qk_status rc = x_launch<true, 2>(g1, st);
  if (rc != QK_OK) return rc;

  k_gmx_hsplit<<<P, kRowThreads, 0, st>>>(W, E, I, P);
  if (cudaGetLastError() != cudaSuccess) return QK_ERR_CUDA;

  GmxArgs g2 = {};
  g2.W = W;
  g2.sf_a = a.down.scales;
  g2.sf_b = a.down.scales;
  g2.sfb = W.sfh;
  g2.out = W.dperm;
  g2.K = I;
  g2.rows_per_e = H;
  g2.MB = H / kXM;
  g2.MBA = H / kXM;
  g2.out_ld = H;
  g2.F = F;
  if (!x_map_weights(&g2.ta, a.down.q, (int64_t)E * H, I) || !x_map_terms(g2.tx, W.hq, 3, P, I)) return QK_ERR_CUDA;
  g2.tb = g2.ta;
  return x_launch<false, 3>(g2, st);
}

}  // namespace qk
