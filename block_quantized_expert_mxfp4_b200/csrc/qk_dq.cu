// qk_dq.cu -- decode path (a few tokens) on the fp4 x fp4 block-scaled tensor
// cores: tcgen05.mma kind::mxf4 with the weights as the 128-row A operand.
//
// At decode sizes the expert projections are weight-streaming matrix-vector
// products ("DeepSeek-v4-Flash-REAP-K180-NVFP4", "Why this mix?": gate+up
// carry about 2/3 of the expert bytes), so the design goal is to keep HBM
// streaming packed e2m1 bytes with as few instructions per byte as possible:
//
//  * The packed e2m1 nibbles go from HBM to shared memory by TMA exactly as
//    stored (one 128-byte row segment = 256 elements of K per row, 128 rows
//    per step, 16 KB) and from there to the tensor core: no unpacking, no
//    register traffic.  The e8m0 scales (one per 32) go to tensor memory as
//    stored.
//  * The tensor core's other operand must be fp4 too (kind::mxf4 multiplies
//    e2m1 by e2m1).  Each activation row is therefore written as a sum of 8
//    e2m1 terms with their own e8m0 scale per 32 elements: term i has scale
//    2^X_i, X_i = floor(log2 max|r_i|) - 2 over the block (the OCP
//    Microscaling rule), and r_{i+1} = r_i - RN_e2m1(r_i / 2^X_i) 2^X_i.
//    Every residual is exact in fp32 and each term lowers the block's
//    largest residual by at least a factor 4, so 8 terms leave at most
//    2^-14 of the block maximum (bf16 x is reproduced exactly unless a block
//    spans more than about 2^14; fp32 h to about 2^-16 of its block maximum).
//    The terms are the N dimension of the MMA (8 columns per pair), which is
//    nearly free: the instruction's cost is set by its 128 weight rows.
//  * One step = 128 weight rows x 256 elements of K = 4 MMAs (K = 64 each),
//    two weight-scale atom copies and one commit; its own accumulator (up to
//    64 TMEM columns, 7 in flight), so the epilogue never stalls the MMAs.
//
//   k_dq<gate/up>  steps ordered (virtual expert, K block, row block) so a
//                  CTA's consecutive steps share one activation image (x
//                  terms of the pairs for one K block), built by the CTA
//                  itself; each step's fp32 result per pair goes to
//                  p1[pair][row block][K block][128].
//   k_dq<down>     (programmatic dependent launch) steps ordered (virtual
//                  expert, K block, output row block).  Its weight copies
//                  start before the gate/up kernel has finished; the h image
//                  of each (virtual expert, K block) -- h = silu(gate) * up
//                  summed from p1 in K-block order, split into 8 terms -- is
//                  built once, by the first CTA of each builder warp's share
//                  to claim it, and copied by the others.  Each step's result
//                  goes to p2; the last warp to finish an output row block
//                  (a counter) forms y for those rows in slot order
//                  (deterministic).
//
// Units are split evenly and contiguously over one CTA per SM (a deep weight
// ring: 11 stages, 176 KB in flight per SM).  Warp roles (12 warps): 0 weight
// TMA, 1 MMA issuer, 2 weight-scale atoms, 4-7 epilogue (TMEM lane quarters),
// 8-11 activation images.  Every wait is bounded.
#include <cuda.h>

#include "qk_common.cuh"
#include "qk_route_table.cuh"
#include "qk_tmap.h"

namespace qk {

constexpr int kQRows = 128;                 // weight rows per step (MMA M)
constexpr int kQK = 256;                    // elements of K per step
constexpr int kQStage = kQRows * kQK / 2;   // 16 KB of packed e2m1
constexpr int kQTerms = 8;                  // e2m1 terms per activation row
constexpr int kQBRows = kTileN * kQTerms;   // 64 B rows at most (8 pairs x 8 terms)
constexpr int kQImg = kQBRows * 128 + 2 * 512;  // one activation image: rows + two scale atoms
constexpr int kQAcc = 7;                    // accumulators of 64 columns in flight
constexpr int kQTSfa = 448, kQTSfb = 456;   // TMEM columns of the scale atoms
constexpr int kQWarps = 12;
constexpr int kQThreads = kQWarps * 32;
constexpr int kQMaxStages = 12;
constexpr int kQClaimParts = 4;             // builder warps: one claim per warp's share of an image
constexpr int kQSfAhead = 4;                // steps of weight scales loaded ahead
constexpr int kMaxTopK = 8;

struct DqArgs {
  qk_weight A, B;        // gate/up kernel: gate, up; down kernel: down, down
  const uint16_t* x;     // bf16 [T][H]
  const int32_t* ids;    // [T][k]
  const float* w;        // [T][k]
  void* y;               // [T][H] fp32 or bf16
  float* p1;             // [P][2I/128][H/256][128] gate/up results per step
  float* p2;             // [P][H/128][I/256][128] down results per step
  uint8_t* himg;         // [kMaxPairs][I/256][kQImg] h images (global copies)
  uint32_t* claim;       // [kMaxPairs][I/256][4]: 0 free, 1 building, 2 ready
  float* pds;            // [P][H/128][128] down results of each pair summed over K blocks
  uint32_t* cnt1;        // [kMaxPairs][H/128] epilogue warps finished per (virtual expert, output row block)
  uint32_t* cnt;         // [H/128] virtual experts finished per output row block
  int T, k, E, H, I, P, y_bf16, stages;
  alignas(64) CUtensorMap ta, tb;  // packed rows as bytes [E*rows][K/2], box {128 B, 128 rows}, 128B swizzle
};

struct DqHead {
  alignas(8) uint64_t wfull[kQMaxStages];
  alignas(8) uint64_t wempty[kQMaxStages];  // MMAs of the stage done: weights and scale atoms free
  alignas(8) uint64_t sfull[kQMaxStages];   // the stage's weight-scale atoms written
  alignas(8) uint64_t bfull[2];             // activation image slot built (4 builder warps)
  alignas(8) uint64_t bempty[2];
  alignas(8) uint64_t afull[kQAcc];         // accumulator holds a finished step
  alignas(8) uint64_t aempty[kQAcc];        // the 4 epilogue warps have read it
  alignas(8) uint64_t drained;
  uint32_t tmem;
  int abort;
};

// Dynamic shared memory: 1 KB alignment slack, weight stages, two image
// slots, scale atoms per stage, routing table, barriers.
__host__ __device__ constexpr int dq_smem_bytes(int stages) {
  return 1024 + stages * kQStage + 2 * kQImg + stages * 1024 + (((int)sizeof(Route) + 15) & ~15) +
         (((int)sizeof(DqHead) + 15) & ~15);
}

__host__ __device__ constexpr uint32_t dq_idesc_mxf4(int N) {
  // A, B e2m1 (format 1), K-major, ue8m0 scales (bit 23), M = 128, N.
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void umma_mxf4(uint32_t tmem_d, uint64_t desc_a, uint64_t desc_b, uint32_t idesc,
                                          uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(
          tmem_d),
      "l"(desc_a), "l"(desc_b), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb));
}

// 32 lanes x 16 consecutive 32-bit TMEM columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
  uint32_t u[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15}, [%16];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) r[i] = __uint_as_float(u[i]);
}

// e2m1 code of v (round to nearest even, saturating at 6) and its value.
__device__ __forceinline__ uint32_t e2m1_rn(float v, float& back) {
  uint16_t b;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n mov.b16 %0, {t, 0};\n}\n"
      : "=h"(b)
      : "f"(0.0f), "f"(v));
  const uint32_t c = b & 0xFu;
  const uint32_t h2 = e2m1x2_to_f16x2<0>(c);
  back = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
  return c;
}

// One e2m1 term of the 32-element block a warp holds (element = lane): the
// block's e8m0 scale code c = X + 127 (X = floor(log2 max|v|) - 2, clamped at
// code 0) and this lane's 4-bit code; v becomes the exact residual.
__device__ __forceinline__ int dq_term(float& v, uint32_t& code) {
  float m = fabsf(v);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int e = (int)((__float_as_uint(m) >> 23) & 0xFFu);
  const int c = e > 2 ? e - 2 : 0;  // <= 253
  const float up = __uint_as_float((uint32_t)(254 - c) << 23);                          // 2^-X
  const float dn = c ? __uint_as_float((uint32_t)c << 23) : __uint_as_float(0x00400000u);  // 2^X
  float back;
  code = e2m1_rn(v * up, back);
  v = fmaf(-back, dn, v);  // exact: back * 2^X is within a factor 2 of v, or 0
  return c;
}

// Writes the 8 terms of the warp's 32-element block (value v of this lane)
// into image rows 8 j + t, 16-byte chunk blk (128-byte swizzle), and the
// scale bytes into the image's two atoms.  img: smem or global image base.
__device__ __forceinline__ void dq_put_terms(float v, int j, int blk, uint8_t* img, uint8_t* img2) {
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int t = 0; t < kQTerms; ++t) {
    uint32_t code;
    const int c = dq_term(v, code);
    uint32_t wd = code << (4 * (lane & 7));
    wd |= __shfl_xor_sync(0xffffffffu, wd, 1);
    wd |= __shfl_xor_sync(0xffffffffu, wd, 2);
    wd |= __shfl_xor_sync(0xffffffffu, wd, 4);
    const int r = kQTerms * j + t;
    const int off = r * 128 + ((blk ^ (r & 7)) << 4) + 4 * (lane >> 3);
    const int soff = kQBRows * 128 + (blk >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (blk & 3);
    if ((lane & 7) == 0) {
      *reinterpret_cast<uint32_t*>(img + off) = wd;
      if (img2) *reinterpret_cast<uint32_t*>(img2 + off) = wd;
    }
    if (lane == 0) {
      img[soff] = (uint8_t)c;
      if (img2) img2[soff] = (uint8_t)c;
    }
  }
}

// Scale bytes of the (absent) pair j of an image: code 0, so the stale rows
// behind them contribute nothing measurable to columns nobody reads.
__device__ __forceinline__ void dq_zero_scales(int j, int blk, uint8_t* img, uint8_t* img2) {
  const int lane = threadIdx.x & 31;
  if (lane < kQTerms) {
    const int r = kQTerms * j + lane;
    const int soff = kQBRows * 128 + (blk >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (blk & 3);
    img[soff] = 0;
    if (img2) img2[soff] = 0;
  }
}

template <bool GATEUP>
__global__ void __launch_bounds__(kQThreads, 1) k_dq(const __grid_constant__ DqArgs G) {
  extern __shared__ __align__(16) uint8_t smem_raw[];  // rounded up to 1024 below, at run time
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int S = G.stages;
  uint8_t* sW = base;                       // S x 16 KB
  uint8_t* sB = sW + S * kQStage;           // 2 x kQImg (1024-aligned)
  uint8_t* sSa = sB + 2 * kQImg;            // S x 1 KB: two weight-scale atoms per stage
  Route& R = *reinterpret_cast<Route*>(sSa + S * 1024);
  DqHead& H = *reinterpret_cast<DqHead*>(reinterpret_cast<uint8_t*>(&R) + ((sizeof(Route) + 15) & ~(size_t)15));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned long long limit = g_wait_limit_ns;
  const int K = GATEUP ? G.H : G.I;
  const int KB = K / kQK;                              // K blocks
  const int NB = GATEUP ? 2 * G.I / kQRows : G.H / kQRows;  // row blocks per virtual expert
  const int KB2 = G.I / kQK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&H.wfull[s], 1);
      mbar_init(&H.wempty[s], 1);
      mbar_init(&H.sfull[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&H.bfull[s], 4);
      mbar_init(&H.bempty[s], 1);
    }
    for (int a = 0; a < kQAcc; ++a) {
      mbar_init(&H.afull[a], 1);
      mbar_init(&H.aempty[a], 4);
    }
    mbar_init(&H.drained, 1);
    H.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&H.tmem, 512);
  if (GATEUP) {
    pdl_wait();  // the ids may come from the kernel launched just before (router)
    if (blockIdx.x == 0) {  // the down kernel's claims and counters (it reads them after this kernel completes)
      const int nc = kMaxPairs * KB2 * kQClaimParts;
      for (int i = threadIdx.x; i < nc; i += blockDim.x) G.claim[i] = 0u;
      for (int i = threadIdx.x; i < kMaxPairs * (G.H / kQRows); i += blockDim.x) G.cnt1[i] = 0u;
      for (int i = threadIdx.x; i < G.H / kQRows; i += blockDim.x) G.cnt[i] = 0u;
    }
  }
  build_route(G.ids, G.P, G.E, R);  // ends with __syncthreads
  if (GATEUP) pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = H.tmem;
  const int U = R.n_v * KB * NB;
  if (!GATEUP && U == 0 && blockIdx.x == 0)  // every id invalid: no step writes y
    for (int i = threadIdx.x; i < G.T * G.H; i += blockDim.x) {
      if (G.y_bf16)
        reinterpret_cast<__nv_bfloat16*>(G.y)[i] = __float2bfloat16_rn(0.f);
      else
        reinterpret_cast<float*>(G.y)[i] = 0.f;
    }
  const int u0 = (int)((long long)blockIdx.x * U / gridDim.x), u1 = (int)((long long)(blockIdx.x + 1) * U / gridDim.x);
  auto step = [&](int u, int& v, int& kb, int& rb) {
    rb = u % NB;
    const int t = u / NB;
    kb = t % KB;
    v = t / KB;
  };
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(&H.abort)) return false;
    if (mbar_wait_bounded(bar, parity, limit)) return true;
    set_status(QK_ERR_TIMEOUT);
    *reinterpret_cast<volatile int*>(&H.abort) = 1;
    return false;
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile int*>(&H.abort) != 0; };
  // First global row of a step's weight rows, its tensor map and scale rows.
  auto wrow = [&](int v, int rb, const void*& map, const uint8_t*& sc) {
    const int e = R.v_expert[v];
    if (GATEUP && rb >= NB / 2) {
      map = &G.tb;
      sc = G.B.scales;
      return e * G.I + (rb - NB / 2) * kQRows;
    }
    map = &G.ta;
    sc = G.A.scales;
    return e * (GATEUP ? G.I : G.H) + rb * kQRows;
  };
  auto npad = [&](int v) { return max(16, (kQTerms * R.v_n[v] + 15) & ~15); };

  if (warp == 0) {
    // ------------------------------------------------------------ weights --
    if (lane == 0) {
      const uint64_t pw = policy_evict_first();
      int q = 0;
      for (int u = u0; u < u1 && !aborted(); ++u, ++q) {
        int v, kb, rb;
        step(u, v, kb, rb);
        const void* m;
        const uint8_t* sc;
        const int y = wrow(v, rb, m, sc);
        const int s = q % S;
        if (q >= S && !wait(&H.wempty[s], (uint32_t)((q / S - 1) & 1))) break;
        mbar_arrive_expect_tx(&H.wfull[s], (uint32_t)kQStage);
        tma_load_2d(sW + s * kQStage, m, kb * (kQK / 2), y, &H.wfull[s], pw);
      }
      for (int r = q > S ? q - S : 0; r < q; ++r)  // nothing may still be landing at exit
        if (!mbar_wait_bounded(&H.wfull[r % S], (uint32_t)((r / S) & 1), kDrainLimitNs)) break;
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------------------------------------- weight-scale atoms --
    // Per step: 8 bytes (8 blocks of 32) of each of the 128 rows, 4 rows per
    // lane, loaded one step ahead; atom 0 = blocks 0-3, atom 1 = blocks 4-7.
    const int srow = K / 32;
    auto load = [&](int u, uint2 (&r)[4]) {
      int v, kb, rb;
      step(u, v, kb, rb);
      const void* m;
      const uint8_t* sc;
      const int r0 = wrow(v, rb, m, sc);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        r[j] = __ldg(reinterpret_cast<const uint2*>(sc + (size_t)(r0 + 32 * j + lane) * srow + kb * 8));
    };
    // A ring of kQSfAhead steps of scale rows in registers (static indices):
    // the loads for step n + kQSfAhead go out as step n is written.
    uint2 ring[kQSfAhead][4];
#pragma unroll
    for (int i = 0; i < kQSfAhead; ++i)
      if (u0 + i < u1) load(u0 + i, ring[i]);
    const int cnt_steps = u1 - u0;
    bool ok = true;
    for (int n0 = 0; n0 < cnt_steps && ok; n0 += kQSfAhead) {
#pragma unroll
      for (int i = 0; i < kQSfAhead; ++i) {
        const int n = n0 + i;
        if (n >= cnt_steps) break;
        uint32_t ff = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) ff |= __vcmpeq4(ring[i][j].x, 0xFFFFFFFFu) | __vcmpeq4(ring[i][j].y, 0xFFFFFFFFu);
        if (ff) set_status(QK_ERR_NAN_SCALE);
        const int s = n % S;
        if (n >= S && !__all_sync(0xffffffffu, wait(&H.wempty[s], (uint32_t)((n / S - 1) & 1)))) {
          ok = false;
          break;
        }
        uint8_t* d = sSa + s * 1024 + lane * 16;
        *reinterpret_cast<uint4*>(d) = make_uint4(ring[i][0].x, ring[i][1].x, ring[i][2].x, ring[i][3].x);
        *reinterpret_cast<uint4*>(d + 512) = make_uint4(ring[i][0].y, ring[i][1].y, ring[i][2].y, ring[i][3].y);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_one(&H.sfull[s]);
        if (n + kQSfAhead < cnt_steps) load(u0 + n + kQSfAhead, ring[i]);
      }
    }
  } else if (warp >= 8) {
    // -------------------------------------------------- activation images --
    // Image of (virtual expert, K block): rows 8 j + t = term t of pair j, one
    // 16-byte chunk per 32-element block.  Task (j, blk) belongs to builder
    // warp (8 j + blk) % 4.
    const int bw = warp - 8;
    if (!GATEUP) pdl_wait();  // the gate/up results
    int img = -1, pv = -1, pkb = -1;
    for (int u = u0; u < u1; ++u) {
      int v, kb, rb;
      step(u, v, kb, rb);
      if (v == pv && kb == pkb) continue;
      pv = v;
      pkb = kb;
      ++img;
      const int b = img & 1;
      if (img >= 2 && !__all_sync(0xffffffffu, wait(&H.bempty[b], (uint32_t)((img / 2 - 1) & 1)))) break;
      uint8_t* dst = sB + b * kQImg;
      const int np = R.v_n[v], p0 = R.v_p0[v];
      if (GATEUP) {
        for (int task = bw; task < kTileN * 8; task += 4) {
          const int j = task >> 3, blk = task & 7;
          if (j >= np) {
            dq_zero_scales(j, blk, dst, nullptr);
            continue;
          }
          const int tok = R.pair_list[p0 + j] / G.k;
          const float xv = bf16_bits_to_f32(G.x[(size_t)tok * G.H + kb * kQK + blk * 32 + lane]);
          if (!finite_bits(xv)) set_status(QK_ERR_NONFINITE);
          dq_put_terms(xv, j, blk, dst, nullptr);
        }
      } else {
        // Claim this warp's share of the h image, or wait for it and copy it.
        uint8_t* gimg = G.himg + ((size_t)v * KB2 + kb) * kQImg;
        uint32_t* cl = G.claim + ((size_t)v * KB2 + kb) * kQClaimParts + bw;
        uint32_t won = 0;
        if (lane == 0) won = atomicCAS(cl, 0u, 1u) == 0u;
        won = __shfl_sync(0xffffffffu, won, 0);
        if (won) {
          const int NB1 = 2 * G.I / kQRows, KB1 = G.H / kQK;
          for (int task = bw; task < kTileN * 8; task += 4) {
            const int j = task >> 3, blk = task & 7;
            if (j >= np) {
              dq_zero_scales(j, blk, dst, gimg);
              continue;
            }
            const int i = kb * kQK + blk * 32 + lane;  // element of h
            const float* pg = G.p1 + (((size_t)(p0 + j) * NB1 + (i >> 7)) * KB1) * kQRows + (i & 127);
            const float* pu = G.p1 + (((size_t)(p0 + j) * NB1 + NB1 / 2 + (i >> 7)) * KB1) * kQRows + (i & 127);
            float g = 0.f, uu = 0.f;
            for (int c0 = 0; c0 < KB1; c0 += 16) {  // 16 K blocks of loads in flight, added in order
              float ga[16], ua[16];
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const bool in = c0 + c < KB1;
                ga[c] = in ? __ldcg(pg + (size_t)(c0 + c) * kQRows) : 0.f;
                ua[c] = in ? __ldcg(pu + (size_t)(c0 + c) * kQRows) : 0.f;
              }
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                g += ga[c];
                uu += ua[c];
              }
            }
            const float h = __fdividef(g, 1.0f + __expf(-g)) * uu;
            if (!finite_bits(h)) set_status(QK_ERR_NONFINITE);
            dq_put_terms(h, j, blk, dst, gimg);
          }
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicExch(cl, 2u);
        } else {
          bool ok = true;
          if (lane == 0) {
            const unsigned long long t0 = globaltimer();
            while (atomicAdd(cl, 0u) != 2u) {
              if (globaltimer() - t0 >= limit || aborted()) {
                ok = false;
                break;
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
          if (!ok) {
            set_status(QK_ERR_TIMEOUT);
            *reinterpret_cast<volatile int*>(&H.abort) = 1;
            break;
          }
          __threadfence();
          for (int task = bw; task < kTileN * 8; task += 4) {
            const int j = task >> 3, blk = task & 7;
            if (j >= np) {
              dq_zero_scales(j, blk, dst, nullptr);
              continue;
            }
            const int r = kQTerms * j + (lane >> 2);
            const int off = r * 128 + ((blk ^ (r & 7)) << 4) + 4 * (lane & 3);
            *reinterpret_cast<uint32_t*>(dst + off) = __ldcg(reinterpret_cast<const uint32_t*>(gimg + off));
            if (lane < kQTerms) {
              const int rr = kQTerms * j + lane;
              const int soff = kQBRows * 128 + (blk >> 2) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (blk & 3);
              dst[soff] = *reinterpret_cast<const volatile uint8_t*>(gimg + soff);
            }
          }
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&H.bfull[b]);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t t_sfa = tmem + kQTSfa, t_sfb = tmem + kQTSfb;
      int img = -1, pv = -1, pkb = -1, n = 0;
      for (int u = u0; u < u1 && !aborted(); ++u, ++n) {
        int v, kb, rb;
        step(u, v, kb, rb);
        const int N = npad(v);
        if (v != pv || kb != pkb) {
          pv = v;
          pkb = kb;
          if (img >= 0) umma_commit(&H.bempty[img & 1]);  // the previous image's MMAs done
          ++img;
          if (!wait(&H.bfull[img & 1], (uint32_t)((img / 2) & 1))) break;
          tc_fence_after();
          const uint8_t* sb = sB + (img & 1) * kQImg + kQBRows * 128;
          utccp_32x128b_x4(t_sfb, umma_desc_sf(sb));
          utccp_32x128b_x4(t_sfb + 4, umma_desc_sf(sb + 512));
        }
        const int a = n % kQAcc, s = n % S;
        if (n >= kQAcc && !wait(&H.aempty[a], (uint32_t)((n / kQAcc - 1) & 1))) break;
        if (!wait(&H.wfull[s], (uint32_t)((n / S) & 1)) || !wait(&H.sfull[s], (uint32_t)((n / S) & 1))) break;
        tc_fence_after();
        utccp_32x128b_x4(t_sfa, umma_desc_sf(sSa + s * 1024));
        utccp_32x128b_x4(t_sfa + 4, umma_desc_sf(sSa + s * 1024 + 512));
        const uint64_t da = umma_desc_k_sw128(sW + s * kQStage);
        const uint64_t db = umma_desc_k_sw128(sB + (img & 1) * kQImg);
        const uint32_t id = dq_idesc_mxf4(N);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t sid = (uint32_t)(k & 1) * 2;
          umma_mxf4(tmem + (uint32_t)(a * 64), da + 2 * k, db + 2 * k, umma_idesc_sf_ids(id, (int)sid, (int)sid),
                    (t_sfa + 4 * (k >> 1)) | (sid << 30), (t_sfb + 4 * (k >> 1)) | (sid << 30), k > 0 ? 1u : 0u);
        }
        umma_commit(&H.wempty[s]);
        umma_commit(&H.afull[a]);
      }
      umma_commit(&H.drained);  // every MMA issued here completes before the accumulators are freed
      mbar_wait_bounded(&H.drained, 0, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ----------------------------------------------------------- epilogue --
    // Thread = weight row 32 ew + lane; columns 8 j .. 8 j + 7 = pair j's
    // terms, added here.
    const int ew = warp - 4;
    const int row = 32 * ew + lane;
    const uint32_t lane_base = (uint32_t)(32 * ew) << 16;
    float* part = GATEUP ? G.p1 : G.p2;
    int n = 0;
    for (int u = u0; u < u1; ++u, ++n) {
      int v, kb, rb;
      step(u, v, kb, rb);
      const int np = R.v_n[v], p0 = R.v_p0[v], N = npad(v);
      const int a = n % kQAcc;
      if (!__all_sync(0xffffffffu, wait(&H.afull[a], (uint32_t)((n / kQAcc) & 1)))) break;
      tc_fence_after();
      float sum[kTileN];
#pragma unroll
      for (int j = 0; j < kTileN; ++j) sum[j] = 0.f;
#pragma unroll
      for (int g = 0; g < kQBRows / 16; ++g) {
        if (16 * g < N) {
          float r[16];
          tmem_ld16(tmem + lane_base + (uint32_t)(a * 64 + 16 * g), r);
#pragma unroll
          for (int t = 0; t < kQTerms; ++t) {
            sum[2 * g] += r[t];
            sum[2 * g + 1] += r[kQTerms + t];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&H.aempty[a]);
      for (int j = 0; j < np; ++j) part[(((size_t)(p0 + j) * NB + rb) * KB + kb) * kQRows + row] = sum[j];
      if (!GATEUP) {
        // Level 1: the last of the 4 x KB epilogue warps of (virtual expert v,
        // output row block rb) adds each of v's pairs' K-block results in
        // order; level 2: the last virtual expert of rb forms y for those rows
        // (slots in order).  Both orders are fixed: deterministic bytes.
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(&G.cnt1[v * NB + rb], 1u) == (unsigned)(4 * KB - 1);
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          for (int j = 0; j < np; ++j) {
            const float4* src = reinterpret_cast<const float4*>(G.p2 + ((size_t)(p0 + j) * NB + rb) * KB * kQRows) + lane;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int c0 = 0; c0 < KB; c0 += 8) {
              float4 d[8];
#pragma unroll
              for (int c = 0; c < 8; ++c)
                d[c] = c0 + c < KB ? __ldcg(src + (size_t)(c0 + c) * (kQRows / 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                acc.x += d[c].x;
                acc.y += d[c].y;
                acc.z += d[c].z;
                acc.w += d[c].w;
              }
            }
            reinterpret_cast<float4*>(G.pds + ((size_t)(p0 + j) * NB + rb) * kQRows)[lane] = acc;
          }
          __threadfence();
          __syncwarp();
          int last2 = 0;
          if (lane == 0) last2 = atomicAdd(&G.cnt[rb], 1u) == (unsigned)(R.n_v - 1);
          last2 = __shfl_sync(0xffffffffu, last2, 0);
          if (last2) {
            __threadfence();
            for (int t = 0; t < G.T; ++t) {
              float4 d[kMaxTopK];
              float wt[kMaxTopK];
#pragma unroll
              for (int s2 = 0; s2 < kMaxTopK; ++s2) {
                d[s2] = make_float4(0.f, 0.f, 0.f, 0.f);
                wt[s2] = 0.f;
                if (s2 < G.k) {
                  const int p = t * G.k + s2, pvv = R.pair_v[p];
                  if (pvv >= 0) {
                    const int sp = R.v_p0[pvv] + R.pair_j[p];
                    d[s2] = __ldcg(reinterpret_cast<const float4*>(G.pds + ((size_t)sp * NB + rb) * kQRows) + lane);
                    wt[s2] = G.w[p];
                  }
                }
              }
              float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int s2 = 0; s2 < kMaxTopK; ++s2) {
                acc[0] = fmaf(wt[s2], d[s2].x, acc[0]);
                acc[1] = fmaf(wt[s2], d[s2].y, acc[1]);
                acc[2] = fmaf(wt[s2], d[s2].z, acc[2]);
                acc[3] = fmaf(wt[s2], d[s2].w, acc[3]);
              }
              if (!(finite_bits(acc[0]) && finite_bits(acc[1]) && finite_bits(acc[2]) && finite_bits(acc[3])))
                set_status(QK_ERR_NONFINITE);
              const size_t o = (size_t)t * G.H + rb * kQRows + lane * 4;
              if (G.y_bf16) {
                __nv_bfloat16* yb = reinterpret_cast<__nv_bfloat16*>(G.y) + o;
#pragma unroll
                for (int q = 0; q < 4; ++q) yb[q] = __float2bfloat16_rn(acc[q]);
              } else {
                *reinterpret_cast<float4*>(reinterpret_cast<float*>(G.y) + o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
              }
            }
          }
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_free(tmem, 512);
  }
}

// ================================================================= host ==
bool dq_eligible(const qk_weight& gate, const qk_weight& up, const qk_weight& down, int H, int I) {
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (gate.fmt != QK_FMT_MXFP4 || up.fmt != QK_FMT_MXFP4 || down.fmt != QK_FMT_MXFP4) return false;
  if (H % kQK != 0 || I % kQK != 0) return false;
  return al(gate.q, 16) && al(up.q, 16) && al(down.q, 16) && al(gate.scales, 8) && al(up.scales, 8) &&
         al(down.scales, 8);
}

struct DqWs {
  size_t p1, p2, pds, himg, claim, cnt1, cnt, total;
};
static DqWs dq_layout(int T, int k, int H, int I) {
  const size_t P = (size_t)T * k;
  DqWs L;
  size_t o = 0;
  L.p1 = o; o += align256(P * (2 * I / kQRows) * (H / kQK) * kQRows * 4);
  L.p2 = o; o += align256(P * (H / kQRows) * (I / kQK) * kQRows * 4);
  L.pds = o; o += align256(P * (H / kQRows) * kQRows * 4);
  L.himg = o; o += align256(P * (I / kQK) * (size_t)kQImg);
  L.claim = o; o += align256((size_t)kMaxPairs * (I / kQK) * kQClaimParts * 4);
  L.cnt1 = o; o += align256((size_t)kMaxPairs * (H / kQRows) * 4);
  L.cnt = o; o += align256((size_t)(H / kQRows) * 4);
  L.total = o;
  return L;
}
size_t dq_workspace_bytes(int T, int k, int H, int I) { return dq_layout(T, k, H, I).total; }

static bool dq_map(CUtensorMap* m, const uint8_t* q, int64_t rows, int K) {
  const uint64_t dims[2] = {(uint64_t)K / 2, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)K / 2};
  const uint32_t box[2] = {(uint32_t)(kQK / 2), (uint32_t)kQRows};
  return tmap_get(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

qk_status dq_forward(const DecodeArgs& a, void* workspace, cudaStream_t st) {
  const DqWs L = dq_layout(a.T, a.k, a.H, a.I);
  uint8_t* p = static_cast<uint8_t*>(workspace);
  DqArgs g = {};
  g.x = a.x;
  g.ids = a.ids;
  g.w = a.w;
  g.y = a.y;
  g.p1 = reinterpret_cast<float*>(p + L.p1);
  g.p2 = reinterpret_cast<float*>(p + L.p2);
  g.himg = p + L.himg;
  g.claim = reinterpret_cast<uint32_t*>(p + L.claim);
  g.pds = reinterpret_cast<float*>(p + L.pds);
  g.cnt1 = reinterpret_cast<uint32_t*>(p + L.cnt1);
  g.cnt = reinterpret_cast<uint32_t*>(p + L.cnt);
  g.T = a.T;
  g.k = a.k;
  g.E = a.E;
  g.H = a.H;
  g.I = a.I;
  g.P = a.P;
  g.y_bf16 = a.y_bf16;
  const int optin = max_smem_optin();
  int stages = kQMaxStages;
  while (stages > 2 && dq_smem_bytes(stages) > optin) --stages;
  if (dq_smem_bytes(stages) > optin) return QK_ERR_UNSUPPORTED;
  g.stages = stages;
  const size_t smem = (size_t)dq_smem_bytes(stages);
  const int sms = num_sms();
  g.A = a.gate;
  g.B = a.up;
  if (!dq_map(&g.ta, a.gate.q, (int64_t)a.E * a.I, a.H) || !dq_map(&g.tb, a.up.q, (int64_t)a.E * a.I, a.H))
    return QK_ERR_CUDA;
  // Steps: at most P virtual experts; one CTA per SM, no more CTAs than steps.
  const int u1max = a.P * (a.H / kQK) * (2 * a.I / kQRows);
  qk_status rc = launch_ex(k_dq<true>, dim3(std::max(1, std::min(sms, u1max))), dim3(kQThreads), smem, st, true, g);
  if (rc != QK_OK) return rc;
  g.A = a.down;
  g.B = a.down;
  if (!dq_map(&g.ta, a.down.q, (int64_t)a.E * a.H, a.I)) return QK_ERR_CUDA;
  g.tb = g.ta;
  const int u2max = a.P * (a.I / kQK) * (a.H / kQRows);
  return launch_ex(k_dq<false>, dim3(std::max(1, std::min(sms, u2max))), dim3(kQThreads), smem, st, true, g);
}

}  // namespace qk
