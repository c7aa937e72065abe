// qk_gmx.cu -- MXFP4 grouped path on the block-scaled tensor cores.
//
// The pages store MXFP4 experts as e2m1 codes with one e8m0 scale per 32
// weights ("DeepSeek-v4-Flash-REAP-K180-NVFP4", "NVFP4: lossless MXFP4->NVFP4
// conversion") and run the expert projections as one grouped GEMM per
// projection ("DeepSeekv4 Flash for 1x Spark [REAP25]", "What's actually
// different").  sm_100a multiplies that format directly: tcgen05.mma
// kind::mxf8f6f4.block_scale takes e4m3 A and e2m1 B, each with a ue8m0 scale
// per 32 elements of K, and accumulates in fp32.  The weights go from HBM to
// the tensor core unchanged (TMA expands each 8-byte group of 16 codes into
// the 16-byte slot the tensor core reads); nothing is dequantized in
// registers.
//
// Activations are bf16 (and h is fp32), so each is written as a sum of e4m3
// terms with per-32 scales:  v = t0 2^(c0-127) + t1 2^(c1-127) [+ t2 ...],
// t_i = RN_e4m3(residual / 2^(c_i-127)), c_i chosen so the block's largest
// residual maps into [128, 256).  A bf16 value has 8 significant bits and
// each e4m3 term takes 4, and the first residual of a bf16 value needs at most
// 4 bits, so two terms reproduce x exactly (except for values within the e4m3
// subnormal range of their block, below 2^-13 of its largest element).  h is
// fp32: three terms keep its relative error below 2^-12.
//
// Orientation: A (M = 128 TMEM lanes) holds a token tile's terms, B (N = 256)
// 256 weight rows.  Lane 32 q + n_t t + i carries term t of token n_t q + i
// (n_t = 16 tokens per lane quadrant for x with 2 terms, 10 for h with 3), so
// the epilogue sums a token's terms with shuffles inside one warp.  Each MMA
// instruction covers 256 weight rows x 32 elements of K.
//
// Activation-quantized modes (QK_ACT_E4M3, QK_ACT_MXFP4: one quantized term
// per token, qk_actq.cuh) use the one-term geometry: lane m of A is token m,
// 128 tokens per tile, no shuffles in the epilogue.  In QK_ACT_MXFP4 the token
// blocks hold packed e2m1 (256 elements of K per 128-byte row, a plain byte
// tensor map for the weights too) and each instruction is kind::mxf4
// .block_scale.block32 over 64 elements of K, both operands fp4 as stored.
// The pages' own W8A8/W4A8 kernels keep the activations in 8 bits; fp4 x fp4
// at 4 x the bf16 rate is what sm_100a adds.  A third mode keeps the weights
// in e4m3 (kind::mxf8f6f4 with e4m3 on both sides, 128-block scales expanded
// to per-32 codes): the FP8 shared expert at large M.
//
//   k_gmx_xsplit  per token: x -> 2 e4m3 terms (1 term, or packed e2m1, in
//                 the quantized modes), written into the tile blocks of each
//                 of its pairs (gate/up tiles of 64 tokens, 128 quantized).
//   k_gmx<gate/up>  per (expert, 128 gate rows + the same 128 up rows, token
//                 tile): the epilogue forms h = silu(gate) * up and writes
//                 its 3 e4m3 terms into the down tile blocks (40 tokens per
//                 tile; 1 term or packed e2m1 and 128 tokens in the quantized
//                 modes).  NVFP4 layers in the fp4 mode instead write gate and
//                 up (fp32) to gu, and
//   k_gmx_hsplit  per sorted row forms and splits h (its scales anchor at the
//                 row's largest, known once the whole row is in).
//   k_gmx<down>   per (expert, 256 down rows, token tile): d (fp32).
//
// Token block (one reduction step of a tile, the MMA's A operand as it sits
// in shared memory): 128 rows x 128 bytes, 128-byte swizzle (16-byte chunk c
// of row m at m * 128 + ((c ^ (m % 8)) * 16)).  Scale-factor atom (the layout
// tcgen05.cp 32x128b.warpx4 copies into tensor memory): 512 bytes for 128
// rows x 4 blocks of 32 along K; row r, block b at byte
// (r % 32) * 16 + (r / 32) * 4 + b.
#include <cuda.h>
#include <cuda_fp8.h>

#include "qk_actq.cuh"
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

// Write one 32-element block (32 codes, block b of the row) of term t of
// tile row j into the tile's step block, and its scale code into the atom.
// npq: tokens per lane quadrant.
__device__ __forceinline__ void put_term(uint8_t* blocks, uint8_t* atoms, int f, int ns, int npq, int j, int t,
                                         int b, const uint32_t (&q)[8], int c) {
  const int m = 32 * (j / npq) + npq * t + j % npq;  // A row (TMEM lane)
  const int step = b >> 2, kb = b & 3;
  uint8_t* row = blocks + ((size_t)f * ns + step) * kXBlock + m * kXK;
  const int c0 = 2 * kb;  // the block's two 16-byte chunks within the 128-byte row
  *reinterpret_cast<uint4*>(row + ((c0 ^ (m & 7)) << 4)) = make_uint4(q[0], q[1], q[2], q[3]);
  *reinterpret_cast<uint4*>(row + (((c0 + 1) ^ (m & 7)) << 4)) = make_uint4(q[4], q[5], q[6], q[7]);
  atoms[((size_t)f * ns + step) * kSfAtom + (m & 31) * 16 + (m >> 5) * 4 + kb] = (uint8_t)c;
}

// Packed e2m1 (the fp4 x fp4 tiles of QK_ACT_MXFP4): one reduction step is
// 256 elements, a 128-byte row of eight 16-byte chunks, one per 32-block
// (chunk b % 8 of row j, swizzled), and two scale atoms (blocks 0-3 and 4-7
// of the step).  Row j = token j of the 128-token tile.
__device__ __forceinline__ void put_fp4(uint8_t* blocks, uint8_t* atoms, int f, int ns4, int j, int b,
                                        const uint32_t (&q)[4], int c) {
  const int step = b >> 3, c8 = b & 7;
  uint8_t* row = blocks + ((size_t)f * ns4 + step) * kXBlock + j * kXK;
  *reinterpret_cast<uint4*>(row + ((c8 ^ (j & 7)) << 4)) = make_uint4(q[0], q[1], q[2], q[3]);
  atoms[(((size_t)f * ns4 + step) * 2 + (c8 >> 2)) * kSfAtom + (j & 31) * 16 + (j >> 5) * 4 + (c8 & 3)] = (uint8_t)c;
}

// The same tiles with ue4m3 scales per 16 (NVFP4 layers, kind::mxf4nvf4):
// four atoms per step, atom a holding blocks 4 a .. 4 a + 3 of 16; the
// 32-block's two halves take the same code.
__device__ __forceinline__ void put_nv(uint8_t* blocks, uint8_t* atoms, int f, int ns4, int j, int b,
                                       const uint32_t (&q)[4], uint32_t code) {
  const int step = b >> 3, c8 = b & 7;
  uint8_t* row = blocks + ((size_t)f * ns4 + step) * kXBlock + j * kXK;
  *reinterpret_cast<uint4*>(row + ((c8 ^ (j & 7)) << 4)) = make_uint4(q[0], q[1], q[2], q[3]);
  *reinterpret_cast<uint16_t*>(atoms + (((size_t)f * ns4 + step) * 4 + (c8 >> 1)) * kSfAtom + (j & 31) * 16 +
                               (j >> 5) * 4 + 2 * (c8 & 1)) = (uint16_t)(code * 0x0101u);
}

// NVFP4 layers in QK_ACT_MXFP4: the row's 32-block scale codes c (the OCP
// rule, as for MXFP4 layers) become ue4m3 codes of 2^(c - cmax + 8), cmax the
// row's largest, and the row's factor 2^(cmax - 135) goes to the epilogue:
// the product is exact while c >= cmax - 17; a block further below its row's
// largest (values under 2^-17 of them) is flushed to zero.
__device__ __forceinline__ int row_max_code(int c) {
  __shared__ int cm;
  if (threadIdx.x == 0) cm = 0;
  __syncthreads();
  atomicMax(&cm, c);
  __syncthreads();
  const int r = cm;
  __syncthreads();
  return r;
}

// One block per token: its pairs' sorted rows (counting-sort scatter) and
// tile positions, then x split into two e4m3 terms per 32-block (QK_ACT_NONE,
// 64-token tiles) or quantized to one term (the activation-quantized modes,
// 128-token tiles: e4m3 codes, or packed e2m1 for QK_ACT_MXFP4), written into
// the gate/up tile of each pair.
__global__ void __launch_bounds__(kRowThreads) k_gmx_xsplit(GroupWs W, const uint16_t* __restrict__ x,
                                                            const int32_t* __restrict__ ids, int k, int E, int H,
                                                            int act_quant, int nv) {
  const int tok1 = gmx_tok1(act_quant), tok2 = gmx_tok2(act_quant);
  __shared__ int fj[8];
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    const int p = t * k + threadIdx.x;
    const int e = ids[p];
    int r = -1, tj = -1;
    if (e >= 0 && e < E) {
      const int o = W.offsets[e];
      r = o + atomicAdd(&W.fill[e], 1);
      const int rel = r - o;
      tj = ((W.L1.exp_tile0[e] + rel / tok1) << 8) | (rel % tok1);
      W.rtile2[r] = ((W.L2.exp_tile0[e] + rel / tok2) << 8) | (rel % tok2);
    } else {
      set_status(QK_ERR_INVALID_ARG);
    }
    W.inv[p] = r;
    fj[threadIdx.x] = tj;
  }
  __syncthreads();
  const int nb = H / 32, ns = H / kXK;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  auto load = [&](int b, float (&v)[32]) {
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
  };
  if (nv) {  // QK_ACT_MXFP4 on an NVFP4 layer: the codes twice, the row's largest scale between
    int cm = 0;
    for (int b = threadIdx.x; b < nb; b += kRowThreads) {
      float v[32];
      uint32_t q4[4];
      load(b, v);
      if (!all_finite32(v)) set_status(QK_ERR_NONFINITE);
      cm = max(cm, actq_block_fp4(v, q4));
    }
    cm = row_max_code(cm);
    for (int b = threadIdx.x; b < nb; b += kRowThreads) {
      float v[32];
      uint32_t q4[4];
      load(b, v);
      const uint32_t code = actq_nv_code(actq_block_fp4(v, q4) - cm + 8);
      for (int s = 0; s < k; ++s)
        if (fj[s] >= 0) put_nv(W.xt, W.sfx, fj[s] >> 8, H / 256, fj[s] & 255, b, q4, code);
    }
    if (threadIdx.x < k && fj[threadIdx.x] >= 0) W.fac1[W.inv[t * k + threadIdx.x]] = actq_pow2(cm - 135);
    return;
  }
  for (int b = threadIdx.x; b < nb; b += kRowThreads) {
    float v[32];
    load(b, v);
    if (!all_finite32(v)) set_status(QK_ERR_NONFINITE);
    if (act_quant == QK_ACT_MXFP4) {
      uint32_t q4[4];
      const int c = actq_block_fp4(v, q4);
      for (int s = 0; s < k; ++s)
        if (fj[s] >= 0) put_fp4(W.xt, W.sfx, fj[s] >> 8, H / 256, fj[s] & 255, b, q4, c);
      continue;
    }
    uint32_t q0[8], q1[8];
    if (act_quant == QK_ACT_E4M3) {
      const int c = actq_block(v, q0, 0);
      for (int s = 0; s < k; ++s)
        if (fj[s] >= 0) put_term(W.xt, W.sfx, fj[s] >> 8, ns, 32, fj[s] & 255, 0, b, q0, c);
      continue;
    }
    const int c0 = split_term(v, q0), c1 = split_term(v, q1);
    for (int s = 0; s < k; ++s) {
      const int tj = fj[s];
      if (tj < 0) continue;
      put_term(W.xt, W.sfx, tj >> 8, ns, kXTok1 / 4, tj & 255, 0, b, q0, c0);
      put_term(W.xt, W.sfx, tj >> 8, ns, kXTok1 / 4, tj & 255, 1, b, q1, c1);
    }
  }
}

// One block per sorted row: h = silu(gate) * up in fp32, split into three
// e4m3 terms per 32-block (QK_ACT_NONE, 40-token tiles) or quantized to one
// term (the activation-quantized modes, 128-token tiles: e4m3 codes, or
// packed e2m1 for QK_ACT_MXFP4), written into the row's down tile.
__global__ void __launch_bounds__(kRowThreads) k_gmx_hsplit(GroupWs W, int E, int I, int act_quant, int nv) {
  const int r = blockIdx.x;
  if (r >= W.offsets[E]) return;  // block-uniform
  const int tj = W.rtile2[r], f = tj >> 8, j = tj & 255;
  const float4* g4 = reinterpret_cast<const float4*>(W.gu + (size_t)r * 2 * I);
  const float4* u4 = g4 + I / 4;
  const int nb = I / 32, ns = I / kXK;
  auto swiglu = [&](int b, float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 g = __ldcg(g4 + b * 8 + q), u = __ldcg(u4 + b * 8 + q);
      v[4 * q + 0] = __fdividef(g.x, 1.0f + __expf(-g.x)) * u.x;
      v[4 * q + 1] = __fdividef(g.y, 1.0f + __expf(-g.y)) * u.y;
      v[4 * q + 2] = __fdividef(g.z, 1.0f + __expf(-g.z)) * u.z;
      v[4 * q + 3] = __fdividef(g.w, 1.0f + __expf(-g.w)) * u.w;
    }
  };
  if (nv) {  // QK_ACT_MXFP4 on an NVFP4 layer (see k_gmx_xsplit)
    int cm = 0;
    for (int b = threadIdx.x; b < nb; b += kRowThreads) {
      float v[32];
      uint32_t q4[4];
      swiglu(b, v);
      if (!all_finite32(v)) set_status(QK_ERR_NONFINITE);
      cm = max(cm, actq_block_fp4(v, q4));
    }
    cm = row_max_code(cm);
    for (int b = threadIdx.x; b < nb; b += kRowThreads) {
      float v[32];
      uint32_t q4[4];
      swiglu(b, v);
      const uint32_t code = actq_nv_code(actq_block_fp4(v, q4) - cm + 8);
      put_nv(W.ht, W.sfh, f, I / 256, j, b, q4, code);
    }
    if (threadIdx.x == 0) W.fac2[r] = actq_pow2(cm - 135);
    return;
  }
  for (int b = threadIdx.x; b < nb; b += kRowThreads) {
    float v[32];
    swiglu(b, v);
    if (!all_finite32(v)) set_status(QK_ERR_NONFINITE);
    if (act_quant == QK_ACT_NONE) {
#pragma unroll
      for (int term = 0; term < 3; ++term) {
        uint32_t q[8];
        const int c = split_term(v, q);
        put_term(W.ht, W.sfh, f, ns, kXTok2 / 4, j, term, b, q, c);
      }
    } else if (act_quant == QK_ACT_MXFP4) {  // one packed e2m1 term, 128-token tiles
      uint32_t q4[4];
      const int c = actq_block_fp4(v, q4);
      put_fp4(W.ht, W.sfh, f, I / 256, j, b, q4, c);
    } else {  // one e4m3 term, 128-token tiles
      uint32_t q[8];
      const int c = actq_block(v, q, 0);
      put_term(W.ht, W.sfh, f, ns, 32, j, 0, b, q, c);
    }
  }
}

}  // namespace qk

namespace qk {

// ---------------------------------------------------------- grouped GEMM --
constexpr int kWN = 256;               // weight rows per tile (tcgen05 N)
constexpr int kXThreads = 12 * 32;     // warp 0 weights, 1 MMA, 2 tokens, 3 weight scales, 4-11 epilogue
constexpr int kXStageW = kWN * kXK;    // 32 KB: 256 rows x 128 codes, one code per byte position
constexpr int kXWS = 4;                // weight stages (one reduction step each)
constexpr int kXTS = 2;                // token stages (two steps each)
constexpr int kXStageT = 2 * kXBlock;  // 32 KB
constexpr int kXSS = 2;                // weight-scale chunk slots (4 steps x 2 atoms each)
constexpr int kXSfaCol = 256;          // token scales: 4 columns; weight scales: 8 columns after them
constexpr int kXTmemCols = 512;
constexpr int kXTSa = 8;               // token scale atoms per token stage (2 steps x up to 4)
constexpr int kXSmem = 1024 + kXWS * kXStageW + kXTS * (kXStageT + kXTSa * kSfAtom) + kXSS * 8 * kSfAtom + 256;

struct GmxArgs {
  TileList L;            // token tiles of this phase
  const uint8_t* blocks; // [F][K / 128] token blocks (16 KB) of this phase
  const uint8_t* atoms;  // [F][K / 128][512] their scale atoms
  const uint8_t* sf_a;   // e8m0 scales [E * rows][K / 32] of the gate (or down) rows
  const uint8_t* sf_b;   // e8m0 scales of the up rows (gate/up phase)
  float* out;            // gate/up: gu [P][2 I]; down: dperm [P][H]
  int K, rows_per_e, MB, MBA, out_ld;  // MBA: weight blocks taken from ta / sf_a (the rest: tb / sf_b)
  int wfp8;              // 0: MXFP4 weights (e2m1, e8m0 per 32 in [rows][K / 32]); 1: FP8 E4M3 weights with
  int sblk;              //    UE8M0 tile scales, one per sblk x sblk tile (128 or 32) in [rows / sblk][K / sblk]
  const float* s2a;      // NVFP4 weights: scale_2 [E] of the gate (or down) projection
  const float* s2b;      //    and of the up projection
  const float* fac;      // NVFP4 weights: per sorted row, the factor of its token scales
  // Fused gate/up (fuse = 1): a tile is 128 gate rows and the same 128 up
  // rows (two 128-row boxes per step), and the epilogue writes h = silu(gate)
  // * up straight into the down tiles in the mode's split (no gu, no h split
  // kernel).
  int fuse, act_quant, I;
  const int* rtile2;     // [P] per sorted row: (down tile << 8) | row within it
  uint8_t* ht;           // down token blocks
  uint8_t* sfh;          // their scale atoms
  alignas(64) CUtensorMap ta, tb;  // MXFP4: 16 x 4-bit -> 16-byte slots; FP8: bytes; box {128, 256}, 128B swizzle
};

struct GmxHead {
  alignas(8) uint64_t wfull[kXWS];   // weight tile landed (TMA)
  alignas(8) uint64_t wempty[kXWS];  // its MMAs completed
  alignas(8) uint64_t tfull[kXTS];   // token blocks and their scale atoms landed
  alignas(8) uint64_t tempty[kXTS];
  alignas(8) uint64_t sfull[kXSS];   // four steps' weight scale atoms written (scale warp)
  alignas(8) uint64_t sempty[kXSS];
  alignas(8) uint64_t acc_full;
  alignas(8) uint64_t acc_empty;     // the epilogue has read the accumulator
  alignas(8) uint64_t drained;
  uint32_t tmem;
  int abort;
};

__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Work tile t: the tiles of one expert are ordered weight block major, so
// consecutive blocks share a weight block (read from HBM once, then from L2)
// and differ in their token tile.
__device__ __forceinline__ void gmx_tile(const TileList& L, int MB, int t, int& f, int& mb) {
  const int f0 = t / MB;
  const int first = L.tile_first[f0], cnt = L.tile_cnt[f0];
  const int u = t - first * MB;
  mb = u / cnt;
  f = first + (u - mb * cnt);
}

// NT: terms per token (2 for x, 3 for h, 1 in the activation-quantized
// modes).  FP4: both operands packed e2m1 (QK_ACT_MXFP4), kind::mxf4 with a
// reduction step of 256 elements (the weights copied as stored, 32 KB per
// stage), two token scale atoms per step and two steps per weight-scale
// chunk; otherwise kind::mxf8f6f4 with steps of 128.  NV (with FP4): NVFP4
// weights, kind::mxf4nvf4 with ue4m3 scales per 16: four token and eight
// weight scale atoms per step (one per instruction and 128 rows), one step
// per weight-scale chunk, and the epilogue applies scale_2 and the row factor.
template <bool GATEUP, int NT, bool FP4, bool NV = false>
__global__ void __launch_bounds__(kXThreads, 1) k_gmx(const __grid_constant__ GmxArgs G) {
  static_assert(!FP4 || NT == 1, "the fp4 x fp4 tiles hold one term");
  static_assert(!NV || FP4, "NVFP4 weights run fp4 x fp4 only");
  constexpr int NPQ = NT == 1 ? 32 : NT == 2 ? kXTok1 / 4 : kXTok2 / 4;  // tokens per TMEM lane quadrant
  constexpr int AT = NV ? 4 : FP4 ? 2 : 1;   // token scale atoms per step
  constexpr int SPC = NV ? 1 : FP4 ? 2 : 4;  // steps per weight-scale chunk (16 bytes of each row)
  constexpr bool FUSE = GATEUP && !NV;       // instantiations that may run the fused gate/up (G.fuse)
  extern __shared__ __align__(16) uint8_t smem_raw[];  // rounded up to 1024 below, at run time
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sW = base;                                  // kXWS weight stages
  uint8_t* sT = sW + kXWS * kXStageW;                  // kXTS token stages
  uint8_t* sTa = sT + kXTS * kXStageT;                 // kXTS x kXTSa token scale atoms (2 steps x AT)
  uint8_t* sSa = sTa + kXTS * kXTSa * kSfAtom;         // kXSS x 8 weight scale atoms
  GmxHead& S = *reinterpret_cast<GmxHead*>(sSa + kXSS * 8 * kSfAtom);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const TileList& L = G.L;
  const int MB = G.MB, KS = G.K / (FP4 ? 2 * kXK : kXK);
  const unsigned long long limit = g_wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kXWS; ++s) {
      mbar_init(&S.wfull[s], 1);
      mbar_init(&S.wempty[s], 1);
    }
    for (int s = 0; s < kXTS; ++s) {
      mbar_init(&S.tfull[s], 1);
      mbar_init(&S.tempty[s], 1);
    }
    for (int s = 0; s < kXSS; ++s) {
      mbar_init(&S.sfull[s], 1);
      mbar_init(&S.sempty[s], 1);
    }
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.acc_empty, 8);
    mbar_init(&S.drained, 1);
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&S.tmem, kXTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem;
  const int n_tiles = *L.n_tiles * MB;
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(&S.abort)) return false;
    if (mbar_wait_bounded(bar, parity, limit)) return true;
    set_status(QK_ERR_TIMEOUT);
    *reinterpret_cast<volatile int*>(&S.abort) = 1;
    return false;
  };
  auto aborted = [&]() { return *reinterpret_cast<volatile int*>(&S.abort) != 0; };

  if (warp == 0) {
    // ----------------------------------------------------- weight tiles --
    // Loads only: an L2 prefetch of later steps costs the SM's TMA unit as
    // much as a load, and measured slower (the 2048-token fp4 x fp4 layer
    // 1.13 -> 0.97 ms without it).
    if (lane == 0) {
      const uint64_t pw = policy_evict_normal();
      auto coords = [&](int t, const void*& map, int& wrow) {
        int f, mb;
        gmx_tile(L, MB, t, f, mb);
        if (FUSE && G.fuse) {  // gate rows, then the same up rows (map tb)
          map = &G.ta;
          wrow = L.tile_e[f] * G.rows_per_e + mb * (kWN / 2);
          return;
        }
        const bool b = mb >= G.MBA;
        map = b ? &G.tb : &G.ta;
        wrow = L.tile_e[f] * G.rows_per_e + (b ? mb - G.MBA : mb) * kWN;
      };
      int n = 0;
      for (int t = blockIdx.x; t < n_tiles && !aborted(); t += gridDim.x) {
        const void* map = nullptr;
        int wrow = 0;
        coords(t, map, wrow);
        for (int ks = 0; ks < KS; ++ks, ++n) {
          const int s = n % kXWS;
          if (n >= kXWS && !wait(&S.wempty[s], (uint32_t)((n / kXWS - 1) & 1))) break;
          // counted in global bytes: packed (4-bit) codes, or one byte per FP8 code
          mbar_arrive_expect_tx(&S.wfull[s], (uint32_t)(G.wfp8 || FP4 ? kXStageW : kXStageW / 2));
          if (FUSE && G.fuse) {
            tma_load_2d(sW + s * kXStageW, &G.ta, ks * kXK, wrow, &S.wfull[s], pw);
            tma_load_2d(sW + s * kXStageW + kXStageW / 2, &G.tb, ks * kXK, wrow, &S.wfull[s], pw);
          } else {
            tma_load_2d(sW + s * kXStageW, map, ks * kXK, wrow, &S.wfull[s], pw);
          }
        }
      }
      for (int q = n > kXWS ? n - kXWS : 0; q < n; ++q)  // nothing may still be landing at exit
        if (!mbar_wait_bounded(&S.wfull[q % kXWS], (uint32_t)((q / kXWS) & 1), kDrainLimitNs)) break;
    }
    __syncwarp();
  } else if (warp == 3) {
    // ----------------------------------------------------- weight scales --
    // Four reduction steps at a time: every lane loads 16 bytes (4 steps x 4
    // blocks) of eight of the tile's 256 rows, one chunk ahead, and writes
    // the four steps' two atoms each; one proxy fence and one arrival.  FP8
    // tile scales are expanded to the same per-32 bytes: a 128 x 128 tile's
    // code serves its rows' four blocks of each step, a 32 x 32 tile's code
    // one block of 32 rows.
    const int srow = G.K / (NV ? 16 : 32);  // MXFP4 (NVFP4) scale bytes per weight row
    // the 16 bytes of chunk `chunk` (4 steps) of rows lane + 32 j of tile t
    auto fetch = [&](int t, int chunk, uint4 (&r)[8]) {
      int f, mb;
      gmx_tile(L, MB, t, f, mb);
      if (FUSE && G.fuse) {  // rows 0-127 gate, 128-255 the same up rows
        const int base = L.tile_e[f] * G.rows_per_e + mb * (kWN / 2);
        if (!G.wfp8) {
          const uint8_t* ra = G.sf_a + (size_t)(base + lane) * srow + chunk * 16;
          const uint8_t* rb = G.sf_b + (size_t)(base + lane) * srow + chunk * 16;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            r[j] = __ldg(reinterpret_cast<const uint4*>(ra + (size_t)32 * j * srow));
            r[4 + j] = __ldg(reinterpret_cast<const uint4*>(rb + (size_t)32 * j * srow));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint8_t* sf = j < 4 ? G.sf_a : G.sf_b;
            const int r0 = base + 32 * (j & 3);  // first of the 32 rows
            if (G.sblk == 128) {
              const uint32_t c4 =
                  __ldg(reinterpret_cast<const uint32_t*>(sf + (size_t)(r0 / 128) * (G.K / 128) + 4 * chunk));
              r[j] = make_uint4((c4 & 0xFFu) * 0x01010101u, ((c4 >> 8) & 0xFFu) * 0x01010101u,
                                ((c4 >> 16) & 0xFFu) * 0x01010101u, (c4 >> 24) * 0x01010101u);
            } else {
              r[j] = __ldg(reinterpret_cast<const uint4*>(sf + (size_t)(r0 / 32) * (G.K / 32) + 16 * chunk));
            }
          }
        }
        return;
      }
      const bool b = mb >= G.MBA;
      const uint8_t* sf = b ? G.sf_b : G.sf_a;
      const int base = L.tile_e[f] * G.rows_per_e + (b ? mb - G.MBA : mb) * kWN;
      if (!G.wfp8) {
        const uint8_t* rp = sf + (size_t)(base + lane) * srow + chunk * 16;
#pragma unroll
        for (int j = 0; j < 8; ++j) r[j] = __ldg(reinterpret_cast<const uint4*>(rp + (size_t)32 * j * srow));
      } else if (G.sblk == 128) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t c4 = __ldg(reinterpret_cast<const uint32_t*>(
              sf + (size_t)((base + 32 * j) / 128) * (G.K / 128) + 4 * chunk));
          r[j] = make_uint4((c4 & 0xFFu) * 0x01010101u, ((c4 >> 8) & 0xFFu) * 0x01010101u,
                            ((c4 >> 16) & 0xFFu) * 0x01010101u, (c4 >> 24) * 0x01010101u);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          r[j] = __ldg(reinterpret_cast<const uint4*>(sf + (size_t)((base + 32 * j) / 32) * (G.K / 32) + 16 * chunk));
      }
    };
    uint4 cur[8], nxt[8];
    if ((int)blockIdx.x < n_tiles) fetch(blockIdx.x, 0, nxt);
    int n = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
      for (int c = 0; c < KS / SPC; ++c, ++n) {
#pragma unroll
        for (int j = 0; j < 8; ++j) cur[j] = nxt[j];
        const int tn = c + 1 < KS / SPC ? t : t + (int)gridDim.x;
        if (tn < n_tiles) fetch(tn, tn == t ? c + 1 : 0, nxt);
        uint32_t ff = 0;
        const uint32_t nm = NV ? 0x80808080u : 0u;  // e4m3 NaN: 0x7F and 0xFF; e8m0 NaN: 0xFF
#pragma unroll
        for (int j = 0; j < 8; ++j)
          ff |= __vcmpeq4(cur[j].x | nm, 0xFFFFFFFFu) | __vcmpeq4(cur[j].y | nm, 0xFFFFFFFFu) |
                __vcmpeq4(cur[j].z | nm, 0xFFFFFFFFu) | __vcmpeq4(cur[j].w | nm, 0xFFFFFFFFu);
        if (ff) set_status(QK_ERR_NAN_SCALE);
        const int s = n % kXSS;
        if (n >= kXSS && !__all_sync(0xffffffffu, wait(&S.sempty[s], (uint32_t)((n / kXSS - 1) & 1)))) {
          ok = false;
          break;
        }
        // slot: [step q][atom a][line lane], line = rows lane + 128 a + {0, 32, 64, 96}
        uint8_t* d = sSa + s * 8 * kSfAtom + lane * 16;
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const uint4* r = cur + 4 * a;
          *reinterpret_cast<uint4*>(d + (0 * 2 + a) * kSfAtom) = make_uint4(r[0].x, r[1].x, r[2].x, r[3].x);
          *reinterpret_cast<uint4*>(d + (1 * 2 + a) * kSfAtom) = make_uint4(r[0].y, r[1].y, r[2].y, r[3].y);
          *reinterpret_cast<uint4*>(d + (2 * 2 + a) * kSfAtom) = make_uint4(r[0].z, r[1].z, r[2].z, r[3].z);
          *reinterpret_cast<uint4*>(d + (3 * 2 + a) * kSfAtom) = make_uint4(r[0].w, r[1].w, r[2].w, r[3].w);
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_one(&S.sfull[s]);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------ token blocks --
    // Two reduction steps per stage: the tile's two 16-KB blocks and two scale
    // atoms are contiguous in global memory (one bulk copy each).
    if (lane == 0) {
      int n = 0;
      for (int t = blockIdx.x; t < n_tiles && !aborted(); t += gridDim.x) {
        int f, mb;
        gmx_tile(L, MB, t, f, mb);
        for (int k0 = 0; k0 < KS; k0 += 2, ++n) {
          const int s = n % kXTS;
          if (k0 + 2 * kXTS < KS)  // the stage after the ring into L2
            bulk_prefetch_l2(G.blocks + ((size_t)f * KS + k0 + 2 * kXTS) * kXBlock, (uint32_t)kXStageT);
          if (n >= kXTS && !wait(&S.tempty[s], (uint32_t)((n / kXTS - 1) & 1))) break;
          mbar_arrive_expect_tx(&S.tfull[s], (uint32_t)(kXStageT + 2 * AT * kSfAtom));
          const size_t blk = (size_t)f * KS + k0;
          bulk_g2s(sT + s * kXStageT, G.blocks + blk * kXBlock, (uint32_t)kXStageT, &S.tfull[s]);
          bulk_g2s(sTa + s * kXTSa * kSfAtom, G.atoms + blk * AT * kSfAtom, (uint32_t)(2 * AT * kSfAtom), &S.tfull[s]);
        }
      }
      for (int q = n > kXTS ? n - kXTS : 0; q < n; ++q)
        if (!mbar_wait_bounded(&S.tfull[q % kXTS], (uint32_t)((q / kXTS) & 1), kDrainLimitNs)) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t t_sfa = tmem + kXSfaCol, t_sfb = t_sfa + 4 * AT;
      // A e4m3 (token terms); B e2m1 (MXFP4 weights) or e4m3 (FP8 weights);
      // FP4: both e2m1 (format 1 of kind::mxf4)
      const uint32_t idesc = NV ? umma_idesc_nv(128, kWN)
                             : FP4 ? umma_idesc_mx(128, kWN, 1, 1) : umma_idesc_mx(128, kWN, 0, G.wfp8 ? 0 : 5);
      int nw = 0, nt = 0, nc = 0, i = 0;
      for (int t = blockIdx.x; t < n_tiles && !aborted(); t += gridDim.x, ++i) {
        if (i >= 1 && !wait(&S.acc_empty, (uint32_t)((i - 1) & 1))) break;
        tc_fence_after();
        bool ok = true;
        for (int ks = 0; ks < KS; ++ks, ++nw) {
          const int sw = nw % kXWS, st = nt % kXTS, sc = nc % kXSS, j = ks & 1, q = ks % SPC;
          if (!wait(&S.wfull[sw], (uint32_t)((nw / kXWS) & 1)) ||
              (j == 0 && !wait(&S.tfull[st], (uint32_t)((nt / kXTS) & 1))) ||
              (q == 0 && !wait(&S.sfull[sc], (uint32_t)((nc / kXSS) & 1)))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = umma_desc_k_sw128(sT + st * kXStageT + j * kXBlock);
          const uint64_t db = umma_desc_k_sw128(sW + sw * kXStageW);
          if (!FP4) {
            utccp_32x128b_x4(t_sfa, umma_desc_sf(sTa + (st * kXTSa + j) * kSfAtom));
            utccp_32x128b_x4(t_sfb, umma_desc_sf(sSa + (sc * 8 + q * 2) * kSfAtom));
            utccp_32x128b_x4(t_sfb + 4, umma_desc_sf(sSa + (sc * 8 + q * 2 + 1) * kSfAtom));
#pragma unroll
            for (int kb = 0; kb < kXK / 32; ++kb)
              umma_mx(tmem, da + 2 * kb, db + 2 * kb, umma_idesc_sf_ids(idesc, kb, kb), t_sfa | ((uint32_t)kb << 30),
                      t_sfb | ((uint32_t)kb << 30), (ks | kb) != 0 ? 1u : 0u);
          } else if (NV) {
            // instruction kk (K = 64: blocks 4 kk .. 4 kk + 3 of 16): token atom
            // kk of the step at t_sfa + 4 kk, weight atoms (rows 0-127,
            // 128-255) at t_sfb + 8 kk and + 4; all four bytes of the column
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              utccp_32x128b_x4(t_sfa + 4 * kk, umma_desc_sf(sTa + (st * kXTSa + j * 4 + kk) * kSfAtom));
              utccp_32x128b_x4(t_sfb + 8 * kk, umma_desc_sf(sSa + (sc * 8 + kk * 2) * kSfAtom));
              utccp_32x128b_x4(t_sfb + 8 * kk + 4, umma_desc_sf(sSa + (sc * 8 + kk * 2 + 1) * kSfAtom));
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_nvf4(tmem, da + 2 * kk, db + 2 * kk, idesc, t_sfa + 4 * kk, t_sfb + 8 * kk, (ks | kk) != 0 ? 1u : 0u);
          } else {
            // blocks 0-3 and 4-7 of the step: token atoms in columns t_sfa and
            // t_sfa + 4, weight atoms (rows 0-127, 128-255) at t_sfb + 8 g and
            // + 4; MMA k (K = 64) takes blocks 2 k, 2 k + 1: group k / 2, byte
            // pair 2 (k % 2)
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              utccp_32x128b_x4(t_sfa + 4 * g, umma_desc_sf(sTa + (st * kXTSa + j * 2 + g) * kSfAtom));
              utccp_32x128b_x4(t_sfb + 8 * g, umma_desc_sf(sSa + (sc * 8 + (2 * q + g) * 2) * kSfAtom));
              utccp_32x128b_x4(t_sfb + 8 * g + 4, umma_desc_sf(sSa + (sc * 8 + (2 * q + g) * 2 + 1) * kSfAtom));
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t sid = (uint32_t)(kk & 1) * 2;
              umma_mxf4(tmem, da + 2 * kk, db + 2 * kk, umma_idesc_sf_ids(idesc, (int)sid, (int)sid),
                        (t_sfa + 4 * (kk >> 1)) | (sid << 30), (t_sfb + 8 * (kk >> 1)) | (sid << 30),
                        (ks | kk) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&S.wempty[sw]);
          if (j == 1) {
            umma_commit(&S.tempty[st]);
            ++nt;
          }
          if (q == SPC - 1) {
            umma_commit(&S.sempty[sc]);
            ++nc;
          }
        }
        if (!ok) break;
        umma_commit(&S.acc_full);
      }
      umma_commit(&S.drained);  // every MMA issued here completes before the accumulator is freed
      mbar_wait_bounded(&S.drained, 0, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue --
    // Warp (quadrant q, half h) reads TMEM lanes 32 q .. 32 q + 31, columns
    // 128 h .. 128 h + 127; lane NPQ t + l holds term t of token NPQ q + l.
    const int quad = warp & 3, half = (warp - 4) >> 2;
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      int f, mb;
      gmx_tile(L, MB, t, f, mb);
      const int row0 = L.tile_row0[f], nrow = L.tile_n[f];
      if (!__all_sync(0xffffffffu, wait(&S.acc_full, (uint32_t)(i & 1)))) break;
      tc_fence_after();
      const int tok = NPQ * quad + lane;
      const bool st = lane < NPQ && tok < nrow;
      if (FUSE && G.fuse) {
        // Columns c (gate) and 128 + c (up) are intermediate index 128 mb + c
        // of the same token: warp half h takes the 32-column chunks 2 h and
        // 2 h + 1, forms h = silu(gate) * up (the h split kernel's
        // arithmetic) and writes its 32-blocks into the down tiles.
        const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16);
        float hv[2][32];
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int cc = 2 * half + k2;
          uint32_t g[32], u[32];
          tmem_ld32(tq + (uint32_t)(cc * 32), g);
          tmem_ld32(tq + (uint32_t)(kWN / 2 + cc * 32), u);
          if (k2 == 1) {  // the accumulator is read: the next tile's MMAs may start
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_one(&S.acc_empty);
          }
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            float a = __uint_as_float(g[jj]), b = __uint_as_float(u[jj]);
            if (NT > 1) {
              a += __shfl_down_sync(0xffffffffu, a, NPQ);
              b += __shfl_down_sync(0xffffffffu, b, NPQ);
              if (NT == 3) {
                a += __shfl_down_sync(0xffffffffu, __uint_as_float(g[jj]), 2 * NPQ);
                b += __shfl_down_sync(0xffffffffu, __uint_as_float(u[jj]), 2 * NPQ);
              }
            }
            hv[k2][jj] = __fdividef(a, 1.0f + __expf(-a)) * b;
          }
        }
        if (st) {
          const int tj = __ldg(G.rtile2 + row0 + tok), f2 = tj >> 8, j2 = tj & 255;
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            float (&v)[32] = hv[k2];
            const int b = mb * 4 + 2 * half + k2;  // 32-block of the h row
            if (!all_finite32(v)) set_status(QK_ERR_NONFINITE);
            if (G.act_quant == QK_ACT_NONE) {
#pragma unroll
              for (int term = 0; term < 3; ++term) {
                uint32_t q[8];
                const int c = split_term(v, q);
                put_term(G.ht, G.sfh, f2, G.I / kXK, kXTok2 / 4, j2, term, b, q, c);
              }
            } else if (G.act_quant == QK_ACT_MXFP4) {
              uint32_t q4[4];
              const int c = actq_block_fp4(v, q4);
              put_fp4(G.ht, G.sfh, f2, G.I / 256, j2, b, q4, c);
            } else {
              uint32_t q[8];
              const int c = actq_block(v, q, 0);
              put_term(G.ht, G.sfh, f2, G.I / kXK, 32, j2, 0, b, q, c);
            }
          }
        }
        continue;
      }
      float* out = G.out + (size_t)(row0 + (st ? tok : 0)) * G.out_ld + mb * kWN + half * 128;
      float mul = 1.f;  // NVFP4: scale_2 of the tile's expert and projection, times the row's factor
      if (NV && st) mul = __ldg((mb >= G.MBA ? G.s2b : G.s2a) + L.tile_e[f]) * __ldg(G.fac + row0 + tok);
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(half * 128);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(taddr + (uint32_t)(c * 32), v);
        if (c == 3) {  // the accumulator is read: the next tile's MMAs may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_one(&S.acc_empty);
        }
        if (NT > 1) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            float a = __uint_as_float(v[jj]);
            a += __shfl_down_sync(0xffffffffu, a, NPQ);
            if (NT == 3) a += __shfl_down_sync(0xffffffffu, __uint_as_float(v[jj]), 2 * NPQ);
            v[jj] = __float_as_uint(a);
          }
        }
        if (NV) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) v[jj] = __float_as_uint(__uint_as_float(v[jj]) * mul);
        }
        if (st) {
          float4* o4 = reinterpret_cast<float4*>(out + c * 32);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            o4[jj] = make_float4(__uint_as_float(v[4 * jj]), __uint_as_float(v[4 * jj + 1]),
                                 __uint_as_float(v[4 * jj + 2]), __uint_as_float(v[4 * jj + 3]));
        }
      }
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
  if (H % 512 != 0 || I % 512 != 0) return false;  // 16-byte scale chunks per row (4 steps of 128), 256-row blocks
  return al(gate.q, 32) && al(up.q, 32) && al(down.q, 32) && al(gate.scales, 16) && al(up.scales, 16) &&
         al(down.scales, 16);
}

bool gmx_nv_eligible(const qk_weight& gate, const qk_weight& up, const qk_weight& down, int H, int I) {
  auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (gate.fmt != QK_FMT_NVFP4 || up.fmt != QK_FMT_NVFP4 || down.fmt != QK_FMT_NVFP4) return false;
  if (!gate.scale_2 || !up.scale_2 || !down.scale_2) return false;
  if (H % 512 != 0 || I % 512 != 0) return false;  // 16-byte scale chunks per row (one step of 256), 256-row blocks
  return al(gate.q, 32) && al(up.q, 32) && al(down.q, 32) && al(gate.scales, 16) && al(up.scales, 16) &&
         al(down.scales, 16);
}

// Packed e2m1 rows [rows][K / 2]: 16 codes (8 bytes) per 16-byte slot in
// shared memory, boxes {128 codes, 256 rows}, 128-byte swizzle.  A box reads
// 64 bytes of each row; 256-byte L2 promotion brings the row's next three
// steps into L2 with the first.
static bool x_map_weights(CUtensorMap* m, const uint8_t* q, int64_t rows, int K, int box_rows = kWN) {
  const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)K / 2};
  const uint32_t box[2] = {(uint32_t)kXK, (uint32_t)box_rows};
  return tmap_get(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// FP8 E4M3 rows [rows][K] bytes, boxes {128, 256}, 128-byte swizzle: the same
// shared-memory layout as the expanded e2m1 slots (one code per byte).
static bool x_map_fp8(CUtensorMap* m, const uint8_t* q, int64_t rows, int K, int box_rows = kWN) {
  const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)K};
  const uint32_t box[2] = {(uint32_t)kXK, (uint32_t)box_rows};
  return tmap_get(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

template <bool GATEUP, int NT, bool FP4 = false, bool NV = false>
static qk_status x_launch(const GmxArgs& A, cudaStream_t st) {
  static_assert(sizeof(GmxHead) <= 256, "head");
  if (kXSmem > max_smem_optin()) return QK_ERR_UNSUPPORTED;
  return launch_ex(k_gmx<GATEUP, NT, FP4, NV>, dim3(num_sms()), dim3(kXThreads), (size_t)kXSmem, st, false, A);
}

// Packed e2m1 rows [rows][K / 2] as bytes, boxes {128 bytes (256 codes), 256
// rows}, 128-byte swizzle: the fp4 x fp4 path reads the weights as stored.
static bool x_map_packed(CUtensorMap* m, const uint8_t* q, int64_t rows, int K, int box_rows = kWN) {
  const uint64_t dims[2] = {(uint64_t)K / 2, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)K / 2};
  const uint32_t box[2] = {(uint32_t)kXK, (uint32_t)box_rows};
  return tmap_get(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

qk_status gmx_forward_act(const DecodeArgs& a, const GroupWs& W, int act_quant, cudaStream_t st) {
  const int T = a.T, k = a.k, E = a.E, H = a.H, I = a.I;
  const bool fp4 = act_quant == QK_ACT_MXFP4, one = act_quant != QK_ACT_NONE;
  const bool nv = fp4 && a.gate.fmt == QK_FMT_NVFP4;  // an all-NVFP4 layer (gmx_nv_eligible): kind::mxf4nvf4
  k_gmx_xsplit<<<T, kRowThreads, 0, st>>>(W, a.x, a.ids, k, E, H, act_quant, nv ? 1 : 0);
  if (cudaGetLastError() != cudaSuccess) return QK_ERR_CUDA;
  auto wmap = [&](CUtensorMap* m, const uint8_t* q, int64_t rows, int K, int box_rows = kWN) {
    return fp4 ? x_map_packed(m, q, rows, K, box_rows) : x_map_weights(m, q, rows, K, box_rows);
  };
  // MXFP4 layers: the gate/up epilogue forms h and writes the down tiles
  // itself (NVFP4 layers keep the h split kernel: their h scales are
  // anchored at the row's largest, known only once the whole row is in).
  const bool fuse = !nv;

  GmxArgs g1 = {};
  g1.L = W.L1;
  g1.blocks = W.xt;
  g1.atoms = W.sfx;
  g1.sf_a = a.gate.scales;
  g1.sf_b = a.up.scales;
  g1.out = W.gu;
  g1.K = H;
  g1.rows_per_e = I;
  g1.MB = 2 * I / kWN;  // gate blocks, then up blocks
  g1.MBA = I / kWN;
  g1.out_ld = 2 * I;
  g1.s2a = a.gate.scale_2;
  g1.s2b = a.up.scale_2;
  g1.fac = W.fac1;
  if (fuse) {
    g1.fuse = 1;
    g1.MB = I / (kWN / 2);  // 128 gate rows and the same 128 up rows per tile
    g1.MBA = g1.MB;
    g1.act_quant = act_quant;
    g1.I = I;
    g1.rtile2 = W.rtile2;
    g1.ht = W.ht;
    g1.sfh = W.sfh;
  }
  const int br = fuse ? kWN / 2 : kWN;
  if (!wmap(&g1.ta, a.gate.q, (int64_t)E * I, H, br) || !wmap(&g1.tb, a.up.q, (int64_t)E * I, H, br))
    return QK_ERR_CUDA;
  qk_status rc = nv    ? x_launch<true, 1, true, true>(g1, st)
                 : fp4 ? x_launch<true, 1, true>(g1, st)
                 : one ? x_launch<true, 1>(g1, st)
                       : x_launch<true, 2>(g1, st);
  if (rc != QK_OK) return rc;

  if (!fuse) {
    k_gmx_hsplit<<<a.P, kRowThreads, 0, st>>>(W, E, I, act_quant, nv ? 1 : 0);
    if (cudaGetLastError() != cudaSuccess) return QK_ERR_CUDA;
  }

  GmxArgs g2 = {};
  g2.L = W.L2;
  g2.blocks = W.ht;
  g2.atoms = W.sfh;
  g2.sf_a = a.down.scales;
  g2.sf_b = a.down.scales;
  g2.out = W.dperm;
  g2.K = I;
  g2.rows_per_e = H;
  g2.MB = H / kWN;
  g2.MBA = H / kWN;
  g2.out_ld = H;
  g2.s2a = a.down.scale_2;
  g2.s2b = a.down.scale_2;
  g2.fac = W.fac2;
  if (!wmap(&g2.ta, a.down.q, (int64_t)E * H, I)) return QK_ERR_CUDA;
  g2.tb = g2.ta;
  return nv    ? x_launch<false, 1, true, true>(g2, st)
         : fp4 ? x_launch<false, 1, true>(g2, st)
         : one ? x_launch<false, 1>(g2, st)
               : x_launch<false, 3>(g2, st);
}

// The FP8 SwiGLU FFN of a shared expert at large M on the same kernels: the M
// tokens form one group (one expert), x splits into 2 e4m3 terms, gate/up and
// down run as block-scaled GEMMs with e4m3 weights, and h splits into 3 terms
// between them.  The caller has counted and tiled the group (W) and adds
// W.dperm into y.
qk_status gmx_fp8_ffn(const GroupWs& W, const uint16_t* x, const int32_t* ids, int M, int H, int I,
                      const uint8_t* wg, const uint8_t* sg, const uint8_t* wu, const uint8_t* su,
                      const uint8_t* wd, const uint8_t* sd, int blk, cudaStream_t st) {
  k_gmx_xsplit<<<M, kRowThreads, 0, st>>>(W, x, ids, 1, 1, H, QK_ACT_NONE, 0);
  if (cudaGetLastError() != cudaSuccess) return QK_ERR_CUDA;
  GmxArgs g1 = {};
  g1.L = W.L1;
  g1.blocks = W.xt;
  g1.atoms = W.sfx;
  g1.sf_a = sg;
  g1.sf_b = su;
  g1.out = W.gu;
  g1.K = H;
  g1.rows_per_e = I;
  g1.MB = 2 * I / kWN;
  g1.MBA = I / kWN;
  g1.out_ld = 2 * I;
  g1.wfp8 = 1;
  g1.sblk = blk;
  g1.fuse = 1;  // h formed and split in the gate/up epilogue
  g1.MB = I / (kWN / 2);
  g1.MBA = g1.MB;
  g1.act_quant = QK_ACT_NONE;
  g1.I = I;
  g1.rtile2 = W.rtile2;
  g1.ht = W.ht;
  g1.sfh = W.sfh;
  if (!x_map_fp8(&g1.ta, wg, I, H, kWN / 2) || !x_map_fp8(&g1.tb, wu, I, H, kWN / 2)) return QK_ERR_CUDA;
  qk_status rc = x_launch<true, 2>(g1, st);
  if (rc != QK_OK) return rc;
  GmxArgs g2 = {};
  g2.L = W.L2;
  g2.blocks = W.ht;
  g2.atoms = W.sfh;
  g2.sf_a = sd;
  g2.sf_b = sd;
  g2.out = W.dperm;
  g2.K = I;
  g2.rows_per_e = H;
  g2.MB = H / kWN;
  g2.MBA = H / kWN;
  g2.out_ld = H;
  g2.wfp8 = 1;
  g2.sblk = blk;
  if (!x_map_fp8(&g2.ta, wd, H, I)) return QK_ERR_CUDA;
  g2.tb = g2.ta;
  return x_launch<false, 3>(g2, st);
}

}  // namespace qk
