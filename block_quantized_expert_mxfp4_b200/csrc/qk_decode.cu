// qk_decode.cu -- decode path of moe_expert_forward (up to 16 tokens per call).
//
// The routed-expert FFN of a DeepSeek-V4-Flash-style MoE layer
// ("DeepSeek-V4-Flash-W4A16-FP8", base-model table: hidden 4096, 256 routed
// experts, top-6) with MXFP4 / NVFP4 expert weights
// ("DeepSeek-v4-Flash-REAP-K180-NVFP4", "NVFP4: lossless MXFP4->NVFP4
// conversion"; gate+up carry ~2/3 of the expert bytes, "Why this mix?").
//
// Two kernels, chained with programmatic dependent launch:
//   k_gateup  h[p][n] = silu(gate_n . x_t) * (up_n . x_t)       for pair p = (t, s)
//   k_down    y[t][m] = sum_s w[t][s] * (down_m . h_p)          (fixed slot order)
//
// Work decomposition.  A "virtual expert" is an expert together with up to 8
// of its routed pairs (one m16n8k16 N-tile); experts with more pairs become
// several virtual experts.  A unit is one 16-row MMA tile of a virtual expert
// (k_gateup: 8 gate rows + the same 8 up rows; k_down: 16 down rows) over the
// full reduction length, cut into chunks of Kc.  The units of the call are
// split evenly over the CTAs (whole units), and each CTA's chunks evenly and
// contiguously over its warps, so every warp streams about the same number of
// bytes.  A unit cut by a warp boundary is summed in shared memory by the warp
// holding its first chunk, adding the pieces in chunk order (deterministic for
// a given grid).  k_down writes each unit's 16 x 8 result; k_decode_y, the
// next launch, forms y in fixed slot order.
//
// Data path.  Each warp streams its chunks through its own ring of shared-
// memory stages.  Packed rows arrive by tensor-map TMA as 3-D boxes of 8 or 16
// rows x Kc/2 bytes in the 128-byte-swizzled layout (16-byte chunk c of row r
// stored at c ^ (r & 7)), so ldmatrix reads them without bank conflicts; the
// matching scale-row slices arrive by cp.async; both complete on the stage's
// mbarrier.  (Shapes whose rows or scale slices are not 256 / 16-byte
// multiples fall back to one cp.async per 16 bytes into padded rows.)  A
// thread forms m16n8k16 A fragments with ldmatrix and the hardware
// e2m1x2 -> f16x2 conversion (exact) and multiplies on the tensor cores with
// f16 activations (fp32 accumulate):
//   MXFP4: the fp32 partial of each 32-block is scaled by 2^(c-127) (exact);
//   NVFP4: the e4m3 scale is folded into the f16 fragment (e2m1 * e4m3 is exact
//          in f16) and scale_2 is applied at the end.
// Activations are staged once per CTA segment as f16 rows scaled by a power of
// two per row, chosen so the row's largest magnitude sits in [2^14, 2^15); their
// loads are issued ahead of the weight stream.
#include <cuda.h>

#include <algorithm>

#include "qk_common.cuh"
#include "qk_route_table.cuh"
#include "qk_tmap.h"

namespace qk {

constexpr int kDW = 8;    // warps per CTA
constexpr int kXCap = 8;  // activation rows staged per segment
constexpr int kMaxD = 4;  // deepest ring per warp

// Routing tables: qk_route_table.cuh.


// ------------------------------------------------------------- geometry --
// Shared by host and device.  Per warp: D nibble stages (1024-byte aligned)
// and D scale stages; then the staged activation rows.
struct DGeo {
  int K, Kc;        // reduction length, chunk length
  int nk;           // chunks per unit
  int nbc;          // 32-blocks per chunk
  int tmap;         // 1: packed rows by tensor-map TMA (swizzled), 0: cp.async rows
  int nseg;         // 128-byte segments per packed chunk row
  int nib;          // padded bytes per packed smem row (row mode)
  int nib_stage;    // bytes of one stage's packed rows (1024-multiple)
  int sca, scb;     // scale bytes per chunk row, rows 0..7 / 8..15
  int sca_g, scb_g; // scale bytes per global row (full K)
  int sc_vec;       // bytes per scale cp.async (16 or 4)
  int sc_stage;     // bytes of one stage's scale rows (16-multiple)
  int act_stride;   // halves per staged activation row
  int xcap;         // staged activation rows
  int fast;         // every row of the call is staged once (rows <= xcap)
  int D;            // stages per warp
  int off_rings, off_scales, off_act;  // from the 1024-aligned base
  int off_raw;      // k_down, every pair row staged at once: the fp32 h rows as copied
  int raw;          // bytes of that area (0: h is read with plain loads)
  int smem;         // total dynamic shared memory (with alignment slack)
};

__host__ __device__ inline int sc_row_bytes(int fmt, int K) {
  return fmt == QK_FMT_MXFP4 ? K / 32 : K / 16;
}

struct DHead {
  Route R;
  int seg_u0, seg_u1, seg_v0, seg_rows;  // units [seg_u0, seg_u1) of the current segment
  int16_t row_key[kXCap];               // staged row -> token (k_gateup) or pair (k_down)
  int8_t col_row[kMaxPairs * kTileN];   // (v - seg_v0, column) -> staged row
  int shift[kXCap];
  int dead;                             // a warp's copies did not land in time
  int pu[kDW][2];                       // unit of the warp's first / last piece (-1: none)
  int pstart[kDW][2];                   // first chunk of that piece within its unit
  int wempty[kDW];                      // the warp has no chunk in this segment
  unsigned amax_bits[kXCap];            // row maxima (bit patterns of non-negative floats)
  float4 piece[kDW][2][32];             // partial sums of units cut by a warp boundary
  alignas(8) uint64_t full[kDW][kMaxD];
};
constexpr int kDHead = (int)((sizeof(DHead) + 127) / 128 * 128);

__host__ __device__ inline int up_to(int x, int a) { return (x + a - 1) / a * a; }

__host__ __device__ inline DGeo make_dgeo(int K, int Kc, int fa, int fb, int xcap, int D, bool tmap_ok,
                                          int raw = 0) {
  DGeo g;
  g.K = K;
  g.Kc = Kc;
  g.nk = K / Kc;
  g.nbc = Kc / 32;
  g.sca_g = sc_row_bytes(fa, K);
  g.scb_g = sc_row_bytes(fb, K);
  g.sca = sc_row_bytes(fa, Kc);
  g.scb = sc_row_bytes(fb, Kc);
  g.sc_vec = (g.sca % 16 || g.scb % 16 || g.sca_g % 16 || g.scb_g % 16) ? 4 : 16;
  g.tmap = (tmap_ok && K % 256 == 0 && Kc % 256 == 0) ? 1 : 0;
  g.nseg = Kc / 256;
  g.nib = Kc / 2 + 16;
  g.nib_stage = g.tmap ? 16 * (Kc / 2) : up_to(16 * g.nib, 1024);
  g.sc_stage = up_to(8 * g.sca + 8 * g.scb, 16);
  g.act_stride = K + 32;  // 2K+64 bytes: conflict-free 16-byte fragment loads
  g.xcap = xcap;
  g.fast = 0;
  g.D = D;
  g.off_rings = up_to(kDHead, 1024);
  g.off_scales = g.off_rings + kDW * D * g.nib_stage;
  g.off_act = up_to(g.off_scales + kDW * D * g.sc_stage, 16);
  // k_down stages h before its weight stream starts: the raw rows borrow the
  // rings when they fit there
  const bool in_rings = raw <= kDW * D * g.nib_stage;
  g.off_raw = in_rings ? g.off_rings : up_to(g.off_act + xcap * g.act_stride * 2, 16);
  g.raw = raw;
  g.smem = up_to(g.off_act + xcap * g.act_stride * 2, 16) + (in_rings ? 0 : raw) + 1024;  // + alignment slack
  return g;
}

struct DArgs {
  DecodeArgs a;
  DGeo G;
  int RT;          // units (row tiles) per virtual expert
  int U_max;       // upper bound of units (grid sizing only)
  alignas(64) CUtensorMap tqa, tqb;  // packed rows of the A / B projections (tensor-map mode)
};

// ---------------------------------------------------------- fragments --
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Four e8m0 codes -> fp32 2^(c-127) (code 0 -> the subnormal 2^-127 exactly).
__device__ __forceinline__ void ue8m0x4(uint32_t c4, float (&f)[4]) {
  uint32_t lo, hi;
  asm("{\n .reg .b16 a, b;\n mov.b32 {a, b}, %2;\n cvt.rn.bf16x2.ue8m0x2 %0, a;\n"
      " cvt.rn.bf16x2.ue8m0x2 %1, b;\n}\n"
      : "=r"(lo), "=r"(hi)
      : "r"(c4));
  f[0] = __uint_as_float(lo << 16);
  f[1] = __uint_as_float(lo & 0xFFFF0000u);
  f[2] = __uint_as_float(hi << 16);
  f[3] = __uint_as_float(hi & 0xFFFF0000u);
}

__device__ __forceinline__ bool has_ff_byte(uint32_t c4) {
  const uint32_t v = ~c4;
  return ((v - 0x01010101u) & c4 & 0x80808080u) != 0u;
}

// Scales of 4 consecutive 32-blocks for one fragment row.
template <int FMT>
struct Scale4;

template <>
struct Scale4<QK_FMT_MXFP4> {
  float f[4];
  __device__ __forceinline__ void load(const uint8_t* row, int b, int /*t*/, bool& bad) {
    const uint32_t c4 = *reinterpret_cast<const uint32_t*>(row + b);
    bad |= has_ff_byte(c4);
    ue8m0x4(c4, f);
  }
};

template <>
struct Scale4<QK_FMT_NVFP4> {
  uint32_t h2[4];  // f16x2 broadcast of this thread's 16-half scale, per block
  __device__ __forceinline__ void load(const uint8_t* row, int b, int t, bool& bad) {
    const uint2 c = *reinterpret_cast<const uint2*>(row + 2 * b);
    bad |= has_ff_byte(c.x | 0x80808080u) | has_ff_byte(c.y | 0x80808080u);
    // thread t holds elements 8t..8t+7 of each 32-block: 16-half number t>>1
    const uint32_t sel = (t >> 1) ? 0x3232u : 0x1010u;
    const uint32_t w[2] = {c.x, c.y};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t h = (i & 1) ? e4m3x2_to_f16x2<1>(w[i >> 1]) : e4m3x2_to_f16x2<0>(w[i >> 1]);
      h2[i] = __byte_perm(h, h, sel);
    }
  }
};

// One 32-block of the 16-row tile against one 8-column activation tile.
// wa: A word of rows g (tile rows 0..7), wb: rows g+8.  xb: the thread's
// 8 f16 activations of this block.  acc rows g -> acc[0..1], g+8 -> acc[2..3].
template <int FA, int FB>
__device__ __forceinline__ void block_mma(float (&acc)[4], uint32_t wa, uint32_t wb,
                                          const uint4& xb, const Scale4<FA>& sa,
                                          const Scale4<FB>& sb, int i) {
  uint32_t a0 = e2m1x2_to_f16x2<0>(wa), a1 = e2m1x2_to_f16x2<0>(wb);
  uint32_t a2 = e2m1x2_to_f16x2<1>(wa), a3 = e2m1x2_to_f16x2<1>(wb);
  uint32_t c0 = e2m1x2_to_f16x2<2>(wa), c1 = e2m1x2_to_f16x2<2>(wb);
  uint32_t c2 = e2m1x2_to_f16x2<3>(wa), c3 = e2m1x2_to_f16x2<3>(wb);
  if constexpr (FA == QK_FMT_NVFP4) {
    a0 = hmul2(a0, sa.h2[i]); a2 = hmul2(a2, sa.h2[i]);
    c0 = hmul2(c0, sa.h2[i]); c2 = hmul2(c2, sa.h2[i]);
  }
  if constexpr (FB == QK_FMT_NVFP4) {
    a1 = hmul2(a1, sb.h2[i]); a3 = hmul2(a3, sb.h2[i]);
    c1 = hmul2(c1, sb.h2[i]); c3 = hmul2(c3, sb.h2[i]);
  }
  if constexpr (FA == QK_FMT_NVFP4 && FB == QK_FMT_NVFP4) {
    mma_f16_16816(acc, a0, a1, a2, a3, xb.x, xb.y);
    mma_f16_16816(acc, c0, c1, c2, c3, xb.z, xb.w);
  } else {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    mma_f16_16816(d, a0, a1, a2, a3, xb.x, xb.y);
    mma_f16_16816(d, c0, c1, c2, c3, xb.z, xb.w);
    if constexpr (FA == QK_FMT_MXFP4) {
      acc[0] = fmaf(d[0], sa.f[i], acc[0]);
      acc[1] = fmaf(d[1], sa.f[i], acc[1]);
    } else {
      acc[0] += d[0];
      acc[1] += d[1];
    }
    if constexpr (FB == QK_FMT_MXFP4) {
      acc[2] = fmaf(d[2], sb.f[i], acc[2]);
      acc[3] = fmaf(d[3], sb.f[i], acc[3]);
    } else {
      acc[2] += d[2];
      acc[3] += d[3];
    }
  }
}

// One chunk of one unit (warp): 16 rows x Kc against one token tile.
// st: the stage's packed rows; sc: its scale rows; xrow: this thread's
// activation row at the chunk's first block.
template <int FA, int FB, bool GATEUP>
__device__ __forceinline__ void chunk_mma(float (&acc)[4], const uint8_t* st, const uint8_t* sc,
                                          const DGeo& G, const __half* xrow, int lane, bool& bad) {
  const int g = lane >> 2, t = lane & 3;
  const int mj = lane >> 3, mr = lane & 7;
  // ldmatrix: lane supplies row r = (mj&1)*8 + mr of block b + (mj>>1)
  const int r = (mj & 1) * 8 + mr;
  constexpr int RB = GATEUP ? 8 : 16;  // rows per TMA box
  const uint8_t* lbase = G.tmap ? st + (r / RB) * (RB * 128 * G.nseg) + (r % RB) * 128
                                : st + r * G.nib;
  const uint8_t* sa = sc + g * G.sca;
  const uint8_t* sb = sc + 8 * G.sca + g * G.scb;
  auto laddr = [&](int bb) -> const uint8_t* {
    return G.tmap ? lbase + (bb >> 3) * (RB * 128) + (((bb & 7) ^ mr) << 4) : lbase + bb * 16;
  };
#pragma unroll 2
  for (int b = 0; b < G.nbc; b += 4) {
    uint32_t w[8];
    ldmatrix_x4(w[0], w[1], w[2], w[3], laddr(b + (mj >> 1)));
    ldmatrix_x4(w[4], w[5], w[6], w[7], laddr(b + 2 + (mj >> 1)));
    Scale4<FA> s_a;
    Scale4<FB> s_b;
    s_a.load(sa, b, t, bad);
    s_b.load(sb, b, t, bad);
    const uint4 x0 = *reinterpret_cast<const uint4*>(xrow + (b + 0) * 32);
    const uint4 x1 = *reinterpret_cast<const uint4*>(xrow + (b + 1) * 32);
    const uint4 x2 = *reinterpret_cast<const uint4*>(xrow + (b + 2) * 32);
    const uint4 x3 = *reinterpret_cast<const uint4*>(xrow + (b + 3) * 32);
    block_mma<FA, FB>(acc, w[0], w[1], x0, s_a, s_b, 0);
    block_mma<FA, FB>(acc, w[2], w[3], x1, s_a, s_b, 1);
    block_mma<FA, FB>(acc, w[4], w[5], x2, s_a, s_b, 2);
    block_mma<FA, FB>(acc, w[6], w[7], x3, s_a, s_b, 3);
  }
}

// Release the writes of this thread (and, through the preceding warp barrier,
// of its warp) and acquire those of earlier arrivals.
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// cp.async global -> shared (L2 only), 16 bytes with an L2 evict-first hint, or 4 bytes.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)),
               "l"(src), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
// The mbarrier receives one (pre-counted) arrival once this thread's earlier
// cp.asyncs land.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ------------------------------------------------------------- staging --
// The segment's activation rows are staged as f16 scaled by 2^-shift[row], the
// shift putting the row's largest magnitude in [2^14, 2^15):
//   k_gateup: token rows of x (bf16 [T][H]) are copied raw into the staging
//     area by cp.async (issued before the weight stream), then converted in
//     place once the row maxima are known;
//   k_down: pair rows of h (fp32 [P][I]); the row maxima come from k_gateup's
//     per-tile maxima.
// The loops stay rolled: they run once per segment, and compact code keeps the
// cold start of the block short.  With `ident`, row i is token / pair i (every
// row of the call staged; row_key is not read).
__device__ __forceinline__ void cp_async16_nohint(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ float bf16x8_absmax(const uint4& v) {
  const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32(wv[e] & 0xFFFFu)), fabsf(bf16_bits_to_f32(wv[e] >> 16))));
  return m;
}

// Max of m into the row's slot; `row` is warp-uniform when `uniform`.
__device__ __forceinline__ void row_max(DHead& S, int row, float m, bool uniform) {
  if (uniform) {
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(&S.amax_bits[row], __float_as_uint(m));
  } else {
    atomicMax(&S.amax_bits[row], __float_as_uint(m));
  }
}

// Shifts from the row maxima (non-negative floats order like their bit patterns).
__device__ __forceinline__ void rows_shift(DHead& S, int nrows) {
  __syncthreads();
  if (threadIdx.x < nrows) S.shift[threadIdx.x] = clamp_shift(f16_shift_for(__uint_as_float(S.amax_bits[threadIdx.x])));
  __syncthreads();
}

__device__ __forceinline__ void stage_x_issue(const DecodeArgs& a, const DHead& S, __half* act, int stride,
                                              int nrows, bool ident) {
  const int nvec = a.H / 8;
  for (int j = threadIdx.x; j < nrows * nvec; j += kDW * 32) {
    const int row = j / nvec, q = j - row * nvec;
    const int key = ident ? row : S.row_key[row];
    cp_async16_nohint(act + (size_t)row * stride + q * 8, a.x + (size_t)key * a.H + q * 8);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void stage_x_finish(const DecodeArgs& a, DHead& S, __half* act, int stride,
                                               int nrows) {
  const int nvec = a.H / 8;
  const bool uniform = nvec % 32 == 0;  // a warp's 32 vectors lie in one row
  if (threadIdx.x < kXCap) S.amax_bits[threadIdx.x] = 0u;
  asm volatile("cp.async.wait_group 0;" ::: "memory");  // the x group only: ring copies are not grouped
  __syncthreads();
  for (int j = threadIdx.x; j < nrows * nvec; j += kDW * 32) {
    const int row = j / nvec, q = j - row * nvec;
    row_max(S, row, bf16x8_absmax(*reinterpret_cast<const uint4*>(act + (size_t)row * stride + q * 8)), uniform);
  }
  rows_shift(S, nrows);
  for (int j = threadIdx.x; j < nrows * nvec; j += kDW * 32) {  // bf16 -> f16 in place
    const int row = j / nvec, q = j - row * nvec;
    uint4* pv = reinterpret_cast<uint4*>(act + (size_t)row * stride + q * 8);
    const uint4 v = *pv;
    const float sc = pow2f(-S.shift[row]);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = pack_f16x2(bf16_bits_to_f32(wv[e] & 0xFFFFu) * sc, bf16_bits_to_f32(wv[e] >> 16) * sc);
    *pv = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

__device__ __forceinline__ void stage_h(const DecodeArgs& a, DHead& S, __half* act, int stride, int nrows,
                                        bool ident) {
  const int R1 = a.I / 8;  // maxima per pair row
  if (threadIdx.x < kXCap) S.amax_bits[threadIdx.x] = 0u;
  __syncthreads();
  for (int j = threadIdx.x; j < nrows * R1; j += kDW * 32) {
    const int row = j / R1;
    const int key = ident ? row : S.row_key[row];
    row_max(S, row, __ldcg(a.hmax + (size_t)key * R1 + (j - row * R1)), R1 % 32 == 0);
  }
  rows_shift(S, nrows);
  const int nvec = a.I / 4;
#pragma unroll 4
  for (int j = threadIdx.x; j < nrows * nvec; j += kDW * 32) {
    const int row = j / nvec, q = j - row * nvec;
    const int key = ident ? row : S.row_key[row];
    const float4 v = __ldcg(reinterpret_cast<const float4*>(a.h + (size_t)key * a.I) + q);
    const float sc = pow2f(-S.shift[row]);
    reinterpret_cast<uint2*>(act + (size_t)row * stride)[q] =
        make_uint2(pack_f16x2(v.x * sc, v.y * sc), pack_f16x2(v.z * sc, v.w * sc));
  }
}

// Every pair row at once (pairs 0 .. nrows-1, contiguous in h): one round of
// cp.async into the raw area, then maxima and conversion from shared memory.
__device__ __forceinline__ void stage_h_raw(const DecodeArgs& a, DHead& S, __half* act, int stride, int nrows,
                                            float* raw) {
  const int nvec = a.I / 4;
  const int total = nrows * nvec;
  for (int j = threadIdx.x; j < total; j += kDW * 32) cp_async16_nohint(raw + 4 * j, a.h + 4 * j);
  asm volatile("cp.async.commit_group;" ::: "memory");
  if (threadIdx.x < kXCap) S.amax_bits[threadIdx.x] = 0u;
  asm volatile("cp.async.wait_group 0;" ::: "memory");  // the h group only: ring copies come later
  __syncthreads();
  const bool uniform = nvec % 32 == 0;  // a warp's 32 vectors lie in one row
  for (int j = threadIdx.x; j < total; j += kDW * 32) {
    const float4 v = *reinterpret_cast<const float4*>(raw + 4 * j);
    row_max(S, j / nvec, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))), uniform);
  }
  rows_shift(S, nrows);
  for (int j = threadIdx.x; j < total; j += kDW * 32) {
    const int row = j / nvec, q = j - row * nvec;
    const float4 v = *reinterpret_cast<const float4*>(raw + 4 * j);
    const float sc = pow2f(-S.shift[row]);
    reinterpret_cast<uint2*>(act + (size_t)row * stride)[q] =
        make_uint2(pack_f16x2(v.x * sc, v.y * sc), pack_f16x2(v.z * sc, v.w * sc));
  }
  // the raw area may be the rings: order these accesses before the copies into them
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ the kernel --
// Unit u = v * RT + r; chunk c = u * nk + kc.
// Every warp fills its own ring: its lanes cp.async the chunk's scale slices
// (and, in row mode, its packed rows) and lane 0 issues the tensor-map copies
// of the packed rows.  A stage's mbarrier completes on 33 arrivals (one
// deferred arrival per lane once its cp.asyncs land, plus lane 0's
// expect-tx arrival) and the TMA bytes.  Issuing from every warp keeps the
// per-instruction cost of a tensor copy off any single warp's critical path.
template <int FA, int FB, bool GATEUP>
__global__ void __launch_bounds__(kDW * 32, 1) k_decode(const __grid_constant__ DArgs P) {
  extern __shared__ __align__(16) uint8_t smem_raw[];  // rounded up to 1024 below, at run time
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  DHead& S = *reinterpret_cast<DHead*>(smem);
  const DecodeArgs& a = P.a;
  const DGeo& G = P.G;
  __half* act = reinterpret_cast<__half*>(smem + G.off_act);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  uint8_t* nring = smem + G.off_rings + (size_t)warp * G.D * G.nib_stage;
  uint8_t* sring = smem + G.off_scales + (size_t)warp * G.D * G.sc_stage;
  uint64_t* full = S.full[warp];
  const int RT = P.RT, nk = G.nk;
  const qk_weight& WA = GATEUP ? a.gate : a.down;
  const qk_weight& WB = GATEUP ? a.up : a.down;
  const int rows_per_e = GATEUP ? a.I : a.H;  // weight rows of one expert
  const bool fast = G.fast != 0;

  pdl_launch_dependents();  // the next kernel (k_down, then k_decode_y) may start its prologue
  if (lane == 0) {
    for (int i = 0; i < G.D; ++i) mbar_init(&full[i], 33);
    fence_mbar_init();
    if (G.tmap && warp == 0) {
      tmap_prefetch(&P.tqa);
      if (GATEUP) tmap_prefetch(&P.tqb);
    }
  }
  if (threadIdx.x == 0) S.dead = 0;
  if (GATEUP && fast) stage_x_issue(a, S, act, G.act_stride, a.T, true);  // x does not depend on the routing
  // k_gateup may start while the router that writes ids and w is finishing
  // (programmatic dependent launch): wait for it before reading them
  if (GATEUP) pdl_wait();
  build_route(a.ids, a.P, a.E, S.R);  // ends with a block barrier
  const int n_v = S.R.n_v;
  const int U = n_v * RT;
  const int u_beg = (int)((int64_t)U * blockIdx.x / gridDim.x);
  const int u_end = (int)((int64_t)U * (blockIdx.x + 1) / gridDim.x);
  if (u_beg >= u_end) return;
  if (fast) {  // one segment: every virtual expert, rows = all tokens / pairs
    for (int i = threadIdx.x; i < n_v * kTileN; i += blockDim.x) {
      const int v = i / kTileN, j = i - v * kTileN;
      if (j < S.R.v_n[v]) {
        const int pr = S.R.pair_list[S.R.v_p0[v] + j];
        S.col_row[i] = (int8_t)(GATEUP ? pr / a.k : pr);
      }
    }
    if (threadIdx.x < kXCap) S.row_key[threadIdx.x] = (int16_t)threadIdx.x;
  }

  const uint64_t pol = policy_evict_first();
  const unsigned long long limit = g_wait_limit_ns;
  const int vpr = G.Kc / 32;  // 16-byte vectors per packed chunk row
  // Chunk c into stage `slot`.
  // This lane's scale pieces of a chunk (the same for every chunk): source
  // offsets from the A / B scale slice, destination offsets in the stage.
  constexpr int kMaxPc = 4;
  int pc_src[kMaxPc], pc_dst[kMaxPc];
  bool pc_b[kMaxPc];
  int npc = 0;
  {
    const int pa = G.sca / G.sc_vec, pb = G.scb / G.sc_vec;  // pieces per row
    for (int idx = lane; idx < 8 * (pa + pb) && npc < kMaxPc; idx += 32, ++npc) {
      const bool isb = idx >= 8 * pa;
      const int k2 = isb ? idx - 8 * pa : idx;
      const int pr = isb ? pb : pa;
      const int row = k2 / pr, pc = k2 - row * pr;
      pc_b[npc] = isb;
      pc_src[npc] = row * (isb ? G.scb_g : G.sca_g) + pc * G.sc_vec;
      pc_dst[npc] = (isb ? 8 * G.sca + row * G.scb : row * G.sca) + pc * G.sc_vec;
    }
  }
  // Unit order: expert-major (u = v * RT + r).
  auto unit_vr = [&](int u, int& v, int& r) {
    v = u / RT;
    r = u - v * RT;
  };
  // Position of a chunk: unit u (expert slot v, row tile r), chunk kc of the unit.
  struct Cur {
    int u, kc, v, r;
  };
  auto cur_at = [&](int c) -> Cur {
    Cur q;
    q.u = c / nk;
    q.kc = c - q.u * nk;
    unit_vr(q.u, q.v, q.r);
    return q;
  };
  auto cur_next = [&](Cur& q) {
    if (++q.kc == nk) {
      q.kc = 0;
      ++q.u;
      if (++q.r == RT) {
        q.r = 0;
        ++q.v;
      }
    }
  };
  auto issue = [&](const Cur& q, int slot) {
    uint8_t* st = nring + (size_t)slot * G.nib_stage;
    uint8_t* sd = sring + (size_t)slot * G.sc_stage;
    uint64_t* bar = &full[slot];
    const int kc = q.kc, r = q.r;
    const int e = S.R.v_expert[q.v];
    const int64_t rowA0 = (int64_t)e * rows_per_e + (GATEUP ? r * 8 : r * 16);
    const int64_t rowB0 = GATEUP ? rowA0 : rowA0 + 8;
    if (!G.tmap) {
      const uint8_t* qa = WA.q + rowA0 * (G.K / 2) + (size_t)kc * (G.Kc / 2);
      const uint8_t* qb = WB.q + rowB0 * (G.K / 2) + (size_t)kc * (G.Kc / 2);
      for (int idx = lane; idx < 16 * vpr; idx += 32) {
        const int row = idx / vpr, vi = idx - row * vpr;
        const uint8_t* src =
            (row < 8 ? qa + (size_t)row * (G.K / 2) : qb + (size_t)(row - 8) * (G.K / 2)) + vi * 16;
        cp_async16(st + row * G.nib + vi * 16, src, pol);
      }
    }
    const uint8_t* sa = WA.scales + rowA0 * G.sca_g + (size_t)kc * G.sca;
    const uint8_t* sb = WB.scales + rowB0 * G.scb_g + (size_t)kc * G.scb;
#pragma unroll
    for (int q2 = 0; q2 < kMaxPc; ++q2) {
      if (q2 >= npc) break;
      const uint8_t* src = (pc_b[q2] ? sb : sa) + pc_src[q2];
      uint8_t* dst = sd + pc_dst[q2];
      if (G.sc_vec == 16) cp_async16(dst, src, pol);
      else cp_async4(dst, src);
    }
    cp_async_arrive(bar);
    if (lane == 0) {
      if (G.tmap) {
        mbar_arrive_expect_tx(bar, 16u * (uint32_t)(G.Kc / 2));
        const int z = kc * G.nseg;
        if (GATEUP) {
          tma_load_3d(st, &P.tqa, 0, (int)rowA0, z, bar, pol);
          tma_load_3d(st + 8 * (G.Kc / 2), &P.tqb, 0, (int)rowB0, z, bar, pol);
        } else {
          tma_load_3d(st, &P.tqa, 0, (int)rowA0, z, bar, pol);
        }
      } else {
        mbar_arrive_expect_tx(bar, 0u);
      }
    }
  };

  // A finished unit: scale, then SwiGLU into h (k_gateup) or the unit result (k_down).
  auto finalize = [&](int u, float4 f, int seg_v0) {
    int v, r;
    unit_vr(u, v, r);
    const int e = S.R.v_expert[v], n = S.R.v_n[v];
    const float s2a = WA.fmt == QK_FMT_NVFP4 ? WA.scale_2[e] : 1.f;
    const float s2b = WB.fmt == QK_FMT_NVFP4 ? WB.scale_2[e] : 1.f;
    float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const int col = 2 * t + jj;
      const float sx = col < n ? pow2f(S.shift[S.col_row[(v - seg_v0) * kTileN + col]]) : 0.f;
      fv[jj] *= sx * s2a;
      fv[2 + jj] *= sx * s2b;
    }
    if (GATEUP) {
      float hm[2];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int col = 2 * t + jj;
        hm[jj] = 0.f;
        if (col < n) {
          const float hv = silu_mul(fv[jj], fv[2 + jj]);
          if (!finite_bits(hv)) set_status(QK_ERR_NONFINITE);
          const int p = S.R.pair_list[S.R.v_p0[v] + col];
          a.h[(size_t)p * a.I + r * 8 + g] = hv;
          hm[jj] = fabsf(hv);
        }
      }
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) hm[jj] = fmaxf(hm[jj], __shfl_xor_sync(0xffffffffu, hm[jj], o));
      if (g == 0) {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int col = 2 * t + jj;
          if (col < n) a.hmax[(size_t)S.R.pair_list[S.R.v_p0[v] + col] * (a.I / 8) + r] = hm[jj];
        }
      }
    } else {
      // stored expert-major whatever the processing order (the combine reads v * RT + r)
      reinterpret_cast<float4*>(a.ures)[((size_t)v * RT + r) * 32 + lane] = make_float4(fv[0], fv[1], fv[2], fv[3]);
    }
  };

  int done = 0;  // chunks consumed by this warp (ring position)
  bool dead = false, bad = false;
  bool waited_pdl = false;
  int u_seg = u_beg;
  while (u_seg < u_end) {
    // ---- plan a segment: consecutive virtual experts whose rows fit xcap
    if (fast) {
      if (threadIdx.x == 0) {
        S.seg_u0 = u_beg;
        S.seg_u1 = u_end;
        S.seg_v0 = 0;
        S.seg_rows = GATEUP ? a.T : a.P;
      }
    } else if (threadIdx.x == 0) {
      const int v0 = u_seg / RT;
      const int vlast = (u_end - 1) / RT;
      int rows = 0, v = v0;
      for (; v <= vlast; ++v) {
        const int n = S.R.v_n[v];
        int add = 0;
        bool fits = true;
        int8_t cr[kTileN];
        for (int j = 0; j < n && fits; ++j) {
          const int pr = S.R.pair_list[S.R.v_p0[v] + j];
          const int key = GATEUP ? pr / a.k : pr;
          int found = -1;
          for (int i = 0; i < rows + add; ++i)
            if (S.row_key[i] == key) found = i;
          if (found < 0) {
            if (rows + add >= G.xcap) {
              fits = false;
            } else {
              S.row_key[rows + add] = (int16_t)key;
              found = rows + add;
              ++add;
            }
          }
          cr[j] = (int8_t)found;
        }
        if (!fits) break;  // v starts the next segment
        for (int j = 0; j < n; ++j) S.col_row[(v - v0) * kTileN + j] = cr[j];
        rows += add;
      }
      S.seg_u0 = u_seg;
      S.seg_u1 = min(u_end, v * RT);  // v > v0 always (one virtual expert has <= xcap rows)
      S.seg_v0 = v0;
      S.seg_rows = rows;
    }
    __syncthreads();
    const int seg_u0 = S.seg_u0, seg_u1 = S.seg_u1, seg_v0 = S.seg_v0, seg_rows = S.seg_rows;
    if (seg_u1 <= seg_u0) {  // cannot happen; never loop forever
      set_status(QK_ERR_INVALID_ARG);
      break;
    }
    const int cs = seg_u0 * nk, n_seg = (seg_u1 - seg_u0) * nk;
    const int w0 = cs + (int)((int64_t)n_seg * warp / kDW);
    const int w1 = cs + (int)((int64_t)n_seg * (warp + 1) / kDW);
    const int wn = w1 - w0;
    if (lane == 0) {
      S.pu[warp][0] = S.pu[warp][1] = -1;
      S.wempty[warp] = wn == 0;
    }

    // ---- k_gateup: x copies (their own cp.async group), weight prefetch (D-1
    // chunks), then the conversion of x.  k_down: h first (it is in L2 and must
    // not queue behind the weight stream), then the weight prefetch.
    // issue cursor (chunk w0 + issued) and ring slots of issue and consumption
    Cur icur = cur_at(w0);
    int islot = done % G.D;
    int issued = 0;
    auto issue_next = [&]() {
      issue(icur, islot);
      cur_next(icur);
      if (++islot == G.D) islot = 0;
      ++issued;
    };
    if (GATEUP) {
      if (!fast) stage_x_issue(a, S, act, G.act_stride, seg_rows, false);
      for (int i = 0; i < G.D - 1 && i < wn; ++i) issue_next();
      stage_x_finish(a, S, act, G.act_stride, seg_rows);
    } else {
      if (!waited_pdl) {
        pdl_wait();  // h and hmax come from k_gateup
        waited_pdl = true;
      }
      if (fast && G.raw) stage_h_raw(a, S, act, G.act_stride, seg_rows, reinterpret_cast<float*>(smem + G.off_raw));
      else stage_h(a, S, act, G.act_stride, seg_rows, fast);
      for (int i = 0; i < G.D - 1 && i < wn; ++i) issue_next();
    }
    __syncthreads();

    // ---- stream this warp's chunks
    int cur_u = -1, kc_start = 0, kc_last = 0, npieces = 0;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    auto close = [&]() {
      const float4 f = make_float4(acc[0], acc[1], acc[2], acc[3]);
      if (kc_start == 0 && kc_last == nk - 1) {
        finalize(cur_u, f, seg_v0);
      } else {  // cut by a warp boundary: the first or the last unit of this warp
        const int sl = npieces++;
        S.piece[warp][sl][lane] = f;
        if (lane == 0) {
          S.pu[warp][sl] = cur_u;
          S.pstart[warp][sl] = kc_start;
        }
      }
    };
    Cur ccur = cur_at(w0);  // consumption cursor
    int slot = done % G.D;
    uint32_t phase = (uint32_t)((done / G.D) & 1);
    for (int i = 0; i < wn; ++i) {
      // keep D-1 chunks in flight: issue chunk i+D-1, then wait for chunk i
      if (issued < wn) issue_next();
      const bool landed = mbar_wait_bounded(&full[slot], phase, limit);
      if (__any_sync(0xffffffffu, !landed)) {
        // the copies did not land in time: report, drain what this warp has in
        // flight, and stop the block at the end of the segment
        set_status(QK_ERR_TIMEOUT);
        const int inflight = min(wn - i, G.D);
        for (int q = 0; q < inflight; ++q)
          if (!mbar_wait_bounded(&full[(done + q) % G.D], (uint32_t)(((done + q) / G.D) & 1),
                                 kDrainLimitNs))
            break;
        dead = true;
        break;
      }
      const int u = ccur.u, kc = ccur.kc, v = ccur.v;
      if (u != cur_u) {
        if (cur_u >= 0) close();
        cur_u = u;
        kc_start = kc;
        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
      }
      kc_last = kc;
      const int n = S.R.v_n[v];
      const int row = S.col_row[(v - seg_v0) * kTileN + (g < n ? g : 0)];
      const __half* xrow = act + (size_t)row * G.act_stride + 8 * t + (size_t)kc * G.Kc;
      chunk_mma<FA, FB, GATEUP>(acc, nring + (size_t)slot * G.nib_stage, sring + (size_t)slot * G.sc_stage,
                                G, xrow, lane, bad);
      ++done;
      cur_next(ccur);
      if (++slot == G.D) {
        slot = 0;
        phase ^= 1u;
      }
      __syncwarp();  // every lane is done with this stage before it is refilled
    }
    if (dead) {
      if (lane == 0) S.dead = 1;
    } else if (cur_u >= 0) {
      close();
    }
    __syncthreads();
    if (S.dead) break;
    // ---- units cut by warp boundaries: the warp holding the first chunk adds
    // the pieces in chunk order
    for (int sl = 0; sl < 2; ++sl) {
      const int u = S.pu[warp][sl];
      if (u < 0 || S.pstart[warp][sl] != 0) continue;
      float4 f = S.piece[warp][sl][lane];
      for (int w2 = warp + 1; w2 < kDW; ++w2) {
        if (S.wempty[w2]) continue;
        if (S.pu[w2][0] != u) break;
        const float4 q = S.piece[w2][0][lane];
        f.x += q.x; f.y += q.y; f.z += q.z; f.w += q.w;
      }
      finalize(u, f, seg_v0);
    }
    __syncthreads();  // the next segment reuses the staged rows and the pieces
    u_seg = seg_u1;
  }
  if (bad) set_status(QK_ERR_NAN_SCALE);
}

// y[t][m] = sum over slots s in order of w[t][s] * (the k_down unit result of
// pair (t, s) for row m): one thread per output, the loads of up to 8 slots in
// flight together.  Launched after k_down (programmatic dependent launch): the
// routing table is built while k_down runs; griddepcontrol.wait returns when
// the unit results are complete and visible.
__global__ void __launch_bounds__(256) k_decode_y(const __grid_constant__ DecodeArgs a) {
  __shared__ Route R;
  build_route(a.ids, a.P, a.E, R);  // ends with __syncthreads
  pdl_wait();
  const int RT = a.H / 16;
  const float* ures = a.ures;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < a.T * a.H; idx += gridDim.x * blockDim.x) {
    const int tok = idx / a.H, row = idx - tok * a.H, r = row >> 4, m = row & 15;
    const int ln = (m & 7) * 4, el = (m >= 8) ? 2 : 0;
    float d[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      d[s] = 0.f;
      if (s < a.k) {
        const int p = tok * a.k + s;
        const int pv = R.pair_v[p];
        if (pv >= 0) {
          const int j = R.pair_j[p];
          d[s] = __ldcg(ures + (((size_t)pv * RT + r) * 32 + ln + (j >> 1)) * 4 + el + (j & 1));
        }
      }
    }
    float yv = 0.f;
#pragma unroll
    for (int s = 0; s < 8; ++s)
      if (s < a.k) yv = fmaf(__ldg(a.w + tok * a.k + s), d[s], yv);
    if (!finite_bits(yv)) set_status(QK_ERR_NONFINITE);
    if (a.y_bf16) reinterpret_cast<__nv_bfloat16*>(a.y)[idx] = __float2bfloat16_rn(yv);
    else reinterpret_cast<float*>(a.y)[idx] = yv;
  }
}

// ================================================================= host ==
// Largest chunk (<= 1024, dividing K, >= 128) whose rings of at least 3 stages
// per warp fit in shared memory (else 2 stages), ring depth up to kMaxD.
static DGeo plan_geo(int K, int fa, int fb, int xcap, bool tmap_ok, int raw) {
  const int cap = max_smem_optin();
  DGeo two = make_dgeo(K, 128, fa, fb, xcap, 2, tmap_ok, raw);
  two.smem = 0;
  for (int Kc = 1024; Kc >= 128; Kc >>= 1) {
    if (K % Kc) continue;
    for (int D = kMaxD; D >= 2; --D) {
      const DGeo g = make_dgeo(K, Kc, fa, fb, xcap, D, tmap_ok, raw);
      if (g.smem > cap) continue;
      if (D >= 3) return g;
      if (!two.smem) two = g;
      break;
    }
  }
  return two;
}

// Packed rows [rows][K/2] bytes as a 3-D map of 4-byte words:
// {32 words of a 128-byte segment, row, segment}, boxes of `box_rows` rows x
// `nseg` segments, 128-byte swizzle.
static bool encode_rows(CUtensorMap* m, const uint8_t* q, int64_t rows, int K, int box_rows, int nseg) {
  const uint64_t dims[3] = {32, (uint64_t)rows, (uint64_t)(K / 256)};
  const uint64_t strides[2] = {(uint64_t)K / 2, 128};
  const uint32_t box[3] = {32, (uint32_t)box_rows, (uint32_t)nseg};
  return tmap_get(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, q, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int FA, int FB, bool GATEUP>
static qk_status go(DArgs& P, cudaStream_t st, bool pdl) {
  const int grid = std::max(1, std::min(num_sms(), P.U_max));
  return launch_ex(k_decode<FA, FB, GATEUP>, dim3(grid), dim3(kDW * 32), (size_t)P.G.smem, st, pdl, P);
}

// Geometry of one kernel: tensor-map mode when the maps encode, else rows by cp.async.
static DGeo plan_kernel(int K, int fa, int fb, int rows, CUtensorMap* ta, CUtensorMap* tb,
                        const uint8_t* qa, const uint8_t* qb, int64_t n_rows, int box_rows, bool raw_h) {
  const int xcap = std::min(rows, kXCap);
  // k_down with every pair row staged at once copies h raw (fp32) first, when it fits
  const int raw = raw_h && rows <= kXCap ? rows * K * 4 : 0;
  DGeo G = plan_geo(K, fa, fb, xcap, true, raw);
  if (!G.smem && raw) G = plan_geo(K, fa, fb, xcap, true, 0);
  const int raw_used = G.raw;
  if (G.smem && G.tmap) {
    bool ok = encode_rows(ta, qa, n_rows, K, box_rows, G.nseg);
    if (ok && tb) ok = encode_rows(tb, qb, n_rows, K, box_rows, G.nseg);
    if (!ok) G = plan_geo(K, fa, fb, xcap, false, raw_used);
  }
  G.fast = rows <= kXCap ? 1 : 0;
  return G;
}

qk_status decode_forward(DecodeArgs args, cudaStream_t st) {
  DArgs P1 = {};
  P1.a = args;
  P1.RT = args.I / 8;
  P1.G = plan_kernel(args.H, args.gate.fmt, args.up.fmt, args.T, &P1.tqa, &P1.tqb, args.gate.q,
                     args.up.q, (int64_t)args.E * args.I, 8, false);
  if (!P1.G.smem) return QK_ERR_UNSUPPORTED;
  P1.U_max = args.P * P1.RT;  // virtual experts <= pairs
  DArgs P2 = {};
  P2.a = args;
  P2.RT = args.H / 16;
  P2.G = plan_kernel(args.I, args.down.fmt, args.down.fmt, args.P, &P2.tqa, nullptr, args.down.q,
                     nullptr, (int64_t)args.E * args.H, 16, true);
  if (!P2.G.smem) return QK_ERR_UNSUPPORTED;
  P2.U_max = args.P * P2.RT;
  constexpr int MX = QK_FMT_MXFP4, NV = QK_FMT_NVFP4;
  const int fg = args.gate.fmt, fu = args.up.fmt, fd = args.down.fmt;
  qk_status rc;
  // k_gateup overlaps its prologue with the end of the previous kernel only
  // when that kernel allows it (the router does); otherwise it waits as usual
  if (fg == MX && fu == MX) rc = go<MX, MX, true>(P1, st, true);
  else if (fg == MX) rc = go<MX, NV, true>(P1, st, true);
  else if (fu == MX) rc = go<NV, MX, true>(P1, st, true);
  else rc = go<NV, NV, true>(P1, st, true);
  if (rc != QK_OK) return rc;
  rc = fd == MX ? go<MX, MX, false>(P2, st, true) : go<NV, NV, false>(P2, st, true);
  if (rc != QK_OK) return rc;
  const int grid = std::max(1, std::min(2 * num_sms(), (args.T * args.H + 255) / 256));
  return launch_ex(k_decode_y, dim3(grid), dim3(256), 0, st, true, args);
}

// Workspace: h [P][I] f32 | hmax [P][I/8] | ures [P*H/16][32] float4.
struct WsLayout {
  size_t h, hmax, ures, total;
};

static WsLayout ws_layout(int T, int k, int H, int I) {
  const size_t P = (size_t)T * k;
  WsLayout L;
  size_t o = 0;
  L.h = o; o += align256(P * I * 4);
  L.hmax = o; o += align256(P * (I / 8) * 4);
  L.ures = o; o += align256(P * (H / 16) * 512);
  L.total = o;
  return L;
}

size_t decode_workspace_bytes(int T, int k, int H, int I) { return ws_layout(T, k, H, I).total; }

void decode_carve(DecodeArgs& a, void* ws) {
  const WsLayout L = ws_layout(a.T, a.k, a.H, a.I);
  uint8_t* p = static_cast<uint8_t*>(ws);
  a.h = reinterpret_cast<float*>(p + L.h);
  a.hmax = reinterpret_cast<float*>(p + L.hmax);
  a.ures = reinterpret_cast<float*>(p + L.ures);
}

}  // namespace qk
