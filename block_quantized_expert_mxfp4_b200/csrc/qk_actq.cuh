// Activation-quantized modes of moe_expert_forward (QK_ACT_E4M3, QK_ACT_MXFP4).
//
// "DeepSeekv4 Flash for 1x Spark [REAP25]", v0.2.3 update: the routed MXFP4
// experts run fp4 weights x dynamic E4M3 activations on block-scaled f8f6f4
// tensor cores, the numerics the model's own config names.  The block-scaled
// MMA takes one e8m0 scale per 32 activations; the scale rule (the pages give
// none) is the OCP Microscaling v1.0 one: X = floor(log2 amax) - emax with
// emax = 8 (e4m3) or 2 (e2m1), scale code X + 127 clamped to [0, 254] (0 for
// an all-zero block), elements rounded to nearest even and saturated.
//
// Each activation is then ONE term in the grouped path's token tiles,
// instead of the two or three exact e4m3 terms of QK_ACT_NONE, so a tile
// holds 128 tokens (gmx_tok1/gmx_tok2 give the tile heights per mode).
// QK_ACT_E4M3 feeds e4m3 codes (one byte each) to kind::mxf8f6f4 against the
// e2m1 weights; QK_ACT_MXFP4 packs two e2m1 codes per byte (element 2 i in
// the low nibble of byte i, the weights' own packing) and runs kind::mxf4
// with both operands as stored, 64 elements of K per instruction.
//
// The arithmetic below is host and device code: a CPU test compiles it for
// the host (QK_ACTQ_ARITHMETIC_ONLY: without the path declarations at the end)
// and checks it bit for bit against the oracle's quantizer.
#pragma once
#include <cuda_fp8.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef __CUDACC__
#define QK_HD __host__ __device__ __forceinline__
#else
#define QK_HD inline
#endif

namespace qk {

QK_HD uint32_t actq_bits(float f) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(f);
#else
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
#endif
}

QK_HD float actq_float(uint32_t u) {
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float f;
  memcpy(&f, &u, 4);
  return f;
#endif
}

// emax of the element format of a mode: 8 for e4m3 (448 = 1.75 * 2^8), 2 for
// e2m1 (6 = 1.5 * 2^2).
QK_HD int actq_emax(int fp4) { return fp4 ? 2 : 8; }

// e8m0 code of a block whose largest magnitude is m (finite, >= 0).  The
// biased exponent field of m is floor(log2 m) + 127 for a normal m; zero and
// fp32 subnormals (floor(log2 m) < -126) clamp to code 0.
QK_HD int actq_scale_code(float m, int emax) {
  const int ef = (int)((actq_bits(m) >> 23) & 0xFFu);
  const int c = ef - emax;
  return ef == 0 || c < 0 ? 0 : (c > 254 ? 254 : c);
}

// 2^(127 - c) for a code from actq_scale_code (c <= 252, so a normal float).
QK_HD float actq_up(int c) { return actq_float((uint32_t)(254 - c) << 23); }

// Nearest value of the e2m1 grid {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the even
// code, saturating at 6.  Within each range the grid step is fixed (0.5 below
// 2, then 1, then 2), so rint of the value over the step is the RNE choice
// and an even quotient is an even code.
QK_HD float actq_e2m1_rn(float a) {
  const float m = fabsf(a);
  float r;
  if (m >= 6.f) r = 6.f;
  else if (m < 2.f) r = rintf(m * 2.f) * 0.5f;
  else if (m < 4.f) r = rintf(m);
  else r = fminf(rintf(m * 0.5f) * 2.f, 6.f);
  return copysignf(r, a);
}

// Two values of a block (already times actq_up) to e4m3 codes, low byte = a.
// e2m1 mode rounds to the e2m1 grid first; the e4m3 cast is then exact.
QK_HD uint32_t actq_pair(float a, float b, int fp4) {
  if (fp4) {
    a = actq_e2m1_rn(a);
    b = actq_e2m1_rn(b);
  }
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

// One term of 32 values (one scale block): e4m3 codes into q (byte i =
// element i), returns the e8m0 code.
QK_HD int actq_block(const float (&v)[32], uint32_t (&q)[8], int fp4) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
  const int c = actq_scale_code(m, actq_emax(fp4));
  const float up = actq_up(c);
#pragma unroll
  for (int i = 0; i < 32; i += 4)
    q[i / 4] = actq_pair(v[i] * up, v[i + 1] * up, fp4) | (actq_pair(v[i + 2] * up, v[i + 3] * up, fp4) << 16);
  return c;
}

// e2m1 code (bit 3: sign) of a value already on the e2m1 grid.
QK_HD uint32_t actq_e2m1_code(float r) {
  const float m = fabsf(r);
  const uint32_t c = m < 2.f ? (uint32_t)(m * 2.f) : m < 4.f ? (uint32_t)m + 2u : m < 6.f ? 6u : 7u;
  return c | (signbit(r) ? 8u : 0u);
}

// One e2m1 term of 32 values as packed codes for the fp4 x fp4 tensor core
// (element 2 i in the low nibble of byte i, 16 bytes in q): the same values
// and e8m0 code as actq_block with fp4 set.
QK_HD int actq_block_fp4(const float (&v)[32], uint32_t (&q)[4]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
  const int c = actq_scale_code(m, actq_emax(1));
  const float up = actq_up(c);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) word |= actq_e2m1_code(actq_e2m1_rn(v[8 * w + i] * up)) << (4 * i);
    q[w] = word;
  }
  return c;
}

// NVFP4 layers in QK_ACT_MXFP4 (kind::mxf4nvf4 takes ue4m3 scales per 16):
// a row's 32-block code c becomes the ue4m3 code of 2^(c - cmax + 8), cmax
// the row's largest, and the row's factor is 2^(cmax - 135), so that code x
// factor = 2^(c - 127) exactly while c >= cmax - 17.
// ue4m3 code of 2^d (d <= 8); 0 below 2^-9, the smallest subnormal.
QK_HD uint32_t actq_nv_code(int d) {
  if (d >= -6) return (uint32_t)(d + 7) << 3;
  return d >= -9 ? 1u << (d + 9) : 0u;
}

// 2^e as fp32 for -149 <= e <= 127 (subnormal below -126): the row factor.
QK_HD float actq_pow2(int e) {
  return e >= -126 ? actq_float((uint32_t)(e + 127) << 23) : actq_float(1u << (e + 149));
}

}  // namespace qk

#if defined(__CUDACC__) && !defined(QK_ACTQ_ARITHMETIC_ONLY)
#include "qk_group.cuh"
#include "qk_internal.h"

namespace qk {
// The grouped path with an activation mode (QK_ACT_*): group_forward is
// group_forward_act(a, QK_ACT_NONE, ...); gmx_forward_act runs the x split
// and the two block-scaled GEMMs (the sort and both tile lists are done, the
// combine follows).
qk_status group_forward_act(const DecodeArgs& a, int act_quant, void* workspace, cudaStream_t st);
qk_status gmx_forward_act(const DecodeArgs& a, const GroupWs& W, int act_quant, cudaStream_t st);
// Token tile heights of the grouped block-scaled path: 64 (gate/up, x as 2
// terms) and 40 (down, h as 3) with exact activations; 128 for both in the
// activation-quantized modes (one term per token, every TMEM lane a token).
__host__ __device__ inline int gmx_tok1(int act_quant) { return act_quant == QK_ACT_NONE ? kXTok1 : 128; }
__host__ __device__ inline int gmx_tok2(int act_quant) { return act_quant == QK_ACT_NONE ? kXTok2 : 128; }
}  // namespace qk
#endif
