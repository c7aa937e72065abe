/*
 * qk_oracle.h -- plain CPU oracle for the block-quantized expert FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the CPU-baseline
 * leg of bench.py may load this library.  It shares no code, header, table or
 * helper with the CUDA library; the two meet only in the byte layouts, which
 * are the storage formats themselves.
 *
 * Everything here is the plain definition: decode every code to its value,
 * form the dequantized weights exactly (fp64), accumulate dot products in
 * fp64, apply SwiGLU in fp64, and sum the routed experts in slot order.  No blocking, fusion or
 * reordering beyond that.
 *
 * Sources (pages on DeepSeek-V4-Flash quantized checkpoints):
 *  - "DeepSeek-v4-Flash-REAP-K180-NVFP4", section "NVFP4: lossless MXFP4->NVFP4
 *    conversion": MXFP4 = e2m1 nibbles + e8m0 scale per 32; NVFP4 = e2m1 +
 *    e4m3 scale per 16 + per-expert fp32 scale_2; the conversion changes
 *    scales only and keeps the nibbles.
 *  - "DeepSeekv4 Flash for 1x Spark [REAP25]", section "What's actually
 *    different": MXFP4 is 4.25 bits per weight.
 *  - "DeepSeek-V4-Flash-IQ2XXS-Q2K-FP8-120GB-target", component table: dense
 *    linears are FP8 E4M3 with block-128 UE8M0 scales.
 *  - "DeepSeek-V4-Flash-W4A16-FP8", base-model table: hidden 4096, 256 routed
 *    experts, top-6.
 * The pages give no bit encodings, nibble order, SwiGLU form or router; the
 * readings adopted for those are listed where each function is defined.
 *
 * Parity pins: every function is checked in tests/ against values fixed
 * outside this file (library decoders, hand-worked blocks, closed forms,
 * invariants, brute force).  No function here is "parity unpinned".
 */
#ifndef QK_ORACLE_H
#define QK_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { QKO_OK = 0, QKO_ERR_INVALID_ARG = 1, QKO_ERR_NAN_SCALE = 4 };
enum { QKO_FMT_MXFP4 = 1, QKO_FMT_NVFP4 = 2 };
enum { QKO_ACT_NONE = 0, QKO_ACT_MXFP4 = 1, QKO_ACT_E4M3 = 2 }; /* activation quantization */

/* Element codes. */
double qko_e2m1_value(uint8_t code);      /* low 4 bits: s|e1 e0|m */
double qko_e8m0_value(uint8_t code);      /* 2^(c-127); NaN for 255 */
double qko_e4m3_value(uint8_t code);      /* E4M3FN; NaN for 0x7F/0xFF */
uint8_t qko_e4m3_encode(double v);        /* round-to-nearest-even, saturate to +-448 */
uint8_t qko_e2m1_encode(double v);        /* round-to-nearest-even, saturate to +-6 */
double qko_bf16_value(uint16_t bits);

/* One projection of one layer: nibbles [E][rows][cols/2], scales
 * [E][rows][cols/32] (MXFP4, e8m0) or [E][rows][cols/16] (NVFP4, e4m3), and
 * scale_2 [E] (NVFP4 only). */
typedef struct {
  int32_t fmt;
  const uint8_t* q;
  const uint8_t* scales;
  const float* scale_2;
  int32_t n_experts, rows, cols;
} qko_weight;

typedef struct {
  qko_weight gate, up, down; /* gate/up: [E][inter][hidden]; down: [E][hidden][inter] */
  int32_t hidden, inter;
} qko_layer;

/* Dequantize one row of expert e, exactly (fp64). Returns QKO_ERR_NAN_SCALE on a NaN scale. */
int qko_dequant_row(const qko_weight* w, int32_t e, int32_t row, double* out);

/* Scale-only MXFP4 -> NVFP4 conversion of one projection. */
int qko_convert_mx_to_nv(const uint8_t* e8m0, int32_t E, int32_t N, int32_t K,
                         uint8_t* e4m3, float* scale_2, uint64_t* n_inexact);

/* NVFP4 -> MXFP4, scales only: exact blocks (equal power-of-two half scales)
 * map to their code, others are counted and take the code nearest in log2 to
 * the larger half scale. */
int qko_convert_nv_to_mx(const uint8_t* e4m3, const float* scale_2, int32_t E, int32_t N, int32_t K,
                         uint8_t* e8m0, uint64_t* n_inexact);

/* Softmax over E logits, top-k, renormalised; fp64 weights. */
int qko_route_topk(const float* logits, int32_t T, int32_t E, int32_t k,
                   int32_t* ids, double* w);

/* Routed-expert FFN for T tokens: y[t] = sum_s w[t][s] * FFN_{ids[t][s]}(x[t]). */
int qko_moe_forward(const qko_layer* L, const uint16_t* x_bf16, int32_t T,
                    const int32_t* ids, const double* w, int32_t k, double* y);

/* One expert's FFN on one token, with intermediates (any pointer may be NULL). */
int qko_expert_ffn(const qko_layer* L, int32_t e, const uint16_t* x_bf16,
                   double* g, double* u, double* h, double* d);

/* Activation quantization of n values (n % 32 == 0) to MXFP4 or E4M3 with one
 * e8m0 scale per 32 (OCP MX scale rule): element codes [n], scale codes
 * [n/32], dequantized values [n]; any output may be NULL. */
int qko_act_quant(const double* v, int32_t n, int32_t aq, uint8_t* codes, uint8_t* scales,
                  double* out);

/* The FFN and the routed sum with activation quantization `aq` (QKO_ACT_*):
 * x quantized before gate/up, h (rounded to fp32) quantized before down. */
int qko_expert_ffn_aq(const qko_layer* L, int32_t e, const uint16_t* x_bf16, int32_t aq,
                      double* g, double* u, double* h, double* d);
int qko_moe_forward_aq(const qko_layer* L, const uint16_t* x_bf16, int32_t T,
                       const int32_t* ids, const double* w, int32_t k, int32_t aq, double* y);

/* y[M][N] = x[M][K] . dq(W)^T with W e4m3 [N][K], scales ue8m0 [N/b][K/b]. */
int qko_fp8_block_linear(const uint16_t* x_bf16, int32_t M, int32_t K,
                         const uint8_t* w, const uint8_t* w_scale, int32_t N,
                         int32_t block, double* y);

/* Shared-expert SwiGLU FFN with FP8 block weights: gate/up [I][H], down [H][I]. */
int qko_fp8_swiglu_ffn(const uint16_t* x_bf16, int32_t M, int32_t H, int32_t I,
                       const uint8_t* wg, const uint8_t* sg,
                       const uint8_t* wu, const uint8_t* su,
                       const uint8_t* wd, const uint8_t* sd,
                       int32_t block, double* y);

void qko_set_threads(int32_t n);
int32_t qko_get_threads(void);

#ifdef __cplusplus
}
#endif
#endif
