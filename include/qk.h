/*
 * qk.h -- C ABI of libqk.so: the routed-expert FFN of a DeepSeek-V4-Flash-style
 * MoE layer with block-quantized expert weights, on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages on quantized DeepSeek-V4-Flash checkpoints; cited by page
 * title and section):
 *  [REAP-K180]  "DeepSeek-v4-Flash-REAP-K180-NVFP4", "NVFP4: lossless
 *               MXFP4->NVFP4 conversion" and "Why this mix?".
 *  [REAP25]     "DeepSeekv4 Flash for 1x Spark [REAP25] [PrismaAURA]",
 *               "What's actually different" and the v0.2.3 update.
 *  [IQ2-FP8]    "DeepSeek-V4-Flash-IQ2XXS-Q2K-FP8-120GB-target", component table.
 *  [W4A16-FP8]  "DeepSeek-V4-Flash-W4A16-FP8", "Architecture & precision".
 *  [V41-Q2]     "DeepSeek-V4.1-Flash mixed-Q2 GGUF (IQ2_XXS gate/up + Q2_K
 *               down)", "Recipe".
 *
 * Storage formats (the byte layouts are the interface):
 *  MXFP4   nibbles  uint8 [E][rows][cols/2]  element 2i = low nibble of byte i
 *          scales   uint8 [E][rows][cols/32] e8m0 (2^(c-127); 255 = NaN)
 *  NVFP4   nibbles  same bytes as MXFP4 (a converted layer shares them)
 *          scales   uint8 [E][rows][cols/16] e4m3 (E4M3FN)
 *          scale_2  float [E]                per-expert fp32 second-level scale
 *  FP8     weight   uint8 [N][K] e4m3, scales uint8 [ceil(N/128)][ceil(K/128)] ue8m0
 *  e2m1 nibble: bit 3 sign, bits 2..1 exponent, bit 0 mantissa; magnitudes
 *  0, .5, 1, 1.5, 2, 3, 4, 6.  Rows are contiguous along the input dimension
 *  and the quantization blocks run along it.  Gate and up are [E][inter][hidden],
 *  down is [E][hidden][inter].
 *
 * Conventions:
 *  - Every pointer argument is DEVICE memory owned by the caller, unless the
 *    comment says host.  The library never allocates on a call path; scratch is
 *    the caller's workspace, sized by the *_workspace_size query.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *  - Argument errors are returned synchronously and nothing is launched.
 *    Errors found on the device (a NaN scale code, an expert id out of range,
 *    a bounded wait that ran out) are recorded in a per-device status word,
 *    first error wins, and read by qk_last_device_status().
 *  - Calls on one stream are ordered; concurrent calls on different streams
 *    must use different workspaces and outputs.
 */
#ifndef QK_H
#define QK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* qk_stream_t; /* same type as cudaStream_t */

typedef int32_t qk_status;
enum {
  QK_OK = 0,
  QK_ERR_INVALID_ARG = 1, /* null pointer, bad size, unsupported shape, expert id out of range */
  QK_ERR_UNSUPPORTED = 2, /* a valid request this build does not implement */
  QK_ERR_WORKSPACE = 3,   /* workspace pointer null or smaller than the query */
  QK_ERR_NAN_SCALE = 4,   /* an e8m0 code 255 or an e4m3 scale code 0x7F/0xFF was read */
  QK_ERR_CUDA = 5,        /* a CUDA runtime call failed (launch, attribute, copy) */
  QK_ERR_TIMEOUT = 6,     /* a bounded device wait ran out; outputs are undefined */
  QK_ERR_NONFINITE = 7    /* an activation, or an fp32 intermediate (h = silu(gate) * up, y), is
                             inf or NaN: an input was not finite or a sum overflowed fp32 (the
                             kernels accumulate in fp32); the affected outputs are undefined */
};

enum { QK_FMT_MXFP4 = 1, QK_FMT_NVFP4 = 2 };

/* Activation handling inside moe_expert_forward.
 *  QK_ACT_NONE   bf16 activations, used as they are (weights exact on chip,
 *                activations exact or as exact sums of e4m3 terms).
 *  QK_ACT_E4M3   W4A8: activations quantized to E4M3 with one e8m0 scale per
 *                32 ([REAP25] v0.2.3 update: fp4 weights x dynamic E4M3
 *                activations on block-scaled f8f6f4 tensor cores, the model's
 *                own expert numerics), x before gate/up and h before down.
 *  QK_ACT_MXFP4  the same with e2m1 activations (fp4 x fp4, run on the
 *                kind::mxf4 block-scaled tensor cores with both operands
 *                packed e2m1; NVFP4 layers on kind::mxf4nvf4, whose scales
 *                are ue4m3 per 16: each row's e8m0 activation scales are
 *                re-anchored as ue4m3 2^(c - cmax + 8), cmax the row's
 *                largest, and 2^(cmax - 135) times scale_2 multiplies the
 *                result; exact while a block's code is within 17 of cmax, a
 *                block further below, under 2^-17 of the row's largest
 *                values, is dropped).
 * Scale rule for both (the pages give none; OCP Microscaling v1.0): X =
 * floor(log2 max|v|) - 8 (e4m3) or - 2 (e2m1) per 32 values, clamped to the
 * e8m0 range; elements rounded to nearest even, saturating (E4M3 to 448,
 * e2m1 to 6).  The quantized modes need an all-MXFP4 layer that qualifies for
 * the block-scaled grouped kernels (see moe_expert_forward), or for
 * QK_ACT_MXFP4 an all-NVFP4 one with the same shape and alignment, and run
 * on them at every token count; other layers (mixed formats, and NVFP4 in
 * QK_ACT_E4M3: the f8f6f4 kind takes ue8m0 scales only) return
 * QK_ERR_UNSUPPORTED. */
enum { QK_ACT_NONE = 0, QK_ACT_MXFP4 = 1, QK_ACT_E4M3 = 2 };

/* One projection of one layer, all experts.  Device pointers. */
typedef struct qk_weight {
  int32_t fmt;            /* QK_FMT_MXFP4 or QK_FMT_NVFP4 */
  const uint8_t* q;       /* nibbles [n_experts][rows][cols/2], 16-byte aligned */
  const uint8_t* scales;  /* [n_experts][rows][cols/32] (MX) or [..][cols/16] (NV) */
  const float* scale_2;   /* [n_experts] (NV only; ignored for MX) */
  int32_t n_experts, rows, cols;
} qk_weight;

/* gate, up: rows = inter, cols = hidden; down: rows = hidden, cols = inter.
 * Each projection may use its own format.  n_experts must agree. */
typedef struct qk_moe_layer {
  qk_weight gate, up, down;
  int32_t hidden, inter;
} qk_moe_layer;

/* ------------------------------------------------------------------------
 * moe_expert_forward -- routed-expert FFN, weighted combine.
 *   y[t] = sum_{s<k} w[t][s] * down_e( silu(gate_e x[t]) * up_e x[t] ),  e = ids[t][s]
 * [REAP-K180] "Why this mix?" (gate/up/down expert projections; gate+up are
 * ~2/3 of expert bytes); [W4A16-FP8] base-model table (hidden 4096, 256 routed
 * experts, top-6).  SwiGLU form silu(gate)*up and the slot-order combine are
 * the readings adopted (the pages do not print them).
 *
 *  x_bf16    [T][hidden] bf16.        topk_ids [T][top_k] int32 in [0, E).
 *  topk_w    [T][top_k] fp32.         y        [T][hidden] fp32 (y_is_bf16=0) or bf16.
 *  act_quant QK_ACT_* (above).        workspace >= moe_expert_workspace_size(), 256-B aligned.
 * Shapes: hidden and inter multiples of 128; 1 <= top_k <= 8.  Up to
 * floor(128/top_k) tokens run the decode kernels: for all-MXFP4 layers with
 * hidden and inter multiples of 1024 and 32-byte aligned weights, the
 * block-scaled tensor cores (tcgen05 kind::mxf8f6f4 block_scale) with the
 * e2m1 weights and e8m0 scales as stored and the activations as e4m3 terms
 * with e8m0 scales per 32 (bf16 x as two terms, exact; h as three, relative
 * error below 2^-12); for other layers nibbles and scales decoded in
 * registers and tensor-core m16n8k16 f16 products; fp32 accumulation in
 * both.  More tokens run the grouped path ([REAP25] "What's actually different": one
 * grouped GEMM per projection): the pairs are sorted by expert and each
 * projection is a grouped tcgen05 GEMM -- on the block-scaled tensor cores
 * with the e2m1 weights and e8m0 scales as stored and the activations as
 * exact e4m3 terms when all three projections are MXFP4, hidden and inter
 * are multiples of 512, q is 32-byte and scales 16-byte aligned; otherwise
 * with the weights expanded to f16 on chip.  All kernels run in order on
 * `stream`.  T = 0 returns QK_OK and launches nothing.
 * Errors: QK_ERR_INVALID_ARG (shapes, pointers, formats, an unknown
 * act_quant), QK_ERR_WORKSPACE, QK_ERR_UNSUPPORTED (a quantized act_quant on
 * a layer the block-scaled kernels do not take), QK_ERR_CUDA; device:
 * QK_ERR_NAN_SCALE,
 * QK_ERR_INVALID_ARG (id out of range: that pair contributes nothing),
 * QK_ERR_TIMEOUT, QK_ERR_NONFINITE (an inf or NaN in x, or a gate/up/h/y
 * value that overflowed fp32: the kernels accumulate in fp32, so products of
 * scale codes near 254 with ordinary activations exceed its range where the
 * exact result does not).
 * moe_expert_workspace_size returns the workspace bytes of the path the same
 * (layer, n_tokens, top_k, act_quant) call takes, or 0 for arguments the call
 * would reject (including a quantized act_quant the layer does not take).
 * ---------------------------------------------------------------------- */
size_t moe_expert_workspace_size(const qk_moe_layer* L, int32_t n_tokens, int32_t top_k,
                                 int32_t act_quant);

qk_status moe_expert_forward(const qk_moe_layer* L, const void* x_bf16, int32_t n_tokens,
                             const int32_t* topk_ids, const float* topk_w, int32_t top_k,
                             void* y, int32_t y_is_bf16, int32_t act_quant,
                             void* workspace, size_t workspace_bytes, qk_stream_t stream);

/* ------------------------------------------------------------------------
 * moe_expert_forward_noalloc -- moe_expert_forward (act_quant QK_ACT_NONE)
 * with its scratch taken from a fixed 16 MiB device array inside libqk.so
 * instead of a caller workspace.  The pages have no counterpart: it exists for
 * callers that cannot allocate device memory on the call path (a C caller
 * embedded in a runtime that owns every device allocation).
 *  Arguments as moe_expert_forward.  The call needs
 *  moe_expert_workspace_size(L, n_tokens, top_k, QK_ACT_NONE) <= 16 MiB (hidden
 *  4096, inter 2048: every launch of an all-MXFP4 layer on the block-scaled
 *  decode kernels (up to 128 pairs) fits; other layers up to 114 pairs at
 *  top-6, 118 at top-2; the grouped kernels above 128 pairs do not fit);
 *  larger requests return
 *  QK_ERR_WORKSPACE and launch nothing.  Nothing in the array has to start at
 *  zero.  The array is shared by every call on a device: calls that overlap on
 *  the GPU (other streams, other host threads) race on it and must not be
 *  issued.  Every call looks up the array's address in the current context
 *  (a host-side runtime query, no device work); the first call in a context
 *  may also load the library's device code, so make it before beginning any
 *  stream capture in that context.
 * Errors: as moe_expert_forward; QK_ERR_WORKSPACE when the fixed array is too
 * small.
 * ---------------------------------------------------------------------- */
qk_status moe_expert_forward_noalloc(const qk_moe_layer* L, const void* x_bf16, int32_t n_tokens,
                                     const int32_t* topk_ids, const float* topk_w, int32_t top_k,
                                     void* y, int32_t y_is_bf16, qk_stream_t stream);

/* ------------------------------------------------------------------------
 * moe_route_topk -- router: softmax over E logits, the top_k largest
 * (equal values: lower expert id first), renormalised to sum 1, in
 * descending order.  Only the top_k logits enter the weights:
 *   w[t][s] = exp(l_s - l_max) / sum_{s'} exp(l_{s'} - l_max).
 * [W4A16-FP8] (256 experts, top-6; hash routing is mentioned, so callers may
 * also pass their own ids and weights to moe_expert_forward).
 *  logits [T][E] fp32 (-inf allowed); ids [T][top_k] int32; w [T][top_k] fp32.
 *  1 <= E <= 2048, 1 <= top_k <= min(E, 32).
 * Errors: QK_ERR_INVALID_ARG, QK_ERR_CUDA; device: QK_ERR_INVALID_ARG when a
 * token has no finite logit.
 * ---------------------------------------------------------------------- */
qk_status moe_route_topk(const float* logits, int32_t n_tokens, int32_t n_experts,
                         int32_t top_k, int32_t* ids, float* w, qk_stream_t stream);

/* ------------------------------------------------------------------------
 * quant_convert_mxfp4_to_nvfp4 -- scale-only MXFP4 -> NVFP4 conversion.
 * [REAP-K180] "NVFP4: lossless MXFP4->NVFP4 conversion": the e2m1 nibbles are
 * not touched (this call never reads or writes them); each e8m0 code per 32
 * becomes two equal e4m3 codes (one per 16) and each expert gets an fp32
 * scale_2.  Rule (reading adopted): c_max = the expert's largest code,
 * scale_2 = 2^(c_max-135), e4m3 = round-to-nearest-even cast of
 * 2^(c-c_max+8).  Exact when c >= c_max-17; otherwise the block's scale
 * becomes 0 and counts once in *n_inexact.
 *  e8m0 [E][N][K/32] -> e4m3 [E][N][K/16], scale_2 [E] fp32,
 *  n_inexact: device uint64, overwritten with the count of inexact 32-blocks.
 *  K multiple of 32.
 * Errors: QK_ERR_INVALID_ARG, QK_ERR_CUDA; device: QK_ERR_NAN_SCALE (a code
 * 255; its outputs are e4m3 NaN 0x7F).
 * ---------------------------------------------------------------------- */
qk_status quant_convert_mxfp4_to_nvfp4(const uint8_t* e8m0, int32_t n_experts, int32_t rows,
                                       int32_t cols, uint8_t* e4m3, float* scale_2,
                                       unsigned long long* n_inexact, qk_stream_t stream);

/* ------------------------------------------------------------------------
 * quant_convert_nvfp4_to_mxfp4 -- scale-only NVFP4 -> MXFP4, the reverse of
 * the conversion above (the pages give only the forward direction; rule
 * adopted): a 32-block whose half scales e4m3(s0) * scale_2 and
 * e4m3(s1) * scale_2 are equal and a power of two 2^p (-127 <= p <= 127)
 * converts exactly to code p + 127.  Any other block counts once in
 * *n_inexact and takes the code whose power of two is nearest in log2 to the
 * larger magnitude of the two (code 0 for two zero scales).  The nibbles are
 * not touched; the reverse of a lossless forward conversion is the identity.
 *  e4m3 [E][N][K/16], scale_2 [E] fp32 -> e8m0 [E][N][K/32];
 *  n_inexact: device uint64, overwritten.  K multiple of 32.
 * Errors: QK_ERR_INVALID_ARG, QK_ERR_CUDA; device: QK_ERR_NAN_SCALE (an e4m3
 * code 0x7F/0xFF or a non-finite scale product; that block's code is 255).
 * ---------------------------------------------------------------------- */
qk_status quant_convert_nvfp4_to_mxfp4(const uint8_t* e4m3, const float* scale_2, int32_t n_experts,
                                       int32_t rows, int32_t cols, uint8_t* e8m0,
                                       unsigned long long* n_inexact, qk_stream_t stream);

/* ------------------------------------------------------------------------
 * fp8_block_linear -- y[M][N] = x[M][K] . dq(W)^T, dq = e4m3 * 2^(s-127) per
 * B x B tile, B = scale_block.  [IQ2-FP8] component table ("FP8 E4M3,
 * block-128, UE8M0 scales"); [W4A16-FP8] ("FP8_BLOCK 128x128"); [V41-Q2]
 * "Recipe": DeepSeek-V4.1's FP8 dense weights carry 32x32 E8M0 block
 * scales where V4's carry 128x128.
 *  x bf16 [M][K]; w e4m3 [N][K]; w_scale ue8m0 [ceil(N/B)][ceil(K/B)];
 *  scale_block B = 128 or 32; y fp32 or bf16 [M][N].
 *  N multiple of 16, K multiple of 128, M >= 1.
 * Errors: QK_ERR_INVALID_ARG, QK_ERR_CUDA; device: QK_ERR_NAN_SCALE.
 * ---------------------------------------------------------------------- */
qk_status fp8_block_linear(const void* x_bf16, int32_t M, int32_t K, const uint8_t* w,
                           const uint8_t* w_scale, int32_t N, int32_t scale_block, void* y,
                           int32_t y_is_bf16, qk_stream_t stream);

/* ------------------------------------------------------------------------
 * fp8_shared_expert_forward -- the shared expert as a SwiGLU FFN with FP8
 * block-scaled weights (B x B tiles, B = scale_block, 128 or 32), ADDED into
 * an fp32 output:
 *   y[t] += down( silu(gate x[t]) * up x[t] )
 * Shared experts are kept at 8 bits on the pages ([REAP25] MXFP8, [REAP-K180]
 * Q8_0); FP8 E4M3 block-128 is the dense-layer format of [IQ2-FP8].
 *  x bf16 [M][H]; gate/up e4m3 [I][H] + scales [I/B][H/B];
 *  down e4m3 [H][I] + scales [H/B][I/B]; y fp32 [M][H] (read and written).
 *  H, I multiples of 128; workspace >= fp8_shared_expert_workspace_size().
 * Errors: as fp8_block_linear, plus QK_ERR_WORKSPACE.
 * ---------------------------------------------------------------------- */
size_t fp8_shared_expert_workspace_size(int32_t M, int32_t hidden, int32_t inter);

qk_status fp8_shared_expert_forward(const void* x_bf16, int32_t M, int32_t hidden, int32_t inter,
                                    const uint8_t* w_gate, const uint8_t* s_gate,
                                    const uint8_t* w_up, const uint8_t* s_up,
                                    const uint8_t* w_down, const uint8_t* s_down, int32_t scale_block,
                                    float* y, void* workspace, size_t workspace_bytes,
                                    qk_stream_t stream);

/* ------------------------------------------------------------------------
 * Status.  qk_last_device_status synchronizes `stream`, returns the first
 * device-side error recorded on the current device since the last read, and
 * clears it.  qk_status_string returns a static string (never NULL).
 * ---------------------------------------------------------------------- */
qk_status qk_last_device_status(qk_stream_t stream);
const char* qk_status_string(qk_status status);

/* Test hook: limit, in nanoseconds, of every bounded device wait (default
 * 1e9).  A limit of 0 makes the first wait that is not already complete run
 * out, which exercises the QK_ERR_TIMEOUT path without any hang.  Host call,
 * applies to launches made after it on the current device. */
qk_status qk_debug_set_wait_limit_ns(unsigned long long limit_ns);

#ifdef __cplusplus
}
#endif
#endif /* QK_H */
