// qk_internal.h -- host-side declarations shared by the libqk translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "qk.h"

namespace qk {

constexpr int kMaxPairs = 128;  // decode path: tokens * top_k
constexpr int kMaxStages = 6;   // deepest bulk-copy ring

inline size_t align256(size_t n) { return (n + 255) / 256 * 256; }

// Dynamic shared memory above the 48 KB default: cudaFuncSetAttribute is
// called once per (kernel, device, size) and remembered, not on every launch.
// smem_attr_forget drops the record (a launch that was refused, e.g. after a
// cudaDeviceReset cleared the attribute, sets it again and retries once).
bool smem_attr(const void* kernel, size_t bytes);
void smem_attr_forget(const void* kernel);

// Arguments of the decode kernels (passed by value as a kernel parameter).
struct DecodeArgs {
  qk_weight gate, up, down;
  const uint16_t* x;  // bf16 [T][H]
  const int32_t* ids; // [T][k]
  const float* w;     // [T][k]
  void* y;
  int T, k, E, H, I, P;
  int y_bf16;
  // workspace
  float* h;           // [P][I] fp32 SwiGLU output
  float* hmax;        // [P][I/8] absmax of h per 8-row tile
  float* ures;        // [units][32] float4: k_down result of each (virtual expert, row tile)
};

qk_status decode_forward(DecodeArgs args, cudaStream_t st);
// Grouped (prefill) path: pairs grouped by expert, tcgen05 grouped GEMMs.
size_t group_workspace_bytes(const qk_moe_layer* L, int T, int k);
// The same with an activation mode (QK_ACT_E4M3 / QK_ACT_MXFP4): 0 if refused.
size_t group_workspace_bytes_act(const qk_moe_layer* L, int T, int k, int act_quant);
qk_status group_forward(const DecodeArgs& a, void* workspace, cudaStream_t st);
// Decode path for all-MXFP4 layers on the block-scaled tensor cores.
bool dmx_eligible(const qk_weight& gate, const qk_weight& up, const qk_weight& down, int H, int I);
size_t dmx_workspace_bytes(int T, int k, int H, int I);
qk_status dmx_forward(const DecodeArgs& a, void* workspace, cudaStream_t st);
size_t decode_workspace_bytes(int T, int k, int H, int I);
void decode_carve(DecodeArgs& a, void* ws);

qk_status route_topk_launch(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                            cudaStream_t st);
qk_status convert_launch(const uint8_t* e8m0, int E, int N, int K, uint8_t* e4m3, float* scale_2,
                         unsigned long long* n_inexact, cudaStream_t st);
qk_status fp8_linear_launch(const void* x, int M, int K, const uint8_t* w, const uint8_t* ws, int N,
                            void* y, int y_bf16, cudaStream_t st);
size_t fp8_ffn_workspace_bytes(int M, int H, int I);
// The FP8 shared expert at large M on the block-scaled grouped kernels (one
// group of M tokens); fp8_ffn_launch_blk takes it where fp8_big_eligible.
size_t fp8_group_workspace_bytes(int M, int H, int I);
qk_status fp8_group_forward(const void* x, int M, int H, int I, const uint8_t* wg, const uint8_t* sg,
                            const uint8_t* wu, const uint8_t* su, const uint8_t* wd, const uint8_t* sd, int blk,
                            float* y, void* workspace, cudaStream_t st);
qk_status fp8_ffn_launch(const void* x, int M, int H, int I, const uint8_t* wg, const uint8_t* sg,
                         const uint8_t* wu, const uint8_t* su, const uint8_t* wd, const uint8_t* sd,
                         float* y, void* ws, cudaStream_t st);

}  // namespace qk
