// qk_capi.cu -- the extern "C" entry points of libqk.so declared in qk.h:
// argument validation, workspace carving, dispatch, and the device status word.
#include <cuda_runtime.h>

#include <mutex>

#include "qk_actq.cuh"
#include "qk_convert_nv.h"
#include "qk_fp8.h"
#include "qk_device.cuh"
#include "qk_internal.h"

namespace qk {
__device__ int g_status = 0;
__device__ unsigned long long g_wait_limit_ns = 1000000000ull;

namespace {
struct SmemAttr {
  const void* fn;
  int dev;
  size_t bytes;
};
constexpr int kSmemAttrs = 256;
SmemAttr g_smem_attr[kSmemAttrs];
int g_smem_attr_n = 0;
std::mutex g_smem_attr_mu;
}  // namespace

bool smem_attr(const void* kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return true;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(g_smem_attr_mu);
  int slot = -1;
  for (int i = 0; i < g_smem_attr_n; ++i)
    if (g_smem_attr[i].fn == kernel && g_smem_attr[i].dev == dev) {
      if (g_smem_attr[i].bytes >= bytes) return true;
      slot = i;
      break;
    }
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
    return false;
  if (slot < 0 && g_smem_attr_n < kSmemAttrs) slot = g_smem_attr_n++;
  if (slot >= 0) g_smem_attr[slot] = {kernel, dev, bytes};
  return true;
}

void smem_attr_forget(const void* kernel) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  std::lock_guard<std::mutex> lock(g_smem_attr_mu);
  for (int i = 0; i < g_smem_attr_n; ++i)
    if (g_smem_attr[i].fn == kernel && g_smem_attr[i].dev == dev) g_smem_attr[i].bytes = 0;
}
}  // namespace qk

using namespace qk;

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool weight_ok(const qk_weight& w, int rows, int cols, int E) {
  if (w.fmt != QK_FMT_MXFP4 && w.fmt != QK_FMT_NVFP4) return false;
  if (!w.q || !w.scales || !aligned16(w.q) || !aligned16(w.scales)) return false;
  if (w.fmt == QK_FMT_NVFP4 && !w.scale_2) return false;
  return w.rows == rows && w.cols == cols && w.n_experts == E;
}

static qk_status layer_ok(const qk_moe_layer* L) {
  if (!L) return QK_ERR_INVALID_ARG;
  const int H = L->hidden, I = L->inter, E = L->gate.n_experts;
  if (H < 128 || I < 128 || H % 128 || I % 128 || E <= 0 || E > 32767) return QK_ERR_INVALID_ARG;
  if (!weight_ok(L->gate, I, H, E) || !weight_ok(L->up, I, H, E) || !weight_ok(L->down, H, I, E))
    return QK_ERR_INVALID_ARG;
  return QK_OK;
}

extern "C" {

// Tokens per decode launch: the routing tables of one launch hold kMaxPairs
// pairs; more tokens take the grouped path.
static int decode_chunk(int top_k) { return kMaxPairs / top_k; }

// The activation-quantized modes run on the grouped block-scaled kernels at
// every token count: all-MXFP4 layers that qualify for them, and all-NVFP4
// layers in QK_ACT_MXFP4 (kind::mxf4nvf4).
static bool act_quant_ok(const qk_moe_layer* L, int32_t act_quant) {
  return group_workspace_bytes_act(L, 1, 1, act_quant) > 0;
}

size_t moe_expert_workspace_size(const qk_moe_layer* L, int32_t n_tokens, int32_t top_k, int32_t act_quant) {
  if (layer_ok(L) != QK_OK || n_tokens < 0 || top_k < 1 || top_k > 8) return 0;
  if (act_quant != QK_ACT_NONE)
    return group_workspace_bytes_act(L, n_tokens, top_k, act_quant);
  if (n_tokens > decode_chunk(top_k))
    return group_workspace_bytes(L, n_tokens, top_k);
  if (dmx_eligible(L->gate, L->up, L->down, L->hidden, L->inter))
    return dmx_workspace_bytes(n_tokens, top_k, L->hidden, L->inter);
  return decode_workspace_bytes(n_tokens, top_k, L->hidden, L->inter);
}

qk_status moe_expert_forward(const qk_moe_layer* L, const void* x_bf16, int32_t n_tokens,
                             const int32_t* topk_ids, const float* topk_w, int32_t top_k,
                             void* y, int32_t y_is_bf16, int32_t act_quant, void* workspace,
                             size_t workspace_bytes, qk_stream_t stream) {
  const qk_status lrc = layer_ok(L);
  if (lrc != QK_OK) return lrc;
  if (n_tokens < 0 || top_k < 1 || top_k > 8) return QK_ERR_INVALID_ARG;
  if (act_quant != QK_ACT_NONE && act_quant != QK_ACT_MXFP4 && act_quant != QK_ACT_E4M3)
    return QK_ERR_INVALID_ARG;
  if (act_quant != QK_ACT_NONE && !act_quant_ok(L, act_quant)) return QK_ERR_UNSUPPORTED;
  if (n_tokens == 0) return QK_OK;
  if (!x_bf16 || !topk_ids || !topk_w || !y || !aligned16(x_bf16)) return QK_ERR_INVALID_ARG;
  const size_t need = moe_expert_workspace_size(L, n_tokens, top_k, act_quant);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return QK_ERR_WORKSPACE;
  DecodeArgs a = {};
  a.gate = L->gate;
  a.up = L->up;
  a.down = L->down;
  a.x = static_cast<const uint16_t*>(x_bf16);
  a.ids = topk_ids;
  a.w = topk_w;
  a.y = y;
  a.T = n_tokens;
  a.k = top_k;
  a.E = L->gate.n_experts;
  a.H = L->hidden;
  a.I = L->inter;
  a.P = n_tokens * top_k;
  a.y_bf16 = y_is_bf16 ? 1 : 0;
  // The activation-quantized modes, and token counts above one decode launch's
  // routing capacity, take the grouped path.
  if (act_quant != QK_ACT_NONE)
    return group_forward_act(a, act_quant, workspace, reinterpret_cast<cudaStream_t>(stream));
  if (n_tokens > decode_chunk(top_k)) return group_forward(a, workspace, reinterpret_cast<cudaStream_t>(stream));
  // All-MXFP4 layers: weights straight to the fp4 block-scaled tensor cores.
  if (dmx_eligible(a.gate, a.up, a.down, a.H, a.I))
    return dmx_forward(a, workspace, reinterpret_cast<cudaStream_t>(stream));
  decode_carve(a, workspace);
  return decode_forward(a, reinterpret_cast<cudaStream_t>(stream));
}

qk_status moe_route_topk(const float* logits, int32_t n_tokens, int32_t n_experts, int32_t top_k,
                         int32_t* ids, float* w, qk_stream_t stream) {
  if (n_tokens < 0 || n_experts < 1 || n_experts > 2048 || top_k < 1 || top_k > 32 ||
      top_k > n_experts)
    return QK_ERR_INVALID_ARG;
  if (n_tokens == 0) return QK_OK;
  if (!logits || !ids || !w) return QK_ERR_INVALID_ARG;
  return route_topk_launch(logits, n_tokens, n_experts, top_k, ids, w,
                           reinterpret_cast<cudaStream_t>(stream));
}

qk_status quant_convert_mxfp4_to_nvfp4(const uint8_t* e8m0, int32_t n_experts, int32_t rows,
                                       int32_t cols, uint8_t* e4m3, float* scale_2,
                                       unsigned long long* n_inexact, qk_stream_t stream) {
  if (n_experts < 0 || rows < 0 || cols <= 0 || cols % 32) return QK_ERR_INVALID_ARG;
  if (!e8m0 || !e4m3 || !scale_2 || !n_inexact) return QK_ERR_INVALID_ARG;
  return convert_launch(e8m0, n_experts, rows, cols, e4m3, scale_2, n_inexact,
                        reinterpret_cast<cudaStream_t>(stream));
}

qk_status quant_convert_nvfp4_to_mxfp4(const uint8_t* e4m3, const float* scale_2, int32_t n_experts,
                                       int32_t rows, int32_t cols, uint8_t* e8m0,
                                       unsigned long long* n_inexact, qk_stream_t stream) {
  if (n_experts < 0 || rows < 0 || cols <= 0 || cols % 32) return QK_ERR_INVALID_ARG;
  if (!e4m3 || !scale_2 || !e8m0 || !n_inexact) return QK_ERR_INVALID_ARG;
  return convert_nv_launch(e4m3, scale_2, n_experts, rows, cols, e8m0, n_inexact,
                           reinterpret_cast<cudaStream_t>(stream));
}

qk_status fp8_block_linear(const void* x_bf16, int32_t M, int32_t K, const uint8_t* w,
                           const uint8_t* w_scale, int32_t N, int32_t scale_block, void* y,
                           int32_t y_is_bf16, qk_stream_t stream) {
  if (M < 1 || K < 128 || K % 128 || N < 16 || N % 16) return QK_ERR_INVALID_ARG;
  if (scale_block != 128 && scale_block != 32) return QK_ERR_INVALID_ARG;
  if (!x_bf16 || !w || !w_scale || !y || !aligned16(x_bf16) || !aligned16(w))
    return QK_ERR_INVALID_ARG;
  return fp8_linear_launch_blk(x_bf16, M, K, w, w_scale, N, y, y_is_bf16 ? 1 : 0, scale_block,
                               reinterpret_cast<cudaStream_t>(stream));
}

size_t fp8_shared_expert_workspace_size(int32_t M, int32_t hidden, int32_t inter) {
  if (M < 1 || hidden < 128 || inter < 128 || hidden % 128 || inter % 128) return 0;
  return fp8_ffn_workspace_bytes(M, hidden, inter);
}

qk_status fp8_shared_expert_forward(const void* x_bf16, int32_t M, int32_t hidden, int32_t inter,
                                    const uint8_t* w_gate, const uint8_t* s_gate,
                                    const uint8_t* w_up, const uint8_t* s_up,
                                    const uint8_t* w_down, const uint8_t* s_down, int32_t scale_block,
                                    float* y, void* workspace, size_t workspace_bytes,
                                    qk_stream_t stream) {
  if (M < 1 || hidden < 128 || inter < 128 || hidden % 128 || inter % 128) return QK_ERR_INVALID_ARG;
  if (scale_block != 128 && scale_block != 32) return QK_ERR_INVALID_ARG;
  if (!x_bf16 || !w_gate || !s_gate || !w_up || !s_up || !w_down || !s_down || !y)
    return QK_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down))
    return QK_ERR_INVALID_ARG;
  const size_t need = fp8_shared_expert_workspace_size(M, hidden, inter);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return QK_ERR_WORKSPACE;
  return fp8_ffn_launch_blk(x_bf16, M, hidden, inter, w_gate, s_gate, w_up, s_up, w_down, s_down, y,
                            workspace, scale_block, reinterpret_cast<cudaStream_t>(stream));
}

qk_status qk_last_device_status(qk_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return QK_ERR_CUDA;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return QK_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return QK_ERR_CUDA;
  return v;
}

const char* qk_status_string(qk_status s) {
  switch (s) {
    case QK_OK: return "ok";
    case QK_ERR_INVALID_ARG: return "invalid argument";
    case QK_ERR_UNSUPPORTED: return "unsupported";
    case QK_ERR_WORKSPACE: return "workspace missing or too small";
    case QK_ERR_NAN_SCALE: return "NaN scale code";
    case QK_ERR_CUDA: return "CUDA runtime error";
    case QK_ERR_TIMEOUT: return "bounded device wait ran out";
    case QK_ERR_NONFINITE: return "activation or fp32 intermediate not finite";
    default: return "unknown status";
  }
}

qk_status qk_debug_set_wait_limit_ns(unsigned long long limit_ns) {
  return cudaMemcpyToSymbol(g_wait_limit_ns, &limit_ns, sizeof(limit_ns)) == cudaSuccess
             ? QK_OK
             : QK_ERR_CUDA;
}

}  // extern "C"
