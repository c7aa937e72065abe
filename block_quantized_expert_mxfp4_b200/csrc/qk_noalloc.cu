// qk_noalloc.cu -- moe_expert_forward_noalloc: moe_expert_forward whose decode
// scratch is a fixed device array of this library instead of a caller
// workspace.
//
// It serves callers that cannot allocate device memory on the call path: a
// C caller embedded in another runtime that owns every device allocation (and
// exposes no allocator to plugins), or a host that must not grow its device
// footprint after start-up.  Such callers cannot size and pass a workspace per
// call; here the scratch is part of the library image, its address looked up
// with cudaGetSymbolAddress on every call (a host-side query: no device work),
// so it is always the address in the context current at the call, also after
// a cudaDeviceReset or in a second context on the same device.  Nothing is
// allocated: no cudaMalloc/cudaFree, no allocating library.
//
// The kernels are the decode kernels of moe_expert_forward, unchanged; only
// the origin of the workspace differs.  Nothing in the scratch has to start at
// zero: every buffer in it is written before it is read within a call.
#include <cuda_runtime.h>

#include "qk_internal.h"

namespace qk {

constexpr size_t kNoallocScratchBytes = (size_t)16 << 20;  // 16 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

// Device address of the scratch array in the current context.  The host-side
// name g_noalloc_scratch is only a stand-in; kernels get this address.
static void* noalloc_scratch() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace qk

using namespace qk;

extern "C" qk_status moe_expert_forward_noalloc(const qk_moe_layer* L, const void* x_bf16,
                                                int32_t n_tokens, const int32_t* topk_ids,
                                                const float* topk_w, int32_t top_k, void* y,
                                                int32_t y_is_bf16, qk_stream_t stream) {
  if (n_tokens < 0) return QK_ERR_INVALID_ARG;
  // validates the layer and top_k (0 = invalid); the size for >= 1 token
  const size_t need = moe_expert_workspace_size(L, n_tokens > 0 ? n_tokens : 1, top_k, QK_ACT_NONE);
  if (need == 0) return QK_ERR_INVALID_ARG;
  if (n_tokens == 0) return QK_OK;
  if (need > kNoallocScratchBytes) return QK_ERR_WORKSPACE;  // beyond the fixed array
  void* scratch = noalloc_scratch();
  if (!scratch) return QK_ERR_CUDA;
  return moe_expert_forward(L, x_bf16, n_tokens, topk_ids, topk_w, top_k, y, y_is_bf16,
                            QK_ACT_NONE, scratch, kNoallocScratchBytes, stream);
}
