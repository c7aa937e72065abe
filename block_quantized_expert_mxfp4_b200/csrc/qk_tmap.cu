// qk_tmap.cu -- tensor-map encoding through the driver entry point
// cuTensorMapEncodeTiled (obtained with cudaGetDriverEntryPoint, so the
// library does not link libcuda), with a small cache keyed by every argument.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "qk_tmap.h"

namespace qk {

namespace {

struct Key {
  int dtype, rank, swizzle, l2promo;
  const void* base;
  uint64_t dims[4], strides[3];
  uint32_t box[4];
  bool operator==(const Key& o) const { return std::memcmp(this, &o, sizeof(Key)) == 0; }
};

struct Entry {
  Key key;
  CUtensorMap map;
  bool used;
};

constexpr int kCache = 64;
Entry g_cache[kCache];
int g_next = 0;
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

}  // namespace

bool tmap_get(CUtensorMap* out, int dtype, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box, int swizzle, int l2promo) {
  Key k;
  std::memset(&k, 0, sizeof(k));
  k.dtype = dtype;
  k.rank = rank;
  k.swizzle = swizzle;
  k.l2promo = l2promo;
  k.base = base;
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides_bytes[i];
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < kCache; ++i)
    if (g_cache[i].used && g_cache[i].key == k) {
      *out = g_cache[i].map;
      return true;
    }
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        !fn)
      return false;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  cuuint64_t d[4], s[3];
  cuuint32_t b[4], es[4] = {1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
  CUtensorMap m;
  const CUresult r = g_encode(&m, (CUtensorMapDataType)dtype, rank, const_cast<void*>(base), d, s,
                              b, es, CU_TENSOR_MAP_INTERLEAVE_NONE, (CUtensorMapSwizzle)swizzle,
                              (CUtensorMapL2promotion)l2promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  Entry& e = g_cache[g_next];
  g_next = (g_next + 1) % kCache;
  e.key = k;
  e.map = m;
  e.used = true;
  *out = m;
  return true;
}

}  // namespace qk
