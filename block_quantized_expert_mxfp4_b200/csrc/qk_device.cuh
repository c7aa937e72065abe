// qk_device.cuh -- device helpers shared by the libqk kernels (sm_100a only).
//
// Thin wrappers over PTX instructions documented in the PTX ISA (mbarrier,
// cp.async.bulk, ldmatrix, mma.sync, cvt with e2m1x2 / e4m3x2 / ue8m0x2
// sources, griddepcontrol), the per-device status word, and bounded waits.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qk.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libqk targets sm_100a (B200) only"
#endif

namespace qk {

// ---------------------------------------------------------------- status --
// First device-side error wins (except that any other error replaces
// QK_ERR_NONFINITE, which is usually its consequence: a NaN scale code makes
// NaN products); read and cleared by qk_last_device_status().
extern __device__ int g_status;
// Limit of every bounded wait, in ns (qk_debug_set_wait_limit_ns).
extern __device__ unsigned long long g_wait_limit_ns;
// Limit used when draining copies after a wait ran out (never 0).
constexpr unsigned long long kDrainLimitNs = 1000000000ull;

__device__ __forceinline__ void set_status(int code) {
  const int old = atomicCAS(&g_status, 0, code);
  if (old == QK_ERR_NONFINITE && code != QK_ERR_NONFINITE) atomicCAS(&g_status, QK_ERR_NONFINITE, code);
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// -------------------------------------------------------------- mbarrier --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_one(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Phase `parity` of `bar` complete now (no suspension).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about `ns` nanoseconds have passed.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` for at most `limit_ns`; false if it ran out.
// A limit of 0 takes one non-suspending look.  Otherwise the thread sleeps in
// hardware between looks (a suspend hint of 1 us, woken by the phase
// completing) and reads the timer once per look: waiting warps that poll in
// software take the issue slots and the barrier unit away from the few busy
// threads (the one issuing copies or tensor-core instructions), which slows
// those down severalfold.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  unsigned long long limit_ns) {
  if (limit_ns == 0) return mbar_test_wait(bar, parity);
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 1000u)) return true;
    if (globaltimer() - t0 >= limit_ns) return false;
  }
}

// 1-D bulk copy global -> shared, completing `bytes` on `bar`.  dst, src and
// bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same with an L2 eviction hint: weights are streamed once per call.
__device__ __forceinline__ void bulk_g2s_evict_first(void* dst, const void* src, uint32_t bytes,
                                                     uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Tiled tensor copies (TMA) global -> shared through a CUtensorMap held in
// kernel-parameter space.  The innermost coordinate must be 16-byte aligned.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int c0, int c1, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int c0, int c1, int c2,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)),
      "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const void* tmap, int c0, int c1, int c2, int c3,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar)),
      "l"(policy)
      : "memory");
}

// Prefetch a byte range from global memory into L2; no shared memory, no
// completion.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Bring a tensor map (kernel-parameter space) into the descriptor cache.
__device__ __forceinline__ void tmap_prefetch(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ------------------------------------------------------ PDL (griddepcontrol)
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;");
}

// ------------------------------------------------------------- ldmatrix --
// Four 8x8 b16 matrices: lane l supplies the row address for matrix l/8, row
// l%8; register j of lane (g = l/4, t = l%4) receives bytes [4t, 4t+4) of row
// g of matrix j.
__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(row_addr)));
}

// Two matrices (lanes 0..15 supply the row addresses).
__device__ __forceinline__ void ldmatrix_x2(uint32_t& r0, uint32_t& r1, const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(smem_u32(row_addr)));
}

// ------------------------------------------------------------------ mma --
// D = A(16x16 f16, row) * B(16x8 f16, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------- converts --
// Byte I of `w` (two e2m1 codes) -> f16x2, low nibble -> low half.
template <int I>
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t w);
#define QK_E2M1X2(IDX)                                                              \
  template <>                                                                       \
  __device__ __forceinline__ uint32_t e2m1x2_to_f16x2<IDX>(uint32_t w) {            \
    uint32_t out;                                                                   \
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n"            \
        " cvt.rn.f16x2.e2m1x2 %0, b" #IDX ";\n}\n"                                   \
        : "=r"(out)                                                                 \
        : "r"(w));                                                                  \
    return out;                                                                     \
  }
QK_E2M1X2(0)
QK_E2M1X2(1)
QK_E2M1X2(2)
QK_E2M1X2(3)
#undef QK_E2M1X2

// Low (I=0) or high (I=1) 16 bits of `w` (two e4m3 codes) -> f16x2.
template <int I>
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t w);
#define QK_E4M3X2(IDX)                                                              \
  template <>                                                                       \
  __device__ __forceinline__ uint32_t e4m3x2_to_f16x2<IDX>(uint32_t w) {            \
    uint32_t out;                                                                   \
    asm("{\n .reg .b16 h0, h1;\n mov.b32 {h0, h1}, %1;\n"                           \
        " cvt.rn.f16x2.e4m3x2 %0, h" #IDX ";\n}\n"                                   \
        : "=r"(out)                                                                 \
        : "r"(w));                                                                  \
    return out;                                                                     \
  }
QK_E4M3X2(0)
QK_E4M3X2(1)
#undef QK_E4M3X2

// e8m0 code -> fp32 2^(c-127) (c = 0 gives the subnormal 2^-127; c = 255 is
// reported by the caller).
__device__ __forceinline__ float e8m0_to_f32(uint32_t c) {
  return __uint_as_float(c ? (c << 23) : 0x00400000u);
}

// e4m3 (E4M3FN) code -> fp32, via the hardware e4m3x2 -> f16x2 conversion.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const uint32_t h = e4m3x2_to_f16x2<0>(c & 0xFFu);
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Power-of-two exponent s such that amax * 2^-s lies in [2^14, 2^15): the
// largest magnitude keeps full f16 precision with headroom below 65504.
__device__ __forceinline__ int f16_shift_for(float amax) {
  if (!(amax > 0.f) || !isfinite(amax)) return 0;
  return ilogbf(amax) - 14;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

// True when every value is finite (not inf, not NaN).  Non-finite inputs or
// fp32 intermediates are reported as QK_ERR_NONFINITE.
__device__ __forceinline__ bool finite_bits(float v) { return (__float_as_uint(v) & 0x7F800000u) != 0x7F800000u; }
__device__ __forceinline__ bool all_finite32(const float (&v)[32]) {
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 32; ++i) ok &= finite_bits(v[i]);
  return ok;
}

}  // namespace qk

// -------------------------------------------------------- tcgen05 / TMEM --
// 5th-generation tensor core: accumulators in tensor memory (TMEM), operands
// in shared memory described by 64-bit matrix descriptors.
namespace qk {

// Shared-memory matrix descriptor of a K-major tile in the 128-byte-swizzled
// canonical layout: rows of 128 bytes, 8-row groups 1024 bytes apart, the tile
// base 1024-byte aligned.  Fields: start address >> 4 (bits 0-13), leading
// byte offset >> 4 (16-29; unused for this layout, 1), stride byte offset >> 4
// (32-45; 1024 B), version 1 (46-47), base offset 0 (49-51), layout type
// 2 = 128-byte swizzle (61-63).
__device__ __forceinline__ uint64_t umma_desc_k_sw128(const void* smem_tile) {
  const uint64_t addr = (uint64_t)(smem_u32(smem_tile) >> 4) & 0x3FFFu;
  return addr | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: f16 A and B (K-major), fp32 accumulator,
// M x N (M = 64 or 128; N a multiple of 16 up to 256 when M = 128).
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t desc_a, uint64_t desc_b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(tmem_d),
      "l"(desc_a), "l"(desc_b), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// Block-scaled MMA (kind::mxf8f6f4): operand formats 0 = e4m3, 5 = e2m1 (in
// shared memory one element per byte position: sixteen 4-bit values in the
// low 8 bytes of each 16-byte chunk), one ue8m0 scale per 32 elements of K
// for every row of A and of B, fp32 accumulator, K = 32 per instruction.
// Fields: B scale id (bits 4-5), A format (7-9), B format (10-12), K-major
// A and B, N >> 3 (17-22), scale type ue8m0 (bit 23), M >> 4 (24-28), A
// scale id (29-30).  The scale ids select the byte of the 32-bit tensor-memory
// word that holds the scale for this instruction's 32 elements of K.
__host__ __device__ constexpr uint32_t umma_idesc_mx(int M, int N, int a_fmt, int b_fmt) {
  return ((uint32_t)a_fmt << 7) | ((uint32_t)b_fmt << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
         ((uint32_t)(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t umma_idesc_sf_ids(uint32_t idesc, int a_id, int b_id) {
  return idesc | ((uint32_t)b_id << 4) | ((uint32_t)a_id << 29);
}

// D[tmem] (+)= (A * sA) (B * sB)^T; tsfa / tsfb are the tensor-memory
// addresses of the scale columns with the byte index in bits 30-31.
__device__ __forceinline__ void umma_mx(uint32_t tmem_d, uint64_t desc_a, uint64_t desc_b, uint32_t idesc,
                                        uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(tmem_d),
      "l"(desc_a), "l"(desc_b), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb));
}

// The same with both operands packed e2m1 (kind::mxf4, K = 64 per
// instruction, one ue8m0 scale per 32: the scale column's byte pair from the
// index in bits 30-31).
__device__ __forceinline__ void umma_mxf4(uint32_t tmem_d, uint64_t desc_a, uint64_t desc_b, uint32_t idesc,
                                          uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(
          tmem_d),
      "l"(desc_a), "l"(desc_b), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb));
}

// Instruction descriptor of kind::mxf4nvf4 with both operands e2m1 and ue4m3
// scales (bit 23 clear): the NVFP4 block-16 form.
__host__ __device__ constexpr uint32_t umma_idesc_nv(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Both operands packed e2m1 with one ue4m3 scale per 16 elements
// (kind::mxf4nvf4, block16: K = 64 per instruction, the scale column's four
// bytes are the instruction's four blocks).
__device__ __forceinline__ void umma_nvf4(uint32_t tmem_d, uint64_t desc_a, uint64_t desc_b, uint32_t idesc,
                                          uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n}\n" ::"r"(
          tmem_d),
      "l"(desc_a), "l"(desc_b), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb));
}

// Shared-memory descriptor of a scale-factor atom for tcgen05.cp: 32 rows of
// 16 bytes, contiguous (no swizzle; 8-row groups 128 bytes apart).
__device__ __forceinline__ uint64_t umma_desc_sf(const void* smem_atom) {
  const uint64_t addr = (uint64_t)(smem_u32(smem_atom) >> 4) & 0x3FFFu;
  return addr | (8ull << 32) | (1ull << 46);
}

// Copy 32 rows x 128 bits from shared memory into 4 tensor-memory columns of
// lanes 0-31, replicated into the lanes of all four sub-partitions.  Ordered
// with the tcgen05.mma instructions the same thread issues.
__device__ __forceinline__ void utccp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc));
}

// The mbarrier receives one arrival when every tcgen05 operation this thread
// issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Allocation by one whole warp; the TMEM address is written to *dst (smem).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_free(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Writes of this thread to shared memory become visible to the async proxy
// (tensor core, TMA) before a following barrier arrival.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base lane + i),
// registers r[j] = column (base column + j).  The warp may access only the
// lanes 32 * (warp % 4) .. + 31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
      "[%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

}  // namespace qk
