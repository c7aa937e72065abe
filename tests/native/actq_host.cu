// Host build of the library's activation-quantization arithmetic
// (qk_actq.cuh), for the CPU test that compares it with the oracle.  Test
// infrastructure only: built into tests/_build by tests/test_actq_host.py.
#define QK_ACTQ_ARITHMETIC_ONLY
#include "qk_actq.cuh"

// n values (n % 32 == 0) -> one e4m3 code per value (e4m3 of the e2m1 value
// in fp4 mode) and one e8m0 code per 32.
extern "C" void actq_host(const float* v, int n, int fp4, uint8_t* codes, uint8_t* scales) {
  for (int b = 0; b < n / 32; ++b) {
    float blk[32];
    uint32_t q[8];
    for (int i = 0; i < 32; ++i) blk[i] = v[b * 32 + i];
    scales[b] = (uint8_t)qk::actq_block(blk, q, fp4);
    memcpy(codes + b * 32, q, 32);
  }
}

// The packed e2m1 form of the fp4 x fp4 tiles: 16 bytes per 32 values
// (element 2 i in the low nibble of byte i) and one e8m0 code per 32.
extern "C" void actq_host_fp4packed(const float* v, int n, uint8_t* packed, uint8_t* scales) {
  for (int b = 0; b < n / 32; ++b) {
    float blk[32];
    uint32_t q[4];
    for (int i = 0; i < 32; ++i) blk[i] = v[b * 32 + i];
    scales[b] = (uint8_t)qk::actq_block_fp4(blk, q);
    memcpy(packed + b * 16, q, 16);
  }
}

// The NVFP4 form of the same tiles (kind::mxf4nvf4): per row of n values
// (n % 32 == 0) the packed codes, one ue4m3 code per 32-block (both 16-halves
// take it) re-anchored at the row's largest 32-block code, and the row's
// factor; the split kernels' two passes, in order.
extern "C" void actq_host_nv_rows(const float* v, int rows, int n, uint8_t* packed, uint8_t* codes, float* fac) {
  for (int r = 0; r < rows; ++r) {
    const float* row = v + (size_t)r * n;
    int cm = 0;
    for (int b = 0; b < n / 32; ++b) {
      float blk[32];
      uint32_t q[4];
      for (int i = 0; i < 32; ++i) blk[i] = row[b * 32 + i];
      const int c = qk::actq_block_fp4(blk, q);
      cm = cm > c ? cm : c;
    }
    for (int b = 0; b < n / 32; ++b) {
      float blk[32];
      uint32_t q[4];
      for (int i = 0; i < 32; ++i) blk[i] = row[b * 32 + i];
      const int c = qk::actq_block_fp4(blk, q);
      codes[(size_t)r * (n / 32) + b] = (uint8_t)qk::actq_nv_code(c - cm + 8);
      memcpy(packed + (size_t)r * (n / 2) + b * 16, q, 16);
    }
    fac[r] = qk::actq_pow2(cm - 135);
  }
}

extern "C" unsigned actq_host_nv_code(int d) { return qk::actq_nv_code(d); }
extern "C" float actq_host_pow2(int e) { return qk::actq_pow2(e); }
