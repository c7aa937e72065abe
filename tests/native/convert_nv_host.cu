// Host build of the library's NVFP4 -> MXFP4 block rule (qk_convert_nv.h),
// for the CPU test that compares it with the oracle.  Test infrastructure
// only: built into tests/_build by tests/test_convert_nv_host.py.
#include "qk_convert_nv.h"

// Blocks given as e4m3 code pairs (2 bytes each) with one scale_2 per block.
extern "C" void convert_nv_host(const uint8_t* e4m3, const float* scale_2, int n, uint8_t* e8m0,
                                unsigned long long* n_inexact, int* n_nan) {
  unsigned long long bad = 0;
  int nn = 0;
  for (int i = 0; i < n; ++i) {
    const double s2 = (double)scale_2[i];
    bool inexact = false, nan = false;
    e8m0[i] = (uint8_t)qk::nv_block_code(qk::nv_e4m3_to_double(e4m3[2 * i]) * s2,
                                         qk::nv_e4m3_to_double(e4m3[2 * i + 1]) * s2, inexact, nan);
    bad += inexact;
    nn += nan;
  }
  *n_inexact = bad;
  *n_nan = nn;
}
