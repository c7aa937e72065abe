// qk_group.cuh -- workspace of the grouped (prefill) path, shared by the f16
// grouped GEMMs (qk_group.cu) and the MXFP4 block-scaled ones (qk_gmx.cu).
#pragma once

#include <cuda_fp16.h>

#include "qk_internal.h"

namespace qk {

constexpr int kGN = 256;          // f16 path: token rows per tile (largest tcgen05 N)
constexpr int kXN = 80;           // MXFP4 path: token rows per tile (terms x rows <= 240 MMA columns)
constexpr int kXK = 128;          // MXFP4 path: reduction per stage (four 32-element scale blocks)
constexpr int kSfAtom = 512;      // scale-factor atom: 128 rows x 4 blocks, tensor-memory copy layout
constexpr int kScanThreads = 1024;
constexpr int kRowThreads = 128;

struct GroupWs {
  int* counts;      // [E] pairs per expert
  int* offsets;     // [E + 1] first sorted row of each expert
  int* fill;        // [E] scatter cursors
  int* tile_e;      // [F] expert of token tile f
  int* tile_row0;   // [F] first sorted row of token tile f
  int* tile_n;      // [F] rows in token tile f
  int* n_tiles;     // [1] token tiles
  int* inv;         // [P] pair -> sorted row
  float* dperm;     // [P][H] fp32 down-projection result of each sorted row
  unsigned long long* n_flush;  // [1] MXFP4 blocks flushed by the relative scaling (f16 path)
  size_t zero_bytes;            // bytes zeroed from `counts` on every call
  // f16 path
  int* xshift;      // [P] per sorted row: x scaled by 2^-xshift
  int* hshift;      // [P] per sorted row: h scaled by 2^-hshift
  __half* xperm;    // [P][H] f16
  float* hperm;     // [P][I] fp32
  __half* h16;      // [P][I] f16
  // MXFP4 block-scaled path
  int* tile_first;  // [F] first token tile of the expert of tile f
  int* tile_cnt;    // [F] token tiles of the expert of tile f
  int* exp_tile0;   // [E] first token tile of expert e
  int* rtile;       // [P] per sorted row: (token tile << 8) | row within the tile
  uint8_t* xq;      // [2][P][H] e4m3 terms of x (x = t0 * 2^s0 + t1 * 2^s1 per 32-block)
  uint8_t* sfx;     // [F][H / 128][2][512] ue8m0 block scales of the stacked x terms, atom layout
  float* gu;        // [P][2 I] fp32 gate (first I) and up (last I) projections
  uint8_t* hq;      // [3][P][I] e4m3 terms of h = silu(gate) * up
  uint8_t* sfh;     // [F][I / 128][2][512] ue8m0 block scales of the stacked h terms, atom layout
};

// The MXFP4 block-scaled path takes a layer when all three projections are
// MXFP4, hidden and inter are multiples of 512 and the packed weights (32 B)
// and scales (16 B) are aligned for its copies.
bool gmx_eligible(const qk_weight& gate, const qk_weight& up, const qk_weight& down, int H, int I);

// x split, gate/up GEMM, h split, down GEMM of the MXFP4 path (the counting
// sort has run; the combine follows).
qk_status gmx_forward(const DecodeArgs& a, const GroupWs& W, cudaStream_t st);

}  // namespace qk
