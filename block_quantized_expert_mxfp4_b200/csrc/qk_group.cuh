// qk_group.cuh -- workspace of the grouped (prefill) path, shared by the f16
// grouped GEMMs (qk_group.cu) and the MXFP4 block-scaled ones (qk_gmx.cu).
#pragma once

#include <cuda_fp16.h>

#include "qk_internal.h"

namespace qk {

constexpr int kGN = 256;          // f16 path: token rows per tile (largest tcgen05 N)
constexpr int kXK = 128;          // MXFP4 path: reduction per step (four 32-element scale blocks)
constexpr int kXTok1 = 64;        // MXFP4 path: tokens per gate/up tile (2 terms x 16 per TMEM lane quadrant)
constexpr int kXTok2 = 40;        // MXFP4 path: tokens per down tile (3 terms x 10 per quadrant)
constexpr int kSfAtom = 512;      // scale-factor atom: 128 rows x 4 blocks, tensor-memory copy layout
constexpr int kXBlock = 128 * kXK;  // one reduction step of a token tile: 128 rows x 128 e4m3 (16 KB)
constexpr int kScanThreads = 1024;
constexpr int kRowThreads = 128;

// Token tiles (<= tn rows of one expert's sorted rows).
struct TileList {
  int* tile_e;      // [F] expert of token tile f
  int* tile_row0;   // [F] first sorted row of token tile f
  int* tile_n;      // [F] rows in token tile f
  int* tile_first;  // [F] first token tile of the expert of tile f (MXFP4 path)
  int* tile_cnt;    // [F] token tiles of the expert of tile f (MXFP4 path)
  int* exp_tile0;   // [E] first token tile of expert e (MXFP4 path)
  int* n_tiles;     // [1] token tiles
};

struct GroupWs {
  int* counts;      // [E] pairs per expert
  int* offsets;     // [E + 1] first sorted row of each expert
  int* fill;        // [E] scatter cursors
  TileList L1;      // f16 path: tiles of kGN rows; MXFP4 path: gate/up tiles of kXTok1 rows
  TileList L2;      // MXFP4 path: down tiles of kXTok2 rows
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
  // MXFP4 block-scaled path.  A token tile's operand per reduction step is a
  // 128-row block (the tcgen05 A operand, 128-byte swizzled): row
  // 32 q + n_t t + i holds term t of the tile's token n_t q + i (n_t = 16
  // tokens per quadrant for x, 10 for h), and its 512-byte scale atom.
  int* rtile2;      // [P] per sorted row: (down tile << 8) | row within it
  uint8_t* xt;      // [F1][H / 128] blocks of the x terms (x = t0 2^s0 + t1 2^s1 per 32-block)
  uint8_t* sfx;     // [F1][H / 128][512] ue8m0 scales of the x terms, atom layout
  float* gu;        // [P][2 I] fp32 gate (first I) and up (last I) projections
  uint8_t* ht;      // [F2][I / 128] blocks of the 3 e4m3 terms of h = silu(gate) * up
  uint8_t* sfh;     // [F2][I / 128][512] ue8m0 scales of the h terms, atom layout
  // NVFP4 layers in QK_ACT_MXFP4 (kind::mxf4nvf4): the token scales are ue4m3
  // per 16 (twice the atoms of the MXFP4 tiles), re-anchored per row; the row's
  // factor 2^(cmax - 135) restores them in the epilogue.
  float* fac1;      // [P] per sorted row: x scale factor
  float* fac2;      // [P] per sorted row: h scale factor
};

// The MXFP4 block-scaled path takes a layer when all three projections are
// MXFP4, hidden and inter are multiples of 512 and the packed weights (32 B)
// and scales (16 B) are aligned for its copies.
bool gmx_eligible(const qk_weight& gate, const qk_weight& up, const qk_weight& down, int H, int I);
// The same kernels take an all-NVFP4 layer in QK_ACT_MXFP4 (fp4 x fp4 on
// kind::mxf4nvf4, ue4m3 block scales per 16): same shape and alignment rules.
bool gmx_nv_eligible(const qk_weight& gate, const qk_weight& up, const qk_weight& down, int H, int I);
// The FP8 shared expert's two GEMMs on the block-scaled grouped kernels.
qk_status gmx_fp8_ffn(const GroupWs& W, const uint16_t* x, const int32_t* ids, int M, int H, int I,
                      const uint8_t* wg, const uint8_t* sg, const uint8_t* wu, const uint8_t* su,
                      const uint8_t* wd, const uint8_t* sd, int blk, cudaStream_t st);

inline int g_max_tiles(int P, int E, int tn) { return P / tn + E + 1; }

}  // namespace qk
