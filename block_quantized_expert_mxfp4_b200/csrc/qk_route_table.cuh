// qk_route_table.cuh -- routing tables of the decode kernels: the (token,
// slot) pairs grouped by expert into virtual experts of at most kTileN pairs.
#pragma once

#include "qk_common.cuh"

namespace qk {

// --------------------------------------------------------------- routing --
struct Route {
  int n_v;                         // virtual experts
  int16_t v_expert[kMaxPairs];
  int16_t v_p0[kMaxPairs];         // first entry in pair_list
  int8_t v_n[kMaxPairs];           // pairs (1..8)
  int16_t pair_list[kMaxPairs];    // pairs grouped by expert, ascending pair index
  int16_t pair_v[kMaxPairs];       // virtual expert of pair p (-1: invalid id)
  int8_t pair_j[kMaxPairs];        // column of pair p in its virtual expert
  int16_t tmp_e[kMaxPairs];
  int8_t tmp_first[kMaxPairs];
  int16_t act_cnt[kMaxPairs];
  int16_t act_off[kMaxPairs + 1];
  int16_t act_v0[kMaxPairs + 1];
};

__device__ __forceinline__ void place_pair(Route& R, int p, int e, int slot, int rank, int total) {
  const int pos = R.act_off[slot] + rank;
  R.pair_list[pos] = (int16_t)p;
  const int v = R.act_v0[slot] + rank / kTileN;
  R.pair_v[p] = (int16_t)v;
  R.pair_j[p] = (int8_t)(rank % kTileN);
  if (rank % kTileN == 0) {
    R.v_expert[v] = (int16_t)e;
    R.v_p0[v] = (int16_t)pos;
    R.v_n[v] = (int8_t)min(kTileN, total - rank);
  }
}

// Routing tables from the ids.  Active experts ascend by id; the pairs of one
// expert ascend by pair index.  P <= 32: one warp with match/ballot; larger P:
// one pair per thread (P <= kMaxPairs <= blockDim).
__device__ inline void build_route(const int32_t* __restrict__ ids, int P, int E, Route& R) {
  const int tid = threadIdx.x, lane = tid & 31;
  if (P <= 32) {
    if (tid < 32) {
      int e = -1;
      if (lane < P) {
        e = ids[lane];
        if (e < 0 || e >= E) {
          set_status(QK_ERR_INVALID_ARG);
          e = -1;
        }
        R.pair_v[lane] = -1;
      }
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      const bool valid = e >= 0;
      const bool first = valid && (__ffs(peers) - 1 == lane);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int total = __popc(peers);
      const unsigned firsts = __ballot_sync(0xffffffffu, first);
      int slot = 0;
      for (int i = 0; i < 32; ++i) {
        const int ei = __shfl_sync(0xffffffffu, e, i);
        slot += ((firsts >> i) & 1u) && ei < e;
      }
      const int n_active = __popc(firsts);
      if (first) R.act_cnt[slot] = (int16_t)total;
      __syncwarp();
      const int cnt = lane < n_active ? R.act_cnt[lane] : 0;
      const int vcnt = (cnt + kTileN - 1) / kTileN;
      int off = cnt, v0 = vcnt;  // inclusive scans over active slots
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, off, o), b = __shfl_up_sync(0xffffffffu, v0, o);
        if (lane >= o) {
          off += a;
          v0 += b;
        }
      }
      if (lane <= n_active) {
        R.act_off[lane] = (int16_t)(off - cnt);
        R.act_v0[lane] = (int16_t)(v0 - vcnt);
      }
      const int n_v = __shfl_sync(0xffffffffu, v0, 31);
      if (lane == 0) R.n_v = n_v;
      __syncwarp();
      if (valid) place_pair(R, lane, e, slot, rank, total);
    }
    __syncthreads();
    return;
  }
  const int p = tid;
  int e = -1;
  if (p < P) {
    e = ids[p];
    if (e < 0 || e >= E) {
      set_status(QK_ERR_INVALID_ARG);
      e = -1;
    }
    R.tmp_e[p] = (int16_t)e;
    R.pair_v[p] = -1;
  }
  __syncthreads();
  int first = (e >= 0);
  for (int q = 0; q < p && first && p < P; ++q) first = (R.tmp_e[q] != e);
  if (p < P) R.tmp_first[p] = (int8_t)first;
  const int n_active = __syncthreads_count(first);
  int slot = 0, rank = 0, total = 0;
  if (e >= 0) {
    for (int q = 0; q < P; ++q) {
      const int eq = R.tmp_e[q];
      slot += (R.tmp_first[q] && eq >= 0 && eq < e);
      rank += (q < p && eq == e);
      total += (eq == e);
    }
    if (first) R.act_cnt[slot] = (int16_t)total;
  }
  __syncthreads();
  if (p <= n_active) {
    int off = 0, v0 = 0;
    for (int a = 0; a < p; ++a) {
      off += R.act_cnt[a];
      v0 += (R.act_cnt[a] + kTileN - 1) / kTileN;
    }
    R.act_off[p] = (int16_t)off;
    R.act_v0[p] = (int16_t)v0;
  }
  __syncthreads();
  if (e >= 0) place_pair(R, p, e, slot, rank, total);
  if (p == 0) R.n_v = R.act_v0[n_active];
  __syncthreads();
}

}  // namespace qk
