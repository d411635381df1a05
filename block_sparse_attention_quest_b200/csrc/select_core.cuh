// Helpers shared by the score/selection kernels (select.cu) and the
// one-launch decode kernel (decode_coop.cu): the transposed segment sum of
// the pooled Quest bound, the order-preserving score keys, block scans and
// the exact ranking of a threshold bin's members.
#pragma once

#include "launch.h"

namespace resa {

// Sum U per-lane values over aligned segments of W lanes, transposed so that
// each round halves the number of live values: after the call lane `l` holds
// the full segment sum of value index seg_value_index<U, W>(l) in v[0].
template <int U, int W>
__device__ __forceinline__ float transpose_reduce(float (&v)[U], int lane) {
  int count = U;
#pragma unroll
  for (int m = W / 2; m >= 1; m >>= 1) {
    if (count > 1) {
      const int half = count / 2;
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < U / 2; ++i) {
        if (i < half) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      count = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
  return v[0];
}
template <int U, int W>
__device__ __forceinline__ int seg_value_index(int lane) {
  int idx = 0, count = U;
#pragma unroll
  for (int m = W / 2; m >= 1; m >>= 1) {
    if (count > 1) {
      count /= 2;
      if (lane & m) idx += count;
    }
  }
  return idx;
}

// lanes that hold a unique reduced value: the low log2(W / U) lane bits are 0
template <int U, int W>
__device__ __forceinline__ bool seg_value_owner(int lane) {
  constexpr int dup = W / U;   // lanes sharing one value
  return (lane % dup) == 0;
}

constexpr int kBins = 2048;           // first pass: the top 11 bits of the key offset
constexpr int kCand = 1024;           // threshold-bin candidates resolved by rank

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f == 0.0f) u = 0u;                          // -0 and +0 are the same score
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// exclusive prefix sum over the block; returns the thread's offset and writes
// the block total to *total
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t x, uint32_t* warp_tot,
                                                         uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    uint32_t t = lane < nw ? warp_tot[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    if (lane < nw) warp_tot[lane] = ti - t;        // exclusive warp offsets
    if (lane == 31) *total = ti;
  }
  __syncthreads();
  const uint32_t r = warp_tot[warp] + inc - x;
  __syncthreads();
  return r;
}

// Sum of x over the block's warps (one value per warp, lane 0 holds it);
// returns the exclusive prefix of this warp and writes the total.
__device__ __forceinline__ uint32_t warp_exclusive_offset(uint32_t x, uint32_t* warp_tot,
                                                          uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    const uint32_t t = lane < nw ? warp_tot[lane] : 0u;
    uint32_t inc = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane < nw) warp_tot[lane] = inc - t;
    if (lane == 31) *total = inc;
  }
  __syncthreads();
  const uint32_t r = warp_tot[warp];
  __syncthreads();
  return r;
}

// The threshold bin's c members (any order) ranked by key descending, then
// index ascending: the member of rank take - 1 is the last one kept (the cut).
// One warp per member, its lanes comparing it with 32 members at a time, so a
// member costs c / 32 ballots rather than c dependent shared-memory reads.
// Indices are distinct, so ranks are too and exactly one member writes the cut.
__device__ __forceinline__ void rank_cut(const uint32_t* cand_rel, const int* cand_j, int c,
                                         uint32_t take, uint32_t* cut_rel, int* cut_j) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int i = warp; i < c; i += nw) {
    const uint32_t r = cand_rel[i];
    const int j = cand_j[i];
    uint32_t rank = 0;
    for (int k0 = 0; k0 < c; k0 += 32) {
      const int k = k0 + lane;
      bool better = false;
      if (k < c) {
        const uint32_t rk = cand_rel[k];
        better = rk > r || (rk == r && cand_j[k] < j);
      }
      rank += __popc(__ballot_sync(0xffffffffu, better));
    }
    if (lane == 0 && rank + 1 == take) {
      *cut_rel = r;
      *cut_j = j;
    }
  }
}

// kept: at or above the cut in (key descending, index ascending) order
__device__ __forceinline__ bool at_or_above(uint32_t rel, int j, uint32_t cut_rel, int cut_j) {
  return rel > cut_rel || (rel == cut_rel && j <= cut_j);
}

}  // namespace resa
