// schedule.cuh -- how the split-KV decode partitions work, shared by the decode kernel
// (which writes partial results) and the combine kernel (which finds and merges them).
//
// The batch's cached tokens are cut into tiles of NT tokens per sequence
// (ceil(L_s / NT) tiles for sequence s) and the tiles of all sequences are laid end to
// end.  Group g of G (one group = d_c / 128 CTAs, one per 128-wide slice of the latent) streams
// the contiguous tile range [floor(g*T/G), floor((g+1)*T/G)), which may cover the end of
// one sequence and the start of the next.  Each (group, sequence) pair it touches is one
// "segment" and leaves one partial softmax state in workspace slot g + s; that map is
// one-to-one because a group's sequences are contiguous and groups advance monotonically.
#pragma once

#include <cstdint>

namespace hra {

constexpr int kMaxBatch = 1024;

// Group whose tile range contains tile t (T tiles over G groups, T > 0).
__device__ __forceinline__ int group_of_tile(int t, int G, int T) {
  return static_cast<int>(((static_cast<long long>(t) + 1) * G - 1) / T);
}
__device__ __forceinline__ int group_tile_begin(int g, int G, int T) {
  return static_cast<int>(static_cast<long long>(g) * T / G);
}

// Sequence that owns tile t (0 <= t < prefix[B]): the smallest s with prefix[s + 1] > t.
__device__ __forceinline__ int seq_of_tile(const int* prefix, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid + 1] > t) hi = mid; else lo = mid + 1;
  }
  return lo;
}

// Exclusive prefix of tiles per sequence into prefix[0..B] (prefix[B] = total), computed
// by one full warp; lanes load 32 lengths at a time.
__device__ __forceinline__ void tile_prefix_warp(const int32_t* __restrict__ seq_lens, int B, int NT,
                                                 int* prefix) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int base = 0; base < B; base += 32) {
    const int s = base + lane;
    int L = s < B ? seq_lens[s] : 0;
    int tiles = L > 0 ? (L + NT - 1) / NT : 0;
    int incl = tiles;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (s < B) prefix[s] = carry + incl - tiles;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) prefix[B] = carry;
}

}  // namespace hra
