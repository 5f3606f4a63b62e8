// Warp-level router of one token (top-k of E logits, ties to the lower index, NaN lowest,
// softmax over the k selected in f32), shared by the router kernels and the fused decode
// kernel so that both select and weight experts identically.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kMaxE = 1024;
constexpr int kMaxPerLane = kMaxE / 32;

// Order-preserving key of a logit: larger logit -> larger key; -0.0 == +0.0; NaN lowest (0).
__device__ __forceinline__ uint32_t rank_key(float v) {
  uint32_t b = __float_as_uint(v);
  if (v != v) return 0u;
  if ((b << 1) == 0u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One warp selects the top k (k <= 32) of a row of E (<= 1024) logits.  Lane j < k gets the
// rank-j expert and its softmax weight.  Keys combine the logit key with the complemented
// index so that a larger combined key is a higher rank (ties to the lower index).
template <int PER_LANE>
__device__ void warp_route_row(const float* __restrict__ row, int E, int k, int lane, int& id,
                               float& weight) {
  uint64_t key[PER_LANE];
  uint64_t best = 0;
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0;
    if (e < E) key[i] = ((uint64_t)rank_key(__ldg(row + e)) << 32) | (uint32_t)(0xFFFFFFFFu - e);
    best = key[i] > best ? key[i] : best;
  }
  id = 0;
  for (int r = 0; r < k; ++r) {
    uint64_t m = best;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xFFFFFFFFu, m, off);
      m = o > m ? o : m;
    }
    const int e = (int)(0xFFFFFFFFu - (uint32_t)m);
    if (lane == r) id = e;
    if (lane == (e & 31)) {
      const int slot = e >> 5;
      best = 0;
#pragma unroll
      for (int i = 0; i < PER_LANE; ++i) {
        if (i == slot) key[i] = 0;
        best = key[i] > best ? key[i] : best;
      }
    }
  }
  const float l = lane < k ? __ldg(row + id) : 0.0f;
  const float lmax = __shfl_sync(0xFFFFFFFFu, l, 0);
  float ex = lane < k ? expf(l - lmax) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
  weight = ex / sum;
}

__device__ __forceinline__ void route_row(const float* row, int E, int k, int lane, int& id, float& w) {
  if (E <= 32 * 8)
    warp_route_row<8>(row, E, k, lane, id, w);
  else
    warp_route_row<kMaxPerLane>(row, E, k, lane, id, w);
}


}  // namespace moe
