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
// rank-j expert and its softmax weight.  Expert e sits in lane e % 32, slot e / 32.  Each round
// takes the largest key over the lanes' current candidates with one warp max-reduction, then
// the lowest expert index among the lanes holding that key with one min-reduction (ties to the
// lower index); the winning lane drops that entry and rescans its own slots.
template <int PER_LANE>
__device__ void warp_route_row(const float* __restrict__ row, int E, int k, int lane, int& id,
                               float& weight) {
  uint32_t key[PER_LANE];
  uint32_t avail = 0;                                    // bit i: slot i is still a candidate
#pragma unroll
  for (int i = 0; i < PER_LANE; ++i) {
    const int e = lane + 32 * i;
    key[i] = 0;
    if (e < E) {
      key[i] = rank_key(__ldg(row + e));
      avail |= 1u << i;
    }
  }
  // The lane's best candidate: the largest key, the lowest slot on ties; slot -1 if none.
  uint32_t bk = 0;
  int bi = -1;
  auto rescan = [&]() {
    bk = 0;
    bi = -1;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i)
      if (((avail >> i) & 1u) && (bi < 0 || key[i] > bk)) {
        bk = key[i];
        bi = i;
      }
  };
  rescan();
  id = 0;
  for (int r = 0; r < k; ++r) {
    const bool has = bi >= 0;
    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, has ? bk : 0u);
    const uint32_t e = __reduce_min_sync(0xFFFFFFFFu, (has && bk == m) ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu);
    if (lane == r) id = (int)e;
    // Every lane rescans (no divergence); only the winning lane's candidates changed.
    if (lane == (int)(e & 31u)) avail &= ~(1u << (e >> 5));
    rescan();
  }
  const float l = lane < k ? __ldg(row + id) : 0.0f;
  const float lmax = __shfl_sync(0xFFFFFFFFu, l, 0);
  float ex = lane < k ? expf(l - lmax) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
  weight = ex / sum;
}

// The same selection for E <= 256 with each lane's 8 candidates sorted once (bitonic network
// on (key, complemented index) pairs): a round then only compares the lanes' list heads and
// shifts the winning lane's list, with no per-round rescan.
__device__ __forceinline__ void warp_route_row_sorted8(const float* __restrict__ row, int E, int k, int lane,
                                                       int& id, float& weight) {
  uint64_t v[8];                                         // (key << 32) | (2^32 - 1 - e); 0 = none
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? ((uint64_t)rank_key(__ldg(row + e)) << 32) | (uint32_t)(0xFFFFFFFFu - e) : 0ull;
  }
#pragma unroll
  for (int kk = 2; kk <= 8; kk <<= 1)
#pragma unroll
    for (int jj = kk >> 1; jj > 0; jj >>= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int l = i ^ jj;
        if (l > i) {
          const bool desc = (i & kk) == 0;
          const uint64_t a = v[i], b = v[l];
          if ((a < b) == desc) {
            v[i] = b;
            v[l] = a;
          }
        }
      }
  id = 0;
  for (int r = 0; r < k; ++r) {
    const uint64_t head = v[0];
    const uint32_t hi = (uint32_t)(head >> 32);
    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, head != 0ull ? hi : 0u);
    const uint32_t e =
        __reduce_min_sync(0xFFFFFFFFu, (head != 0ull && hi == m) ? 0xFFFFFFFFu - (uint32_t)head : 0xFFFFFFFFu);
    if (lane == r) id = (int)e;
    const bool pop = lane == (int)(e & 31u);
#pragma unroll
    for (int i = 0; i < 7; ++i) v[i] = pop ? v[i + 1] : v[i];
    v[7] = pop ? 0ull : v[7];
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
    warp_route_row_sorted8(row, E, k, lane, id, w);
  else
    warp_route_row<kMaxPerLane>(row, E, k, lane, id, w);
}


}  // namespace moe
