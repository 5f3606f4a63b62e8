// Router (top-k + softmax over the selected logits) and token permutation.
//
// Method statement: top-k over the F32 router logits with warp-level selection, ties to the
// lower expert index, softmax over the k selected logits; then a per-expert histogram, the
// exclusive prefix sum of the counts, and a stable placement of the routed rows expert by
// expert.  Page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents",
// section "What this pack holds" (256 routed experts, 8 active per token); page
// "Beam-1.0-501B-A23B VQ GGUF", section "What stays native" (router logits in FP32).
#include "common.cuh"
#include "internal.h"
#include "route_warp.cuh"

namespace moe {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// Stable placement of rows r0 .. r0+n-1 (n <= 32, one per lane, bins from bin_of) by one warp:
// lanes with the same bin take consecutive slots in lane order, from run[bin] on, and the
// lowest lane of each bin advances run[bin] for the next call.
template <typename BinOf>
__device__ __forceinline__ void place32(int64_t r0, int n, int lane, int* run, const RouteBufs& b, BinOf bin_of) {
  const bool have = lane < n;
  const unsigned act = __ballot_sync(kFull, have);
  if (have) {
    const int64_t r = r0 + lane;
    const int bin = bin_of(r);
    const unsigned peers = __match_any_sync(act, bin);
    const unsigned below = peers & ((1u << lane) - 1u);
    const int pos = run[bin] + __popc(below);
    b.perm[pos] = (int32_t)r;
    b.inv[r] = pos;
    __syncwarp(act);
    if (below == 0u) run[bin] += __popc(peers);
  }
  __syncwarp();
}

// Per-bin exclusive prefix over chunks, in place in chunk_counts ([nchunks][stride]); returns
// bin e's total.  Loads go out 16 at a time so that their latencies overlap.
__device__ __forceinline__ int chunk_prefix(int32_t* cc, int nchunks, int stride, int e) {
  int run = 0;
  int c = 0;
  for (; c + 16 <= nchunks; c += 16) {
    int v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = cc[(size_t)(c + i) * stride + e];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      cc[(size_t)(c + i) * stride + e] = run;
      run += v[i];
    }
  }
  for (; c < nchunks; ++c) {
    int* p = cc + (size_t)c * stride + e;
    const int v = *p;
    *p = run;
    run += v;
  }
  return run;
}

// Exclusive prefix sums of four arrays of n ints in shared memory, in place, by one warp (each
// lane a contiguous run, then a shuffle scan of the runs' sums); the four totals go to tot[0..3].
__device__ __forceinline__ void warp_scan4_excl(int* a0, int* a1, int* a2, int* a3, int n, int* tot) {
  const int lane = threadIdx.x & 31, per = (n + 31) / 32;
  const int lo = min(n, lane * per), hi = min(n, lo + per);
  int s[4] = {0, 0, 0, 0};
  for (int i = lo; i < hi; ++i) {
    s[0] += a0[i];
    s[1] += a1[i];
    s[2] += a2[i];
    s[3] += a3[i];
  }
  int inc[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
  for (int o = 1; o < 32; o <<= 1)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int v = __shfl_up_sync(kFull, inc[j], o);
      if (lane >= o) inc[j] += v;
    }
  int run[4] = {inc[0] - s[0], inc[1] - s[1], inc[2] - s[2], inc[3] - s[3]};
  for (int i = lo; i < hi; ++i) {
    int v = a0[i];
    a0[i] = run[0];
    run[0] += v;
    v = a1[i];
    a1[i] = run[1];
    run[1] += v;
    v = a2[i];
    a2[i] = run[2];
    run[2] += v;
    v = a3[i];
    a3[i] = run[3];
    run[3] += v;
  }
  if (lane == 31)
#pragma unroll
    for (int j = 0; j < 4; ++j) tot[j] = inc[j];
}

// From per-expert counts in shared memory: offsets and the two group lists.  An expert's rows
// are cut into groups of group_rows; when split_singles is set, a last group of a single row
// goes to the one-row list instead.  All full groups (exactly group_rows rows) come first, in
// expert order, then the partial ones: a kernel that hands out groups in list order starts
// with the large work items and fills in with the small ones.  With expert_major, each expert's
// groups are listed together instead (its full groups, then its partial one), so that a kernel
// streaming the list in order reads an expert's weights for all of its groups at about the same
// time (the repeats then come from L2).
__device__ void finish_counts(int* cnt, int* tmp, int* tmp1, int* tmp2, int* warp_tmp, int E, int group_rows,
                              const RouteBufs& b) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = cnt[e], full = c / group_rows, r = c - full * group_rows;
    const int single = (b.split_singles && r == 1) ? 1 : 0;
    const int part = (r > 0 && !single) ? 1 : 0;
    b.counts[e] = c;
    tmp[e] = b.expert_major ? full + part : full;
    tmp2[e] = b.expert_major ? 0 : part;
    tmp1[e] = single;
  }
  __syncthreads();
  // tmp: first full group of e; tmp2: its partial group, after the full ones; tmp1: its one-row
  // group slot; cnt -> offsets (in place)
  if (threadIdx.x < 32) warp_scan4_excl(tmp, tmp2, tmp1, cnt, E, warp_tmp);
  __syncthreads();
  const int nf = warp_tmp[0], np = warp_tmp[1], ns = warp_tmp[2], R = warp_tmp[3];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    b.offsets[e] = cnt[e];
    const int c = b.counts[e];
    const int full = c / group_rows;
    const int single = (b.split_singles && c % group_rows == 1) ? 1 : 0;
    const int rest = c - full * group_rows - single;        // rows of the partial group
    for (int q = 0; q < full; ++q)
      b.groups[tmp[e] + q] = make_int4(e, cnt[e] + q * group_rows, group_rows, 0);
    if (rest > 0)
      b.groups[b.expert_major ? tmp[e] + full : nf + tmp2[e]] = make_int4(e, cnt[e] + full * group_rows, rest, 0);
    if (single) b.singles[tmp1[e]] = make_int4(e, cnt[e] + c - 1, 1, 0);
  }
  if (threadIdx.x == 0) {
    b.offsets[E] = R;
    *b.ngroups = nf + np;
    *b.nsingles = ns;
  }
}

// Single-CTA routing for T <= kOneCtaTokens: router, histogram, scan, groups, stable placement.
__global__ void __launch_bounds__(1024) route_one_cta_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                             RouteBufs b) {
  __shared__ int cnt[kMaxE], tmp[kMaxE], tmp1[kMaxE], tmp2[kMaxE], run[kMaxE], warp_tmp[32];
  __shared__ int sids[kOneCtaTokens * 32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int t = wid; t < T; t += nw) {
    int id;
    float w;
    route_row(logits + (size_t)t * E, E, k, lane, id, w);
    if (lane < k) {
      b.ids[t * k + lane] = id;
      b.w[t * k + lane] = w;
      sids[t * k + lane] = id;
      atomicAdd(&cnt[id], 1);
    }
  }
  __syncthreads();
  finish_counts(cnt, tmp, tmp1, tmp2, warp_tmp, E, b.group_rows, b);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) run[e] = cnt[e];   // cnt now = offsets
  __syncthreads();
  if (wid == 0) {
    const int R = T * k;
    for (int r0 = 0; r0 < R; r0 += 32)
      place32(r0, min(32, R - r0), lane, run, b, [&](int64_t r) { return sids[r]; });
  }
}

// Routing of T <= kRouteChunk tokens in one launch: CTA c routes tokens kSmallTok c .. (one per
// warp) and counts its rows per expert; the last CTA to finish (a counter in the workspace, zero
// at launch) takes every CTA's counts, forms counts, offsets and groups, and places the rows, one
// warp per CTA's rows, each from its own running positions.
__global__ void __launch_bounds__(32 * kSmallTok) route_small_kernel(const float* __restrict__ logits, int T, int E,
                                                                     int k, RouteBufs b) {
  __shared__ int cnt[kMaxE], tmp[kMaxE], tmp1[kMaxE], tmp2[kMaxE], warp_tmp[32];
  __shared__ int s_last;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nch = gridDim.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int t = blockIdx.x * kSmallTok + wid;
  if (t < T) {
    int id;
    float w;
    route_row(logits + (size_t)t * E, E, k, lane, id, w);
    if (lane < k) {
      b.ids[t * k + lane] = id;
      b.w[t * k + lane] = w;
      atomicAdd(&cnt[id], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) b.chunk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();                                   // this CTA's ids and counts before the count
    s_last = atomicAdd(b.done, 1u) == (unsigned)(nch - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();                                     // every CTA's ids and counts after the count
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = chunk_prefix(b.chunk_counts, nch, E, e);
  __syncthreads();
  finish_counts(cnt, tmp, tmp1, tmp2, warp_tmp, E, b.group_rows, b);
  __syncthreads();                                     // cnt = offsets
  // running position of chunk c's next row of expert e, in place in chunk_counts
  for (int i = threadIdx.x; i < nch * E; i += blockDim.x) b.chunk_counts[i] += cnt[i % E];
  __syncthreads();
  for (int c = wid; c < nch; c += kSmallTok) {
    const int r_begin = c * kSmallTok * k, r_end = min(T, (c + 1) * kSmallTok) * k;
    for (int r0 = r_begin; r0 < r_end; r0 += 32)
      place32(r0, min(32, r_end - r0), lane, b.chunk_counts + (size_t)c * E, b,
              [&](int64_t r) { return __ldcg(b.ids + r); });
  }
  if (threadIdx.x == 0) *b.done = 0;                   // for the next call on this workspace
}

// Multi-CTA routing, step 1: route the chunk's tokens and count its rows per expert.
__global__ void __launch_bounds__(512) route_chunk_kernel(const float* __restrict__ logits,
                                                          int64_t T, int E, int k, RouteBufs b) {
  __shared__ int cnt[kMaxE];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kRouteChunk;
  const int nt = (int)(T - t0 < kRouteChunk ? T - t0 : kRouteChunk);
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int i = wid; i < nt; i += nw) {
    const int64_t t = t0 + i;
    int id;
    float w;
    route_row(logits + t * E, E, k, lane, id, w);
    if (lane < k) {
      b.ids[t * k + lane] = id;
      b.w[t * k + lane] = w;
      atomicAdd(&cnt[id], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    b.chunk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

// Multi-CTA routing, step 2 (one CTA): per-expert prefix over chunks, counts, offsets, groups.
__global__ void __launch_bounds__(1024) route_scan_kernel(int nchunks, int E, RouteBufs b) {
  __shared__ int cnt[kMaxE], tmp[kMaxE], tmp1[kMaxE], tmp2[kMaxE], warp_tmp[32];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = chunk_prefix(b.chunk_counts, nchunks, E, e);
  __syncthreads();
  finish_counts(cnt, tmp, tmp1, tmp2, warp_tmp, E, b.group_rows, b);
}

// Multi-CTA routing, step 3: stable placement of the chunk's rows.
__global__ void __launch_bounds__(32) route_scatter_kernel(int64_t T, int E, int k, RouteBufs b) {
  __shared__ int run[kMaxE];
  const int lane = threadIdx.x;
  const int64_t t0 = (int64_t)blockIdx.x * kRouteChunk;
  const int nt = (int)(T - t0 < kRouteChunk ? T - t0 : kRouteChunk);
  for (int e = lane; e < E; e += 32)
    run[e] = b.offsets[e] + b.chunk_counts[(size_t)blockIdx.x * E + e];
  __syncwarp();
  const int64_t r_begin = t0 * k, n = (int64_t)nt * k;
  for (int64_t i = 0; i < n; i += 32)
    place32(r_begin + i, (int)min((int64_t)32, n - i), lane, run, b, [&](int64_t r) { return b.ids[r]; });
}

// Rows with given expert ids (k = 1), step 1: this chunk's rows per bin, bins 0 .. E-1 for the
// experts and bin E for rows whose id lies outside [0, E) (padding rows).
__global__ void __launch_bounds__(256) ids_count_kernel(const int32_t* __restrict__ rows, int64_t R, int E,
                                                        RouteBufs b) {
  __shared__ int cnt[kMaxE + 1];
  const int64_t r0 = (int64_t)blockIdx.x * kRouteChunk;
  const int nr = (int)(R - r0 < kRouteChunk ? R - r0 : kRouteChunk);
  for (int e = threadIdx.x; e <= E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < nr; i += blockDim.x) {
    const int id = rows[r0 + i];
    const bool ok = id >= 0 && id < E;
    b.ids[r0 + i] = ok ? id : -1;
    b.w[r0 + i] = 1.0f;
    atomicAdd(&cnt[ok ? id : E], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e <= E; e += blockDim.x)
    b.chunk_counts[(size_t)blockIdx.x * (E + 1) + e] = cnt[e];
}

// Step 2 (one CTA): per-bin prefix over chunks, then counts, offsets and groups of the experts;
// the padding bin's chunk prefixes are left in chunk_counts and its rows go after all expert
// rows (offsets[E] is the number of expert rows).
__global__ void __launch_bounds__(1024) ids_scan_kernel(int nchunks, int E, RouteBufs b) {
  __shared__ int cnt[kMaxE], tmp[kMaxE], tmp1[kMaxE], tmp2[kMaxE], warp_tmp[32];
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    const int run = chunk_prefix(b.chunk_counts, nchunks, E + 1, e);
    if (e < E) cnt[e] = run;
  }
  __syncthreads();
  finish_counts(cnt, tmp, tmp1, tmp2, warp_tmp, E, b.group_rows, b);
}

// Step 3: stable placement of the chunk's rows, expert rows by expert, padding rows at the end.
__global__ void __launch_bounds__(32) ids_scatter_kernel(int64_t R, int E, RouteBufs b) {
  __shared__ int run[kMaxE + 1];
  const int lane = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.x * kRouteChunk;
  const int nr = (int)(R - r0 < kRouteChunk ? R - r0 : kRouteChunk);
  for (int e = lane; e <= E; e += 32)
    run[e] = b.offsets[e] + b.chunk_counts[(size_t)blockIdx.x * (E + 1) + e];
  __syncwarp();
  for (int i = 0; i < nr; i += 32)
    place32(r0 + i, min(32, nr - i), lane, run, b, [&](int64_t r) {
      const int id = b.ids[r];
      return id < 0 ? E : id;
    });
}

}  // namespace

int launch_route(const float* logits, int64_t T, int E, int k, const RouteBufs& b,
                 cudaStream_t s) {
  if (T <= kOneCtaTokens) {
    route_one_cta_kernel<<<1, 1024, 0, s>>>(logits, (int)T, E, k, b);
    const cudaError_t err = cudaGetLastError();
    return err == cudaSuccess ? 1 : -(int)err;
  }
  if (T <= kRouteChunk) {
    cudaError_t err = cudaMemsetAsync(b.done, 0, sizeof(unsigned), s);
    if (err != cudaSuccess) return -(int)err;
    route_small_kernel<<<(unsigned)((T + kSmallTok - 1) / kSmallTok), 32 * kSmallTok, 0, s>>>(logits, (int)T, E, k, b);
    err = cudaGetLastError();
    return err == cudaSuccess ? 1 : -(int)err;
  }
  const int nch = route_chunks(T);
  route_chunk_kernel<<<nch, 512, 0, s>>>(logits, T, E, k, b);
  route_scan_kernel<<<1, 1024, 0, s>>>(nch, E, b);
  route_scatter_kernel<<<nch, 32, 0, s>>>(T, E, k, b);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 3 : -(int)err;
}

int launch_route_ids(const int32_t* rows, int64_t R, int E, const RouteBufs& b, cudaStream_t s) {
  const int nch = route_chunks(R);
  ids_count_kernel<<<nch, 256, 0, s>>>(rows, R, E, b);
  ids_scan_kernel<<<1, 1024, 0, s>>>(nch, E, b);
  ids_scatter_kernel<<<nch, 32, 0, s>>>(R, E, b);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 3 : -(int)err;
}

}  // namespace moe
