// Expert parallelism across GPUs: the layer's experts split evenly over G ranks (rank d holds
// global experts d*El .. d*El+El-1, El = E / G), each rank routing its own tokens over all E.
// Three kernels move the routed rows over peer memory (NVLink / NVSwitch) without a collective
// on the data path:
//   plan      from the count matrix C[s][g] (rows rank s routes to global expert g, gathered
//             from every rank) the place of this rank's rows in every receiver's buffer and the
//             local expert id of every row this rank receives;
//   dispatch  reads each token's row once and stores it straight into the receive buffer of the
//             owner of each of its k experts (a peer pointer), expert-major there: for local
//             expert e, the rows of rank 0, then of rank 1, ...; the receiver's expert kernels
//             then read them in place;
//   combine   reads each routed row's expert output back from the owner's output buffer (peer
//             loads) and forms out[t] = bf16(sum_j w[t, j] * y[t, j]) with the layer's own f32
//             accumulation order.
// The official deployment of the model runs tensor and expert parallelism over eight GPUs (page
// "Beam 1.0 501B", the model-information page's introduction: TP8/EP8); the workstation recipe
// uses tensor parallelism over four (page "Running Beam-1.0 (501B) on workstation GPUs", its
// serving command).
#include <cuda_runtime.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kPlanThreads = 1024;
constexpr int kPlanRowsPerCta = 8 * kPlanThreads;

// C [G][E] row-major.  Layout 0 (expert-major receive buffers, the dispatch kernel's): rank d's
// buffer holds, for e = 0 .. El-1, the rows of global expert d*El+e from rank 0, 1, ....
// Layout 1 (source-major, an all-to-all's): the rows from rank 0 (expert by expert), then from
// rank 1, ....  CTA 0 writes dst_off[g], where this rank's first row of expert g lands in its
// owner's buffer; every CTA fills its share of recv_ids, the local expert of each row of this
// rank's own buffer (-1 past the rows the count matrix sends here).
__global__ void __launch_bounds__(kPlanThreads) ep_plan_kernel(const int32_t* __restrict__ C, int G, int E, int rank,
                                                               int layout, int32_t* __restrict__ dst_off,
                                                               int32_t* __restrict__ recv_ids, int64_t recv_rows) {
  extern __shared__ int sm[];
  int* tot = sm;            // [E]: rows of expert g over all ranks
  int* seg = sm + E;        // [El * G]: this rank's receive segments in buffer order -> their starts
  __shared__ int s_total;      // rows sent to this rank
  const int El = E / G, nseg = El * G;
  for (int i = threadIdx.x; i < nseg; i += blockDim.x) {
    int e, s;
    if (layout == 0) e = i / G, s = i - (i / G) * G;
    else s = i / El, e = i - (i / El) * El;
    seg[i] = C[(size_t)s * E + rank * El + e];
  }
  if (blockIdx.x == 0) {
    for (int g = threadIdx.x; g < E; g += blockDim.x) {
      int a = 0;
      for (int s = 0; s < G; ++s) a += C[(size_t)s * E + g];
      tot[g] = a;
    }
  }
  __syncthreads();
  // exclusive prefix of seg by warp 0: each lane a contiguous run
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x, per = (nseg + 31) / 32;
    const int lo = lane * per, hi = min(nseg, lo + per);
    int sum = 0;
    for (int i = lo; i < hi; ++i) sum += seg[i];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int i = lo; i < hi; ++i) {
      const int v = seg[i];
      seg[i] = run;
      run += v;
    }
    if (lane == 31) s_total = incl;
  }
  __syncthreads();
  const int total = s_total;
  if (blockIdx.x == 0) {
    for (int g = threadIdx.x; g < E; g += blockDim.x) {
      const int d = g / El, e = g - d * El;
      int off = 0;
      if (layout == 0) {
        for (int e2 = 0; e2 < e; ++e2) off += tot[d * El + e2];
        for (int s = 0; s < rank; ++s) off += C[(size_t)s * E + g];
      } else {
        for (int s = 0; s < rank; ++s)
          for (int e2 = 0; e2 < El; ++e2) off += C[(size_t)s * E + d * El + e2];
        for (int e2 = 0; e2 < e; ++e2) off += C[(size_t)rank * E + d * El + e2];
      }
      dst_off[g] = off;
    }
  }
  // each row: the last segment whose start is <= the row (earlier segments with the same start
  // are empty)
  const int64_t r0 = (int64_t)blockIdx.x * kPlanRowsPerCta;
  const int64_t r1 = min(recv_rows, r0 + kPlanRowsPerCta);
  for (int64_t r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
    if (r >= total) {
      recv_ids[r] = -1;
      continue;
    }
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (seg[mid] <= r) lo = mid; else hi = mid - 1;
    }
    recv_ids[r] = layout == 0 ? lo / G : lo % El;
  }
}

constexpr int kMoveThreads = 128;
constexpr int kMaxVec = 8;          // 16-byte vectors per thread per row: H <= 8 * 128 * 8 = 8192

struct PeerPtrs {
  void* p[kEpMaxRanks];
};

// One CTA per token in turn (grid-stride over tokens): the token's row of x is read once into
// registers and stored to the owner of each of its k experts, routed row r = t*k+j going to row
// dst_off[g] + (inv[r] - offsets[g]) of that owner's receive buffer.
__global__ void __launch_bounds__(kMoveThreads) ep_dispatch_kernel(const uint16_t* __restrict__ x, int64_t T, int k,
                                                                   int H, const int32_t* __restrict__ ids,
                                                                   const int32_t* __restrict__ inv,
                                                                   const int32_t* __restrict__ offsets,
                                                                   const int32_t* __restrict__ dst_off, int El,
                                                                   int E, int64_t cap, PeerPtrs recv) {
  const int nv = H / 8;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    uint4 v[kMaxVec];
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i)
      if (threadIdx.x + i * kMoveThreads < nv) v[i] = src[threadIdx.x + i * kMoveThreads];
    for (int j = 0; j < k; ++j) {
      const int64_t r = t * k + j;
      const int g = ids[r];
      if ((unsigned)g >= (unsigned)E) continue;     // not an expert id: store nothing
      const int d = g / El;
      const int64_t pos = (int64_t)dst_off[g] + (inv[r] - offsets[g]);
      if (pos < 0 || pos >= cap) continue;          // a plan that does not fit: store nothing
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(recv.p[d]) + (size_t)pos * H);
#pragma unroll
      for (int i = 0; i < kMaxVec; ++i)
        if (threadIdx.x + i * kMoveThreads < nv) dst[threadIdx.x + i * kMoveThreads] = v[i];
    }
  }
  // Order the CTA's stores (to peers) before anything the stream does after the kernel, at system
  // scope: the barrier that follows the dispatch then publishes them to their owners.  The CTA
  // barrier orders every thread's stores before thread 0's fence, which is cumulative; one fence
  // per CTA instead of one per thread (a system-scope fence in every thread was this kernel's
  // largest stall).
  __syncthreads();
  if (threadIdx.x == 0) __threadfence_system();
}

// out[t] = bf16(sum_j w[t, j] * y_owner(t, j)), j = 0 .. k-1 in order with fmaf, as the layer's
// combine; y of routed row r = t*k+j is row dst_off[g] + (inv[r] - offsets[g]) of the output
// buffer of g's owner.  One thread per 8 columns of a token.
__global__ void __launch_bounds__(256) ep_combine_kernel(int64_t T, int k, int H, const int32_t* __restrict__ ids,
                                                         const float* __restrict__ w,
                                                         const int32_t* __restrict__ inv,
                                                         const int32_t* __restrict__ offsets,
                                                         const int32_t* __restrict__ dst_off, int El, int E,
                                                         int64_t cap, PeerPtrs ys,
                                                         const uint16_t* __restrict__ x, uint16_t* __restrict__ out,
                                                         uint16_t* __restrict__ x_next) {
  const int per_row = H / 8;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * per_row) return;
  const int64_t t = idx / per_row;
  const int c = (int)(idx - t * per_row) * 8;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int j = 0; j < k; ++j) {
    const int64_t r = t * k + j;
    const int g = ids[r];
    if ((unsigned)g >= (unsigned)E) continue;     // not an expert id: the row adds nothing
    const int d = g / El;
    const int64_t pos = (int64_t)dst_off[g] + (inv[r] - offsets[g]);
    if (pos < 0 || pos >= cap) continue;          // a plan that does not fit: the row adds nothing
    const float wj = w[r];
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(ys.p[d]) + (size_t)pos * H + c);
    const float4 a = src[0], b = src[1];
    acc[0] = fmaf(wj, a.x, acc[0]);
    acc[1] = fmaf(wj, a.y, acc[1]);
    acc[2] = fmaf(wj, a.z, acc[2]);
    acc[3] = fmaf(wj, a.w, acc[3]);
    acc[4] = fmaf(wj, b.x, acc[4]);
    acc[5] = fmaf(wj, b.y, acc[5]);
    acc[6] = fmaf(wj, b.z, acc[6]);
    acc[7] = fmaf(wj, b.w, acc[7]);
  }
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = f32_to_bf16_bits(acc[i]);
  *reinterpret_cast<uint4*>(out + t * H + c) =
      make_uint4(o[0] | (o[1] << 16), o[2] | (o[3] << 16), o[4] | (o[5] << 16), o[6] | (o[7] << 16));
  if (x_next != nullptr) {
    const uint4 xv = *reinterpret_cast<const uint4*>(x + t * H + c);
    const uint32_t xs[8] = {xv.x & 0xFFFF, xv.x >> 16, xv.y & 0xFFFF, xv.y >> 16,
                            xv.z & 0xFFFF, xv.z >> 16, xv.w & 0xFFFF, xv.w >> 16};
    uint32_t q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = f32_to_bf16_bits(bf16_bits_to_f32(xs[i]) + bf16_bits_to_f32(o[i]));
    *reinterpret_cast<uint4*>(x_next + t * H + c) =
        make_uint4(q[0] | (q[1] << 16), q[2] | (q[3] << 16), q[4] | (q[5] << 16), q[6] | (q[7] << 16));
  }
}

}  // namespace

size_t ep_plan_smem_bytes(int E) { return (size_t)(E + E) * sizeof(int); }   // tot[E] and seg[El * G = E]

int launch_ep_plan(const int32_t* C, int G, int E, int rank, int layout, int32_t* dst_off, int32_t* recv_ids,
                   int64_t recv_rows, cudaStream_t s) {
  const size_t smem = ep_plan_smem_bytes(E);
  const int64_t ctas = recv_rows > 0 ? (recv_rows + kPlanRowsPerCta - 1) / kPlanRowsPerCta : 1;
  ep_plan_kernel<<<(unsigned)ctas, kPlanThreads, smem, s>>>(C, G, E, rank, layout, dst_off, recv_ids, recv_rows);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

bool ep_move_supported(int H) { return H % 8 == 0 && H / 8 <= kMaxVec * kMoveThreads; }

int launch_ep_dispatch(const uint16_t* x, int64_t T, int k, int H, const int32_t* ids, const int32_t* inv,
                       const int32_t* offsets, const int32_t* dst_off, int El, int64_t cap, void* const* recv, int G,
                       int num_sms, cudaStream_t s) {
  PeerPtrs pp{};
  for (int d = 0; d < G; ++d) pp.p[d] = recv[d];
  const int64_t blocks = T < (int64_t)num_sms * 16 ? T : (int64_t)num_sms * 16;
  ep_dispatch_kernel<<<(unsigned)blocks, kMoveThreads, 0, s>>>(x, T, k, H, ids, inv, offsets, dst_off, El, El * G, cap,
                                                               pp);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

int launch_ep_combine(int64_t T, int k, int H, const int32_t* ids, const float* w, const int32_t* inv,
                      const int32_t* offsets, const int32_t* dst_off, int El, int64_t cap, const float* const* ys,
                      int G, const uint16_t* x, uint16_t* out, uint16_t* x_next, cudaStream_t s) {
  PeerPtrs pp{};
  for (int d = 0; d < G; ++d) pp.p[d] = const_cast<float*>(ys[d]);
  const int64_t n = T * (H / 8);
  ep_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(T, k, H, ids, w, inv, offsets, dst_off, El, El * G,
                                                                 cap, pp, x, out, x_next);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

}  // namespace moe

// ---- C ABI --------------------------------------------------------------------------------------

#include "moe_nvfp4.h"

namespace {

bool al(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int done(int rc, const char* what) {
  if (rc < 0) return moe::api_cuda_fail(-rc, what);
  moe::api_set_launches(rc);
  return MOE_NVFP4_OK;
}

int check_ranks(int32_t G, int32_t E) {
  if (G < 1 || G > moe::kEpMaxRanks)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "ranks must be 1 .. 64");
  if (E < 1 || E > 1024 || E % G)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "num_experts must be 1 .. 1024 and a multiple of the ranks");
  return MOE_NVFP4_OK;
}

}  // namespace

extern "C" {

int moe_nvfp4_ep_plan(const int32_t* counts_all_dev, int32_t ranks, int32_t num_experts, int32_t rank,
                      int32_t layout, int32_t* dst_off_dev, int32_t* recv_ids_dev, int64_t recv_rows, void* stream) {
  moe::api_set_launches(0);
  int rc = check_ranks(ranks, num_experts);
  if (rc) return rc;
  if (rank < 0 || rank >= ranks) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "rank outside 0 .. ranks-1");
  if (layout != MOE_NVFP4_EP_EXPERT_MAJOR && layout != MOE_NVFP4_EP_SOURCE_MAJOR)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "layout is not MOE_NVFP4_EP_EXPERT_MAJOR or _SOURCE_MAJOR");
  if (recv_rows < 0 || recv_rows > ((int64_t)1 << 31) - 1)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "recv_rows outside 0 .. 2^31-1");
  if (!counts_all_dev || !dst_off_dev || (recv_rows > 0 && !recv_ids_dev))
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "counts_all, dst_off and recv_ids must not be NULL");
  int dev, sms;
  if ((rc = moe::api_device(&dev, &sms))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return done(moe::launch_ep_plan(counts_all_dev, ranks, num_experts, rank, layout, dst_off_dev, recv_ids_dev,
                                  recv_rows, s), "ep plan");
}

int moe_nvfp4_ep_dispatch(const void* x_dev, int64_t T, int32_t k, int32_t hidden, int32_t num_experts,
                          const int32_t* ids_dev, const int32_t* inv_dev, const int32_t* offsets_dev,
                          const int32_t* dst_off_dev, int32_t ranks, void* const* recv_x_ptrs_host,
                          int64_t capacity_rows, void* stream) {
  moe::api_set_launches(0);
  int rc = check_ranks(ranks, num_experts);
  if (rc) return rc;
  if (T < 0 || k < 1 || k > 32 || k > num_experts || T > ((int64_t)1 << 31) / 32)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "T or k out of range");
  if (hidden < 8 || !moe::ep_move_supported(hidden))
    return moe::api_fail(MOE_NVFP4_ERR_UNSUPPORTED, "hidden must be a multiple of 8 and at most 8192");
  int dev, sms;
  if ((rc = moe::api_device(&dev, &sms))) return rc;
  if (T == 0) return MOE_NVFP4_OK;
  if (!x_dev || !ids_dev || !inv_dev || !offsets_dev || !dst_off_dev || !recv_x_ptrs_host)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!al(x_dev, 16)) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "x must be 16-byte aligned");
  if (capacity_rows < 0) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "capacity_rows is negative");
  for (int d = 0; d < ranks; ++d)
    if (!recv_x_ptrs_host[d] || !al(recv_x_ptrs_host[d], 16))
      return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "every receive buffer must be non-NULL and 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return done(moe::launch_ep_dispatch(static_cast<const uint16_t*>(x_dev), T, k, hidden, ids_dev, inv_dev,
                                      offsets_dev, dst_off_dev, num_experts / ranks, capacity_rows, recv_x_ptrs_host,
                                      ranks, sms, s),
              "ep dispatch");
}

int moe_nvfp4_ep_combine(const void* x_dev, int64_t T, int32_t k, int32_t hidden, int32_t num_experts,
                         const int32_t* ids_dev, const float* w_dev, const int32_t* inv_dev,
                         const int32_t* offsets_dev, const int32_t* dst_off_dev, int32_t ranks,
                         const float* const* recv_y_ptrs_host, int64_t capacity_rows, void* out_dev,
                         void* x_next_dev, void* stream) {
  moe::api_set_launches(0);
  int rc = check_ranks(ranks, num_experts);
  if (rc) return rc;
  if (T < 0 || k < 1 || k > 32 || k > num_experts || T > ((int64_t)1 << 31) / 32)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "T or k out of range");
  if (hidden < 8 || hidden % 8 || hidden > 8192)
    return moe::api_fail(MOE_NVFP4_ERR_UNSUPPORTED, "hidden must be a multiple of 8 and at most 8192");
  int dev, sms;
  if ((rc = moe::api_device(&dev, &sms))) return rc;
  if (T == 0) return MOE_NVFP4_OK;
  if (!ids_dev || !w_dev || !inv_dev || !offsets_dev || !dst_off_dev || !recv_y_ptrs_host || !out_dev ||
      (x_next_dev && !x_dev))
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!al(out_dev, 16) || (x_next_dev && (!al(x_next_dev, 16) || !al(x_dev, 16))))
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "out, x and x_next must be 16-byte aligned");
  if (capacity_rows < 0) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "capacity_rows is negative");
  for (int d = 0; d < ranks; ++d)
    if (!recv_y_ptrs_host[d] || !al(recv_y_ptrs_host[d], 16))
      return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "every output buffer must be non-NULL and 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return done(moe::launch_ep_combine(T, k, hidden, ids_dev, w_dev, inv_dev, offsets_dev, dst_off_dev,
                                     num_experts / ranks, capacity_rows, recv_y_ptrs_host, ranks,
                                     static_cast<const uint16_t*>(x_dev),
                                     static_cast<uint16_t*>(out_dev), static_cast<uint16_t*>(x_next_dev), s),
              "ep combine");
}

int moe_nvfp4_gather_rows(const void* x_dev, const int32_t* perm_dev, int64_t T, int32_t k, int32_t hidden,
                          void* rows_dev, void* stream) {
  moe::api_set_launches(0);
  if (T < 0 || k < 1 || k > 32 || T > ((int64_t)1 << 31) / 32)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "T or k out of range");
  if (hidden < 8 || hidden % 8 || hidden > 8192)
    return moe::api_fail(MOE_NVFP4_ERR_UNSUPPORTED, "hidden must be a multiple of 8 and at most 8192");
  int dev, sms;
  int rc = moe::api_device(&dev, &sms);
  if (rc) return rc;
  if (T == 0) return MOE_NVFP4_OK;
  if (!x_dev || !perm_dev || !rows_dev) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!al(x_dev, 16) || !al(rows_dev, 16))
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "x and rows must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return done(moe::launch_gather(static_cast<const uint16_t*>(x_dev), perm_dev, k, T * k, hidden, rows_dev, s),
              "gather rows");
}

int moe_nvfp4_combine(const float* y_dev, const float* w_dev, const int32_t* inv_dev, int64_t T, int32_t k,
                      int32_t hidden, const void* x_dev, void* out_dev, void* x_next_dev, void* stream) {
  moe::api_set_launches(0);
  if (T < 0 || k < 1 || k > 32 || T > ((int64_t)1 << 31) / 32)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "T or k out of range");
  if (hidden < 8 || hidden % 8 || hidden > 8192)
    return moe::api_fail(MOE_NVFP4_ERR_UNSUPPORTED, "hidden must be a multiple of 8 and at most 8192");
  int dev, sms;
  int rc = moe::api_device(&dev, &sms);
  if (rc) return rc;
  if (T == 0) return MOE_NVFP4_OK;
  if (!y_dev || !w_dev || !inv_dev || !out_dev || (x_next_dev && !x_dev))
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "a pointer argument is NULL");
  if (!al(y_dev, 16) || !al(out_dev, 16) || (x_next_dev && (!al(x_next_dev, 16) || !al(x_dev, 16))))
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "y, out, x and x_next must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return done(moe::launch_combine(y_dev, w_dev, inv_dev, T, k, hidden, static_cast<const uint16_t*>(x_dev),
                                  static_cast<uint16_t*>(out_dev), static_cast<uint16_t*>(x_next_dev), s),
              "combine");
}

int moe_nvfp4_ep_buffer_create(uint64_t bytes, void** dev_ptr, uint8_t* handle_host) {
  if (!dev_ptr || !handle_host || bytes == 0)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "dev_ptr and handle must not be NULL, bytes > 0");
  *dev_ptr = nullptr;
  int dev, sms;
  int rc = moe::api_device(&dev, &sms);
  if (rc) return rc;
  void* p = nullptr;
  cudaError_t e = cudaMalloc(&p, bytes);
  if (e != cudaSuccess) return moe::api_cuda_fail(e, "ep buffer allocation");
  cudaIpcMemHandle_t h;
  e = cudaIpcGetMemHandle(&h, p);
  if (e != cudaSuccess) {
    cudaFree(p);
    return moe::api_cuda_fail(e, "ep buffer handle");
  }
  memcpy(handle_host, &h, sizeof(h));
  *dev_ptr = p;
  return MOE_NVFP4_OK;
}

int moe_nvfp4_ep_buffer_open(const uint8_t* handle_host, void** peer_ptr) {
  if (!handle_host || !peer_ptr)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "handle and peer_ptr must not be NULL");
  *peer_ptr = nullptr;
  int dev, sms;
  int rc = moe::api_device(&dev, &sms);
  if (rc) return rc;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle_host, sizeof(h));
  const cudaError_t e = cudaIpcOpenMemHandle(peer_ptr, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return moe::api_cuda_fail(e, "open a peer's ep buffer");
  return MOE_NVFP4_OK;
}

int moe_nvfp4_ep_buffer_close(void* peer_ptr) {
  if (!peer_ptr) return MOE_NVFP4_OK;
  const cudaError_t e = cudaIpcCloseMemHandle(peer_ptr);
  if (e != cudaSuccess) return moe::api_cuda_fail(e, "close a peer's ep buffer");
  return MOE_NVFP4_OK;
}

int moe_nvfp4_ep_buffer_destroy(void* dev_ptr) {
  if (!dev_ptr) return MOE_NVFP4_OK;
  const cudaError_t e = cudaFree(dev_ptr);
  if (e != cudaSuccess) return moe::api_cuda_fail(e, "free an ep buffer");
  return MOE_NVFP4_OK;
}

}  // extern "C"
