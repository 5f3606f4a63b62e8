// Weighted combine of the k expert outputs of each token, and the residual add of stacked
// layers: out[t] = bf16(sum_j w[t, j] * y[inv[t*k + j]]) with f32 accumulation in rank
// order j = 0 .. k-1; if requested, x_next[t] = bf16(x[t] + out[t]) (the sum of two BF16
// values rounded once).  The combine is part of the method statement of the routed-expert
// layer; the residual add between stacked layers is the verify-across-depth workload's.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ inv, int64_t T,
                                                      int k, int H, const uint16_t* __restrict__ x,
                                                      uint16_t* __restrict__ out,
                                                      uint16_t* __restrict__ x_next) {
  const int per_row = H / 8;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * per_row) return;
  const int64_t t = idx / per_row;
  const int c = (int)(idx - t * per_row) * 8;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int j = 0; j < k; ++j) {
    const float wj = w[t * k + j];
    const float4* src = reinterpret_cast<const float4*>(y + (size_t)inv[t * k + j] * H + c);
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
  uint4 ov = make_uint4(o[0] | (o[1] << 16), o[2] | (o[3] << 16), o[4] | (o[5] << 16),
                        o[6] | (o[7] << 16));
  *reinterpret_cast<uint4*>(out + t * H + c) = ov;
  if (x_next != nullptr) {
    const uint4 xv = *reinterpret_cast<const uint4*>(x + t * H + c);
    const uint32_t xs[8] = {xv.x & 0xFFFF, xv.x >> 16, xv.y & 0xFFFF, xv.y >> 16,
                            xv.z & 0xFFFF, xv.z >> 16, xv.w & 0xFFFF, xv.w >> 16};
    uint32_t r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      r[i] = f32_to_bf16_bits(bf16_bits_to_f32(xs[i]) + bf16_bits_to_f32(o[i]));
    *reinterpret_cast<uint4*>(x_next + t * H + c) =
        make_uint4(r[0] | (r[1] << 16), r[2] | (r[3] << 16), r[4] | (r[5] << 16),
                   r[6] | (r[7] << 16));
  }
}

// Experts-only calls: y_rows[r] = y[inv[r]] (the expert output of row r, which the expert
// kernels wrote at its place in expert order), zero for padding rows (id < 0).
__global__ void __launch_bounds__(256) unpermute_kernel(const float* __restrict__ y, const int32_t* __restrict__ inv,
                                                        const int32_t* __restrict__ ids, int64_t R, int H,
                                                        float* __restrict__ y_rows) {
  const int per_row = H / 4;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= R * per_row) return;
  const int64_t r = idx / per_row;
  const int c = (int)(idx - r * per_row) * 4;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (ids[r] >= 0) v = *reinterpret_cast<const float4*>(y + (size_t)inv[r] * H + c);
  *reinterpret_cast<float4*>(y_rows + (size_t)r * H + c) = v;
}

}  // namespace

int launch_combine(const float* y, const float* w, const int32_t* inv, int64_t T, int k, int H,
                   const uint16_t* x, uint16_t* out, uint16_t* x_next, cudaStream_t s) {
  const int64_t n = T * (H / 8);
  const int blocks = (int)((n + 255) / 256);
  combine_kernel<<<blocks, 256, 0, s>>>(y, w, inv, T, k, H, x, out, x_next);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

int launch_unpermute(const float* y, const int32_t* inv, const int32_t* ids, int64_t R, int H, float* y_rows,
                     cudaStream_t s) {
  const int64_t n = R * (H / 4);
  unpermute_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(y, inv, ids, R, H, y_rows);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

}  // namespace moe
