// NVFP4 encoder: BF16 weights [n, out, in] -> E2M1 codes, E4M3 block scales and one f32 global per
// projection, written straight into expert records (any record stride and part offsets).
//
// The rule (page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents",
// section "What this pack holds": a block's scale is e4m3(block scale) x (g / 2688), 2688 being
// 6 x 448; page "Running Beam-1.0 (501B) on workstation GPUs": data-free NVFP4A16 quantization
// of the experts): the per-tensor multiplier s2 = f32(amax / 2688) maps the tensor's largest
// magnitude onto the largest product 6 x 448; each block of 16 inputs takes the E4M3 value
// nearest to f32(amax_b / f32(6 s2)) (ties to even, saturating at 448); each weight takes the E2M1
// value nearest to f32(w / f32(e4m3 x s2)) (ties to even, saturating at 6) with the weight's sign
// bit.  Every quotient and product is one f32 operation rounded to nearest even, because each one
// decides a stored integer.
//
// Four launches, no scratch memory: (1) clear each projection's global slot, (2) collect each
// projection's max |w| there (atomicMax on the f32 bit pattern: non-negative f32 values order like
// their patterns), (3) encode the blocks, one thread per block of 16 inputs, reading amax from the
// slot, (4) replace amax by the stored global (s2, or g = amax itself in global mode 1, since
// f32(amax / 2688) is s2 by construction).  Streams: input read twice (the amax pass and the
// encode pass), 0.5625 B written per weight.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kEncThreads = 256;
constexpr int kAmaxPerThread = 8;      // 16-byte loads (8 weights) per thread of the amax pass

__device__ __forceinline__ float* slot_of(uint8_t* dst, uint64_t stride, uint64_t global_off, int64_t p) {
  return reinterpret_cast<float*>(dst + (uint64_t)p * stride + global_off);
}

__global__ void enc_clear_kernel(uint8_t* dst, uint64_t stride, uint64_t global_off, int64_t n) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p < n) *slot_of(dst, stride, global_off, p) = 0.0f;
}

// Chunk c of projection p (flattened over blockIdx.x): kEncThreads x kAmaxPerThread 16-byte loads.
__global__ void __launch_bounds__(kEncThreads) enc_amax_kernel(const uint16_t* w, int64_t per, int64_t chunks,
                                                               uint8_t* dst, uint64_t stride, uint64_t global_off) {
  const int64_t p = blockIdx.x / chunks, c = blockIdx.x - p * chunks;
  const uint4* src = reinterpret_cast<const uint4*>(w + p * per);
  const int64_t n8 = per / 8;
  const int64_t base = c * (int64_t)(kEncThreads * kAmaxPerThread);
  uint32_t m = 0;
#pragma unroll
  for (int t = 0; t < kAmaxPerThread; ++t) {
    const int64_t i = base + t * kEncThreads + threadIdx.x;
    if (i < n8) m = max(m, bf16x8_abs_max_bits(__ldg(src + i)));
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t s_m[kEncThreads / 32];
  if ((threadIdx.x & 31) == 0) s_m[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t v = 0;
#pragma unroll
    for (int i = 0; i < kEncThreads / 32; ++i) v = max(v, s_m[i]);
    // the BF16 magnitude pattern widened to f32 (exact); f32 patterns of non-negative values
    // order like the values
    if (v) atomicMax(reinterpret_cast<unsigned*>(slot_of(dst, stride, global_off, p)), v << 16);
  }
}

// Sign bits of eight BF16 values (four packed pairs) at the code positions 4i + 3.
__device__ __forceinline__ uint32_t e2m1x8_signs(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t p3) {
  const uint32_t p[4] = {p0, p1, p2, p3};
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) s |= ((p[i] >> 15) & 1u) << (8 * i + 3) | (p[i] >> 31) << (8 * i + 7);
  return s;
}

struct EncParams {
  const uint16_t* w;       // [n, out, in] bf16
  int64_t n;
  int out_f, in_f;
  uint8_t* dst;
  uint64_t stride, codes_off, scales_off, global_off;
};

__global__ void __launch_bounds__(kEncThreads) enc_blocks_kernel(const EncParams p) {
  const int nb = p.in_f / 16;                                   // blocks per row
  const int64_t per_proj = (int64_t)p.out_f * nb;
  const int64_t total = p.n * per_proj;
  for (int64_t g = (int64_t)blockIdx.x * kEncThreads + threadIdx.x; g < total; g += (int64_t)gridDim.x * kEncThreads) {
    const int64_t pj = g / per_proj, rb = g - pj * per_proj;
    const int row = (int)(rb / nb), b = (int)(rb - (int64_t)row * nb);
    const uint4* src = reinterpret_cast<const uint4*>(p.w + pj * (int64_t)p.out_f * p.in_f + (int64_t)row * p.in_f + 16 * b);
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    uint8_t* rec = p.dst + (uint64_t)pj * p.stride;
    const float amax = __ldcg(reinterpret_cast<const float*>(rec + p.global_off));
    const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t scale = 0;
    float eff = 0.0f;
    if (amax > 0.0f) {
      const float s2 = __fdiv_rn(amax, 2688.0f);
      const float amax_b = __uint_as_float(max(bf16x8_abs_max_bits(v0), bf16x8_abs_max_bits(v1)) << 16);
      scale = f32_to_e4m3_byte(__fdiv_rn(amax_b, __fmul_rn(6.0f, s2)));
      eff = __fmul_rn(e4m3_byte_to_f32(scale), s2);
    }
    // the weights' sign bits in every case; magnitudes only where the block scale is not zero
    uint32_t lo = e2m1x8_signs(wv[0], wv[1], wv[2], wv[3]), hi = e2m1x8_signs(wv[4], wv[5], wv[6], wv[7]);
    if (eff > 0.0f) {
      float r[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        r[2 * i] = fabsf(__fdiv_rn(bf16_bits_to_f32(wv[i] & 0xFFFFu), eff));
        r[2 * i + 1] = fabsf(__fdiv_rn(bf16_bits_to_f32(wv[i] >> 16), eff));
      }
      lo |= e2m1x8_mag(r);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        r[2 * i] = fabsf(__fdiv_rn(bf16_bits_to_f32(wv[4 + i] & 0xFFFFu), eff));
        r[2 * i + 1] = fabsf(__fdiv_rn(bf16_bits_to_f32(wv[4 + i] >> 16), eff));
      }
      hi |= e2m1x8_mag(r);
    }
    *reinterpret_cast<uint2*>(rec + p.codes_off + (uint64_t)row * (p.in_f / 2) + 8 * b) = make_uint2(lo, hi);
    rec[p.scales_off + (uint64_t)row * nb + b] = (uint8_t)scale;
  }
}

__global__ void enc_finalize_kernel(uint8_t* dst, uint64_t stride, uint64_t global_off, int64_t n, int mode) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n) return;
  float* slot = slot_of(dst, stride, global_off, p);
  const float amax = *slot;
  if (mode == 0) *slot = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 0.0f;
}

}  // namespace

int launch_encode(const uint16_t* w, int64_t n, int out_f, int in_f, int global_mode, uint8_t* dst, uint64_t stride,
                  uint64_t codes_off, uint64_t scales_off, uint64_t global_off, int num_sms, cudaStream_t s) {
  const int64_t per = (int64_t)out_f * in_f;
  const unsigned nblk = (unsigned)((n + 255) / 256);
  enc_clear_kernel<<<nblk, 256, 0, s>>>(dst, stride, global_off, n);
  const int64_t chunks = (per / 8 + kEncThreads * kAmaxPerThread - 1) / (kEncThreads * kAmaxPerThread);
  enc_amax_kernel<<<(unsigned)(n * chunks), kEncThreads, 0, s>>>(w, per, chunks, dst, stride, global_off);
  EncParams p{w, n, out_f, in_f, dst, stride, codes_off, scales_off, global_off};
  const int64_t blocks = n * per / 16;
  const int64_t want = (blocks + kEncThreads - 1) / kEncThreads;
  const int64_t cap = (int64_t)num_sms * 16;                   // grid-stride beyond 16 CTAs per SM
  enc_blocks_kernel<<<(unsigned)(want < cap ? want : cap), kEncThreads, 0, s>>>(p);
  enc_finalize_kernel<<<nblk, 256, 0, s>>>(dst, stride, global_off, n, global_mode);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 4 : -(int)err;
}

}  // namespace moe
