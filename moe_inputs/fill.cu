// Device writer of synthetic expert banks: the same counter-based SplitMix64 streams as
// moe_inputs/gen.py (Steele, Lea & Flood, OOPSLA 2014), so a record written here is
// byte-identical to gen.record_bytes() for the same (seed, layer, expert).  Input
// generation only: nothing here belongs to the MoE layer's arithmetic.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, uint64_t layer, uint64_t expert,
                                               uint64_t stream) {
  uint64_t k = mix64(seed + kGolden);
  k = mix64(k ^ (layer + kGolden));
  k = mix64(k ^ (expert + kGolden));
  k = mix64(k ^ (stream + kGolden));
  return k;
}

struct FillArgs {
  uint8_t* base;
  uint64_t stride;
  uint64_t code_words;   // u64 words of codes per record (3*I*H/16)
  uint64_t scale_bytes;  // scale bytes per record (3*I*H/16), a multiple of 8
  uint64_t global_off;   // byte offset of the 3 f32 globals
  uint64_t seed;
  uint32_t layer;
  int expert0, experts;
  float gval;
};

__global__ void fill_codes(FillArgs a) {
  const uint64_t per = a.code_words;
  const uint64_t total = per * (uint64_t)a.experts;
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < total;
       i += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t e = i / per, w = i - e * per;
    const uint64_t key = stream_key(a.seed, a.layer, a.expert0 + e, 0);
    const uint64_t v = mix64(key + (w + 1) * kGolden);
    reinterpret_cast<uint64_t*>(a.base + (a.expert0 + e) * a.stride)[w] = v;
  }
}

__global__ void fill_scales(FillArgs a) {
  const uint64_t per = a.scale_bytes / 8;
  const uint64_t total = per * (uint64_t)a.experts;
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < total;
       i += (uint64_t)gridDim.x * blockDim.x) {
    const uint64_t e = i / per, q = i - e * per;
    const uint64_t key = stream_key(a.seed, a.layer, a.expert0 + e, 1);
    uint64_t packed = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint64_t h = mix64(key + (q * 8 + j + 1) * kGolden) & 0xFFFFFFFFull;
      const uint64_t b = 0x18 + ((h * 49ull) >> 32);
      packed |= b << (8 * j);
    }
    uint8_t* rec = a.base + (a.expert0 + e) * a.stride;
    reinterpret_cast<uint64_t*>(rec + a.code_words * 8)[q] = packed;
  }
}

__global__ void fill_globals(FillArgs a) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= a.experts) return;
  float* g = reinterpret_cast<float*>(a.base + (a.expert0 + e) * a.stride + a.global_off);
  g[0] = a.gval;
  g[1] = a.gval;
  g[2] = a.gval;
}

}  // namespace

extern "C" {

// Writes records expert0 .. expert0+experts-1 of the bank at `base` (device memory,
// records `stride` bytes apart) for shapes H, I: codes, then scales, then 3 f32 globals
// equal to `gval`.  Returns 0 or the CUDA error code.
int moe_inputs_fill_bank(void* base, uint64_t stride, int H, int I, uint64_t seed,
                         uint32_t layer, int expert0, int experts, float gval,
                         void* stream) {
  FillArgs a;
  a.base = static_cast<uint8_t*>(base);
  a.stride = stride;
  a.code_words = 3ull * (uint64_t)I * (uint64_t)H / 16;
  a.scale_bytes = 3ull * (uint64_t)I * (uint64_t)H / 16;
  a.global_off = a.code_words * 8 + a.scale_bytes;
  a.seed = seed;
  a.layer = layer;
  a.expert0 = expert0;
  a.experts = experts;
  a.gval = gval;
  if (a.scale_bytes % 8 != 0 || (reinterpret_cast<uintptr_t>(base) & 7) || (stride & 7))
    return (int)cudaErrorInvalidValue;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  fill_codes<<<148 * 8, 256, 0, s>>>(a);
  fill_scales<<<148 * 8, 256, 0, s>>>(a);
  fill_globals<<<(experts + 255) / 256, 256, 0, s>>>(a);
  return (int)cudaGetLastError();
}

// Host copy of the stream key (for tests that compare the two implementations).
uint64_t moe_inputs_stream_key(uint64_t seed, uint32_t layer, uint32_t expert, uint32_t stream) {
  return stream_key(seed, layer, expert, stream);
}

}  // extern "C"
