// Device helpers of the fused decode kernels (single token and few tokens): packed f16 math,
// shared loads, the 32-input NVFP4 unit dot product, bounded counter waits, work shares.
#pragma once

#include "common.cuh"

namespace moe {
namespace fused {

__device__ __forceinline__ uint32_t hfma2_(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
__device__ __forceinline__ uint32_t hadd2_(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// acc += the dot product of one 32-input unit: codes (4 words) and its two E4M3 block scales
// against 16 f16x2 of x.  Each 16-input block is summed with packed f16 FMAs (two chains per
// half), its two halves are added in f16, and each half times the block's f16 scale is added
// to acc by an f32 FMA on f16 operands (fma.rn.f32.f16: the product is exact in f32, one
// rounding per addition), so no f16 -> f32 conversions are issued.
__device__ __forceinline__ void unit_dot_acc(const uint4 c, uint32_t sc2, const uint32_t (&x)[16], float& acc) {
  const uint32_t s = e4m3x2_to_f16x2((uint16_t)sc2);     // block 0 scale low, block 1 high
  uint32_t e0[4], e1[4], e2[4], e3[4];
  e2m1x8_to_f16x8(c.x, e0);
  e2m1x8_to_f16x8(c.y, e1);
  e2m1x8_to_f16x8(c.z, e2);
  e2m1x8_to_f16x8(c.w, e3);
  uint32_t p0 = hfma2_(e0[0], x[0], 0u), p0b = hfma2_(e0[1], x[1], 0u);
  uint32_t p1 = hfma2_(e2[0], x[8], 0u), p1b = hfma2_(e2[1], x[9], 0u);
  p0 = hfma2_(e0[2], x[2], p0), p0b = hfma2_(e0[3], x[3], p0b);
  p1 = hfma2_(e2[2], x[10], p1), p1b = hfma2_(e2[3], x[11], p1b);
  p0 = hfma2_(e1[0], x[4], p0), p0b = hfma2_(e1[1], x[5], p0b);
  p1 = hfma2_(e3[0], x[12], p1), p1b = hfma2_(e3[1], x[13], p1b);
  p0 = hfma2_(e1[2], x[6], p0), p0b = hfma2_(e1[3], x[7], p0b);
  p1 = hfma2_(e3[2], x[14], p1), p1b = hfma2_(e3[3], x[15], p1b);
  const uint32_t a = hadd2_(p0, p0b), b = hadd2_(p1, p1b);
  asm("{\n\t.reg .f16 al, ah, bl, bh, s0, s1;\n\t"
      "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\tmov.b32 {s0, s1}, %3;\n\t"
      "fma.rn.f32.f16 %0, al, s0, %0;\n\tfma.rn.f32.f16 %0, ah, s0, %0;\n\t"
      "fma.rn.f32.f16 %0, bl, s1, %0;\n\tfma.rn.f32.f16 %0, bh, s1, %0;\n\t}"
      : "+f"(acc)
      : "r"(a), "r"(b), "r"(s));
}

// The same unit's dot product on its own.
__device__ __forceinline__ float unit_dot(const uint4 c, uint32_t sc2, const uint32_t (&x)[16]) {
  float acc = 0.0f;
  unit_dot_acc(c, sc2, x, acc);
  return acc;
}

// Waits until *counter reaches target (other CTAs of the persistent grid add to it; all are
// resident: cooperative launch).  Bounded: gives up after kWaitCycles, records a timeout and
// returns false.
__device__ __forceinline__ bool wait_count(const unsigned* counter, unsigned target) {
  const long long t0 = clock64();
  while (ld_acquire(counter) < target) {
    if (clock64() - t0 > kWaitCycles) {
      atomicExch(&g_status, kStatusTimeout);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// Contiguous share [lo, hi) of n work units for CTA c of G.
__device__ __forceinline__ void share(int n, int c, int G, int& lo, int& hi) {
  lo = (int)(((long long)n * c) / G);
  hi = (int)(((long long)n * (c + 1)) / G);
}

}  // namespace fused
}  // namespace moe
