// Device helpers shared by the kernels of the NVFP4 MoE library (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace moe {

// Sticky device status: set by a kernel whose bounded wait gave up.
extern __device__ int g_status;

constexpr int kStatusTimeout = -5;

// Bounded waits give up after this many clock cycles (~1 s at B200 clocks).
constexpr long long kWaitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the async proxy (TMA) before first use.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with this parity to complete.  Gives up after kWaitCycles, records
// a timeout in g_status and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) {
      atomicExch(&g_status, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------- bulk copies (TMA, 1-D)

// L2 policy for data read once per call (expert weights): evict first.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// L2 policy for data fetched early and read once later: evict last.
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Bulk prefetch of [src, src + bytes) into L2 (TMA; no completion to wait for).  src 16-byte
// aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes, uint64_t policy) {
  asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;" ::"l"(src), "r"(bytes), "l"(policy)
               : "memory");
}

// Global -> shared bulk copy completing on `bar`; dst, src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// ---------------------------------------------------------------- named barriers

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---------------------------------------------------------------- conversions

// Eight E2M1 codes (one little-endian u32, code i in bits 4i..4i+3) -> four f16x2; out[j]
// holds codes 2j (low half) and 2j+1 (high half).  Exact.
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t out[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w));
}

// Eight E2M1 codes (one u32, code i in bits 4i..4i+3) times an f16x2 block scale (both halves
// equal) -> four bf16x2; out[j] holds codes 2j (low half) and 2j+1 (high half).  Exact: each
// product has at most 5 significant bits and lies in [2^-10, 2688], so it is exact in f16, in
// f32 and in bf16.
__device__ __forceinline__ void e2m1x8_scaled_to_bf16x8(uint32_t w, uint32_t scale2, uint32_t out[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      ".reg .b32 h0, h1, h2, h3;\n\t"
      ".reg .b16 l0, u0, l1, u1, l2, u2, l3, u3;\n\t"
      ".reg .f32 a0, c0, a1, c1, a2, c2, a3, c3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 h0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 h1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 h2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 h3, b3;\n\t"
      "mul.rn.f16x2 h0, h0, %5;\n\t"
      "mul.rn.f16x2 h1, h1, %5;\n\t"
      "mul.rn.f16x2 h2, h2, %5;\n\t"
      "mul.rn.f16x2 h3, h3, %5;\n\t"
      "mov.b32 {l0, u0}, h0;\n\t"
      "mov.b32 {l1, u1}, h1;\n\t"
      "mov.b32 {l2, u2}, h2;\n\t"
      "mov.b32 {l3, u3}, h3;\n\t"
      "cvt.f32.f16 a0, l0;\n\t cvt.f32.f16 c0, u0;\n\t"
      "cvt.f32.f16 a1, l1;\n\t cvt.f32.f16 c1, u1;\n\t"
      "cvt.f32.f16 a2, l2;\n\t cvt.f32.f16 c2, u2;\n\t"
      "cvt.f32.f16 a3, l3;\n\t cvt.f32.f16 c3, u3;\n\t"
      "cvt.rn.bf16x2.f32 %0, c0, a0;\n\t"
      "cvt.rn.bf16x2.f32 %1, c1, a1;\n\t"
      "cvt.rn.bf16x2.f32 %2, c2, a2;\n\t"
      "cvt.rn.bf16x2.f32 %3, c3, a3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w), "r"(scale2));
}

// Two E4M3 bytes (low byte first) -> f16x2.  Exact (every E4M3 value is an f16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// f16x2 with both halves equal to the low (hi = false) or high half of v.
__device__ __forceinline__ uint32_t bcast_half(uint32_t v, bool hi) {
  return hi ? __byte_perm(v, 0, 0x3232) : __byte_perm(v, 0, 0x1010);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

__device__ __forceinline__ uint32_t f32_to_bf16_bits(float v) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(v));
  return r;
}

// ---------------------------------------------------------------- warp MMA

// D += A * B with A 16x16 f16 (row), B 16x8 f16 (col), D 16x8 f32.
__device__ __forceinline__ void mma_16816(float c[4], const uint32_t a[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- power-of-two prescale
//
// The decode kernels multiply NVFP4 weights with the activations in f16 (packed f16 FMAs, or
// mma.sync with f16 operands).  BF16 activations and f32 mid values span far more than f16, so
// every activation vector (one token's x, one routed row's h) is first multiplied by an exact
// power of two 2^s taken from its largest magnitude: s = min(136 - emax, 126), with emax the
// largest biased exponent (the 8-bit field that f32 and BF16 share), puts max |v| 2^s in
// [2^9, 2^10) (below 1 for vectors whose maximum is under 2^-126).
//  * A sum of 8 products e2m1 x v (|e2m1| <= 6) then stays below 48 x 2^10 = 49152 < 65504.
//  * Values down to 2^-23 of the vector's maximum stay normal f16 (11 significant bits); below
//    that they lose bits as f16 subnormals, and below 2^-34 of the maximum they become zero.
//    Every BF16 value times 2^126 is at least 2^-7, so x never underflows for that reason.
//  * Results are multiplied by 2^-s in f32, which is exact unless the result itself leaves
//    the normal f32 range, so the outcome is that of the unscaled arithmetic wherever f16 would
//    have held the unscaled values.
// s lies in [-119, 126], so 2^s and 2^-s are both normal f32 values.

// Largest |bf16| bit pattern (sign cleared) of the two halves of a packed pair: magnitudes of
// finite values order like their patterns, and inf / NaN compare above every finite value.
__device__ __forceinline__ uint32_t bf16x2_abs_max_bits(uint32_t v) {
  const uint32_t a = v & 0x7FFF7FFFu;
  return max(a & 0xFFFFu, a >> 16);
}
__device__ __forceinline__ uint32_t f32_abs_bits(float v) { return __float_as_uint(v) & 0x7FFFFFFFu; }

// s from the largest |bf16| pattern / the largest |f32| pattern.
__device__ __forceinline__ int prescale_shift_bf16(uint32_t max_abs_bits) {
  return min(136 - (int)(max_abs_bits >> 7), 126);
}
__device__ __forceinline__ int prescale_shift_f32(uint32_t max_abs_bits) {
  return min(136 - (int)(max_abs_bits >> 23), 126);
}

// 2^s for s in [-126, 127].
__device__ __forceinline__ float exp2_int(int s) { return __int_as_float((s + 127) << 23); }

// Two BF16 values (a packed pair) times the power of two f, as a BF16 pair.  Exact unless a
// scaled value falls below the normal BF16 range, which only happens to values that lie more
// than 2^-126 below the largest of their vector (f16 flushes those to zero anyway).
__device__ __forceinline__ uint32_t bf16x2_scaled(uint32_t v, float f) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
      : "=r"(r)
      : "f"(bf16_bits_to_f32(v >> 16) * f), "f"(bf16_bits_to_f32(v & 0xFFFFu) * f));
  return r;
}
__device__ __forceinline__ uint4 bf16x8_scaled(uint4 v, float f) {
  return make_uint4(bf16x2_scaled(v.x, f), bf16x2_scaled(v.y, f), bf16x2_scaled(v.z, f), bf16x2_scaled(v.w, f));
}
__device__ __forceinline__ uint32_t bf16x8_abs_max_bits(uint4 v) {
  return max(max(bf16x2_abs_max_bits(v.x), bf16x2_abs_max_bits(v.y)),
             max(bf16x2_abs_max_bits(v.z), bf16x2_abs_max_bits(v.w)));
}

// SwiGLU of one pair: silu(g) * u = g / (1 + e^-g) * u, in f32.
// ---------------------------------------------------------------- NVFP4 encoding
// Every decision (a scale byte, a code) is taken on an f32 quotient rounded to nearest even.

// E4M3 byte of a non-negative f32, nearest even, saturating at 448.
__device__ __forceinline__ uint32_t f32_to_e4m3_byte(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// Value of an E4M3 byte (exact: every E4M3 value is an f16 value).
__device__ __forceinline__ float e4m3_byte_to_f32(uint32_t b) {
  const uint32_t h2 = e4m3x2_to_f16x2((uint16_t)b);
  float f;
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, lo;\n\t}" : "=f"(f) : "r"(h2));
  return f;
}

// Eight E2M1 magnitude codes (element i in bits 4i .. 4i+3, bit 4i+3 clear) of non-negative f32
// values, nearest magnitude, ties to even, saturating at 6.
__device__ __forceinline__ uint32_t e2m1x8_mag(const float (&a)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]), "f"(a[7]));
  return r & 0x77777777u;
}

// Encodes one block of 16 f32 values with the positive multiplier s2: the block scale is the E4M3
// value nearest to f32(amax / f32(6 s2)) (ties to even, saturating at 448), each code the E2M1
// value nearest to f32(v / f32(e4m3 x s2)) (ties to even, saturating at 6) with the sign bit of
// v; a block whose f32(e4m3 x s2) is 0 keeps only the signs.  Codes of elements 0..7 go to lo,
// 8..15 to hi (element i at bits 4(i % 8)); returns the scale byte.
__device__ __forceinline__ uint32_t nvfp4_encode16(const float (&v)[16], float s2, uint32_t& lo, uint32_t& hi) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t scale = f32_to_e4m3_byte(__fdiv_rn(amax, __fmul_rn(6.0f, s2)));
  const float eff = __fmul_rn(e4m3_byte_to_f32(scale), s2);
  lo = 0;
  hi = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo |= (__float_as_uint(v[i]) >> 31) << (4 * i + 3);
    hi |= (__float_as_uint(v[8 + i]) >> 31) << (4 * i + 3);
  }
  if (eff > 0.0f) {
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = fabsf(__fdiv_rn(v[i], eff));
    lo |= e2m1x8_mag(r);
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = fabsf(__fdiv_rn(v[8 + i], eff));
    hi |= e2m1x8_mag(r);
  }
  return scale;
}

// The same encoding with the 16 code decisions taken from q = f32(|v| x f32(1 / eff)) instead of
// a division per value, where that gives the same code: q is within about 3 x 2^-24 (relative) of
// f32(v / eff), so when q (1 - 2^-20) and q (1 + 2^-20) round to the same E2M1 code, no code
// boundary (nor a tie on one) lies between q and f32(v / eff), and that code is the one the
// division would give.  Otherwise (rarely) the 8 values of that half are decided by division.
__device__ __forceinline__ uint32_t nvfp4_encode16_fast(const float (&v)[16], float s2, uint32_t& lo, uint32_t& hi) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t scale = f32_to_e4m3_byte(__fdiv_rn(amax, __fmul_rn(6.0f, s2)));
  const float eff = __fmul_rn(e4m3_byte_to_f32(scale), s2);
  lo = 0;
  hi = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo |= (__float_as_uint(v[i]) >> 31) << (4 * i + 3);
    hi |= (__float_as_uint(v[8 + i]) >> 31) << (4 * i + 3);
  }
  if (eff > 0.0f) {
    const float r = __frcp_rn(eff);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float q = __fmul_rn(fabsf(v[8 * h + i]), r);
        a[i] = __fmul_rn(q, 1.0f - 0x1p-20f);
        b[i] = __fmul_rn(q, 1.0f + 0x1p-20f);
      }
      uint32_t c = e2m1x8_mag(a);
      if (c != e2m1x8_mag(b)) {
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = fabsf(__fdiv_rn(v[8 * h + i], eff));
        c = e2m1x8_mag(a);
      }
      if (h)
        hi |= c;
      else
        lo |= c;
    }
  }
  return scale;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

// SwiGLU with the hardware exponential and fast division (a few ulp; used where the result is
// rounded to f16 right after).
__device__ __forceinline__ float silu_mul_fast(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Multiplier of a projection's stored global: mode 0 the value itself, mode 1 f32(g / 2688).
__device__ __forceinline__ float global_mult(float g, int mode) {
  return mode == 1 ? __fdiv_rn(g, 2688.0f) : g;
}

}  // namespace moe

// ---------------------------------------------------------------- tcgen05 / TMEM (sm_100a)

namespace moe {

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrives once on `bar` when all tcgen05 operations issued so far by this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// D (TMEM, f32) (+)= A (smem descriptor) * B (smem descriptor)^T, kind::f16.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Makes this thread's generic-proxy shared-memory writes visible to the async proxy
// (tensor core, TMA) before it signals a barrier.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled TMA load of box (x, y) of `map` into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// 3-D tiled TMA load of box (x, y, z) of `map` into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// Prefetch of box (x, y, z) of a 3-D tensor map into L2 (no shared memory, no completion): issued
// a few stages ahead of the load of the same box, so that the load finds its bytes in L2.
__device__ __forceinline__ void tma_prefetch_3d(const void* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(map), "r"(x), "r"(y),
               "r"(z)
               : "memory");
}

// Shared-memory matrix descriptor (sm_100) for a K-major operand stored in 128-byte swizzle
// atoms (8 rows x 128 B, 1024 B apart): start address, leading offset 1 (unused when
// swizzled), stride offset 1024 B, descriptor version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: f16 A and B, f32 accumulator, both K-major, M x N.
__host__ __device__ __forceinline__ uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// The same with bf16 A and B (a_format = b_format = 1).
__host__ __device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace moe
