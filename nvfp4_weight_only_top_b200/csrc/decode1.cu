// Decode of a single token (T = 1) as ONE persistent kernel: route -> gate/up + SwiGLU ->
// down -> combine, with two grid-wide barriers and no other launch.
//
// With one token every routed row is its own expert, the work is 2 FLOP per weight byte, and
// the layer is a pure stream of k expert records (177 MB at E=256, k=8, H=5120, I=2560) from
// HBM.  What costs time besides the bytes is the number of dependent steps, so:
//   * every CTA routes the token itself (top-k of E logits, the router of route_warp.cuh):
//     no router kernel, no hand-off;
//   * one producer warp per CTA streams the CTA's weight rows with large 1-D bulk copies
//     (TMA) into a 4-stage shared-memory ring -- first its share of the gate/up rows, then,
//     without waiting for anything, its share of the down rows, so HBM stays busy across the
//     grid barrier that makes h visible;
//   * eight consumer warps dot the rows against the activations held in registers (f16, the
//     lane's own K positions) with packed f16 FMAs per 16-input block, fold each block into
//     f32 with its E4M3 scale, and reduce across the warp;
//   * after the last barrier each CTA combines a slice of the output (f32 in slot order, one
//     BF16 rounding, optional residual), exactly as the combine kernel does.
//
// Weight layout: page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit
// residents", section "What this pack holds"; router logits and SwiGLU in FP32: page
// "Beam-1.0-501B-A23B VQ GGUF", section "What stays native".  The pages' "flat decode MoE
// scheduler" (page "Beam-1.0-501B-A23B, EXL3 3-bit, for 2x RTX PRO 6000 Blackwell", section
// "How it fits") likewise runs decode over one flat work list across experts.
#include "common.cuh"
#include "internal.h"
#include "route_warp.cuh"

namespace moe {

namespace {

constexpr int kNW = 8;                       // consumer warps
constexpr int kThreads1 = 32 * (kNW + 1);    // + one producer warp
constexpr int kRing = 4;                     // stages in the ring
constexpr int kMaxK = 32;

struct D1Params {
  const uint8_t* bank;
  uint64_t stride;
  uint64_t codes_off[3], scales_off[3], global_off[3];
  int global_mode;
  int E, k;
  const float* logits;   // [E]
  const uint16_t* x;     // [H] bf16
  uint16_t* out;         // [H] bf16
  uint16_t* x_next;      // [H] bf16 or null
  float* h;              // [k, I] f32 scratch
  float* y;              // [k, H] f32 scratch
  unsigned* bar;         // [2] grid-barrier counters, zero on entry
  int32_t* ids;          // [k] routing result (for inspection)
  float* w;              // [k]
};

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
__device__ __forceinline__ float2 f16x2_to_f2(uint32_t v) {
  float a, b;
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
      : "=f"(a), "=f"(b)
      : "r"(v));
  return make_float2(a, b);
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

// One 32-input unit: codes (4 words) and its two E4M3 block scales against 16 f16x2 of x.
__device__ __forceinline__ float unit_dot(const uint4 c, uint32_t sc2, const uint32_t (&x)[16]) {
  const float2 sf = f16x2_to_f2(e4m3x2_to_f16x2((uint16_t)sc2));
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
  const float2 a = f16x2_to_f2(hadd2_(p0, p0b)), b = f16x2_to_f2(hadd2_(p1, p1b));
  return fmaf(sf.x, a.x + a.y, sf.y * (b.x + b.y));
}

// Grid-wide barrier of the persistent grid (all CTAs resident: cooperative launch).  One
// thread per CTA; bounded: gives up after kWaitCycles, records a timeout and returns false.
__device__ bool grid_arrive_wait(unsigned* counter, unsigned target) {
  __threadfence();
  atomicAdd(counter, 1u);
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

// UG = H / 1024 units per lane per row (gate/up: 32 lanes x UG units x 32 inputs = H);
// UD = I / 512 units per lane over a pair of down rows.
template <int UG, int UD>
__global__ void __launch_bounds__(kThreads1, 1) decode1_kernel(const D1Params p) {
  constexpr int H = UG * 1024, I = UD * 512;
  constexpr int kCodes1 = kNW * H / 2, kScales1 = kNW * H / 16;       // per matrix, 8 rows
  constexpr int kStage1 = 2 * (kCodes1 + kScales1);
  constexpr int kRows2 = 2 * kNW;                                     // down rows per stage
  constexpr int kCodes2 = kRows2 * I / 2, kScales2 = kRows2 * I / 16;
  constexpr int kStage2 = kCodes2 + kScales2;
  constexpr int kStage = kStage1 > kStage2 ? kStage1 : kStage2;
  constexpr int kUnits2 = I / 32;                                     // units per down row

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRing * kStage);
  uint64_t* empty = full + kRing;
  int* s_ids = reinterpret_cast<int*>(empty + kRing);
  float* s_w = reinterpret_cast<float*>(s_ids + kMaxK);
  float* s_gm = s_w + kMaxK;                                // [3][kMaxK] global multipliers
  int* s_ok = reinterpret_cast<int*>(s_gm + 3 * kMaxK);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = p.k;
  const int n1 = k * (I / kNW), n2 = k * (H / kRows2);      // stages of each phase, whole grid
  int lo1, hi1, lo2, hi2;
  share(n1, blockIdx.x, gridDim.x, lo1, hi1);
  share(n2, blockIdx.x, gridDim.x, lo2, hi2);
  const int cnt1 = hi1 - lo1, cnt = cnt1 + (hi2 - lo2);     // this CTA's stages, both phases

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kNW);
    }
    *s_ok = 1;
    fence_barrier_init();
  }
  if (warp == 0) {                                          // every CTA routes the token
    int id;
    float wt;
    route_row(p.logits, p.E, k, lane, id, wt);
    if (lane < k) {
      s_ids[lane] = id;
      s_w[lane] = wt;
      const uint8_t* rec = p.bank + (uint64_t)id * p.stride;
#pragma unroll
      for (int m = 0; m < 3; ++m)
        s_gm[m * kMaxK + lane] =
            global_mult(__ldg(reinterpret_cast<const float*>(rec + p.global_off[m])), p.global_mode);
      if (blockIdx.x == 0) {
        p.ids[lane] = id;
        p.w[lane] = wt;
      }
    }
  }
  __syncthreads();

  if (warp == kNW) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int q = 0;
      for (; q < cnt; ++q) {
        const int s = q % kRing;
        if (!mbar_wait(&empty[s], ((q / kRing) & 1) ^ 1)) break;
        uint8_t* dst = smem + s * kStage;
        if (q < cnt1) {
          const int u = lo1 + q, j = u / (I / kNW), r0 = (u - j * (I / kNW)) * kNW;
          const uint8_t* rec = p.bank + (uint64_t)s_ids[j] * p.stride;
          mbar_arrive_expect_tx(&full[s], kStage1);
          bulk_g2s(dst, rec + p.codes_off[0] + (uint64_t)r0 * (H / 2), kCodes1, &full[s], pol);
          bulk_g2s(dst + kCodes1, rec + p.codes_off[1] + (uint64_t)r0 * (H / 2), kCodes1, &full[s], pol);
          bulk_g2s(dst + 2 * kCodes1, rec + p.scales_off[0] + (uint64_t)r0 * (H / 16), kScales1, &full[s], pol);
          bulk_g2s(dst + 2 * kCodes1 + kScales1, rec + p.scales_off[1] + (uint64_t)r0 * (H / 16), kScales1,
                   &full[s], pol);
        } else {
          const int u = lo2 + (q - cnt1), j = u / (H / kRows2), r0 = (u - j * (H / kRows2)) * kRows2;
          const uint8_t* rec = p.bank + (uint64_t)s_ids[j] * p.stride;
          mbar_arrive_expect_tx(&full[s], kStage2);
          bulk_g2s(dst, rec + p.codes_off[2] + (uint64_t)r0 * (I / 2), kCodes2, &full[s], pol);
          bulk_g2s(dst + kCodes2, rec + p.scales_off[2] + (uint64_t)r0 * (I / 16), kScales2, &full[s], pol);
        }
      }
      // Leave no copy in flight (only an error path gets here with copies outstanding).
      for (int i = q - kRing > 0 ? q - kRing : 0; i < q; ++i) mbar_wait(&full[i % kRing], (i / kRing) & 1);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers
    const uint32_t sbase = smem_addr(smem);
    bool ok = true;
    // Phase 1: gate/up.  Warp w takes row r0 + w of both matrices; lane l its units
    // l + 32 u (u < UG) of the row, with x at those K positions held in registers.
    uint32_t xr[UG][16];
#pragma unroll
    for (int u = 0; u < UG; ++u) {
      const uint16_t* xp = p.x + 32 * (lane + 32 * u);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(xp + 8 * q));
        xr[u][4 * q + 0] = pack_f16x2(bf16_bits_to_f32(b.x & 0xFFFF), bf16_bits_to_f32(b.x >> 16));
        xr[u][4 * q + 1] = pack_f16x2(bf16_bits_to_f32(b.y & 0xFFFF), bf16_bits_to_f32(b.y >> 16));
        xr[u][4 * q + 2] = pack_f16x2(bf16_bits_to_f32(b.z & 0xFFFF), bf16_bits_to_f32(b.z >> 16));
        xr[u][4 * q + 3] = pack_f16x2(bf16_bits_to_f32(b.w & 0xFFFF), bf16_bits_to_f32(b.w >> 16));
      }
    }
    int q = 0;
    for (; q < cnt1 && ok; ++q) {
      const int s = q % kRing;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (q / kRing) & 1))) {
        ok = false;
        break;
      }
      const int u0 = lo1 + q, j = u0 / (I / kNW), r = (u0 - j * (I / kNW)) * kNW + warp;
      const uint32_t st = sbase + s * kStage;
      const uint32_t cg = st + warp * (H / 2), cu = st + kCodes1 + warp * (H / 2);
      const uint32_t sg = st + 2 * kCodes1 + warp * (H / 16), su = sg + kScales1;
      float accG = 0.0f, accU = 0.0f;
#pragma unroll
      for (int u = 0; u < UG; ++u) {
        const int un = lane + 32 * u;
        accG += unit_dot(lds128(cg + un * 16), lds16(sg + un * 2), xr[u]);
      }
#pragma unroll
      for (int u = 0; u < UG; ++u) {
        const int un = lane + 32 * u;
        accU += unit_dot(lds128(cu + un * 16), lds16(su + un * 2), xr[u]);
      }
      fence_proxy_async_smem();            // the reads above come before the slot's next TMA
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        accG += __shfl_xor_sync(0xFFFFFFFFu, accG, off);
        accU += __shfl_xor_sync(0xFFFFFFFFu, accU, off);
      }
      if (lane == 0) p.h[(size_t)j * I + r] = silu_mul(accG * s_gm[j], accU * s_gm[kMaxK + j]);
    }
    // Grid barrier 1: every h row written.
    named_bar_sync(1, 32 * kNW);
    if (threadIdx.x == 0) *s_ok = (ok && grid_arrive_wait(&p.bar[0], gridDim.x)) ? 1 : 0;
    named_bar_sync(1, 32 * kNW);
    ok = ok && *s_ok;

    // Phase 2: down.  Warp w takes rows r0 + 2w, r0 + 2w + 1 of the stage; lane l its units
    // cu = l + 32 u (u < UD) of the two rows laid end to end: row cu / kUnits2, K unit
    // cu % kUnits2, with h at those K positions in registers (reloaded when the slot changes).
    uint32_t hr[UD][16];
    int hj = -1;
    for (; q < cnt && ok; ++q) {
      const int s = q % kRing;
      const int u0 = lo2 + (q - cnt1), j = u0 / (H / kRows2), r0 = (u0 - j * (H / kRows2)) * kRows2 + 2 * warp;
      if (j != hj) {
        hj = j;
        const float* hp = p.h + (size_t)j * I;
#pragma unroll
        for (int u = 0; u < UD; ++u) {
          const int ku = (lane + 32 * u) % kUnits2;
          const float4* src = reinterpret_cast<const float4*>(hp + 32 * ku);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 a = __ldcg(src + q4);
            hr[u][2 * q4] = pack_f16x2(a.x, a.y);
            hr[u][2 * q4 + 1] = pack_f16x2(a.z, a.w);
          }
        }
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (q / kRing) & 1))) {
        ok = false;
        break;
      }
      const uint32_t st = sbase + s * kStage;
      const uint32_t cd = st + 2 * warp * (I / 2), sd = st + kCodes2 + 2 * warp * (I / 16);
      float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
      for (int u = 0; u < UD; ++u) {
        const int cu = lane + 32 * u;                       // unit within the pair of rows
        const float part = unit_dot(lds128(cd + cu * 16), lds16(sd + cu * 2), hr[u]);
        if (cu < kUnits2)
          acc0 += part;
        else
          acc1 += part;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        acc0 += __shfl_xor_sync(0xFFFFFFFFu, acc0, off);
        acc1 += __shfl_xor_sync(0xFFFFFFFFu, acc1, off);
      }
      if (lane < 2) p.y[(size_t)j * H + r0 + lane] = (lane == 0 ? acc0 : acc1) * s_gm[2 * kMaxK + j];
    }
    // Grid barrier 2: every y row written.
    named_bar_sync(1, 32 * kNW);
    if (threadIdx.x == 0) *s_ok = (ok && grid_arrive_wait(&p.bar[1], gridDim.x)) ? 1 : 0;
    named_bar_sync(1, 32 * kNW);
    if (*s_ok) {
      // Combine: out[c] = bf16(sum_j w_j y[j][c]) in slot order; x_next = bf16(x + out).
      int c0, c1;
      share(H / 8, blockIdx.x, gridDim.x, c0, c1);
      for (int cc = c0 + (int)threadIdx.x; cc < c1; cc += 32 * kNW) {
        const int c = 8 * cc;
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int j = 0; j < k; ++j) {
          const float wj = s_w[j];
          const float4* src = reinterpret_cast<const float4*>(p.y + (size_t)j * H + c);
          const float4 a = __ldcg(src), b = __ldcg(src + 1);
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
        *reinterpret_cast<uint4*>(p.out + c) =
            make_uint4(o[0] | (o[1] << 16), o[2] | (o[3] << 16), o[4] | (o[5] << 16), o[6] | (o[7] << 16));
        if (p.x_next != nullptr) {
          const uint4 xv = __ldg(reinterpret_cast<const uint4*>(p.x + c));
          const uint32_t xs[8] = {xv.x & 0xFFFF, xv.x >> 16, xv.y & 0xFFFF, xv.y >> 16,
                                  xv.z & 0xFFFF, xv.z >> 16, xv.w & 0xFFFF, xv.w >> 16};
          uint32_t rr[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) rr[i] = f32_to_bf16_bits(bf16_bits_to_f32(xs[i]) + bf16_bits_to_f32(o[i]));
          *reinterpret_cast<uint4*>(p.x_next + c) =
              make_uint4(rr[0] | (rr[1] << 16), rr[2] | (rr[3] << 16), rr[4] | (rr[5] << 16), rr[6] | (rr[7] << 16));
        }
      }
    }
  }
}

template <int UG, int UD>
int launch_d1(const D1Params& p, int num_sms, cudaStream_t s) {
  constexpr int H = UG * 1024, I = UD * 512;
  constexpr int kStage1 = 2 * (kNW * H / 2 + kNW * H / 16);
  constexpr int kStage2 = 2 * kNW * I / 2 + 2 * kNW * I / 16;
  constexpr int kStage = kStage1 > kStage2 ? kStage1 : kStage2;
  const int smem = kRing * kStage + 2 * kRing * 8 + 5 * kMaxK * 4 + 16;
  auto kern = decode1_kernel<UG, UD>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return -(int)err;
  // Cooperative launch: all CTAs are resident at once, which the grid barriers need.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms);
  cfg.blockDim = dim3(kThreads1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, kern, p);
  return err == cudaSuccess ? 1 : -(int)err;
}

}  // namespace

bool decode1_supported(int H, int I, int k) {
  if (k > kMaxK) return false;
  return (H == 5120 && I == 2560) || (H == 1024 && I == 512) || (H == 2048 && I == 1024) ||
         (H == 4096 && I == 1536);
}

int launch_decode1(const BankView& bank, const float* logits, int k, const uint16_t* x, uint16_t* out,
                   uint16_t* x_next, float* h, float* y, unsigned* bar, int32_t* ids, float* w, int num_sms,
                   cudaStream_t s) {
  D1Params p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  for (int m = 0; m < 3; ++m) {
    p.codes_off[m] = bank.codes_off[m];
    p.scales_off[m] = bank.scales_off[m];
    p.global_off[m] = bank.global_off[m];
  }
  p.global_mode = bank.global_mode;
  p.E = bank.E;
  p.k = k;
  p.logits = logits;
  p.x = x;
  p.out = out;
  p.x_next = x_next;
  p.h = h;
  p.y = y;
  p.bar = bar;
  p.ids = ids;
  p.w = w;
  cudaError_t err = cudaMemsetAsync(bar, 0, 2 * sizeof(unsigned), s);
  if (err != cudaSuccess) return -(int)err;
  if (bank.H == 5120 && bank.I == 2560) return launch_d1<5, 5>(p, num_sms, s);
  if (bank.H == 1024 && bank.I == 512) return launch_d1<1, 1>(p, num_sms, s);
  if (bank.H == 2048 && bank.I == 1024) return launch_d1<2, 2>(p, num_sms, s);
  if (bank.H == 4096 && bank.I == 1536) return launch_d1<4, 3>(p, num_sms, s);
  return -(int)cudaErrorInvalidValue;
}

}  // namespace moe
