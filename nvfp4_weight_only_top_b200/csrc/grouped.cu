// Decode of larger batches (more tokens than the few-token kernel takes, up to the prefill
// switch): after the router, two persistent kernels -- gate/up + SwiGLU, then down -- over the
// router's groups (up to 8 routed rows of one expert, in expert order), then the combine kernel.
//
// A stage is a block of whole weight rows, contiguous in the record: 8 gate rows + the same 8 up
// rows (gate/up), or 32 down rows; the stages of the CTA's contiguous share of the flat (group,
// stage) list stream with 1-D bulk copies (TMA) into a shared-memory ring.  Every stage ends in a
// CTA-wide barrier (the sum of the warps' partials), after which one thread refills the slot just
// read with the stage kGRing ahead -- so no warp is set aside as a producer, and each thread may
// hold 255 registers.
// Eight consumer warps split K: for gate/up warp w takes the 128-input units w, w + 8, ... of the
// stage's one 16-row tile (8 gate rows over 8 up rows); for down, warp w takes the units w % 4,
// w % 4 + 4, ... of tile w / 4 (two 16-row tiles per stage).  Each runs mma.sync m16n8k16 with the
// weights as A (E2M1 -> f16 by cvt, times the E4M3 block scale in f16: both exact) and the
// group's 8 rows of activations as B (N = 8).  The activations of a group stay in registers for
// all its stages, in f16 after an exact power-of-two prescale per row (from the row's largest
// magnitude, collected across the CTA; undone in f32).  The warps' partial sums are added in a
// fixed order through shared memory; the global scales and SwiGLU follow in f32.
//
// The MMA's 16 logical k of a row come from four threads: thread tid4 supplies 4 K values of its
// own 32-wide slice of the unit per k-step (8 steps per unit) and takes the activations at the
// same K positions, so the weights need no exchange between threads and the block scale can be
// applied to A before the MMA.
//
// Weight layout: page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents",
// section "What this pack holds"; SwiGLU in FP32: page "Beam-1.0-501B-A23B VQ GGUF", section
// "What stays native".  The pages' "flat decode MoE scheduler" (page "Beam-1.0-501B-A23B, EXL3
// 3-bit, for 2x RTX PRO 6000 Blackwell", section "How it fits") likewise runs decode over one
// flat work list across experts.
#include "common.cuh"
#include "internal.h"
#include "decode_fused.cuh"

namespace moe {

namespace {

constexpr int kGW = 8;                       // warps (all compute; thread 0 also issues the copies)
constexpr int kGThreads = 32 * kGW;
constexpr int kGRing = 3;                    // stages in the ring
constexpr int kGRows = 8;                    // routed rows per group (MMA N)

struct GParams {
  const uint8_t* bank;
  uint64_t stride;
  uint64_t codes_off[2], scales_off[2], global_off[2];   // gate/up: [0] gate, [1] up; down: [0]
  int global_mode;
  int k;                     // routing top-k: permuted row q holds token perm[q] / k
  const int4* groups;        // (expert, first permuted row, rows 1..8, 0)
  const int32_t* ngroups;
  const int32_t* perm;
  const void* xin;           // gate/up: bf16 x [T, H]; down: f32 h [R, I] (permuted rows)
  float* out;                // gate/up: h [R, I]; down: y [R, H] (permuted rows)
};

// H = UG x 1024, I = UD x 512.  Gate/up: K = H, stage = 8 gate + 8 up rows, UG units per warp.
// Down: K = I, stage = 32 rows (two tiles), UD units per warp.
template <int UG, int UD, bool GATEUP>
__global__ void __launch_bounds__(kGThreads, 1) grouped_kernel(const GParams p) {
  constexpr int H = UG * 1024, I = UD * 512;
  constexpr int K = GATEUP ? H : I;                        // inputs per weight row
  constexpr int NOUT = GATEUP ? I : H;                     // output rows per matrix
  constexpr int U = GATEUP ? UG : UD;                      // 128-input units per warp and stage
  constexpr int kRowsSt = GATEUP ? 8 : 32;                 // rows per stage (per matrix)
  constexpr int kCodesM = kRowsSt * K / 2, kScalesM = kRowsSt * K / 16;
  // A ring slot holds the stage's code rows back to back (each matrix one contiguous copy), then
  // the scale rows.  (One copy per row with a padded pitch would avoid the 2-way bank conflicts of
  // the 8 rows a warp reads at once, but 16-32 small copies per stage streamed far slower.)
  constexpr int kPitch = K / 2;
  constexpr int kMats = GATEUP ? 2 : 1;
  constexpr int kScBase = kMats * kCodesM;                 // scales follow the code rows
  constexpr int kStage = kScBase + kMats * kScalesM;       // bytes of a ring slot
  constexpr int kTx = kStage;                              // bytes the copies of a stage deliver
  constexpr int kSpg = NOUT / kRowsSt;                     // stages per group
  constexpr int kUStep = GATEUP ? kGW : 4;                 // unit stride between a warp's units
  static_assert(kStage % 128 == 0 && kPitch % 16 == 0, "stage alignment");

  extern __shared__ __align__(128) uint8_t smem[];
  float4* red = reinterpret_cast<float4*>(smem + kGRing * kStage);      // [2][kGW][32] partial sums
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 2 * kGW * 32);
  uint32_t* s_wmax = reinterpret_cast<uint32_t*>(full + kGRing);       // [kGW][kGRows] row maxima
  int* s_abort = reinterpret_cast<int*>(s_wmax + kGW * kGRows);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tid4 = lane & 3;
  const int total = *p.ngroups * kSpg;
  const int lo = (int)(((long long)total * blockIdx.x) / gridDim.x);
  const int hi = (int)(((long long)total * (blockIdx.x + 1)) / gridDim.x);
  const int cnt = hi - lo;
  if (cnt <= 0) return;                                    // the same for every thread of the CTA
  // Stage q of this CTA into ring slot q % kGRing (thread 0 only).
  auto issue = [&](int q) {
    const uint64_t pol = policy_evict_first();
    const int s = q % kGRing;
    const int u = lo + q, g = u / kSpg, st = u - g * kSpg;
    const uint8_t* rec = p.bank + (uint64_t)__ldg(&p.groups[g].x) * p.stride;
    const uint64_t r0 = (uint64_t)st * kRowsSt;
    uint8_t* dst = smem + s * kStage;
    mbar_arrive_expect_tx(&full[s], kTx);
#pragma unroll
    for (int m = 0; m < kMats; ++m) {
      bulk_g2s(dst + m * kCodesM, rec + p.codes_off[m] + r0 * (K / 2), kCodesM, &full[s], pol);
      bulk_g2s(dst + kScBase + m * kScalesM, rec + p.scales_off[m] + r0 * (K / 16), kScalesM, &full[s], pol);
    }
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGRing; ++s) mbar_init(&full[s], 1);
    *s_abort = 0;
    fence_barrier_init();
    for (int q = 0; q < cnt && q < kGRing; ++q) issue(q);
  }
  __syncthreads();

  const uint32_t sbase = smem_addr(smem);
  const int tile = GATEUP ? 0 : warp >> 2;                 // down: rows 16 tile .. 16 tile + 15
  const int u0 = GATEUP ? warp : (warp & 3);               // first unit of this warp
  // A rows of this thread inside a stage: gate/up: gate row gid and up row gid; down: rows
  // 16 tile + gid and 16 tile + gid + 8.
  // (the second row is a fixed distance further: the up matrix, or 8 rows down)
  const int row_a = GATEUP ? gid : 16 * tile + gid;
  constexpr uint32_t kCodeB = 8 * kPitch, kScB = GATEUP ? kScalesM : 8 * (K / 16);
  uint32_t xr[U][16];                                      // B: row gid's f16 at this thread's K
  int cur_g = -1, q0 = 0, nrows = 0, issued = cnt < kGRing ? cnt : kGRing;
  float gm0 = 0.0f, gm1 = 0.0f;
  float un0 = 1.0f, un1 = 1.0f;                            // 2^-s of columns 2 tid4 and 2 tid4 + 1
  bool ok = true;
  for (int q = 0; q < cnt; ++q) {
    const int u = lo + q, g = u / kSpg, st = u - g * kSpg;
    if (g != cur_g) {
      // ---- a new group: its rows' activations into registers, prescaled into f16
      cur_g = g;
      const int4 grp = __ldg(&p.groups[g]);
      q0 = grp.y;
      nrows = grp.z;
      const uint8_t* rec = p.bank + (uint64_t)grp.x * p.stride;
      gm0 = global_mult(__ldg(reinterpret_cast<const float*>(rec + p.global_off[0])), p.global_mode);
      gm1 = GATEUP ? global_mult(__ldg(reinterpret_cast<const float*>(rec + p.global_off[1])), p.global_mode) : 0.0f;
      const bool has = gid < nrows;
      uint32_t m = 0;
      // The rows' largest magnitudes first; a second pass loads and converts (L1 hits).
      const uint16_t* xrow = GATEUP ? static_cast<const uint16_t*>(p.xin) +
                                          (size_t)(has ? __ldg(&p.perm[q0 + gid]) / p.k : 0) * H
                                    : nullptr;
      if (GATEUP) {
#pragma unroll 1
        for (int j = 0; j < U; ++j) {
          const uint4* src = reinterpret_cast<const uint4*>(xrow + (u0 + kUStep * j) * 128 + 32 * tid4);
#pragma unroll
          for (int c = 0; c < 4; ++c) m = max(m, bf16x8_abs_max_bits(has ? __ldg(src + c) : make_uint4(0, 0, 0, 0)));
        }
      } else {
        // f32 mid values: the largest magnitude first (a second pass loads and converts)
        const float* hrow = static_cast<const float*>(p.xin) + (size_t)(has ? q0 + gid : 0) * I;
#pragma unroll 1
        for (int j = 0; j < U; ++j) {
          const float4* src = reinterpret_cast<const float4*>(hrow + (u0 + kUStep * j) * 128 + 32 * tid4);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 v = has ? __ldcg(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            m = max(m, max(max(f32_abs_bits(v.x), f32_abs_bits(v.y)), max(f32_abs_bits(v.z), f32_abs_bits(v.w))));
          }
        }
      }
      // row gid's maximum: over the 4 lanes of the row in this warp, then over the warps
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      if (tid4 == 0) s_wmax[warp * kGRows + gid] = m;
      named_bar_sync(1, 32 * kGW);
      uint32_t mg = 0, mc0 = 0, mc1 = 0;
#pragma unroll
      for (int w = 0; w < kGW; ++w) {
        mg = max(mg, s_wmax[w * kGRows + gid]);
        mc0 = max(mc0, s_wmax[w * kGRows + 2 * tid4]);
        mc1 = max(mc1, s_wmax[w * kGRows + 2 * tid4 + 1]);
      }
      named_bar_sync(1, 32 * kGW);                         // s_wmax may be rewritten afterwards
      if (GATEUP) {
        const float f = exp2_int(prescale_shift_bf16(mg));
        un0 = exp2_int(-prescale_shift_bf16(mc0));
        un1 = exp2_int(-prescale_shift_bf16(mc1));
#pragma unroll
        for (int j = 0; j < U; ++j) {
          const uint4* src = reinterpret_cast<const uint4*>(xrow + (u0 + kUStep * j) * 128 + 32 * tid4);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = has ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
              xr[j][4 * c + i] = pack_f16x2(bf16_bits_to_f32(w[i] & 0xFFFFu) * f, bf16_bits_to_f32(w[i] >> 16) * f);
          }
        }
      } else {
        const float f = exp2_int(prescale_shift_f32(mg));
        un0 = exp2_int(-prescale_shift_f32(mc0));
        un1 = exp2_int(-prescale_shift_f32(mc1));
        const float* hrow = static_cast<const float*>(p.xin) + (size_t)(has ? q0 + gid : 0) * I;
#pragma unroll
        for (int j = 0; j < U; ++j) {
          const float4* src = reinterpret_cast<const float4*>(hrow + (u0 + kUStep * j) * 128 + 32 * tid4);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 v = has ? __ldcg(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            xr[j][2 * c] = pack_f16x2(v.x * f, v.y * f);
            xr[j][2 * c + 1] = pack_f16x2(v.z * f, v.w * f);
          }
        }
      }
    }
    // ---- the stage: partial sums over this warp's units
    const int s = q % kGRing;
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (q / kGRing) & 1))) ok = false;
    // four independent accumulators (one per code word of a unit), so that consecutive MMAs do not
    // wait for each other's results; added at the end
    float acc[4][4] = {};
    if (ok) {
      const uint32_t cbase = sbase + s * kStage + row_a * kPitch + u0 * 64 + tid4 * 16;
      const uint32_t sbase2 = sbase + s * kStage + kScBase + row_a * (K / 16) + u0 * 8 + tid4 * 2;
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const uint4 wa = fused::lds128(cbase + j * kUStep * 64);
        const uint4 wb = fused::lds128(cbase + kCodeB + j * kUStep * 64);
        const uint32_t hsa = e4m3x2_to_f16x2((uint16_t)fused::lds16(sbase2 + j * kUStep * 8));
        const uint32_t hsb = e4m3x2_to_f16x2((uint16_t)fused::lds16(sbase2 + kScB + j * kUStep * 8));
        const uint32_t ca[4] = {wa.x, wa.y, wa.z, wa.w}, cb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          // words 0, 1: inputs 0..15 of the thread's 32-input slice (first block), words 2, 3: second
          const uint32_t sA = bcast_half(hsa, w4 >= 2), sB = bcast_half(hsb, w4 >= 2);
          uint32_t fa[4], fb[4];
          e2m1x8_to_f16x8(ca[w4], fa);
          e2m1x8_to_f16x8(cb[w4], fb);
          const uint32_t a0[4] = {hmul2(fa[0], sA), hmul2(fb[0], sB), hmul2(fa[1], sA), hmul2(fb[1], sB)};
          mma_16816(acc[w4], a0, xr[j][4 * w4], xr[j][4 * w4 + 1]);
          const uint32_t a1[4] = {hmul2(fa[2], sA), hmul2(fb[2], sB), hmul2(fa[3], sA), hmul2(fb[3], sB)};
          mma_16816(acc[w4], a1, xr[j][4 * w4 + 2], xr[j][4 * w4 + 3]);
        }
      }
      fence_proxy_async_smem();            // the reads above come before the slot's next TMA
    }
    // ---- fixed-order sum of the warps' partials, then the epilogue
    const int buf = q & 1;
    red[(buf * kGW + warp) * 32 + lane] =
        make_float4((acc[0][0] + acc[1][0]) + (acc[2][0] + acc[3][0]), (acc[0][1] + acc[1][1]) + (acc[2][1] + acc[3][1]),
                    (acc[0][2] + acc[1][2]) + (acc[2][2] + acc[3][2]), (acc[0][3] + acc[1][3]) + (acc[2][3] + acc[3][3]));
    if (!ok) *s_abort = 1;
    named_bar_sync(1, 32 * kGW);
    if (*s_abort) break;                                    // every warp leaves together
    // every warp has read stage q: its slot takes stage q + kGRing
    if (issued < cnt) {
      if (threadIdx.x == 0) issue(issued);
      ++issued;
    }
    // acc[0..1]: A row gid, columns (routed rows of the group) 2 tid4, 2 tid4 + 1; acc[2..3]: row gid + 8
    if (GATEUP) {
      if (warp == q % kGW) {
        float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < kGW; ++w) {
          const float4 v = red[(buf * kGW + w) * 32 + lane];
          c[0] += v.x, c[1] += v.y, c[2] += v.z, c[3] += v.w;
        }
        const int row = st * kRowsSt + gid;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int n = 2 * tid4 + cc;
          const float un = cc ? un1 : un0;
          if (n < nrows) p.out[(size_t)(q0 + n) * I + row] = silu_mul(c[cc] * un * gm0, c[2 + cc] * un * gm1);
        }
      }
    } else {
      if ((warp & 3) == (q & 3)) {                          // one warp per tile
        float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float4 v = red[(buf * kGW + 4 * tile + w) * 32 + lane];
          c[0] += v.x, c[1] += v.y, c[2] += v.z, c[3] += v.w;
        }
        const int row = st * kRowsSt + 16 * tile + gid;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int n = 2 * tid4 + cc;
          const float un = cc ? un1 : un0;
          if (n < nrows) {
            float* o = p.out + (size_t)(q0 + n) * H;
            o[row] = c[cc] * un * gm0;
            o[row + 8] = c[2 + cc] * un * gm0;
          }
        }
      }
    }
  }
  // Leave no copy in flight (only an abandoned run has copies outstanding here): at most the last
  // kGRing stages issued.
  if (threadIdx.x == 0 && *s_abort)
    for (int q = issued - kGRing > 0 ? issued - kGRing : 0; q < issued; ++q) mbar_wait(&full[q % kGRing], (q / kGRing) & 1);
}

template <int UG, int UD, bool GATEUP>
int launch_g(const GParams& p, int num_sms, cudaStream_t s) {
  constexpr int H = UG * 1024, I = UD * 512;
  constexpr int K = GATEUP ? H : I;
  constexpr int kRowsSt = GATEUP ? 8 : 32;
  constexpr int kStage = (GATEUP ? 2 : 1) * (kRowsSt * K / 2 + kRowsSt * K / 16);
  const int smem = kGRing * kStage + 2 * kGW * 32 * 16 + kGRing * 8 + kGW * kGRows * 4 + 16;
  auto kern = grouped_kernel<UG, UD, GATEUP>;
  cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (err != cudaSuccess) return -(int)err;
  kern<<<num_sms, kGThreads, smem, s>>>(p);
  err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

template <bool GATEUP>
int launch_shape(const BankView& bank, const GParams& p, int num_sms, cudaStream_t s) {
  if (bank.H == 5120 && bank.I == 2560) return launch_g<5, 5, GATEUP>(p, num_sms, s);
  if (bank.H == 1024 && bank.I == 512) return launch_g<1, 1, GATEUP>(p, num_sms, s);
  if (bank.H == 2048 && bank.I == 1024) return launch_g<2, 2, GATEUP>(p, num_sms, s);
  if (bank.H == 4096 && bank.I == 1536) return launch_g<4, 3, GATEUP>(p, num_sms, s);
  return -(int)cudaErrorInvalidValue;
}

}  // namespace

bool grouped_supported(int H, int I) {
  return (H == 5120 && I == 2560) || (H == 1024 && I == 512) || (H == 2048 && I == 1024) ||
         (H == 4096 && I == 1536);
}

int launch_grouped_gateup(const BankView& bank, const uint16_t* x, int k, const RouteBufs& rb, float* h, int num_sms,
                          cudaStream_t s) {
  GParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  for (int m = 0; m < 2; ++m) {
    p.codes_off[m] = bank.codes_off[m];
    p.scales_off[m] = bank.scales_off[m];
    p.global_off[m] = bank.global_off[m];
  }
  p.global_mode = bank.global_mode;
  p.k = k;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.perm = rb.perm;
  p.xin = x;
  p.out = h;
  return launch_shape<true>(bank, p, num_sms, s);
}

int launch_grouped_down(const BankView& bank, const float* h, const RouteBufs& rb, float* y, int num_sms,
                        cudaStream_t s) {
  GParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  p.codes_off[0] = p.codes_off[1] = bank.codes_off[2];
  p.scales_off[0] = p.scales_off[1] = bank.scales_off[2];
  p.global_off[0] = p.global_off[1] = bank.global_off[2];
  p.global_mode = bank.global_mode;
  p.k = 1;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.perm = rb.perm;
  p.xin = h;
  p.out = y;
  return launch_shape<false>(bank, p, num_sms, s);
}

}  // namespace moe
