// Decode of a single token (T = 1) as ONE persistent kernel: route -> gate/up + SwiGLU ->
// down -> combine, with no grid-wide barrier and no other launch.
//
// With one token every routed row is its own expert, the work is 2 FLOP per weight byte, and
// the layer is a pure stream of k expert records (177 MB at E=256, k=8, H=5120, I=2560) from
// HBM.  What costs time besides the bytes is the number of dependent steps, so:
//   * every CTA routes the token itself (top-k of E logits in the router's order: logit
//     descending, lower index first; softmax over the k in f32): no router kernel, no hand-off;
//   * one producer warp per CTA streams the CTA's weight rows with large 1-D bulk copies
//     (TMA) into a 4-stage shared-memory ring -- first its share of the gate/up rows, then,
//     without waiting for anything, its share of the down rows;
//   * the work is cut into contiguous shares so that a CTA's down rows belong to the same one
//     or two slots (experts) as its gate/up rows: before its down rows a CTA waits only until
//     the h of those slots is complete (a per-slot counter), not for the whole grid;
//   * eight consumer warps dot the rows against the activations held in registers (f16, the
//     lane's own K positions) with packed f16 FMAs per 16-input block, fold each block into
//     f32 with its E4M3 scale, and reduce across the warp;
//   * the combine of a block of 32 output rows is done by the CTA that writes the block's last
//     y values (a per-block counter), in slot order with f32 accumulation and one BF16
//     rounding (and the optional residual), exactly as the combine kernel does;
//   * the completion counters come from a library-owned pool of counter sets that every call
//     leaves at zero (the last CTA clears its set), so a call is this one launch, nothing else.
//
// Weight layout: page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit
// residents", section "What this pack holds"; router logits and SwiGLU in FP32: page
// "Beam-1.0-501B-A23B VQ GGUF", section "What stays native".  The pages' "flat decode MoE
// scheduler" (page "Beam-1.0-501B-A23B, EXL3 3-bit, for 2x RTX PRO 6000 Blackwell", section
// "How it fits") likewise runs decode over one flat work list across experts.
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "decode_fused.cuh"
#include "route_warp.cuh"

namespace moe {

namespace {

using namespace fused;

constexpr int kNW = 8;                       // consumer warps
constexpr int kThreads1 = 32 * (kNW + 1);    // + one producer warp
constexpr int kRing = 4;                     // stages in the ring
constexpr int kMaxK = 32;
constexpr int kMaxBlocks = 256;              // H / 32 row blocks of the combine
constexpr int kMaxLast = 64;                 // down stages of one CTA (bound checked on the host)
constexpr int kMaxRankE = 256;               // experts routed by the in-kernel rank count
// Completion counters: kMaxK per-slot counts, kMaxBlocks per-block counts, one exit count.
constexpr int kCounterWords = kMaxK + kMaxBlocks + 1;
constexpr int kCounterSets = 64;             // calls that may be in flight at once per device

// Counter sets owned by the library, one used per call in turn.  They start at zero (module
// load) and each call leaves its set at zero again (the last CTA to finish clears it), so no
// call needs a memset.
__device__ unsigned g_d1_counters[kCounterSets][kCounterWords];

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
  unsigned* bar;         // [kCounterWords] completion counters: zero on entry, zero again on exit
  int32_t* ids;          // [k] routing result (for inspection)
  float* w;              // [k]
};

// UG = H / 1024 units per lane per row (gate/up: 32 lanes x UG units x 32 inputs = H);
// UD = I / 512 units per lane over a pair of down rows.
template <int UG, int UD>
__global__ void __launch_bounds__(kThreads1, 1) decode1_kernel(const D1Params p) {
  constexpr int H = UG * 1024, I = UD * 512;
  constexpr int kCodes1 = kNW * H / 2, kScales1 = kNW * H / 16;       // per matrix, 8 rows
  constexpr int kStage1 = 2 * (kCodes1 + kScales1);
  constexpr int kRows2 = 4 * kNW;                                     // down rows per stage
  constexpr int kCodes2 = kRows2 * I / 2, kScales2 = kRows2 * I / 16;
  constexpr int kStage2 = kCodes2 + kScales2;
  constexpr int kStage = kStage1 > kStage2 ? kStage1 : kStage2;
  constexpr int kUnits2 = I / 32;                                     // units per down row
  static_assert((kRing * kStage + H * 2 + 2 * I * 4) % 16 == 0, "16-byte alignment of the routing keys");

  extern __shared__ __align__(128) uint8_t smem[];
  // ring | x (bf16 [H]) | h of up to two slots (f32 [2][I]) | barriers, routing
  uint16_t* sx = reinterpret_cast<uint16_t*>(smem + kRing * kStage);
  float* sh = reinterpret_cast<float*>(sx + H);
  // Routing keys first: they are read as 16-byte pairs and need 16-byte alignment (the
  // offset here is a multiple of 16: ring stages, x and h all are).
  uint64_t* s_key = reinterpret_cast<uint64_t*>(sh + 2 * I);  // [kMaxRankE] routing keys
  uint64_t* full = s_key + kMaxRankE;
  uint64_t* empty = full + kRing;
  uint64_t* gm_full = empty + kRing;                        // the global multipliers are in s_gm
  int* s_ids = reinterpret_cast<int*>(gm_full + 1);
  float* s_w = reinterpret_cast<float*>(s_ids + kMaxK);
  float* s_gm = s_w + kMaxK;                                // [3][kMaxK]
  int* s_ok = reinterpret_cast<int*>(s_gm + 3 * kMaxK);
  // After s_ok and the kMaxLast blocks to combine: largest |x| pattern per warp ([0, 9)) and
  // largest |h| pattern per consumer warp and down slot ([16 + 2 w + slot]).
  uint32_t* s_amax = reinterpret_cast<uint32_t*>(s_ok + 1 + kMaxLast);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = p.k;
  const int n1 = k * (I / kNW), n2 = k * (H / kRows2);      // stages of each phase, whole grid
  int lo1, hi1, lo2, hi2;
  share(n1, blockIdx.x, gridDim.x, lo1, hi1);
  share(n2, blockIdx.x, gridDim.x, lo2, hi2);
  const int cnt1 = hi1 - lo1, cnt = cnt1 + (hi2 - lo2);     // this CTA's stages, both phases
  unsigned* slot_done = p.bar;                              // [k]: gate/up stages completed
  unsigned* block_done = p.bar + kMaxK;                     // [H/32]: down stages written

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kNW);
    }
    mbar_init(gm_full, 1);
    *s_ok = 1;
    fence_barrier_init();
  }
  // Every CTA routes the token itself.  Expert e's rank is the number of experts ahead of it
  // in the order (logit desc, index asc) -- the order of the warp router -- counted by one
  // thread per expert against all E keys; the experts of rank < k fill slots 0 .. k-1.
  // The logit and this thread's share of x are loaded together.  x goes to shared memory once
  // per CTA, already multiplied by the power of two 2^shx of its prescale into f16 (shx from the
  // largest |x|, reduced across the CTA while the routing keys are ranked), 16-byte chunk c of
  // 32-input unit u at chunk c ^ ((u >> 1) & 3) of the unit, so that the lanes of a warp, which
  // read consecutive units, hit different banks.
  constexpr int kXPer = (H / 8 + kThreads1 - 1) / kThreads1;
  uint4 xv[kXPer];
  {
    const int e = threadIdx.x;
    const float lg = (e < kMaxRankE && e < p.E) ? __ldg(p.logits + e) : 0.0f;
    uint32_t m = 0;
#pragma unroll
    for (int t = 0; t < kXPer; ++t) {
      const int i = (int)threadIdx.x + t * kThreads1;
      if (i < H / 8) {
        xv[t] = __ldg(reinterpret_cast<const uint4*>(p.x) + i);
        m = max(m, bf16x8_abs_max_bits(xv[t]));
      }
    }
    if (e < kMaxRankE) s_key[e] = e < p.E ? ((uint64_t)rank_key(lg) << 32) | (uint32_t)(0xFFFFFFFFu - e) : 0ull;
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (lane == 0) s_amax[warp] = m;
  }
  __syncthreads();
  int shx;                                                  // prescale shift of x
  {
    uint32_t m = 0;
#pragma unroll
    for (int w = 0; w <= kNW; ++w) m = max(m, s_amax[w]);
    shx = prescale_shift_bf16(m);
    const float f = exp2_int(shx);
#pragma unroll
    for (int t = 0; t < kXPer; ++t) {
      const int i = (int)threadIdx.x + t * kThreads1;
      if (i < H / 8) {
        const int u = i >> 2, c = i & 3;
        reinterpret_cast<uint4*>(sx)[4 * u + (c ^ ((u >> 1) & 3))] = bf16x8_scaled(xv[t], f);
      }
    }
  }
  if (threadIdx.x < p.E) {
    const uint64_t me = s_key[threadIdx.x];
    int ahead = 0;
    const ulonglong2* kk = reinterpret_cast<const ulonglong2*>(s_key);
#pragma unroll 8
    for (int i = 0; i < kMaxRankE / 2; ++i) {              // keys beyond E are 0: never ahead
      const ulonglong2 v = kk[i];
      ahead += (v.x > me) + (v.y > me);
    }
    if (ahead < k) s_ids[ahead] = threadIdx.x;
  }
  __syncthreads();
  // The producer starts streaming now; the softmax weights are only needed by the combine at the
  // end (after the consumer warps' later barriers), so warp 0 forms them while the first copies
  // are in flight.
  if (warp == 0) {                                          // softmax over the k selected
    const int id = lane < k ? s_ids[lane] : 0;
    const float l = lane < k ? __ldg(p.logits + id) : 0.0f;
    const float lmax = __shfl_sync(0xFFFFFFFFu, l, 0);
    const float ex = lane < k ? expf(l - lmax) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
    const float wt = ex / sum;
    if (lane < k) {
      s_w[lane] = wt;
      if (blockIdx.x == 0) {
        p.ids[lane] = id;
        p.w[lane] = wt;
      }
    }
  }

  if (warp == kNW) {
    // ---------------------------------------------------------------- producer
    const uint64_t pol = policy_evict_first();
    auto issue = [&](int q) {                               // stage q into its ring slot
      const int s = q % kRing;
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
    };
    const int first = cnt < kRing ? cnt : kRing;            // the ring starts empty
    if (lane == 0)
      for (int q = 0; q < first; ++q) issue(q);
    // With those in flight, the global multipliers of the k slots (one lane per slot).
    if (lane < k) {
      const uint8_t* rec = p.bank + (uint64_t)s_ids[lane] * p.stride;
      float g[3];
#pragma unroll
      for (int m = 0; m < 3; ++m) g[m] = __ldg(reinterpret_cast<const float*>(rec + p.global_off[m]));
#pragma unroll
      for (int m = 0; m < 3; ++m) s_gm[m * kMaxK + lane] = global_mult(g[m], p.global_mode);
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(gm_full);
      int q = first;
      for (; q < cnt; ++q) {
        if (!mbar_wait(&empty[q % kRing], ((q / kRing) & 1) ^ 1)) break;
        issue(q);
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
    // x 2^shx enters the f16 products; the gate and up sums are multiplied back by 2^-shx.
    uint32_t xr[UG][16];
#pragma unroll
    for (int u = 0; u < UG; ++u) {
      const int un = lane + 32 * u;
      const uint4* xp = reinterpret_cast<const uint4*>(sx) + 4 * un;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 b = xp[q ^ ((un >> 1) & 3)];
        xr[u][4 * q + 0] = pack_f16x2(bf16_bits_to_f32(b.x & 0xFFFF), bf16_bits_to_f32(b.x >> 16));
        xr[u][4 * q + 1] = pack_f16x2(bf16_bits_to_f32(b.y & 0xFFFF), bf16_bits_to_f32(b.y >> 16));
        xr[u][4 * q + 2] = pack_f16x2(bf16_bits_to_f32(b.z & 0xFFFF), bf16_bits_to_f32(b.z >> 16));
        xr[u][4 * q + 3] = pack_f16x2(bf16_bits_to_f32(b.w & 0xFFFF), bf16_bits_to_f32(b.w >> 16));
      }
    }
    int q = 0;
    bool have_gm = false;
    for (; q < cnt1 && ok; ++q) {
      const int s = q % kRing;
      const int u0 = lo1 + q, j = u0 / (I / kNW), r = (u0 - j * (I / kNW)) * kNW + warp;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (q / kRing) & 1))) {
        ok = false;
        break;
      }
      const uint32_t st = sbase + s * kStage;
      const uint32_t cg = st + warp * (H / 2), cu = st + kCodes1 + warp * (H / 2);
      const uint32_t sg = st + 2 * kCodes1 + warp * (H / 16), su = sg + kScales1;
      float accG = 0.0f, accU = 0.0f;
#pragma unroll
      for (int u = 0; u < UG; ++u) {
        const int un = lane + 32 * u;
        unit_dot_acc(lds128(cg + un * 16), lds16(sg + un * 2), xr[u], accG);
      }
#pragma unroll
      for (int u = 0; u < UG; ++u) {
        const int un = lane + 32 * u;
        unit_dot_acc(lds128(cu + un * 16), lds16(su + un * 2), xr[u], accU);
      }
      fence_proxy_async_smem();            // the reads above come before the slot's next TMA
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        accG += __shfl_xor_sync(0xFFFFFFFFu, accG, off);
        accU += __shfl_xor_sync(0xFFFFFFFFu, accU, off);
      }
      if (!have_gm) {
        have_gm = true;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(gm_full, 0))) {
          ok = false;
          break;
        }
      }
      if (lane == 0) {
        const float xun = exp2_int(-shx);
        p.h[(size_t)j * I + r] = silu_mul(accG * xun * s_gm[j], accU * xun * s_gm[kMaxK + j]);
      }
    }
    // Publish this CTA's gate/up stages per slot, then wait for the slots of its down rows.
    named_bar_sync(1, 32 * kNW);
    if (threadIdx.x == 0) {
      __threadfence();
      for (int u = lo1; u < hi1;) {
        const int j = u / (I / kNW), uend = min(hi1, (j + 1) * (I / kNW));
        atomicAdd(&slot_done[j], (unsigned)(uend - u));
        u = uend;
      }
      bool good = ok;
      if (hi2 > lo2)
        for (int j = lo2 / (H / kRows2); good && j <= (hi2 - 1) / (H / kRows2); ++j)
          good = wait_count(&slot_done[j], I / kNW);
      *s_ok = good ? 1 : 0;
    }
    named_bar_sync(1, 32 * kNW);
    ok = ok && *s_ok;
    // h of the (at most two) slots of this CTA's down rows into shared memory, once per CTA
    // rather than once per warp: every CTA reads the same few KB, so per-warp loads would
    // pile onto the same L2 lines.
    const int jlo = lo2 / (H / kRows2);
    int sh0 = 0, sh1 = 0;                                   // prescale shifts of h, slots jlo, jlo + 1
    if (ok && hi2 > lo2) {
      // All of a thread's loads are issued before any store, so their latencies overlap.
      constexpr int kPer = (2 * I / 4 + 32 * kNW - 1) / (32 * kNW);
      const int n4 = ((hi2 - 1) / (H / kRows2) - jlo + 1) * I / 4;
      const float4* src = reinterpret_cast<const float4*>(p.h + (size_t)jlo * I);
      float4 v[kPer];
#pragma unroll
      for (int t = 0; t < kPer; ++t) {
        const int i = (int)threadIdx.x + t * 32 * kNW;
        if (i < n4) v[t] = __ldcg(src + i);
      }
      // h enters the f16 products as h 2^sh per slot (sh from the slot's largest magnitude,
      // collected across the consumer warps first); the down sums are multiplied back by 2^-sh.
      uint32_t m0 = 0, m1 = 0;
#pragma unroll
      for (int t = 0; t < kPer; ++t) {
        const int i = (int)threadIdx.x + t * 32 * kNW;
        if (i < n4) {
          const uint32_t a = max(max(f32_abs_bits(v[t].x), f32_abs_bits(v[t].y)),
                                 max(f32_abs_bits(v[t].z), f32_abs_bits(v[t].w)));
          if (i < I / 4)
            m0 = max(m0, a);
          else
            m1 = max(m1, a);
        }
      }
      m0 = __reduce_max_sync(0xFFFFFFFFu, m0);
      m1 = __reduce_max_sync(0xFFFFFFFFu, m1);
      if (lane == 0) {
        s_amax[16 + 2 * warp] = m0;
        s_amax[16 + 2 * warp + 1] = m1;
      }
      named_bar_sync(1, 32 * kNW);
      m0 = m1 = 0;
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        m0 = max(m0, s_amax[16 + 2 * w]);
        m1 = max(m1, s_amax[16 + 2 * w + 1]);
      }
      sh0 = prescale_shift_f32(m0);
      sh1 = prescale_shift_f32(m1);
      const float f0 = exp2_int(sh0), f1 = exp2_int(sh1);
      // Chunk c of unit u (32 floats) of a slot is stored at chunk c ^ (u & 7) of the unit
      // (bank spread for the per-lane reads below).
#pragma unroll
      for (int t = 0; t < kPer; ++t) {
        const int i = (int)threadIdx.x + t * 32 * kNW;
        if (i < n4) {
          const int sl = i / (I / 4), w = i - sl * (I / 4), u = w >> 3, c = w & 7;
          const float f = sl ? f1 : f0;
          reinterpret_cast<float4*>(sh)[sl * (I / 4) + 8 * u + (c ^ (u & 7))] =
              make_float4(v[t].x * f, v[t].y * f, v[t].z * f, v[t].w * f);
        }
      }
    }
    named_bar_sync(1, 32 * kNW);

    // Phase 2: down.  Warp w takes rows 4w .. 4w+3 of the stage as two pairs; in a pair, lane l
    // takes units cu = l + 32 u (u < UD) of the two rows laid end to end: row cu / kUnits2, K
    // unit cu % kUnits2, with h at those K positions in registers (reloaded when the slot
    // changes).
    uint32_t hr[UD][16];
    int hj = -1;
    int shh = 0;                                            // prescale shift of the h in hr
    for (; q < cnt && ok; ++q) {
      const int s = q % kRing;
      const int u0 = lo2 + (q - cnt1), j = u0 / (H / kRows2), r0 = (u0 - j * (H / kRows2)) * kRows2 + 4 * warp;
      if (!have_gm) {
        have_gm = true;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(gm_full, 0))) {
          ok = false;
          break;
        }
      }
      if (j != hj) {
        hj = j;
        const float* hp = sh + (size_t)(j - jlo) * I;
        shh = j == jlo ? sh0 : sh1;
#pragma unroll
        for (int u = 0; u < UD; ++u) {
          const int ku = (lane + 32 * u) % kUnits2;
          const float4* src = reinterpret_cast<const float4*>(hp + 32 * ku);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 a = src[q4 ^ (ku & 7)];
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
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const uint32_t cd = st + (4 * warp + 2 * pr) * (I / 2), sd = st + kCodes2 + (4 * warp + 2 * pr) * (I / 16);
#pragma unroll
        for (int u = 0; u < UD; ++u) {
          const int cu = lane + 32 * u;                     // unit within the pair of rows
          const uint4 cw = lds128(cd + cu * 16);
          const uint32_t sw = lds16(sd + cu * 2);
          if (32 * u + 31 < kUnits2) {                      // every lane in the first row
            unit_dot_acc(cw, sw, hr[u], acc[2 * pr]);
          } else if (32 * u >= kUnits2) {                   // every lane in the second row
            unit_dot_acc(cw, sw, hr[u], acc[2 * pr + 1]);
          } else {
            const float part = unit_dot(cw, sw, hr[u]);
            if (cu < kUnits2)
              acc[2 * pr] += part;
            else
              acc[2 * pr + 1] += part;
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += __shfl_xor_sync(0xFFFFFFFFu, acc[i], off);
      if (lane < 4) {
        const float v = lane == 0 ? acc[0] : lane == 1 ? acc[1] : lane == 2 ? acc[2] : acc[3];
        p.y[(size_t)j * H + r0 + lane] = v * exp2_int(-shh) * s_gm[2 * kMaxK + j];
      }
    }
    // Combine.  Block b = rows 32b .. 32b+31: one down stage per slot, so k contributions.
    // One consumer thread per down stage publishes it (fence, then the block's counter), so the
    // counter round trips overlap instead of queueing behind one thread; a thread that adds a
    // block's last contribution records the block (s_ok counts them), and the CTA combines the
    // blocks it recorded.
    int* s_last = s_ok + 1;                                 // blocks this CTA combines
    if (threadIdx.x == 0) *s_ok = 0;                        // every thread read it long ago
    named_bar_sync(1, 32 * kNW);
    if (ok)
      for (int u = lo2 + (int)threadIdx.x; u < hi2; u += 32 * kNW) {
        const int b = u % (H / kRows2);
        __threadfence();
        if (atomicAdd(&block_done[b], 1u) == (unsigned)k - 1u) {
          __threadfence();
          s_last[atomicAdd(s_ok, 1)] = b;
        }
      }
    named_bar_sync(1, 32 * kNW);
    // The last CTA through here clears the counter set for the call that uses it next.
    // (warp 0: one lane takes the exit count, the whole warp clears the set).
    if (warp == 0) {
      unsigned* exit_count = p.bar + kMaxK + kMaxBlocks;
      unsigned last = 0;
      if (lane == 0) {
        __threadfence();
        last = atomicAdd(exit_count, 1u) == gridDim.x - 1 ? 1u : 0u;
        __threadfence();                    // every other CTA's counter updates come before
      }
      __syncwarp();
      if (__shfl_sync(0xFFFFFFFFu, last, 0)) {
        __threadfence();
        for (int i = lane; i < kMaxK; i += 32) slot_done[i] = 0;
        for (int i = lane; i < H / 32; i += 32) block_done[i] = 0;
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          *exit_count = 0;
          __threadfence();
        }
      }
    }
    // Warps 1.. combine while warp 0 takes the exit count (and, in the last CTA, clears the set).
    for (int i = warp - 1; warp > 0 && i < *s_ok; i += kNW - 1) {
      const int c = 32 * s_last[i] + lane;
      float a = 0.0f;
      for (int jj = 0; jj < k; ++jj) a = fmaf(s_w[jj], __ldcg(p.y + (size_t)jj * H + c), a);
      const uint32_t o = f32_to_bf16_bits(a);
      p.out[c] = (uint16_t)o;
      if (p.x_next != nullptr) p.x_next[c] = (uint16_t)f32_to_bf16_bits(bf16_bits_to_f32(__ldg(p.x + c)) + bf16_bits_to_f32(o));
    }
  }
}

template <int UG, int UD>
int launch_d1(const D1Params& p, int num_sms, cudaStream_t s) {
  constexpr int H = UG * 1024, I = UD * 512;
  constexpr int kStage1 = 2 * (kNW * H / 2 + kNW * H / 16);
  constexpr int kStage2 = 4 * kNW * I / 2 + 4 * kNW * I / 16;
  constexpr int kStage = kStage1 > kStage2 ? kStage1 : kStage2;
  const int smem =
      kRing * kStage + H * 2 + 2 * I * 4 + (2 * kRing + 1) * 8 + kMaxRankE * 8 + 5 * kMaxK * 4 + 4 + 4 * kMaxLast +
      4 * 32;
  auto kern = decode1_kernel<UG, UD>;
  cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(kern), smem);
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

bool decode1_supported(int H, int I, int k, int E, int num_sms) {
  if (E > kMaxRankE || k > kMaxK || H / 32 > kMaxBlocks || num_sms < 1 || (k * (H / 32) + num_sms - 1) / num_sms > kMaxLast) return false;
  return (H == 5120 && I == 2560) || (H == 1024 && I == 512) || (H == 2048 && I == 1024) ||
         (H == 4096 && I == 1536);
}

// Device address of this device's counter sets (the current device), resolved once.
static unsigned* d1_counter_base(int dev) {
  static std::mutex mu;
  static std::vector<unsigned*> base;
  std::lock_guard<std::mutex> lk(mu);
  if ((int)base.size() <= dev) base.resize(dev + 1, nullptr);
  if (!base[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_d1_counters) != cudaSuccess) return nullptr;
    base[dev] = static_cast<unsigned*>(ptr);
  }
  return base[dev];
}

static std::atomic<unsigned> g_d1_next_set{0};

int decode1_reset_pool() {
  void* ptr = nullptr;
  cudaError_t err = cudaGetSymbolAddress(&ptr, g_d1_counters);
  if (err == cudaSuccess) err = cudaMemset(ptr, 0, sizeof(g_d1_counters));
  return err == cudaSuccess ? 0 : -(int)err;
}

int launch_decode1(const BankView& bank, const float* logits, int k, const uint16_t* x, uint16_t* out,
                   uint16_t* x_next, float* h, float* y, int32_t* ids, float* w, int dev, int num_sms,
                   cudaStream_t s) {
  unsigned* sets = d1_counter_base(dev);
  if (!sets) return -(int)cudaErrorInvalidSymbol;
  unsigned* bar = sets + (size_t)(g_d1_next_set.fetch_add(1u) % kCounterSets) * kCounterWords;
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
  if (bank.H == 5120 && bank.I == 2560) return launch_d1<5, 5>(p, num_sms, s);
  if (bank.H == 1024 && bank.I == 512) return launch_d1<1, 1>(p, num_sms, s);
  if (bank.H == 2048 && bank.I == 1024) return launch_d1<2, 2>(p, num_sms, s);
  if (bank.H == 4096 && bank.I == 1536) return launch_d1<4, 3>(p, num_sms, s);
  return -(int)cudaErrorInvalidValue;
}

}  // namespace moe
