// Prefill path: grouped NVFP4 expert GEMM on the 5th-generation tensor cores (tcgen05, TMEM).
//
// Work item (tile) = one group of up to 256 routed rows of one expert x 2 MMA M-tiles of 128
// weight rows: for gate/up the gate rows r0 .. r0+127 and the same up rows (SwiGLU is applied
// in the epilogue), for down 256 consecutive rows of Wd.  The two M-tiles share every tile of
// activations, halving activation traffic per FLOP.
//
// Per CTA (one per SM, persistent over tiles), warp-specialised, all hand-offs on mbarriers:
//   warp 6 (one thread): 3-D TMA of the raw NVFP4 tiles -- codes 128 rows x 32 B per M-tile and
//       stage, E4M3 scales 128 rows x 16 B per M-tile every 4 stages -- straight out of the
//       bank (dims: bytes of a row, rows, expert), so weight bytes cross the L1 once, in bulk;
//   warps 0-3 (one thread per weight row of each M-tile): read their row's codes and scales
//       from shared memory, convert E2M1 with cvt, multiply by the block scale (exact) and store
//       the BF16 row chunk into a 128-byte-swizzled K-major operand stage;
//   warp 4 (one thread): 2-D TMA of the group's BF16 activation rows (expert order) into
//       swizzled stages;
//   warp 5 (one thread): tcgen05.mma kind::f16 with BF16 A and B (M = 128, N = rows of the
//       group rounded up to 16, K = 16) into two f32 accumulators in tensor memory;
//       tcgen05.commit frees a stage.
// After a tile's last K stage warps 0-3 read the accumulators back with tcgen05.ld and apply
// the global scale (and SwiGLU for gate/up, whose result h is stored as BF16).
//
// Tiles are handed out dynamically: the weight-TMA thread takes the next tile index from a
// global counter and passes it to the other roles through a small queue in shared memory.
// The router lists the groups with a full 256 rows first, so the large tiles go out first and
// the small remainder tiles fill in at the end.
//
// Weight layout: page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit
// residents", section "What this pack holds"; SwiGLU in FP32: page "Beam-1.0-501B-A23B VQ
// GGUF", section "What stays native".  The pages' prefill kernels ("decode-once prefill MoE
// GEMM" on sm_120) dequantize each weight tile once for all of a group's tokens; so does this
// one, on sm_100a tensor cores.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kBM = 128;                       // rows per MMA M-tile
constexpr int kKC = 64;                        // K per stage: one 128-byte swizzle row of bf16
constexpr int kStages = 3;                     // operand stages (A and B, bf16)
constexpr int kWStages = 3;                    // raw code stages
constexpr int kSStages = 2;                    // raw scale stages (4 operand stages each)
constexpr int kPrefetch = 8;                   // stages of raw codes prefetched into L2 ahead of their load
constexpr int kMaxN = 256;
constexpr int kBoxRows = 64;                   // activation rows per TMA box
constexpr int kThreads = 32 * 7;
constexpr int kABytes = kBM * kKC * 2;         // 16 KB: one M-tile of one stage
constexpr int kBBytes = kMaxN * kKC * 2;       // 32 KB: activations of one stage
constexpr int kWBytes = kBM * kKC / 2;         // 4 KB: codes of one M-tile of one stage
constexpr int kSBytes = kBM * 16;              // 2 KB: scales of one M-tile, 4 stages
constexpr int kTmemCols = 512;                 // two 256-column f32 accumulators
constexpr int kTQ = 4;                         // tile queue entries
constexpr int kTQConsumers = 4 + 1 + 1;        // producer warps, activation TMA, MMA
constexpr int kOffB = kStages * 2 * kABytes;
constexpr int kOffW = kOffB + kStages * kBBytes;
constexpr int kOffS = kOffW + kWStages * 2 * kWBytes;
constexpr int kOffBar = kOffS + kSStages * 2 * kSBytes;
constexpr int kSmemBytes = kOffBar + 512 /*barriers, tile queue*/ + 1024 /*alignment*/;
static_assert(kSmemBytes <= 232448, "shared memory per block");

struct PrefillParams {
  const uint8_t* bank;
  int f16;                 // 1: F16 operands (gate/up: activations prescaled per row, colscale undoes it)
  const float* colscale;   // f16: per activation row the factor 2^-s of its prescale
  uint64_t stride;
  uint64_t global_off[2];  // global scale of the matrix of M-tile 0 / M-tile 1
  int global_mode;
  int K;                   // inputs per weight row
  int tiles_per_group;     // output-row tiles per group
  int gateup;              // 1: M-tile 0 = gate rows, M-tile 1 = same up rows; 0: 256 consecutive rows
  const int4* groups;      // (expert, first permuted row, rows <= 256, 0)
  const int32_t* ngroups;
  unsigned* tile_ctr;      // tiles handed out so far (zero at launch)
  void* out;               // gate/up: h bf16 [R, out_stride]; down: y f32 [R, out_stride]
  int out_stride;
};

struct Maps {
  CUtensorMap x;           // activations [R, K] bf16
  CUtensorMap codes[2];    // codes of the M-tile 0 / 1 matrix: [E][rows][K/2] bytes
  CUtensorMap scales[2];   // scales: [E][rows][K/16] bytes
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// One thread's share of one stage: 64 codes and 4 scale bytes of each of its two rows.
struct StageFrag {
  uint4 c[2][2];
  uint32_t s[2];
};

// Maps a CTA-local tile number to (group, output-row tile).
struct TileCursor {
  int tiles_per_group;
  __device__ __forceinline__ void at(int tt, int& g, int& m) const {
    g = tt / tiles_per_group;
    m = tt - g * tiles_per_group;
  }
};

__device__ __forceinline__ int row0_of(const PrefillParams& p, int m, int mt) {
  return p.gateup ? m * kBM : m * 2 * kBM + mt * kBM;
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ Maps maps, const PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;                                   // [stage][m-tile] 16 KB bf16, 128B-swizzled
  uint8_t* sB = smem + kOffB;                           // [stage] 32 KB bf16, 128B-swizzled
  uint8_t* sW = smem + kOffW;                           // [stage][m-tile] 128 rows x 32 B
  uint8_t* sS = smem + kOffS;                           // [stage][m-tile] 128 rows x 16 B
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* a_full = bars;                              // [kStages] producers -> MMA
  uint64_t* b_full = a_full + kStages;                  // [kStages] TMA -> MMA
  uint64_t* empty = b_full + kStages;                   // [kStages] MMA commit -> producers, TMA
  uint64_t* w_full = empty + kStages;                   // [kWStages] TMA -> producers
  uint64_t* w_empty = w_full + kWStages;                // [kWStages] producers -> TMA
  uint64_t* s_full = w_empty + kWStages;                // [kSStages]
  uint64_t* s_empty = s_full + kSStages;                // [kSStages]
  uint64_t* d_full = s_empty + kSStages;                // MMA commit -> epilogue
  uint64_t* d_empty = d_full + 1;                       // epilogue -> MMA
  uint64_t* tq_full = d_empty + 1;                      // [kTQ] scheduler -> roles
  uint64_t* tq_empty = tq_full + kTQ;                   // [kTQ] roles -> scheduler
  int* s_tq = reinterpret_cast<int*>(tq_empty + kTQ);   // [kTQ] tile index, -1 = no more
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_tq + kTQ);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = *p.ngroups * p.tiles_per_group;
  const int nst = p.K / kKC;                            // stages per tile (a multiple of 4)
  const TileCursor cur{p.tiles_per_group};
  // Takes tile number i of this CTA from the queue (every role sees the same sequence).
  auto pop_tile = [&](int i, int& tt) -> bool {
    const int slot = i % kTQ;
    if (!mbar_wait(&tq_full[slot], (i / kTQ) & 1)) return false;
    tt = ((volatile int*)s_tq)[slot];
    return true;
  };

  if (threadIdx.x == 0) {
    // Producer-side barriers count one arrival per producer warp (lane 0 after __syncwarp):
    // 128 arrivals on one word would serialise in the shared-memory pipe.
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&a_full[s], 4);
      mbar_init(&b_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], 4);
    }
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 4);
    }
    mbar_init(d_full, 1);
    mbar_init(d_empty, 4);
    for (int s = 0; s < kTQ; ++s) {
      mbar_init(&tq_full[s], 1);
      mbar_init(&tq_empty[s], kTQConsumers);
    }
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------------------ dequant + epilogue
    const int t = threadIdx.x;                      // weight row within each M-tile
    const uint32_t w_base = smem_addr(sW), s_base = smem_addr(sS);
    // The two 16-byte halves of a 32-byte code row are read in an order that alternates every
    // four rows, so a warp's 128-bit shared loads cover all 32 banks without conflicts.
    const uint32_t h0 = ((t >> 2) & 1) * 16, h1 = h0 ^ 16;
    auto fetch = [&](int q, StageFrag& f) {        // raw stage q: shared -> registers
      const int c = q % nst;
      const int ws = q % kWStages, ss = (q >> 2) % kSStages;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t row = w_base + (ws * 2 + mt) * kWBytes + t * 32;
        const uint4 u = ld_shared_v4(row + h0), v = ld_shared_v4(row + h1);
        f.c[mt][0] = h0 ? v : u;
        f.c[mt][1] = h0 ? u : v;
        f.s[mt] = ld_shared_u32(s_base + (ss * 2 + mt) * kSBytes + t * 16 + (c & 3) * 4);
      }
    };
    auto store = [&](int s, const StageFrag& f) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t base = smem_addr(sA + (s * 2 + mt) * kABytes) + t * 128;
        const uint32_t h01 = e4m3x2_to_f16x2((uint16_t)(f.s[mt] & 0xFFFF));
        const uint32_t h23 = e4m3x2_to_f16x2((uint16_t)(f.s[mt] >> 16));
        const uint32_t sc[4] = {bcast_half(h01, false), bcast_half(h01, true), bcast_half(h23, false),
                                bcast_half(h23, true)};
        const uint32_t w[8] = {f.c[mt][0].x, f.c[mt][0].y, f.c[mt][0].z, f.c[mt][0].w,
                               f.c[mt][1].x, f.c[mt][1].y, f.c[mt][1].z, f.c[mt][1].w};
        if (p.f16) {
          // F16 operand: E2M1 -> f16 (cvt) times the block scale in f16 -- two instructions per pair
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t e[4];
            e2m1x8_to_f16x8(w[j], e);
            st_shared_v4(base + ((j ^ (t & 7)) << 4), hmul2(e[0], sc[j >> 1]), hmul2(e[1], sc[j >> 1]),
                         hmul2(e[2], sc[j >> 1]), hmul2(e[3], sc[j >> 1]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {                // word j = K 8j .. 8j+7 = 16-byte chunk j
            uint32_t e[4];
            e2m1x8_scaled_to_bf16x8(w[j], sc[j >> 1], e);
            st_shared_v4(base + ((j ^ (t & 7)) << 4), e[0], e[1], e[2], e[3]);
          }
        }
      }
    };
    auto epilogue = [&](int tt, int i) {
      int g, m;
      cur.at(tt, g, m);
      const int4 grp = __ldg(&p.groups[g]);
      const uint8_t* rec = p.bank + (uint64_t)grp.x * p.stride;
      const float gm0 = global_mult(__ldg(reinterpret_cast<const float*>(rec + p.global_off[0])), p.global_mode);
      const float gm1 = global_mult(__ldg(reinterpret_cast<const float*>(rec + p.global_off[1])), p.global_mode);
      if (!__all_sync(0xffffffffu, mbar_wait(d_full, i & 1))) return;   // tcgen05.ld needs the whole warp
      tc_fence_after();
      const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
      for (int n0 = 0; n0 < grp.z; n0 += 32) {
        uint32_t d0[32], d1[32];
        tmem_ld32(lane_base + n0, d0);
        tmem_ld32(lane_base + 256 + n0, d1);
        tmem_wait_ld();
        const int nn = min(32, grp.z - n0);
        if (p.gateup) {
          uint16_t* o = static_cast<uint16_t*>(p.out) + (size_t)(grp.y + n0) * p.out_stride + m * kBM + t;
          const float* cs = p.colscale + grp.y + n0;     // (f16 operands: undo each row's prescale)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nn) {
              const float c = p.f16 ? __ldg(cs + j) : 1.0f;
              o[(size_t)j * p.out_stride] = (uint16_t)f32_to_bf16_bits(
                  silu_mul_fast(__uint_as_float(d0[j]) * c * gm0, __uint_as_float(d1[j]) * c * gm1));
            }
        } else {
          float* o = static_cast<float*>(p.out) + (size_t)(grp.y + n0) * p.out_stride + m * 2 * kBM + t;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j < nn) {
              o[(size_t)j * p.out_stride] = __uint_as_float(d0[j]) * gm0;
              o[(size_t)j * p.out_stride + kBM] = __uint_as_float(d1[j]) * gm1;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(d_empty);
    };

    bool ok = true;
    const int first = nst < kStages ? nst : kStages;   // stages of a tile stored before the previous epilogue
    int q = 0, i = 0, prev = -1;
    for (; ok; ++i) {
      int tt = -1;
      if (!__all_sync(0xffffffffu, pop_tile(i, tt))) {
        ok = false;
        break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&tq_empty[i % kTQ]);
      if (tt < 0) break;
      for (int c = 0; c < nst; ++c, ++q) {
        const int ws = q % kWStages, ss = (q >> 2) % kSStages;
        const bool got = mbar_wait(&w_full[ws], (q / kWStages) & 1) &&
                         ((c & 3) != 0 || mbar_wait(&s_full[ss], ((q >> 2) / kSStages) & 1));
        if (!__all_sync(0xffffffffu, got)) {     // warp-uniform: the warp arrives as one below
          ok = false;
          break;
        }
        StageFrag f;
        fetch(q, f);
        const int s = q % kStages;
        if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ((q / kStages) & 1) ^ 1))) {
          ok = false;
          break;
        }
        store(s, f);
        fence_proxy_async_smem();
        __syncwarp();
        // The raw slots go back to the TMA only after every lane's proxy fence above: a TMA
        // write (async proxy) into a slot that was read with generic loads must be ordered
        // after those reads, or it can overtake them.
        if (lane == 0) {
          mbar_arrive(&a_full[s]);
          mbar_arrive(&w_empty[ws]);
          if ((c & 3) == 3) mbar_arrive(&s_empty[ss]);
        }
        if (i > 0 && c == first - 1) epilogue(prev, i - 1);
      }
      prev = tt;
    }
    if (ok && i > 0) epilogue(prev, i - 1);
  } else if (warp == 4) {
    // ------------------------------------------------------------ activation TMA
    if (lane == 0) {
      int q = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        int tt = -1;
        if (!pop_tile(i, tt)) break;
        mbar_arrive(&tq_empty[i % kTQ]);
        if (tt < 0) break;
        const int4 grp = __ldg(&p.groups[tt / p.tiles_per_group]);
        const int nbox = (grp.z + kBoxRows - 1) / kBoxRows;
        for (int c = 0; c < nst; ++c, ++q) {
          const int s = q % kStages;
          if (!mbar_wait(&empty[s], ((q / kStages) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&b_full[s], nbox * kBoxRows * kKC * 2);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(sB + s * kBBytes + b * kBoxRows * kKC * 2, &maps.x, c * kKC, grp.y + b * kBoxRows,
                        &b_full[s]);
        }
      }
      for (int j = max(0, q - kStages); j < q; ++j) mbar_wait(&b_full[j % kStages], (j / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------------ weight TMA
    if (lane == 0) {
      bool ok = true;
      int q = 0, qs = 0;
      for (int i = 0; ok; ++i) {
        // Next tile for every role of this CTA.
        const int slot = i % kTQ;
        if (!mbar_wait(&tq_empty[slot], ((i / kTQ) & 1) ^ 1)) break;
        int tt = (int)atomicAdd(p.tile_ctr, 1u);
        if (tt >= ntiles) tt = -1;
        ((volatile int*)s_tq)[slot] = tt;
        mbar_arrive(&tq_full[slot]);
        if (tt < 0) break;
        int g, m;
        cur.at(tt, g, m);
        const int e = __ldg(&p.groups[g].x);
        auto prefetch_stage = [&](int m_, int e_, int cs) {
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            tma_prefetch_3d(&maps.codes[mt], cs * (kKC / 2), row0_of(p, m_, mt), e_);
            if ((cs & 3) == 0) tma_prefetch_3d(&maps.scales[mt], (cs >> 2) * 16, row0_of(p, m_, mt), e_);
          }
        };
        for (int c = 0; c < nst && ok; ++c, ++q) {
          if ((c & 3) == 0) {                       // scales of stages c .. c+3
            const int ss = qs % kSStages;
            if (!mbar_wait(&s_empty[ss], ((qs / kSStages) & 1) ^ 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&s_full[ss], 2 * kSBytes);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
              tma_load_3d(sS + (ss * 2 + mt) * kSBytes, &maps.scales[mt], (c >> 2) * 16, row0_of(p, m, mt), e,
                          &s_full[ss]);
            ++qs;
          }
          // The raw codes come from HBM in 32-byte rows: prefetch them into L2 kPrefetch stages
          // ahead of their load (the ring is only kWStages deep).
          if (c == 0)
            for (int cp = 1; cp < kPrefetch && cp < nst; ++cp) prefetch_stage(m, e, cp);
          if (c + kPrefetch < nst) prefetch_stage(m, e, c + kPrefetch);
          const int ws = q % kWStages;
          if (!mbar_wait(&w_empty[ws], ((q / kWStages) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&w_full[ws], 2 * kWBytes);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
            tma_load_3d(sW + (ws * 2 + mt) * kWBytes, &maps.codes[mt], c * (kKC / 2), row0_of(p, m, mt), e,
                        &w_full[ws]);
        }
      }
      // Leave no copy in flight (only an error path gets here with copies outstanding).
      for (int j = max(0, q - kWStages); j < q; ++j) mbar_wait(&w_full[j % kWStages], (j / kWStages) & 1);
      for (int j = max(0, qs - kSStages); j < qs; ++j) mbar_wait(&s_full[j % kSStages], (j / kSStages) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int q = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        int tt = -1;
        if (!pop_tile(i, tt)) break;
        mbar_arrive(&tq_empty[i % kTQ]);
        if (tt < 0) break;
        const int4 grp = __ldg(&p.groups[tt / p.tiles_per_group]);
        const int N = (grp.z + 15) & ~15;
        const uint32_t idesc = p.f16 ? idesc_f16(kBM, N) : idesc_bf16(kBM, N);
        if (i > 0 && !mbar_wait(d_empty, (i - 1) & 1)) break;
        tc_fence_after();
        for (int c = 0; c < nst; ++c, ++q) {
          const int s = q % kStages;
          const uint32_t ph = (q / kStages) & 1;
          if (!mbar_wait(&a_full[s], ph) || !mbar_wait(&b_full[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b0 = smem_addr(sB + s * kBBytes);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const uint32_t a0 = smem_addr(sA + (s * 2 + mt) * kABytes);
#pragma unroll
            for (int k = 0; k < kKC / 16; ++k)
              tc_mma_f16(tmem + mt * 256, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc,
                         (c | k) != 0);
          }
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(d_full);
      }
      // Do not free tensor memory while MMAs may still run (matters only on the error path).
      if (q > 0) mbar_wait(&empty[(q - 1) % kStages], ((q - 1) / kStages) & 1);
    }
    __syncwarp();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Gathers the routed rows of x (bf16 [T, H]) in expert order into xp as f16 [R, H], each row
// times the exact power of two 2^s that puts its largest magnitude in [2^9, 2^10) (the decode
// kernels' prescale; every BF16 value down to 2^-23 of the row's maximum is exact in f16), and
// writes colscale[p] = 2^-s.  One CTA of 128 threads per token: its row is read and converted
// once (the maximum first), then stored at the place inv[t*k + j] of each of its k routed rows.
constexpr int kGatherThreads = 128;
constexpr int kGatherPer = 8;          // 16-byte chunks per thread (H <= 8192)
__global__ void __launch_bounds__(kGatherThreads) gather_f16_kernel(const uint16_t* __restrict__ x,
                                                                   const int32_t* __restrict__ inv, int k, int H,
                                                                   uint16_t* __restrict__ xp,
                                                                   float* __restrict__ colscale) {
  const int64_t t = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  const int n8 = H / 8;
  uint4 v[kGatherPer];
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < kGatherPer; ++i) {
    const int c = (int)threadIdx.x + i * kGatherThreads;
    if (c < n8) {
      v[i] = __ldg(src + c);
      m = max(m, bf16x8_abs_max_bits(v[i]));
    }
  }
  __shared__ uint32_t s_m[kGatherThreads / 32];
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if ((threadIdx.x & 31) == 0) s_m[threadIdx.x >> 5] = m;
  __syncthreads();
  m = max(max(s_m[0], s_m[1]), max(s_m[2], s_m[3]));
  const int sh = prescale_shift_bf16(m);
  const float f = exp2_int(sh);
#pragma unroll
  for (int i = 0; i < kGatherPer; ++i) {
    const int c = (int)threadIdx.x + i * kGatherThreads;
    if (c < n8) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) o[j] = pack_f16x2(bf16_bits_to_f32(w[j] & 0xFFFFu) * f, bf16_bits_to_f32(w[j] >> 16) * f);
      v[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  // the token's row goes to the place of each of its k routed rows
  for (int j = 0; j < k; ++j) {
    const int64_t p = inv[t * k + j];
    uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)p * H);
#pragma unroll
    for (int i = 0; i < kGatherPer; ++i) {
      const int c = (int)threadIdx.x + i * kGatherThreads;
      if (c < n8) dst[c] = v[i];
    }
    if (threadIdx.x == 0) colscale[p] = exp2_int(-sh);
  }
}

// Gathers the routed rows of x (bf16 [T, H]) in expert order into xp (bf16 [R, H]).
__global__ void gather_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, int k, int64_t R,
                              int H, uint16_t* __restrict__ xp) {
  const int per = H / 8;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= R * per) return;
  const int64_t r = i / per;
  const int c = (int)(i - r * per) * 8;
  const int t = perm[r] / k;
  *reinterpret_cast<uint4*>(xp + r * H + c) = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H + c));
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// Tensor map over a row-major 16-bit matrix [rows, cols]: boxes of 64 columns x 64 rows, 128B
// swizzle (the copy moves bytes; bf16 and f16 rows use the same map).
int make_rows_map(CUtensorMap* map, const void* base, int64_t rows, int cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -(int)cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {kKC, kBoxRows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -(int)cudaErrorInvalidValue;
}

// Tensor map over one byte matrix of every record: [E][rows][row_bytes] with the record stride
// between experts; boxes of box_bytes x 128 rows x 1 expert, no swizzle.
int make_bank_map(CUtensorMap* map, const BankView& bank, uint64_t off, int rows, int row_bytes, int box_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -(int)cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)row_bytes, (cuuint64_t)rows, (cuuint64_t)bank.E};
  const cuuint64_t strides[2] = {(cuuint64_t)row_bytes, (cuuint64_t)bank.stride};
  const cuuint32_t box[3] = {(cuuint32_t)box_bytes, (cuuint32_t)kBM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(bank.base + off), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -(int)cudaErrorInvalidValue;
}

int launch_prefill(const PrefillParams& p, const Maps& maps, int num_sms, cudaStream_t s) {
  cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(prefill_kernel), kSmemBytes);
  if (err != cudaSuccess) return -(int)err;
  prefill_kernel<<<num_sms, kThreads, kSmemBytes, s>>>(maps, p);
  err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

// Weight maps of the two M-tile matrices (proj0, proj1) whose rows hold K inputs.
int make_weight_maps(Maps* maps, const BankView& bank, int proj0, int proj1, int rows, int K) {
  const int projs[2] = {proj0, proj1};
  for (int mt = 0; mt < 2; ++mt) {
    int rc = make_bank_map(&maps->codes[mt], bank, bank.codes_off[projs[mt]], rows, K / 2, kKC / 2);
    if (rc) return rc;
    rc = make_bank_map(&maps->scales[mt], bank, bank.scales_off[projs[mt]], rows, K / 16, 16);
    if (rc) return rc;
  }
  return 0;
}

}  // namespace

int make_tensor_map(CUtensorMap* map, int rank, const void* base, const uint64_t* dims, const uint64_t* strides,
                    const uint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -(int)cudaErrorNotSupported;
  if (rank < 1 || rank > 5) return -(int)cudaErrorInvalidValue;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void*>(base), d, st, b, e,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -(int)cudaErrorInvalidValue;
}

bool prefill_supported(int H, int I) { return H % 256 == 0 && I % 256 == 0; }

int launch_gather_f16(const uint16_t* x, const int32_t* inv, int k, int64_t T, int H, void* xp, float* colscale,
                      cudaStream_t s) {
  if (H / 8 > kGatherPer * kGatherThreads) return -(int)cudaErrorInvalidValue;
  gather_f16_kernel<<<(unsigned)T, kGatherThreads, 0, s>>>(x, inv, k, H, static_cast<uint16_t*>(xp), colscale);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

int launch_gather(const uint16_t* x, const int32_t* perm, int k, int64_t R, int H, void* xp, cudaStream_t s) {
  const int64_t n = R * (H / 8);
  gather_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(x, perm, k, R, H, static_cast<uint16_t*>(xp));
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

int launch_prefill_gateup(const BankView& bank, const void* xp, const float* colscale, int64_t R, const RouteBufs& rb,
                          void* hb, unsigned* tile_ctr, int num_sms, cudaStream_t s) {
  Maps maps;
  int rc = make_rows_map(&maps.x, xp, R, bank.H);
  if (!rc) rc = make_weight_maps(&maps, bank, 0, 1, bank.I, bank.H);
  if (rc) return rc;
  PrefillParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  p.global_off[0] = bank.global_off[0];
  p.global_off[1] = bank.global_off[1];
  p.global_mode = bank.global_mode;
  p.K = bank.H;
  p.tiles_per_group = bank.I / kBM;
  p.gateup = 1;
  p.f16 = colscale != nullptr;
  p.colscale = colscale;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.tile_ctr = tile_ctr;
  p.out = hb;
  p.out_stride = bank.I;
  return launch_prefill(p, maps, num_sms, s);
}

int launch_prefill_down(const BankView& bank, const void* hb, int64_t R, const RouteBufs& rb, float* y,
                        unsigned* tile_ctr, int num_sms, cudaStream_t s) {
  Maps maps;
  int rc = make_rows_map(&maps.x, hb, R, bank.I);
  if (!rc) rc = make_weight_maps(&maps, bank, 2, 2, bank.H, bank.I);
  if (rc) return rc;
  PrefillParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  p.global_off[0] = bank.global_off[2];
  p.global_off[1] = bank.global_off[2];
  p.global_mode = bank.global_mode;
  p.K = bank.I;
  p.tiles_per_group = bank.H / (2 * kBM);
  p.gateup = 0;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.tile_ctr = tile_ctr;
  p.out = y;
  p.out_stride = bank.H;
  return launch_prefill(p, maps, num_sms, s);
}

}  // namespace moe
