// Prefill path on CTA pairs: grouped NVFP4 expert GEMM with tcgen05.mma.cta_group::2 (M = 256
// across the two SMs of a cluster), double-buffered accumulators, the epilogue of one tile
// overlapping the MMAs of the next.
//
// Work item (tile) = one group of up to 256 routed rows of one expert (MMA N = the group's rows
// rounded up to 32) x 256 weight rows (MMA M): for gate/up the gate rows i0 .. i0+127 and the same
// up rows, for down 256 consecutive rows of Wd.  CTA r of the pair holds (and dequantizes) 128 of
// those weight rows -- gate/up: gate rows i0 + 64 r .. +63 in rows 0..63 and the same up rows in
// rows 64..127, so that SwiGLU pairs rows within one CTA -- and half of the group's activation
// rows; the pair's MMA reads both halves of both operands, and each CTA's tensor memory receives
// the products of its own 128 weight rows with all N activation rows.
//
// Per CTA (one persistent pair per two SMs, tiles assigned round-robin to the pairs over the
// router's group list, full groups first):
//   warp 9 (one thread): 3-D TMA of the raw NVFP4 codes (2 x 64 rows x 32 B per stage) and E4M3
//       scales (2 x 64 rows x 16 B every 4 stages) of the CTA's 128 weight rows;
//   warps 4-7 (one thread per weight row): E2M1 -> F16 with cvt, times the block scale (exact),
//       into a 128-byte-swizzled K-major operand stage (F16, or repacked to BF16);
//   warp 8 (one thread): 2-D TMA of the CTA's half of the group's activation rows;
//   warp 10 of CTA 0 (one thread): tcgen05.mma.cta_group::2 (M = 256, N, K = 16) into one of two
//       256-column f32 accumulators; tcgen05.commit multicast to both CTAs frees a stage in both
//       and tells both epilogues that an accumulator is complete;
//   warps 0-3: epilogue on the CTA's 128 TMEM lanes: global scale (and the activation rows'
//       prescale), SwiGLU with the up rows handed from warps 2-3 to warps 0-1 through shared
//       memory, h as BF16 (gate/up) or y as f32 (down).
// The dequantizing warps of both CTAs and both epilogues signal barriers in CTA 0 (remote
// mbarrier arrives); CTA 1's activation TMA completes its bytes on CTA 0's barrier.  Every wait is
// bounded.  No TMA multicast: each CTA loads only its own operands.
//
// Weight layout: page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit
// residents", section "What this pack holds"; SwiGLU in FP32: page "Beam-1.0-501B-A23B VQ GGUF",
// section "What stays native".  As in the pages' "decode-once prefill MoE GEMM" (sm_120), each
// weight tile is dequantized once for all of a group's tokens.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kRows = 128;                      // weight rows per CTA (M = 256 per pair)
constexpr int kKC = 64;                         // K per stage: one 128-byte swizzle row of 16-bit values
constexpr int kSt = 4;                          // operand stages
constexpr int kWSt = 4;                         // raw code stages
constexpr int kSSt = 2;                         // raw scale stages (4 operand stages each)
constexpr int kPrefetch = 8;                    // stages of raw codes prefetched into L2 ahead of their load
constexpr int kMaxN = 256;                      // activation rows per tile (both CTAs)
constexpr int kBoxRows = 64;
constexpr int kABytes = kRows * kKC * 2;        // 16 KB
constexpr int kBBytes = (kMaxN / 2) * kKC * 2;  // 16 KB: this CTA's half of the activations
constexpr int kWBytes = kRows * kKC / 2;        // 4 KB of raw codes
constexpr int kSBytes = kRows * 16;             // 2 KB of raw scales (4 stages)
constexpr int kXPitch = 33;                     // floats per row of the SwiGLU hand-off
constexpr int kOffB = kSt * kABytes;
constexpr int kOffW = kOffB + kSt * kBBytes;
constexpr int kOffS = kOffW + kWSt * kWBytes;
constexpr int kOffX = kOffS + kSSt * kSBytes;
constexpr int kOffBar = kOffX + 64 * kXPitch * 4;
constexpr int kSmem = kOffBar + 512 + 1024;
static_assert(kSmem <= 232448, "shared memory per block");
constexpr int kThreads = 32 * 11;
constexpr int kTmemCols = 512;                  // two 256-column f32 accumulators

struct P2Params {
  const uint8_t* bank;
  int f16;                 // 1: F16 operands (activations prescaled per row, colscale undoes it)
  const float* colscale;
  uint64_t stride;
  uint64_t global_off[2];  // global of rows 0..63 / 64..127 of a CTA (gate, up; or down, down)
  int global_mode;
  int K;
  int tiles_per_group;
  int gateup;
  const int4* groups;      // (expert, first routed row, rows <= 256, 0), full groups first
  const int32_t* ngroups;
  void* out;               // gate/up: h bf16 [R, out_stride]; down: y f32 [R, out_stride]
  int out_stride;
};

struct P2Maps {
  CUtensorMap x;           // activations [R, K] 16-bit as bytes [R, 2K], boxes of 128 B x 64 rows, 128B swizzle
  CUtensorMap codes[2];    // [E][rows][K/2] bytes, boxes of 32 B x 64 rows
  CUtensorMap scales[2];   // [E][rows][K/16] bytes, boxes of 16 B x 64 rows
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on a barrier that threads of the other CTA arrive on.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) {
      atomicExch(&g_status, kStatusTimeout);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// 2-D TMA load into this CTA's shared memory whose completion counts on a barrier of either CTA
// of the pair (cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const void* map, int x, int y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (both CTAs' TMEM) (+)= A (both CTAs' shared memory) * B^T, kind::f16, issued by CTA 0.
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on `bar` (same offset) in both CTAs when the MMAs issued so far complete.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_addr(bar)),
      "h"((uint16_t)3)
      : "memory");
}
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

// N of a tile: the group's rows rounded up to 32 (each CTA holds N / 2, a multiple of 16).
__device__ __forceinline__ int tile_n(int rows) { return (rows + 31) & ~31; }

__global__ void __launch_bounds__(kThreads, 1) prefill2_kernel(const __grid_constant__ P2Maps maps, const P2Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;                                   // [stage] 16 KB, 128B-swizzled
  uint8_t* sB = smem + kOffB;                           // [stage] 16 KB, 128B-swizzled
  uint8_t* sW = smem + kOffW;                           // [stage] 128 rows x 32 B raw codes
  uint8_t* sS = smem + kOffS;                           // [stage] 128 rows x 16 B raw scales
  float* sX = reinterpret_cast<float*>(smem + kOffX);   // [64][kXPitch] up values of a chunk
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* a_full = bars;                              // [kSt] CTA 0: 4 dequant warps x 2 CTAs
  uint64_t* b_full = a_full + kSt;                      // [kSt] CTA 0: expect_tx of both halves
  uint64_t* empty = b_full + kSt;                       // [kSt] both: MMA commit (multicast)
  uint64_t* w_full = empty + kSt;                       // [kWSt] local TMA -> dequant
  uint64_t* w_empty = w_full + kWSt;                    // [kWSt] local dequant -> TMA
  uint64_t* s_full = w_empty + kWSt;                    // [kSSt]
  uint64_t* s_empty = s_full + kSSt;                    // [kSSt]
  uint64_t* d_full = s_empty + kSSt;                    // [2] both: MMA commit (multicast)
  uint64_t* d_empty = d_full + 2;                       // [2] CTA 0: 4 epilogue warps x 2 CTAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_empty + 2);
  volatile int* s_epi = reinterpret_cast<volatile int*>(tmem_slot + 4);   // [2][4] epilogue wait results

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int ntiles = *p.ngroups * p.tiles_per_group;
  const int nst = p.K / kKC;                            // stages per tile (a multiple of 4)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&a_full[s], 8);
      mbar_init(&b_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kWSt; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], 4);
    }
    for (int s = 0; s < kSSt; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&d_full[b], 1);
      mbar_init(&d_empty[b], 8);
    }
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  cluster_sync();                                       // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Row r0 of the CTA's weight rows in matrix mt (0: rows 0..63, 1: rows 64..127) of tile m.
  auto row0 = [&](int m, int mt) -> int {
    return p.gateup ? m * 128 + 64 * (int)rank : m * 256 + 128 * (int)rank + 64 * mt;
  };

  if (warp < 4) {
    // ------------------------------------------------------------ epilogue
    const uint32_t d_empty0 = map_to(smem_addr(d_empty), 0);
    for (int i = 0;; ++i) {
      const int tt = pair + i * npairs;
      if (tt >= ntiles) break;
      const int g = tt / p.tiles_per_group, m = tt - g * p.tiles_per_group;
      const int4 grp = __ldg(&p.groups[g]);
      const uint8_t* rec = p.bank + (uint64_t)grp.x * p.stride;
      const float gm0 = global_mult(__ldg(reinterpret_cast<const float*>(rec + p.global_off[0])), p.global_mode);
      const float gm1 = global_mult(__ldg(reinterpret_cast<const float*>(rec + p.global_off[1])), p.global_mode);
      const int buf = i & 1;
      // The four warps share named barriers below, so they leave together: each publishes
      // whether its (bounded) wait succeeded, and all stop if one gave up.
      const bool got = __all_sync(0xffffffffu, mbar_wait(&d_full[buf], (i >> 1) & 1));   // tcgen05.ld: whole warp
      if (lane == 0) s_epi[4 * (i & 1) + warp] = got ? 1 : 0;
      named_bar_sync(2, 128);
      if (!(s_epi[4 * (i & 1)] && s_epi[4 * (i & 1) + 1] && s_epi[4 * (i & 1) + 2] && s_epi[4 * (i & 1) + 3])) break;
      tc_fence_after();
      const uint32_t lane_base = tmem + 256u * buf + ((uint32_t)(32 * warp) << 16);
      for (int n0 = 0; n0 < grp.z; n0 += 32) {
        uint32_t d[32];
        tmem_ld32(lane_base + n0, d);
        tmem_wait_ld();
        const int nn = min(32, grp.z - n0);
        if (p.gateup) {
          if (warp >= 2) {                              // up rows: hand them to warps 0-1
            float* xr = sX + (32 * (warp - 2) + lane) * kXPitch;
#pragma unroll
            for (int j = 0; j < 32; ++j) xr[j] = __uint_as_float(d[j]);
          }
          named_bar_sync(2, 128);
          if (warp < 2) {
            const int hi = m * 128 + 64 * (int)rank + 32 * warp + lane;     // h column
            const float* xr = sX + (32 * warp + lane) * kXPitch;
            uint16_t* o = static_cast<uint16_t*>(p.out) + (size_t)(grp.y + n0) * p.out_stride + hi;
            const float* cs = p.colscale + grp.y + n0;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nn) {
                const float c = p.f16 ? __ldg(cs + j) : 1.0f;
                o[(size_t)j * p.out_stride] =
                    (uint16_t)f32_to_bf16_bits(silu_mul_fast(__uint_as_float(d[j]) * c * gm0, xr[j] * c * gm1));
              }
          }
          named_bar_sync(2, 128);
        } else {
          const int row = m * 256 + 128 * (int)rank + 32 * warp + lane;
          float* o = static_cast<float*>(p.out) + (size_t)(grp.y + n0) * p.out_stride + row;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nn) o[(size_t)j * p.out_stride] = __uint_as_float(d[j]) * gm0;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(d_empty0 + 8u * buf);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ dequant
    const int t = threadIdx.x - 128;                    // weight row within the CTA's 128
    const uint32_t w_base = smem_addr(sW), s_base = smem_addr(sS);
    const uint32_t a_full0 = map_to(smem_addr(a_full), 0);
    // The two 16-byte halves of a 32-byte code row are read in an order that alternates every
    // four rows, so a warp's 128-bit shared loads cover all 32 banks without conflicts.
    const uint32_t h0 = ((t >> 2) & 1) * 16, h1 = h0 ^ 16;
    int q = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int tt = pair + i * npairs;
      if (tt >= ntiles) break;
      for (int c = 0; c < nst; ++c, ++q) {
        const int ws = q % kWSt, ss = (q >> 2) % kSSt;
        const bool got = mbar_wait(&w_full[ws], (q / kWSt) & 1) &&
                         ((c & 3) != 0 || mbar_wait(&s_full[ss], ((q >> 2) / kSSt) & 1));
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const uint32_t row = w_base + ws * kWBytes + t * 32;
        const uint4 u = ld_shared_v4(row + h0), v = ld_shared_v4(row + h1);
        const uint4 c0 = h0 ? v : u, c1 = h0 ? u : v;
        const uint32_t sc4 = ld_shared_u32(s_base + ss * kSBytes + t * 16 + (c & 3) * 4);
        const int s = q % kSt;
        if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ((q / kSt) & 1) ^ 1))) {
          ok = false;
          break;
        }
        const uint32_t base = smem_addr(sA + s * kABytes) + t * 128;
        const uint32_t h01 = e4m3x2_to_f16x2((uint16_t)(sc4 & 0xFFFF));
        const uint32_t h23 = e4m3x2_to_f16x2((uint16_t)(sc4 >> 16));
        const uint32_t sc[4] = {bcast_half(h01, false), bcast_half(h01, true), bcast_half(h23, false),
                                bcast_half(h23, true)};
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        if (p.f16) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t e[4];
            e2m1x8_to_f16x8(w[j], e);
            st_shared_v4(base + ((j ^ (t & 7)) << 4), hmul2(e[0], sc[j >> 1]), hmul2(e[1], sc[j >> 1]),
                         hmul2(e[2], sc[j >> 1]), hmul2(e[3], sc[j >> 1]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t e[4];
            e2m1x8_scaled_to_bf16x8(w[j], sc[j >> 1], e);
            st_shared_v4(base + ((j ^ (t & 7)) << 4), e[0], e[1], e[2], e[3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        // The raw slots go back to the TMA only after every lane's proxy fence above (a TMA
        // write into a slot read with generic loads must be ordered after those reads).
        if (lane == 0) {
          mbar_arrive_cluster(a_full0 + 8u * s);
          mbar_arrive(&w_empty[ws]);
          if ((c & 3) == 3) mbar_arrive(&s_empty[ss]);
        }
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ activation TMA
    if (lane == 0) {
      const uint32_t b_full0 = map_to(smem_addr(b_full), 0);
      int q = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int tt = pair + i * npairs;
        if (tt >= ntiles) break;
        const int4 grp = __ldg(&p.groups[tt / p.tiles_per_group]);
        const int nh = tile_n(grp.z) / 2;               // this CTA's activation rows
        const int nbox = (nh + kBoxRows - 1) / kBoxRows;
        for (int c = 0; c < nst; ++c, ++q) {
          const int s = q % kSt;
          if (!mbar_wait(&empty[s], ((q / kSt) & 1) ^ 1)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&b_full[s], 2 * nbox * kBoxRows * kKC * 2);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_pair(sB + s * kBBytes + b * kBoxRows * kKC * 2, &maps.x, c * kKC * 2,   // x in bytes
                             grp.y + (int)rank * nh + b * kBoxRows, b_full0 + 8u * s);
        }
      }
      // Leave no copy in flight: CTA 0 waits for its stages' bytes (both halves); CTA 1's copies
      // complete on those same barriers, so it waits for the MMA commits of its last stages.
      if (rank == 0)
        for (int j = max(0, q - kSt); j < q; ++j) mbar_wait(&b_full[j % kSt], (j / kSt) & 1);
      else
        for (int j = max(0, q - kSt); j < q; ++j) mbar_wait(&empty[j % kSt], (j / kSt) & 1);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ weight TMA
    if (lane == 0) {
      int q = 0, qs = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int tt = pair + i * npairs;
        if (tt >= ntiles) break;
        const int g = tt / p.tiles_per_group, m = tt - g * p.tiles_per_group;
        const int e = __ldg(&p.groups[g].x);
        // The raw codes come from HBM in 32-byte rows: prefetch them into L2 kPrefetch stages
        // ahead of their load (the ring is only kWSt deep).
        auto prefetch_stage = [&](int cs) {
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            tma_prefetch_3d(&maps.codes[mt], cs * (kKC / 2), row0(m, mt), e);
            if ((cs & 3) == 0) tma_prefetch_3d(&maps.scales[mt], (cs >> 2) * 16, row0(m, mt), e);
          }
        };
        for (int cp = 1; cp < kPrefetch && cp < nst; ++cp) prefetch_stage(cp);
        for (int c = 0; c < nst && ok; ++c, ++q) {
          if (c + kPrefetch < nst) prefetch_stage(c + kPrefetch);
          if ((c & 3) == 0) {                           // scales of stages c .. c+3
            const int ss = qs % kSSt;
            if (!mbar_wait(&s_empty[ss], ((qs / kSSt) & 1) ^ 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&s_full[ss], kSBytes);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
              tma_load_3d(sS + ss * kSBytes + mt * (kSBytes / 2), &maps.scales[mt], (c >> 2) * 16, row0(m, mt), e,
                          &s_full[ss]);
            ++qs;
          }
          const int ws = q % kWSt;
          if (!mbar_wait(&w_empty[ws], ((q / kWSt) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&w_full[ws], kWBytes);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt)
            tma_load_3d(sW + ws * kWBytes + mt * (kWBytes / 2), &maps.codes[mt], c * (kKC / 2), row0(m, mt), e,
                        &w_full[ws]);
        }
      }
      for (int j = max(0, q - kWSt); j < q; ++j) mbar_wait(&w_full[j % kWSt], (j / kWSt) & 1);
      for (int j = max(0, qs - kSSt); j < qs; ++j) mbar_wait(&s_full[j % kSSt], (j / kSSt) & 1);
    }
    __syncwarp();
  } else if (rank == 0) {
    // ------------------------------------------------------------ MMA issue (CTA 0 of the pair)
    if (lane == 0) {
      int q = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int tt = pair + i * npairs;
        if (tt >= ntiles) break;
        const int4 grp = __ldg(&p.groups[tt / p.tiles_per_group]);
        const int N = tile_n(grp.z);
        const uint32_t idesc = p.f16 ? idesc_f16(2 * kRows, N) : idesc_bf16(2 * kRows, N);
        const int buf = i & 1;
        if (i >= 2 && !mbar_wait_cluster(&d_empty[buf], ((i >> 1) - 1) & 1)) break;
        tc_fence_after();
        const uint32_t dt = tmem + 256u * buf;
        for (int c = 0; c < nst; ++c, ++q) {
          const int s = q % kSt;
          const uint32_t ph = (q / kSt) & 1;
          if (!mbar_wait_cluster(&a_full[s], ph) || !mbar_wait(&b_full[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_addr(sA + s * kABytes), b0 = smem_addr(sB + s * kBBytes);
#pragma unroll
          for (int k = 0; k < kKC / 16; ++k)
            tc_mma_pair(dt, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc, (c | k) != 0);
          tc_commit_pair(&empty[s]);
        }
        if (ok) tc_commit_pair(&d_full[buf]);
      }
      // Do not free tensor memory while MMAs may still run (matters only on the error path).
      if (q > 0) mbar_wait(&empty[(q - 1) % kSt], ((q - 1) / kSt) & 1);
    }
    __syncwarp();
  }
  tc_fence_before();
  cluster_sync();                                       // no CTA leaves while its pair may still use it
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

// Pairs that can be resident at once (one pair per two SMs, or fewer if the cluster placement
// leaves SMs unpaired); 0 if the device cannot run the kernel.
int prefill2_pairs(int num_sms) {
  static int cached = -1;
  if (cached >= 0) return cached;
  cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(prefill2_kernel), kSmem);
  if (err != cudaSuccess) return cached = 0;
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(num_sms & ~1));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  err = cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(prefill2_kernel), &cfg);
  if (err != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return cached = n;
}

int launch_prefill2(const P2Params& p, const P2Maps& maps, int pairs, cudaStream_t s) {
  cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(prefill2_kernel), kSmem);
  if (err != cudaSuccess) return -(int)err;
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, prefill2_kernel, maps, p);
  if (err == cudaSuccess) err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

int make_p2_maps(P2Maps* maps, const BankView& bank, const void* xp, int64_t R, int K, int proj0, int proj1,
                 int rows) {
  {
    const uint64_t d[2] = {(uint64_t)K * 2, (uint64_t)R}, st[1] = {(uint64_t)K * 2};
    const uint32_t b[2] = {kKC * 2, kBoxRows};
    int rc = make_tensor_map(&maps->x, 2, xp, d, st, b, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
  }
  const int projs[2] = {proj0, proj1};
  for (int mt = 0; mt < 2; ++mt) {
    const uint64_t cd[3] = {(uint64_t)K / 2, (uint64_t)rows, (uint64_t)bank.E};
    const uint64_t cs[2] = {(uint64_t)K / 2, bank.stride};
    const uint32_t cb[3] = {kKC / 2, kBoxRows, 1};
    int rc = make_tensor_map(&maps->codes[mt], 3, bank.base + bank.codes_off[projs[mt]], cd, cs, cb,
                             CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
    const uint64_t sd[3] = {(uint64_t)K / 16, (uint64_t)rows, (uint64_t)bank.E};
    const uint64_t ss[2] = {(uint64_t)K / 16, bank.stride};
    const uint32_t sb[3] = {16, kBoxRows, 1};
    rc = make_tensor_map(&maps->scales[mt], 3, bank.base + bank.scales_off[projs[mt]], sd, ss, sb,
                         CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  return 0;
}

int launch_prefill2_gateup(const BankView& bank, const void* xp, const float* colscale, int64_t R,
                           const RouteBufs& rb, void* hb, int pairs, cudaStream_t s) {
  P2Maps maps;
  int rc = make_p2_maps(&maps, bank, xp, R, bank.H, 0, 1, bank.I);
  if (rc) return rc;
  P2Params p{};
  p.bank = bank.base;
  p.f16 = colscale != nullptr;
  p.colscale = colscale;
  p.stride = bank.stride;
  p.global_off[0] = bank.global_off[0];
  p.global_off[1] = bank.global_off[1];
  p.global_mode = bank.global_mode;
  p.K = bank.H;
  p.tiles_per_group = bank.I / 128;
  p.gateup = 1;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.out = hb;
  p.out_stride = bank.I;
  return launch_prefill2(p, maps, pairs, s);
}

int launch_prefill2_down(const BankView& bank, const void* hb, int64_t R, const RouteBufs& rb, float* y, int pairs,
                         cudaStream_t s) {
  P2Maps maps;
  int rc = make_p2_maps(&maps, bank, hb, R, bank.I, 2, 2, bank.H);
  if (rc) return rc;
  P2Params p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  p.global_off[0] = bank.global_off[2];
  p.global_off[1] = bank.global_off[2];
  p.global_mode = bank.global_mode;
  p.K = bank.I;
  p.tiles_per_group = bank.H / 256;
  p.gateup = 0;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.out = y;
  p.out_stride = bank.H;
  return launch_prefill2(p, maps, pairs, s);
}

}  // namespace moe
