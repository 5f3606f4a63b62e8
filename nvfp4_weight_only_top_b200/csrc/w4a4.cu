// W4A4 path: NVFP4 weights times NVFP4 activations on the block-scaled tensor cores
// (tcgen05.mma kind::mxf4nvf4: E2M1 operands, one UE4M3 scale per 16 inputs on each side, f32
// accumulators in tensor memory).
//
// What it computes (page "Beam-1.0-501B-A23B, EXL3 3-bit ...", section "Fidelity": the official
// NVFP4 release served on Blackwell with FP4 activations; page "Beam 1.0 501B-A23B, streaming
// pack, NVFP4 experts / MLX 8-bit residents", section "What this pack holds": the release's
// activation scales, unused by the BF16-activation build).  A routed row of expert e quantizes its
// token's x with the expert's input multiplier s_x[e] as the NVFP4 global (block scales and codes
// found from the values, each decision on an f32 quotient rounded to nearest even, as the
// encoder does), runs gate and up on the tensor cores, forms h = silu(g) * u in f32 and
// quantizes it with s_h[e] in the same way, then runs down.  The combine is the BF16 path's.
//
// Kernels:
//   w4a4_quant_x_kernel -- one warp per routed row (expert order): 16 BF16 inputs per lane and
//       step -> 8 code bytes and one scale byte;
//   w4a4_gemm_kernel<stages, gate/up | down> -- one persistent CTA per SM, tiles handed out from a
//       global counter.  Tile = one group of up to 128 routed rows of one expert (MMA M = 128) x
//       256 weight rows (MMA N = 256; gate/up: 128 gate rows and the same 128 up rows).  Per K
//       stage of 256 inputs (one 128-byte swizzle row of codes; 54 KB; four stages in flight for
//       gate/up, three for down, whose epilogue staging takes the room of the fourth):
//         warp 8 (one thread)  TMA: activation codes 128 x 128 B, weight codes 2 x 128 x 128 B (both
//                              128B-swizzled, K-major), scale bytes 128 x 16 B and 2 x 128 x 16 B;
//         warp 9               rearranges the scale bytes in place into the layout the tensor core
//                              reads them in: per MMA (64 inputs) and 128 rows, 512 bytes with row
//                              32j + i at byte 16 i + 4 j (its four block scales in one 32-bit word);
//         warp 10 (one thread) tcgen05.cp of those 512-byte chunks into tensor memory (32 lanes x
//                              128 bits, broadcast to the four lane quarters), then four MMAs of
//                              K = 64; tcgen05.commit frees the stage;
//         warps 0-7            epilogue: each thread owns one routed row (a TMEM lane) and copies
//                              its accumulator columns to registers first, handing the accumulator
//                              back to the next tile's MMAs; gate/up then forms h from gate and up
//                              columns and quantizes it per block of 16 in registers, storing codes
//                              and scales; down stores y in f32 through a per-warp shared tile, a
//                              row's 32 columns per warp store.
// Tensor memory: accumulator columns 0..255, then two sets of 48 scale-factor columns (one per
// stage parity: 4 MMAs x (4 columns for the activations + 8 for the weights)).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kM = 128;                   // routed rows per tile (MMA M)
constexpr int kN = 256;                   // weight rows per tile (MMA N)
constexpr int kKS = 256;                  // inputs per stage
constexpr int kACodes = kM * kKS / 2;     // 16 KB
constexpr int kBCodes = kN * kKS / 2;     // 32 KB
constexpr int kARaw = kM * 16;            // 2 KB: 16 scale bytes per row and stage
constexpr int kBRaw = kN * 16;            // 4 KB
constexpr int kEpiPitch = 36;             // floats per staged row (16-byte aligned, 4 wavefronts per v4 store)
constexpr int kEpiBytes = 8 * 32 * kEpiPitch * 4;   // per epilogue warp: 32 rows x 32 floats

// Shared-memory layout with ST stages: activation codes | weight codes | activation scale bytes |
// weight scale bytes (both rearranged in place into the tensor core's layout) | barriers | (down
// only) the epilogue's staging of y.  Gate/up keeps four stages in flight, down three (its
// epilogue staging takes the room of the fourth).
template <int ST, bool GATEUP>
struct Layout {
  static constexpr int kOffBc = ST * kACodes;
  static constexpr int kOffAr = kOffBc + ST * kBCodes;
  static constexpr int kOffBr = kOffAr + ST * kARaw;
  static constexpr int kOffBars = kOffBr + ST * kBRaw;
  static constexpr int kOffEpi = kOffBars + 512;  // barriers, tile queue
  static constexpr int kSmem = kOffEpi + (GATEUP ? 0 : kEpiBytes) + 1024 /*alignment*/;
  static_assert(kSmem <= 232448, "shared memory per block");
};
constexpr int kStGateUp = 4, kStDown = 3;
constexpr int kPrefetch = 6;              // stages of weights prefetched into L2 ahead of their load
constexpr int kEpiWarps = 8;
constexpr int kWarpTma = kEpiWarps, kWarpSf = kEpiWarps + 1, kWarpMma = kEpiWarps + 2;
constexpr int kThreads = 32 * (kEpiWarps + 3);
constexpr int kTmemCols = 512;
constexpr int kSfCol = 256;               // first scale-factor column
constexpr int kSfSet = 48;                // columns of one stage's scale factors
constexpr int kTQ = 4;
constexpr int kTQConsumers = kEpiWarps + 2;   // epilogue warps, scale warp, MMA thread
constexpr uint32_t kStageTx = kACodes + kBCodes + kARaw + kBRaw;

struct GemmParams {
  const uint8_t* bank;
  uint64_t stride;
  uint64_t global_off[2];     // gate/up: gate, up; down: down, down
  int global_mode;
  const float* act_scales;    // [E][2]: input multiplier of gate/up, of down
  int K;                      // inputs per weight row
  int tiles_per_group;        // 256-row weight tiles per group
  int gateup;
  const int4* groups;         // (expert, first routed row, rows <= 128, 0)
  const int32_t* ngroups;
  unsigned* tile_ctr;         // zero at launch
  uint8_t* h_codes;           // gate/up: [R][I/2], expert order
  uint8_t* h_scales;          // gate/up: [R][I/16]
  float* y;                   // down: [R][H] f32
  int I, H;
  const int32_t* perm;        // routed row -> slot t*k + j (for the taps)
  float* tap_h;               // optional, slot order: h f32 [R][I] before quantization
  uint8_t* tap_codes;         // optional (with tap_scales), slot order: [R][I/2]
  uint8_t* tap_scales;        // [R][I/16]
};

struct GemmMaps {
  CUtensorMap a_codes, a_scales;          // activations: [R][K/2], [R][K/16] bytes
  CUtensorMap b_codes[2], b_scales[2];    // weight rows 0..127 / 128..255 of a tile: [E][rows][K/2], [K/16]
};

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_shared_v4f(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Shared-memory descriptor of one 512-byte scale chunk for tcgen05.cp (32 rows x 16 B, K-major,
// no swizzle: 8-row core matrices 128 B apart; a single core matrix across, so the leading
// offset is unused).
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

// Copies a 512-byte chunk (32 rows x 128 bits) into 4 columns of all four TMEM lane quarters.
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D (TMEM, f32) (+)= (A x SFA) (B x SFB)^T, E2M1 operands with UE4M3 scales per 16 inputs, K = 64.
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Instruction descriptor of the block-scaled MMA: E2M1 A and B (format 1), UE4M3 scale factors
// (bit 23 clear), both K-major, scale-factor ids 0, K = 64, M x N.
__host__ __device__ __forceinline__ uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int kSt, bool GATEUP>
__global__ void __launch_bounds__(kThreads, 1) w4a4_gemm_kernel(const __grid_constant__ GemmMaps maps,
                                                                const GemmParams p) {
  using L = Layout<kSt, GATEUP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sAc = smem;
  uint8_t* sBc = smem + L::kOffBc;
  uint8_t* sAr = smem + L::kOffAr;                     // scale bytes: raw, then the tensor core's layout
  uint8_t* sBr = smem + L::kOffBr;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBars);
  uint64_t* full = bars;                   // [kSt] TMA -> scale warp, MMA
  uint64_t* sf_full = full + kSt;          // [kSt] scale warp -> MMA
  uint64_t* empty = sf_full + kSt;         // [kSt] MMA commit -> TMA
  uint64_t* d_full = empty + kSt;          // MMA commit -> epilogue
  uint64_t* d_empty = d_full + 1;          // epilogue warps -> MMA
  uint64_t* tq_full = d_empty + 1;         // [kTQ]
  uint64_t* tq_empty = tq_full + kTQ;      // [kTQ]
  int* s_tq = reinterpret_cast<int*>(tq_empty + kTQ);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_tq + kTQ);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = *p.ngroups * p.tiles_per_group;
  const int nst = p.K / kKS;
  auto pop_tile = [&](int i, int& tt) -> bool {
    const int slot = i % kTQ;
    if (!mbar_wait(&tq_full[slot], (i / kTQ) & 1)) return false;
    tt = ((volatile int*)s_tq)[slot];
    return true;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sf_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(d_full, 1);
    mbar_init(d_empty, kEpiWarps);
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

  if (warp < kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3, hf = warp >> 2;       // TMEM lane quarter, column half
    const int r = 32 * q4 + lane;                  // routed row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
    for (int i = 0;; ++i) {
      int tt = -1;
      if (!__all_sync(0xffffffffu, pop_tile(i, tt))) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&tq_empty[i % kTQ]);
      if (tt < 0) break;
      const int g = tt / p.tiles_per_group, m = tt - g * p.tiles_per_group;
      const int4 grp = __ldg(&p.groups[g]);
      const uint8_t* rec = p.bank + (uint64_t)grp.x * p.stride;
      const float gm0 = global_mult(__ldg(reinterpret_cast<const float*>(rec + p.global_off[0])), p.global_mode);
      const float gm1 = global_mult(__ldg(reinterpret_cast<const float*>(rec + p.global_off[1])), p.global_mode);
      const float sx = __ldg(p.act_scales + 2 * grp.x), sh = __ldg(p.act_scales + 2 * grp.x + 1);
      if (!__all_sync(0xffffffffu, mbar_wait(d_full, i & 1))) break;   // tcgen05.ld needs the whole warp
      tc_fence_after();
      const bool valid = r < grp.z;
      const int64_t row = (int64_t)grp.y + r;
      // All of this warp's accumulator columns go to registers first (128 per thread), and the
      // accumulator is handed back before any arithmetic, so the next tile's MMAs overlap the
      // rest of this epilogue.
      uint32_t d[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(lane_base + (GATEUP ? (c & 1) * 128 + 64 * hf + 32 * (c >> 1) : 128 * hf + 32 * c), d[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(d_empty);
      if (GATEUP) {
        // d[2c] = gate, d[2c + 1] = up columns of h columns 64 hf + 32 c .. +31
        const float cg = gm0 * sx, cu = gm1 * sx;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col = 64 * hf + 32 * c;          // h column within the tile
          float hv[32];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            hv[j] = silu_mul_fast(__uint_as_float(d[2 * c][j]) * cg, __uint_as_float(d[2 * c + 1][j]) * cu);
          uint32_t cw[4], sc[2];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float blk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) blk[j] = hv[16 * b + j];
            sc[b] = nvfp4_encode16_fast(blk, sh, cw[2 * b], cw[2 * b + 1]);
          }
          if (valid) {
            const int hcol = m * kM + col;           // h index
            const uint4 cv = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            const uint16_t sv = (uint16_t)(sc[0] | (sc[1] << 8));
            *reinterpret_cast<uint4*>(p.h_codes + row * (p.I / 2) + hcol / 2) = cv;
            *reinterpret_cast<uint16_t*>(p.h_scales + row * (p.I / 16) + hcol / 16) = sv;
            if (p.tap_h || p.tap_codes) {
              const int64_t slot = __ldg(p.perm + row);
              if (p.tap_h) {
                float4* o = reinterpret_cast<float4*>(p.tap_h + slot * p.I + hcol);
#pragma unroll
                for (int j = 0; j < 8; ++j) o[j] = make_float4(hv[4 * j], hv[4 * j + 1], hv[4 * j + 2], hv[4 * j + 3]);
              }
              if (p.tap_codes) {
                *reinterpret_cast<uint4*>(p.tap_codes + slot * (p.I / 2) + hcol / 2) = cv;
                *reinterpret_cast<uint16_t*>(p.tap_scales + slot * (p.I / 16) + hcol / 16) = sv;
              }
            }
          }
        }
      } else {
        // y through a per-warp shared-memory tile: a thread holds 32 columns of one row, a warp
        // store writes 32 columns of one row (128 contiguous bytes) -- row by row.
        const float cy = gm0 * sh;
        float* stg = reinterpret_cast<float*>(smem + L::kOffEpi) + warp * 32 * kEpiPitch;
        const uint32_t my = smem_addr(stg + lane * kEpiPitch);
        const int nrows = min(32, grp.z - 32 * q4);    // valid rows of this lane quarter
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4f(my + 16 * j, __uint_as_float(d[c][4 * j]) * cy, __uint_as_float(d[c][4 * j + 1]) * cy,
                          __uint_as_float(d[c][4 * j + 2]) * cy, __uint_as_float(d[c][4 * j + 3]) * cy);
          __syncwarp();
          float* o = p.y + ((int64_t)grp.y + 32 * q4) * p.H + m * kN + 128 * hf + 32 * c + lane;
          for (int rr = 0; rr < nrows; ++rr) o[(int64_t)rr * p.H] = stg[rr * kEpiPitch + lane];
          __syncwarp();
        }
      }
    }
  } else if (warp == kWarpTma) {
    // ------------------------------------------------------------ tile scheduler + TMA
    if (lane == 0) {
      bool ok = true;
      int q = 0;
      for (int i = 0; ok; ++i) {
        const int slot = i % kTQ;
        if (!mbar_wait(&tq_empty[slot], ((i / kTQ) & 1) ^ 1)) break;
        int tt = (int)atomicAdd(p.tile_ctr, 1u);
        if (tt >= ntiles) tt = -1;
        ((volatile int*)s_tq)[slot] = tt;
        mbar_arrive(&tq_full[slot]);
        if (tt < 0) break;
        const int g = tt / p.tiles_per_group, m = tt - g * p.tiles_per_group;
        const int4 grp = __ldg(&p.groups[g]);
        const int row0 = GATEUP ? m * 128 : m * kN, row1 = GATEUP ? m * 128 : m * kN + 128;
        // Weight boxes come from HBM: prefetch them into L2 kPrefetch stages ahead of their load.
        auto prefetch_stage = [&](int cs) {
          tma_prefetch_3d(&maps.b_codes[0], cs * (kKS / 2), row0, grp.x);
          tma_prefetch_3d(&maps.b_codes[1], cs * (kKS / 2), row1, grp.x);
          tma_prefetch_3d(&maps.b_scales[0], cs * 16, row0, grp.x);
          tma_prefetch_3d(&maps.b_scales[1], cs * 16, row1, grp.x);
        };
        for (int cp = 1; cp < kPrefetch && cp < nst; ++cp) prefetch_stage(cp);
        for (int c = 0; c < nst; ++c, ++q) {
          if (c + kPrefetch < nst) prefetch_stage(c + kPrefetch);
          const int s = q % kSt;
          if (!mbar_wait(&empty[s], ((q / kSt) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kStageTx);
          tma_load_2d(sAc + s * kACodes, &maps.a_codes, c * (kKS / 2), grp.y, &full[s]);
          tma_load_2d(sAr + s * kARaw, &maps.a_scales, c * 16, grp.y, &full[s]);
          tma_load_3d(sBc + s * kBCodes, &maps.b_codes[0], c * (kKS / 2), row0, grp.x, &full[s]);
          tma_load_3d(sBc + s * kBCodes + kBCodes / 2, &maps.b_codes[1], c * (kKS / 2), row1, grp.x, &full[s]);
          tma_load_3d(sBr + s * kBRaw, &maps.b_scales[0], c * 16, row0, grp.x, &full[s]);
          tma_load_3d(sBr + s * kBRaw + kBRaw / 2, &maps.b_scales[1], c * 16, row1, grp.x, &full[s]);
        }
      }
      // Leave no copy in flight (only an error path gets here with copies outstanding).
      for (int j = max(0, q - kSt); j < q; ++j) mbar_wait(&full[j % kSt], (j / kSt) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpSf) {
    // ------------------------------------------------------------ scale bytes -> tensor-core layout
    // Lane l handles rows 32 j + i with j = l & 3 and i = 8 it + (l >> 2): its loads cover four
    // runs of 8 consecutive 16-byte rows and its stores one run of 128 bytes per MMA, both free
    // of bank conflicts.
    const int j4 = lane & 3, i8 = lane >> 2;
    int q = 0;
    for (int i = 0;; ++i) {
      int tt = -1;
      if (!__all_sync(0xffffffffu, pop_tile(i, tt))) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&tq_empty[i % kTQ]);
      if (tt < 0) break;
      bool ok = true;
      for (int c = 0; c < nst; ++c, ++q) {
        const int s = q % kSt;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (q / kSt) & 1))) {
          ok = false;
          break;
        }
        // In place: every lane loads its 12 rows before any lane stores.
        const uint32_t ar = smem_addr(sAr + s * kARaw), br = smem_addr(sBr + s * kBRaw);
        uint4 va[4], vb[8];
#pragma unroll
        for (int it = 0; it < 4; ++it) va[it] = lds_v4(ar + 16 * (32 * j4 + 8 * it + i8));
#pragma unroll
        for (int it = 0; it < 8; ++it) vb[it] = lds_v4(br + 16 * (128 * (it >> 2) + 32 * j4 + 8 * (it & 3) + i8));
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const uint32_t dst = ar + 16 * (8 * it + i8) + 4 * j4;
          st_shared_u32(dst, va[it].x);
          st_shared_u32(dst + 512, va[it].y);
          st_shared_u32(dst + 1024, va[it].z);
          st_shared_u32(dst + 1536, va[it].w);
        }
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const uint32_t dst = br + 512 * (it >> 2) + 16 * (8 * (it & 3) + i8) + 4 * j4;
          st_shared_u32(dst, vb[it].x);
          st_shared_u32(dst + 1024, vb[it].y);
          st_shared_u32(dst + 2048, vb[it].z);
          st_shared_u32(dst + 3072, vb[it].w);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[s]);
      }
      if (!ok) break;
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_nvf4(kM, kN);
      int q = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        int tt = -1;
        if (!pop_tile(i, tt)) break;
        mbar_arrive(&tq_empty[i % kTQ]);
        if (tt < 0) break;
        if (i > 0 && !mbar_wait(d_empty, (i - 1) & 1)) break;
        tc_fence_after();
        for (int c = 0; c < nst; ++c, ++q) {
          const int s = q % kSt;
          const uint32_t ph = (q / kSt) & 1;
          if (!mbar_wait(&full[s], ph) || !mbar_wait(&sf_full[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf = tmem + kSfCol + (uint32_t)((q & 1) * kSfSet);
          const uint32_t aa = smem_addr(sAr + s * kARaw), ba = smem_addr(sBr + s * kBRaw);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            tc_cp_sf(sf + 12 * k, smem_desc_sf(aa + 512 * k));
            tc_cp_sf(sf + 12 * k + 4, smem_desc_sf(ba + 1024 * k));
            tc_cp_sf(sf + 12 * k + 8, smem_desc_sf(ba + 1024 * k + 512));
          }
          const uint32_t a0 = smem_addr(sAc + s * kACodes), b0 = smem_addr(sBc + s * kBCodes);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_nvf4(tmem, smem_desc_sw128(a0 + 32 * k), smem_desc_sw128(b0 + 32 * k), idesc, sf + 12 * k,
                        sf + 12 * k + 4, (c | k) != 0);
          tc_commit(&empty[s]);
        }
        if (ok) tc_commit(d_full);
      }
      // Do not free tensor memory while MMAs may still run (matters only on the error path).
      if (q > 0) mbar_wait(&empty[(q - 1) % kSt], ((q - 1) / kSt) & 1);
    }
    __syncwarp();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// One warp per routed row r (expert order): x[perm[r] / k] (BF16, exact in f32) quantized with
// the input multiplier of the row's expert; codes [R][H/2] and scales [R][H/16], and the same in
// slot order when tap_codes is given.
constexpr int kQuantWarps = 8;
__global__ void __launch_bounds__(32 * kQuantWarps)
    w4a4_quant_x_kernel(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm, const int32_t* __restrict__ ids,
                        int k, int64_t R, int H, const float* __restrict__ act_scales, uint8_t* __restrict__ codes,
                        uint8_t* __restrict__ scales, uint8_t* __restrict__ tap_codes, uint8_t* __restrict__ tap_scales) {
  const int64_t r = (int64_t)blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (r >= R) return;
  const int lane = threadIdx.x & 31;
  const int slot = __ldg(perm + r);
  const int t = slot / k, e = __ldg(ids + slot);
  const float s2 = __ldg(act_scales + 2 * e);
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  const int nb = H / 16;
  for (int b = lane; b < nb; b += 32) {
    const uint4 v0 = __ldg(src + 2 * b), v1 = __ldg(src + 2 * b + 1);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
      v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
    uint32_t lo, hi;
    const uint32_t sc = nvfp4_encode16_fast(v, s2, lo, hi);
    *reinterpret_cast<uint2*>(codes + r * (H / 2) + 8 * b) = make_uint2(lo, hi);
    scales[r * (H / 16) + b] = (uint8_t)sc;
    if (tap_codes) {
      *reinterpret_cast<uint2*>(tap_codes + (int64_t)slot * (H / 2) + 8 * b) = make_uint2(lo, hi);
      tap_scales[(int64_t)slot * (H / 16) + b] = (uint8_t)sc;
    }
  }
}

int make_act_maps(GemmMaps* m, const uint8_t* codes, const uint8_t* scales, int64_t R, int K) {
  const uint64_t cd[2] = {(uint64_t)K / 2, (uint64_t)R}, cs[1] = {(uint64_t)K / 2};
  const uint32_t cb[2] = {kKS / 2, kM};
  int rc = make_tensor_map(&m->a_codes, 2, codes, cd, cs, cb, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  const uint64_t sd[2] = {(uint64_t)K / 16, (uint64_t)R}, ss[1] = {(uint64_t)K / 16};
  const uint32_t sb[2] = {16, kM};
  return make_tensor_map(&m->a_scales, 2, scales, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE);
}

int make_weight_maps(GemmMaps* m, const BankView& bank, int proj0, int proj1, int rows, int K) {
  const int projs[2] = {proj0, proj1};
  for (int h = 0; h < 2; ++h) {
    const uint64_t cd[3] = {(uint64_t)K / 2, (uint64_t)rows, (uint64_t)bank.E};
    const uint64_t cs[2] = {(uint64_t)K / 2, bank.stride};
    const uint32_t cb[3] = {kKS / 2, 128, 1};
    int rc = make_tensor_map(&m->b_codes[h], 3, bank.base + bank.codes_off[projs[h]], cd, cs, cb,
                             CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    const uint64_t sd[3] = {(uint64_t)K / 16, (uint64_t)rows, (uint64_t)bank.E};
    const uint64_t ss[2] = {(uint64_t)K / 16, bank.stride};
    const uint32_t sb[3] = {16, 128, 1};
    rc = make_tensor_map(&m->b_scales[h], 3, bank.base + bank.scales_off[projs[h]], sd, ss, sb,
                         CU_TENSOR_MAP_SWIZZLE_NONE);
    if (rc) return rc;
  }
  return 0;
}

template <int ST, bool GATEUP>
int launch_gemm_t(const GemmParams& p, const GemmMaps& maps, int num_sms, cudaStream_t s) {
  constexpr int smem = Layout<ST, GATEUP>::kSmem;
  cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(w4a4_gemm_kernel<ST, GATEUP>), smem);
  if (err != cudaSuccess) return -(int)err;
  w4a4_gemm_kernel<ST, GATEUP><<<num_sms, kThreads, smem, s>>>(maps, p);
  err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

int launch_gemm(const GemmParams& p, const GemmMaps& maps, int num_sms, cudaStream_t s) {
  return p.gateup ? launch_gemm_t<kStGateUp, true>(p, maps, num_sms, s)
                  : launch_gemm_t<kStDown, false>(p, maps, num_sms, s);
}

}  // namespace

bool w4a4_supported(int H, int I) { return H % 256 == 0 && I % 256 == 0; }

int launch_w4a4_quant_x(const uint16_t* x, const RouteBufs& rb, int k, int64_t R, int H, const float* act_scales,
                        uint8_t* codes, uint8_t* scales, uint8_t* tap_codes, uint8_t* tap_scales, cudaStream_t s) {
  const int64_t blocks = (R + kQuantWarps - 1) / kQuantWarps;
  w4a4_quant_x_kernel<<<(unsigned)blocks, 32 * kQuantWarps, 0, s>>>(x, rb.perm, rb.ids, k, R, H, act_scales, codes,
                                                                    scales, tap_codes, tap_scales);
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

int launch_w4a4_gateup(const BankView& bank, const float* act_scales, const uint8_t* x_codes, const uint8_t* x_scales,
                       int64_t R, const RouteBufs& rb, uint8_t* h_codes, uint8_t* h_scales, const W4A4Taps& taps,
                       unsigned* tile_ctr, int num_sms, cudaStream_t s) {
  GemmMaps maps;
  int rc = make_act_maps(&maps, x_codes, x_scales, R, bank.H);
  if (!rc) rc = make_weight_maps(&maps, bank, 0, 1, bank.I, bank.H);
  if (rc) return rc;
  GemmParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  p.global_off[0] = bank.global_off[0];
  p.global_off[1] = bank.global_off[1];
  p.global_mode = bank.global_mode;
  p.act_scales = act_scales;
  p.K = bank.H;
  p.tiles_per_group = bank.I / 128;
  p.gateup = 1;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.tile_ctr = tile_ctr;
  p.h_codes = h_codes;
  p.h_scales = h_scales;
  p.I = bank.I;
  p.H = bank.H;
  p.perm = rb.perm;
  p.tap_h = taps.h;
  p.tap_codes = taps.h_codes;
  p.tap_scales = taps.h_scales;
  return launch_gemm(p, maps, num_sms, s);
}

int launch_w4a4_down(const BankView& bank, const float* act_scales, const uint8_t* h_codes, const uint8_t* h_scales,
                     int64_t R, const RouteBufs& rb, float* y, unsigned* tile_ctr, int num_sms, cudaStream_t s) {
  GemmMaps maps;
  int rc = make_act_maps(&maps, h_codes, h_scales, R, bank.I);
  if (!rc) rc = make_weight_maps(&maps, bank, 2, 2, bank.H, bank.I);
  if (rc) return rc;
  GemmParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  p.global_off[0] = bank.global_off[2];
  p.global_off[1] = bank.global_off[2];
  p.global_mode = bank.global_mode;
  p.act_scales = act_scales;
  p.K = bank.I;
  p.tiles_per_group = bank.H / kN;
  p.gateup = 0;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.tile_ctr = tile_ctr;
  p.y = y;
  p.I = bank.I;
  p.H = bank.H;
  return launch_gemm(p, maps, num_sms, s);
}

}  // namespace moe
