// Decode path: memory-bound grouped NVFP4 expert GEMV/GEMM.
//
// Work item = (group, row tile): a group is <= 8 routed rows of one expert (in permuted
// order), a row tile is 16 MMA rows x the full input width K.  For gate/up the 16 MMA rows
// are 8 gate rows and the same 8 up rows, so SwiGLU is applied in-thread in the epilogue;
// for down they are 16 rows of Wd.
//
// One CTA per SM walks a contiguous range of items.  Warp kNW (the producer) streams each
// tile's codes and scales into a ring of shared-memory stages with 1-D bulk copies (TMA),
// one copy per weight row so that rows land at a padded pitch (conflict-free reads).  The
// kNW consumer warps split K: warp w takes 128-wide K units w, w + kNW, ...  Each thread
// dequantizes its codes in registers (E2M1 -> f16 by cvt, times the E4M3 block scale in
// f16, both exact), and feeds mma.sync m16n8k16 with the weights as A (16 rows) and the
// group's activations as B (N = 8 token slots, f32 accumulators).  Partial sums of the
// warps are added through shared memory; the global scale and SwiGLU are applied in f32.
//
// Within one MMA the 16 logical k of a row come from four threads; thread tid4 supplies
// K offsets 32*tid4 + 4*s .. +3 of the unit for k-step s, and the activations are staged
// in shared memory in the matching order, so no data is shuffled between threads.
//
// Weight layout: page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit
// residents", section "What this pack holds"; SwiGLU in FP32: page "Beam-1.0-501B-A23B VQ
// GGUF", section "What stays native".
#include "common.cuh"
#include "internal.h"

namespace moe {

__device__ int g_status = 0;

namespace {

constexpr int kNW = 10;                    // consumer warps
constexpr int kThreads = 32 * (kNW + 1);   // + one producer warp
constexpr int kTileRows = 16;
constexpr int kMaxStages = 8;
constexpr int kSmemLimit = 232448;         // 227 KB opt-in per block on sm_100

struct DecodeParams {
  const uint8_t* bank;
  uint64_t stride;
  uint64_t codes_off[2], scales_off[2], global_off[2];  // [0] gate (or down), [1] up
  int global_mode;
  int K, N;       // inputs per weight row, output rows per matrix
  int k;          // routing top-k: routed row r belongs to token r / k
  int stages;
  int xrows;      // activation rows staged per group (1 .. 8)
  const int4* groups;
  const int32_t* ngroups;
  const int32_t* perm;
  const void* xin;  // gate/up: bf16 x [T, K]; down: f32 h [R, K] (permuted rows)
  float* out;       // [R, N] (permuted rows)
};

struct Layout {
  int code_pitch, stage_codes, stage_bytes, xs_pitch, off_xs, off_red, off_bar, total;
};

__host__ __device__ inline Layout make_layout(int K, int stages, int xrows) {
  Layout L;
  const int rowb = K / 2;
  L.code_pitch = rowb + ((rowb % 128) == 0 ? 64 : 0);   // pitch = 64 (mod 128)
  L.stage_codes = kTileRows * L.code_pitch;
  L.stage_bytes = (L.stage_codes + kTileRows * (K / 16) + 127) & ~127;
  L.xs_pitch = K * 2 + 64;                              // = 64 (mod 128)
  L.off_xs = stages * L.stage_bytes;
  L.off_red = L.off_xs + ((xrows * L.xs_pitch + 127) & ~127);
  L.off_bar = L.off_red + 2 * kNW * 32 * 16;
  L.total = L.off_bar + 2 * stages * 8;
  return L;
}

// Stage the group's activations as f16 in the fragment order: inside each 128-wide K unit,
// the 8 values K0 .. K0+7 with K0 = 32*t + 8*i go to 16-byte chunk 4*i + t.
template <bool GATEUP>
__device__ void fill_xs(const DecodeParams& p, const Layout& L, uint8_t* xs, int row0, int nrows,
                        int ctid) {
  const int cpr = p.K / 8;  // chunks of 8 values per row
  for (int c = ctid; c < p.xrows * cpr; c += kNW * 32) {
    const int n = c / cpr, kk = (c - n * cpr) * 8;
    const int u = kk >> 7, q = kk & 127;
    uint4* dst = reinterpret_cast<uint4*>(xs + n * L.xs_pitch + u * 256 +
                                          (((q & 31) >> 3) * 4 + (q >> 5)) * 16);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n < nrows) {
      if (GATEUP) {
        const int t = p.perm[row0 + n] / p.k;
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(
            static_cast<const uint16_t*>(p.xin) + (size_t)t * p.K + kk));
        v.x = pack_f16x2(bf16_bits_to_f32(b.x & 0xFFFF), bf16_bits_to_f32(b.x >> 16));
        v.y = pack_f16x2(bf16_bits_to_f32(b.y & 0xFFFF), bf16_bits_to_f32(b.y >> 16));
        v.z = pack_f16x2(bf16_bits_to_f32(b.z & 0xFFFF), bf16_bits_to_f32(b.z >> 16));
        v.w = pack_f16x2(bf16_bits_to_f32(b.w & 0xFFFF), bf16_bits_to_f32(b.w >> 16));
      } else {
        const float4* src = reinterpret_cast<const float4*>(
            static_cast<const float*>(p.xin) + (size_t)(row0 + n) * p.K + kk);
        const float4 a = src[0], b = src[1];
        v.x = pack_f16x2(a.x, a.y);
        v.y = pack_f16x2(a.z, a.w);
        v.z = pack_f16x2(b.x, b.y);
        v.w = pack_f16x2(b.z, b.w);
      }
    }
    *dst = v;
  }
}

template <bool GATEUP>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Layout L = make_layout(p.K, p.stages, p.xrows);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.off_bar);
  uint64_t* empty = full + p.stages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = GATEUP ? p.N / 8 : p.N / kTileRows;
  const int items = *p.ngroups * tiles;
  const int per = items / (int)gridDim.x, rem = items % (int)gridDim.x;
  const int i0 = (int)blockIdx.x * per + min((int)blockIdx.x, rem);
  const int i1 = i0 + per + ((int)blockIdx.x < rem ? 1 : 0);
  const uint32_t rowb = p.K / 2, scb = p.K / 16;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kNW);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kNW) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int issued = 0;
      for (int it = i0; it < i1; ++it, ++issued) {
        const int j = it - i0, s = j % p.stages;
        const uint32_t ph = (j / p.stages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1)) break;
        const int g = it / tiles, tile = it - g * tiles;
        const uint8_t* rec = p.bank + (uint64_t)p.groups[g].x * p.stride;
        uint8_t* st = smem + s * L.stage_bytes;
        mbar_arrive_expect_tx(&full[s], kTileRows * (rowb + scb));
        if (GATEUP) {
          const int n0 = tile * 8;
          const uint8_t* gc = rec + p.codes_off[0] + (size_t)n0 * rowb;
          const uint8_t* uc = rec + p.codes_off[1] + (size_t)n0 * rowb;
#pragma unroll 1
          for (int r = 0; r < 8; ++r) {
            bulk_g2s(st + r * L.code_pitch, gc + (size_t)r * rowb, rowb, &full[s], pol);
            bulk_g2s(st + (8 + r) * L.code_pitch, uc + (size_t)r * rowb, rowb, &full[s], pol);
          }
          bulk_g2s(st + L.stage_codes, rec + p.scales_off[0] + (size_t)n0 * scb, 8 * scb, &full[s], pol);
          bulk_g2s(st + L.stage_codes + 8 * scb, rec + p.scales_off[1] + (size_t)n0 * scb, 8 * scb,
                   &full[s], pol);
        } else {
          const int n0 = tile * kTileRows;
          const uint8_t* dc = rec + p.codes_off[0] + (size_t)n0 * rowb;
#pragma unroll 1
          for (int r = 0; r < kTileRows; ++r)
            bulk_g2s(st + r * L.code_pitch, dc + (size_t)r * rowb, rowb, &full[s], pol);
          bulk_g2s(st + L.stage_codes, rec + p.scales_off[0] + (size_t)n0 * scb, kTileRows * scb,
                   &full[s], pol);
        }
      }
      // Do not leave while copies may still be landing (matters only on the error path).
      for (int j = max(0, issued - p.stages); j < issued; ++j)
        mbar_wait(&full[j % p.stages], (j / p.stages) & 1);
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int gid = lane >> 2, tid4 = lane & 3;
  const int units = p.K / 128;
  uint8_t* xs = smem + L.off_xs;
  float4* red = reinterpret_cast<float4*>(smem + L.off_red);
  int cur_g = -1, row0 = 0, nrows = 0;
  float gm0 = 0.0f, gm1 = 0.0f;
  const bool has_x = gid < p.xrows;
  const uint8_t* xrow = xs + (has_x ? gid : 0) * L.xs_pitch + tid4 * 16;

  for (int it = i0; it < i1; ++it) {
    const int j = it - i0, s = j % p.stages;
    const uint32_t ph = (j / p.stages) & 1;
    const int g = it / tiles, tile = it - g * tiles;
    if (g != cur_g) {
      named_bar_sync(1, kNW * 32);
      const int4 grp = p.groups[g];
      row0 = grp.y;
      nrows = grp.z;
      const uint8_t* rec = p.bank + (uint64_t)grp.x * p.stride;
      gm0 = global_mult(*reinterpret_cast<const float*>(rec + p.global_off[0]), p.global_mode);
      gm1 = GATEUP ? global_mult(*reinterpret_cast<const float*>(rec + p.global_off[1]), p.global_mode)
                   : 0.0f;
      fill_xs<GATEUP>(p, L, xs, row0, nrows, threadIdx.x);
      named_bar_sync(1, kNW * 32);
      cur_g = g;
    }
    if (!mbar_wait(&full[s], ph)) break;

    const uint8_t* st = smem + s * L.stage_bytes;
    const uint8_t* rowA = st + gid * L.code_pitch + tid4 * 16;
    const uint8_t* rowB = rowA + 8 * L.code_pitch;
    const uint8_t* scA = st + L.stage_codes + gid * scb + tid4 * 2;
    const uint8_t* scB = scA + 8 * scb;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
    for (int u = warp; u < units; u += kNW) {
      const uint4 qa = *reinterpret_cast<const uint4*>(rowA + u * 64);
      const uint4 qb = *reinterpret_cast<const uint4*>(rowB + u * 64);
      const uint32_t hsa = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(scA + u * 8));
      const uint32_t hsb = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(scB + u * 8));
      uint4 xq[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        xq[i] = has_x ? *reinterpret_cast<const uint4*>(xrow + u * 256 + i * 64)
                      : make_uint4(0, 0, 0, 0);
      const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
      const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t sA = bcast_half(hsa, q >= 2), sB = bcast_half(hsb, q >= 2);
        uint32_t fa[4], fb[4];
        e2m1x8_to_f16x8(wa[q], fa);
        e2m1x8_to_f16x8(wb[q], fb);
        const uint32_t a0[4] = {hmul2(fa[0], sA), hmul2(fb[0], sB), hmul2(fa[1], sA), hmul2(fb[1], sB)};
        mma_16816(acc, a0, xq[q].x, xq[q].y);
        const uint32_t a1[4] = {hmul2(fa[2], sA), hmul2(fb[2], sB), hmul2(fa[3], sA), hmul2(fb[3], sB)};
        mma_16816(acc, a1, xq[q].z, xq[q].w);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    const int buf = j & 1;
    red[(buf * kNW + warp) * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    named_bar_sync(1, kNW * 32);
    if (warp == j % kNW) {
      float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        const float4 v = red[(buf * kNW + w) * 32 + lane];
        c[0] += v.x;
        c[1] += v.y;
        c[2] += v.z;
        c[3] += v.w;
      }
      // c[0], c[1]: MMA row gid, token slots 2*tid4, 2*tid4+1; c[2], c[3]: MMA row gid + 8.
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int n = 2 * tid4 + cc;
        if (n < nrows) {
          float* o = p.out + (size_t)(row0 + n) * p.N;
          if (GATEUP) {
            const float gv = c[cc] * gm0, uv = c[2 + cc] * gm1;
            o[tile * 8 + gid] = gv / (1.0f + expf(-gv)) * uv;
          } else {
            o[tile * kTileRows + gid] = c[cc] * gm0;
            o[tile * kTileRows + gid + 8] = c[2 + cc] * gm0;
          }
        }
      }
    }
  }
}

int pick_stages(int K, int xrows, int stage_cap) {
  for (int s = stage_cap; s >= 2; --s)
    if (make_layout(K, s, xrows).total <= kSmemLimit) return s;
  return 0;
}

template <bool GATEUP>
int launch(const DecodeParams& p0, int num_sms, cudaStream_t s) {
  DecodeParams p = p0;
  p.stages = pick_stages(p.K, p.xrows, kMaxStages);
  if (p.stages == 0) return -(int)cudaErrorInvalidValue;
  const int bytes = make_layout(p.K, p.stages, p.xrows).total;
  cudaError_t err = cudaFuncSetAttribute(decode_kernel<GATEUP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err != cudaSuccess) return -(int)err;
  decode_kernel<GATEUP><<<num_sms, kThreads, bytes, s>>>(p);
  err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

}  // namespace

size_t decode_smem_bytes(int K, int xrows, bool gateup) {
  (void)gateup;
  const int st = pick_stages(K, xrows, kMaxStages);
  return st ? (size_t)make_layout(K, st, xrows).total : 0;
}

int launch_decode_gateup(const BankView& bank, const uint16_t* x, int k, const RouteBufs& rb,
                         int xrows, float* h, int num_sms, cudaStream_t s) {
  DecodeParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  p.codes_off[0] = bank.codes_off[0];
  p.codes_off[1] = bank.codes_off[1];
  p.scales_off[0] = bank.scales_off[0];
  p.scales_off[1] = bank.scales_off[1];
  p.global_off[0] = bank.global_off[0];
  p.global_off[1] = bank.global_off[1];
  p.global_mode = bank.global_mode;
  p.K = bank.H;
  p.N = bank.I;
  p.k = k;
  p.xrows = xrows;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.perm = rb.perm;
  p.xin = x;
  p.out = h;
  return launch<true>(p, num_sms, s);
}

int launch_decode_down(const BankView& bank, const float* h, const RouteBufs& rb, int xrows,
                       float* y, int num_sms, cudaStream_t s) {
  DecodeParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  p.codes_off[0] = bank.codes_off[2];
  p.scales_off[0] = bank.scales_off[2];
  p.global_off[0] = bank.global_off[2];
  p.global_mode = bank.global_mode;
  p.K = bank.I;
  p.N = bank.H;
  p.k = 1;
  p.xrows = xrows;
  p.groups = rb.groups;
  p.ngroups = rb.ngroups;
  p.perm = rb.perm;
  p.xin = h;
  p.out = y;
  return launch<false>(p, num_sms, s);
}

}  // namespace moe
