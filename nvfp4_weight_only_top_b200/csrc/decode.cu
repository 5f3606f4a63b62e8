// Decode path: memory-bound grouped NVFP4 expert GEMV/GEMM.
//
// Work item = (group, row tile): a group is <= 8 routed rows of one expert (in permuted
// order); a row tile is 16 weight rows x the full input width K, one MMA M-tile.  For gate/up
// the 16 rows are 8 gate rows and the same 8 up rows, so SwiGLU is applied in-thread in the
// epilogue; for down they are 16 rows of Wd.
//
// Two CTAs per SM, each walking a contiguous range of items.  The kNW warps of a CTA split K
// into 128-wide units (warp w takes units w, w + kNW, ...).  A thread streams its share of
// every unit straight from HBM with 128-bit loads into a 3-slot register ring (two units in
// flight while it computes a third), dequantizes 2 rows x 32 codes in registers (E2M1 -> f16
// by cvt, times the E4M3 block scale in f16: both exact) and issues 8 mma.sync m16n8k16 with
// the weights as A and the group's activations (N = 8 token slots, staged once per group in
// shared memory) as B, alternating between two accumulators.  The warps' partial sums are
// added through shared memory in a fixed order; the global scale and SwiGLU follow in f32.
//
// The MMA's 16 logical k of a row come from four threads: thread tid4 supplies 4 K values of
// its own 32-wide slice of the unit per k-step, and the activations are staged in the same
// order, so no data moves between threads.
//
// Weight layout: page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit
// residents", section "What this pack holds"; SwiGLU in FP32: page "Beam-1.0-501B-A23B VQ
// GGUF", section "What stays native".
#include "common.cuh"
#include "internal.h"

namespace moe {

__device__ int g_status = 0;

namespace {

constexpr int kNW = 10;                  // warps per CTA
constexpr int kThreads = 32 * kNW;
constexpr int kCtasPerSm = 2;
constexpr int kSmemLimit = 113 * 1024;   // per CTA, two CTAs per SM

struct DecodeParams {
  const uint8_t* bank;
  uint64_t stride;
  uint64_t codes_off[2], scales_off[2], global_off[2];  // [0] gate (or down), [1] up
  int global_mode;
  int K, N;       // inputs per weight row, output rows per matrix
  int k;          // routing top-k: routed row r belongs to token r / k
  int xrows;      // activation rows staged per group (1 .. 8)
  const int4* groups;
  const int32_t* ngroups;
  const int32_t* perm;
  const void* xin;  // gate/up: bf16 x [T, K]; down: f32 h [R, K] (permuted rows)
  float* out;       // gate/up: h [R, N] = silu(G) * U; down: y [R, N] (permuted rows)
};

__host__ __device__ inline int xs_pitch(int K) { return K * 2 + 64; }   // = 64 (mod 128)
__host__ __device__ inline int off_red(int K, int xrows) { return (xrows * xs_pitch(K) + 127) & ~127; }
// + the prescale shifts of the group's activation rows (8 ints).
__host__ __device__ inline int smem_total(int K, int xrows) { return off_red(K, xrows) + 2 * kNW * 32 * 16 + 32; }

// Stage the group's activations as f16 in fragment order: inside each 128-wide K unit the 8
// values K0 .. K0+7 with K0 = 32*t + 8*i go to 16-byte chunk 4*i + t.  Row n is stored times
// 2^xsh[n], its power-of-two prescale into f16, taken first from its largest magnitude (one warp
// per row); callers bracket the call with CTA barriers.
template <bool GATEUP>
__device__ void fill_xs(const DecodeParams& p, uint8_t* xs, int* xsh, int row0, int nrows) {
  const int cpr = p.K / 8;  // chunks of 8 values per row
  const int pitch = xs_pitch(p.K);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int n = warp; n < nrows; n += kNW) {
    uint32_t m = 0;
    if (GATEUP) {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.xin) +
                                                        (size_t)(p.perm[row0 + n] / p.k) * p.K);
      for (int c = lane; c < cpr; c += 32) m = max(m, bf16x8_abs_max_bits(__ldg(src + c)));
    } else {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.xin) + (size_t)(row0 + n) * p.K);
      for (int c = lane; c < 2 * cpr; c += 32) {
        const float4 a = __ldg(src + c);
        m = max(m, max(max(f32_abs_bits(a.x), f32_abs_bits(a.y)), max(f32_abs_bits(a.z), f32_abs_bits(a.w))));
      }
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (lane == 0) xsh[n] = GATEUP ? prescale_shift_bf16(m) : prescale_shift_f32(m);
  }
  named_bar_sync(1, kThreads);
  for (int c = threadIdx.x; c < p.xrows * cpr; c += kThreads) {
    const int n = c / cpr, kk = (c - n * cpr) * 8;
    const int u = kk >> 7, q = kk & 127;
    uint4* dst = reinterpret_cast<uint4*>(xs + n * pitch + u * 256 + (((q & 31) >> 3) * 4 + (q >> 5)) * 16);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n < nrows) {
      const float f = exp2_int(xsh[n]);
      if (GATEUP) {
        const int t = p.perm[row0 + n] / p.k;
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(
            static_cast<const uint16_t*>(p.xin) + (size_t)t * p.K + kk));
        v.x = pack_f16x2(bf16_bits_to_f32(b.x & 0xFFFF) * f, bf16_bits_to_f32(b.x >> 16) * f);
        v.y = pack_f16x2(bf16_bits_to_f32(b.y & 0xFFFF) * f, bf16_bits_to_f32(b.y >> 16) * f);
        v.z = pack_f16x2(bf16_bits_to_f32(b.z & 0xFFFF) * f, bf16_bits_to_f32(b.z >> 16) * f);
        v.w = pack_f16x2(bf16_bits_to_f32(b.w & 0xFFFF) * f, bf16_bits_to_f32(b.w >> 16) * f);
      } else {
        const float4* src = reinterpret_cast<const float4*>(
            static_cast<const float*>(p.xin) + (size_t)(row0 + n) * p.K + kk);
        const float4 a = src[0], b = src[1];
        v = make_uint4(pack_f16x2(a.x * f, a.y * f), pack_f16x2(a.z * f, a.w * f), pack_f16x2(b.x * f, b.y * f),
                       pack_f16x2(b.z * f, b.w * f));
      }
    }
    *dst = v;
  }
}

// One thread's share of one unit of one item: 16 code bytes and 2 scale bytes of each of the
// MMA rows gid and gid + 8.
struct Frag {
  uint4 c0, c1;
  uint32_t s0, s1;
};

// Walks the (item, unit) steps of one warp.  All warps take the same number of steps per
// item (units beyond K are empty steps), so item boundaries line up across the CTA.
struct Cursor {
  int item, q, g, tile;
  const uint8_t* rec;
};

__device__ __forceinline__ uint32_t ld_u16_nc(const uint8_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_v4_stream(const uint8_t* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

template <bool GATEUP>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* xs = smem;
  float4* red = reinterpret_cast<float4*>(smem + off_red(p.K, p.xrows));
  int* xsh = reinterpret_cast<int*>(red + 2 * kNW * 32);     // [8] prescale shifts of the group's rows
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tid4 = lane & 3;
  const int tiles = GATEUP ? p.N / 8 : p.N / 16;
  const int items = *p.ngroups * tiles;
  const int per = items / (int)gridDim.x, rem = items % (int)gridDim.x;
  const int i0 = (int)blockIdx.x * per + min((int)blockIdx.x, rem);
  const int i1 = i0 + per + ((int)blockIdx.x < rem ? 1 : 0);
  if (i0 >= i1) return;
  const int units = p.K / 128;
  const int U = (units + kNW - 1) / kNW;           // steps per item
  const uint32_t rowb = p.K / 2, scb = p.K / 16;
  const uint64_t pol = policy_evict_first();

  // Per-thread byte offsets (inside a record) of rows gid and gid + 8 of tile 0.
  const uint64_t c0_off = p.codes_off[0] + (uint64_t)gid * rowb + tid4 * 16;
  const uint64_t s0_off = p.scales_off[0] + (uint64_t)gid * scb + tid4 * 2;
  const uint64_t c1_off = GATEUP ? p.codes_off[1] + (uint64_t)gid * rowb + tid4 * 16 : c0_off + 8 * rowb;
  const uint64_t s1_off = GATEUP ? p.scales_off[1] + (uint64_t)gid * scb + tid4 * 2 : s0_off + 8 * scb;
  const int tile_rows = GATEUP ? 8 : 16;

  auto start = [&](Cursor& c, int item) {
    c.item = item;
    c.q = 0;
    c.g = item / tiles;
    c.tile = item - c.g * tiles;
    c.rec = p.bank + (uint64_t)__ldg(&p.groups[c.g].x) * p.stride;
  };
  auto advance = [&](Cursor& c) {
    if (++c.q == U) {
      c.q = 0;
      ++c.item;
      if (++c.tile == tiles && c.item < i1) {
        c.tile = 0;
        ++c.g;
        c.rec = p.bank + (uint64_t)__ldg(&p.groups[c.g].x) * p.stride;
      }
    }
  };
  auto load = [&](const Cursor& c, Frag& f) {
    const int u = warp + kNW * c.q;
    if (c.item < i1 && u < units) {
      const uint64_t row = (uint64_t)c.tile * tile_rows;
      const uint8_t* b = c.rec + u * 64;
      f.c0 = ld_v4_stream(b + c0_off + row * rowb, pol);
      f.c1 = ld_v4_stream(b + c1_off + row * rowb, pol);
      const uint8_t* sb = c.rec + u * 8;
      f.s0 = ld_u16_nc(sb + s0_off + row * scb);
      f.s1 = ld_u16_nc(sb + s1_off + row * scb);
    }
  };

  const bool has_x = gid < p.xrows;
  const uint8_t* xrow = xs + (has_x ? gid : 0) * xs_pitch(p.K) + tid4 * 16;
  int cur_g = -1, row0 = 0, nrows = 0, j = 0;
  float gm0 = 0.0f, gm1 = 0.0f;
  float acc[2][4];

  auto compute = [&](const Cursor& c, const Frag& f) {
    if (c.q == 0) {
      if (c.g != cur_g) {
        named_bar_sync(1, kThreads);
        const int4 grp = p.groups[c.g];
        row0 = grp.y;
        nrows = grp.z;
        gm0 = global_mult(*reinterpret_cast<const float*>(c.rec + p.global_off[0]), p.global_mode);
        gm1 = GATEUP ? global_mult(*reinterpret_cast<const float*>(c.rec + p.global_off[1]), p.global_mode) : 0.0f;
        fill_xs<GATEUP>(p, xs, xsh, row0, nrows);
        named_bar_sync(1, kThreads);
        cur_g = c.g;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[0][i] = acc[1][i] = 0.0f;
    }
    const int u = warp + kNW * c.q;
    if (u < units) {
      uint4 xq[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        xq[i] = has_x ? *reinterpret_cast<const uint4*>(xrow + u * 256 + i * 64) : make_uint4(0, 0, 0, 0);
      const uint32_t hs0 = e4m3x2_to_f16x2((uint16_t)f.s0);
      const uint32_t hs1 = e4m3x2_to_f16x2((uint16_t)f.s1);
      const uint32_t w0[4] = {f.c0.x, f.c0.y, f.c0.z, f.c0.w};
      const uint32_t w1[4] = {f.c1.x, f.c1.y, f.c1.z, f.c1.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t sA = bcast_half(hs0, w >= 2), sB = bcast_half(hs1, w >= 2);
        uint32_t fa[4], fb[4];
        e2m1x8_to_f16x8(w0[w], fa);
        e2m1x8_to_f16x8(w1[w], fb);
        const uint32_t a0[4] = {hmul2(fa[0], sA), hmul2(fb[0], sB), hmul2(fa[1], sA), hmul2(fb[1], sB)};
        mma_16816(acc[0], a0, xq[w].x, xq[w].y);
        const uint32_t a1[4] = {hmul2(fa[2], sA), hmul2(fb[2], sB), hmul2(fa[3], sA), hmul2(fb[3], sB)};
        mma_16816(acc[1], a1, xq[w].z, xq[w].w);
      }
    }
    if (c.q == U - 1) {
      const int buf = j & 1;
      red[(buf * kNW + warp) * 32 + lane] =
          make_float4(acc[0][0] + acc[1][0], acc[0][1] + acc[1][1], acc[0][2] + acc[1][2], acc[0][3] + acc[1][3]);
      named_bar_sync(1, kThreads);
      if (warp == j % kNW) {
        float cs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int w = 0; w < kNW; ++w) {
          const float4 v = red[(buf * kNW + w) * 32 + lane];
          cs[0] += v.x, cs[1] += v.y, cs[2] += v.z, cs[3] += v.w;
        }
        // cs[0..1]: MMA row gid, token slots 2*tid4, 2*tid4+1; cs[2..3]: MMA row gid + 8.
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int n = 2 * tid4 + cc;
          if (n < nrows) {
            const float un = exp2_int(-xsh[n]);             // undo the row's prescale
            if (GATEUP) {
              p.out[(size_t)(row0 + n) * p.N + c.tile * 8 + gid] = silu_mul(cs[cc] * un * gm0, cs[2 + cc] * un * gm1);
            } else {
              float* o = p.out + (size_t)(row0 + n) * p.N;
              o[c.tile * 16 + gid] = cs[cc] * un * gm0;
              o[c.tile * 16 + gid + 8] = cs[2 + cc] * un * gm0;
            }
          }
        }
      }
      ++j;
    }
  };

  // Three-slot ring: loads run two steps ahead of the step being computed.
  const int S = (i1 - i0) * U;
  Cursor lc, cc;
  start(lc, i0);
  start(cc, i0);
  Frag fA, fB, fC;
  load(lc, fA);
  advance(lc);
  load(lc, fB);
  advance(lc);
  for (int s = 0; s < S; s += 3) {
    load(lc, fC);
    advance(lc);
    compute(cc, fA);
    advance(cc);
    if (s + 1 >= S) break;
    load(lc, fA);
    advance(lc);
    compute(cc, fB);
    advance(cc);
    if (s + 2 >= S) break;
    load(lc, fB);
    advance(lc);
    compute(cc, fC);
    advance(cc);
  }
}

template <bool GATEUP>
int launch(const DecodeParams& p, int num_sms, cudaStream_t s) {
  const int bytes = smem_total(p.K, p.xrows);
  if (bytes > kSmemLimit) return -(int)cudaErrorInvalidValue;
  cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(decode_kernel<GATEUP>), bytes);
  if (err != cudaSuccess) return -(int)err;
  decode_kernel<GATEUP><<<num_sms * kCtasPerSm, kThreads, bytes, s>>>(p);
  err = cudaGetLastError();
  return err == cudaSuccess ? 1 : -(int)err;
}

}  // namespace

size_t decode_smem_bytes(int K, int xrows, bool gateup) {
  (void)gateup;
  const int b = smem_total(K, xrows);
  return b <= kSmemLimit ? (size_t)b : 0;
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
  p.codes_off[1] = bank.codes_off[2];
  p.scales_off[0] = bank.scales_off[2];
  p.scales_off[1] = bank.scales_off[2];
  p.global_off[0] = bank.global_off[2];
  p.global_off[1] = bank.global_off[2];
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
