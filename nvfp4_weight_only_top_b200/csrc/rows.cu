// Decode path for one-row groups (an expert that received a single routed row): warp-per-row
// NVFP4 GEMV on CUDA cores.
//
// With one token, an MMA would waste 7/8 of its N = 8 columns, and mma.sync throughput on
// sm_100 caps such a kernel well below the HBM rate; here every lane works on real data.
// Work item = two weight rows of one expert: for gate/up the gate row and the up row of the
// same output (they share the activations, and SwiGLU is applied to the pair), for down two
// consecutive rows.  An item is
// 32 * UPL 16-byte units: lane l takes units l, l + 32, ... of the two rows laid end to end.
// Each warp walks a contiguous range of items; there is no block-level synchronisation.
//
// Per unit (32 weights of one row) a lane converts its 4 code words with cvt (E2M1 -> f16,
// exact), forms the two 16-input block dot products with packed f16 FMAs against the
// activations -- f16 at the lane's own K positions, staged once per group in the warp's slab
// of shared memory -- then adds e4m3(scale) x block sum in f32.  A warp butterfly adds the lanes'
// partial row sums; the global scale is applied once per row.  Code and scale loads are
// 128-bit / 16-bit streaming loads issued DEPTH - 1 items ahead through a register ring.
//
// Weight layout: page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit
// residents", section "What this pack holds"; SwiGLU in FP32: page "Beam-1.0-501B-A23B VQ
// GGUF", section "What stays native".
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {


struct RowParams {
  const uint8_t* bank;
  uint64_t stride;
  uint64_t codes_off[2], scales_off[2], global_off[2];   // matrix of row A, matrix of row B
  int global_mode;
  int K;            // inputs per row
  int N;            // rows per matrix
  int pair_rows;    // 1: item = row r of matrix A and row r of matrix B; 0: rows 2r, 2r+1 of A
  int k;            // routing top-k: routed row r belongs to token r / k
  int out_stride;   // floats per output row
  const int4* singles;
  const int32_t* nsingles;
  const int32_t* perm;
  const void* xin;  // gate/up: bf16 x [T, K]; down: f32 h [R, K]
  float* out;       // gate/up: h [R, N] = silu(G) * U; down: y [R, N]
};

template <int UPL>
struct RowFrag {
  uint4 c[UPL];
  uint32_t s[UPL];
};

__device__ __forceinline__ uint4 ld_v4_stream(const uint8_t* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

__device__ __forceinline__ uint32_t ld_u16_stream(const uint8_t* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t hadd2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t v) {
  float a, b;
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
      : "=f"(a), "=f"(b)
      : "r"(v));
  return make_float2(a, b);
}

// Stores the group's activations as f16 at the lane's own K positions in the warp's slab of
// shared memory.  Slot (m, q) of lane l -- the 8 values at K = kpos[m] + 8q .. +7 -- lives at
// 16-byte chunk (4m + q) * 32 + l, so a warp-wide 128-bit read of one slot is conflict-free.
// Each lane reads back only what it wrote itself.  The values are stored times 2^s, the
// power-of-two prescale into f16 taken from the row's largest magnitude (the lanes of the warp
// together cover the whole row: a first pass finds it); returns s.
template <int NX, bool GATEUP>
__device__ __forceinline__ int load_x(const RowParams& p, int prow, const int (&kpos)[NX], uint4* slab, int lane) {
  if (GATEUP) {
    const int t = __ldg(&p.perm[prow]) / p.k;
    const uint16_t* xrow = static_cast<const uint16_t*>(p.xin) + (size_t)t * p.K;
    uint32_t mx = 0;
#pragma unroll 1
    for (int m = 0; m < NX; ++m)
#pragma unroll
      for (int q = 0; q < 4; ++q)
        mx = max(mx, bf16x8_abs_max_bits(__ldg(reinterpret_cast<const uint4*>(xrow + kpos[m] + 8 * q))));
    const int sh = prescale_shift_bf16(__reduce_max_sync(0xFFFFFFFFu, mx));
    const float f = exp2_int(sh);
#pragma unroll
    for (int m = 0; m < NX; ++m)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(xrow + kpos[m] + 8 * q));
        slab[(4 * m + q) * 32 + lane] =
            make_uint4(pack_f16x2(bf16_bits_to_f32(b.x & 0xFFFF) * f, bf16_bits_to_f32(b.x >> 16) * f),
                       pack_f16x2(bf16_bits_to_f32(b.y & 0xFFFF) * f, bf16_bits_to_f32(b.y >> 16) * f),
                       pack_f16x2(bf16_bits_to_f32(b.z & 0xFFFF) * f, bf16_bits_to_f32(b.z >> 16) * f),
                       pack_f16x2(bf16_bits_to_f32(b.w & 0xFFFF) * f, bf16_bits_to_f32(b.w >> 16) * f));
      }
    return sh;
  } else {
    const float* hp = static_cast<const float*>(p.xin) + (size_t)prow * p.K;
    uint32_t mx = 0;
#pragma unroll 1
    for (int m = 0; m < NX; ++m)
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(hp + kpos[m] + 4 * q));
        mx = max(mx, max(max(f32_abs_bits(a.x), f32_abs_bits(a.y)), max(f32_abs_bits(a.z), f32_abs_bits(a.w))));
      }
    const int sh = prescale_shift_f32(__reduce_max_sync(0xFFFFFFFFu, mx));
    const float f = exp2_int(sh);
#pragma unroll
    for (int m = 0; m < NX; ++m)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(hp + kpos[m] + 8 * q));
        const float4 b = __ldg(reinterpret_cast<const float4*>(hp + kpos[m] + 8 * q + 4));
        slab[(4 * m + q) * 32 + lane] = make_uint4(pack_f16x2(a.x * f, a.y * f), pack_f16x2(a.z * f, a.w * f),
                                                   pack_f16x2(b.x * f, b.y * f), pack_f16x2(b.z * f, b.w * f));
      }
    return sh;
  }
}

// Position of a warp inside its item range: one-row group g, item t within the group.
struct Cursor {
  int g, t;
  const uint8_t* rec;
  int prow;
};

// UPL units per lane per item; NX distinct K units per lane (UPL / 2 when the two rows share
// K positions, else UPL); DEPTH items in the register ring; WARPS warps per CTA (one CTA per
// SM; 8 warps allow 255 registers per thread, 12 allow 168: each SM sub-partition holds 16K).
template <int UPL, int NX, int DEPTH, int WARPS, bool GATEUP>
__global__ void __launch_bounds__(32 * WARPS, 1) rows_kernel(const RowParams p) {
  const int lane = threadIdx.x & 31;
  const int gw = (int)blockIdx.x * WARPS + (int)(threadIdx.x >> 5);
  const int nw = (int)gridDim.x * WARPS;
  const int ipg = p.pair_rows ? p.N : p.N / 2;    // items per group
  const int items = *p.nsingles * ipg;
  const int per = items / nw, rem = items % nw;
  const int w0 = gw * per + min(gw, rem);
  const int w1 = w0 + per + (gw < rem ? 1 : 0);
  if (w0 >= w1) return;
  const int urow = p.K / 32;                       // 32-wide units per row
  const uint32_t rowb = p.K / 2, scb = p.K / 16;
  const uint64_t pol = policy_evict_first();

  // The lane's units: row rb[m] (0 = A, 1 = B) of the item, x slot xi(m), byte offsets from
  // the start of that row.
  // Unit m of the lane is unit cu = lane + 32 m of the item: row cu / urow (with pair rows,
  // NX < UPL, that is m >= NX), 32-wide K unit cu % urow of that row.
  auto row_of = [&](int m) { return NX < UPL ? (m >= NX ? 1 : 0) : (lane + 32 * m) / urow; };
  auto unit_of = [&](int m) {
    const int cu = lane + 32 * (NX < UPL ? m % NX : m);
    return NX < UPL ? cu : cu - row_of(m) * urow;
  };
  int kpos[NX];
#pragma unroll
  for (int m = 0; m < NX; ++m) kpos[m] = 32 * unit_of(m);

  auto open = [&](Cursor& c, int it) {
    c.g = it / ipg;
    c.t = it - c.g * ipg;
    const int4 grp = __ldg(&p.singles[c.g]);
    c.rec = p.bank + (uint64_t)grp.x * p.stride;
    c.prow = grp.y;
  };
  auto next = [&](Cursor& c, int it_next) {
    if (++c.t == ipg && it_next < w1) open(c, it_next);
  };
  auto row_a = [&](int t) { return p.pair_rows ? t : 2 * t; };
  auto row_b = [&](int t) { return p.pair_rows ? t : 2 * t + 1; };
  auto load = [&](const Cursor& c, int it, RowFrag<UPL>& f) {
    if (it >= w1) return;
    const uint8_t* ca = c.rec + p.codes_off[0] + (uint64_t)row_a(c.t) * rowb;
    const uint8_t* cbp = c.rec + p.codes_off[1] + (uint64_t)row_b(c.t) * rowb;
    const uint8_t* sa = c.rec + p.scales_off[0] + (uint64_t)row_a(c.t) * scb;
    const uint8_t* sbp = c.rec + p.scales_off[1] + (uint64_t)row_b(c.t) * scb;
#pragma unroll
    for (int m = 0; m < UPL; ++m) {
      const int ku = unit_of(m), r = row_of(m);
      f.c[m] = ld_v4_stream((r ? cbp : ca) + ku * 16, pol);
      f.s[m] = ld_u16_stream((r ? sbp : sa) + ku * 2);
    }
  };

  extern __shared__ __align__(16) uint4 x_slabs[];
  uint4* slab = x_slabs + (threadIdx.x >> 5) * (NX * 4 * 32);   // this warp's activations
  int cur_g = -1, xsh = 0;          // current group, prescale shift of its activations
  float gmA = 0.0f, gmB = 0.0f;     // global multipliers

  auto compute = [&](const Cursor& c, const RowFrag<UPL>& f) {
    if (c.g != cur_g) {
      cur_g = c.g;
      gmA = global_mult(__ldg(reinterpret_cast<const float*>(c.rec + p.global_off[0])), p.global_mode);
      gmB = global_mult(__ldg(reinterpret_cast<const float*>(c.rec + p.global_off[1])), p.global_mode);
      xsh = load_x<NX, GATEUP>(p, c.prow, kpos, slab, lane);
      __syncwarp();
    }
    float accA = 0.0f, accB = 0.0f;
#pragma unroll
    for (int m = 0; m < UPL; ++m) {
      const uint4* xs = slab + 4 * (m % NX) * 32 + lane;
      const uint4 xa = xs[0], xb = xs[32], xc = xs[64], xd = xs[96];
      const uint32_t x[16] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w,
                              xc.x, xc.y, xc.z, xc.w, xd.x, xd.y, xd.z, xd.w};
      const float2 sf = f16x2_to_float2(e4m3x2_to_f16x2((uint16_t)f.s[m]));
      uint32_t e0[4], e1[4], e2[4], e3[4];
      e2m1x8_to_f16x8(f.c[m].x, e0);
      e2m1x8_to_f16x8(f.c[m].y, e1);
      e2m1x8_to_f16x8(f.c[m].z, e2);
      e2m1x8_to_f16x8(f.c[m].w, e3);
      // block 0 = words 0, 1 and block 1 = words 2, 3; two interleaved chains per block
      uint32_t p0 = hfma2(e0[0], x[0], 0u), p0b = hfma2(e0[1], x[1], 0u);
      uint32_t p1 = hfma2(e2[0], x[8], 0u), p1b = hfma2(e2[1], x[9], 0u);
      p0 = hfma2(e0[2], x[2], p0), p0b = hfma2(e0[3], x[3], p0b);
      p1 = hfma2(e2[2], x[10], p1), p1b = hfma2(e2[3], x[11], p1b);
      p0 = hfma2(e1[0], x[4], p0), p0b = hfma2(e1[1], x[5], p0b);
      p1 = hfma2(e3[0], x[12], p1), p1b = hfma2(e3[1], x[13], p1b);
      p0 = hfma2(e1[2], x[6], p0), p0b = hfma2(e1[3], x[7], p0b);
      p1 = hfma2(e3[2], x[14], p1), p1b = hfma2(e3[3], x[15], p1b);
      const float2 a = f16x2_to_float2(hadd2(p0, p0b)), b = f16x2_to_float2(hadd2(p1, p1b));
      const float part = fmaf(sf.x, a.x + a.y, sf.y * (b.x + b.y));
      if (row_of(m) == 0)
        accA += part;
      else
        accB += part;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      accA += __shfl_xor_sync(0xFFFFFFFFu, accA, off);
      accB += __shfl_xor_sync(0xFFFFFFFFu, accB, off);
    }
    const float un = exp2_int(-xsh);
    if (GATEUP) {
      if (lane == 0) p.out[(size_t)c.prow * p.out_stride + c.t] = silu_mul(accA * un * gmA, accB * un * gmB);
    } else if (lane < 2) {
      p.out[(size_t)c.prow * p.out_stride + (lane == 0 ? row_a(c.t) : row_b(c.t))] =
          lane == 0 ? accA * un * gmA : accB * un * gmB;
    }
  };

  // Register ring of DEPTH items: loads run DEPTH - 1 items ahead of the one computed.
  RowFrag<UPL> f[DEPTH];
  Cursor lc, cc;
  open(lc, w0);
  open(cc, w0);
#pragma unroll
  for (int d = 0; d < DEPTH - 1; ++d) {
    load(lc, w0 + d, f[d]);
    next(lc, w0 + d + 1);
  }
  for (int it = w0; it < w1; it += DEPTH) {
#pragma unroll
    for (int d = 0; d < DEPTH; ++d) {
      if (it + d >= w1) break;
      load(lc, it + d + DEPTH - 1, f[(d + DEPTH - 1) % DEPTH]);
      next(lc, it + d + DEPTH);
      compute(cc, f[d]);
      next(cc, it + d + 1);
    }
  }
}

// Units per lane for an item of two rows of width K, or 0 if K does not split evenly.
int units_per_lane(int K) { return (K % 512 == 0 && K / 512 <= 10) ? K / 512 : 0; }

template <int UPL, int NX, int DEPTH, int WARPS, bool GATEUP>
cudaError_t launch_one(const RowParams& p, int num_sms, cudaStream_t s) {
  const int smem = WARPS * NX * 4 * 32 * 16;
  cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(rows_kernel<UPL, NX, DEPTH, WARPS, GATEUP>), smem);
  if (err != cudaSuccess) return err;
  rows_kernel<UPL, NX, DEPTH, WARPS, GATEUP><<<num_sms, 32 * WARPS, smem, s>>>(p);
  return cudaGetLastError();
}

// gate/up: the gate row and the up row of an item share K positions (NX = UPL / 2);
// down: two consecutive rows, each lane at its own K positions (NX = UPL).
int launch_gateup_rows(const RowParams& p, int num_sms, cudaStream_t s) {
  cudaError_t err = cudaErrorInvalidValue;
  switch (units_per_lane(p.K)) {
    case 2: err = launch_one<2, 1, 4, 12, true>(p, num_sms, s); break;
    case 4: err = launch_one<4, 2, 3, 12, true>(p, num_sms, s); break;
    case 6: err = launch_one<6, 3, 3, 8, true>(p, num_sms, s); break;
    case 8: err = launch_one<8, 4, 3, 8, true>(p, num_sms, s); break;
    case 10: err = launch_one<10, 5, 2, 8, true>(p, num_sms, s); break;
    default: break;
  }
  return err == cudaSuccess ? 1 : -(int)err;
}

int launch_down_rows(const RowParams& p, int num_sms, cudaStream_t s) {
  cudaError_t err = cudaErrorInvalidValue;
  switch (units_per_lane(p.K)) {
    case 1: err = launch_one<1, 1, 4, 12, false>(p, num_sms, s); break;
    case 3: err = launch_one<3, 3, 4, 8, false>(p, num_sms, s); break;
    case 5: err = launch_one<5, 5, 2, 8, false>(p, num_sms, s); break;
    default: break;
  }
  return err == cudaSuccess ? 1 : -(int)err;
}

}  // namespace

bool rows_supported(int K, bool gateup) {
  const int upl = units_per_lane(K);
  if (gateup) return K % 1024 == 0 && (upl == 2 || upl == 4 || upl == 6 || upl == 8 || upl == 10);
  return upl == 1 || upl == 3 || upl == 5;
}

int launch_rows_gateup(const BankView& bank, const uint16_t* x, int k, const RouteBufs& rb,
                       float* h, int num_sms, cudaStream_t s) {
  RowParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  for (int m = 0; m < 2; ++m) {
    p.codes_off[m] = bank.codes_off[m];
    p.scales_off[m] = bank.scales_off[m];
    p.global_off[m] = bank.global_off[m];
  }
  p.global_mode = bank.global_mode;
  p.K = bank.H;
  p.N = bank.I;
  p.pair_rows = 1;
  p.k = k;
  p.out_stride = bank.I;
  p.singles = rb.singles;
  p.nsingles = rb.nsingles;
  p.perm = rb.perm;
  p.xin = x;
  p.out = h;
  return launch_gateup_rows(p, num_sms, s);
}

int launch_rows_down(const BankView& bank, const float* h, const RouteBufs& rb, float* y,
                     int num_sms, cudaStream_t s) {
  RowParams p{};
  p.bank = bank.base;
  p.stride = bank.stride;
  p.codes_off[0] = p.codes_off[1] = bank.codes_off[2];
  p.scales_off[0] = p.scales_off[1] = bank.scales_off[2];
  p.global_off[0] = p.global_off[1] = bank.global_off[2];
  p.global_mode = bank.global_mode;
  p.K = bank.I;
  p.N = bank.H;
  p.pair_rows = 0;
  p.k = 1;
  p.out_stride = bank.H;
  p.singles = rb.singles;
  p.nsingles = rb.nsingles;
  p.perm = rb.perm;
  p.xin = h;
  p.out = y;
  return launch_down_rows(p, num_sms, s);
}

}  // namespace moe
