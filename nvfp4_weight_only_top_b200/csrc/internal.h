// Internal launch interface between the C ABI (moe_nvfp4.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Routing outputs and scratch, all device pointers into one workspace.
struct RouteBufs {
  int32_t* ids;        // [T, k]
  float* w;            // [T, k]
  int32_t* counts;     // [E]
  int32_t* offsets;    // [E + 1]
  int32_t* perm;       // [T * k]
  int32_t* inv;        // [T * k]
  int4* groups;        // [max_groups]: (expert, first permuted row, rows, 0), rows >= 2
  int32_t* ngroups;    // [1]
  int4* singles;       // [max_groups]: (expert, permuted row, 1, 0): one-row groups
  int32_t* nsingles;   // [1]
  int32_t* chunk_counts;  // [nchunks, E]: kRouteChunk tokens per chunk (T > kRouteChunk), or
                          // kSmallTok tokens per chunk (T <= kRouteChunk)
  unsigned* done;         // [1]: CTAs of the one-launch router that finished (reset by its last)
  int group_rows;      // rows per group (decode token tile)
  int split_singles;   // 1: one-row groups go to `singles`; 0: they stay in `groups`
  int expert_major;    // 1: each expert's groups are listed together (full, then its partial);
                       // 0: all full groups first, then the partial ones
};

// Tokens per routing chunk in the multi-launch router, used for T > kRouteChunk; up to
// kRouteChunk tokens are routed in one launch, by one CTA up to kOneCtaTokens, else kSmallTok
// tokens (one per warp) per CTA.
constexpr int kRouteChunk = 64;
constexpr int kSmallTok = 8;
// Up to this many tokens one CTA routes them alone (measured faster than the one-launch
// multi-CTA router below about 32 tokens, which pays for a memset and the last-CTA hand-off).
constexpr int kOneCtaTokens = 32;

inline int route_chunks(int64_t T) { return (int)((T + kRouteChunk - 1) / kRouteChunk); }
// Ints of RouteBufs::chunk_counts the router needs for T tokens and E experts.
inline size_t route_chunk_ints(int64_t T, int E) {
  return T > kRouteChunk ? (size_t)route_chunks(T) * E : (size_t)((T + kSmallTok - 1) / kSmallTok) * E;
}
inline int64_t max_groups(int64_t R, int E, int group_rows) {
  int64_t g = (R + group_rows - 1) / group_rows + E;
  return g < R ? g : R;
}

// Launches the router and the permutation; returns the number of kernels launched or a
// negative cudaError_t.
int launch_route(const float* logits, int64_t T, int E, int k, const RouteBufs& b,
                 cudaStream_t s);

// Routing of rows whose expert ids are given (k = 1, weights 1): ids [R] of the caller; ids
// outside [0, E) mark padding rows, placed after all expert rows and in no group.  chunk_counts
// must hold route_chunks(R) * (E + 1) ints.  Returns the number of kernels launched.
int launch_route_ids(const int32_t* rows, int64_t R, int E, const RouteBufs& b, cudaStream_t s);

struct BankView {
  const uint8_t* base;
  uint64_t stride;
  uint64_t codes_off[3], scales_off[3], global_off[3];
  int global_mode;
  int E, H, I;
};

// Decode path, groups of 2..8 rows: grouped NVFP4 GEMM on mma.sync.
// gate/up: h [R, I] f32 = silu(x Wg^T gg) * (x Wu^T gu) for every routed row.
int launch_decode_gateup(const BankView& bank, const uint16_t* x, int k, const RouteBufs& rb,
                         int xrows, float* h, int num_sms, cudaStream_t s);
// down: y [R, H] f32 = h Wd^T gd for every routed row.
int launch_decode_down(const BankView& bank, const float* h, const RouteBufs& rb, int xrows,
                       float* y, int num_sms, cudaStream_t s);

// Decode path, one-row groups: warp-per-row NVFP4 GEMV on CUDA cores (same outputs).
bool rows_supported(int K, bool gateup);
int launch_rows_gateup(const BankView& bank, const uint16_t* x, int k, const RouteBufs& rb,
                       float* h, int num_sms, cudaStream_t s);
int launch_rows_down(const BankView& bank, const float* h, const RouteBufs& rb, float* y,
                     int num_sms, cudaStream_t s);

// out [T, H] bf16 = sum_j w[t, j] * y[inv[t*k+j]]; optional x_next = bf16(x + out).
int launch_combine(const float* y, const float* w, const int32_t* inv, int64_t T, int k, int H,
                   const uint16_t* x, uint16_t* out, uint16_t* x_next, cudaStream_t s);

// y_rows [R, H] f32 = y[inv[r]] for rows with ids[r] >= 0, zero for the others.
int launch_unpermute(const float* y, const int32_t* inv, const int32_t* ids, int64_t R, int H, float* y_rows,
                     cudaStream_t s);
size_t decode_smem_bytes(int K, int xrows, bool gateup);

// Decode of larger batches on the router's groups (up to 8 routed rows of one expert, group_rows
// 8, singles kept in the groups): persistent gate/up + SwiGLU and down kernels (bulk-TMA stage
// ring, mma.sync with the group's activations as N = 8).  h [R, I] and y [R, H] f32 in permuted
// row order, as the combine kernel reads them.
bool grouped_supported(int H, int I);
int launch_grouped_gateup(const BankView& bank, const uint16_t* x, int k, const RouteBufs& rb, float* h, int num_sms,
                          cudaStream_t s);
int launch_grouped_down(const BankView& bank, const float* h, const RouteBufs& rb, float* y, int num_sms,
                        cudaStream_t s);

// Decode of a single token: route, gate/up, down and combine in one persistent kernel.  h [k, I]
// and y [k, H] are f32 scratch; its completion counters come from a library-owned pool of
// self-clearing counter sets on device dev (the current device).
bool decode1_supported(int H, int I, int k, int E, int num_sms);
int launch_decode1(const BankView& bank, const float* logits, int k, const uint16_t* x, uint16_t* out,
                   uint16_t* x_next, float* h, float* y, int32_t* ids, float* w, int dev, int num_sms,
                   cudaStream_t s);
int decode1_reset_pool();

// Decode of 2 .. 16 tokens (T k <= number of SMs) in one persistent kernel after the router:
// gate/up, down and combine over one slot per routed row, in the router's permutation order.
// h [T k, I] and y [T k, H] are f32 scratch; counters as for the single-token kernel.
bool decode_few_supported(int H, int I, int k, int T, int num_sms);
int launch_decode_few(const BankView& bank, int T, int k, const uint16_t* x, uint16_t* out, uint16_t* x_next,
                      float* h, float* y, const int32_t* ids, const float* w, const int32_t* perm,
                      const int32_t* inv, int dev, int num_sms, cudaStream_t s);
int decode_few_reset_pool();

// Prefill path: grouped NVFP4 GEMM on tcgen05 tensor cores, groups of up to kPrefillRows rows.
constexpr int kPrefillRows = 256;
bool prefill_supported(int H, int I);
// xp [R, H] bf16 = x[perm[r] / k] for every routed row r (expert order).
int launch_gather(const uint16_t* x, const int32_t* perm, int k, int64_t R, int H, void* xp, cudaStream_t s);
// xp [T k, H] f16: row inv[t k + j] = x[t] 2^s_t (s_t the token's prescale), colscale there = 2^-s_t.
int launch_gather_f16(const uint16_t* x, const int32_t* inv, int k, int64_t T, int H, void* xp, float* colscale,
                      cudaStream_t s);
// hb [R, I] bf16 = silu(xp Wg^T gg) * (xp Wu^T gu); with colscale, xp holds prescaled f16 rows
// (F16 MMA operands) whose results are multiplied by colscale[r], else bf16 rows.
// tile_ctr: a counter zeroed before the launch (tiles are handed out dynamically).
int launch_prefill_gateup(const BankView& bank, const void* xp, const float* colscale, int64_t R, const RouteBufs& rb,
                          void* hb, unsigned* tile_ctr, int num_sms, cudaStream_t s);
// y [R, H] f32 = hb Wd^T gd.
int launch_prefill_down(const BankView& bank, const void* hb, int64_t R, const RouteBufs& rb, float* y,
                        unsigned* tile_ctr, int num_sms, cudaStream_t s);

// Prefill path on CTA pairs (tcgen05 cta_group::2, M = 256): the same outputs as
// launch_prefill_gateup / launch_prefill_down.  prefill2_pairs: pairs resident at once (0: not
// available on this device).
int prefill2_pairs(int num_sms);
int launch_prefill2_gateup(const BankView& bank, const void* xp, const float* colscale, int64_t R,
                           const RouteBufs& rb, void* hb, int pairs, cudaStream_t s);
int launch_prefill2_down(const BankView& bank, const void* hb, int64_t R, const RouteBufs& rb, float* y, int pairs,
                         cudaStream_t s);

// W4A4 path (NVFP4 activations on tcgen05 kind::mxf4nvf4), groups of up to kW4A4Rows rows.
constexpr int kW4A4Rows = 128;
bool w4a4_supported(int H, int I);
// Optional outputs of the gate/up kernel in slot order (row perm[r]); NULL members are skipped.
struct W4A4Taps {
  float* h;                // [R][I] f32, h before quantization
  uint8_t* h_codes;        // [R][I/2]
  uint8_t* h_scales;       // [R][I/16]
};
// x[perm[r] / k] quantized with act_scales[2 e] (e the row's expert): codes [R][H/2], scales
// [R][H/16] in expert order, and in slot order too when tap_codes is not NULL.
int launch_w4a4_quant_x(const uint16_t* x, const RouteBufs& rb, int k, int64_t R, int H, const float* act_scales,
                        uint8_t* codes, uint8_t* scales, uint8_t* tap_codes, uint8_t* tap_scales, cudaStream_t s);
// h = silu(xq Wg^T gg sx) * (xq Wu^T gu sx), quantized with act_scales[2 e + 1] into h_codes [R][I/2]
// and h_scales [R][I/16] (expert order).  tile_ctr: a counter zeroed before the launch.
int launch_w4a4_gateup(const BankView& bank, const float* act_scales, const uint8_t* x_codes, const uint8_t* x_scales,
                       int64_t R, const RouteBufs& rb, uint8_t* h_codes, uint8_t* h_scales, const W4A4Taps& taps,
                       unsigned* tile_ctr, int num_sms, cudaStream_t s);
// y [R][H] f32 = hq Wd^T gd sh.
int launch_w4a4_down(const BankView& bank, const float* act_scales, const uint8_t* h_codes, const uint8_t* h_scales,
                     int64_t R, const RouteBufs& rb, float* y, unsigned* tile_ctr, int num_sms, cudaStream_t s);

// Expert parallelism over peer memory (ep.cu).  Ranks G <= kEpMaxRanks; the plan writes dst_off [E]
// and recv_ids [recv_rows]; dispatch and combine take G peer pointers (host array).
constexpr int kEpMaxRanks = 64;
size_t ep_plan_smem_bytes(int E);
int launch_ep_plan(const int32_t* C, int G, int E, int rank, int layout, int32_t* dst_off, int32_t* recv_ids,
                   int64_t recv_rows, cudaStream_t s);
bool ep_move_supported(int H);
int launch_ep_dispatch(const uint16_t* x, int64_t T, int k, int H, const int32_t* ids, const int32_t* inv,
                       const int32_t* offsets, const int32_t* dst_off, int El, int64_t cap, void* const* recv, int G,
                       int num_sms, cudaStream_t s);
int launch_ep_combine(int64_t T, int k, int H, const int32_t* ids, const float* w, const int32_t* inv,
                      const int32_t* offsets, const int32_t* dst_off, int El, int64_t cap, const float* const* ys,
                      int G, const uint16_t* x, uint16_t* out, uint16_t* x_next, cudaStream_t s);

// Tiled tensor map over a byte tensor of the given rank (dims innermost first, strides in bytes
// of dims 1.., box sizes); 0 or a negative cudaError_t.
int make_tensor_map(CUtensorMap* map, int rank, const void* base, const uint64_t* dims, const uint64_t* strides,
                    const uint32_t* box, CUtensorMapSwizzle swizzle);

// NVFP4 encoder: n projections [n, out_f, in_f] of BF16 weights -> codes, block scales and the
// stored global of projection i at dst + i * stride + {codes_off, scales_off, global_off}.
// Returns the number of kernels launched or a negative cudaError_t.
int launch_encode(const uint16_t* w, int64_t n, int out_f, int in_f, int global_mode, uint8_t* dst, uint64_t stride,
                  uint64_t codes_off, uint64_t scales_off, uint64_t global_off, int num_sms, cudaStream_t s);

// Sets a kernel's dynamic shared-memory limit on the current device, once per (kernel, device,
// size): the attribute call costs host time on every launch otherwise.
cudaError_t set_smem_limit(const void* kernel, int bytes);

// C-ABI bridge (moe_nvfp4.cu): status and message of the calling host thread, the current
// device (sm_100 check, SM count).
int api_fail(int code, const char* msg);
void api_set_launches(int n);          // moe_nvfp4_last_launch_count of the calling thread
int api_cuda_fail(int err, const char* what);
int api_device(int* dev, int* sms);

}  // namespace moe
