// C ABI of the NVFP4 weight-only routed-expert MoE layer: host-side validation, workspace
// management and the launch sequence (route -> expert GEMMs -> combine).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <memory>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "moe_nvfp4.h"

namespace {

thread_local std::string t_last_error;
thread_local int t_last_launches = 0;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MOE_NVFP4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct DeviceInfo {
  int sms = 0;
  int major = 0;
  int smem_optin = 0;
};

std::mutex g_mu;
std::vector<DeviceInfo> g_info;

struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::vector<Workspace> g_ws;

// Staging of moe_nvfp4_forward_host: x and the logits go to the device in one copy, through a
// pinned host buffer (in) into one device buffer (x at 0, logits at the next 256-byte boundary).
// A captured small host call (copy in, layer, copy out) for one (T, k, bank) and the staging and
// workspace buffers it was captured with; replayed with one graph launch.
struct HostGraph {
  int64_t T = 0;
  int k = 0;
  moe_nvfp4_bank bank{};
  const void* in_dev = nullptr;
  const void* in_host = nullptr;
  const void* out = nullptr;
  const void* out_host = nullptr;
  const void* ws = nullptr;
  cudaGraphExec_t exec = nullptr;
  int launches = 0;
  uint64_t used = 0;
};
struct HostStage {
  void* in_dev = nullptr;      // x | logits
  void* in_host = nullptr;     // pinned x | logits
  void* out = nullptr;
  void* out_host = nullptr;    // pinned out (graph replays)
  size_t in_bytes = 0, out_bytes = 0, out_host_bytes = 0;
  cudaStream_t capture = nullptr;
  std::vector<HostGraph> graphs;
  uint64_t tick = 0;
};
// One record per device, held by pointer so that growing the vector for another device never
// moves a record a caller is using.
std::vector<std::unique_ptr<HostStage>> g_stage;

int current_device(int* dev, DeviceInfo* info) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return fail(MOE_NVFP4_ERR_UNSUPPORTED, "no CUDA device: %s", cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(g_mu);
  if ((int)g_info.size() <= *dev) {
    g_info.resize(*dev + 1);
    g_ws.resize(*dev + 1);
    g_stage.resize(*dev + 1);
  }
  if (!g_stage[*dev]) g_stage[*dev].reset(new HostStage());
  DeviceInfo& d = g_info[*dev];
  if (d.sms == 0) {
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, *dev);
    cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, *dev);
    cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, *dev);
  }
  *info = d;
  if (d.major != 10)
    return fail(MOE_NVFP4_ERR_UNSUPPORTED, "device %d has compute capability %d.x; this library needs sm_100",
                *dev, d.major);
  return MOE_NVFP4_OK;
}

// Sizes of the workspace sub-buffers, each 256-byte aligned.
struct WsLayout {
  size_t ids, w, counts, offsets, perm, inv, groups, ngroups, singles, nsingles, chunk_counts, done, bar, h, y, total;
};

size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

// given_ids: the routing of an experts-only call (rows with given expert ids), whose chunk
// counts carry a padding bin and exist for every R.
WsLayout ws_layout(int64_t T, int E, int k, int H, int I, int path, bool given_ids = false) {
  (void)path;
  WsLayout L{};
  const size_t R = (size_t)T * k;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += up256(bytes);
    return at;
  };
  L.ids = take(R * 4);
  L.w = take(R * 4);
  L.counts = take((size_t)E * 4);
  L.offsets = take((size_t)(E + 1) * 4);
  L.perm = take(R * 4);
  L.inv = take(R * 4);
  L.groups = take((size_t)moe::max_groups((int64_t)R, E, 8) * 16);
  L.ngroups = take(4);
  L.singles = take((size_t)E * 16);
  L.nsingles = take(4);
  L.chunk_counts = take(given_ids ? (size_t)moe::route_chunks(T) * (E + 1) * 4 : moe::route_chunk_ints(T, E) * 4);
  L.done = take(4);
  L.bar = take(2 * sizeof(unsigned));        // tile counters of the tensor-core path
  L.h = take(R * (size_t)I * 4);
  L.y = take(R * (size_t)H * 4);
  L.total = o;
  return L;
}

int check_bank(const moe_nvfp4_bank* b) {
  if (!b) return fail(MOE_NVFP4_ERR_INVALID_ARG, "bank is NULL");
  if (!b->base_dev) return fail(MOE_NVFP4_ERR_INVALID_ARG, "bank->base_dev is NULL");
  if (b->num_experts < 1 || b->num_experts > 1024)
    return fail(MOE_NVFP4_ERR_UNSUPPORTED, "num_experts %d outside 1..1024", b->num_experts);
  if (b->hidden < 128 || b->hidden % 128 || b->intermediate < 128 || b->intermediate % 128)
    return fail(MOE_NVFP4_ERR_UNSUPPORTED, "hidden %d and intermediate %d must be positive multiples of 128",
                b->hidden, b->intermediate);
  if (b->hidden > 8192 || b->intermediate > 8192)
    return fail(MOE_NVFP4_ERR_UNSUPPORTED, "hidden and intermediate are limited to 8192");
  if (b->global_mode != 0 && b->global_mode != 1)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "global_mode %d is not 0 or 1", b->global_mode);
  if (!aligned(b->base_dev, 16) || b->record_stride % 16)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "bank base and record_stride must be 16-byte aligned");
  const uint64_t H = b->hidden, I = b->intermediate;
  for (int p = 0; p < 3; ++p) {
    if (b->codes_off[p] % 16 || b->scales_off[p] % 16 || b->global_off[p] % 4)
      return fail(MOE_NVFP4_ERR_INVALID_ARG, "projection %d offsets misaligned (codes/scales 16 B, global 4 B)", p);
    if (b->codes_off[p] + H * I / 2 > b->record_stride || b->scales_off[p] + H * I / 16 > b->record_stride ||
        b->global_off[p] + 4 > b->record_stride)
      return fail(MOE_NVFP4_ERR_INVALID_ARG, "projection %d does not fit in record_stride", p);
  }
  return MOE_NVFP4_OK;
}

moe::BankView view_of(const moe_nvfp4_bank* b) {
  moe::BankView v;
  v.base = static_cast<const uint8_t*>(b->base_dev);
  v.stride = b->record_stride;
  for (int p = 0; p < 3; ++p) {
    v.codes_off[p] = b->codes_off[p];
    v.scales_off[p] = b->scales_off[p];
    v.global_off[p] = b->global_off[p];
  }
  v.global_mode = b->global_mode;
  v.E = b->num_experts;
  v.H = b->hidden;
  v.I = b->intermediate;
  return v;
}

// Decode kernels for more than one token, for comparisons: MOE_NVFP4_DECODE=grouped takes the
// grouped kernels for every T > 1 that their shapes allow, =rows the older row and mma.sync group
// kernels; unset, 2 .. 11 tokens take the few-token kernel and larger batches the grouped kernels.
enum { kDecodeDefault = 0, kDecodeGrouped = 1, kDecodeRows = 2 };
constexpr int64_t kGroupedMinT = 12;     // fewest tokens the grouped kernels take by default
int decode_kernel_choice() {
  static const int v = [] {
    const char* s = getenv("MOE_NVFP4_DECODE");
    if (s && strcmp(s, "grouped") == 0) return (int)kDecodeGrouped;
    if (s && strcmp(s, "rows") == 0) return (int)kDecodeRows;
    return (int)kDecodeDefault;
  }();
  return v;
}

// Prefill kernel: the single-CTA kernel; MOE_NVFP4_PREFILL=pair selects the CTA-pair kernel
// (cta_group::2), which computes the same result (see prefill2.cu).
bool prefill_pair_kernel() {
  static const bool v = [] {
    const char* s = getenv("MOE_NVFP4_PREFILL");
    return s && strcmp(s, "pair") == 0;
  }();
  return v;
}

bool sync_each_kernel() {
  static const bool on = [] {
    const char* s = getenv("MOE_NVFP4_SYNC");
    return s && s[0] == '1';
  }();
  return on;
}

// Per-thread kernel timing (moe_nvfp4_profile_begin / _end).
struct ProfPair {
  int kind;
  cudaEvent_t a, b;
};
thread_local bool t_prof_on = false;
thread_local std::vector<ProfPair> t_prof;

cudaEvent_t prof_event() {
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// While a stream captures, an event record only becomes a timing node of the graph when it
// is recorded as an external event.
void prof_record(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(s, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
  else
    cudaEventRecord(e, s);
}

void prof_before(int kind, cudaStream_t s) {
  if (!t_prof_on) return;
  ProfPair p{kind, prof_event(), prof_event()};
  prof_record(p.a, s);
  t_prof.push_back(p);
}

void prof_after(cudaStream_t s) {
  if (!t_prof_on || t_prof.empty()) return;
  prof_record(t_prof.back().b, s);
}

int after_launch(int rc, cudaStream_t s, const char* what, int* count) {
  prof_after(s);
  if (rc < 0) return cuda_fail((cudaError_t)(-rc), what);
  *count += rc;
  if (sync_each_kernel()) {
    const cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, what);
  }
  return MOE_NVFP4_OK;
}

// Makes sure the internal workspace of `dev` holds `bytes`.
int ensure_workspace(int dev, size_t bytes, cudaStream_t s, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& w = g_ws[dev];
  if (w.bytes < bytes) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &cs);
    if (cs != cudaStreamCaptureStatusNone)
      return fail(MOE_NVFP4_ERR_WORKSPACE,
                  "internal workspace must grow to %zu bytes while the stream is capturing; run once "
                  "outside capture or pass a workspace",
                  bytes);
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "synchronise before workspace growth");
    if (w.ptr) cudaFree(w.ptr);
    w.ptr = nullptr;
    w.bytes = 0;
    e = cudaMalloc(&w.ptr, bytes);
    if (e != cudaSuccess) return cuda_fail(e, "workspace allocation");
    w.bytes = bytes;
  }
  *out = w.ptr;
  return MOE_NVFP4_OK;
}

moe::RouteBufs route_bufs(uint8_t* ws, const WsLayout& L) {
  moe::RouteBufs b;
  b.ids = reinterpret_cast<int32_t*>(ws + L.ids);
  b.w = reinterpret_cast<float*>(ws + L.w);
  b.counts = reinterpret_cast<int32_t*>(ws + L.counts);
  b.offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  b.perm = reinterpret_cast<int32_t*>(ws + L.perm);
  b.inv = reinterpret_cast<int32_t*>(ws + L.inv);
  b.groups = reinterpret_cast<int4*>(ws + L.groups);
  b.ngroups = reinterpret_cast<int32_t*>(ws + L.ngroups);
  b.singles = reinterpret_cast<int4*>(ws + L.singles);
  b.nsingles = reinterpret_cast<int32_t*>(ws + L.nsingles);
  b.chunk_counts = reinterpret_cast<int32_t*>(ws + L.chunk_counts);
  b.done = reinterpret_cast<unsigned*>(ws + L.done);
  b.group_rows = 8;
  b.split_singles = 0;
  b.expert_major = 0;
  return b;
}

int check_k_T(int64_t T, int E, int k) {
  if (T < 0) return fail(MOE_NVFP4_ERR_INVALID_ARG, "T = %lld is negative", (long long)T);
  if (k < 1 || k > 32 || k > E) return fail(MOE_NVFP4_ERR_INVALID_ARG, "k = %d outside 1..min(E=%d, 32)", k, E);
  if (T > ((int64_t)1 << 31) / 32) return fail(MOE_NVFP4_ERR_UNSUPPORTED, "T = %lld too large", (long long)T);
  return MOE_NVFP4_OK;
}

// AUTO takes the tensor-core path once experts average more than 8 routed rows and the
// shapes allow it (H and I multiples of 256).
int resolve_path(int path, int64_t T, int k, int E, int H, int I) {
  if (path != MOE_NVFP4_PATH_AUTO) return path;
  return (T * k > (int64_t)8 * E && moe::prefill_supported(H, I)) ? MOE_NVFP4_PATH_PREFILL
                                                                  : MOE_NVFP4_PATH_DECODE;
}

// Prefill path: route (groups of up to 256 rows) -> gather -> tcgen05 gate/up -> tcgen05 down
// -> combine.  The bf16 gathered rows live in the y region and the bf16 intermediate in the h
// region, so the workspace is the decode path's.
int prefill_impl(const void* x, const float* logits, int64_t T, const moe_nvfp4_bank* bank, int32_t k, void* out,
                 void* x_next, void* workspace, size_t workspace_bytes, void* stream, int dev,
                 const DeviceInfo& info) {
  const int E = bank->num_experts, H = bank->hidden, I = bank->intermediate;
  const WsLayout L = ws_layout(T, E, k, H, I, MOE_NVFP4_PATH_PREFILL);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  int rc;
  if (ws) {
    if (workspace_bytes < L.total)
      return fail(MOE_NVFP4_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes,
                  L.total);
    if (!aligned(ws, 256)) return fail(MOE_NVFP4_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  } else if ((rc = ensure_workspace(dev, L.total, s, &ws))) {
    return rc;
  }
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  moe::RouteBufs rb = route_bufs(w8, L);
  rb.group_rows = moe::kPrefillRows;
  rb.split_singles = 0;
  const moe::BankView bv = view_of(bank);
  const int64_t R = T * k;
  void* hb = w8 + L.h;
  unsigned* tile_ctr = reinterpret_cast<unsigned*>(w8 + L.bar);   // two tile counters, zeroed here
  {
    const cudaError_t e = cudaMemsetAsync(tile_ctr, 0, 2 * sizeof(unsigned), s);
    if (e != cudaSuccess) return cuda_fail(e, "clear tile counters");
  }
  void* xp = w8 + L.y;
  float* y = reinterpret_cast<float*>(w8 + L.y);
  int launches = 0;
  prof_before(MOE_NVFP4_KERNEL_ROUTE, s);
  if ((rc = after_launch(moe::launch_route(logits, T, E, k, rb, s), s, "route", &launches))) return rc;
  // Gate/up runs on F16 operands: the gathered rows are prescaled into f16 and the per-row factors
  // that undo it sit in the unused second half of the h region (h is bf16 [R, I] there).
  float* colscale = reinterpret_cast<float*>(w8 + L.h + up256((size_t)R * I * 2));
  prof_before(MOE_NVFP4_KERNEL_PREFILL_GATHER, s);
  if ((rc = after_launch(moe::launch_gather_f16(static_cast<const uint16_t*>(x), rb.inv, k, T, H, xp, colscale, s), s,
                         "gather", &launches)))
    return rc;
  const int pairs = prefill_pair_kernel() ? moe::prefill2_pairs(info.sms) : 0;
  prof_before(MOE_NVFP4_KERNEL_PREFILL_GATEUP, s);
  rc = pairs > 0 ? moe::launch_prefill2_gateup(bv, xp, colscale, R, rb, hb, pairs, s)
                 : moe::launch_prefill_gateup(bv, xp, colscale, R, rb, hb, tile_ctr, info.sms, s);
  if ((rc = after_launch(rc, s, "prefill gate/up", &launches))) return rc;
  prof_before(MOE_NVFP4_KERNEL_PREFILL_DOWN, s);
  rc = pairs > 0 ? moe::launch_prefill2_down(bv, hb, R, rb, y, pairs, s)
                 : moe::launch_prefill_down(bv, hb, R, rb, y, tile_ctr + 1, info.sms, s);
  if ((rc = after_launch(rc, s, "prefill down", &launches))) return rc;
  prof_before(MOE_NVFP4_KERNEL_COMBINE, s);
  if ((rc = after_launch(moe::launch_combine(y, rb.w, rb.inv, T, k, H, static_cast<const uint16_t*>(x),
                                             static_cast<uint16_t*>(out), static_cast<uint16_t*>(x_next), s),
                         s, "combine", &launches)))
    return rc;
  t_last_launches = launches;
  return MOE_NVFP4_OK;
}

int forward_impl(const void* x, const float* logits, int64_t T, const moe_nvfp4_bank* bank, int32_t k,
                 void* out, void* x_next, void* workspace, size_t workspace_bytes, int32_t path,
                 void* stream) {
  t_last_launches = 0;
  int rc = check_bank(bank);
  if (rc) return rc;
  const int E = bank->num_experts, H = bank->hidden, I = bank->intermediate;
  if ((rc = check_k_T(T, E, k))) return rc;
  if (path < MOE_NVFP4_PATH_AUTO || path > MOE_NVFP4_PATH_PREFILL)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "path %d unknown", path);
  int dev;
  DeviceInfo info;
  if ((rc = current_device(&dev, &info))) return rc;
  if (T == 0) return MOE_NVFP4_OK;
  if (!x || !logits || !out) return fail(MOE_NVFP4_ERR_INVALID_ARG, "x, logits and out must not be NULL");
  if (!aligned(x, 16) || !aligned(logits, 16) || !aligned(out, 16) || (x_next && !aligned(x_next, 16)))
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "x, logits, out and x_next must be 16-byte aligned");
  const int use = resolve_path(path, T, k, E, H, I);
  if (use == MOE_NVFP4_PATH_PREFILL) {
    if (!moe::prefill_supported(H, I))
      return fail(MOE_NVFP4_ERR_UNSUPPORTED, "prefill path needs H %% 256 == 0 and I %% 256 == 0 (H=%d, I=%d)", H,
                  I);
    return prefill_impl(x, logits, T, bank, k, out, x_next, workspace, workspace_bytes, stream, dev, info);
  }
  const int xrows = (int)(T < 8 ? T : 8);
  if (moe::decode_smem_bytes(H, xrows, true) == 0 || moe::decode_smem_bytes(I, xrows, false) == 0 ||
      (int)moe::decode_smem_bytes(H, xrows, true) > info.smem_optin)
    return fail(MOE_NVFP4_ERR_UNSUPPORTED, "H=%d / I=%d exceed the decode kernel's shared memory", H, I);

  const WsLayout L = ws_layout(T, E, k, H, I, use);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  if (ws) {
    if (workspace_bytes < L.total)
      return fail(MOE_NVFP4_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes,
                  L.total);
    if (!aligned(ws, 256)) return fail(MOE_NVFP4_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  } else if ((rc = ensure_workspace(dev, L.total, s, &ws))) {
    return rc;
  }
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  moe::RouteBufs rb = route_bufs(w8, L);
  const moe::BankView bv = view_of(bank);
  int launches = 0;
  if (T == 1 && moe::decode1_supported(H, I, k, E, info.sms)) {
    prof_before(MOE_NVFP4_KERNEL_DECODE_FUSED, s);
    if ((rc = after_launch(moe::launch_decode1(bv, logits, k, static_cast<const uint16_t*>(x),
                                               static_cast<uint16_t*>(out), static_cast<uint16_t*>(x_next),
                                               reinterpret_cast<float*>(w8 + L.h), reinterpret_cast<float*>(w8 + L.y),
                                               rb.ids, rb.w, dev, info.sms, s),
                           s, "fused single-token decode", &launches)))
      return rc;
    t_last_launches = launches;
    return MOE_NVFP4_OK;
  }
  // 2 .. 11 tokens: the few-token kernel (one launch after the router, combine inside); from 12
  // tokens on the grouped kernels read each expert once per group of 8 rows instead of once per
  // routed row and are faster (measured: 16 tokens 529 -> 480 us, equal at 12).
  if (moe::decode_few_supported(H, I, k, (int)T, info.sms) && T < kGroupedMinT &&
      decode_kernel_choice() == kDecodeDefault) {
    // A few tokens: the router, then one persistent kernel over one slot per routed row in the
    // router's permutation order (expert order).
    prof_before(MOE_NVFP4_KERNEL_ROUTE, s);
    if ((rc = after_launch(moe::launch_route(logits, T, E, k, rb, s), s, "route", &launches))) return rc;
    prof_before(MOE_NVFP4_KERNEL_DECODE_FUSED, s);
    if ((rc = after_launch(moe::launch_decode_few(bv, (int)T, k, static_cast<const uint16_t*>(x),
                                                  static_cast<uint16_t*>(out), static_cast<uint16_t*>(x_next),
                                                  reinterpret_cast<float*>(w8 + L.h),
                                                  reinterpret_cast<float*>(w8 + L.y), rb.ids, rb.w, rb.perm, rb.inv,
                                                  dev, info.sms, s),
                           s, "fused few-token decode", &launches)))
      return rc;
    t_last_launches = launches;
    return MOE_NVFP4_OK;
  }
  if (moe::grouped_supported(H, I) && decode_kernel_choice() != kDecodeRows) {
    // Larger batches: the router's groups of up to 8 rows of one expert (single rows included),
    // the persistent gate/up and down kernels, then the combine.
    rb.group_rows = 8;
    rb.split_singles = 0;
    rb.expert_major = 1;           // an expert's groups stream together (repeat reads hit L2)
    float* h = reinterpret_cast<float*>(w8 + L.h);
    float* y = reinterpret_cast<float*>(w8 + L.y);
    prof_before(MOE_NVFP4_KERNEL_ROUTE, s);
    if ((rc = after_launch(moe::launch_route(logits, T, E, k, rb, s), s, "route", &launches))) return rc;
    prof_before(MOE_NVFP4_KERNEL_DECODE_GATEUP, s);
    if ((rc = after_launch(moe::launch_grouped_gateup(bv, static_cast<const uint16_t*>(x), k, rb, h, info.sms, s), s,
                           "grouped gate/up", &launches)))
      return rc;
    prof_before(MOE_NVFP4_KERNEL_DECODE_DOWN, s);
    if ((rc = after_launch(moe::launch_grouped_down(bv, h, rb, y, info.sms, s), s, "grouped down", &launches)))
      return rc;
    prof_before(MOE_NVFP4_KERNEL_COMBINE, s);
    if ((rc = after_launch(moe::launch_combine(y, rb.w, rb.inv, T, k, H, static_cast<const uint16_t*>(x),
                                               static_cast<uint16_t*>(out), static_cast<uint16_t*>(x_next), s),
                           s, "combine", &launches)))
      return rc;
    t_last_launches = launches;
    return MOE_NVFP4_OK;
  }
  // One-row groups take the CUDA-core row kernels when both widths allow; groups of two or
  // more rows (none when T == 1) take the mma.sync kernels.
  const bool rows = moe::rows_supported(H, true) && moe::rows_supported(I, false);
  const bool multi = !rows || T > 1;
  rb.split_singles = rows ? 1 : 0;
  float* h = reinterpret_cast<float*>(w8 + L.h);
  float* y = reinterpret_cast<float*>(w8 + L.y);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  prof_before(MOE_NVFP4_KERNEL_ROUTE, s);
  if ((rc = after_launch(moe::launch_route(logits, T, E, k, rb, s), s, "route", &launches))) return rc;
  prof_before(MOE_NVFP4_KERNEL_DECODE_GATEUP, s);
  if (rows && (rc = after_launch(moe::launch_rows_gateup(bv, xb, k, rb, h, info.sms, s), s, "rows gate/up",
                                 &launches)))
    return rc;
  if (multi && (rc = after_launch(moe::launch_decode_gateup(bv, xb, k, rb, xrows, h, info.sms, s), s,
                                  "decode gate/up", &launches)))
    return rc;
  prof_before(MOE_NVFP4_KERNEL_DECODE_DOWN, s);
  if (rows && (rc = after_launch(moe::launch_rows_down(bv, h, rb, y, info.sms, s), s, "rows down", &launches)))
    return rc;
  if (multi && (rc = after_launch(moe::launch_decode_down(bv, h, rb, xrows, y, info.sms, s), s, "decode down",
                                  &launches)))
    return rc;
  prof_before(MOE_NVFP4_KERNEL_COMBINE, s);
  if ((rc = after_launch(moe::launch_combine(y, rb.w, rb.inv, T, k, H, static_cast<const uint16_t*>(x),
                                             static_cast<uint16_t*>(out), static_cast<uint16_t*>(x_next), s),
                         s, "combine", &launches)))
    return rc;
  t_last_launches = launches;
  return MOE_NVFP4_OK;
}

// Experts-only call: y_rows[r] = expert ids[r] applied to x_rows[r] (no router, no weights, no
// combine), for expert parallelism, where a rank runs its own experts on the rows other ranks
// sent it.  The same expert kernels as the layer: the ids router (k = 1) places the rows in
// expert order, the tensor-core or the grouped/row kernels compute y in that order, and the
// unpermute kernel writes each row's result back at its own index.
int experts_impl(const void* x_rows, const int32_t* ids, int64_t R, const moe_nvfp4_bank* bank, float* y_rows,
                 void* workspace, size_t workspace_bytes, int32_t path, int32_t flags, void* stream) {
  t_last_launches = 0;
  int rc = check_bank(bank);
  if (rc) return rc;
  const int E = bank->num_experts, H = bank->hidden, I = bank->intermediate;
  if ((rc = check_k_T(R, E, 1))) return rc;
  if (path < MOE_NVFP4_PATH_AUTO || path > MOE_NVFP4_PATH_PREFILL)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "path %d unknown", path);
  if (flags & ~MOE_NVFP4_EXPERTS_SORTED) return fail(MOE_NVFP4_ERR_INVALID_ARG, "flags 0x%x unknown", flags);
  const bool sorted = (flags & MOE_NVFP4_EXPERTS_SORTED) != 0;
  int dev;
  DeviceInfo info;
  if ((rc = current_device(&dev, &info))) return rc;
  if (R == 0) return MOE_NVFP4_OK;
  if (!x_rows || !ids || !y_rows) return fail(MOE_NVFP4_ERR_INVALID_ARG, "x_rows, ids and y_rows must not be NULL");
  if (!aligned(x_rows, 16) || !aligned(y_rows, 16) || !aligned(ids, 4))
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "x_rows and y_rows must be 16-byte aligned, ids 4-byte aligned");
  const int use = resolve_path(path, R, 1, E, H, I);
  if (use == MOE_NVFP4_PATH_PREFILL && !moe::prefill_supported(H, I))
    return fail(MOE_NVFP4_ERR_UNSUPPORTED, "prefill path needs H %% 256 == 0 and I %% 256 == 0 (H=%d, I=%d)", H, I);
  const int xrows = (int)(R < 8 ? R : 8);
  if (use != MOE_NVFP4_PATH_PREFILL &&
      (moe::decode_smem_bytes(H, xrows, true) == 0 || moe::decode_smem_bytes(I, xrows, false) == 0 ||
       (int)moe::decode_smem_bytes(H, xrows, true) > info.smem_optin))
    return fail(MOE_NVFP4_ERR_UNSUPPORTED, "H=%d / I=%d exceed the decode kernel's shared memory", H, I);
  const WsLayout L = ws_layout(R, E, 1, H, I, use, true);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  if (ws) {
    if (workspace_bytes < L.total)
      return fail(MOE_NVFP4_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes,
                  L.total);
    if (!aligned(ws, 256)) return fail(MOE_NVFP4_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  } else if ((rc = ensure_workspace(dev, L.total, s, &ws))) {
    return rc;
  }
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  moe::RouteBufs rb = route_bufs(w8, L);
  const moe::BankView bv = view_of(bank);
  const uint16_t* xb = static_cast<const uint16_t*>(x_rows);
  float* h = reinterpret_cast<float*>(w8 + L.h);
  // Rows already in expert order: the router's permutation is the identity, so the down
  // kernels write each row's result in place and no unpermute follows.
  float* y = sorted ? y_rows : reinterpret_cast<float*>(w8 + L.y);
  int launches = 0;
  if (use == MOE_NVFP4_PATH_PREFILL) {
    rb.group_rows = moe::kPrefillRows;
    unsigned* tile_ctr = reinterpret_cast<unsigned*>(w8 + L.bar);
    const cudaError_t e = cudaMemsetAsync(tile_ctr, 0, 2 * sizeof(unsigned), s);
    if (e != cudaSuccess) return cuda_fail(e, "clear tile counters");
    prof_before(MOE_NVFP4_KERNEL_ROUTE, s);
    if ((rc = after_launch(moe::launch_route_ids(ids, R, E, rb, s), s, "ids route", &launches))) return rc;
    void* xp = w8 + L.y;
    void* hb = w8 + L.h;
    float* colscale = reinterpret_cast<float*>(w8 + L.h + up256((size_t)R * I * 2));
    prof_before(MOE_NVFP4_KERNEL_PREFILL_GATHER, s);
    if ((rc = after_launch(moe::launch_gather_f16(xb, rb.inv, 1, R, H, xp, colscale, s), s, "gather", &launches)))
      return rc;
    const int pairs = prefill_pair_kernel() ? moe::prefill2_pairs(info.sms) : 0;
    prof_before(MOE_NVFP4_KERNEL_PREFILL_GATEUP, s);
    rc = pairs > 0 ? moe::launch_prefill2_gateup(bv, xp, colscale, R, rb, hb, pairs, s)
                   : moe::launch_prefill_gateup(bv, xp, colscale, R, rb, hb, tile_ctr, info.sms, s);
    if ((rc = after_launch(rc, s, "prefill gate/up", &launches))) return rc;
    prof_before(MOE_NVFP4_KERNEL_PREFILL_DOWN, s);
    rc = pairs > 0 ? moe::launch_prefill2_down(bv, hb, R, rb, y, pairs, s)
                   : moe::launch_prefill_down(bv, hb, R, rb, y, tile_ctr + 1, info.sms, s);
    if ((rc = after_launch(rc, s, "prefill down", &launches))) return rc;
  } else if (moe::grouped_supported(H, I) && decode_kernel_choice() != kDecodeRows) {
    rb.group_rows = 8;
    rb.split_singles = 0;
    rb.expert_major = 1;
    prof_before(MOE_NVFP4_KERNEL_ROUTE, s);
    if ((rc = after_launch(moe::launch_route_ids(ids, R, E, rb, s), s, "ids route", &launches))) return rc;
    prof_before(MOE_NVFP4_KERNEL_DECODE_GATEUP, s);
    if ((rc = after_launch(moe::launch_grouped_gateup(bv, xb, 1, rb, h, info.sms, s), s, "grouped gate/up",
                           &launches)))
      return rc;
    prof_before(MOE_NVFP4_KERNEL_DECODE_DOWN, s);
    if ((rc = after_launch(moe::launch_grouped_down(bv, h, rb, y, info.sms, s), s, "grouped down", &launches)))
      return rc;
  } else {
    const bool rows = moe::rows_supported(H, true) && moe::rows_supported(I, false);
    const bool multi = !rows || R > 1;       // groups of two or more rows exist only then
    rb.split_singles = rows ? 1 : 0;
    prof_before(MOE_NVFP4_KERNEL_ROUTE, s);
    if ((rc = after_launch(moe::launch_route_ids(ids, R, E, rb, s), s, "ids route", &launches))) return rc;
    prof_before(MOE_NVFP4_KERNEL_DECODE_GATEUP, s);
    if (rows && (rc = after_launch(moe::launch_rows_gateup(bv, xb, 1, rb, h, info.sms, s), s, "rows gate/up",
                                   &launches)))
      return rc;
    if (multi && (rc = after_launch(moe::launch_decode_gateup(bv, xb, 1, rb, xrows, h, info.sms, s), s, "decode gate/up",
                           &launches)))
      return rc;
    prof_before(MOE_NVFP4_KERNEL_DECODE_DOWN, s);
    if (rows && (rc = after_launch(moe::launch_rows_down(bv, h, rb, y, info.sms, s), s, "rows down", &launches)))
      return rc;
    if (multi && (rc = after_launch(moe::launch_decode_down(bv, h, rb, xrows, y, info.sms, s), s, "decode down",
                                    &launches)))
      return rc;
  }
  if (!sorted) {
    prof_before(MOE_NVFP4_KERNEL_COMBINE, s);
    if ((rc = after_launch(moe::launch_unpermute(y, rb.inv, rb.ids, R, H, y_rows, s), s, "unpermute", &launches)))
      return rc;
  }
  t_last_launches = launches;
  return MOE_NVFP4_OK;
}

int ensure_stage(void** p, size_t* have, size_t need) {
  if (*have >= need) return MOE_NVFP4_OK;
  if (*p) cudaFree(*p);
  *p = nullptr;
  *have = 0;
  const cudaError_t e = cudaMalloc(p, need);
  if (e != cudaSuccess) return cuda_fail(e, "staging allocation");
  *have = need;
  return MOE_NVFP4_OK;
}

// Fixed scratch for moe_nvfp4_forward_noalloc: a file-scope device array, so the entry point
// never allocates.  Every device that loads the library holds it until the process exits.
constexpr size_t kNoAllocBytes = (size_t)16 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch per device (host code only sees a stand-in for it).
std::vector<void*> g_noalloc_addr;

int noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if ((int)g_noalloc_addr.size() <= dev) g_noalloc_addr.resize(dev + 1, nullptr);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // current device = dev
    if (e != cudaSuccess) return cuda_fail(e, "resolve the fixed scratch array");
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return MOE_NVFP4_OK;
}

// W4A4 path: route (groups of up to 128 rows) -> quantize x -> tcgen05 kind::mxf4nvf4 gate/up (h
// quantized in its epilogue) -> down -> combine.  The x codes and scales live in the y region
// (dead once gate/up has run), the h codes and scales in the h region: the prefill path's
// workspace.
int w4a4_impl(const void* x, const float* logits, int64_t T, const moe_nvfp4_bank* bank, const float* act_scales,
              int32_t k, void* out, void* x_next, void* workspace, size_t workspace_bytes,
              const moe_nvfp4_w4a4_taps* taps, void* stream) {
  t_last_launches = 0;
  int rc = check_bank(bank);
  if (rc) return rc;
  const int E = bank->num_experts, H = bank->hidden, I = bank->intermediate;
  if ((rc = check_k_T(T, E, k))) return rc;
  if (!moe::w4a4_supported(H, I))
    return fail(MOE_NVFP4_ERR_UNSUPPORTED, "W4A4 path needs H %% 256 == 0 and I %% 256 == 0 (H=%d, I=%d)", H, I);
  int dev;
  DeviceInfo info;
  if ((rc = current_device(&dev, &info))) return rc;
  if (T == 0) return MOE_NVFP4_OK;
  if (!x || !logits || !out || !act_scales)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "x, logits, act_scales and out must not be NULL");
  if (!aligned(x, 16) || !aligned(logits, 16) || !aligned(out, 16) || !aligned(act_scales, 16) ||
      (x_next && !aligned(x_next, 16)))
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "x, logits, act_scales, out and x_next must be 16-byte aligned");
  moe_nvfp4_w4a4_taps tp{};
  if (taps) tp = *taps;
  if (!tp.x_codes_dev != !tp.x_scales_dev || !tp.h_codes_dev != !tp.h_scales_dev)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "taps: codes and scales come in pairs (both set or both NULL)");
  const void* tps[5] = {tp.x_codes_dev, tp.x_scales_dev, tp.h_dev, tp.h_codes_dev, tp.h_scales_dev};
  for (const void* q : tps)
    if (q && !aligned(q, 16)) return fail(MOE_NVFP4_ERR_INVALID_ARG, "taps must be 16-byte aligned");
  const WsLayout L = ws_layout(T, E, k, H, I, MOE_NVFP4_PATH_PREFILL);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  if (ws) {
    if (workspace_bytes < L.total)
      return fail(MOE_NVFP4_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", workspace_bytes,
                  L.total);
    if (!aligned(ws, 256)) return fail(MOE_NVFP4_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  } else if ((rc = ensure_workspace(dev, L.total, s, &ws))) {
    return rc;
  }
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  moe::RouteBufs rb = route_bufs(w8, L);
  rb.group_rows = moe::kW4A4Rows;
  rb.split_singles = 0;
  const moe::BankView bv = view_of(bank);
  const int64_t R = T * k;
  uint8_t* xc = w8 + L.y;
  uint8_t* xs = xc + up256((size_t)R * H / 2);
  uint8_t* hc = w8 + L.h;
  uint8_t* hs = hc + up256((size_t)R * I / 2);
  float* y = reinterpret_cast<float*>(w8 + L.y);
  unsigned* tile_ctr = reinterpret_cast<unsigned*>(w8 + L.bar);
  {
    const cudaError_t e = cudaMemsetAsync(tile_ctr, 0, 2 * sizeof(unsigned), s);
    if (e != cudaSuccess) return cuda_fail(e, "clear tile counters");
  }
  int launches = 0;
  prof_before(MOE_NVFP4_KERNEL_ROUTE, s);
  if ((rc = after_launch(moe::launch_route(logits, T, E, k, rb, s), s, "route", &launches))) return rc;
  prof_before(MOE_NVFP4_KERNEL_W4A4_QUANT, s);
  if ((rc = after_launch(moe::launch_w4a4_quant_x(static_cast<const uint16_t*>(x), rb, k, R, H, act_scales, xc, xs,
                                                  tp.x_codes_dev, tp.x_scales_dev, s),
                         s, "W4A4 quantize x", &launches)))
    return rc;
  const moe::W4A4Taps wt{tp.h_dev, tp.h_codes_dev, tp.h_scales_dev};
  prof_before(MOE_NVFP4_KERNEL_W4A4_GATEUP, s);
  if ((rc = after_launch(moe::launch_w4a4_gateup(bv, act_scales, xc, xs, R, rb, hc, hs, wt, tile_ctr, info.sms, s), s,
                         "W4A4 gate/up", &launches)))
    return rc;
  prof_before(MOE_NVFP4_KERNEL_W4A4_DOWN, s);
  if ((rc = after_launch(moe::launch_w4a4_down(bv, act_scales, hc, hs, R, rb, y, tile_ctr + 1, info.sms, s), s,
                         "W4A4 down", &launches)))
    return rc;
  prof_before(MOE_NVFP4_KERNEL_COMBINE, s);
  if ((rc = after_launch(moe::launch_combine(y, rb.w, rb.inv, T, k, H, static_cast<const uint16_t*>(x),
                                             static_cast<uint16_t*>(out), static_cast<uint16_t*>(x_next), s),
                         s, "combine", &launches)))
    return rc;
  t_last_launches = launches;
  return MOE_NVFP4_OK;
}

}  // namespace

// Bridge for the other translation units of the C ABI (pack.cu): error reporting and the
// current device's checks, with the same semantics as the entry points here.
namespace moe {

cudaError_t set_smem_limit(const void* kernel, int bytes) {
  struct Key {
    const void* k;
    int dev, bytes;
  };
  static std::mutex mu;
  static std::vector<Key> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  for (const Key& d : done)
    if (d.k == kernel && d.dev == dev && d.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back(Key{kernel, dev, bytes});
  return e;
}

int api_fail(int code, const char* msg) { return fail(code, "%s", msg); }

void api_set_launches(int n) { t_last_launches = n; }

int api_cuda_fail(int err, const char* what) { return cuda_fail((cudaError_t)err, what); }

int api_device(int* dev, int* sms) {
  DeviceInfo info;
  const int rc = current_device(dev, &info);
  if (rc == MOE_NVFP4_OK) *sms = info.sms;
  return rc;
}

}  // namespace moe

// Host inputs of at least this many bytes in page-locked memory are copied to the device directly.
static constexpr size_t kDirectCopyBytes = (size_t)1 << 20;

static bool is_pinned(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();                       // pageable memory of old runtimes reports an error
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

extern "C" {

int moe_nvfp4_forward(const void* x_dev, const float* logits_dev, int64_t T, const moe_nvfp4_bank* bank, int32_t k,
                      void* out_dev, void* stream) {
  return forward_impl(x_dev, logits_dev, T, bank, k, out_dev, nullptr, nullptr, 0, MOE_NVFP4_PATH_AUTO, stream);
}

int moe_nvfp4_forward_ex(const void* x_dev, const float* logits_dev, int64_t T, const moe_nvfp4_bank* bank,
                         int32_t k, void* out_dev, void* x_next_dev, void* workspace_dev, size_t workspace_bytes,
                         int32_t path, void* stream) {
  return forward_impl(x_dev, logits_dev, T, bank, k, out_dev, x_next_dev, workspace_dev, workspace_bytes, path,
                      stream);
}

int moe_nvfp4_forward_w4a4(const void* x_dev, const float* logits_dev, int64_t T, const moe_nvfp4_bank* bank,
                           const float* act_scales_dev, int32_t k, void* out_dev, void* x_next_dev,
                           void* workspace_dev, size_t workspace_bytes, const moe_nvfp4_w4a4_taps* taps,
                           void* stream) {
  return w4a4_impl(x_dev, logits_dev, T, bank, act_scales_dev, k, out_dev, x_next_dev, workspace_dev, workspace_bytes,
                   taps, stream);
}

// Host calls whose inputs fit in this many bytes replay a captured graph.
static constexpr size_t kGraphMaxBytes = (size_t)64 << 10;
static constexpr size_t kMaxHostGraphs = 8;

// The graph of a small host call: H2D copy of the staged x | logits, the layer on the internal
// workspace, D2H copy into the pinned out staging buffer.  Captured on a library stream (the
// caller's may be the legacy stream, which cannot capture), launched on the caller's.
// With build false, only looks the graph up (*out_g = NULL when there is none).
static int host_graph(HostStage* st, int dev, int64_t T, const moe_nvfp4_bank* bank, int32_t k, size_t ib,
                      size_t lo, size_t xb, bool build, HostGraph** out_g) {
  const int E = bank->num_experts, H = bank->hidden, I = bank->intermediate;
  void* ws = nullptr;
  int rc;
  const size_t need = ws_layout(T, E, k, H, I, resolve_path(MOE_NVFP4_PATH_AUTO, T, k, E, H, I)).total;
  if (!st->capture) {
    const cudaError_t e = cudaStreamCreateWithFlags(&st->capture, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "capture stream");
  }
  if ((rc = ensure_workspace(dev, need, st->capture, &ws))) return rc;
  for (HostGraph& g : st->graphs)
    if (g.T == T && g.k == k && !memcmp(&g.bank, bank, sizeof(*bank)) && g.in_dev == st->in_dev && g.in_host == st->in_host &&
        g.out == st->out && g.out_host == st->out_host && g.ws == ws) {
      g.used = ++st->tick;
      *out_g = &g;
      return MOE_NVFP4_OK;
    }
  *out_g = nullptr;
  if (!build) return MOE_NVFP4_OK;
  cudaStream_t c = st->capture;
  cudaError_t e = cudaStreamBeginCapture(c, cudaStreamCaptureModeThreadLocal);
  if (e != cudaSuccess) return cuda_fail(e, "begin capture");
  e = cudaMemcpyAsync(st->in_dev, st->in_host, ib, cudaMemcpyHostToDevice, c);
  rc = e != cudaSuccess ? cuda_fail(e, "capture copy in") : MOE_NVFP4_OK;
  if (!rc)
    rc = forward_impl(st->in_dev, reinterpret_cast<const float*>(static_cast<uint8_t*>(st->in_dev) + lo), T, bank, k,
                      st->out, nullptr, nullptr, 0, MOE_NVFP4_PATH_AUTO, c);
  const int launches = t_last_launches;
  if (!rc) {
    e = cudaMemcpyAsync(st->out_host, st->out, xb, cudaMemcpyDeviceToHost, c);
    if (e != cudaSuccess) rc = cuda_fail(e, "capture copy out");
  }
  cudaGraph_t graph = nullptr;
  e = cudaStreamEndCapture(c, &graph);
  if (!rc && e != cudaSuccess) rc = cuda_fail(e, "end capture");
  cudaGraphExec_t exec = nullptr;
  if (!rc) {
    e = cudaGraphInstantiate(&exec, graph, 0);
    if (e != cudaSuccess) rc = cuda_fail(e, "instantiate");
  }
  if (graph) cudaGraphDestroy(graph);
  if (rc) return rc;
  if (st->graphs.size() >= kMaxHostGraphs) {
    size_t lru = 0;
    for (size_t i = 1; i < st->graphs.size(); ++i)
      if (st->graphs[i].used < st->graphs[lru].used) lru = i;
    cudaGraphExecDestroy(st->graphs[lru].exec);
    st->graphs.erase(st->graphs.begin() + lru);
  }
  HostGraph g;
  g.T = T;
  g.k = k;
  g.bank = *bank;
  g.in_dev = st->in_dev;
  g.in_host = st->in_host;
  g.out = st->out;
  g.out_host = st->out_host;
  g.ws = ws;
  g.exec = exec;
  g.launches = launches;
  g.used = ++st->tick;
  st->graphs.push_back(g);
  *out_g = &st->graphs.back();
  return MOE_NVFP4_OK;
}

int moe_nvfp4_forward_host(const void* x_host, const float* logits_host, int64_t T, const moe_nvfp4_bank* bank,
                           int32_t k, void* out_host, void* stream) {
  int rc = check_bank(bank);
  if (rc) return rc;
  if ((rc = check_k_T(T, bank->num_experts, k))) return rc;
  int dev;
  DeviceInfo info;
  if ((rc = current_device(&dev, &info))) return rc;
  if (T == 0) return MOE_NVFP4_OK;
  if (!x_host || !logits_host || !out_host)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "x_host, logits_host and out_host must not be NULL");
  const size_t xb = (size_t)T * bank->hidden * 2, lb = (size_t)T * bank->num_experts * 4;
  HostStage* st;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    st = g_stage[dev].get();
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t lo = up256(xb), ib = lo + lb;          // logits after x, 256-byte aligned
  if (ib > st->in_bytes || xb > st->out_bytes) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "synchronise before staging growth");
    if (ib > st->in_bytes) {
      if (st->in_host) cudaFreeHost(st->in_host);
      st->in_host = nullptr;
      size_t have = st->in_bytes;
      if ((rc = ensure_stage(&st->in_dev, &have, ib))) return rc;
      e = cudaHostAlloc(&st->in_host, ib, cudaHostAllocDefault);
      if (e != cudaSuccess) {
        st->in_bytes = 0;
        return cuda_fail(e, "pinned staging allocation");
      }
      st->in_bytes = ib;
    }
    if ((rc = ensure_stage(&st->out, &st->out_bytes, xb))) return rc;
  }
  if (ib <= kGraphMaxBytes && !t_prof_on && !sync_each_kernel()) {
    // Small call: stage x and the logits, replay (or capture once) copy in + layer + copy out.
    if (xb > st->out_host_bytes) {
      cudaError_t e = cudaStreamSynchronize(s);
      if (e != cudaSuccess) return cuda_fail(e, "synchronise before staging growth");
      if (st->out_host) cudaFreeHost(st->out_host);
      st->out_host = nullptr;
      st->out_host_bytes = 0;
      e = cudaHostAlloc(&st->out_host, kGraphMaxBytes, cudaHostAllocDefault);
      if (e != cudaSuccess) return cuda_fail(e, "pinned staging allocation");
      st->out_host_bytes = kGraphMaxBytes;
    }
    HostGraph* g = nullptr;
    if ((rc = host_graph(st, dev, T, bank, k, ib, lo, xb, false, &g))) return rc;
    memcpy(st->in_host, x_host, xb);
    memcpy(static_cast<uint8_t*>(st->in_host) + lo, logits_host, lb);
    cudaError_t e;
    int launches;
    if (g) {
      e = cudaGraphLaunch(g->exec, s);
      launches = g->launches;
    } else {
      // First call of this kind: run it eagerly (every kernel attribute is then set outside any
      // capture), and capture the graph for the next calls once it has completed.
      e = cudaMemcpyAsync(st->in_dev, st->in_host, ib, cudaMemcpyHostToDevice, s);
      if (e == cudaSuccess) {
        rc = forward_impl(st->in_dev, reinterpret_cast<const float*>(static_cast<uint8_t*>(st->in_dev) + lo), T,
                          bank, k, st->out, nullptr, nullptr, 0, MOE_NVFP4_PATH_AUTO, stream);
        if (rc) {
          cudaStreamSynchronize(s);
          return rc;
        }
        e = cudaMemcpyAsync(st->out_host, st->out, xb, cudaMemcpyDeviceToHost, s);
      }
      launches = t_last_launches;
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "host call");
    memcpy(out_host, st->out_host, xb);
    if (!g && (rc = host_graph(st, dev, T, bank, k, ib, lo, xb, true, &g))) return rc;
    t_last_launches = launches;
    return MOE_NVFP4_OK;
  }
  cudaError_t e;
  if (ib >= kDirectCopyBytes && is_pinned(x_host) && is_pinned(logits_host)) {
    // Large inputs already in page-locked memory: two direct copies (a host memcpy into the
    // staging buffer would cost more than the second copy's launch).
    e = cudaMemcpyAsync(st->in_dev, x_host, xb, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<uint8_t*>(st->in_dev) + lo, logits_host, lb, cudaMemcpyHostToDevice, s);
  } else {
    // Small or pageable inputs: one host copy into the pinned staging buffer (free again here:
    // every call ends with a stream synchronisation), then one copy to the device.
    memcpy(st->in_host, x_host, xb);
    memcpy(static_cast<uint8_t*>(st->in_host) + lo, logits_host, lb);
    e = cudaMemcpyAsync(st->in_dev, st->in_host, ib, cudaMemcpyHostToDevice, s);
  }
  if (e != cudaSuccess) {
    cudaStreamSynchronize(s);
    return cuda_fail(e, "copy x and logits to device");
  }
  const void* xd = st->in_dev;
  const float* ld = reinterpret_cast<const float*>(static_cast<uint8_t*>(st->in_dev) + lo);
  rc = forward_impl(xd, ld, T, bank, k, st->out, nullptr, nullptr, 0,
                    MOE_NVFP4_PATH_AUTO, stream);
  if (rc) {
    cudaStreamSynchronize(s);                 // the copy from the pinned buffer may still run
    return rc;
  }
  e = cudaMemcpyAsync(out_host, st->out, xb, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) {
    cudaStreamSynchronize(s);
    return cuda_fail(e, "copy out to host");
  }
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "synchronise");
  return MOE_NVFP4_OK;
}

int moe_nvfp4_route(const float* logits_dev, int64_t T, int32_t E, int32_t k, int32_t* ids_dev, float* w_dev,
                    int32_t* counts_dev, int32_t* offsets_dev, int32_t* perm_dev, int32_t* inv_dev, void* stream) {
  t_last_launches = 0;
  if (E < 1 || E > 1024) return fail(MOE_NVFP4_ERR_UNSUPPORTED, "E = %d outside 1..1024", E);
  int rc = check_k_T(T, E, k);
  if (rc) return rc;
  int dev;
  DeviceInfo info;
  if ((rc = current_device(&dev, &info))) return rc;
  if (!counts_dev || !offsets_dev) return fail(MOE_NVFP4_ERR_INVALID_ARG, "counts and offsets must not be NULL");
  if (T > 0 && (!logits_dev || !ids_dev || !w_dev || !perm_dev || !inv_dev))
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "logits, ids, w, perm and inv must not be NULL");
  const WsLayout L = ws_layout(T, E, k, 128, 128, MOE_NVFP4_PATH_DECODE);
  const size_t need = L.h;  // routing part only
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws;
  if ((rc = ensure_workspace(dev, need, s, &ws))) return rc;
  moe::RouteBufs rb = route_bufs(static_cast<uint8_t*>(ws), L);
  rb.ids = ids_dev;
  rb.w = w_dev;
  rb.counts = counts_dev;
  rb.offsets = offsets_dev;
  rb.perm = perm_dev;
  rb.inv = inv_dev;
  if (T == 0) {
    cudaError_t e = cudaMemsetAsync(counts_dev, 0, (size_t)E * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(offsets_dev, 0, (size_t)(E + 1) * 4, s);
    return e == cudaSuccess ? MOE_NVFP4_OK : cuda_fail(e, "clear counts");
  }
  int launches = 0;
  if ((rc = after_launch(moe::launch_route(logits_dev, T, E, k, rb, s), s, "route", &launches))) return rc;
  t_last_launches = launches;
  return MOE_NVFP4_OK;
}

size_t moe_nvfp4_workspace_bytes(int64_t T, int32_t E, int32_t k, int32_t H, int32_t I, int32_t path) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > 32 || k > E || H < 128 || I < 128) return 0;
  return ws_layout(T, E, k, H, I, resolve_path(path, T, k, E, H, I)).total;
}

int moe_nvfp4_experts(const void* x_rows_dev, const int32_t* expert_ids_dev, int64_t R, const moe_nvfp4_bank* bank,
                      float* y_rows_dev, void* workspace_dev, size_t workspace_bytes, int32_t path, int32_t flags,
                      void* stream) {
  return experts_impl(x_rows_dev, expert_ids_dev, R, bank, y_rows_dev, workspace_dev, workspace_bytes, path, flags,
                      stream);
}

size_t moe_nvfp4_experts_workspace_bytes(int64_t R, int32_t E, int32_t H, int32_t I, int32_t path) {
  if (R < 0 || E < 1 || E > 1024 || H < 128 || I < 128) return 0;
  return ws_layout(R, E, 1, H, I, resolve_path(path, R, 1, E, H, I), true).total;
}

const char* moe_nvfp4_last_error(void) { return t_last_error.c_str(); }

int moe_nvfp4_device_status(void) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, moe::g_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  const int zero = 0;
  e = cudaMemcpyToSymbol(moe::g_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear device status");
  if (v != 0) {
    // A kernel that gave up may have left its completion counters set: clear them all.
    int rc = moe::decode1_reset_pool();
    if (rc == 0) rc = moe::decode_few_reset_pool();
    if (rc < 0) return cuda_fail((cudaError_t)(-rc), "clear decode counters");
    return fail(MOE_NVFP4_ERR_TIMEOUT, "a bounded device wait gave up (status %d)", v);
  }
  return MOE_NVFP4_OK;
}

int moe_nvfp4_forward_noalloc(const void* x_dev, const float* logits_dev, int64_t T, const moe_nvfp4_bank* bank,
                              int32_t k, void* out_dev, void* stream) {
  t_last_launches = 0;
  int rc = check_bank(bank);
  if (rc) return rc;
  if ((rc = check_k_T(T, bank->num_experts, k))) return rc;
  const size_t need = ws_layout(T, bank->num_experts, k, bank->hidden, bank->intermediate, MOE_NVFP4_PATH_AUTO).total;
  if (need > kNoAllocBytes)
    return fail(MOE_NVFP4_ERR_WORKSPACE,
                "this call needs %zu bytes of scratch; the fixed array of moe_nvfp4_forward_noalloc holds %zu "
                "(MOE_NVFP4_NOALLOC_MAX_BYTES); use moe_nvfp4_forward_ex with a caller workspace",
                need, kNoAllocBytes);
  int dev;
  DeviceInfo info;
  if ((rc = current_device(&dev, &info))) return rc;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(dev, &scratch))) return rc;
  return forward_impl(x_dev, logits_dev, T, bank, k, out_dev, nullptr, scratch, kNoAllocBytes,
                      MOE_NVFP4_PATH_AUTO, stream);
}

int moe_nvfp4_encode(const void* w_dev, int64_t n, int32_t out_features, int32_t in_features, int32_t global_mode,
                     void* dst_dev, uint64_t dst_stride, uint64_t codes_off, uint64_t scales_off, uint64_t global_off,
                     void* stream) {
  t_last_launches = 0;
  if (n < 0) return fail(MOE_NVFP4_ERR_INVALID_ARG, "n = %lld is negative", (long long)n);
  if (out_features < 1 || in_features < 16 || in_features % 16)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "shape [%d, %d]: out must be >= 1 and in a positive multiple of 16",
                out_features, in_features);
  if (global_mode != 0 && global_mode != 1)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "global_mode %d is not 0 or 1", global_mode);
  const uint64_t weights = (uint64_t)out_features * (uint64_t)in_features;
  const uint64_t cb = weights / 2, sb = weights / 16;
  if (codes_off % 16 || global_off % 4 || dst_stride % 16)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "codes_off and dst_stride must be multiples of 16, global_off of 4");
  auto overlap = [](uint64_t a, uint64_t al, uint64_t b, uint64_t bl) { return a < b + bl && b < a + al; };
  if (overlap(codes_off, cb, scales_off, sb) || overlap(codes_off, cb, global_off, 4) ||
      overlap(scales_off, sb, global_off, 4))
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "the codes, scales and global parts overlap");
  const uint64_t end = std::max(codes_off + cb, std::max(scales_off + sb, global_off + 4));
  if (n > 1 && end > dst_stride)
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "a projection's parts (%llu bytes) do not fit in dst_stride %llu",
                (unsigned long long)end, (unsigned long long)dst_stride);
  int dev, rc;
  DeviceInfo info;
  if ((rc = current_device(&dev, &info))) return rc;
  if (n == 0) return MOE_NVFP4_OK;
  if (!w_dev || !dst_dev) return fail(MOE_NVFP4_ERR_INVALID_ARG, "w and dst must not be NULL");
  if (!aligned(w_dev, 16) || !aligned(dst_dev, 16))
    return fail(MOE_NVFP4_ERR_INVALID_ARG, "w and dst must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int launches = 0;
  if ((rc = after_launch(moe::launch_encode(static_cast<const uint16_t*>(w_dev), n, out_features, in_features,
                                            global_mode, static_cast<uint8_t*>(dst_dev), dst_stride, codes_off,
                                            scales_off, global_off, info.sms, s),
                         s, "encode", &launches)))
    return rc;
  t_last_launches = launches;
  return MOE_NVFP4_OK;
}

int moe_nvfp4_last_launch_count(void) { return t_last_launches; }

int moe_nvfp4_profile_begin(void) {
  for (auto& p : t_prof) {
    cudaEventDestroy(p.a);
    cudaEventDestroy(p.b);
  }
  t_prof.clear();
  t_prof_on = true;
  return MOE_NVFP4_OK;
}

int moe_nvfp4_profile_end(double* ms, int64_t* launches, int32_t n) {
  t_prof_on = false;
  if ((!ms || !launches) && n > 0) return fail(MOE_NVFP4_ERR_INVALID_ARG, "ms and launches must not be NULL");
  for (int i = 0; i < n; ++i) {
    ms[i] = 0.0;
    launches[i] = 0;
  }
  int rc = MOE_NVFP4_OK;
  for (auto& p : t_prof) {
    float t = 0.0f;
    cudaError_t e = cudaEventSynchronize(p.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, p.a, p.b);
    if (e != cudaSuccess && rc == MOE_NVFP4_OK) rc = cuda_fail(e, "profile event");
    if (p.kind < n) {
      ms[p.kind] += t;
      launches[p.kind] += 1;
    }
    cudaEventDestroy(p.a);
    cudaEventDestroy(p.b);
  }
  t_prof.clear();
  return rc;
}

}  // extern "C"
