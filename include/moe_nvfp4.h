/*
 * moe_nvfp4.h -- C ABI of the NVFP4 weight-only routed-expert MoE layer for B200 (sm_100a).
 *
 * One call computes one routed-expert SwiGLU MoE layer of a large sparse model: for each
 * token, the top-k of E router logits (ties to the lower expert index) with softmax
 * weights over the k selected logits, then for every selected expert e
 *     y = Wd_e (silu(Wg_e x) * (Wu_e x)),
 * and out = sum over the k experts of weight * y, rounded to BF16.  Expert weights are
 * NVFP4 (weight = e2m1(code) * e4m3(block scale) * global); activations are BF16.
 *
 * Sources (pages on Reflection's Beam-1.0-501B-A23B):
 *  - "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents", section
 *    "What this pack holds": the expert record (gate, up and down, each E2M1 codes in U32
 *    words, one E4M3 block scale per 16 inputs and one F32 global scale), the MLX block
 *    scale e4m3(s) x (g / 2688) in f32, 256 routed experts with 8 active per token,
 *    activations in BF16.
 *  - "Beam-1.0-501B-A23B VQ GGUF", section "What stays native": router logits and SwiGLU
 *    are FP32 numerics; section "Kernel budget on GB10": hidden 5,120, intermediate 2,560,
 *    mid values staged as BF16.
 *
 * Conventions for every entry point:
 *  - Pointers named *_dev are device memory of the current CUDA device, *_host are host
 *    memory; the caller owns all of them and the library keeps none after the call.
 *  - Tensors are dense row-major.  x [T, H] and out [T, H] are BF16 (uint16 bit patterns),
 *    logits [T, E] are f32.  Device tensors must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Device work is only
 *    enqueued: errors raised by a kernel at run time surface at the caller's next
 *    synchronisation, or through moe_nvfp4_device_status().
 *  - Arguments are validated on the host before anything is enqueued; on a negative return
 *    nothing was enqueued (except MOE_NVFP4_ERR_CUDA from a launch) and
 *    moe_nvfp4_last_error() gives a message for the calling thread.
 *  - There is no CPU fallback: without an sm_100 device every compute entry point returns
 *    MOE_NVFP4_ERR_UNSUPPORTED.
 */
#ifndef MOE_NVFP4_H_
#define MOE_NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define MOE_NVFP4_OK               0
#define MOE_NVFP4_ERR_INVALID_ARG (-1)  /* null pointer, bad k, T < 0, misaligned pointer   */
#define MOE_NVFP4_ERR_UNSUPPORTED (-2)  /* shape outside the supported set, no sm_100 device */
#define MOE_NVFP4_ERR_CUDA        (-3)  /* a CUDA runtime call or launch failed              */
#define MOE_NVFP4_ERR_WORKSPACE   (-4)  /* caller workspace too small, or growth refused
                                           during stream capture                             */
#define MOE_NVFP4_ERR_TIMEOUT     (-5)  /* a bounded device-side wait gave up (device status) */
#define MOE_NVFP4_ERR_IO          (-6)  /* a pack file could not be opened or read            */
#define MOE_NVFP4_ERR_INTEGRITY   (-7)  /* a pack record's sha256 differs from its manifest    */

/*
 * Expert-GEMM path selection for moe_nvfp4_forward_ex.
 * DECODE (memory-bound, CUDA cores):
 *   T = 1, H x I in {5120x2560, 4096x1536, 2048x1024, 1024x512}, E <= 256: the whole layer in
 *     one persistent kernel (routing, gate/up, down and combine; one launch);
 *   2 <= T <= 16 with T k <= the SM count, same shapes: the router kernel, then one persistent
 *     kernel over the routed rows (two launches);
 *   otherwise: router kernel(s), grouped GEMV/GEMM kernels, combine.
 *   The persistent kernels take completion counters from 64 library-owned counter sets per
 *   device and kernel, one per call in turn, chosen on the host when the call is made (and so
 *   fixed inside a captured CUDA graph).  Two such calls whose GPU work overlaps -- calls on
 *   different streams with no ordering between them, concurrent replays of one graph, or a
 *   graph replay beside an eager call -- may share a set and return wrong results: order them
 *   on one stream (calls and replays in one stream run one after another).
 * PREFILL (tcgen05 tensor cores, BF16 x BF16 -> F32): H and I multiples of 256.
 */
#define MOE_NVFP4_PATH_AUTO    0
#define MOE_NVFP4_PATH_DECODE  1   /* memory-bound kernels, any number of tokens */
#define MOE_NVFP4_PATH_PREFILL 2   /* tensor-core (tcgen05) grouped GEMM          */

/*
 * Expert bank: E records in device memory, record e at base + e * record_stride.
 * Inside a record, projection p (0 = gate [I, H], 1 = up [I, H], 2 = down [H, I]; shape
 * [out, in], row-major) has
 *   codes   at codes_off[p]:  [out, in/8] little-endian uint32 words; input i of a row is
 *           the 4-bit E2M1 field at bits 4*(i%8) .. 4*(i%8)+3 of word i/8 (low nibble first);
 *   scales  at scales_off[p]: [out, in/16] E4M3 (OCP "FN") bytes, scale b covering inputs
 *           16b .. 16b+15 of its row;
 *   global  at global_off[p]: one f32.
 * global_mode 0: the weight is e2m1 * e4m3 * global.  global_mode 1: the stored f32 is the
 * streaming pack's g and the multiplier is f32(g / 2688), as the pack page says MLX forms it.
 * base, record_stride, codes_off and scales_off must be multiples of 16; global_off of 4.
 * The bank is read only; several calls may share it.
 */
typedef struct moe_nvfp4_bank {
  int32_t num_experts;    /* E, 1 .. 1024                                    */
  int32_t hidden;         /* H, a multiple of 128                            */
  int32_t intermediate;   /* I, a multiple of 128                            */
  int32_t global_mode;    /* 0 or 1                                          */
  const void* base_dev;   /* device pointer to record 0                      */
  uint64_t record_stride; /* bytes between records                           */
  uint64_t codes_off[3];
  uint64_t scales_off[3];
  uint64_t global_off[3];
} moe_nvfp4_bank;

/*
 * The layer, out = MoE(x).  Inputs: x_dev [T, H] BF16, logits_dev [T, E] f32, T >= 0
 * (T = 0 returns OK and enqueues nothing), 1 <= k <= min(E, 32).  Output: out_dev [T, H]
 * BF16 (round to nearest even).  Scratch comes from a per-device workspace owned by the
 * library that grows on demand (a growth synchronises the device; it is refused with
 * MOE_NVFP4_ERR_WORKSPACE while `stream` is capturing -- call once outside capture first,
 * or use moe_nvfp4_forward_ex with a caller workspace).  Not thread-safe per device when
 * the internal workspace is used from several host threads on different streams.
 */
int moe_nvfp4_forward(const void* x_dev, const float* logits_dev, int64_t T,
                      const moe_nvfp4_bank* bank, int32_t k, void* out_dev, void* stream);

/*
 * As moe_nvfp4_forward, plus:
 *  x_next_dev     if not NULL, also writes x_next [T, H] = bf16(x + out) (the residual add of
 *                 stacked layers; the sum of the two BF16 values rounded once);
 *  workspace_dev  caller scratch of workspace_bytes >= moe_nvfp4_workspace_bytes(...), 256-byte
 *                 aligned; if NULL the internal workspace is used;
 *  path           MOE_NVFP4_PATH_*; AUTO picks the prefill path when T*k > 8*E and H and I
 *                 are multiples of 256, else the decode path.
 * With a caller workspace nothing is allocated, so the call can be captured in a CUDA graph.
 * When the call's work has completed, the caller workspace starts with the routing result of
 * the call, on every path: ids [T, k] int32 at byte 0 and the softmax weights w [T, k] f32 at
 * byte 256 * ceil(T*k*4 / 256), both as moe_nvfp4_route describes them.
 */
int moe_nvfp4_forward_ex(const void* x_dev, const float* logits_dev, int64_t T,
                         const moe_nvfp4_bank* bank, int32_t k, void* out_dev,
                         void* x_next_dev, void* workspace_dev, size_t workspace_bytes,
                         int32_t path, void* stream);

/*
 * W4A4 variant of the layer: NVFP4 weights and NVFP4 activations on the block-scaled tensor
 * cores.  Source: page "Beam-1.0-501B-A23B, EXL3 3-bit ...", section "Fidelity" (the official
 * NVFP4 release served on Blackwell with FP4 activations, against the weights-only build); page
 * "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents", section "What this
 * pack holds" (the release's activation scales, which the BF16-activation build leaves unused).
 *
 * act_scales_dev [E][2] f32, positive and finite (not checked on the device): for a routed row
 * of expert e, x is quantized to NVFP4 with act_scales[e][0] as its global multiplier s, and the
 * mid values h = silu(g) * u, formed in f32, with act_scales[e][1].  Per block of 16 values the
 * block scale is the E4M3 value nearest to f32(amax / f32(6 s)) and each code the E2M1 value
 * nearest to f32(v / f32(e4m3 x s)), ties to even, saturating at 448 and 6, with the value's sign
 * bit (the encoder's rule, moe_nvfp4_encode, with s fixed in advance).  g, u and y accumulate in
 * f32 on the tensor cores; y is scaled by the weight global and s and combined as in
 * moe_nvfp4_forward.  The bank's block-scale bytes must be below 0x80 (the tensor cores read them
 * as unsigned E4M3; every encoder output is); this is not checked.  H and I must be multiples of
 * 256 (else MOE_NVFP4_ERR_UNSUPPORTED).
 *
 * x_next_dev as in moe_nvfp4_forward_ex.  workspace_dev: NULL for the internal workspace, else
 * at least moe_nvfp4_workspace_bytes(T, E, k, H, I, MOE_NVFP4_PATH_PREFILL) bytes, 256-byte
 * aligned; afterwards it starts with the routing result as moe_nvfp4_forward_ex describes.
 * taps (may be NULL, and so may each member; codes and scales come in pairs): the quantized
 * activations and the mid values of every routed slot t*k + j, written in addition to the
 * layer's own work, for inspection and tests.  Codes hold two E2M1 values per byte, the lower
 * index in the low nibble; scales are E4M3 bytes, one per 16 values.  Each must be 16-byte
 * aligned.
 */
typedef struct moe_nvfp4_w4a4_taps {
  uint8_t* x_codes_dev;   /* [T*k, H/2]  quantized x of the slot                 */
  uint8_t* x_scales_dev;  /* [T*k, H/16]                                        */
  float* h_dev;           /* [T*k, I]    f32 mid values before quantization      */
  uint8_t* h_codes_dev;   /* [T*k, I/2]  quantized mid values                    */
  uint8_t* h_scales_dev;  /* [T*k, I/16]                                        */
} moe_nvfp4_w4a4_taps;

int moe_nvfp4_forward_w4a4(const void* x_dev, const float* logits_dev, int64_t T,
                           const moe_nvfp4_bank* bank, const float* act_scales_dev, int32_t k,
                           void* out_dev, void* x_next_dev, void* workspace_dev,
                           size_t workspace_bytes, const moe_nvfp4_w4a4_taps* taps, void* stream);

/*
 * End-to-end call with host tensors: copies x_host [T, H] BF16 and logits_host [T, E] f32 to
 * the device, runs the layer on the resident bank, copies out [T, H] BF16 back to out_host and
 * synchronises `stream` before returning.  Host buffers may be pageable or pinned (pinned
 * copies are asynchronous and faster).  Uses the internal workspace and internal staging
 * buffers for x, logits and out.
 */
int moe_nvfp4_forward_host(const void* x_host, const float* logits_host, int64_t T,
                           const moe_nvfp4_bank* bank, int32_t k, void* out_host, void* stream);

/*
 * As moe_nvfp4_forward, but allocating nothing: the scratch comes from one fixed array of
 * MOE_NVFP4_NOALLOC_MAX_BYTES that the library places in device memory when it is loaded
 * (every device the process uses holds it until exit).  The pages this library follows have
 * no counterpart for this call; it exists for callers that cannot call cudaMalloc: runtimes
 * that reserve all device memory up front and forbid later allocations, and latency-critical
 * loops that must not pay for the device-wide synchronisation an allocation can cause.
 *  - Inputs and outputs are the caller's, as for moe_nvfp4_forward.
 *  - Calls needing more scratch than the array holds (about T*k*(H+I)*4 bytes plus routing
 *    tables; T <= 64 at E=256, k=8, H=5120, I=2560) return MOE_NVFP4_ERR_WORKSPACE and enqueue
 *    nothing.
 *  - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *    that device current; make that first call before any stream capture.
 *  - All calls share the one array and it keeps the last call's contents; nothing in it needs
 *    to start at zero (each call writes every entry it reads).  Calls whose GPU work overlaps
 *    -- different streams, or several host threads -- race on it: order them on one stream.
 */
#define MOE_NVFP4_NOALLOC_MAX_BYTES ((size_t)16 << 20)
int moe_nvfp4_forward_noalloc(const void* x_dev, const float* logits_dev, int64_t T,
                              const moe_nvfp4_bank* bank, int32_t k, void* out_dev, void* stream);

/*
 * Routing only (router + permutation), for inspection:
 *  ids_dev [T, k] int32 expert ids in rank order;   w_dev [T, k] f32 softmax weights;
 *  counts_dev [E] int32;  offsets_dev [E+1] int32 exclusive prefix sum of counts;
 *  perm_dev [T*k] int32: position p holds the routed row r = t*k + j, expert by expert,
 *           ascending r inside an expert;   inv_dev [T*k] int32 with perm[inv[r]] = r.
 * Ranking key: larger logit first, ties to the lower index, -0.0 equal to +0.0, NaN below
 * -inf.  Scratch comes from the internal workspace.
 */
int moe_nvfp4_route(const float* logits_dev, int64_t T, int32_t E, int32_t k, int32_t* ids_dev,
                    float* w_dev, int32_t* counts_dev, int32_t* offsets_dev, int32_t* perm_dev,
                    int32_t* inv_dev, void* stream);

/*
 * Experts only: y_rows[r] = Wd_e (silu(Wg_e x) * (Wu_e x)) for row r of x_rows with e =
 * expert_ids[r], in f32, unweighted -- the routed-expert step of the layer without the router
 * and the combine, for expert parallelism (a rank runs its own experts on the rows other ranks
 * send it; the layer's method statement is moe_nvfp4_forward's).  x_rows_dev [R, H] BF16,
 * expert_ids_dev [R] int32 in any order, y_rows_dev [R, H] f32.  An id outside [0, E) marks a
 * padding row: its y row is zero and it costs no expert work.  The same expert kernels as the
 * layer (path as in moe_nvfp4_forward_ex with T = R, k = 1): for a row, the result is the one
 * the layer computes for that row and expert on the same path.  workspace_dev: NULL for the
 * internal workspace, else at least moe_nvfp4_experts_workspace_bytes(...) bytes, 256-byte
 * aligned.  R = 0 returns OK.  flags: 0, or MOE_NVFP4_EXPERTS_SORTED when the caller knows the
 * ids are non-decreasing and all in [0, E) (rows already in expert order, as an expert-major
 * receive buffer holds them): the results are then written in place, saving one pass over y
 * (with unsorted ids the flag leaves rows in the wrong places, within y_rows).
 */
#define MOE_NVFP4_EXPERTS_SORTED 1
int moe_nvfp4_experts(const void* x_rows_dev, const int32_t* expert_ids_dev, int64_t R,
                      const moe_nvfp4_bank* bank, float* y_rows_dev, void* workspace_dev,
                      size_t workspace_bytes, int32_t path, int32_t flags, void* stream);
size_t moe_nvfp4_experts_workspace_bytes(int64_t R, int32_t E, int32_t H, int32_t I,
                                         int32_t path);

/*
 * Expert parallelism (EP) over G ranks, one process per GPU.  Source: the official deployment of
 * the model runs tensor and expert parallelism over eight GPUs (page "Beam 1.0 501B", the
 * model-information page's introduction: TP8/EP8); the workstation recipe uses tensor
 * parallelism over four (page "Running Beam-1.0 (501B) on workstation GPUs", its serving
 * command).  The layer is the one of moe_nvfp4_forward;
 * EP only changes where each expert runs.  Rank d holds global experts d*El .. d*El+El-1
 * (El = E / G) as a bank of El records (a moe_nvfp4_bank whose base points at record d*El of the
 * full bank layout) and routes its own tokens over all E with moe_nvfp4_route (ids, w, counts,
 * offsets, perm, inv).  counts_all [G][E] int32 is every rank's counts, row s from rank s (an
 * all-gather the caller performs).  One step, on every rank:
 *   route -> all-gather counts -> ep_plan -> ep_dispatch -> barrier -> moe_nvfp4_experts on the
 *   rows received (recv_ids as expert ids) -> barrier -> ep_combine.
 * The barriers are the caller's (any stream-ordered cross-rank barrier, e.g. an all-reduce of
 * one element); dispatch ends with a system-scope fence so that a barrier after it publishes its
 * peer stores.  Receive buffers: rank d's recv_x [Rd, H] BF16 and recv_y [Rd, H] f32, with Rd =
 * sum over s of counts_all[s][d*El .. d*El+El-1] (the rows the plan sends there), allocated with
 * moe_nvfp4_ep_buffer_create and opened in every other rank's process with
 * moe_nvfp4_ep_buffer_open; the caller checks Rd against their capacity before dispatching.
 */
#define MOE_NVFP4_EP_EXPERT_MAJOR 0   /* rank d's rows: for e, the rows from rank 0, 1, ...   */
#define MOE_NVFP4_EP_SOURCE_MAJOR 1   /* rank d's rows: from rank 0 (expert by expert), 1, ... */

/*
 * From counts_all_dev [G][E]: dst_off_dev [E], the row of the owner's buffer (layout as given)
 * that receives this rank's first row of global expert g (the others follow in the order of
 * perm), and recv_ids_dev [recv_rows], the local expert (0 .. El-1) of each row of this rank's
 * buffer, -1 for rows past the ones the count matrix sends here.  SOURCE_MAJOR is the order an
 * all-to-all of the rows gathered in perm order delivers (moe_nvfp4_gather_rows, then each
 * rank's share of them in rank order).  One launch; E % G == 0, G <= 64.
 */
int moe_nvfp4_ep_plan(const int32_t* counts_all_dev, int32_t ranks, int32_t num_experts,
                      int32_t rank, int32_t layout, int32_t* dst_off_dev, int32_t* recv_ids_dev,
                      int64_t recv_rows, void* stream);

/*
 * Stores every routed row of this rank (x_dev [T, H] BF16; routed row r = t*k+j) into the
 * receive buffer of the owner of g = ids[r], at row dst_off[g] + (inv[r] - offsets[g]) of an
 * EXPERT_MAJOR plan; each token's row is read once and stored k times.  recv_x_ptrs_host: host
 * array of G device pointers valid in this process (this rank's own buffer, the others opened
 * with moe_nvfp4_ep_buffer_open), each 16-byte aligned.  ids, inv and offsets are
 * moe_nvfp4_route's for this rank's tokens.
 * capacity_rows: rows every receive buffer holds; a row whose place falls outside
 * [0, capacity_rows) is not stored (a plan from counts that do not match the routing).
 */
int moe_nvfp4_ep_dispatch(const void* x_dev, int64_t T, int32_t k, int32_t hidden,
                          int32_t num_experts, const int32_t* ids_dev, const int32_t* inv_dev,
                          const int32_t* offsets_dev, const int32_t* dst_off_dev, int32_t ranks,
                          void* const* recv_x_ptrs_host, int64_t capacity_rows, void* stream);

/*
 * out_dev [T, H] BF16 = bf16(sum_j w[t, j] * y(t, j)), j ascending with f32 fused multiply-adds
 * (the layer's combine, bit for bit), where y(t, j) is row dst_off[g] + (inv[r] - offsets[g]) of
 * the recv_y buffer of the owner of g = ids[r], r = t*k+j, read over peer memory.
 * recv_y_ptrs_host: host array of G device pointers (f32 [capacity_rows, H] each); a row whose
 * place falls outside [0, capacity_rows) adds nothing.  x_next_dev as in moe_nvfp4_forward_ex
 * (x_dev is needed only with it).
 */
int moe_nvfp4_ep_combine(const void* x_dev, int64_t T, int32_t k, int32_t hidden,
                         int32_t num_experts, const int32_t* ids_dev, const float* w_dev,
                         const int32_t* inv_dev, const int32_t* offsets_dev,
                         const int32_t* dst_off_dev, int32_t ranks,
                         const float* const* recv_y_ptrs_host, int64_t capacity_rows, void* out_dev,
                         void* x_next_dev, void* stream);

/*
 * The two ends of an all-to-all exchange of the rows (for a collective library in place of the
 * peer-memory kernels): rows_dev [T*k, H] BF16 = x[perm[p] / k] (the routed rows in expert
 * order), and out = the layer's combine of y_dev [T*k, H] f32 held in that same order (row p is
 * the result of routed row perm[p]); out[t] = bf16(sum_j w[t, j] * y[inv[t*k+j]]).
 */
int moe_nvfp4_gather_rows(const void* x_dev, const int32_t* perm_dev, int64_t T, int32_t k,
                          int32_t hidden, void* rows_dev, void* stream);
int moe_nvfp4_combine(const float* y_dev, const float* w_dev, const int32_t* inv_dev, int64_t T,
                      int32_t k, int32_t hidden, const void* x_dev, void* out_dev,
                      void* x_next_dev, void* stream);

/*
 * Peer-visible buffers (CUDA IPC): create allocates `bytes` of device memory on the current
 * device and writes its 64-byte handle to handle_host; open maps another process's buffer
 * from its handle into this process (peer access over NVLink) -- a process cannot open its own
 * handle; close unmaps it, destroy frees a buffer made by create.  The caller exchanges the
 * handles (e.g. an all-gather of bytes) and keeps each buffer alive until every peer closed it.
 */
#define MOE_NVFP4_EP_HANDLE_BYTES 64
int moe_nvfp4_ep_buffer_create(uint64_t bytes, void** dev_ptr, uint8_t* handle_host);
int moe_nvfp4_ep_buffer_open(const uint8_t* handle_host, void** peer_ptr);
int moe_nvfp4_ep_buffer_close(void* peer_ptr);
int moe_nvfp4_ep_buffer_destroy(void* dev_ptr);

/*
 * NVFP4 encoder: turns BF16 weights into the bank's NVFP4 parts, so that BF16 experts can feed
 * the layer.  w_dev holds n projections [n, out_features, in_features] BF16, row-major (rows =
 * outputs); projection i is written to dst_dev + i * dst_stride: its E2M1 codes at + codes_off
 * ([out, in/8] little-endian u32 words, low nibble first), its E4M3 block scales at + scales_off
 * ([out, in/16] bytes, one per 16 inputs of a row) and its f32 global at + global_off -- with
 * the bank's record layout, one call writes one part role (gate, up or down) of n experts.
 * The rule (pages "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit residents",
 * section "What this pack holds", whose MLX block scale is e4m3(s) x (g / 2688), and "Running
 * Beam-1.0 (501B) on workstation GPUs", data-free NVFP4A16 quantization): amax = max |w| of the
 * projection, s2 = f32(amax / 2688); block scale = the E4M3 value nearest to
 * f32(amax_block / f32(6 s2)) (ties to even, saturating at 448); code = the E2M1 value nearest
 * to f32(w / f32(e4m3 x s2)) (ties to even, saturating at 6) with the sign bit of w, magnitude
 * 0 where the block scale is 0; every step one f32 operation rounded to nearest even.  The
 * stored global is s2 (global_mode 0) or g = amax (global_mode 1, the streaming pack's
 * convention: f32(g / 2688) is then exactly s2).  A projection of zeros stores 0 everywhere.
 * Inputs must be finite.  Requirements: in_features a multiple of 16; w_dev, dst_dev,
 * dst_stride and codes_off multiples of 16, global_off of 4; the three parts must not overlap
 * and (for n > 1) must lie inside dst_stride.  Nothing is allocated (the global slot holds the
 * running amax until the last of the call's four kernels).  n = 0 returns OK.
 */
int moe_nvfp4_encode(const void* w_dev, int64_t n, int32_t out_features, int32_t in_features,
                     int32_t global_mode, void* dst_dev, uint64_t dst_stride, uint64_t codes_off,
                     uint64_t scales_off, uint64_t global_off, void* stream);

/*
 * Streaming packs (page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts / MLX 8-bit
 * residents", sections "What this pack holds" and "How to run").  experts.bin holds one record
 * per (layer, expert), each starting at a multiple of 4 KiB; expert-manifest.json names the
 * format (mlx-stream-nvfp4-expert-bank-v1) and layout (nvfp4-gud-9part), the source pin, the 9
 * parts of a record, and the offset, length and sha256 of each record, plus the projections
 * whose global scale is inexact (global_scale_inexact).  The page prints these fields but not
 * the JSON schema; this library reads top-level keys "format", "layout", "layers", "experts",
 * "hidden", "intermediate", "record_bytes", "record_stride", "parts" (objects with "name" in
 * gate|up|down . codes|scales|global, "offset", "length" inside a record), "records" (objects
 * with "layer", "expert", "offset", "length", "sha256" as 64 hex digits) and
 * "global_scale_inexact" (a list).  The pack's globals follow the page's convention: a bank
 * built from it has global_mode 1 (multiplier f32(g / 2688)).
 *
 * moe_nvfp4_pack_open    parses manifest_path and opens bin_path (NULL: experts.bin beside the
 *                        manifest); checks the format and layout names, the part sizes against
 *                        hidden and intermediate, 4 KiB-aligned record offsets inside the file.
 *                        *pack receives an opaque handle (host memory owned by the library until
 *                        moe_nvfp4_pack_close).  Needs no GPU.
 * moe_nvfp4_pack_get_info fills the geometry (below).
 * moe_nvfp4_pack_verify  recomputes the sha256 of every record of `layer` (-1: all layers) on
 *                        `threads` host threads (0: one per core); *bad receives the number of
 *                        records whose digest differs, and MOE_NVFP4_ERR_INTEGRITY is returned
 *                        if any does.  Needs no GPU.
 * moe_nvfp4_pack_load    copies the records (layer, experts[i]) for i < n (experts NULL: every
 *                        expert of the layer in order, n ignored) to dst_dev + i * dst_stride:
 *                        file -> pinned staging buffers (a ring, reused once its copy is done)
 *                        -> cudaMemcpyAsync on `stream`; with verify != 0 each record's sha256 is
 *                        checked before its copy and a mismatch stops the load with
 *                        MOE_NVFP4_ERR_INTEGRITY.  dst_stride >= record_bytes, multiple of 16.
 *                        Returns once every copy is enqueued.
 */
typedef struct moe_nvfp4_pack_info {
  int32_t layers, experts, hidden, intermediate;
  uint64_t record_bytes, record_stride;           /* record size and spacing in experts.bin */
  uint64_t codes_off[3], scales_off[3], global_off[3];  /* gate, up, down parts in a record */
  int32_t global_mode;                            /* 1: the pack stores g, multiplier f32(g/2688) */
  int32_t inexact_globals;                        /* entries of global_scale_inexact           */
} moe_nvfp4_pack_info;

int moe_nvfp4_pack_open(const char* manifest_path, const char* bin_path, void** pack);
int moe_nvfp4_pack_get_info(const void* pack, moe_nvfp4_pack_info* info);
int moe_nvfp4_pack_verify(void* pack, int32_t layer, int32_t threads, int64_t* bad);
int moe_nvfp4_pack_load(void* pack, int32_t layer, const int32_t* experts_host, int32_t n, void* dst_dev,
                        uint64_t dst_stride, int32_t verify, void* stream);
int moe_nvfp4_pack_close(void* pack);

/* SHA-256 (FIPS 180-4) of len bytes of host memory into digest_host[32]; the digest the pack
 * loader checks records with.  Needs no GPU. */
int moe_nvfp4_sha256(const void* data_host, uint64_t len, uint8_t* digest_host);

/*
 * Expert rows: a bounded cache of one layer's expert records on the GPU, fed from a pack (the
 * page's "rows": the expert slots the GPU keeps per routed layer, filled from experts.bin as the
 * router selects experts).  A layer whose experts do not all fit in device memory runs through
 * its rows:
 *  moe_nvfp4_rows_create   allocates `slots` record slots on the current device (slots <= E,
 *                          <= 256 for the single-token kernel), a copy stream and pinned staging.
 *  moe_nvfp4_rows_forward  the layer on x_dev [T, H] / logits_dev [T, E] (finite logits) into
 *                          out_dev [T, H]: routes on the GPU, reads back which experts were
 *                          selected (one synchronisation of `stream`), loads the missing ones
 *                          into free slots or the least recently used slots that this call does
 *                          not need (file -> pinned staging -> the cache's copy stream, which
 *                          `stream` then waits for), and runs the layer on the slots: each
 *                          token's logits are mapped onto the slots (selected experts keep their
 *                          logit, every other slot gets -inf), so the routing, the weights and
 *                          the output are those of the full layer.  A call that selects more
 *                          experts than there are slots returns MOE_NVFP4_ERR_UNSUPPORTED.
 *                          One stream at a time per cache; not capturable (it synchronises).
 *  moe_nvfp4_rows_stats    hits and misses (selected experts found resident / loaded) and bytes
 *                          loaded since creation.
 *  moe_nvfp4_rows_destroy  frees the cache (synchronises its streams).
 * The pack must stay open while a cache made from it exists.
 */
int moe_nvfp4_rows_create(void* pack, int32_t layer, int32_t slots, void** rows);
int moe_nvfp4_rows_forward(void* rows, const void* x_dev, const float* logits_dev, int64_t T, int32_t k,
                           void* out_dev, void* stream);
int moe_nvfp4_rows_stats(const void* rows, int64_t* hits, int64_t* misses, int64_t* bytes_loaded);
int moe_nvfp4_rows_destroy(void* rows);

/* Bytes of caller workspace moe_nvfp4_forward_ex needs for these sizes and path (AUTO
 * gives the size of the path AUTO would take).  Returns 0 for invalid sizes. */
size_t moe_nvfp4_workspace_bytes(int64_t T, int32_t E, int32_t k, int32_t H, int32_t I,
                                 int32_t path);

/* Message for the last non-OK status returned to the calling host thread ("" if none). */
const char* moe_nvfp4_last_error(void);

/*
 * Reads and clears the current device's sticky kernel status (synchronises the device):
 * MOE_NVFP4_OK, or MOE_NVFP4_ERR_TIMEOUT if a bounded wait inside a kernel gave up since the
 * last call.  A timeout means the kernel returned early and its outputs are invalid; the
 * persistent decode kernels' counter sets are then cleared so that later calls start clean.
 */
int moe_nvfp4_device_status(void);

/* Number of kernels the last successful compute call on this host thread enqueued. */
int moe_nvfp4_last_launch_count(void);

/* Kernel kinds reported by moe_nvfp4_profile_end. */
#define MOE_NVFP4_KERNEL_ROUTE          0  /* router + permutation (1 or 3 kernels)   */
#define MOE_NVFP4_KERNEL_DECODE_GATEUP  1
#define MOE_NVFP4_KERNEL_DECODE_DOWN    2
#define MOE_NVFP4_KERNEL_COMBINE        3
#define MOE_NVFP4_KERNEL_PREFILL_GATHER 4
#define MOE_NVFP4_KERNEL_PREFILL_GATEUP 5
#define MOE_NVFP4_KERNEL_PREFILL_DOWN   6
#define MOE_NVFP4_KERNEL_DECODE_FUSED   7  /* single-token decode: the whole layer in one kernel */
#define MOE_NVFP4_KERNEL_W4A4_QUANT     8  /* W4A4: quantize the routed rows of x            */
#define MOE_NVFP4_KERNEL_W4A4_GATEUP    9
#define MOE_NVFP4_KERNEL_W4A4_DOWN     10
#define MOE_NVFP4_KERNEL_KINDS         11

/*
 * Kernel timing for benchmarks.  Between moe_nvfp4_profile_begin() and
 * moe_nvfp4_profile_end(), every kernel kind a compute call launches on the calling host
 * thread is bracketed by two CUDA events recorded on the call's stream (also while the stream
 * is capturing into a CUDA graph: the events become event-record nodes and hold the times of
 * the graph's latest replay).  moe_nvfp4_profile_end() synchronises on the events and writes,
 * for each kind, the summed milliseconds into ms[kind] and the number of bracketed launches
 * into launches[kind], for kinds < n; both arrays are caller-owned host memory.
 */
int moe_nvfp4_profile_begin(void);
int moe_nvfp4_profile_end(double* ms, int64_t* launches, int32_t n);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MOE_NVFP4_H_ */
