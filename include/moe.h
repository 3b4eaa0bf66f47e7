/*
 * moe.h -- C ABI of libmoe: the per-layer quantized Mixture-of-Experts step
 * (route -> permute -> block-quantized SwiGLU experts -> combine) and the
 * frequency-driven expert cache, for NVIDIA B200 (sm_100a).
 *
 * Sources (web pages on running large MoE models on small GPUs):
 *  - Strata article (tech.hub77a.com), 30-second summary and section 2
 *    items 1-3: 10 of 24,576 experts active per token; hot experts resident
 *    in VRAM, all experts in RAM; a routed expert that is resident is
 *    computed at once, the others must first be moved in; verify passes of
 *    drafted tokens; prompt chunks of up to 8,192 tokens.
 *  - Strata code review (qaqmin.com), sections 1, 3, 4: CUDA MoE and
 *    dequantisation kernels, an expert cache, a page-locked stage buffer,
 *    512 experts per layer.
 *  - 27B dense report (trawling.dev), model-file paragraph: a Q4_0 value
 *    costs 0.5625 B (32 four-bit codes + one fp16 scale); Strata article,
 *    summary table: the Q2_0 size.
 *  - Janas-LLM page (onedev.kr): a RAM expert cache keeps experts that are
 *    used again.
 *
 * Conventions shared by every call
 *  - Pointers named "device" are CUDA device pointers; "host" are CPU
 *    pointers.  The caller owns all memory; the library allocates only
 *    host-side handle state (expert cache) and never calls cudaMalloc.
 *  - Compute calls are asynchronous on the caller's cudaStream_t (0 = the
 *    legacy default stream).  They validate arguments on the host before
 *    launching anything and return a status; nothing throws or aborts.
 *  - Device buffers must be 16-byte aligned unless stated otherwise.
 *  - Status: MOE_OK (0) on success; on failure one of the positive codes
 *    below and a message readable with moe_last_error() (thread-local, valid
 *    until the next call on the same thread).
 *  - Kernels never trap.  Problems found on the device (an expert id out of
 *    range, a missing expert blob, a non-finite selected logit) set a
 *    per-device error word that moe_device_error() reads.
 *
 * Expert blob (one contiguous buffer per expert, "b" = 4 or 2 bits):
 *    codes Wg [I][H/32][4b B], codes Wu [I][H/32][4b B], codes Wd [H][I/32][4b B],
 *    scales Wg [I][H/32], Wu [I][H/32], Wd [H][I/32] as IEEE fp16.
 *  A weight is d * (q - 2^(b-1)).  4-bit block: element i in byte i%16, low
 *  nibble for i < 16, high nibble otherwise.  2-bit block: element i in byte
 *  i%8 at bit 2*(i/8).  Wg, Wu map hidden H -> intermediate I, Wd maps back.
 *  Blob pointers must be 16-byte aligned.  Shapes: H and I multiples of 128.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t;   /* same type as cudaStream_t */

/* status codes */
#define MOE_OK 0
#define MOE_EINVAL 1      /* bad argument (shape, pointer, alignment, workspace size) */
#define MOE_ENOMEM 2      /* host allocation failed */
#define MOE_ECUDA 3       /* a CUDA runtime call failed */
#define MOE_EBUSY 4       /* expert cache: not enough evictable slots */
#define MOE_ETIMEDOUT 5   /* expert cache: wait ran out of time */
#define MOE_EIO 6         /* expert cache: a staging copy failed */
#define MOE_EDEVICE 7     /* the device error word was set */

/* activation / router dtypes */
#define MOE_F32 0
#define MOE_BF16 1

/* expert FFN modes */
#define MOE_MODE_AUTO 0   /* GEMV when T <= 16 and the shape suits it, else GEMM */
#define MOE_MODE_GEMV 1   /* CUDA-core kernels, fp32 math, any T (slow for large T) */
#define MOE_MODE_GEMM 2   /* tcgen05 tensor-core grouped GEMM, fp16 operands */

/* device error word bits (moe_device_error) */
#define MOE_DEVERR_BAD_EXPERT 1u     /* expert id outside [0, E) */
#define MOE_DEVERR_NULL_BLOB 2u      /* an active expert had no blob pointer */
#define MOE_DEVERR_NONFINITE 4u      /* a selected logit was NaN or +inf */
#define MOE_DEVERR_BAD_ROW 8u        /* offsets/perm_src inconsistent */
#define MOE_DEVERR_TIMEOUT 16u       /* a bounded in-kernel wait ran out */
#define MOE_DEVERR_MISALIGNED 32u    /* an expert blob pointer was not 16-byte aligned */

/* Thread-local message of the last failing call ("" if none). */
const char *moe_last_error(void);

/* Library version (major * 10000 + minor * 100 + patch). */
int moe_version(void);

/* Build variant of the loaded library: MOE_BUILD_DEBUG set for the MOE_DEBUG
 * build (python -m quantized_expert_ffn_route_b200.build --debug, output in
 * _build_debug/), in which every index read from a caller's buffer before it
 * addresses memory (permutation entries, the active-expert count, expert ids
 * and row ranges of the tensor-core path) also sets its MOE_DEVERR_* bit when
 * it is out of range.  Every build keeps such an index in range (it becomes 0,
 * or the group is skipped); only the debug build reports it. */
#define MOE_BUILD_DEBUG 1
int moe_build_flags(void);

/* Number of kernel launches this library has issued in this process (host-side
 * count; launches recorded into a CUDA graph are counted once, at capture). */
uint64_t moe_kernel_launches(void);

/* Reads the calling device's error word after synchronizing `s`; clears it if
 * `clear` != 0.  *bits_out receives MOE_DEVERR_* bits.  Returns MOE_OK, or
 * MOE_EDEVICE if any bit was set, or MOE_ECUDA. */
int moe_device_error(uint32_t *bits_out, int clear, moe_stream_t s);

/* Test hooks: settings that only tests change, to drive bounded in-kernel
 * waits into their timeout path without a GPU fault.  Process-wide; read
 * when a call launches its kernels; 0 restores the default.  Returns
 * MOE_EINVAL for an unknown hook or a negative value.
 *  MOE_HOOK_WAIT_LIMIT_NS         time limit of the fused decode kernel's
 *                                 waits (grid barriers, copies); default 1 s.
 *  MOE_HOOK_DECODE_EXTRA_ARRIVALS arrivals the fused decode kernel's grid
 *                                 barriers wait for beyond its own CTAs, so
 *                                 a value > 0 makes every barrier time out.
 *  MOE_HOOK_GEMM_SPIN             polls before a grouped-GEMM mbarrier wait
 *                                 gives up; default 4,194,304 (about a
 *                                 second).
 *  MOE_HOOK_DECODE_ONE_KERNEL     1: moe_layer_decode runs the one-kernel
 *                                 persistent step where it applies instead
 *                                 of the three-kernel chain (to test and
 *                                 time both). */
#define MOE_HOOK_WAIT_LIMIT_NS 1
#define MOE_HOOK_DECODE_EXTRA_ARRIVALS 2
#define MOE_HOOK_GEMM_SPIN 3
#define MOE_HOOK_DECODE_ONE_KERNEL 4
int moe_test_hook(int which, int64_t value);

/* Bytes of one expert blob (see layout above). */
size_t moe_expert_blob_bytes(int bits, int H, int I);

/* ------------------------------------------------------------------ route
 * Router logits and top-k gate (Strata article, summary table and section 2
 * item 2: 10 of 24,576 experts per token; the router's choice decides the
 * compute path).
 *   l[t,e]  = sum_h x[t,h] * w_router[e,h] (+ bias[e]), fp32 accumulation
 *             (bf16 x and w_router with T >= 64 and H % 64 == 0: a tensor-core
 *             bf16 GEMM, fp32 accumulation; else CUDA-core dot products);
 *             or, when w_router == NULL, l = logits_in [T,E] fp32 (device).
 *   ids[t,:] = the k experts first in the order (l descending, id ascending);
 *             NaN ranks below -inf.
 *   w[t,j]  = exp(l_j - l_0) / sum_i exp(l_i - l_0) over the k selected.
 *  x        device [T,H], dtype x_dtype (MOE_F32 | MOE_BF16), row-major.
 *  w_router device [E,H], dtype w_dtype, row-major; NULL -> use logits_in.
 *  bias     device [E] fp32 or NULL (added to logits from x, not to logits_in).
 *  topk_ids device [T,k] int32 out.  topk_w device [T,k] fp32 out.
 *  logits_out device [T,E] fp32 out, or NULL.
 *  ws       device workspace of at least moe_route_ws_size(T,E,k) bytes:
 *           the logits when they are computed here and logits_out is NULL,
 *           and, when E > 1024, the chunked top-k's candidates (so with
 *           E > 1024 ws is needed even with logits_in or logits_out).
 * Limits: 1 <= k <= min(E, 32), 1 <= E <= 32768, T >= 0.  T = 0 is a no-op.
 * A selected NaN/+inf logit sets MOE_DEVERR_NONFINITE and yields NaN gates. */
size_t moe_route_ws_size(int T, int E, int k);
int moe_route_topk(const void *x, int x_dtype, const void *w_router, int w_dtype,
                   const float *logits_in, const float *bias, int T, int H, int E, int k,
                   int32_t *topk_ids, float *topk_w, float *logits_out,
                   void *ws, size_t ws_bytes, moe_stream_t s);

/* ---------------------------------------------------------------- permute
 * Token-to-expert permute: a stable counting sort of the T*k (token, slot)
 * pairs by expert id, so each expert's rows are contiguous and in ascending
 * token order.
 *  expert_offsets device [E+1] out: exclusive prefix sum of per-expert counts.
 *  perm_src device [T*k] out: row -> token index.
 *  perm_dst device [T*k] out: (t*k + j) -> row.
 *  active   device [1 + min(E, T*k)] out or NULL: number of experts with rows,
 *           then those expert ids ascending.
 * An id outside [0, E) sets MOE_DEVERR_BAD_EXPERT; the outputs are then
 * unspecified.  ws: at least moe_permute_ws_size(T,k,E) bytes. */
size_t moe_permute_ws_size(int T, int k, int E);
int moe_permute(const int32_t *topk_ids, int T, int k, int E, int32_t *expert_offsets,
                int32_t *perm_src, int32_t *perm_dst, int32_t *active,
                void *ws, size_t ws_bytes, moe_stream_t s);

/* ------------------------------------------------------------- expert FFN
 * Block-quantized SwiGLU experts over the permuted rows:
 *   y_perm[r] = Wd_e (silu(Wg_e x_t) * (Wu_e x_t)),  t = perm_src[r],
 *   for every row r of every expert e listed in `active` (offsets give the
 *   rows), and, if shared_blob != NULL, y_shared[t] = the same FFN of the
 *   shared expert for every token t (Strata code review, section 1: CUDA MoE
 *   and dequantisation kernels; the shared expert is a reading).
 * Weights are dequantised on the fly from the blobs (never materialised in
 * HBM).  GEMV mode: fp32 arithmetic throughout.  GEMM mode: weights and
 * activations as fp16 tensor-core operands with fp32 accumulation; the
 * intermediate h is rounded to fp16.
 *  expert_blobs device array [E] of device blob pointers (expert id -> blob);
 *           entries of experts that are not active are not read.
 *  expert_offsets, active, perm_src: as produced by moe_permute.  Rows of
 *           experts absent from `active` are left untouched in y_perm.
 *  x        device [T,H] dtype x_dtype.
 *  y_perm   device [T*k, H] fp32 out.  y_shared device [T,H] fp32 out (or
 *           NULL when shared_blob is NULL).
 *  mode     MOE_MODE_AUTO | _GEMV | _GEMM.  GEMV needs H <= 2048 and I/32
 *           (4-bit) or I/64 (2-bit) in {2, 4, 8, 16, 32}; GEMM needs at most
 *           4095 groups (min(E, T*k) + shared).  Else MOE_EINVAL.
 *  ws       at least moe_expert_ffn_ws_size(bits,T,k,H,I,E,mode) bytes.
 * _q4 reads 4-bit blobs, _q2 2-bit blobs. */
size_t moe_expert_ffn_ws_size(int bits, int T, int k, int H, int I, int E, int mode);
int moe_expert_ffn_q4(const void *const *expert_blobs, const int32_t *expert_offsets,
                      const int32_t *active, const int32_t *perm_src, const void *x,
                      int x_dtype, int T, int k, int H, int I, int E,
                      const void *shared_blob, float *y_perm, float *y_shared, int mode,
                      void *ws, size_t ws_bytes, moe_stream_t s);
int moe_expert_ffn_q2(const void *const *expert_blobs, const int32_t *expert_offsets,
                      const int32_t *active, const int32_t *perm_src, const void *x,
                      int x_dtype, int T, int k, int H, int I, int E,
                      const void *shared_blob, float *y_perm, float *y_shared, int mode,
                      void *ws, size_t ws_bytes, moe_stream_t s);

/* ------------------------------------------------------- fused decode step
 * The whole step for ONE token: router logits (or logits_in), top-k + gates,
 * the k routed experts and the shared expert, and the combine
 *   y = sum_{j<k} w_j * FFN_{ids_j}(x) + FFN_shared(x)    (fp32, slot order),
 * with the same definitions as moe_route_topk -> moe_permute ->
 * moe_expert_ffn_q4/q2 (GEMV mode) -> moe_combine (Strata article, section 2
 * item 2: only the experts the router picks are computed; at one token the
 * step is bound by streaming those experts' weights).
 * The step runs as three kernels chained with programmatic dependent launch:
 * route (router logits, then the last of its CTAs selects the top-k, computes
 * the gates and publishes the selected blob pointers), gate/up (the shared
 * expert's CTAs start before the route kernel ends; every CTA prefetches its
 * share of its expert's down matrix into L2) and down + combine.  With the
 * test hook MOE_HOOK_DECODE_ONE_KERNEL set, shapes with H and I multiples of
 * 256, H <= 2048, I / (32 for 4-bit, 64 for 2-bit) in {4, 8, 16, 32} and a
 * per-SM share of the weights that fits in shared memory run instead as ONE
 * persistent kernel (one CTA per SM, launched cooperatively so all CTAs are
 * resident) with two grid-wide barriers kept in the workspace; on B200 it is
 * the slower of the two.
 *  x [H] (x_dtype), w_router [E,H] (w_dtype) or NULL with logits_in [E];
 *  expert_blobs device [E] blob pointers (16-byte aligned; a misaligned one
 *  sets MOE_DEVERR_MISALIGNED and that expert is left out); shared_blob or
 *  NULL; topk_ids [k] int32 out, topk_w [k] fp32 out, logits_out [E] or NULL
 *  (written only when the logits are computed here), y [H] fp32 out.
 *  ws: moe_layer_decode_ws_size() bytes of scratch.  It must be zero-filled
 *  before its first use (cudaMemsetAsync once): it holds the route kernel's
 *  ticket count and the one-kernel step's barrier count, which every call
 *  leaves ready for the next.  After a call that set MOE_DEVERR_TIMEOUT (a
 *  grid barrier or copy wait of the one-kernel step ran out) zero it again.
 *  Calls sharing one ws must not overlap.
 * Supported shapes (else MOE_EINVAL: use the separate calls): E <= 1024,
 * k <= 32, H <= 2048 and a multiple of 128, I a multiple of 128 with I/32
 * (4-bit) or I/64 (2-bit) in {4, 8, 16, 32}, and the down kernel's tasks,
 * (k + 1) * (rows per block) / (32 / that number), at most 64 (rows per
 * block 8 when k + 1 <= 16, else 4). */
size_t moe_layer_decode_ws_size(int E, int k, int I);
int moe_layer_decode(int bits, const void *x, int x_dtype, const void *w_router, int w_dtype,
                     const float *bias, const float *logits_in, const void *const *expert_blobs,
                     const void *shared_blob, int H, int I, int E, int k, int32_t *topk_ids,
                     float *topk_w, float *logits_out, float *y, void *ws, size_t ws_bytes,
                     moe_stream_t s);

/* ------------------------------------------------------ decode session
 * moe_layer_decode for a serving loop with host buffers: at creation the
 * host->device copy of x_host, the fused step (router logits from w_router,
 * top-k, experts, combine) and the device->host copies of y (and of the ids
 * when ids_host is given) are recorded once into a CUDA graph on stream `s`
 * (after one eager call that checks every argument as moe_layer_decode does
 * and zero-fills ws); each moe_decode_session_run replays it and returns when
 * y_host holds the step's output.  x_host [H] (x_dtype) and y_host [H] fp32
 * (ids_host [k] int32 or NULL) are page-locked host buffers the caller
 * fills / reads between runs; x_dev [H], ids_dev [k], w_dev [k], y_dev [H] and
 * ws (moe_layer_decode_ws_size bytes) are device buffers; all stay owned by
 * the caller and must outlive the session.  `s` must not be the legacy
 * default stream.  Runs of one session must not overlap. */
typedef struct moe_decode_session moe_decode_session;
int moe_decode_session_create(int bits, const void *x_host, int x_dtype, const void *w_router, int w_dtype,
                              const float *bias, const void *const *expert_blobs, const void *shared_blob,
                              int H, int I, int E, int k, float *y_host, int32_t *ids_host, void *x_dev,
                              int32_t *ids_dev, float *w_dev, float *y_dev, void *ws, size_t ws_bytes,
                              moe_stream_t s, moe_decode_session **out);
int moe_decode_session_run(moe_decode_session *ds);
void moe_decode_session_destroy(moe_decode_session *ds);

/* ------------------------------------------------- allocation-free FFN
 * The pages have no counterpart of this call; it serves callers that cannot
 * allocate device memory when they run the step: engines held to a device
 * memory budget fixed at start-up, C hosts with no device allocator to hand
 * out a workspace, and latency-critical loops where an allocation could
 * synchronise the device.
 * Same computation and arguments as moe_expert_ffn_q4/q2 in MOE_MODE_GEMV
 * (bits = 4 or 2 selects the blob format), but without ws/ws_bytes: the
 * scratch (the fp32 intermediate h, T*(k+1)*I*4 bytes) comes from one array
 * built into the library of moe_expert_ffn_noalloc_max_bytes() bytes (8 MiB),
 * which every GPU that loads the library holds until the process exits.
 *  - Calls whose scratch, T*(k+1)*I*4 bytes, exceeds that size, H/I outside
 *    [128, 2048], or an I
 *    that GEMV mode does not take (see above), are rejected with MOE_EINVAL
 *    before anything is launched.
 *  - It never calls cudaMalloc, cudaFree or any allocating routine.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any stream
 *    capture.  MOE_ECUDA if the lookup fails.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents (nothing in it needs to start at zero).  Calls whose kernels
 *    overlap on the GPU (other streams, other threads) race on it: serialise
 *    them. */
size_t moe_expert_ffn_noalloc_max_bytes(void);
int moe_expert_ffn_noalloc(int bits, const void *const *expert_blobs, const int32_t *expert_offsets,
                           const int32_t *active, const int32_t *perm_src, const void *x, int x_dtype,
                           int T, int k, int H, int I, int E, const void *shared_blob,
                           float *y_perm, float *y_shared, moe_stream_t s);

/* ---------------------------------------------------------------- combine
 *   y[t] = sum_{j=0}^{k-1} topk_w[t,j] * y_perm[perm_dst[t,j]] (+ y_shared[t]),
 *   summed in slot order, fp32.  y_shared may be NULL.  y device [T,H] out. */
int moe_combine(const float *y_perm, const int32_t *perm_dst, const float *topk_w,
                const float *y_shared, int T, int k, int H, float *y, moe_stream_t s);

/* ----------------------------------------------------------- expert cache
 * Frequency-driven residency of expert blobs in an HBM slab, paged in from a
 * page-locked host pool (Strata article, section 2 item 2 and section 3:
 * hot experts resident in VRAM, everything in RAM, part of the RAM pinned
 * for the GPU; Strata code review, section 3: the stage buffer; Janas-LLM:
 * repeated experts stay cached).
 * Policy, per step (one call of expcache_stage with the step's distinct ids):
 *  - at the start of step s > 0 with s % decay_period == 0, all counters halve;
 *  - each id: counter += 1, last use = s; resident -> hit; otherwise miss:
 *    the lowest free slot, else evict the resident expert not among this
 *    step's ids with the smallest (counter, last use, id); misses always enter.
 * Copies run on the cache's own stream (cudaMemcpyAsync from the pinned pool,
 * one per miss) after the work already queued on the compute stream, then a
 * tiny kernel patches the device table; expcache_join makes a stream wait for
 * all of it.  Expert blobs of hits may be used at once.
 */
typedef struct moe_expcache moe_expcache;

typedef struct {
    int32_t n_experts;      /* experts in the host pool */
    int32_t capacity;       /* HBM slots */
    int64_t blob_bytes;     /* bytes per expert (multiple of 16) */
    int64_t slot_stride;    /* bytes between slots and pool entries (>= blob_bytes, multiple of 256) */
    void *host_pool;        /* host [n_experts * slot_stride], caller-owned; page-locked unless use_staging */
    void *hbm_slab;         /* device [capacity * slot_stride], caller-owned */
    void *dev_table;        /* device [n_experts] pointers, caller-owned; set to NULL at create */
    void *stage_buffer;     /* host, page-locked, >= 2 * slot_stride bytes; used only with use_staging */
    int32_t decay_period;   /* steps between halvings; 0 = never */
    int32_t use_staging;    /* 1: pool may be pageable; copies bounce through stage_buffer (double-buffered) */
} moe_expcache_desc;

typedef struct {
    int64_t steps, hits, misses, evictions, bytes_staged;
    int32_t resident;
    int64_t prefetched;     /* experts admitted by expcache_prefetch */
} moe_expcache_stats;

/* Creates the cache (empty).  Returns MOE_EINVAL on bad descriptors. */
int expcache_create(const moe_expcache_desc *d, moe_expcache **out);
void expcache_destroy(moe_expcache *c);

/* Query only, no state change: slots_out[i] = slot of ids_host[i] or -1. */
int expcache_lookup(moe_expcache *c, const int32_t *ids_host, int n, int32_t *slots_out, int *n_miss);

/* One step: policy bookkeeping for the n distinct ids (host array), then the
 * copies of the misses.  Outputs (host, optional, n entries each): hit[i]
 * 1 = resident and usable at once, 2 = resident but admitted by
 * expcache_prefetch since the last expcache_join (its copy may still be in
 * flight: use it after expcache_join), 0 = miss; slot[i], victim[i] (-1 =
 * none).  The compute stream's work queued so
 * far is ordered before any slot is overwritten.  Returns MOE_EBUSY if
 * n > capacity, MOE_EINVAL for bad or repeated ids, MOE_EIO/MOE_ECUDA if
 * issuing a copy failed (the step's bookkeeping is then rolled back). */
int expcache_stage(moe_expcache *c, const int32_t *ids_host, int n, moe_stream_t compute,
                   int32_t *hit_out, int32_t *slot_out, int32_t *victim_out);

/* expcache_stage with the misses copied from caller-given page-locked host
 * addresses (src_host[i] for ids_host[i]; entries of hits are ignored and may
 * be NULL) instead of host_pool + id * slot_stride: the RAM tier of an
 * expert store (expstore_fetch) feeding the cache.  A miss with a NULL
 * source returns MOE_EINVAL before anything changes.  Not with use_staging. */
int expcache_stage_from(moe_expcache *c, const int32_t *ids_host, int n, const void *const *src_host,
                        moe_stream_t compute, int32_t *hit_out, int32_t *slot_out, int32_t *victim_out);

/* Loads experts expected soon (the next layer's likely experts) without a
 * use: for each id of ids_host (-1 = none), in order, a resident id is left
 * alone; otherwise it enters the lowest free slot, else the slot of the
 * resident expert smallest in (counter, last use, id) that is neither one of
 * the last expcache_stage call's ids nor on this list; if every resident
 * expert is protected the id is skipped.  Counters and last uses do not
 * change.  Copies and the table patch are queued like expcache_stage's (after
 * the compute stream's queued work); expcache_join covers them.  Outputs
 * (host, optional): slot_out[i] (-1 = not admitted), victim_out[i],
 * *n_admitted.  MOE_EINVAL for an id outside [-1, n_experts) or n > 32. */
int expcache_prefetch(moe_expcache *c, const int32_t *ids_host, int n, moe_stream_t compute,
                      int32_t *slot_out, int32_t *victim_out, int *n_admitted);

/* Makes `s` wait (cudaStreamWaitEvent) for every copy and table update issued
 * so far; experts admitted by earlier prefetches count as settled from then on
 * (expcache_stage reports them as hit 1). */
int expcache_join(moe_expcache *c, moe_stream_t s);

/* Host wait for the staged copies with a time limit; MOE_ETIMEDOUT if not done. */
int expcache_wait(moe_expcache *c, int64_t timeout_us);

/* Evicts the given resident ids (NULL/0 = nothing).  Non-resident ids are ignored. */
int expcache_evict(moe_expcache *c, const int32_t *ids_host, int n);

/* The descriptor's dev_table: device [n_experts] blob pointers (NULL = not
 * resident), for the FFN calls. */
const void *const *expcache_device_table(moe_expcache *c);

int expcache_stats(moe_expcache *c, moe_expcache_stats *out);

/* Host copy of the per-expert counters and slots (n_experts entries each; either may be NULL). */
int expcache_snapshot(moe_expcache *c, int64_t *counts_out, int32_t *slot_of_out);

/* Timing of the most recent step that staged copies: milliseconds from
 * `ref_event` (a cudaEvent_t the caller recorded with timing enabled, on the
 * cache's device) to the start of that step's first copy (*start_ms) and to
 * the end of its table update (*end_ms).  Both events must have completed
 * (synchronize first): MOE_ECUDA otherwise.  MOE_EINVAL before any step has
 * staged a copy.  Used to measure how much copy time compute hides. */
int expcache_copy_times(moe_expcache *c, const void *ref_event, float *start_ms, float *end_ms);

/* Histogram of the copy time of the steps that staged copies (first copy
 * issued -> table patched, from events on the cache's stream): bins_out[i]
 * (MOE_COPY_HIST_BINS entries) counts the steps whose copies took
 * [2^i, 2^(i+1)) microseconds, bin 0 also everything shorter and the last bin
 * everything longer.  A step is counted once its copies have completed (all
 * are after expcache_wait); *steps_out (optional) = the steps counted. */
#define MOE_COPY_HIST_BINS 24
int expcache_copy_histogram(moe_expcache *c, int64_t *bins_out, int64_t *steps_out);

/* Test hook: the next `n` copies report failure before being issued (MOE_EIO). */
int expcache_inject_copy_failures(moe_expcache *c, int n);

/* ------------------------------------------------ NVMe tier (expert store)
 * The third tier below the page-locked RAM pool: a file holding every expert
 * blob (expert e at byte offset e * slot_stride), read on demand into a RAM
 * tier of `ram_slots` slots of the caller's page-locked buffer (Strata
 * article, section 2 item 2 and its three-tier summary: experts on SSD, the
 * hot ones in RAM and VRAM; Janas-LLM page: experts read from NVMe per token
 * with O_DIRECT into a RAM cache of capped size).  Host calls only.
 * expstore_fetch makes the given experts resident in the RAM tier: the
 * missing ones are read by io_threads threads in parallel (pread; with
 * use_direct the file is opened O_DIRECT, so reads bypass the page cache --
 * then slot_stride and ram_buffer must be 4096-byte aligned and each read is
 * rounded up to whole 4096-byte blocks inside the slot), each taking the
 * least recently fetched slot that holds none of the call's ids.  It returns
 * once every read has landed.  A slot may be reused by the next fetch, so
 * copies out of it (expcache_stage_from) must have completed before then
 * (expcache_wait).  Calls on one store must not overlap.
 */
typedef struct moe_expstore moe_expstore;

typedef struct {
    const char *path;       /* the file of n_experts * slot_stride bytes (the last blob may end the file) */
    int32_t n_experts;
    int64_t blob_bytes;     /* bytes per expert */
    int64_t slot_stride;    /* bytes between experts in the file and between RAM slots (multiple of 256) */
    int32_t ram_slots;      /* experts the RAM tier holds */
    void *ram_buffer;       /* host [ram_slots * slot_stride], page-locked, caller-owned */
    int32_t io_threads;     /* concurrent reads, 1..64 */
    int32_t use_direct;     /* 1: O_DIRECT */
} moe_expstore_desc;

typedef struct {
    int64_t fetches, hits, reads, bytes_read, evictions;
    double read_seconds;    /* wall time spent waiting for reads */
} moe_expstore_stats;

/* Opens the file.  MOE_EIO if it cannot be opened (O_DIRECT on a file system
 * without it included), MOE_EINVAL if it is too short or the descriptor is bad. */
int expstore_create(const moe_expstore_desc *d, moe_expstore **out);
void expstore_destroy(moe_expstore *s);

/* ids: n distinct experts (n <= 32 and <= ram_slots, else MOE_EINVAL /
 * MOE_EBUSY).  ram_ptrs_out[i] (optional): id i's address in the RAM tier;
 * hit_out[i] (optional): 1 if it was already there.  A failed read returns
 * MOE_EIO (that expert's pointer is NULL; the others are valid). */
int expstore_fetch(moe_expstore *s, const int32_t *ids, int n, void **ram_ptrs_out, int8_t *hit_out);
int expstore_stats(moe_expstore *s, moe_expstore_stats *out);
/* Host copy of each expert's RAM slot (-1 = on the drive only), n_experts entries. */
int expstore_snapshot(moe_expstore *s, int32_t *slot_of_out);

/* ------------------------------------------ device-initiated expert staging
 * The expert cache's policy and copies on the GPU (Strata article, section 2
 * item 2: resident experts are computed at once, the others move in from
 * host memory; the host-driven expcache_* calls above are the form that
 * hands each step's ids to the host).  devcache_stage reads the step's ids
 * from DEVICE memory and enqueues, with no host synchronisation:
 *  1. one policy kernel on `compute`: the policy of expcache_stage (halving
 *     decay every decay_period steps; count += 1 and last use = step for each
 *     id in order; resident -> hit; a miss takes the lowest free slot, else
 *     the slot of the resident expert outside this step with the smallest
 *     (count, last use, id)), the device table patched at once (victims
 *     NULL, admitted misses -> their slot), and the FFN lists written;
 *  2. one copy kernel on `copy`, after the policy kernel: the admitted
 *     misses' blobs from the host pool into their slots, read by the SMs
 *     through the pool's device mapping (16-byte loads over the host link).
 * devcache_join(c, s) makes `s` wait for the copy kernel.  The sequence is
 * fixed by the host arguments alone, so a CUDA graph can hold whole steps.
 * Zero-copy compute for cold experts: with admit_min > 1 a missed expert
 * whose count (after this use) is below admit_min is not admitted; for this
 * step its table entry points at its blob in the host pool, which the
 * expert FFN in MOE_MODE_GEMV reads in place (only that mode: the other
 * paths read blobs with bulk copies, which this build keeps off host
 * memory); the next devcache_stage clears the entry.  admit_min 0 or 1:
 * every miss is admitted (the policy of expcache_stage exactly).
 */
typedef struct moe_devcache moe_devcache;

typedef struct {
    int32_t n_experts;      /* experts in the host pool */
    int32_t capacity;       /* HBM slots (<= n_experts) */
    int64_t blob_bytes;     /* bytes per expert (multiple of 16, <= 1 GiB) */
    int64_t slot_stride;    /* bytes between slots and pool entries (>= blob_bytes, multiple of 256) */
    void *host_pool;        /* host [n_experts * slot_stride], page-locked and mapped (cudaHostAlloc, or
                               cudaHostRegister with cudaHostRegisterMapped), caller-owned */
    void *hbm_slab;         /* device [capacity * slot_stride], caller-owned */
    void *dev_table;        /* device [n_experts] pointers, caller-owned; set to NULL at create */
    int32_t decay_period;   /* steps between halvings; 0 = never */
    int32_t admit_min;      /* see above; 0 or 1 = admit every miss */
    int32_t log_steps;      /* steps of per-id events kept on the device (ring) for devcache_events; 0 = none */
} moe_devcache_desc;

typedef struct {
    int64_t steps, hits, misses, evictions;
    int64_t in_place;       /* misses computed in place (not admitted) */
    int64_t bytes_copied;   /* bytes of admitted misses */
    int64_t bad_steps;      /* steps whose ids were out of range or repeated (nothing changed) */
} moe_devcache_stats;

/* Creates the cache (empty, every table entry NULL); synchronises the device.
 * MOE_EINVAL on a bad descriptor (including a host_pool the device cannot
 * address), MOE_ENOMEM/MOE_ECUDA on allocation failures. */
int devcache_create(const moe_devcache_desc *d, moe_devcache **out);
void devcache_destroy(moe_devcache *c);

/* One step.  ids_dev: device int32 [n] (n <= 32, n <= capacity, else
 * MOE_EINVAL / MOE_EBUSY), the step's distinct ids, each offset by id_base
 * into the pool (a layer's experts id_base .. id_base + E_l - 1).  act_dev:
 * device int32 [66] out, two active-expert lists in the layout the expert
 * FFN takes: act_dev[0] = n_a, act_dev[1..n_a] the ids (without id_base) of
 * the hits and of experts computed in place -- usable at once; act_dev[33] =
 * n_b, act_dev[34..33+n_b] the admitted misses -- usable on a stream after
 * devcache_join.  Ids that are out of range or repeated set
 * MOE_DEVERR_BAD_EXPERT and leave both lists empty and the cache unchanged.
 * compute and copy may be the same stream; when they differ, the previous
 * step must have been joined (devcache_join) first, else MOE_EINVAL. */
int devcache_stage(moe_devcache *c, const int32_t *ids_dev, int n, int32_t id_base, int32_t *act_dev,
                   moe_stream_t compute, moe_stream_t copy);

/* Makes `s` wait for the copy kernel of the last devcache_stage. */
int devcache_join(moe_devcache *c, moe_stream_t s);

/* Host copies (after a device synchronisation) of the logged events of steps
 * [first_step, first_step + n_steps): per step 32 entries, entry j for the
 * step's j-th id: hit 1 = hit, 0 = admitted miss, 3 = computed in place;
 * slot (-1 if none), victim (-1 if none).  The steps must still be in the
 * log ring of log_steps steps, else MOE_EINVAL.  Any output may be NULL. */
int devcache_events(moe_devcache *c, int64_t first_step, int n_steps, int8_t *hit_out, int32_t *slot_out,
                    int32_t *victim_out);

/* Counters (a synchronous copy from the device). */
int devcache_stats(moe_devcache *c, moe_devcache_stats *out);

/* Host copies of the per-expert counts and slots (n_experts entries each; either may be NULL). */
int devcache_snapshot(moe_devcache *c, int64_t *counts_out, int32_t *slot_of_out);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
