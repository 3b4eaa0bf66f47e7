// The whole MoE step for one decode token as ONE persistent kernel: one CTA
// per SM, all CTAs resident at once (cooperative launch), two grid-wide
// barriers.
//
// At one token the step moves ~21.6 MB (router rows + 10 routed experts + the
// shared expert, 4-bit) and does little arithmetic, so what costs time is the
// chain of dependent DRAM round trips: logits -> top-k -> expert weights ->
// h -> down weights.  The kernel keeps that chain to two round trips of data
// plus two grid barriers:
//
//   A  every CTA stages x in shared memory (in natural order for the router
//      and as the pieces the dequantising dot products read), issues bulk
//      copies (cp.async.bulk, completion counted on an mbarrier) of its share
//      of the shared expert's rows -- they do not depend on the routing --
//      then computes its share of the router logits, eight warps per router
//      row, each over one eighth of H, the eight partial sums added in a
//      fixed order, and publishes them;                     grid barrier 1
//   B  every CTA selects the top-k from the E logits itself (a merge tree:
//      each warp sorts 32 keys with a bitonic network, sorted lists of 16
//      merge pairwise), looks the k blobs up in a copy of the expert table
//      staged in shared memory, and issues bulk copies of ALL its remaining
//      weights at once: its slice of the routed gate/up rows (in chunks of 8
//      rows, one mbarrier each, each chunk's copies issued by lane 0 of its
//      own warp so that issue is spread over the CTA) and its output rows of
//      every routed down matrix.  Each CTA's share is ~130 KB, so the whole
//      ~19.5 MB of expert weights is in flight together;
//   C  each warp takes gate/up units (one row of W_g and W_u of one group) as
//      their chunk lands: h = silu(W_g x) * (W_u x), written to the
//      workspace;                                             grid barrier 2
//   D  one warp per group holds its slice of h_g (from L2) in registers and
//      computes the CTA's output rows of W_d,g . h_g from the down rows that
//      arrived during C; y[r] = sum_j w_j (W_d,e_j[r] . h_j) + W_d,shared[r] .
//      h_s is summed in slot order (the combine).
//
// This path is opt-in (moe_test_hook MOE_HOOK_DECODE_ONE_KERNEL): on B200 the
// three-kernel chain of decode.cu, whose launches overlap through
// programmatic dependent launch, is faster, because each grid barrier here
// costs about as much as a dependent launch and phase C runs on 1 CTA per SM.
//
// The grid barriers share one monotonic 64-bit arrival count in the caller's
// workspace (zero before the first call; every call adds two arrivals per
// CTA, so calls on one workspace stay in step).
// Every wait is bounded: a barrier or copy that does not complete within the
// limit sets MOE_DEVERR_TIMEOUT and the CTA leaves after its own copies have
// landed.
//
// Strata article, section 2 item 2: the router's choice decides which
// experts are computed; only those experts' weights are streamed.
#include "common.cuh"
#include "kernels.h"
#include "qdot.cuh"
#include "sm100.cuh"
#include "topk.cuh"

namespace moe {
using namespace sm100;

constexpr int kStepThreads = 1024;
constexpr int kStepWarps = kStepThreads / 32;
constexpr int kChunkRows = 8;                  // gate/up rows per copy chunk (one mbarrier each)
constexpr int kMaxChunks = 16;                 // routed gate/up chunks per CTA
constexpr int kStepRowsMax = 16;               // output rows per CTA (H <= 2048 over >= 128 SMs)
constexpr int kRouterSlices = 8;               // warps per router row (each a slice of H / 8)
constexpr size_t kStepSmemLimit = 227 * 1024;  // dynamic + static shared memory per CTA

struct StepArgs {
    int H, I, E, k, ng, G;
    const void *x;
    int x_bf16;
    const void *w_router;
    int w_bf16;
    const float *bias;
    const float *logits_in;
    const uint8_t *const *blobs;
    const uint8_t *shared;
    int32_t *ids_out;
    float *w_out;
    float *logits_out;
    float *y;
    float *logits_ws;              // [E]
    float *h_ws;                   // [ng][I]
    unsigned *bar;                 // 64-bit monotonic grid-barrier arrival count (8-byte aligned)
    unsigned *err;
    unsigned long long wait_ns;    // limit of every wait
    unsigned extra_arrivals;       // test hook: arrivals the barriers wait for in addition to the grid's
};

// Shared-memory layout (bytes from the dynamic base; all offsets 16-aligned
// for the shapes this kernel takes: H and I multiples of 256).
struct StepLayout {
    int ru, su, rd;                  // per CTA at most: routed units, shared units, down rows
    uint32_t CB, SB, DCB, DSB, UB;   // code / scale bytes of a gate/up row, of a down row; one unit
    uint32_t off_table, off_x, off_xn, off_cs, off_rp, off_gu, off_dn, off_h, off_hcs, off_part, total;
};

__host__ __device__ inline uint32_t al16(uint32_t v) { return (v + 15u) & ~15u; }

__host__ __device__ inline StepLayout step_layout(int bits, int H, int I, int E, int k, int ng, int G) {
    StepLayout L;
    const long R = static_cast<long>(k) * I;
    L.ru = static_cast<int>((R + G - 1) / G);
    L.su = ng > k ? (I + G - 1) / G : 0;
    L.rd = (H + G - 1) / G;
    L.CB = static_cast<uint32_t>(H) * bits / 8;
    L.SB = static_cast<uint32_t>(H) / 16;
    L.DCB = static_cast<uint32_t>(I) * bits / 8;
    L.DSB = static_cast<uint32_t>(I) / 16;
    L.UB = 2 * (L.CB + L.SB);
    uint32_t o = 0;
    L.off_table = o;
    o += al16(static_cast<uint32_t>(E) * 8);
    L.off_x = o;                                   // x as pieces: piece q of chunk c at [q][c]
    o += static_cast<uint32_t>(H) * 4;
    L.off_xn = o;                                  // x in natural order (router slices)
    o += static_cast<uint32_t>(H) * 4;
    L.off_cs = o;                                  // pre-scaled block sums of x
    o += al16(static_cast<uint32_t>(H) / 32 * 4);
    L.off_rp = o;                                  // router partial sums [rows][slices]
    o += al16(static_cast<uint32_t>((E + G - 1) / G) * kRouterSlices * 4);
    L.off_gu = o;
    o += static_cast<uint32_t>(L.ru + L.su) * L.UB;
    L.off_dn = o;
    o += static_cast<uint32_t>(ng) * L.rd * (L.DCB + L.DSB);
    L.off_h = o;
    o += static_cast<uint32_t>(ng) * I * 4;
    L.off_hcs = o;
    o += al16(static_cast<uint32_t>(ng) * (I / 32) * 4);
    L.off_part = o;
    o += al16(static_cast<uint32_t>(ng) * L.rd * 4);
    L.total = o;
    return L;
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// completing on `bar`; nothing for zero bytes.
__device__ __forceinline__ void bulk(uint8_t *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    if (bytes) bulk_g2s(smem_addr(dst), src, bytes, bar);
}

// Gate/up rows [i, i + m) of blob b into a region of n rows at `base`, laid
// out [gate codes][up codes][gate scales][up scales], starting at row `off`.
template <int BITS>
__device__ __forceinline__ void copy_rows(const StepLayout &L, uint8_t *base, int n, int off, const uint8_t *b, int i,
                                          int m, int H, int I, uint64_t *bar) {
    const BlobView v = blob_view(b, BITS, H, I);
    bulk(base + off * L.CB, v.cg + static_cast<size_t>(i) * L.CB, m * L.CB, bar);
    bulk(base + (n + off) * L.CB, v.cu + static_cast<size_t>(i) * L.CB, m * L.CB, bar);
    bulk(base + 2 * n * L.CB + off * L.SB, reinterpret_cast<const uint8_t *>(v.sg) + static_cast<size_t>(i) * L.SB,
         m * L.SB, bar);
    bulk(base + 2 * n * L.CB + (n + off) * L.SB, reinterpret_cast<const uint8_t *>(v.su) + static_cast<size_t>(i) * L.SB,
         m * L.SB, bar);
}

// Output rows [r0, r0 + nr) of blob b's down matrix (codes, then scales)
// into a down slot.
template <int BITS>
__device__ __forceinline__ void copy_down(const StepLayout &L, uint8_t *slot, const uint8_t *b, int r0, int nr, int H,
                                          int I, uint64_t *bar) {
    const BlobView v = blob_view(b, BITS, H, I);
    bulk(slot, v.cd + static_cast<size_t>(r0) * L.DCB, nr * L.DCB, bar);
    bulk(slot + L.rd * L.DCB, reinterpret_cast<const uint8_t *>(v.sd) + static_cast<size_t>(r0) * L.DSB, nr * L.DSB, bar);
}

// Bounded wait for phase 0 of a copy barrier; false after `limit_ns`.  The
// clock is read only every 1024 polls (each poll may suspend the thread
// briefly), so waiting warps leave the issue slots and the clock unit to the
// warps that compute.
__device__ __forceinline__ bool copies_landed(uint64_t *bar, unsigned long long limit_ns) {
    unsigned long long t0 = 0;
    for (unsigned it = 0;; ++it) {
        if (mbar_try_wait(bar, 0)) return true;
        if ((it & 1023u) == 1023u) {
            const unsigned long long t = globaltimer_ns();
            if (t0 == 0) t0 = t;
            else if (t - t0 > limit_ns) return false;
        }
    }
}

__device__ __forceinline__ unsigned long long atom_add_release_u64(unsigned long long *p, unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.release.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
    return old;
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Grid barrier on a monotonic 64-bit arrival count, for the thread that
// represents its CTA (after a CTA barrier).  Every call makes exactly G
// arrivals per barrier and two barriers, so the arrivals of one barrier are
// the G consecutive tickets [m G, (m + 1) G) and an arrival waits until the
// count reaches the end of its block (plus the test hook's extra arrivals,
// which never come).  No arrival has to release the others: the count itself
// is the flag.  `wait` false: arrive only.
__device__ bool grid_arrive(unsigned long long *count, unsigned G, unsigned extra, bool wait,
                            unsigned long long limit_ns) {
    const unsigned long long old = atom_add_release_u64(count, 1ull);
    if (!wait) return true;
    const unsigned long long target = (old / G + 1) * G + extra;
    unsigned long long t0 = 0;
    for (unsigned it = 1;; ++it) {
        if (ld_acquire_u64(count) >= target) return true;
        if ((it & 255u) == 0) {                            // look at the clock now and then
            const unsigned long long t = globaltimer_ns();
            if (t0 == 0) t0 = t;
            else if (t - t0 > limit_ns) return false;
        }
    }
}

// Eight bf16 (16 bytes) -> two float4.
__device__ __forceinline__ void bf16x8(const uint4 u, float4 &lo, float4 &hi) {
    lo = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xffff0000u));
    hi = make_float4(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xffff0000u), __uint_as_float(u.w << 16),
                     __uint_as_float(u.w & 0xffff0000u));
}

template <int BITS, int LPR>
__global__ void __launch_bounds__(kStepThreads, 1) k_dec_step(StepArgs a) {
    using Q = QT<BITS>;
    constexpr int S = 2048 / Q::EPC / 32;            // x chunks per lane (H <= 2048)
    constexpr int RPP = 32 / LPR;                    // down rows per warp pass
    constexpr int I = LPR * Q::EPC;                  // the intermediate size
    constexpr int DNSC = I / 32;                     // quant blocks of a down row
    extern __shared__ __align__(128) uint8_t sm[];
    __shared__ uint64_t bars[2 + kMaxChunks];        // shared-expert copies, routed down copies, gate/up chunks
    __shared__ uint64_t lists[kStepWarps * 32], sel[32];   // top-k candidates (tree: 16 per warp; merge: k)
    __shared__ float gates_s[33];
    __shared__ const uint8_t *gblob_s[33];           // blob of each group; NULL: the group is skipped
    __shared__ int fail_s;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H, E = a.E, k = a.k, ng = a.ng, G = a.G, c = blockIdx.x;
    const StepLayout L = step_layout(BITS, H, I, E, k, ng, G);
    uint64_t *barS = bars, *barD = bars + 1, *barG = bars + 2;
    const bool has_shared = ng > k;
    const long R = static_cast<long>(k) * I;
    const int u0 = static_cast<int>(c * R / G), u1 = static_cast<int>((c + 1) * R / G);
    const int s0 = has_shared ? static_cast<int>(static_cast<long>(c) * I / G) : 0;
    const int s1 = has_shared ? static_cast<int>(static_cast<long>(c + 1) * I / G) : 0;
    const int r0 = static_cast<int>(static_cast<long>(c) * H / G), r1 = static_cast<int>(static_cast<long>(c + 1) * H / G);
    const int ns = s1 - s0, nru = u1 - u0, nrd = r1 - r0;
    const int nchunks = (nru + kChunkRows - 1) / kChunkRows;
    const int NCH = H / Q::EPC;
    const uint8_t **tab = reinterpret_cast<const uint8_t **>(sm + L.off_table);
    unsigned long long *count = reinterpret_cast<unsigned long long *>(a.bar);
    uint8_t *sh_base = sm + L.off_gu;                // the shared expert's rows: one region of ns rows
    uint8_t *rt_base = sm + L.off_gu + static_cast<uint32_t>(ns) * L.UB;   // routed chunks of 8 rows
    bool routed_issued = false;

    // ---------------------------------------------------------------- A
    // every load of this phase goes out before any is used: this thread's
    // slice of a router row (kRouterSlices warps per row), its entry of the
    // expert table, its 16 bytes of x
    const int e0 = static_cast<int>(static_cast<long>(c) * E / G), e1 = static_cast<int>(static_cast<long>(c + 1) * E / G);
    const int nrow = e1 - e0, HS = H / kRouterSlices;
    const int rp = warp;                              // (row, slice) pair of this warp's first router task
    uint4 wr4[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
    const bool router_here = !a.logits_in && rp < nrow * kRouterSlices && lane * 8 < HS;
    if (router_here) {
        const int e = e0 + rp / kRouterSlices, h0 = (rp % kRouterSlices) * HS + lane * 8;
        if (a.w_bf16) {
            wr4[0] = ldg_stream(static_cast<const __nv_bfloat16 *>(a.w_router) + static_cast<size_t>(e) * H + h0);
        } else {
            wr4[0] = ldg_stream(static_cast<const float *>(a.w_router) + static_cast<size_t>(e) * H + h0);
            wr4[1] = ldg_stream(static_cast<const float *>(a.w_router) + static_cast<size_t>(e) * H + h0 + 4);
        }
    }
    const uint8_t *tab_e = tid < E ? a.blobs[tid] : nullptr;
    float4 x8[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    uint4 xr = make_uint4(0, 0, 0, 0);
    if (tid * 8 < H) {
        if (a.x_bf16) {
            xr = *reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.x) + tid * 8);
        } else {
            x8[0] = *reinterpret_cast<const float4 *>(static_cast<const float *>(a.x) + tid * 8);
            x8[1] = *reinterpret_cast<const float4 *>(static_cast<const float *>(a.x) + tid * 8 + 4);
        }
    }
    if (tid == 0) {
        fail_s = 0;
        for (int j = 0; j < 2 + kMaxChunks; ++j) mbar_init(bars + j, 1);
        fence_barrier_init();
    }
    __syncthreads();
    // the shared expert's rows do not depend on the routing: copy them now,
    // one bulk copy per region, issued by lane 0 of the last six warps
    if (has_shared && lane == 0 && warp >= kStepWarps - 6) {
        const BlobView v = blob_view(a.shared, BITS, H, I);
        const int q = warp - (kStepWarps - 6);
        uint8_t *dslot = sm + L.off_dn + static_cast<uint32_t>(k) * L.rd * (L.DCB + L.DSB);
        if (q == 0) bulk(sh_base, v.cg + static_cast<size_t>(s0) * L.CB, ns * L.CB, barS);
        if (q == 1) bulk(sh_base + ns * L.CB, v.cu + static_cast<size_t>(s0) * L.CB, ns * L.CB, barS);
        if (q == 2) bulk(sh_base + 2 * ns * L.CB, reinterpret_cast<const uint8_t *>(v.sg) + static_cast<size_t>(s0) * L.SB,
                         ns * L.SB, barS);
        if (q == 3) bulk(sh_base + 2 * ns * L.CB + ns * L.SB,
                         reinterpret_cast<const uint8_t *>(v.su) + static_cast<size_t>(s0) * L.SB, ns * L.SB, barS);
        if (q == 4) bulk(dslot, v.cd + static_cast<size_t>(r0) * L.DCB, nrd * L.DCB, barS);
        if (q == 5) bulk(dslot + L.rd * L.DCB, reinterpret_cast<const uint8_t *>(v.sd) + static_cast<size_t>(r0) * L.DSB,
                         nrd * L.DSB, barS);
    }
    if (tid == 0) mbar_arrive_expect_tx(barS, has_shared ? ns * L.UB + nrd * (L.DCB + L.DSB) : 0u);
    // stage x: natural order (router) and as pieces (expert rows: piece q of
    // chunk c at [q][c], so the lanes of a warp read consecutive pieces)
    float4 *xs = reinterpret_cast<float4 *>(sm + L.off_x);
    float *xn = reinterpret_cast<float *>(sm + L.off_xn);
    float *cs = reinterpret_cast<float *>(sm + L.off_cs);
    if (tid * 8 < H) {
        if (a.x_bf16) bf16x8(xr, x8[0], x8[1]);
        reinterpret_cast<float4 *>(xn)[2 * tid] = x8[0];
        reinterpret_cast<float4 *>(xn)[2 * tid + 1] = x8[1];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int g4 = 2 * tid + h, cch = g4 / Q::PPC, q = g4 % Q::PPC;
            xs[q * NCH + cch] = x8[h];
        }
    }
    if (tid < E) tab[tid] = tab_e;
    __syncthreads();
    if (tid < H / 32) {                               // (128 + half) * sum of x over each quant block
        float sum = 0.f;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float4 v = reinterpret_cast<const float4 *>(xn)[8 * tid + p];
            sum += (v.x + v.y) + (v.z + v.w);
        }
        cs[tid] = static_cast<float>(128 + Q::HALF) * sum;
    }
    if (!a.logits_in) {
        // router: warp task p = (row p / slices, slice p % slices), a partial
        // dot over H / slices elements; the partials meet in shared memory
        float *rpart = reinterpret_cast<float *>(sm + L.off_rp);
        for (int p = warp; p < nrow * kRouterSlices; p += kStepWarps) {
            const int e = e0 + p / kRouterSlices, h0 = (p % kRouterSlices) * HS + lane * 8;
            float acc = 0.f;
            if (lane * 8 < HS) {
                if (p != rp) {
                    if (a.w_bf16) {
                        wr4[0] = ldg_stream(static_cast<const __nv_bfloat16 *>(a.w_router) + static_cast<size_t>(e) * H + h0);
                    } else {
                        wr4[0] = ldg_stream(static_cast<const float *>(a.w_router) + static_cast<size_t>(e) * H + h0);
                        wr4[1] = ldg_stream(static_cast<const float *>(a.w_router) + static_cast<size_t>(e) * H + h0 + 4);
                    }
                }
                float4 w0, w1;
                if (a.w_bf16) {
                    bf16x8(wr4[0], w0, w1);
                } else {
                    w0 = make_float4(__uint_as_float(wr4[0].x), __uint_as_float(wr4[0].y), __uint_as_float(wr4[0].z),
                                     __uint_as_float(wr4[0].w));
                    w1 = make_float4(__uint_as_float(wr4[1].x), __uint_as_float(wr4[1].y), __uint_as_float(wr4[1].z),
                                     __uint_as_float(wr4[1].w));
                }
                const float4 xa = reinterpret_cast<const float4 *>(xn + h0)[0];
                const float4 xb = reinterpret_cast<const float4 *>(xn + h0)[1];
                acc = fmaf(w0.x, xa.x, acc); acc = fmaf(w0.y, xa.y, acc);
                acc = fmaf(w0.z, xa.z, acc); acc = fmaf(w0.w, xa.w, acc);
                acc = fmaf(w1.x, xb.x, acc); acc = fmaf(w1.y, xb.y, acc);
                acc = fmaf(w1.z, xb.z, acc); acc = fmaf(w1.w, xb.w, acc);
            }
            acc = warp_sum(acc);
            if (lane == 0) rpart[p] = acc;
        }
        __syncthreads();
        if (tid < nrow) {
            float l = 0.f;
            for (int q = 0; q < kRouterSlices; ++q) l += rpart[tid * kRouterSlices + q];   // slice order
            l += a.bias ? a.bias[e0 + tid] : 0.f;
            __stcg(a.logits_ws + e0 + tid, l);
            if (a.logits_out) a.logits_out[e0 + tid] = l;
        }
    }
    __syncthreads();                                 // this CTA's logits are written
    // barrier 1: every call arrives, so the count stays in step; only a call
    // that computed the logits here waits
    if (tid == 0) __threadfence();
    if (tid == 0 && !grid_arrive(count, G, a.extra_arrivals, !a.logits_in, a.wait_ns)) {
        fail_s = 1;
        report(a.err, MOE_DEVERR_TIMEOUT);
    }
    __syncthreads();
    if (fail_s) goto finish;

    // ---------------------------------------------------------------- B
    {
        const float *lg = a.logits_in ? a.logits_in : a.logits_ws;
        if (k <= 16 && E <= 32 * kStepWarps) block_topk_tree<kStepWarps>(lg, E, k, lists, sel);
        else block_topk_merge<kStepWarps, 1>(lg, E, k, lists, sel);
        if (warp == 0) {
            const uint64_t key = lane < k ? sel[lane] : 0ull;
            const float my_v = key_float(static_cast<uint32_t>(key >> 32));
            const int my_id = static_cast<int>(0xffffffffu - static_cast<uint32_t>(key));
            const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
            const bool bad = lane < k && (my_v != my_v || my_v == __int_as_float(0x7f800000));
            const bool any_bad = __any_sync(0xffffffffu, bad);
            const float ex = lane < k ? expf(my_v - v0) : 0.f;
            float sum = 0.f;
            for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, ex, j);   // slot order
            const uint8_t *b = nullptr;
            if (lane < k) {
                const float wj = any_bad ? __int_as_float(0x7fc00000) : ex / sum;
                const bool in_range = my_id >= 0 && my_id < E;
                b = in_range ? tab[my_id] : nullptr;
                unsigned e_bits = 0;
                if (!b) e_bits = in_range ? MOE_DEVERR_NULL_BLOB : MOE_DEVERR_BAD_EXPERT;
                else if (reinterpret_cast<uintptr_t>(b) & 15u) e_bits = MOE_DEVERR_MISALIGNED;
                if (e_bits) b = nullptr;
                gates_s[lane] = wj;
                gblob_s[lane] = b;
                if (c == 0) {
                    a.ids_out[lane] = my_id;
                    a.w_out[lane] = wj;
                    if (e_bits) report(a.err, e_bits);
                }
            }
            if (lane == 0) {
                gblob_s[k] = a.shared;
                gates_s[k] = 1.0f;
                if (c == 0 && any_bad) report(a.err, MOE_DEVERR_NONFINITE);
            }
            // arm the routed barriers with the bytes their copies will bring:
            // lane j < nchunks the gate/up chunk j, lane 31 the down rows
            __syncwarp();
            if (lane < nchunks) {
                const int c0 = u0 + lane * kChunkRows, c1 = min(u1, c0 + kChunkRows);
                uint32_t bytes = 0;
                for (int p = c0; p < c1; ++p) bytes += gblob_s[p / I] ? L.UB : 0u;
                mbar_arrive_expect_tx(barG + lane, bytes);
            }
            if (lane == 31) {
                uint32_t bytes = 0;
                for (int g = 0; g < k; ++g) bytes += gblob_s[g] ? static_cast<uint32_t>(nrd) * (L.DCB + L.DSB) : 0u;
                mbar_arrive_expect_tx(barD, bytes);
            }
        }
        __syncthreads();
        routed_issued = true;
        // the copies: gate/up chunk j (up to two groups, four regions each) by
        // lane 0 of warp j; the down rows of routed group g by lane 0 of warp
        // (nchunks + g) mod 16
        if (lane == 0) {
            for (int cj = warp; cj < nchunks; cj += kStepWarps) {
                const int c0 = u0 + cj * kChunkRows, c1 = min(u1, c0 + kChunkRows), n = c1 - c0;
                uint8_t *base = rt_base + static_cast<uint32_t>(cj) * kChunkRows * L.UB;
                for (int p = c0; p < c1;) {
                    const int g = p / I, q = min(c1, (g + 1) * I);
                    if (gblob_s[g]) copy_rows<BITS>(L, base, n, p - c0, gblob_s[g], p - g * I, q - p, H, I, barG + cj);
                    p = q;
                }
            }
            for (int g = (warp - nchunks % kStepWarps + kStepWarps) % kStepWarps; g < k; g += kStepWarps)
                if (gblob_s[g])
                    copy_down<BITS>(L, sm + L.off_dn + static_cast<uint32_t>(g) * L.rd * (L.DCB + L.DSB), gblob_s[g], r0,
                                    nrd, H, I, barD);
        }
    }

    // ---------------------------------------------------------------- C
    {
        const int nunits = ns + nru;
        for (int j = warp; j < nunits; j += kStepWarps) {
            int g, i, rj, n;
            const uint8_t *base;
            uint64_t *bar;
            if (j < ns) {
                g = k;
                i = s0 + j;
                rj = j;
                n = ns;
                base = sh_base;
                bar = barS;
            } else {
                const int jr = j - ns, u = u0 + jr;
                g = u / I;
                i = u - g * I;
                const int cj = jr / kChunkRows;
                rj = jr - cj * kChunkRows;
                n = min(kChunkRows, nru - cj * kChunkRows);
                base = rt_base + static_cast<uint32_t>(cj) * kChunkRows * L.UB;
                bar = barG + cj;
            }
            float hv = 0.f;
            if (gblob_s[g]) {
                // every lane observes the copies; the warp leaves together on a timeout
                if (!__all_sync(0xffffffffu, copies_landed(bar, a.wait_ns))) {
                    if (lane == 0) {
                        fail_s = 1;
                        report(a.err, MOE_DEVERR_TIMEOUT);
                    }
                    break;
                }
                const uint8_t *gc = base + rj * L.CB, *uc = base + (n + rj) * L.CB;
                const __half *gs = reinterpret_cast<const __half *>(base + 2 * n * L.CB + rj * L.SB);
                const __half *us = reinterpret_cast<const __half *>(base + 2 * n * L.CB + (n + rj) * L.SB);
                float dg = 0.f, du = 0.f;
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const int cc = lane + 32 * s;
                    if (cc < NCH) {
                        const uint4 cv[2] = {*reinterpret_cast<const uint4 *>(gc + cc * 16),
                                             *reinterpret_cast<const uint4 *>(uc + cc * 16)};
                        float sg[Q::BPC], su[Q::BPC], csum[Q::BPC], fx[2][Q::BPC];
                        load_scales<BITS>(gs, cc, true, sg);
                        load_scales<BITS>(us, cc, true, su);
#pragma unroll
                        for (int b = 0; b < Q::BPC; ++b) csum[b] = cs[cc * Q::BPC + b];
                        rows_fx<BITS, 2>(cv, xs + cc, NCH, fx);      // both rows share each x piece read
                        dg = chunk_finish<BITS>(fx[0], sg, csum, dg);
                        du = chunk_finish<BITS>(fx[1], su, csum, du);
                    }
                }
                dg = warp_sum(dg);
                du = warp_sum(du);
                hv = dg / (1.0f + expf(-dg)) * du;
            }
            if (lane == 0) __stcg(a.h_ws + static_cast<size_t>(g) * I + i, hv);
        }
        __syncthreads();
        const bool ok = !fail_s;
        // barrier 2: h complete everywhere (every CTA arrives, even after a failure here)
        if (tid == 0) __threadfence();
        if (tid == 0 && !grid_arrive(count, G, a.extra_arrivals, ok, a.wait_ns)) {
            fail_s = 1;
            report(a.err, MOE_DEVERR_TIMEOUT);
        }
        __syncthreads();
        if (fail_s) goto finish;
    }

    // ---------------------------------------------------------------- D
    {
        float4 *hs = reinterpret_cast<float4 *>(sm + L.off_h);     // [ng][PPC][LPR] pieces
        float *hcs = reinterpret_cast<float *>(sm + L.off_hcs);    // [ng][I/32] pre-scaled block sums
        float *part = reinterpret_cast<float *>(sm + L.off_part);  // [ng][rd]
        // hs[(t * PPC + q) * LPR + c] = piece q of chunk c of h_t: consecutive
        // threads store consecutive pieces (no bank conflicts)
        for (int i4 = tid; i4 < ng * (I / 4); i4 += kStepThreads) {
            const int t = i4 / (I / 4), rem = i4 % (I / 4);
            const int q = rem / LPR, cch = rem % LPR;
            hs[i4] = __ldcg(reinterpret_cast<const float4 *>(a.h_ws) + t * (I / 4) + cch * Q::PPC + q);
        }
        __syncthreads();
        for (int b = tid; b < ng * DNSC; b += kStepThreads) {
            const int t = b / DNSC, bb = b % DNSC;
            const int cch = bb / Q::BPC, beta = bb % Q::BPC;
            float s_acc = 0.f;
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const float4 v = hs[(t * Q::PPC + 8 * beta + p) * LPR + cch];
                s_acc += (v.x + v.y) + (v.z + v.w);
            }
            hcs[b] = static_cast<float>(128 + Q::HALF) * s_acc;
        }
        __syncthreads();
        // tasks (group, RPP rows): each lane one 16-byte code chunk of one row
        const int RG = (nrd + RPP - 1) / RPP;
        const int seg = lane % LPR, sub = lane / LPR;
        for (int t = warp; t < ng * RG; t += kStepWarps) {
            const int g = t / RG, rl = (t - g * RG) * RPP + sub;
            float v = 0.f;
            if (gblob_s[g]) {
                if (!__all_sync(0xffffffffu, copies_landed(g < k ? barD : barS, a.wait_ns))) {
                    if (lane == 0) {
                        fail_s = 1;
                        report(a.err, MOE_DEVERR_TIMEOUT);
                    }
                    break;
                }
                if (rl < nrd) {
                    const uint8_t *slot = sm + L.off_dn + static_cast<uint32_t>(g) * L.rd * (L.DCB + L.DSB);
                    const uint4 code = *reinterpret_cast<const uint4 *>(slot + rl * L.DCB + seg * 16);
                    const __half *sc = reinterpret_cast<const __half *>(slot + L.rd * L.DCB + rl * L.DSB);
                    float d[Q::BPC], fx[Q::BPC], csum[Q::BPC];
                    load_scales<BITS>(sc, seg, true, d);
                    float4 hp[Q::PPC];
#pragma unroll
                    for (int q = 0; q < Q::PPC; ++q) hp[q] = hs[(g * Q::PPC + q) * LPR + seg];
#pragma unroll
                    for (int b = 0; b < Q::BPC; ++b) csum[b] = hcs[g * DNSC + seg * Q::BPC + b];
                    chunk_fx<BITS>(code, hp, fx);
                    v = chunk_finish<BITS>(fx, d, csum, 0.f);
                }
            }
#pragma unroll
            for (int o = LPR >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (seg == 0 && rl < nrd) part[g * L.rd + rl] = v;
        }
        __syncthreads();
        if (!fail_s)
            for (int rl = tid; rl < nrd; rl += kStepThreads) {
                float acc = 0.f;
                for (int g = 0; g < ng; ++g) acc = fmaf(gates_s[g], part[g * L.rd + rl], acc);   // slot order
                a.y[r0 + rl] = acc;
            }
    }

finish:
    // every copy this CTA issued has landed before it exits (bounded)
    if (warp == 0) {
        bool ok = copies_landed(barS, a.wait_ns);
        if (routed_issued) {
            ok = copies_landed(barD, a.wait_ns) && ok;
            for (int j = 0; j < nchunks; ++j) ok = copies_landed(barG + j, a.wait_ns) && ok;
        }
        if (!ok && lane == 0) report(a.err, MOE_DEVERR_TIMEOUT);
    }
}

// ------------------------------------------------------------------ host
// Upper bound on the kernel's static shared memory (barriers, top-k
// candidates, per-group gates and blobs).
constexpr size_t kStepStaticSmem = 10 * 1024;

static int step_lpr(int bits, int I) { return I / (bits == 4 ? 32 : 64); }

static size_t step_smem(int bits, int H, int I, int E, int k, int ng, int G) {
    return step_layout(bits, H, I, E, k, ng, G).total;
}

bool decode_step_supported(int bits, int H, int I, int E, int k, bool shared) {
    if (H < 256 || H > 2048 || H % 256 != 0 || I % 256 != 0 || E > 1024 || k > 32) return false;
    const int lpr = step_lpr(bits, I);
    if (lpr != 4 && lpr != 8 && lpr != 16 && lpr != 32) return false;
    const int G = num_sms();
    const int ng = k + (shared ? 1 : 0);
    const StepLayout L = step_layout(bits, H, I, E, k, ng, G);
    if ((L.ru + kChunkRows - 1) / kChunkRows > kMaxChunks || L.rd > kStepRowsMax) return false;
    return static_cast<size_t>(L.total) + kStepStaticSmem <= kStepSmemLimit;
}

template <int BITS, int LPR>
static int launch_step_t(const StepArgs &a, cudaStream_t s) {
    const size_t smem = step_smem(BITS, a.H, a.I, a.E, a.k, a.ng, a.G);
    int rc = cuda_status(cudaFuncSetAttribute(k_dec_step<BITS, LPR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(smem)),
                         "decode step smem attribute");
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.G);
    cfg.blockDim = dim3(kStepThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeCooperative;          // all CTAs resident at once (grid barriers)
    attr.val.cooperative = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    rc = cuda_status(cudaLaunchKernelEx(&cfg, k_dec_step<BITS, LPR>, a), "decode step launch");
    count_launches(1);
    return rc;
}

int launch_decode_step(int bits, const void *x, int x_dtype, const void *w_router, int w_dtype, const float *bias,
                       const float *logits_in, const uint8_t *const *blobs, const uint8_t *shared, int H, int I,
                       int E, int k, int32_t *ids, float *w, float *logits_out, float *y, float *logits_ws,
                       float *h_ws, unsigned *bar, unsigned *err, cudaStream_t s) {
    StepArgs a;
    a.H = H; a.I = I; a.E = E; a.k = k;
    a.ng = k + (shared ? 1 : 0);
    a.G = num_sms();
    a.x = x; a.x_bf16 = x_dtype == MOE_BF16;
    a.w_router = w_router; a.w_bf16 = w_dtype == MOE_BF16;
    a.bias = bias; a.logits_in = logits_in;
    a.blobs = blobs; a.shared = shared;
    a.ids_out = ids; a.w_out = w; a.logits_out = logits_out;
    a.y = y;
    a.logits_ws = logits_ws;
    a.h_ws = h_ws;
    a.bar = bar;
    a.err = err;
    const long long lim = test_hook_value(MOE_HOOK_WAIT_LIMIT_NS);
    a.wait_ns = lim > 0 ? static_cast<unsigned long long>(lim) : 1000000000ull;
    a.extra_arrivals = static_cast<unsigned>(test_hook_value(MOE_HOOK_DECODE_EXTRA_ARRIVALS));
    const int lpr = step_lpr(bits, I);
    if (bits == 4) {
        switch (lpr) {
            case 8: return launch_step_t<4, 8>(a, s);
            case 16: return launch_step_t<4, 16>(a, s);
            default: return launch_step_t<4, 32>(a, s);
        }
    }
    switch (lpr) {
        case 4: return launch_step_t<2, 4>(a, s);
        case 8: return launch_step_t<2, 8>(a, s);
        case 16: return launch_step_t<2, 16>(a, s);
        default: return launch_step_t<2, 32>(a, s);
    }
}

}  // namespace moe
