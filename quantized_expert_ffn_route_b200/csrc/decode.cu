// The whole MoE step for one decode token: three kernels chained with
// programmatic dependent launch (each starts while its predecessor runs and
// waits with griddepcontrol only where it reads the predecessor's results).
//
//   1. route: the logits (one warp per router row, E/4 CTAs; one CTA when
//      the caller gives the logits), then the last CTA to finish selects the
//      top-k, computes the gates and publishes ids, gates and the selected
//      blob pointers.  Selecting once here rather than in every gate/up CTA
//      keeps the selection off hundreds of CTAs' critical paths.
//   2. gate/up (all selected experts + the shared expert, 16 rows per CTA):
//      h_g[i] = silu(Wg_g[i] . x) * (Wu_g[i] . x).  The shared expert's CTAs
//      never wait for the route kernel; every CTA prefetches its share of
//      its expert's down rows into L2 for kernel 3.
//   3. down + combine (a few output rows per CTA, all groups; each lane one
//      chunk of one row): every code load is issued before h is staged, then
//      y[r] = sum_j w_j (Wd_{e_j}[r] . h_j) + Wd_shared[r] . h_shared, summed
//      in slot order.
// At one token the step streams ~20 MB of expert weights with little
// arithmetic, so the kernels keep every weight load of a warp in flight
// before touching shared memory, and every shape-dependent index is a
// compile-time shift.
//
// Strata article, section 2 item 2: the router's choice decides which
// experts are computed; only those experts' weights are streamed.
#include "common.cuh"
#include "kernels.h"
#include "qdot.cuh"
#include "sm100.cuh"
#include "topk.cuh"

namespace moe {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Workspace layout (bytes): ids [32] int32 @0 | gates [32] fp32 @128 |
// grid-barrier arrival count (uint64) @256 (used by the one-kernel step) |
// route-CTA ticket count (uint32) @264 | selected blob pointers [32] @512 |
// logits [E] @1024 | h [(k+1) * I] fp32 (256-aligned).  Both counts are zero
// before the first call, and every call leaves them so.
constexpr size_t kDecWsHeader = 1024;
struct DecodeWs {
    int32_t *ids;
    float *gates;
    unsigned *tickets;
    const uint8_t **blob;
    float *logits;
    float *h;
};
__host__ __device__ inline DecodeWs decode_ws(void *ws, int E) {
    uint8_t *p = static_cast<uint8_t *>(ws);
    DecodeWs w;
    w.ids = reinterpret_cast<int32_t *>(p);
    w.gates = reinterpret_cast<float *>(p + 128);
    w.tickets = reinterpret_cast<unsigned *>(p + 264);
    w.blob = reinterpret_cast<const uint8_t **>(p + 512);
    w.logits = reinterpret_cast<float *>(p + kDecWsHeader);
    w.h = reinterpret_cast<float *>(p + kDecWsHeader + ((static_cast<size_t>(E) * 4 + 255) / 256) * 256);
    return w;
}

struct DecodeArgs {
    int H, I, E, k;
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
    float *logits_out;   // may be NULL
    float *y;            // [H]
    DecodeWs ws;
    unsigned *err;
};

// ------------------------------------------------------------- 1. route
// One warp per router row, kLogitRows rows per CTA, so the E rows are read by
// E / kLogitRows SMs at once; every lane issues all of its weight loads
// before it stages x.  Each CTA then takes a ticket; the CTA that takes the
// last one sees every logit (each CTA fences its writes before its ticket)
// and selects.
constexpr int kLogitRows = 8;

__global__ void __launch_bounds__(kLogitRows * 32) k_dec_route(DecodeArgs a) {
    __shared__ __align__(16) float xs[2048];
    __shared__ uint64_t cand[kLogitRows * 32], sel[32];
    __shared__ const uint8_t *tab_s[1024];
    __shared__ int last;
    pdl_trigger();                                       // the gate/up kernel may start its prologue
    const int H = a.H, E = a.E, k = a.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (!a.logits_in) {
        const int e = blockIdx.x * kLogitRows + warp;
        uint4 w[8];                                      // bf16 rows: 8 x 16 B per lane covers H <= 2048
        if (a.w_bf16) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int hh = lane * 8 + 256 * j;
                w[j] = make_uint4(0, 0, 0, 0);
                if (e < E && hh < H)
                    w[j] = ldg_stream(static_cast<const __nv_bfloat16 *>(a.w_router) + static_cast<size_t>(e) * H + hh);
            }
        }
        {
            float4 v[4];                                 // H <= 2048: at most 4 loads per thread, all in flight
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = threadIdx.x + u * kLogitRows * 32;
                if (i < H / 4)
                    v[u] = a.x_bf16 ? load4(static_cast<const __nv_bfloat16 *>(a.x) + 4 * i)
                                    : load4(static_cast<const float *>(a.x) + 4 * i);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = threadIdx.x + u * kLogitRows * 32;
                if (i < H / 4) reinterpret_cast<float4 *>(xs)[i] = v[u];
            }
        }
        __syncthreads();
        if (e < E) {
            float s = 0.f;
            if (a.w_bf16) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int hh = lane * 8 + 256 * j;
                    if (hh < H) {
                        const float4 x0 = reinterpret_cast<const float4 *>(xs + hh)[0];
                        const float4 x1 = reinterpret_cast<const float4 *>(xs + hh)[1];
                        const uint4 u = w[j];
                        s = fmaf(__uint_as_float(u.x << 16), x0.x, s);
                        s = fmaf(__uint_as_float(u.x & 0xffff0000u), x0.y, s);
                        s = fmaf(__uint_as_float(u.y << 16), x0.z, s);
                        s = fmaf(__uint_as_float(u.y & 0xffff0000u), x0.w, s);
                        s = fmaf(__uint_as_float(u.z << 16), x1.x, s);
                        s = fmaf(__uint_as_float(u.z & 0xffff0000u), x1.y, s);
                        s = fmaf(__uint_as_float(u.w << 16), x1.z, s);
                        s = fmaf(__uint_as_float(u.w & 0xffff0000u), x1.w, s);
                    }
                }
            } else {
                for (int hh = lane * 4; hh < H; hh += 128) {
                    const float4 wv = load4(static_cast<const float *>(a.w_router) + static_cast<size_t>(e) * H + hh);
                    const float4 xv = reinterpret_cast<const float4 *>(xs + hh)[0];
                    s = fmaf(wv.x, xv.x, s); s = fmaf(wv.y, xv.y, s);
                    s = fmaf(wv.z, xv.z, s); s = fmaf(wv.w, xv.w, s);
                }
            }
            s = warp_sum(s);
            if (lane == 0) {
                const float l = s + (a.bias ? a.bias[e] : 0.f);
                a.ws.logits[e] = l;
                if (a.logits_out) a.logits_out[e] = l;
            }
        }
    }
    __syncthreads();                                     // every row of this CTA written
    if (threadIdx.x == 0)                                // release this CTA's rows; the last also acquires all
        last = sm100::atom_add_acq_rel_gpu(a.ws.tickets, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!last) return;
    // the expert table (E <= 1024 pointers) is read together with the logits,
    // so that the selected blob pointers need no further round trip
    constexpr int kTabPerThread = 1024 / (kLogitRows * 32);
    const uint8_t *tv[kTabPerThread];
#pragma unroll
    for (int u = 0; u < kTabPerThread; ++u) {
        const int e = threadIdx.x + u * kLogitRows * 32;
        tv[u] = e < E ? a.blobs[e] : nullptr;
    }
    const float *lg = a.logits_in ? a.logits_in : a.ws.logits;
    if (k <= 16 && E <= 32 * 2 * kLogitRows) block_topk_tree_n<kLogitRows, 2>(lg, E, k, cand, sel);
    else block_topk_merge<kLogitRows, 1024 / (32 * kLogitRows)>(lg, E, k, cand, sel);
#pragma unroll
    for (int u = 0; u < kTabPerThread; ++u) {
        const int e = threadIdx.x + u * kLogitRows * 32;
        if (e < E) tab_s[e] = tv[u];
    }
    __syncthreads();
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
        if (lane < k) {
            const float wj = any_bad ? __int_as_float(0x7fc00000) : ex / sum;
            const bool id_ok = my_id >= 0 && my_id < E;
            const uint8_t *b = id_ok ? tab_s[my_id] : nullptr;
            if (!b) {
                report(a.err, id_ok ? MOE_DEVERR_NULL_BLOB : MOE_DEVERR_BAD_EXPERT);
            } else if (reinterpret_cast<uintptr_t>(b) & 15u) {   // 16-byte loads need an aligned blob
                report(a.err, MOE_DEVERR_MISALIGNED);
                b = nullptr;
            }
            a.ws.ids[lane] = my_id;
            a.ws.gates[lane] = wj;
            a.ws.blob[lane] = b;
            a.ids_out[lane] = my_id;
            a.w_out[lane] = wj;
        }
        if (lane == 0 && any_bad) report(a.err, MOE_DEVERR_NONFINITE);
        if (lane == 0) *a.ws.tickets = 0u;               // ready for the next call
    }
}

// x as fp32 pieces in the order the chunk loops read them (piece q of chunk
// c at q * nch + c) plus the pre-scaled block sums (128 + h) * sum(x over the
// block); every divisor is a compile-time constant.
template <int BITS>
__device__ __forceinline__ void stage_x(float4 *xs, float *cs, int H, const void *x, int bf16) {
    using Q = QT<BITS>;
    const int nch = H / Q::EPC;
    constexpr int kB = 4;                                // loads of a thread in flight together
    for (int base = threadIdx.x; base < H / 4; base += kB * blockDim.x) {
        float4 v[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int g4 = base + u * blockDim.x;
            if (g4 < H / 4)
                v[u] = bf16 ? load4(static_cast<const __nv_bfloat16 *>(x) + 4 * g4)
                            : load4(static_cast<const float *>(x) + 4 * g4);
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int g4 = base + u * blockDim.x;
            if (g4 < H / 4) xs[(g4 % Q::PPC) * nch + g4 / Q::PPC] = v[u];
        }
    }
    __syncthreads();
    for (int b = threadIdx.x; b < H / 32; b += blockDim.x) {
        const int c = b / Q::BPC, beta = b % Q::BPC;
        float s = 0.f;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float4 v = xs[(8 * beta + p) * nch + c];
            s += (v.x + v.y) + (v.z + v.w);
        }
        cs[b] = static_cast<float>(128 + Q::HALF) * s;
    }
    __syncthreads();
}

// This CTA's share (1 / rblocks of the rows) of a blob's down matrix, codes
// and scales, into L2: the down kernel's loads, which may only start once the
// whole gate/up grid is done, then come from L2 instead of HBM.
template <int BITS>
__device__ __forceinline__ void prefetch_down_share(const uint8_t *blob, int H, int I, int rb, int rblocks) {
    const BlobView bv = blob_view(blob, BITS, H, I);
    const size_t r0 = static_cast<size_t>(rb) * H / rblocks, r1 = static_cast<size_t>(rb + 1) * H / rblocks;
    const size_t drowb = static_cast<size_t>(I) * BITS / 8, srow = static_cast<size_t>(I) / 16;
    sm100::prefetch_l2(bv.cd + r0 * drowb, static_cast<uint32_t>((r1 - r0) * drowb));
    const size_t s0 = (r0 * srow) & ~size_t(15), s1 = (r1 * srow) & ~size_t(15);
    sm100::prefetch_l2(reinterpret_cast<const uint8_t *>(bv.sd) + s0, static_cast<uint32_t>(s1 - s0));
}

// ----------------------------------------------------------- 2. gate/up
// Block = 8 warps x 2 row pairs = 16 rows of one group; grid = groups x I/16.
// The last group (when present) is the shared expert.  Each lane keeps the
// activation pieces of one chunk in registers and applies them to the four
// weight rows of its warp (gate and up of two rows).
template <int BITS>
__global__ void __launch_bounds__(kDecThreads, 3) k_dec_gateup(DecodeArgs a) {
    using Q = QT<BITS>;
    extern __shared__ __align__(16) float4 gsm[];
    const int H = a.H, I = a.I, k = a.k;
    constexpr int RPB = kDecWarps * 2;
    const int rblocks = I / RPB;
    const int g = blockIdx.x / rblocks;
    const int i0 = (blockIdx.x - g * rblocks) * RPB;
    const bool shared_group = g == k;
    // The down kernel is launched once every CTA here has triggered: the
    // shared expert's CTAs trigger at once, the routed ones only after their
    // wait on the route kernel, so that the down kernel may read the route
    // kernel's outputs (gates, blob pointers) before its own wait on h.
    if (shared_group) pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float4 *xs = gsm;
    float *cs = reinterpret_cast<float *>(gsm + H / 4);
    const int nch = H / Q::EPC;
    const int nscx = H / 32;
    const size_t xrowb = static_cast<size_t>(H) * BITS / 8;
    constexpr int S = 2048 / Q::EPC / 32;               // chunks per lane (H <= 2048)
    uint4 code[4][S];
    float dsc[4][S][Q::BPC];
    // all code loads of the warp's four row vectors
    auto load_codes = [&](const uint8_t *blob) {
        const BlobView bv = blob_view(blob, BITS, H, I);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int i = i0 + warp * 2 + (v >> 1);
            const uint8_t *cbase = (v & 1) ? bv.cu : bv.cg;
            const __half *sbase = (v & 1) ? bv.su : bv.sg;
#pragma unroll
            for (int s = 0; s < S; ++s) {
                const int cc = lane + 32 * s;
                const bool valid = cc < nch;
                code[v][s] = valid ? ldg_stream(cbase + static_cast<size_t>(i) * xrowb + static_cast<size_t>(cc) * 16)
                                   : make_uint4(0, 0, 0, 0);
                load_scales<BITS>(sbase + static_cast<size_t>(i) * nscx, cc, valid, dsc[v][s]);
            }
        }
    };
    stage_x<BITS>(xs, cs, H, a.x, a.x_bf16);
    if (shared_group) {
        if (threadIdx.x == 0) prefetch_down_share<BITS>(a.shared, H, I, blockIdx.x - g * rblocks, rblocks);
        load_codes(a.shared);                            // independent of the routing
    } else {
        pdl_wait();                                      // ids, gates and blob pointers are final from here on
        pdl_trigger();
        const uint8_t *blob = reinterpret_cast<const uint8_t *>(
            __ldcg(reinterpret_cast<const unsigned long long *>(a.ws.blob) + g));
        if (!blob) return;                               // reported by the route kernel; uniform over the CTA
        if (threadIdx.x == 0) prefetch_down_share<BITS>(blob, H, I, blockIdx.x - g * rblocks, rblocks);
        load_codes(blob);
    }
    float dot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const int cc = lane + 32 * s;
        if (cc < nch) {
            float csum[Q::BPC];
#pragma unroll
            for (int b = 0; b < Q::BPC; ++b) csum[b] = cs[cc * Q::BPC + b];
            const uint4 cv[4] = {code[0][s], code[1][s], code[2][s], code[3][s]};
            float fx[4][Q::BPC];
            rows_fx<BITS, 4>(cv, xs + cc, nch, fx);
#pragma unroll
            for (int v = 0; v < 4; ++v) dot[v] = chunk_finish<BITS>(fx[v], dsc[v][s], csum, dot[v]);
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float gv = warp_sum(dot[2 * j]);
        const float uv = warp_sum(dot[2 * j + 1]);
        if (lane == 0) a.ws.h[static_cast<size_t>(g) * I + i0 + warp * 2 + j] = gv / (1.0f + expf(-gv)) * uv;
    }
}

// ------------------------------------------------------ 3. down + combine
// Block = RB output rows x all groups.  Tasks (group, RPP rows) are spread
// over the 8 warps; each lane takes one chunk of one row (LPR = I / chunk
// lanes per row), with every code load of the warp issued before h is
// staged.  Per-group partials meet in shared memory and are summed in slot
// order.
constexpr int kDownTasks = 8;                            // tasks per warp (checked on the host)

template <int BITS, int LPR, int RB>
__global__ void __launch_bounds__(kDecThreads, 2) k_dec_down(DecodeArgs a, int ng) {
    using Q = QT<BITS>;
    constexpr int RPP = 32 / LPR;                        // rows per task
    constexpr int TPG = RB / RPP;                        // tasks per group
    constexpr int IL = LPR * Q::EPC;                     // the intermediate size I
    static_assert(RB % RPP == 0, "rows per block");
    extern __shared__ __align__(16) float4 dsm[];
    __shared__ const uint8_t *blobs_s[33];
    __shared__ float gates_s[33];
    const int H = a.H, k = a.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ntasks = ng * TPG;
    const int r0 = blockIdx.x * RB;
    constexpr size_t drowb = static_cast<size_t>(IL) * BITS / 8;
    constexpr int dnsc = IL / 32;
    float4 *hs = dsm;                                    // [ng][PPC][LPR] pieces
    float *hcs = reinterpret_cast<float *>(dsm + static_cast<size_t>(ng) * (IL / 4));
    float *part = hcs + static_cast<size_t>(ng) * dnsc;
    // The route kernel's gates and blob pointers are final already (see the
    // gate/up kernel's trigger), so the code loads go out before the wait on h.
    if (threadIdx.x < ng) {
        const int g = threadIdx.x;
        const uint8_t *b = a.shared;
        float gw = 1.0f;
        if (g < k) {
            b = reinterpret_cast<const uint8_t *>(__ldcg(reinterpret_cast<const unsigned long long *>(a.ws.blob) + g));
            gw = __ldcg(a.ws.gates + g);
        }
        blobs_s[g] = b;
        gates_s[g] = gw;
    }
    __syncthreads();
    const int seg = lane % LPR, sub = lane / LPR;
    uint4 code[kDownTasks];
    float dsc[kDownTasks][Q::BPC];
#pragma unroll
    for (int t = 0; t < kDownTasks; ++t) {
        const int task = warp + kDecWarps * t;
        const int g = task / TPG;
        const int r = r0 + (task % TPG) * RPP + sub;
        const uint8_t *blob = task < ntasks ? blobs_s[g] : nullptr;
        const bool valid = blob != nullptr && r < H;
        code[t] = make_uint4(0, 0, 0, 0);
        const BlobView bv = blob_view(valid ? blob : a.shared, BITS, H, IL);
        if (valid) code[t] = ldg_stream(bv.cd + static_cast<size_t>(r) * drowb + static_cast<size_t>(seg) * 16);
        load_scales<BITS>(bv.sd + static_cast<size_t>(valid ? r : 0) * dnsc, seg, valid, dsc[t]);
    }
    pdl_wait();                                          // h (gate/up) is final
    // stage h of every group (gate/up's fp32 output) as pieces + block sums
    {
        constexpr int kB = 8;                            // loads of a thread in flight together
        const int n4 = ng * (IL / 4);
        for (int base = threadIdx.x; base < n4; base += kB * kDecThreads) {
            float4 v[kB];
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const int g4 = base + u * kDecThreads;
                if (g4 < n4) v[u] = __ldcg(reinterpret_cast<const float4 *>(a.ws.h) + g4);
            }
#pragma unroll
            for (int u = 0; u < kB; ++u) {
                const int g4 = base + u * kDecThreads;
                if (g4 < n4) {
                    const int t = g4 / (IL / 4), rem = g4 % (IL / 4);
                    hs[(t * Q::PPC + rem % Q::PPC) * LPR + rem / Q::PPC] = v[u];
                }
            }
        }
    }
    __syncthreads();
    for (int b = threadIdx.x; b < ng * dnsc; b += kDecThreads) {
        const int t = b / dnsc, bb = b % dnsc;
        const int c = bb / Q::BPC, beta = bb % Q::BPC;
        float s = 0.f;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float4 v = hs[(t * Q::PPC + 8 * beta + p) * LPR + c];
            s += (v.x + v.y) + (v.z + v.w);
        }
        hcs[b] = static_cast<float>(128 + Q::HALF) * s;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < kDownTasks; ++t) {
        const int task = warp + kDecWarps * t;
        if (task >= ntasks) break;                       // uniform over the warp
        const int g = task / TPG;
        const int rl = (task % TPG) * RPP + sub;
        float4 xp[Q::PPC];
#pragma unroll
        for (int q = 0; q < Q::PPC; ++q) xp[q] = hs[(g * Q::PPC + q) * LPR + seg];
        float csum[Q::BPC];
#pragma unroll
        for (int b = 0; b < Q::BPC; ++b) csum[b] = hcs[g * dnsc + seg * Q::BPC + b];
        float fx[Q::BPC];
        chunk_fx<BITS>(code[t], xp, fx);
        float v = blobs_s[g] ? chunk_finish<BITS>(fx, dsc[t], csum, 0.f) : 0.f;
#pragma unroll
        for (int o = LPR >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (seg == 0) part[g * RB + rl] = v;
    }
    __syncthreads();
    if (threadIdx.x < RB && r0 + static_cast<int>(threadIdx.x) < H) {
        float acc = 0.f;
        for (int g = 0; g < ng; ++g) acc = fmaf(gates_s[g], part[g * RB + threadIdx.x], acc);   // slot order
        a.y[r0 + threadIdx.x] = acc;
    }
}

// ------------------------------------------------------------------ host
size_t decode_ws_bytes(int E, int k, int I) {
    return kDecWsHeader + ((static_cast<size_t>(E) * 4 + 255) / 256) * 256 + static_cast<size_t>(k + 1) * I * 4;
}

static int down_lpr(int bits, int I) { return I / (bits == 4 ? 32 : 64); }
static int down_rows_per_block(int ng, int lpr) { return (ng <= 16 || lpr == 4) ? 8 : 4; }

bool decode_supported(int bits, int H, int I, int E, int k) {
    if (E > 1024 || k > 32 || H > 2048 || H % 128 != 0 || I % 128 != 0) return false;
    const int lpr = down_lpr(bits, I);
    if (lpr != 4 && lpr != 8 && lpr != 16 && lpr != 32) return false;   // one chunk per lane
    const int rpp = 32 / lpr, ng = k + 1, RB = down_rows_per_block(ng, lpr);
    if (RB % rpp != 0 || ceil_div(ng * (RB / rpp), kDecWarps) > kDownTasks) return false;
    const size_t smem_down = static_cast<size_t>(ng) * I * 4 + static_cast<size_t>(ng) * (I / 32) * 4 +
                             static_cast<size_t>(ng) * RB * 4;
    return smem_down <= 200 * 1024;
}

template <int BITS, int LPR, int RB>
static int launch_down(const DecodeArgs &a, int groups, const cudaLaunchAttribute &pdl, cudaStream_t s) {
    const size_t smem = static_cast<size_t>(groups) * a.I * 4 + static_cast<size_t>(groups) * (a.I / 32) * 4 +
                        static_cast<size_t>(groups) * RB * 4;
    int rc = cuda_status(cudaFuncSetAttribute(k_dec_down<BITS, LPR, RB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(smem)),
                         "down smem attribute");
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ceil_div(a.H, RB));
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr = pdl;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    rc = cuda_status(cudaLaunchKernelEx(&cfg, k_dec_down<BITS, LPR, RB>, a, groups), "decode down launch");
    count_launches(1);
    return rc;
}

template <int BITS, int LPR>
static int launch_down_rb(const DecodeArgs &a, int groups, const cudaLaunchAttribute &pdl, cudaStream_t s) {
    if constexpr (LPR == 4) return launch_down<BITS, LPR, 8>(a, groups, pdl, s);
    else if (down_rows_per_block(groups, LPR) == 8) return launch_down<BITS, LPR, 8>(a, groups, pdl, s);
    else return launch_down<BITS, LPR, 4>(a, groups, pdl, s);
}

template <int BITS>
static int launch_decode_t(DecodeArgs a, int groups, cudaStream_t s) {
    const int H = a.H, I = a.I, E = a.E;
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    // 1. route (one CTA that only selects when the caller supplies the logits)
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(a.logits_in ? 1 : ceil_div(E, kLogitRows));
        cfg.blockDim = dim3(kLogitRows * 32);
        cfg.stream = s;
        int rc = cuda_status(cudaLaunchKernelEx(&cfg, k_dec_route, a), "decode route launch");
        count_launches(1);
        if (rc) return rc;
    }
    // 2. gate/up
    {
        const int rblocks = I / (kDecWarps * 2);
        const size_t smem = static_cast<size_t>(H) * 4 + static_cast<size_t>(H / 32) * 4;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(groups * rblocks);
        cfg.blockDim = dim3(kDecThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cfg.attrs = &pdl;
        cfg.numAttrs = 1;
        int rc = cuda_status(cudaLaunchKernelEx(&cfg, k_dec_gateup<BITS>, a), "decode gate/up launch");
        count_launches(1);
        if (rc) return rc;
    }
    // 3. down + combine
    switch (down_lpr(BITS, I)) {
        case 4: return launch_down_rb<BITS, 4>(a, groups, pdl, s);
        case 8: return launch_down_rb<BITS, 8>(a, groups, pdl, s);
        case 16: return launch_down_rb<BITS, 16>(a, groups, pdl, s);
        default: return launch_down_rb<BITS, 32>(a, groups, pdl, s);
    }
}

int launch_decode(int bits, const void *x, int x_dtype, const void *w_router, int w_dtype, const float *bias,
                  const float *logits_in, const uint8_t *const *blobs, const uint8_t *shared, int H, int I, int E,
                  int k, int32_t *ids, float *w, float *logits_out, float *y, void *ws, unsigned *err,
                  cudaStream_t s) {
    if (test_hook_value(MOE_HOOK_DECODE_ONE_KERNEL) != 0 && decode_step_supported(bits, H, I, E, k, shared != nullptr)) {
        // one persistent kernel (decode_step.cu); its grid-barrier count sits
        // at byte 256 of the workspace, between the gates and the logits
        const DecodeWs dw = decode_ws(ws, E);
        return launch_decode_step(bits, x, x_dtype, w_router, w_dtype, bias, logits_in, blobs, shared, H, I, E, k, ids,
                                  w, logits_out, y, dw.logits, dw.h,
                                  reinterpret_cast<unsigned *>(static_cast<uint8_t *>(ws) + 256), err, s);
    }
    DecodeArgs a;
    a.H = H; a.I = I; a.E = E; a.k = k;
    a.x = x; a.x_bf16 = x_dtype == MOE_BF16;
    a.w_router = w_router; a.w_bf16 = w_dtype == MOE_BF16;
    a.bias = bias; a.logits_in = logits_in;
    a.blobs = blobs; a.shared = shared;
    a.ids_out = ids; a.w_out = w; a.logits_out = logits_out;
    a.y = y;
    a.ws = decode_ws(ws, E);
    a.err = err;
    const int groups = k + (shared ? 1 : 0);
    return bits == 4 ? launch_decode_t<4>(a, groups, s) : launch_decode_t<2>(a, groups, s);
}

}  // namespace moe
