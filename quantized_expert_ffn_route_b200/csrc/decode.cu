// The whole MoE step for one decode token: three kernels chained with
// programmatic dependent launch (each starts while its predecessor runs and
// waits with griddepcontrol only where it reads the predecessor's results).
//
//   1. logits (one warp per router row, spread over E/4 SMs).
//   2. gate/up (all selected experts + the shared expert, 16 rows per CTA):
//      every routed CTA selects the top-k from the logits itself (a block
//      top-k of a few hundred cycles, cheaper than another kernel boundary),
//      then h_g[i] = silu(Wg_g[i] . x) * (Wu_g[i] . x); CTA 0 publishes ids
//      and gates.  The shared expert's CTAs never wait for the logits.
//   3. down + combine (a few output rows per CTA, all groups; each lane one
//      chunk of one row): every code load is issued before h is staged, then
//      y[r] = sum_j w_j (Wd_{e_j}[r] . h_j) + Wd_shared[r] . h_shared, summed
//      in slot order.
// At one token the step streams ~20 MB of expert weights with little
// arithmetic, so everything here is about keeping loads in flight: every warp
// issues all of its weight loads before it touches shared memory.
//
// Strata article, section 2 item 2: the router's choice decides which
// experts are computed; only those experts' weights are streamed.
#include "common.cuh"
#include "kernels.h"
#include "qdot.cuh"
#include "topk.cuh"

namespace moe {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Workspace layout (bytes): ids [32] int32 | gates [32] fp32 | logits [E] | h [(k+1) * I]
struct DecodeWs {
    int32_t *ids;
    float *gates;
    float *logits;
    float *h;
};
__host__ __device__ inline DecodeWs decode_ws(void *ws, int E) {
    uint8_t *p = static_cast<uint8_t *>(ws);
    DecodeWs w;
    w.ids = reinterpret_cast<int32_t *>(p);
    w.gates = reinterpret_cast<float *>(p + 128);
    w.logits = reinterpret_cast<float *>(p + 256);
    w.h = reinterpret_cast<float *>(p + 256 + ((static_cast<size_t>(E) * 4 + 255) / 256) * 256);
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

// ------------------------------------------------------------ 1. logits
// One warp per router row, kLogitRows rows per CTA, so the E rows are read by
// E / kLogitRows SMs at once; every lane issues all of its weight loads
// before it stages x.
constexpr int kLogitRows = 4;

__global__ void __launch_bounds__(kLogitRows * 32) k_dec_logits(DecodeArgs a) {
    __shared__ __align__(16) float xs[2048];
    pdl_trigger();                                       // the gate/up kernel may start its prologue
    const int H = a.H, E = a.E;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x * kLogitRows + warp;
    uint4 w[8];                                          // bf16 rows: 8 x 16 B per lane covers H <= 2048
    if (a.w_bf16) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int hh = lane * 8 + 256 * j;
            w[j] = make_uint4(0, 0, 0, 0);
            if (e < E && hh < H)
                w[j] = ldg_stream(static_cast<const __nv_bfloat16 *>(a.w_router) + static_cast<size_t>(e) * H + hh);
        }
    }
    for (int i = threadIdx.x; i < H / 4; i += blockDim.x)
        reinterpret_cast<float4 *>(xs)[i] = a.x_bf16 ? load4(static_cast<const __nv_bfloat16 *>(a.x) + 4 * i)
                                                     : load4(static_cast<const float *>(a.x) + 4 * i);
    __syncthreads();
    if (e >= E) return;
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

// Top-k (k <= 32) of E <= 1024 logits by one block of kDecThreads threads.
// Each warp first takes the k best of its keys (k rounds of two warp max
// reductions: the value key, then among equal values the larger low word,
// i.e. the lower id), then warp 0 takes the k best of those 8k candidates.
// sel[0..k-1] receives the selection keys in rank order.
template <int N>
__device__ __forceinline__ void warp_take(uint64_t (&keys)[N], int k, int lane, uint64_t *dst) {
    uint64_t best = 0ull;
#pragma unroll
    for (int q = 0; q < N; ++q) best = keys[q] > best ? keys[q] : best;
    for (int r = 0; r < k; ++r) {
        const uint32_t hi = __reduce_max_sync(0xffffffffu, static_cast<uint32_t>(best >> 32));
        const uint32_t lo =
            __reduce_max_sync(0xffffffffu, static_cast<uint32_t>(best >> 32) == hi ? static_cast<uint32_t>(best) : 0u);
        const uint64_t win = (static_cast<uint64_t>(hi) << 32) | lo;
        if (lane == 0) dst[r] = win;
        if (best == win && win != 0ull) {                // keys are distinct: exactly one lane holds it
            best = 0ull;
#pragma unroll
            for (int q = 0; q < N; ++q) {
                if (keys[q] == win) keys[q] = 0ull;
                best = keys[q] > best ? keys[q] : best;
            }
        }
    }
}

__device__ void block_topk(const float *logits, int E, int k, uint64_t *cand, uint64_t *sel) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    {
        uint64_t keys[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int e = threadIdx.x + kDecThreads * q;
            keys[q] = e < E ? sel_key(__ldcg(logits + e), e) : 0ull;
        }
        warp_take(keys, k, lane, cand + warp * k);
    }
    __syncthreads();
    if (warp == 0) {
        uint64_t keys[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int i = lane + 32 * q;
            keys[q] = i < kDecWarps * k ? cand[i] : 0ull;
        }
        warp_take(keys, k, lane, sel);
    }
    __syncthreads();
}

// ----------------------------------------------------------- 2. gate/up
// Block = 8 warps x 2 row pairs = 16 rows of one group; grid = groups x I/16.
// The last group (when present) is the shared expert.  Each lane keeps the
// activation pieces of one chunk in registers and applies them to the four
// weight rows of its warp (gate and up of two rows).
template <int BITS>
__global__ void __launch_bounds__(kDecThreads, BITS == 4 ? 3 : 2) k_dec_gateup(DecodeArgs a) {
    using Q = QT<BITS>;
    extern __shared__ __align__(16) float4 gsm[];
    __shared__ const uint8_t *blob_s;
    const int H = a.H, I = a.I, k = a.k;
    const int rows_per_block = kDecWarps * 2;
    const int rblocks = I / rows_per_block;
    const int g = blockIdx.x / rblocks;
    const int i0 = (blockIdx.x % rblocks) * rows_per_block;
    const bool shared_group = g == k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float4 *xs = gsm;
    float *cs = reinterpret_cast<float *>(gsm + H / 4);
    {
        const void *x = a.x;
        stage_rows_fn<BITS>(xs, cs, 1, 1, H, [x](int) { return x; }, a.x_bf16);   // independent of the routing
    }
    pdl_trigger();                                       // the down kernel may start
    if (!shared_group) {
        pdl_wait();                                      // the logits are final from here on
        __shared__ uint64_t cand[kDecWarps * 32], sel[32];
        block_topk(a.logits_in ? a.logits_in : a.ws.logits, a.E, k, cand, sel);
        if (blockIdx.x == 0 && threadIdx.x < 32) {       // one CTA publishes ids and gates
            const int lane = threadIdx.x;
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
                a.ws.ids[lane] = my_id;
                a.ws.gates[lane] = wj;
                a.ids_out[lane] = my_id;
                a.w_out[lane] = wj;
            }
            if (lane == 0 && any_bad) report(a.err, MOE_DEVERR_NONFINITE);
        }
        if (threadIdx.x == 0) {
            const int e = static_cast<int>(0xffffffffu - static_cast<uint32_t>(sel[g]));
            const uint8_t *b = (e >= 0 && e < a.E) ? a.blobs[e] : nullptr;
            if (!b) report(a.err, (e >= 0 && e < a.E) ? MOE_DEVERR_NULL_BLOB : MOE_DEVERR_BAD_EXPERT);
            blob_s = b;
        }
    } else if (threadIdx.x == 0) {
        blob_s = a.shared;
    }
    __syncthreads();
    const uint8_t *blob = blob_s;
    if (!blob) return;
    const BlobView bv = blob_view(blob, BITS, H, I);
    const int nch = H / Q::EPC;
    const int nscx = H / 32;
    const size_t xrowb = static_cast<size_t>(H) * BITS / 8;
    // all code loads of the warp's four row vectors first
    constexpr int S = 2048 / Q::EPC / 32;               // chunks per lane (H <= 2048)
    uint4 code[4][S];
    float dsc[4][S][Q::BPC];
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
    float dot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const int cc = lane + 32 * s;
        if (cc < nch) {
            float4 xp[Q::PPC];
#pragma unroll
            for (int q = 0; q < Q::PPC; ++q) xp[q] = xs[q * nch + cc];
            float csum[Q::BPC];
#pragma unroll
            for (int b = 0; b < Q::BPC; ++b) csum[b] = cs[cc * Q::BPC + b];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                float fx[Q::BPC];
                chunk_fx<BITS>(code[v][s], xp, fx);
                dot[v] = chunk_finish<BITS>(fx, dsc[v][s], csum, dot[v]);
            }
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
// Block = RB output rows x all groups.  Tasks (group, lane-row group) are
// spread over the 8 warps; each lane takes one chunk of one row (lpr lanes
// per row), with every code load of the warp issued before h is staged.
// Per-group partials meet in shared memory and are summed in slot order.
constexpr int kDownTasks = 8;                            // tasks per warp (checked on the host)

template <int BITS>
__global__ void __launch_bounds__(kDecThreads, 2) k_dec_down(DecodeArgs a, int ng, int RB) {
    using Q = QT<BITS>;
    extern __shared__ __align__(16) float4 dsm[];
    __shared__ const uint8_t *blobs_s[33];
    __shared__ float gates_s[33];
    const int H = a.H, I = a.I, k = a.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nchd = I / Q::EPC;                         // chunks per row == lanes per row (power of two)
    const int lpr = nchd;
    const int rpp = 32 / lpr;                            // rows per task
    const int tpg = RB / rpp;                            // tasks per group
    const int ntasks = ng * tpg;
    const int r0 = blockIdx.x * RB;
    const size_t drowb = static_cast<size_t>(I) * BITS / 8;
    const int dnsc = I / 32;
    float4 *hs = dsm;
    float *hcs = reinterpret_cast<float *>(dsm + static_cast<size_t>(ng) * (I / 4));
    float *part = hcs + static_cast<size_t>(ng) * (I / 32);
    pdl_wait();                                          // ids (route) and h (gate/up) are final
    if (threadIdx.x < ng) {
        const int g = threadIdx.x;
        const uint8_t *b = a.shared;
        float gw = 1.0f;
        if (g < k) {
            const int e = a.ws.ids[g];
            b = (e >= 0 && e < a.E) ? a.blobs[e] : nullptr;
            gw = a.ws.gates[g];
        }
        blobs_s[g] = b;
        gates_s[g] = gw;
    }
    __syncthreads();
    const int seg = lane % lpr, sub = lane / lpr;
    uint4 code[kDownTasks];
    float dsc[kDownTasks][Q::BPC];
#pragma unroll
    for (int t = 0; t < kDownTasks; ++t) {
        const int task = warp + kDecWarps * t;
        const int g = task / tpg;
        const int r = r0 + (task % tpg) * rpp + sub;
        const bool valid = task < ntasks && r < H && blobs_s[g] != nullptr;
        code[t] = make_uint4(0, 0, 0, 0);
        const BlobView bv = blob_view(valid ? blobs_s[g] : a.shared, BITS, H, I);
        if (valid) code[t] = ldg_stream(bv.cd + static_cast<size_t>(r) * drowb + static_cast<size_t>(seg) * 16);
        load_scales<BITS>(bv.sd + static_cast<size_t>(valid ? r : 0) * dnsc, seg, valid, dsc[t]);
    }
    {
        const float *h = a.ws.h;
        stage_rows_fn<BITS>(hs, hcs, ng, ng, I,
                            [h, I](int t) { return static_cast<const void *>(h + static_cast<size_t>(t) * I); }, 0);
    }                                                    // ends with __syncthreads
#pragma unroll
    for (int t = 0; t < kDownTasks; ++t) {
        const int task = warp + kDecWarps * t;
        if (task >= ntasks) break;                       // uniform over the warp
        const int g = task / tpg;
        const int rl = (task % tpg) * rpp + sub;
        float4 xp[Q::PPC];
#pragma unroll
        for (int q = 0; q < Q::PPC; ++q) xp[q] = hs[static_cast<size_t>(g) * (I / 4) + q * nchd + seg];
        float csum[Q::BPC];
#pragma unroll
        for (int b = 0; b < Q::BPC; ++b) csum[b] = hcs[static_cast<size_t>(g) * (I / 32) + seg * Q::BPC + b];
        float fx[Q::BPC];
        chunk_fx<BITS>(code[t], xp, fx);
        float v = blobs_s[g] ? chunk_finish<BITS>(fx, dsc[t], csum, 0.f) : 0.f;
        for (int o = lpr >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
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
    return 256 + ((static_cast<size_t>(E) * 4 + 255) / 256) * 256 + static_cast<size_t>(k + 1) * I * 4;
}

static int down_rows_per_block(int ng) { return ng <= 16 ? 8 : 4; }

bool decode_supported(int bits, int H, int I, int E, int k) {
    if (E > 1024 || k > 32 || H > 2048 || I % 128 != 0) return false;
    const int nchd = I / (bits == 4 ? 32 : 64);
    if (nchd > 32 || (nchd & (nchd - 1)) != 0) return false;    // one chunk per lane, power-of-two lanes per row
    const int rpp = 32 / nchd, ng = k + 1, RB = down_rows_per_block(ng);
    if (RB % rpp != 0 || ceil_div(ng * (RB / rpp), kDecWarps) > kDownTasks) return false;
    const size_t smem_down = static_cast<size_t>(ng) * I * 4 + static_cast<size_t>(ng) * (I / 32) * 4 +
                             static_cast<size_t>(ng) * RB * 4;
    return smem_down <= 200 * 1024;
}

template <int BITS>
static int launch_decode_t(DecodeArgs a, int groups, cudaStream_t s) {
    const int H = a.H, I = a.I, E = a.E;
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    // 1. router logits (skipped when the caller supplies them)
    if (!a.logits_in) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(ceil_div(E, kLogitRows));
        cfg.blockDim = dim3(kLogitRows * 32);
        cfg.stream = s;
        int rc = cuda_status(cudaLaunchKernelEx(&cfg, k_dec_logits, a), "decode logits launch");
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
        cfg.numAttrs = a.logits_in ? 0 : 1;              // x and given logits come from earlier work: no overlap
        int rc = cuda_status(cudaLaunchKernelEx(&cfg, k_dec_gateup<BITS>, a), "decode gate/up launch");
        count_launches(1);
        if (rc) return rc;
    }
    // 3. down + combine
    {
        const int RB = down_rows_per_block(groups);
        const size_t smem = static_cast<size_t>(groups) * I * 4 + static_cast<size_t>(groups) * (I / 32) * 4 +
                            static_cast<size_t>(groups) * RB * 4;
        int rc = cuda_status(cudaFuncSetAttribute(k_dec_down<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  static_cast<int>(smem)),
                             "down smem attribute");
        if (rc) return rc;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(ceil_div(H, RB));
        cfg.blockDim = dim3(kDecThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cfg.attrs = &pdl;
        cfg.numAttrs = 1;
        rc = cuda_status(cudaLaunchKernelEx(&cfg, k_dec_down<BITS>, a, groups, RB), "decode down launch");
        count_launches(1);
        return rc;
    }
}

int launch_decode(int bits, const void *x, int x_dtype, const void *w_router, int w_dtype, const float *bias,
                  const float *logits_in, const uint8_t *const *blobs, const uint8_t *shared, int H, int I, int E,
                  int k, int32_t *ids, float *w, float *logits_out, float *y, void *ws, unsigned *err,
                  cudaStream_t s) {
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
