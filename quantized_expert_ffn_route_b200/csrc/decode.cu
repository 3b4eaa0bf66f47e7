// The whole MoE step for one decode token: three kernels chained with
// programmatic dependent launch (each starts while its predecessor runs and
// waits with griddepcontrol only where it reads the predecessor's results).
//
//   1. route  (one cluster of up to 16 CTAs): router logits, rows split over
//      the cluster and gathered through distributed shared memory; top-k and
//      gates by one warp.
//   2. gate/up (all selected experts + the shared expert, one warp per row
//      pair): h_g[i] = silu(Wg_g[i] . x) * (Wu_g[i] . x).  The shared expert's
//      CTAs do not wait for the route kernel at all.
//   3. down + combine (one warp per output row, all groups): the codes of the
//      row are loaded before h is staged, then
//      y[r] = sum_j w_j (Wd_{e_j}[r] . h_j) + Wd_shared[r] . h_shared, summed
//      in slot order.
// At one token the step streams ~20 MB of expert weights with little
// arithmetic, so everything here is about keeping loads in flight: every warp
// issues all of its weight loads before it touches shared memory.
//
// Strata article, section 2 item 2: the router's choice decides which
// experts are computed; only those experts' weights are streamed.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "qdot.cuh"
#include "topk.cuh"

namespace cg = cooperative_groups;

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

// Top-k of E <= 1024 values in shared memory by one warp (lane l owns experts
// l, l + 32, ...) with single-instruction warp maxima: first the 32-bit value
// key, then, among lanes holding that key, the lowest id.  Lane j < k ends
// with slot j's (value, id).
__device__ __forceinline__ void warp_topk_smem(const float *vals, int E, int k, int lane, float &my_v, int &my_id) {
    const int npl = (E - lane + 31) / 32;
    uint32_t taken = 0u;
    uint32_t bv = 0u;
    int bi = -1;
    auto best = [&]() {
        bv = 0u;
        bi = -1;
        for (int i = 0; i < npl; ++i) {
            if (taken & (1u << i)) continue;
            const uint32_t key = float_key(vals[lane + 32 * i]);
            if (bi < 0 || key > bv) {                   // equal keys keep the lower id (smaller i)
                bv = key;
                bi = lane + 32 * i;
            }
        }
    };
    best();
    for (int j = 0; j < k; ++j) {
        // keys are shifted by one so that "no candidate" (0) ranks below every real key
        const uint32_t hi = __reduce_max_sync(0xffffffffu, bi >= 0 ? bv + 1u : 0u);
        const unsigned lo_in = (bi >= 0 && bv + 1u == hi) ? 0xffffffffu - static_cast<unsigned>(bi) : 0u;
        const unsigned lo = __reduce_max_sync(0xffffffffu, lo_in);
        const int id = static_cast<int>(0xffffffffu - lo);
        if (lane == j) {
            my_v = key_float(hi - 1u);
            my_id = id;
        }
        if (bi == id) {                                   // the winner retires its candidate
            taken |= 1u << ((id - lane) / 32);
            best();
        }
    }
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

// ------------------------------------------------------------ 1. route
// One cluster; CTA rank r computes logit rows [r*er, (r+1)*er) for the single
// token, rank 0 gathers them and selects.  (With logits_in, rank 0 selects
// directly.)  Dynamic smem: x natural [H] + this CTA's logits [er] + all [E].
__global__ void __launch_bounds__(kDecThreads) k_dec_route(DecodeArgs a) {
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(16) float rsm[];
    pdl_trigger();                                       // the gate/up kernel may start its prologue
    const int H = a.H, E = a.E, k = a.k;
    const int C = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int er = ceil_div(E, C);
    float *xnat = rsm;
    float *lg = rsm + H;
    float *lall = lg + er;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (!a.logits_in) {
        for (int i = threadIdx.x; i < H / 4; i += kDecThreads)
            reinterpret_cast<float4 *>(xnat)[i] = a.x_bf16 ? load4(static_cast<const __nv_bfloat16 *>(a.x) + 4 * i)
                                                           : load4(static_cast<const float *>(a.x) + 4 * i);
        __syncthreads();
        const int e0 = min(E, rank * er), e1 = min(E, e0 + er);
        constexpr int RI = 8;                            // H <= 2048: one row's loads all in flight
        for (int e = e0 + warp; e < e1; e += kDecWarps) {
            float4 w0[RI], w1[RI];
#pragma unroll
            for (int j = 0; j < RI; ++j) {
                const int hh = lane * 8 + 256 * j;
                w0[j] = w1[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (hh < H) {
                    if (a.w_bf16) {
                        const __nv_bfloat16 *wr =
                            static_cast<const __nv_bfloat16 *>(a.w_router) + static_cast<size_t>(e) * H + hh;
                        w0[j] = load4(wr);
                        w1[j] = load4(wr + 4);
                    } else {
                        const float *wr = static_cast<const float *>(a.w_router) + static_cast<size_t>(e) * H + hh;
                        w0[j] = load4(wr);
                        w1[j] = load4(wr + 4);
                    }
                }
            }
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < RI; ++j) {
                const int hh = lane * 8 + 256 * j;
                if (hh < H) {
                    const float4 x0 = reinterpret_cast<const float4 *>(xnat + hh)[0];
                    const float4 x1 = reinterpret_cast<const float4 *>(xnat + hh)[1];
                    acc = fmaf(w0[j].x, x0.x, acc); acc = fmaf(w0[j].y, x0.y, acc);
                    acc = fmaf(w0[j].z, x0.z, acc); acc = fmaf(w0[j].w, x0.w, acc);
                    acc = fmaf(w1[j].x, x1.x, acc); acc = fmaf(w1[j].y, x1.y, acc);
                    acc = fmaf(w1[j].z, x1.z, acc); acc = fmaf(w1[j].w, x1.w, acc);
                }
            }
            acc = warp_sum(acc);
            if (lane == 0) {
                const float l = acc + (a.bias ? a.bias[e] : 0.f);
                lg[e - e0] = l;
                if (a.logits_out) a.logits_out[e] = l;
            }
        }
        cluster.sync();                                  // logit rows visible cluster-wide
        if (rank == 0)
            for (int e = threadIdx.x; e < E; e += kDecThreads) lall[e] = cluster.map_shared_rank(lg, e / er)[e % er];
        cluster.sync();                                  // no distributed shared memory reads after this
    } else if (rank == 0) {
        for (int e = threadIdx.x; e < E; e += kDecThreads) lall[e] = a.logits_in[e];
    }
    if (rank != 0) return;
    __syncthreads();
    if (warp == 0) {
        float my_v = 0.f;
        int my_id = 0;
        warp_topk_smem(lall, E, k, lane, my_v, my_id);
        const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
        const bool bad = lane < k && (my_v != my_v || my_v == __int_as_float(0x7f800000));
        const bool any_bad = __any_sync(0xffffffffu, bad);
        const float ex = lane < k ? expf(my_v - v0) : 0.f;
        float s = 0.f;
        for (int j = 0; j < k; ++j) s += __shfl_sync(0xffffffffu, ex, j);   // slot order
        if (lane < k) {
            const float wj = any_bad ? __int_as_float(0x7fc00000) : ex / s;
            a.ws.ids[lane] = my_id;
            a.ws.gates[lane] = wj;
            a.ids_out[lane] = my_id;
            a.w_out[lane] = wj;
        }
        if (lane == 0 && any_bad) report(a.err, MOE_DEVERR_NONFINITE);
    }
}

// ----------------------------------------------------------- 2. gate/up
// Block = 8 warps x 2 row pairs = 16 rows of one group; grid = groups x I/16.
// The last group (when present) is the shared expert.
template <int BITS>
__global__ void __launch_bounds__(kDecThreads, 3) k_dec_gateup(DecodeArgs a) {
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
    // prologue: x pieces + block sums (independent of the routing)
    {
        const void *rows[1] = {a.x};
        stage_rows<BITS>(xs, cs, 1, 1, H, rows, a.x_bf16);
    }
    pdl_trigger();                                       // the down kernel may start
    if (threadIdx.x == 0) {
        const uint8_t *b = a.shared;
        if (!shared_group) {
            pdl_wait();                                  // the route kernel's ids are needed from here on
            const int e = a.ws.ids[g];
            b = (e >= 0 && e < a.E) ? a.blobs[e] : nullptr;
            if (!b) report(a.err, (e >= 0 && e < a.E) ? MOE_DEVERR_NULL_BLOB : MOE_DEVERR_BAD_EXPERT);
        }
        blob_s = b;
    }
    __syncthreads();
    const uint8_t *blob = blob_s;
    if (!blob) return;
    const BlobView bv = blob_view(blob, BITS, H, I);
    const int nch = H / Q::EPC;
    const int nscx = H / 32;
    const size_t xrowb = static_cast<size_t>(H) * BITS / 8;
    uint4 cgv[2][2], cuv[2][2];
    float sgv[2][2][Q::BPC], suv[2][2][Q::BPC];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int i = i0 + warp * 2 + j;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const int cc = lane + 32 * s;
            const bool valid = cc < nch;
            cgv[j][s] = cuv[j][s] = make_uint4(0, 0, 0, 0);
            if (valid) {
                const size_t off = static_cast<size_t>(i) * xrowb + static_cast<size_t>(cc) * 16;
                cgv[j][s] = ldg_stream(bv.cg + off);
                cuv[j][s] = ldg_stream(bv.cu + off);
            }
            load_scales<BITS>(bv.sg + static_cast<size_t>(i) * nscx, cc, valid, sgv[j][s]);
            load_scales<BITS>(bv.su + static_cast<size_t>(i) * nscx, cc, valid, suv[j][s]);
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int i = i0 + warp * 2 + j;
        float dg[1] = {0.f}, du[1] = {0.f};
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const int cc = lane + 32 * s;
            if (cc < nch) {
                chunk_dot<BITS, 1>(cgv[j][s], sgv[j][s], xs, cs, nch, cc, dg);
                chunk_dot<BITS, 1>(cuv[j][s], suv[j][s], xs, cs, nch, cc, du);
            }
        }
        const float gv = warp_sum(dg[0]);
        const float uv = warp_sum(du[0]);
        if (lane == 0) a.ws.h[static_cast<size_t>(g) * I + i] = gv / (1.0f + expf(-gv)) * uv;
    }
}

// ------------------------------------------------------ 3. down + combine
// Warp = RPW output rows x all groups; lanes split a row's chunks (lpr lanes
// per group row, 32/lpr groups at a time).  Codes are loaded before h is
// staged (kDownRows x kMaxPass codes per lane in registers).
constexpr int kDownRows = 2;
constexpr int kMaxPass = 8;                             // passes of 32/lpr groups each (checked on the host)

template <int BITS>
__global__ void __launch_bounds__(kDecThreads, 2) k_dec_down(DecodeArgs a, int ng, int lpr) {
    using Q = QT<BITS>;
    extern __shared__ __align__(16) float4 dsm[];
    __shared__ const uint8_t *blobs_s[33];
    __shared__ float gates_s[33];
    const int H = a.H, I = a.I, k = a.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r0 = (blockIdx.x * kDecWarps + warp) * kDownRows;
    const int gpp = 32 / lpr;                            // groups per warp pass
    const int npass = ceil_div(ng, gpp);
    const int sub = lane / lpr, seg = lane % lpr;
    const int nchd = I / Q::EPC;                         // == lpr (checked on the host)
    const size_t drowb = static_cast<size_t>(I) * BITS / 8;
    const int dnsc = I / 32;
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
    // issue every code load of this warp's rows first
    uint4 code[kDownRows][kMaxPass];
    float sc[kDownRows][kMaxPass][Q::BPC];
#pragma unroll
    for (int rr = 0; rr < kDownRows; ++rr)
#pragma unroll
        for (int p = 0; p < kMaxPass; ++p) {
            const int g = p * gpp + sub;
            const int r = r0 + rr;
            const bool valid = p < npass && g < ng && r < H && blobs_s[g] != nullptr;
            code[rr][p] = make_uint4(0, 0, 0, 0);
            sc[rr][p][0] = 0.f;
            if (Q::BPC > 1) sc[rr][p][Q::BPC - 1] = 0.f;
            if (valid) {
                const BlobView bv = blob_view(blobs_s[g], BITS, H, I);
                code[rr][p] = ldg_stream(bv.cd + static_cast<size_t>(r) * drowb + static_cast<size_t>(seg) * 16);
                load_scales<BITS>(bv.sd + static_cast<size_t>(r) * dnsc, seg, true, sc[rr][p]);
            }
        }
    // h of every group as pieces + block sums
    float4 *hs = dsm;
    float *hcs = reinterpret_cast<float *>(dsm + static_cast<size_t>(ng) * (I / 4));
    {
        const void *rows[33];
        for (int g = 0; g < ng; ++g) rows[g] = a.ws.h + static_cast<size_t>(g) * I;
        stage_rows<BITS>(hs, hcs, ng, ng, I, rows, 0);
    }
#pragma unroll
    for (int rr = 0; rr < kDownRows; ++rr) {
        const int r = r0 + rr;
        float acc = 0.f;
#pragma unroll
        for (int p = 0; p < kMaxPass; ++p) {
            if (p >= npass) break;
            const int g = p * gpp + sub;
            float dot[1] = {0.f};
            if (g < ng && blobs_s[g])
                chunk_dot<BITS, 1>(code[rr][p], sc[rr][p], hs + static_cast<size_t>(g) * (I / 4),
                                   hcs + static_cast<size_t>(g) * (I / 32), nchd, seg, dot);
            float v = dot[0];
            for (int o = lpr >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            for (int s2 = 0; s2 < gpp; ++s2) {           // slot order: groups p*gpp + s2
                const float vs = __shfl_sync(0xffffffffu, v, s2 * lpr);
                const int gg = p * gpp + s2;
                if (gg < ng) acc = fmaf(gates_s[gg], vs, acc);
            }
        }
        if (lane == 0 && r < H) a.y[r] = acc;
    }
}

// ------------------------------------------------------------------ host
size_t decode_ws_bytes(int E, int k, int I) {
    return 256 + ((static_cast<size_t>(E) * 4 + 255) / 256) * 256 + static_cast<size_t>(k + 1) * I * 4;
}

bool decode_supported(int bits, int H, int I, int E, int k) {
    if (E > 1024 || k > 32 || H > 2048 || I % 128 != 0) return false;
    const int nchd = I / (bits == 4 ? 32 : 64);
    if (nchd > 32 || (nchd & (nchd - 1)) != 0) return false;    // one chunk per lane, power-of-two lanes per row
    const int gpp = 32 / nchd;
    if (ceil_div(k + 1, gpp) > kMaxPass) return false;
    const size_t smem_down = static_cast<size_t>(k + 1) * I * 4 + static_cast<size_t>(k + 1) * (I / 32) * 4;
    return smem_down <= 200 * 1024;
}

template <int BITS>
static int launch_decode_t(DecodeArgs a, int groups, cudaStream_t s) {
    const int H = a.H, I = a.I, E = a.E;
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    // 1. route: one cluster (16 CTAs when the router is computed here)
    {
        int C = a.logits_in ? 1 : 16;
        const size_t smem = (static_cast<size_t>(H) + ceil_div(E, C) + E) * 4;
        int rc = cuda_status(cudaFuncSetAttribute(k_dec_route, cudaFuncAttributeNonPortableClusterSizeAllowed, 1),
                             "route cluster attribute");
        if (rc) return rc;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(C);
        cfg.blockDim = dim3(kDecThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        rc = cuda_status(cudaLaunchKernelEx(&cfg, k_dec_route, a), "decode route launch");
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
    {
        const int nchd = I / QT<BITS>::EPC;
        const int lpr = nchd;
        const size_t smem = static_cast<size_t>(groups) * I * 4 + static_cast<size_t>(groups) * (I / 32) * 4;
        int rc = cuda_status(cudaFuncSetAttribute(k_dec_down<BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  static_cast<int>(smem)),
                             "down smem attribute");
        if (rc) return rc;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(ceil_div(H, kDecWarps * kDownRows));
        cfg.blockDim = dim3(kDecThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cfg.attrs = &pdl;
        cfg.numAttrs = 1;
        rc = cuda_status(cudaLaunchKernelEx(&cfg, k_dec_down<BITS>, a, groups, lpr), "decode down launch");
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
