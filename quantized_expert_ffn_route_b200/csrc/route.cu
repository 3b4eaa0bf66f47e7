// Router logits and top-k gate.
//
// Strata article, summary table / section 2 item 1: each token activates 10
// of 24,576 experts; section 2 item 2: the router's choice decides which
// experts are computed.  Selection order: larger logit first, equal logits by
// lower expert id, NaN below -inf.  Gates: softmax over the k selected.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace moe {

// --------------------------------------------------------------- logits
// One warp per (expert row, group of TT tokens): the router row is streamed
// once per token group with 16-byte loads; fp32 accumulation.
template <int TT, typename XT, typename WT>
__global__ void __launch_bounds__(256) k_router_logits(const XT *__restrict__ x, const WT *__restrict__ w,
                                                        const float *__restrict__ bias, int T, int H, int E,
                                                        float *__restrict__ logits) {
    const int lane = threadIdx.x & 31;
    const int warps = blockDim.x >> 5;
    const int n_tg = (T + TT - 1) / TT;
    const long total = static_cast<long>(E) * n_tg;
    for (long task = static_cast<long>(blockIdx.x) * warps + (threadIdx.x >> 5); task < total;
         task += static_cast<long>(gridDim.x) * warps) {
        const int e = static_cast<int>(task % E);
        const int t0 = static_cast<int>(task / E) * TT;
        float acc[TT];
#pragma unroll
        for (int j = 0; j < TT; ++j) acc[j] = 0.f;
        const WT *wr = w + static_cast<size_t>(e) * H;
        for (int h = lane * 8; h < H; h += 256) {
            float4 w0 = load4(wr + h), w1 = load4(wr + h + 4);
#pragma unroll
            for (int j = 0; j < TT; ++j) {
                if (t0 + j < T) {
                    const XT *xr = x + static_cast<size_t>(t0 + j) * H + h;
                    float4 a = load4(xr), b = load4(xr + 4);
                    float s = acc[j];
                    s = fmaf(w0.x, a.x, s); s = fmaf(w0.y, a.y, s); s = fmaf(w0.z, a.z, s); s = fmaf(w0.w, a.w, s);
                    s = fmaf(w1.x, b.x, s); s = fmaf(w1.y, b.y, s); s = fmaf(w1.z, b.z, s); s = fmaf(w1.w, b.w, s);
                    acc[j] = s;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < TT; ++j) {
            float s = warp_sum(acc[j]);
            if (lane == 0 && t0 + j < T) logits[static_cast<size_t>(t0 + j) * E + e] = s + (bias ? bias[e] : 0.f);
        }
    }
}

// One warp per token, E <= 32 * NPL.
template <int NPL>
__global__ void __launch_bounds__(256) k_topk_warp(const float *__restrict__ logits, int T, int E, int k,
                                                    int32_t *__restrict__ ids, float *__restrict__ w,
                                                    unsigned *err) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *l = logits + static_cast<size_t>(t) * E;
    uint64_t key[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        int e = lane + 32 * i;
        key[i] = e < E ? sel_key(l[e], e) : 0ull;
    }
    uint64_t last = ~0ull;
    float my_v = 0.f;
    int my_id = 0;
    for (int j = 0; j < k; ++j) {
        uint64_t m = 0ull;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            uint64_t c = key[i] < last ? key[i] : 0ull;
            m = c > m ? c : m;
        }
        m = shfl_max64(m);
        last = m;
        if (lane == j) {
            my_v = key_float(static_cast<uint32_t>(m >> 32));
            my_id = static_cast<int>(0xffffffffu - static_cast<uint32_t>(m));
        }
    }
    write_gates(lane, k, my_v, my_id, ids + static_cast<size_t>(t) * k, w + static_cast<size_t>(t) * k, err);
}

// One 1024-thread block per token, E <= 1024 * NPT.  32-bit value keys are
// kept in registers; the id half of the selection key is rebuilt on the fly.
template <int NPT>
__global__ void __launch_bounds__(1024) k_topk_block(const float *__restrict__ logits, int T, int E, int k,
                                                      int32_t *__restrict__ ids, float *__restrict__ w,
                                                      unsigned *err) {
    __shared__ uint64_t red[32];
    __shared__ uint64_t chosen[32];
    const int t = blockIdx.x;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const float *l = logits + static_cast<size_t>(t) * E;
    uint32_t vkey[NPT];
#pragma unroll
    for (int i = 0; i < NPT; ++i) {
        int e = threadIdx.x + 1024 * i;
        vkey[i] = e < E ? float_key(l[e]) : 0u;
    }
    uint64_t last = ~0ull;
    for (int j = 0; j < k; ++j) {
        uint64_t m = 0ull;
#pragma unroll
        for (int i = 0; i < NPT; ++i) {
            int e = threadIdx.x + 1024 * i;
            uint64_t c = e < E ? ((static_cast<uint64_t>(vkey[i]) << 32) |
                                  static_cast<uint32_t>(0xffffffffu - static_cast<uint32_t>(e)))
                               : 0ull;
            c = c < last ? c : 0ull;
            m = c > m ? c : m;
        }
        m = shfl_max64(m);
        if (lane == 0) red[wid] = m;
        __syncthreads();
        if (wid == 0) {
            uint64_t v = red[lane];
            v = shfl_max64(v);
            if (lane == 0) chosen[j] = v;
        }
        __syncthreads();
        last = chosen[j];
    }
    if (wid == 0) {
        uint64_t m = lane < k ? chosen[lane] : 0ull;
        float my_v = key_float(static_cast<uint32_t>(m >> 32));
        int my_id = static_cast<int>(0xffffffffu - static_cast<uint32_t>(m));
        write_gates(lane, k, my_v, my_id, ids + static_cast<size_t>(t) * k, w + static_cast<size_t>(t) * k, err);
    }
}

// ------------------------------------------------------------- launchers
template <typename XT, typename WT>
static void launch_logits_t(const void *x, const void *w, const float *bias, int T, int H, int E, float *out,
                            cudaStream_t s) {
    const int threads = 128, warps = threads / 32;
    const int tt = T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : 8;
    const long tasks = static_cast<long>(E) * ((T + tt - 1) / tt);
    long blocks = (tasks + warps - 1) / warps;
    const long cap = static_cast<long>(num_sms()) * 16;
    if (blocks > cap) blocks = cap;
    auto xp = static_cast<const XT *>(x);
    auto wp = static_cast<const WT *>(w);
    switch (tt) {
        case 1: k_router_logits<1, XT, WT><<<blocks, threads, 0, s>>>(xp, wp, bias, T, H, E, out); count_launches(1); break;
        case 2: k_router_logits<2, XT, WT><<<blocks, threads, 0, s>>>(xp, wp, bias, T, H, E, out); count_launches(1); break;
        case 4: k_router_logits<4, XT, WT><<<blocks, threads, 0, s>>>(xp, wp, bias, T, H, E, out); count_launches(1); break;
        default: k_router_logits<8, XT, WT><<<blocks, threads, 0, s>>>(xp, wp, bias, T, H, E, out); count_launches(1); break;
    }
}

void launch_router_logits(const void *x, int x_dtype, const void *w, int w_dtype, const float *bias, int T,
                          int H, int E, float *out, cudaStream_t s) {
    if (x_dtype == MOE_BF16 && w_dtype == MOE_BF16)
        launch_logits_t<__nv_bfloat16, __nv_bfloat16>(x, w, bias, T, H, E, out, s);
    else if (x_dtype == MOE_BF16)
        launch_logits_t<__nv_bfloat16, float>(x, w, bias, T, H, E, out, s);
    else if (w_dtype == MOE_BF16)
        launch_logits_t<float, __nv_bfloat16>(x, w, bias, T, H, E, out, s);
    else
        launch_logits_t<float, float>(x, w, bias, T, H, E, out, s);
}

void launch_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w, unsigned *err,
                 cudaStream_t s) {
    if (E <= 1024) {
        const int threads = 256, per = threads / 32;
        const int blocks = (T + per - 1) / per;
        if (E <= 64) { k_topk_warp<2><<<blocks, threads, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
        else if (E <= 256) { k_topk_warp<8><<<blocks, threads, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
        else if (E <= 512) { k_topk_warp<16><<<blocks, threads, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
        else { k_topk_warp<32><<<blocks, threads, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
    } else {
        if (E <= 8192) { k_topk_block<8><<<T, 1024, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
        else if (E <= 16384) { k_topk_block<16><<<T, 1024, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
        else { k_topk_block<32><<<T, 1024, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
    }
}

}  // namespace moe
