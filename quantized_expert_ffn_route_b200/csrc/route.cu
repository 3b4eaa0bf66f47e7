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

// E > 1024: the logits split into chunks of kTopkChunk; one 256-thread CTA
// per (token, chunk) selects the chunk's best k (block_topk_merge) and writes
// them, as selection keys re-based to global ids, to the workspace; then one
// warp per token merges the sorted chunk lists (lane c holds the head of
// chunk c's list; each round the best head wins and its lane reads on).  The
// whole GPU shares the selection instead of one SM scanning every logit k
// times.  Keys of missing entries (a chunk shorter than k) are 0, below every
// real key.
constexpr int kTopkChunk = 2048;

__global__ void __launch_bounds__(256) k_topk_chunk(const float *__restrict__ logits, int E, int k,
                                                    uint64_t *__restrict__ cand) {
    __shared__ uint64_t c_s[8 * 32], sel[32];
    const int t = blockIdx.x, c = blockIdx.y, C = gridDim.y;
    const int e0 = c * kTopkChunk;
    const int n = min(kTopkChunk, E - e0);
    block_topk_merge<8, kTopkChunk / 256>(logits + static_cast<size_t>(t) * E + e0, n, k, c_s, sel);
    if (threadIdx.x < k) {
        uint64_t key = sel[threadIdx.x];
        if (key) {
            const uint32_t local = 0xffffffffu - static_cast<uint32_t>(key);
            key = (key & 0xffffffff00000000ull) | (0xffffffffu - (local + static_cast<uint32_t>(e0)));
        }
        cand[(static_cast<size_t>(t) * C + c) * k + threadIdx.x] = key;
    }
}

__global__ void __launch_bounds__(32) k_topk_merge_chunks(const uint64_t *__restrict__ cand, int C, int k,
                                                          int32_t *__restrict__ ids, float *__restrict__ w,
                                                          unsigned *err) {
    const int t = blockIdx.x, lane = threadIdx.x;
    const uint64_t *cl = cand + static_cast<size_t>(t) * C * k;
    int pos = 0;
    uint64_t head = lane < C ? cl[static_cast<size_t>(lane) * k] : 0ull, mine = 0ull;
    for (int r = 0; r < k; ++r) {
        const uint32_t hv = static_cast<uint32_t>(head >> 32);
        const uint32_t hi = __reduce_max_sync(0xffffffffu, hv);
        const unsigned tied = __ballot_sync(0xffffffffu, hv == hi);
        int winner;
        if (__popc(tied) == 1) {
            winner = __ffs(tied) - 1;
        } else {
            const uint32_t lo = __reduce_max_sync(0xffffffffu, hv == hi ? static_cast<uint32_t>(head) : 0u);
            winner = __ffs(__ballot_sync(0xffffffffu, hv == hi && static_cast<uint32_t>(head) == lo)) - 1;
        }
        const uint64_t won = __shfl_sync(0xffffffffu, head, winner);
        if (lane == r) mine = won;
        if (lane == winner) {
            ++pos;
            head = pos < k ? cl[static_cast<size_t>(lane) * k + pos] : 0ull;
        }
    }
    const float my_v = key_float(static_cast<uint32_t>(mine >> 32));
    const int my_id = static_cast<int>(0xffffffffu - static_cast<uint32_t>(mine));
    write_gates(lane, k, my_v, my_id, ids + static_cast<size_t>(t) * k, w + static_cast<size_t>(t) * k, err);
}

size_t topk_chunk_ws_offset(int T, int E) { return (static_cast<size_t>(T) * E * sizeof(float) + 255) / 256 * 256; }

size_t topk_chunk_ws_bytes(int T, int E, int k) {
    return static_cast<size_t>(T) * ((E + kTopkChunk - 1) / kTopkChunk) * k * sizeof(uint64_t);
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

void launch_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w, unsigned *err, void *cand_ws,
                 cudaStream_t s) {
    if (E <= 1024) {
        const int threads = 256, per = threads / 32;
        const int blocks = (T + per - 1) / per;
        if (E <= 64) { k_topk_warp<2><<<blocks, threads, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
        else if (E <= 256) { k_topk_warp<8><<<blocks, threads, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
        else if (E <= 512) { k_topk_warp<16><<<blocks, threads, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
        else { k_topk_warp<32><<<blocks, threads, 0, s>>>(logits, T, E, k, ids, w, err); count_launches(1); }
    } else {
        const int C = (E + kTopkChunk - 1) / kTopkChunk;            // <= 16 for E <= 32768
        uint64_t *cand = static_cast<uint64_t *>(cand_ws);
        k_topk_chunk<<<dim3(T, C), 256, 0, s>>>(logits, E, k, cand);
        k_topk_merge_chunks<<<T, 32, 0, s>>>(cand, C, k, ids, w, err);
        count_launches(2);
    }
}

}  // namespace moe
