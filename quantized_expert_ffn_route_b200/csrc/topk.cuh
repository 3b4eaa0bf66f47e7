// Selection keys and the gate softmax shared by the top-k kernels.
// Order: larger logit first, equal logits by lower expert id, NaN below -inf.
#pragma once

#include "common.cuh"

namespace moe {

// Order-preserving 32-bit key of a float: larger float -> larger key,
// -0 and +0 equal, every NaN -> 0 (below -inf, whose key is 0x007fffff).
__device__ __forceinline__ uint32_t float_key(float v) {
    if (v != v) return 0u;
    if (v == 0.0f) v = 0.0f;
    uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    if (k == 0u) return __uint_as_float(0x7fc00000u);
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}
// 64-bit selection key: value key, then the larger the lower the id.
__device__ __forceinline__ uint64_t sel_key(float v, int e) {
    return (static_cast<uint64_t>(float_key(v)) << 32) | static_cast<uint32_t>(0xffffffffu - static_cast<uint32_t>(e));
}
__device__ __forceinline__ uint64_t shfl_max64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

// ------------------------------------------------------------- gate math
// Every lane holds (v_j, id_j) for slot j = lane (< k).  Writes ids and gates.
__device__ __forceinline__ void write_gates(int lane, int k, float my_v, int my_id, int32_t *ids, float *w,
                                            unsigned *err) {
    const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
    const bool bad = lane < k && (my_v != my_v || my_v == __int_as_float(0x7f800000));
    const bool any_bad = __any_sync(0xffffffffu, bad);
    float ex = lane < k ? expf(my_v - v0) : 0.f;
    float s = 0.f;
    for (int j = 0; j < k; ++j) s += __shfl_sync(0xffffffffu, ex, j);   // slot order
    if (lane < k) {
        ids[lane] = my_id;
        w[lane] = any_bad ? __int_as_float(0x7fc00000) : ex / s;
    }
    if (any_bad && lane == 0) report(err, MOE_DEVERR_NONFINITE);
}

// ------------------------------------------------------- block top-k
// k best of N keys per lane by one warp.  Each lane first sorts its keys
// (descending, a bitonic network on registers); then every round the warp
// takes the largest head: a max reduction of the value halves, and only when
// several heads share that value a second one of the low words (the larger
// low word is the lower id).  The winning lane pops its head.  dst[r]
// receives the rank-r key.
template <int N>
__device__ __forceinline__ void warp_take(uint64_t (&keys)[N], int k, int lane, uint64_t *dst) {
#pragma unroll
    for (int k2 = 2; k2 <= N; k2 <<= 1)
#pragma unroll
        for (int j = k2 >> 1; j > 0; j >>= 1)
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int l = i ^ j;
                if (l > i) {
                    const bool desc = (i & k2) == 0;
                    const uint64_t a = keys[i], b = keys[l];
                    if (desc ? a < b : a > b) {
                        keys[i] = b;
                        keys[l] = a;
                    }
                }
            }
    for (int r = 0; r < k; ++r) {
        const uint64_t head = keys[0];
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
        const uint32_t wlo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(head), winner);
        if (lane == 0) dst[r] = (static_cast<uint64_t>(hi) << 32) | wlo;
        if (lane == winner) {
#pragma unroll
            for (int q = 0; q + 1 < N; ++q) keys[q] = keys[q + 1];
            keys[N - 1] = 0ull;
        }
    }
}

// Top-k (k <= 32) of E <= 32 * NW * KPT logits by one block of NW warps in
// two short stages: each warp takes the k best of its keys (KPT per lane),
// then warp 0 merges the NW sorted candidate lists as a tournament (lane l
// holds the head of list l; each round the best head wins and its lane
// reads its next candidate).  sel[0..k-1] receives the keys in rank order.
template <int NW, int KPT>
__device__ void block_topk_merge(const float *logits, int E, int k, uint64_t *cand, uint64_t *sel) {
    static_assert(NW <= 32, "one list per lane in the merge");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    {
        uint64_t keys[KPT];
#pragma unroll
        for (int q = 0; q < KPT; ++q) {
            const int e = threadIdx.x + 32 * NW * q;
            keys[q] = e < E ? sel_key(__ldcg(logits + e), e) : 0ull;
        }
        warp_take(keys, k, lane, cand + warp * k);
    }
    __syncthreads();
    if (warp == 0) {
        int pos = 0;
        uint64_t head = lane < NW ? cand[lane * k] : 0ull;
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
            const uint32_t wlo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(head), winner);
            if (lane == 0) sel[r] = (static_cast<uint64_t>(hi) << 32) | wlo;
            if (lane == winner) {
                ++pos;
                head = pos < k ? cand[lane * k + pos] : 0ull;
            }
        }
    }
    __syncthreads();
}

// Keeps the larger (keep_max) or smaller 64-bit key of this lane and lane ^ j.
__device__ __forceinline__ uint64_t cmpx(uint64_t v, int j, bool keep_max) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, v, j);
    return keep_max ? (o > v ? o : v) : (o < v ? o : v);
}

// Sorts one key per lane in descending order across the warp (lane 0 the
// largest): a bitonic network of 15 compare-exchange steps.
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t v, int lane) {
#pragma unroll
    for (int k2 = 2; k2 <= 32; k2 <<= 1)
#pragma unroll
        for (int j = k2 >> 1; j > 0; j >>= 1) v = cmpx(v, j, ((lane & k2) == 0 || k2 == 32) == ((lane & j) == 0));
    return v;
}

// Top-k (k <= 16) of E <= 32 * NW logits with one key per thread, as a merge
// tree: every warp sorts its 32 keys (bitonic network), keeps its best 16;
// then pairs of lists merge level by level (list a in lanes 0-15, list b
// reversed in lanes 16-31 form a bitonic sequence; five compare-exchange
// steps sort it), the best 16 of each merge going on, until one list is
// left.  sel[0..k-1] receives the keys in rank order.  lists: NW * 16 keys.
template <int NW>
__device__ void block_topk_tree(const float *logits, int E, int k, uint64_t *lists, uint64_t *sel) {
    static_assert((NW & (NW - 1)) == 0, "a power-of-two number of warps");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = threadIdx.x;
    uint64_t key = e < E ? sel_key(__ldcg(logits + e), e) : 0ull;
    key = warp_sort_desc(key, lane);
    if (lane < 16) lists[warp * 16 + lane] = key;
    __syncthreads();
#pragma unroll 1
    for (int n = NW; n > 1; n >>= 1) {
        uint64_t v = 0ull;
        if (warp < n / 2) {
            v = lane < 16 ? lists[(2 * warp) * 16 + lane] : lists[(2 * warp + 1) * 16 + (31 - lane)];
#pragma unroll
            for (int j = 16; j > 0; j >>= 1) v = cmpx(v, j, (lane & j) == 0);
        }
        __syncthreads();                                 // every read of this level before the writes
        if (warp < n / 2 && lane < 16) lists[warp * 16 + lane] = v;
        __syncthreads();
    }
    if (threadIdx.x < k) sel[threadIdx.x] = lists[threadIdx.x];
    __syncthreads();
}

// Sorts 32 * N keys, N per lane (element lane + 32 q in v[q]), in descending
// order across the warp: a bitonic network whose compare-exchanges at
// strides of 32 and more pair two keys of the same lane.
template <int N>
__device__ __forceinline__ void warp_sort_desc_n(uint64_t (&v)[N], int lane) {
#pragma unroll
    for (int k2 = 2; k2 <= 32 * N; k2 <<= 1)
#pragma unroll
        for (int j = k2 >> 1; j > 0; j >>= 1) {
            if (j >= 32) {                               // partner in the same lane
#pragma unroll
                for (int q = 0; q < N; ++q) {
                    const int p = q ^ (j >> 5);
                    if (p > q) {
                        const bool desc = k2 == 32 * N || ((lane + 32 * q) & k2) == 0;
                        const uint64_t lo_i = v[q], hi_i = v[p];
                        const bool swap = desc ? lo_i < hi_i : lo_i > hi_i;
                        v[q] = swap ? hi_i : lo_i;
                        v[p] = swap ? lo_i : hi_i;
                    }
                }
            } else {
#pragma unroll
                for (int q = 0; q < N; ++q) {
                    const int i = lane + 32 * q;
                    const bool desc = k2 == 32 * N || (i & k2) == 0;
                    v[q] = cmpx(v[q], j, desc == ((i & j) == 0));
                }
            }
        }
}

// block_topk_tree with N keys per thread: E <= 32 * N * NW, k <= 16.  Warp w
// sorts the keys of experts [32 N w, 32 N (w + 1)); the merge levels follow.
template <int NW, int N>
__device__ void block_topk_tree_n(const float *logits, int E, int k, uint64_t *lists, uint64_t *sel) {
    static_assert((NW & (NW - 1)) == 0, "a power-of-two number of warps");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t v[N];
#pragma unroll
    for (int q = 0; q < N; ++q) {
        const int e = warp * 32 * N + lane + 32 * q;
        v[q] = e < E ? sel_key(__ldcg(logits + e), e) : 0ull;
    }
    warp_sort_desc_n<N>(v, lane);
    if (lane < 16) lists[warp * 16 + lane] = v[0];
    __syncthreads();
#pragma unroll 1
    for (int n = NW; n > 1; n >>= 1) {
        uint64_t m = 0ull;
        if (warp < n / 2) {
            m = lane < 16 ? lists[(2 * warp) * 16 + lane] : lists[(2 * warp + 1) * 16 + (31 - lane)];
#pragma unroll
            for (int j = 16; j > 0; j >>= 1) m = cmpx(m, j, (lane & j) == 0);
        }
        __syncthreads();                                 // every read of this level before the writes
        if (warp < n / 2 && lane < 16) lists[warp * 16 + lane] = m;
        __syncthreads();
    }
    if (threadIdx.x < k) sel[threadIdx.x] = lists[threadIdx.x];
    __syncthreads();
}

}  // namespace moe
