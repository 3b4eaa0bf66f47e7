// Token-to-expert permute: stable counting sort of the (token, slot) pairs by
// expert id.  Rows of one expert are contiguous and in ascending token order,
// so the result is unique and the kernels are deterministic (no atomics on
// anything but counts, whose values do not depend on order).
#include "common.cuh"
#include "kernels.h"

namespace moe {

// Exclusive scan over n counts held in shared memory (in place), also
// writing offsets[0..n] and the list of nonzero entries to global memory.
// Runs on a whole 1024-thread block.
__device__ void block_scan_counts(int32_t *cnt, int n, int32_t *offsets, int32_t *active, int active_cap) {
    __shared__ int32_t part[1024];
    __shared__ int32_t apart[1024];
    const int tid = threadIdx.x;
    const int per = (n + 1023) / 1024;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    int32_t s = 0, a = 0;
    for (int i = lo; i < hi; ++i) {
        s += cnt[i];
        a += cnt[i] > 0;
    }
    part[tid] = s;
    apart[tid] = a;
    __syncthreads();
    // Hillis-Steele inclusive scan over 1024 partials
    for (int o = 1; o < 1024; o <<= 1) {
        int32_t v = tid >= o ? part[tid - o] : 0;
        int32_t va = tid >= o ? apart[tid - o] : 0;
        __syncthreads();
        part[tid] += v;
        apart[tid] += va;
        __syncthreads();
    }
    int32_t run = tid ? part[tid - 1] : 0;
    int32_t arun = tid ? apart[tid - 1] : 0;
    for (int i = lo; i < hi; ++i) {
        int32_t c = cnt[i];
        offsets[i] = run;
        cnt[i] = run;            // becomes the write cursor
        if (c > 0 && active && arun < active_cap) active[1 + arun] = i;
        arun += c > 0;
        run += c;
    }
    if (tid == 1023) {
        offsets[n] = part[1023];
        if (active) active[0] = apart[1023];
    }
    __syncthreads();
}

// Ranks the pairs [p0, p1) in order with one warp: rows = cursor[e] + rank among
// equal ids inside each 32-pair group; advances the cursors.
__device__ __forceinline__ void warp_scatter(const int32_t *ids, int p0, int p1, int k, int E, int32_t *cursor,
                                             int32_t *perm_src, int32_t *perm_dst) {
    const int lane = threadIdx.x & 31;
    for (int base = p0; base < p1; base += 32) {
        const int p = base + lane;
        const bool live = p < p1;
        const unsigned livemask = __ballot_sync(0xffffffffu, live);
        int e = live ? ids[p] : -1;
        const bool ok = live && e >= 0 && e < E;
        e = ok ? e : -1 - lane;                          // invalid ids never group
        const unsigned peers = __match_any_sync(0xffffffffu, e) & livemask;
        const int rank = __popc(peers & ((1u << lane) - 1u));
        int pos = ok ? cursor[e] : 0;
        __syncwarp();
        const bool last_of_group = ok && (peers >> lane) == 1u;
        if (last_of_group) cursor[e] = pos + rank + 1;
        __syncwarp();
        if (ok) {
            const int r = pos + rank;
            perm_src[r] = p / k;
            perm_dst[p] = r;
        }
    }
}

// Whole permute in one block (small T*k and E): counts in shared memory.
__global__ void __launch_bounds__(1024) k_permute_small(const int32_t *__restrict__ ids, int T, int k, int E,
                                                         int32_t *__restrict__ offsets, int32_t *__restrict__ perm_src,
                                                         int32_t *__restrict__ perm_dst, int32_t *__restrict__ active,
                                                         int active_cap, unsigned *err) {
    extern __shared__ int32_t cnt[];
    const int n = T * k;
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int p = threadIdx.x; p < n; p += blockDim.x) {
        int e = ids[p];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
        else report(err, MOE_DEVERR_BAD_EXPERT);
    }
    __syncthreads();
    block_scan_counts(cnt, E, offsets, active, active_cap);
    if (threadIdx.x < 32) warp_scatter(ids, 0, n, k, E, cnt, perm_src, perm_dst);
}

// Few pairs (n = T*k <= 32, e.g. one decode token) and any E: no counting
// array over the experts.  Warp 0 holds the n ids; the row of a valid pair is
// the number of valid pairs with a smaller id plus the earlier pairs with the
// same id (the stable order) -- its position in the sorted list of valid ids
// -- and each offset is the number of valid pairs with a smaller id, found by
// walking that sorted list alongside the thread's increasing experts.
constexpr int kSparsePairs = 32;

__global__ void __launch_bounds__(1024) k_permute_sparse(const int32_t *__restrict__ ids, int n, int k, int E,
                                                          int32_t *__restrict__ offsets,
                                                          int32_t *__restrict__ perm_src,
                                                          int32_t *__restrict__ perm_dst,
                                                          int32_t *__restrict__ active, int active_cap,
                                                          unsigned *err) {
    __shared__ int ids_s[kSparsePairs], sorted_s[kSparsePairs], nv_s;
    const int tid = threadIdx.x;
    if (tid < 32) {
        const int lane = tid;
        const bool live = lane < n;
        const int e = live ? ids[lane] : -1;
        const bool ok = live && e >= 0 && e < E;
        if (live && !ok) report(err, MOE_DEVERR_BAD_EXPERT);
        ids_s[lane] = ok ? e : -1;                       // -1: no valid pair here
        __syncwarp();
        int r = 0, d = 0;
        bool first = ok;
        for (int q = 0; q < n; ++q) {
            const int f = ids_s[q];
            if (f < 0) continue;
            r += f < e || (f == e && q < lane);
            first &= !(f == e && q < lane);
            if (ok && f < e) {                           // distinct ids below e: count first occurrences
                bool fq = true;
                for (int u = 0; u < q; ++u) fq &= ids_s[u] != f;
                d += fq;
            }
        }
        if (ok) {
            perm_src[r] = lane / k;
            perm_dst[lane] = r;
            sorted_s[r] = e;
            if (first && active && d < active_cap) active[1 + d] = e;
        }
        const unsigned firsts = __ballot_sync(0xffffffffu, first);
        const unsigned valid = __ballot_sync(0xffffffffu, ok);
        if (lane == 0 && active) active[0] = __popc(firsts);
        if (lane == 0) nv_s = __popc(valid);
    }
    __syncthreads();
    const int nv = nv_s;
    int p = 0;                                           // sorted ids below e (e grows with each pass)
    for (int e = tid; e <= E; e += blockDim.x) {
        while (p < nv && sorted_s[p] < e) ++p;
        offsets[e] = p;
    }
}

// General path, step 1: per-chunk counts (chunk c = pairs [c*P, (c+1)*P)).
__global__ void k_permute_count(const int32_t *__restrict__ ids, int n, int E, int P, int32_t *__restrict__ cc,
                                unsigned *err) {
    const int c = blockIdx.x;
    const int p0 = c * P, p1 = min(n, p0 + P);
    for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
        int e = ids[p];
        if (e >= 0 && e < E) atomicAdd(&cc[static_cast<size_t>(c) * E + e], 1);
        else report(err, MOE_DEVERR_BAD_EXPERT);
    }
}

// Step 2 (one block): per-expert running sums over chunks, global offsets,
// active list; cc[c][e] becomes the first row of chunk c's pairs of expert e.
__global__ void __launch_bounds__(1024) k_permute_scan(int32_t *__restrict__ cc, int C, int E,
                                                        int32_t *__restrict__ tot, int32_t *__restrict__ offsets,
                                                        int32_t *__restrict__ active, int active_cap) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = 0;
        for (int c = 0; c < C; ++c) {
            int32_t v = cc[static_cast<size_t>(c) * E + e];
            cc[static_cast<size_t>(c) * E + e] = run;
            run += v;
        }
        tot[e] = run;
    }
    __syncthreads();
    // tot is a global scratch array; scan it in place through the block
    extern __shared__ int32_t stot[];
    const bool in_smem = E <= 32768;
    int32_t *arr = in_smem ? stot : tot;
    if (in_smem) {
        for (int e = threadIdx.x; e < E; e += blockDim.x) stot[e] = tot[e];
        __syncthreads();
    }
    block_scan_counts(arr, E, offsets, active, active_cap);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int32_t o = offsets[e];
        for (int c = 0; c < C; ++c) cc[static_cast<size_t>(c) * E + e] += o;
    }
}

// Step 3: one warp per chunk scatters its pairs in order.
__global__ void k_permute_scatter(const int32_t *__restrict__ ids, int n, int k, int E, int P,
                                  int32_t *__restrict__ cc, int32_t *__restrict__ perm_src,
                                  int32_t *__restrict__ perm_dst) {
    const int c = blockIdx.x;
    const int p0 = c * P, p1 = min(n, p0 + P);
    warp_scatter(ids, p0, p1, k, E, cc + static_cast<size_t>(c) * E, perm_src, perm_dst);
}

static constexpr int kSmallPairs = 4096;
static constexpr int kSmallE = 32768;
static constexpr int kChunkPairs = 1024;

size_t permute_ws_bytes(int T, int k, int E) {
    const long n = static_cast<long>(T) * k;
    if (n <= kSparsePairs || (n <= kSmallPairs && E <= kSmallE)) return 0;
    const long C = (n + kChunkPairs - 1) / kChunkPairs;
    return static_cast<size_t>((C + 1) * E) * sizeof(int32_t);
}

int launch_permute(const int32_t *ids, int T, int k, int E, int32_t *offsets, int32_t *perm_src,
                   int32_t *perm_dst, int32_t *active, void *ws, unsigned *err, cudaStream_t s) {
    const int n = T * k;
    const int active_cap = n < E ? n : E;
    if (n <= kSparsePairs) {
        k_permute_sparse<<<1, 1024, 0, s>>>(ids, n, k, E, offsets, perm_src, perm_dst, active, active_cap, err);
        count_launches(1);
        return cuda_status(cudaGetLastError(), "permute launch");
    }
    if (n <= kSmallPairs && E <= kSmallE) {
        const size_t smem = static_cast<size_t>(E) * sizeof(int32_t);
        cudaFuncSetAttribute(k_permute_small, cudaFuncAttributeMaxDynamicSharedMemorySize, 32768 * 4);
        k_permute_small<<<1, 1024, smem, s>>>(ids, T, k, E, offsets, perm_src, perm_dst, active, active_cap, err); count_launches(1);
        return cuda_status(cudaGetLastError(), "permute launch");
    }
    const int C = (n + kChunkPairs - 1) / kChunkPairs;
    int32_t *cc = static_cast<int32_t *>(ws);
    int32_t *tot = cc + static_cast<size_t>(C) * E;
    int st = cuda_status(cudaMemsetAsync(cc, 0, static_cast<size_t>(C) * E * sizeof(int32_t), s), "permute memset");
    if (st) return st;
    k_permute_count<<<C, 256, 0, s>>>(ids, n, E, kChunkPairs, cc, err); count_launches(1);
    const size_t smem = E <= kSmallE ? static_cast<size_t>(E) * sizeof(int32_t) : 0;
    cudaFuncSetAttribute(k_permute_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, 32768 * 4);
    k_permute_scan<<<1, 1024, smem, s>>>(cc, C, E, tot, offsets, active, active_cap); count_launches(1);
    k_permute_scatter<<<C, 32, 0, s>>>(ids, n, k, E, kChunkPairs, cc, perm_src, perm_dst); count_launches(1);
    return cuda_status(cudaGetLastError(), "permute launch");
}

}  // namespace moe
