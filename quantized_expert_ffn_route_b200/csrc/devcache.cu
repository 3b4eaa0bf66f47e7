// Device-initiated expert staging: the expert cache's policy and its copies
// run on the GPU, so a step never hands the router's ids to the host.
//
// The host-driven cache (expcache.cu) reads the step's ids on the host, runs
// the policy there and issues one cudaMemcpyAsync per miss: every step pays a
// device->host copy of the ids and a host synchronisation before any copy can
// start.  Here the same policy (halving decay, victim = the resident expert
// outside the step with the smallest (count, last use, id), lowest free slot
// first) runs in one CTA on the device, reading the ids where the router left
// them, and a copy kernel pulls the admitted misses from the page-locked host
// pool (mapped into the device address space) with 16-byte loads over the
// host link.  A whole step -- route, permute, policy, copies, FFN, combine --
// is then a fixed sequence of launches that a CUDA graph can hold.
//
// Zero-copy compute for cold experts (optional, admit_min > 1): a missed
// expert whose count after this use is still below admit_min is not admitted;
// its table entry points at its blob in the host pool for this step and the
// FFN reads it over the link in place (no slot is taken, nothing is evicted).
// The next step's policy kernel clears that entry again.
//
// Strata article, section 2 item 2: resident experts are computed at once,
// only the others move in from host memory; Strata code review, section 3:
// the page-locked stage buffer the host-driven design copies through.

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kDcThreads = 1024;
constexpr int kDcWarps = kDcThreads / 32;
constexpr int kDcMaxIds = 32;
constexpr int kDcCopyThreads = 256;
constexpr int kDcCopyUnroll = 8;                   // 16-byte loads of a thread in flight together

struct DcMeta {
    long long step;
    long long hits, misses, evictions, inplace, bytes_copied, bad_steps;
    int n_copy;                                    // admitted misses of the last step
    int n_inplace;                                 // experts computed in place in the last step
    int copy_e[kDcMaxIds], copy_slot[kDcMaxIds];
    int inplace_e[kDcMaxIds];
};

struct DcArgs {
    int E, cap, decay, admit_min, log_steps;
    long long blob_bytes, stride;
    const uint8_t *pool;                           // the host pool as the device addresses it
    uint8_t *slab;
    const uint8_t **table;
    long long *cnt, *last;
    int *slot_of, *expert_in;
    DcMeta *meta;
    signed char *log_hit;                          // [log_steps][kDcMaxIds]
    int *log_slot, *log_victim;
    unsigned *err;
};

// (c, l, id) before (bc, bl, bid) in the eviction order; bid < 0: no candidate yet
__device__ __forceinline__ bool evict_before(long long c, long long l, int id, long long bc, long long bl, int bid) {
    if (bid < 0) return id >= 0;
    if (id < 0) return false;
    if (c != bc) return c < bc;
    if (l != bl) return l < bl;
    return id < bid;
}

__device__ __forceinline__ void reduce_victim(long long &bc, long long &bl, int &bid, int &bsl) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const long long oc = __shfl_xor_sync(0xffffffffu, bc, o);
        const long long ol = __shfl_xor_sync(0xffffffffu, bl, o);
        const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
        const int osl = __shfl_xor_sync(0xffffffffu, bsl, o);
        if (evict_before(oc, ol, oid, bc, bl, bid)) {
            bc = oc;
            bl = ol;
            bid = oid;
            bsl = osl;
        }
    }
}

// One step of the policy in one CTA.  act: [0] = n_a, [1..] ids of list A
// (hits and experts computed in place: usable at once); [33] = n_b, [34..]
// ids of list B (admitted misses: usable after the copy kernel).  Ids in the
// lists are the caller's (id_base not added), in step order.
//
// The sequential policy is evaluated without a sequential loop: a step's ids
// are distinct and never victims, so whether each is resident is fixed at
// the start of the step, and the victims' (count, last use, id) do not change
// during it.  Hence the admitted misses, in step order, take first the
// lowest free slots in increasing order, then the slots of the resident
// experts outside the step in increasing (count, last use, id) -- exactly
// what handling the ids one by one gives.
__global__ void __launch_bounds__(kDcThreads) k_dc_stage(DcArgs a, const int32_t *__restrict__ ids, int n, int base,
                                                         int32_t *__restrict__ act) {
    __shared__ int ids_s[kDcMaxIds], code_s[kDcMaxIds], slot_s[kDcMaxIds], victim_s[kDcMaxIds];
    __shared__ int miss_j[kDcMaxIds];                // step positions of the admitted misses, in order
    __shared__ int ok_s, nmiss_s, nfree_s;
    __shared__ int wsum[kDcWarps], rid[kDcWarps], rsl[kDcWarps];
    __shared__ long long rc[kDcWarps], rl[kDcWarps];
    DcMeta &m = *a.meta;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // last step's in-place entries go back to NULL (they were never admitted)
    if (tid < m.n_inplace) {
        const int e = m.inplace_e[tid];
        if (a.slot_of[e] < 0) a.table[e] = nullptr;
    }
    if (tid == 0) ok_s = 1;
    __syncthreads();
    if (tid < n) {
        const int l = ids[tid];
        const long long e = static_cast<long long>(l) + base;
        ids_s[tid] = static_cast<int>(e);
        if (l < 0 || e < 0 || e >= a.E) ok_s = 0;
    }
    __syncthreads();
    if (tid < n && ok_s)
        for (int j = 0; j < tid; ++j)
            if (ids_s[j] == ids_s[tid]) ok_s = 0;
    __syncthreads();
    if (!ok_s) {                                     // nothing changes; the FFN lists are empty
        if (tid == 0) {
            report(a.err, MOE_DEVERR_BAD_EXPERT);
            act[0] = 0;
            act[33] = 0;
            m.n_copy = 0;
            m.n_inplace = 0;
            m.bad_steps++;
        }
        return;
    }
    const long long s = m.step;
    if (a.decay > 0 && s > 0 && s % a.decay == 0)
        for (int e = tid; e < a.E; e += kDcThreads) a.cnt[e] /= 2;
    __syncthreads();
    // every id at once: count, last use, resident or not, computed in place or not
    if (tid < n) {
        const int e = ids_s[tid];
        const long long c = a.cnt[e] + 1;
        a.cnt[e] = c;
        a.last[e] = s;
        const int res = a.slot_of[e];
        code_s[tid] = res >= 0 ? 1 : (a.admit_min > 1 && c < a.admit_min ? 3 : 0);
        slot_s[tid] = res;
        victim_s[tid] = -1;
    }
    __syncthreads();
    if (tid == 0) {
        int q = 0;
        for (int j = 0; j < n; ++j)
            if (code_s[j] == 0) miss_j[q++] = j;
        nmiss_s = q;
    }
    __syncthreads();
    const int nm = nmiss_s;
    // thread t owns the contiguous slots [lo, hi)
    const int per = (a.cap + kDcThreads - 1) / kDcThreads;
    const int lo = min(a.cap, tid * per), hi = min(a.cap, lo + per);
    if (nm > 0) {
        // the nm lowest free slots, by a block scan of the free counts
        int mine = 0;
        for (int sl = lo; sl < hi; ++sl) mine += a.expert_in[sl] < 0;
        int inc = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        if (lane == 31) wsum[warp] = inc;
        __syncthreads();
        if (warp == 0) {
            int w = wsum[lane], wi = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += v;
            }
            wsum[lane] = wi - w;                         // exclusive prefix of the warps
            if (lane == 31) nfree_s = wi;
        }
        __syncthreads();
        int r = wsum[warp] + inc - mine;                 // free slots before this thread's
        for (int sl = lo; sl < hi && r < nm; ++sl)
            if (a.expert_in[sl] < 0) slot_s[miss_j[r++]] = sl;
        __syncthreads();
        // the remaining misses evict, in (count, last use, id) order
        const int nfree = min(nfree_s, nm);
#pragma unroll 1
        for (int v = nfree; v < nm; ++v) {
            long long bc = 0, bl = 0;
            int bid = -1, bsl = -1;
            for (int sl = lo; sl < hi; ++sl) {
                const int c = a.expert_in[sl];
                if (c < 0) continue;
                bool skip = false;
                for (int jj = 0; jj < n; ++jj) skip |= ids_s[jj] == c;
                for (int q = nfree; q < v; ++q) skip |= victim_s[miss_j[q]] == c;
                if (!skip && evict_before(a.cnt[c], a.last[c], c, bc, bl, bid)) {
                    bc = a.cnt[c];
                    bl = a.last[c];
                    bid = c;
                    bsl = sl;
                }
            }
            reduce_victim(bc, bl, bid, bsl);
            if (lane == 0) {
                rc[warp] = bc;
                rl[warp] = bl;
                rid[warp] = bid;
                rsl[warp] = bsl;
            }
            __syncthreads();
            if (warp == 0) {
                bc = rc[lane];
                bl = rl[lane];
                bid = rid[lane];
                bsl = rsl[lane];
                reduce_victim(bc, bl, bid, bsl);   // bid >= 0: capacity >= n
                if (lane == 0) {
                    victim_s[miss_j[v]] = bid;
                    slot_s[miss_j[v]] = bsl;
                }
            }
            __syncthreads();
        }
    }
    // apply: one thread per id (the effects of different ids are disjoint)
    if (tid < n) {
        const int e = ids_s[tid], code = code_s[tid];
        if (code == 0) {
            const int sl = slot_s[tid], v = victim_s[tid];
            if (v >= 0) {
                a.slot_of[v] = -1;
                a.table[v] = nullptr;
            }
            a.slot_of[e] = sl;
            a.expert_in[sl] = e;
            a.table[e] = a.slab + static_cast<size_t>(sl) * a.stride;
        } else if (code == 3) {
            a.table[e] = a.pool + static_cast<size_t>(e) * a.stride;
        }
        if (a.log_steps > 0) {
            const size_t o = static_cast<size_t>(s % a.log_steps) * kDcMaxIds + tid;
            a.log_hit[o] = static_cast<signed char>(code);
            a.log_slot[o] = code == 3 ? -1 : slot_s[tid];
            a.log_victim[o] = victim_s[tid];
        }
    }
    if (tid == 0) {                                  // lists, copy list and counters, in step order
        int n_a = 0, n_b = 0, n_inpl = 0, nev = 0;
        for (int j = 0; j < n; ++j) {
            const int e = ids_s[j], code = code_s[j];
            if (code == 0) {
                act[34 + n_b] = e - base;
                m.copy_e[n_b] = e;
                m.copy_slot[n_b] = slot_s[j];
                n_b++;
                nev += victim_s[j] >= 0;
            } else {
                act[1 + n_a++] = e - base;
                if (code == 3) m.inplace_e[n_inpl++] = e;
            }
        }
        act[0] = n_a;
        act[33] = n_b;
        m.n_copy = n_b;
        m.n_inplace = n_inpl;
        m.hits += n_a - n_inpl;
        m.misses += n_b + n_inpl;
        m.inplace += n_inpl;
        m.evictions += nev;
        m.bytes_copied += static_cast<long long>(n_b) * a.blob_bytes;
        m.step = s + 1;
    }
}

// The admitted misses of the last policy step, host pool -> slots: 16-byte
// chunks spread over the grid, kDcCopyUnroll loads of a thread in flight.
__global__ void __launch_bounds__(kDcCopyThreads) k_dc_copy(DcArgs a) {
    const DcMeta &m = *a.meta;
    const int n = m.n_copy;
    const unsigned per = static_cast<unsigned>(a.blob_bytes / 16);
    const unsigned total = static_cast<unsigned>(n) * per;
    const unsigned stride = gridDim.x * kDcCopyThreads * kDcCopyUnroll;
    for (unsigned i0 = blockIdx.x * kDcCopyThreads * kDcCopyUnroll + threadIdx.x; i0 < total; i0 += stride) {
        uint4 v[kDcCopyUnroll];
#pragma unroll
        for (int u = 0; u < kDcCopyUnroll; ++u) {
            const unsigned i = i0 + u * kDcCopyThreads;
            if (i < total) {
                const unsigned j = i / per, off = i - j * per;
                v[u] = __ldcv(reinterpret_cast<const uint4 *>(a.pool + static_cast<size_t>(m.copy_e[j]) * a.stride) + off);
            }
        }
#pragma unroll
        for (int u = 0; u < kDcCopyUnroll; ++u) {
            const unsigned i = i0 + u * kDcCopyThreads;
            if (i < total) {
                const unsigned j = i / per, off = i - j * per;
                reinterpret_cast<uint4 *>(a.slab + static_cast<size_t>(m.copy_slot[j]) * a.stride)[off] = v[u];
            }
        }
    }
}

}  // namespace moe

// ------------------------------------------------------------------ C ABI
using namespace moe;

struct moe_devcache {
    moe_devcache_desc d;
    int device = 0;
    DcArgs a{};
    cudaEvent_t ev_policy = nullptr, ev_copied = nullptr;
    int copy_grid = 0;
    long long steps = 0;                            // stage calls so far (host count)
    bool staged = false;
    bool joined = true;                             // a stream joined the last step's copy kernel
};

int devcache_create(const moe_devcache_desc *d, moe_devcache **out) {
    moe::NvtxRange nvtx_range("devcache_create");
    REQUIRE(d && out, "desc/out are NULL");
    *out = nullptr;
    REQUIRE(d->n_experts > 0 && d->capacity > 0 && d->capacity <= d->n_experts, "need 0 < capacity <= n_experts");
    REQUIRE(d->blob_bytes > 0 && d->blob_bytes % 16 == 0 && d->blob_bytes <= (int64_t(1) << 30),
            "blob_bytes must be a positive multiple of 16 up to 1 GiB");
    REQUIRE(d->slot_stride >= d->blob_bytes && d->slot_stride % 256 == 0, "slot_stride must be >= blob_bytes, multiple of 256");
    REQUIRE(static_cast<int64_t>(kDcMaxIds) * (d->blob_bytes / 16) < (int64_t(1) << 32),
            "blob_bytes too large for one step's copies");
    REQUIRE(d->host_pool && d->hbm_slab && d->dev_table, "host_pool/hbm_slab/dev_table must not be NULL");
    REQUIRE(d->decay_period >= 0 && d->admit_min >= 0 && d->log_steps >= 0, "negative decay_period/admit_min/log_steps");
    REQUIRE(aligned16(d->hbm_slab) && aligned16(d->host_pool) && (reinterpret_cast<uintptr_t>(d->dev_table) & 7u) == 0,
            "host_pool/hbm_slab must be 16-byte aligned, dev_table 8-byte aligned");
    cudaPointerAttributes pa{};
    if (cudaPointerGetAttributes(&pa, d->host_pool) != cudaSuccess || pa.type != cudaMemoryTypeHost ||
        pa.devicePointer == nullptr) {
        cudaGetLastError();
        set_error("host_pool is not page-locked host memory mapped for the device");
        return MOE_EINVAL;
    }
    auto *c = new moe_devcache();
    c->d = *d;
    cudaGetDevice(&c->device);
    DcArgs &a = c->a;
    a.E = d->n_experts;
    a.cap = d->capacity;
    a.decay = d->decay_period;
    a.admit_min = d->admit_min;
    a.log_steps = d->log_steps;
    a.blob_bytes = d->blob_bytes;
    a.stride = d->slot_stride;
    a.pool = static_cast<const uint8_t *>(pa.devicePointer);
    a.slab = static_cast<uint8_t *>(d->hbm_slab);
    a.table = static_cast<const uint8_t **>(d->dev_table);
    a.err = device_error_word();
    const size_t E = d->n_experts, cap = d->capacity, L = d->log_steps;
    bool ok = a.err != nullptr;
    ok = ok && cudaMalloc(&a.cnt, E * 8) == cudaSuccess && cudaMalloc(&a.last, E * 8) == cudaSuccess &&
         cudaMalloc(&a.slot_of, E * 4) == cudaSuccess && cudaMalloc(&a.expert_in, cap * 4) == cudaSuccess &&
         cudaMalloc(&a.meta, sizeof(DcMeta)) == cudaSuccess;
    if (ok && L > 0)
        ok = cudaMalloc(&a.log_hit, L * kDcMaxIds) == cudaSuccess &&
             cudaMalloc(&a.log_slot, L * kDcMaxIds * 4) == cudaSuccess &&
             cudaMalloc(&a.log_victim, L * kDcMaxIds * 4) == cudaSuccess;
    ok = ok && cudaMemset(a.cnt, 0, E * 8) == cudaSuccess && cudaMemset(a.last, 0xff, E * 8) == cudaSuccess &&
         cudaMemset(a.slot_of, 0xff, E * 4) == cudaSuccess && cudaMemset(a.expert_in, 0xff, cap * 4) == cudaSuccess &&
         cudaMemset(a.meta, 0, sizeof(DcMeta)) == cudaSuccess &&
         cudaMemset(d->dev_table, 0, E * sizeof(void *)) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&c->ev_policy, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->ev_copied, cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    if (!ok) {
        const int rc = cuda_status(cudaGetLastError(), "devcache_create");
        devcache_destroy(c);
        return rc ? rc : MOE_ENOMEM;
    }
    c->copy_grid = num_sms() * 2;
    *out = c;
    return MOE_OK;
}

void devcache_destroy(moe_devcache *c) {
    if (!c) return;
    DcArgs &a = c->a;
    cudaFree(a.cnt);
    cudaFree(a.last);
    cudaFree(a.slot_of);
    cudaFree(a.expert_in);
    cudaFree(a.meta);
    cudaFree(a.log_hit);
    cudaFree(a.log_slot);
    cudaFree(a.log_victim);
    if (c->ev_policy) cudaEventDestroy(c->ev_policy);
    if (c->ev_copied) cudaEventDestroy(c->ev_copied);
    delete c;
}

int devcache_stage(moe_devcache *c, const int32_t *ids_dev, int n, int32_t id_base, int32_t *act_dev,
                   moe_stream_t compute, moe_stream_t copy) {
    moe::NvtxRange nvtx_range("devcache_stage");
    REQUIRE(c && act_dev && (n == 0 || ids_dev), "cache/act/ids are NULL");
    REQUIRE(n >= 0 && n <= kDcMaxIds, "n must be in [0, 32]");
    if (n > c->d.capacity) {
        set_error("step needs %d experts but the cache holds %d", n, c->d.capacity);
        return MOE_EBUSY;
    }
    REQUIRE(id_base >= 0 && id_base < c->d.n_experts, "id_base outside [0, n_experts)");
    cudaStream_t sc = reinterpret_cast<cudaStream_t>(compute), sk = reinterpret_cast<cudaStream_t>(copy);
    // the policy kernel rewrites the copy list the last copy kernel reads
    REQUIRE(c->joined || sk == sc, "join the previous step (devcache_join) before the next devcache_stage");
    DeviceGuard guard(c->device);
    k_dc_stage<<<1, kDcThreads, 0, sc>>>(c->a, ids_dev, n, id_base, act_dev);
    count_launches(1);
    int rc = cuda_status(cudaGetLastError(), "devcache policy launch");
    if (rc) return rc;
    rc = cuda_status(cudaEventRecord(c->ev_policy, sc), "devcache event");
    if (rc) return rc;
    if (sk != sc) {
        rc = cuda_status(cudaStreamWaitEvent(sk, c->ev_policy, 0), "devcache copy-stream wait");
        if (rc) return rc;
    }
    k_dc_copy<<<c->copy_grid, kDcCopyThreads, 0, sk>>>(c->a);
    count_launches(1);
    rc = cuda_status(cudaGetLastError(), "devcache copy launch");
    if (rc) return rc;
    rc = cuda_status(cudaEventRecord(c->ev_copied, sk), "devcache event");
    if (rc) return rc;
    c->steps++;
    c->staged = true;
    c->joined = sk == sc;
    return MOE_OK;
}

int devcache_join(moe_devcache *c, moe_stream_t s) {
    REQUIRE(c, "cache is NULL");
    if (!c->staged) return MOE_OK;
    DeviceGuard guard(c->device);
    const int rc = cuda_status(cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(s), c->ev_copied, 0), "devcache join");
    if (rc == MOE_OK) c->joined = true;
    return rc;
}

int devcache_events(moe_devcache *c, int64_t first_step, int n_steps, int8_t *hit_out, int32_t *slot_out,
                    int32_t *victim_out) {
    REQUIRE(c, "cache is NULL");
    REQUIRE(n_steps >= 0 && first_step >= 0 && first_step + n_steps <= c->steps,
            "steps [%lld, %lld) not staged yet", static_cast<long long>(first_step),
            static_cast<long long>(first_step + n_steps));
    REQUIRE(c->d.log_steps > 0 && c->steps - first_step <= c->d.log_steps,
            "step %lld is no longer in the event log of %d steps", static_cast<long long>(first_step), c->d.log_steps);
    DeviceGuard guard(c->device);
    int rc = cuda_status(cudaDeviceSynchronize(), "devcache events sync");
    if (rc) return rc;
    const size_t row = kDcMaxIds;
    for (int64_t s = first_step; s < first_step + n_steps; ++s) {
        const size_t src = static_cast<size_t>(s % c->d.log_steps) * row, dst = static_cast<size_t>(s - first_step) * row;
        if (hit_out && (rc = cuda_status(cudaMemcpy(hit_out + dst, c->a.log_hit + src, row, cudaMemcpyDeviceToHost), "log")))
            return rc;
        if (slot_out &&
            (rc = cuda_status(cudaMemcpy(slot_out + dst, c->a.log_slot + src, row * 4, cudaMemcpyDeviceToHost), "log")))
            return rc;
        if (victim_out &&
            (rc = cuda_status(cudaMemcpy(victim_out + dst, c->a.log_victim + src, row * 4, cudaMemcpyDeviceToHost), "log")))
            return rc;
    }
    return MOE_OK;
}

int devcache_stats(moe_devcache *c, moe_devcache_stats *out) {
    REQUIRE(c && out, "cache/out are NULL");
    DeviceGuard guard(c->device);
    DcMeta m;
    int rc = cuda_status(cudaMemcpy(&m, c->a.meta, sizeof(m), cudaMemcpyDeviceToHost), "devcache stats");
    if (rc) return rc;
    out->steps = m.step;
    out->hits = m.hits;
    out->misses = m.misses;
    out->evictions = m.evictions;
    out->in_place = m.inplace;
    out->bytes_copied = m.bytes_copied;
    out->bad_steps = m.bad_steps;
    return MOE_OK;
}

int devcache_snapshot(moe_devcache *c, int64_t *counts_out, int32_t *slot_of_out) {
    REQUIRE(c, "cache is NULL");
    DeviceGuard guard(c->device);
    int rc = 0;
    const size_t E = c->d.n_experts;
    if (counts_out && (rc = cuda_status(cudaMemcpy(counts_out, c->a.cnt, E * 8, cudaMemcpyDeviceToHost), "snapshot")))
        return rc;
    if (slot_of_out && (rc = cuda_status(cudaMemcpy(slot_of_out, c->a.slot_of, E * 4, cudaMemcpyDeviceToHost), "snapshot")))
        return rc;
    return MOE_OK;
}
