// Expert cache: frequency-driven residency of expert blobs in an HBM slab,
// paged in from a page-locked host pool.
//
// Strata article, section 2 item 2: the most-called experts live in VRAM,
// all experts in RAM; an expert the router picks is computed at once when
// resident, otherwise it is first moved in.  Section 3: part of the RAM is
// page-locked for the GPU.  Strata code review, section 3: a stage buffer
// whose page-locking became optional.  Janas-LLM page: experts used again
// stay in the cache.
//
// Host bookkeeping is O(log capacity) per access (an ordered set keyed by
// (counter, last use, id) over the resident experts); each miss is one
// cudaMemcpyAsync on the cache's own stream, after which one small kernel
// patches the device table of blob pointers.
#include <algorithm>
#include <chrono>
#include <cstring>
#include <new>
#include <set>
#include <thread>
#include <tuple>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void k_table_patch(const void **table, TablePatch p) {
    const int i = threadIdx.x;
    if (i < p.n) table[p.ids[i]] = p.ptrs[i];
}

int launch_table_patch(const void **table, const TablePatch &p, cudaStream_t s) {
    if (p.n <= 0) return MOE_OK;
    k_table_patch<<<1, 64, 0, s>>>(table, p); count_launches(1);
    return cuda_status(cudaGetLastError(), "table patch launch");
}

}  // namespace moe

using namespace moe;

struct moe_expcache {
    moe_expcache_desc d;
    int device = 0;
    cudaStream_t copy = nullptr;
    cudaEvent_t ev_compute = nullptr;     // compute stream position at the last stage call
    cudaEvent_t ev_done = nullptr;        // all copies + table patch issued so far
    cudaEvent_t ev_stage[2] = {nullptr, nullptr};   // staging halves free again
    cudaEvent_t ev_t0 = nullptr, ev_t1 = nullptr;     // timed: start / end of the last step's copies
    bool timed = false;                               // ev_t0/ev_t1 have been recorded
    // copy-time histogram: start/end events of the steps whose copies are not
    // yet counted (a ring, oldest at ring_tail; the copy stream completes
    // them in order)
    static constexpr int kRing = 32;
    cudaEvent_t ring0[kRing] = {}, ring1[kRing] = {};
    int ring_tail = 0, ring_pending = 0;
    int64_t hist[MOE_COPY_HIST_BINS] = {};
    int stage_next = 0;
    std::vector<int32_t> slot_of, expert_in;
    std::vector<int64_t> cnt, last;
    std::set<std::tuple<int64_t, int64_t, int32_t>> order;   // resident experts by (cnt, last, id)
    std::set<int32_t> free_slots;
    int64_t step = 0;
    std::vector<int32_t> step_ids;                     // ids of the last stage call (protected from prefetch)
    std::vector<uint8_t> inflight;                     // admitted by a prefetch not yet covered by a join
    moe_expcache_stats st{};
    int inject_fail = 0;
};

static void destroy_events(moe_expcache *c) {
    if (c->ev_compute) cudaEventDestroy(c->ev_compute);
    if (c->ev_done) cudaEventDestroy(c->ev_done);
    for (auto &e : c->ev_stage)
        if (e) cudaEventDestroy(e);
    if (c->ev_t0) cudaEventDestroy(c->ev_t0);
    if (c->ev_t1) cudaEventDestroy(c->ev_t1);
    for (int i = 0; i < moe_expcache::kRing; ++i) {
        if (c->ring0[i]) cudaEventDestroy(c->ring0[i]);
        if (c->ring1[i]) cudaEventDestroy(c->ring1[i]);
    }
    if (c->copy) cudaStreamDestroy(c->copy);
}

// One copy per admitted expert on the cache's stream, after the compute
// stream's work queued so far (it may still read the victims' slots), then
// one table patch; copies that cannot be issued leave their experts out of
// the cache again.
struct PendingCopy {
    int32_t id, slot;
    const uint8_t *src;                                // NULL: the pool entry of id
};

// Counts the timed steps whose copies have completed into the histogram
// (bin i: [2^i, 2^(i+1)) microseconds, the first and last bins open-ended).
// wait_oldest: block on the oldest pending step first (the ring is full).
static int harvest_copy_times(moe_expcache *c, bool wait_oldest) {
    while (c->ring_pending > 0) {
        const int i = c->ring_tail;
        if (wait_oldest) {
            int rc = cuda_status(cudaEventSynchronize(c->ring1[i]), "copy timing wait");
            if (rc) return rc;
            wait_oldest = false;
        } else {
            const cudaError_t q = cudaEventQuery(c->ring1[i]);
            if (q == cudaErrorNotReady) break;
            if (q != cudaSuccess) return cuda_status(q, "copy timing query");
        }
        float ms = 0.f;
        int rc = cuda_status(cudaEventElapsedTime(&ms, c->ring0[i], c->ring1[i]), "copy timing");
        if (rc) return rc;
        int bin = 0;
        for (double us = ms * 1e3; us >= 2.0 && bin < MOE_COPY_HIST_BINS - 1; us /= 2.0) ++bin;
        c->hist[bin]++;
        c->ring_tail = (i + 1) % moe_expcache::kRing;
        c->ring_pending--;
    }
    return MOE_OK;
}

static int issue_copies(moe_expcache *c, const PendingCopy *copies, int nc, TablePatch &patch, moe_stream_t compute) {
    if (nc == 0 && patch.n == 0) return MOE_OK;
    int rc = MOE_OK;
    if (nc > 0) {
        rc = cuda_status(cudaEventRecord(c->ev_compute, reinterpret_cast<cudaStream_t>(compute)), "event record");
        if (!rc) rc = cuda_status(cudaStreamWaitEvent(c->copy, c->ev_compute, 0), "stream wait");
        if (!rc) rc = cuda_status(cudaEventRecord(c->ev_t0, c->copy), "event record");
        if (!rc) rc = harvest_copy_times(c, c->ring_pending == moe_expcache::kRing);
        if (!rc) {
            const int slot = (c->ring_tail + c->ring_pending) % moe_expcache::kRing;
            rc = cuda_status(cudaEventRecord(c->ring0[slot], c->copy), "event record");
        }
    }
    const size_t B = static_cast<size_t>(c->d.blob_bytes), S = static_cast<size_t>(c->d.slot_stride);
    auto *slab = static_cast<uint8_t *>(c->d.hbm_slab);
    auto *pool = static_cast<const uint8_t *>(c->d.host_pool);
    int issued = 0;
    for (int i = 0; i < nc && !rc; ++i) {
        uint8_t *dst = slab + static_cast<size_t>(copies[i].slot) * S;
        const uint8_t *src = copies[i].src ? copies[i].src : pool + static_cast<size_t>(copies[i].id) * S;
        if (c->d.use_staging) {
            const int h = c->stage_next;
            c->stage_next ^= 1;
            rc = cuda_status(cudaEventSynchronize(c->ev_stage[h]), "stage wait");
            uint8_t *buf = static_cast<uint8_t *>(c->d.stage_buffer) + static_cast<size_t>(h) * S;
            if (!rc) std::memcpy(buf, src, B);
            if (!rc) rc = cuda_status(cudaMemcpyAsync(dst, buf, B, cudaMemcpyHostToDevice, c->copy), "stage copy");
            if (!rc) rc = cuda_status(cudaEventRecord(c->ev_stage[h], c->copy), "event record");
        } else {
            rc = cuda_status(cudaMemcpyAsync(dst, src, B, cudaMemcpyHostToDevice, c->copy), "expert copy");
        }
        if (rc) {
            rc = MOE_EIO;
        } else {
            patch.ids[patch.n] = copies[i].id;
            patch.ptrs[patch.n] = dst;
            patch.n++;
            issued++;
            c->st.bytes_staged += static_cast<int64_t>(B);
        }
    }
    // copies that could not be issued leave their experts out of the cache
    for (int i = issued; i < nc; ++i) {
        const int e = copies[i].id;
        c->order.erase(std::make_tuple(c->cnt[e], c->last[e], e));
        c->expert_in[copies[i].slot] = -1;
        c->slot_of[e] = -1;
        c->free_slots.insert(copies[i].slot);
    }
    int rc2 = launch_table_patch(reinterpret_cast<const void **>(c->d.dev_table), patch, c->copy);
    if (!rc2) rc2 = cuda_status(cudaEventRecord(c->ev_done, c->copy), "event record");
    if (!rc2 && nc > 0) rc2 = cuda_status(cudaEventRecord(c->ev_t1, c->copy), "event record");
    if (!rc2 && nc > 0) {
        const int slot = (c->ring_tail + c->ring_pending) % moe_expcache::kRing;
        rc2 = cuda_status(cudaEventRecord(c->ring1[slot], c->copy), "event record");
        if (!rc2) c->ring_pending++;
    }
    if (!rc2 && nc > 0) c->timed = true;
    return rc ? rc : rc2;
}

extern "C" {

int expcache_create(const moe_expcache_desc *d, moe_expcache **out) {
    REQUIRE(d && out, "desc/out are NULL");
    *out = nullptr;
    REQUIRE(d->n_experts >= 1, "n_experts must be >= 1");
    REQUIRE(d->capacity >= 1, "capacity must be >= 1");
    REQUIRE(d->blob_bytes > 0 && d->blob_bytes % 16 == 0, "blob_bytes must be a positive multiple of 16");
    REQUIRE(d->slot_stride >= d->blob_bytes && d->slot_stride % 256 == 0,
            "slot_stride must be >= blob_bytes and a multiple of 256");
    REQUIRE(d->host_pool && d->hbm_slab && d->dev_table, "host_pool/hbm_slab/dev_table must not be NULL");
    REQUIRE(aligned16(d->host_pool) && aligned16(d->hbm_slab) && aligned16(d->dev_table),
            "host_pool/hbm_slab/dev_table must be 16-byte aligned");
    REQUIRE(d->decay_period >= 0, "decay_period must be >= 0");
    REQUIRE(!d->use_staging || d->stage_buffer, "use_staging needs a stage_buffer");
    moe_expcache *c = new (std::nothrow) moe_expcache();
    if (!c) {
        set_error("out of host memory");
        return MOE_ENOMEM;
    }
    c->d = *d;
    cudaGetDevice(&c->device);
    int rc = cuda_status(cudaStreamCreateWithFlags(&c->copy, cudaStreamNonBlocking), "copy stream");
    if (!rc) rc = cuda_status(cudaEventCreateWithFlags(&c->ev_compute, cudaEventDisableTiming), "event");
    if (!rc) rc = cuda_status(cudaEventCreateWithFlags(&c->ev_done, cudaEventDisableTiming), "event");
    for (int i = 0; i < 2 && !rc; ++i)
        rc = cuda_status(cudaEventCreateWithFlags(&c->ev_stage[i], cudaEventDisableTiming), "event");
    if (!rc) rc = cuda_status(cudaEventCreate(&c->ev_t0), "event");
    if (!rc) rc = cuda_status(cudaEventCreate(&c->ev_t1), "event");
    for (int i = 0; i < moe_expcache::kRing && !rc; ++i) {
        rc = cuda_status(cudaEventCreate(&c->ring0[i]), "event");
        if (!rc) rc = cuda_status(cudaEventCreate(&c->ring1[i]), "event");
    }
    if (!rc)
        rc = cuda_status(cudaMemsetAsync(d->dev_table, 0, sizeof(void *) * static_cast<size_t>(d->n_experts), c->copy),
                         "table clear");
    if (!rc) rc = cuda_status(cudaEventRecord(c->ev_done, c->copy), "event record");
    for (int i = 0; i < 2 && !rc; ++i) rc = cuda_status(cudaEventRecord(c->ev_stage[i], c->copy), "event record");
    if (rc) {
        destroy_events(c);
        delete c;
        return rc;
    }
    try {
        c->slot_of.assign(d->n_experts, -1);
        c->inflight.assign(d->n_experts, 0);
        c->expert_in.assign(d->capacity, -1);
        c->cnt.assign(d->n_experts, 0);
        c->last.assign(d->n_experts, -1);
        for (int s = 0; s < d->capacity; ++s) c->free_slots.insert(s);
    } catch (...) {
        destroy_events(c);
        delete c;
        set_error("out of host memory");
        return MOE_ENOMEM;
    }
    *out = c;
    return MOE_OK;
}

void expcache_destroy(moe_expcache *c) {
    if (!c) return;
    DeviceGuard g(c->device);
    cudaStreamSynchronize(c->copy);
    destroy_events(c);
    delete c;
}

int expcache_lookup(moe_expcache *c, const int32_t *ids_host, int n, int32_t *slots_out, int *n_miss) {
    REQUIRE(c && (n == 0 || ids_host), "cache/ids are NULL");
    REQUIRE(n >= 0, "n must be >= 0");
    int miss = 0;
    for (int i = 0; i < n; ++i) {
        const int e = ids_host[i];
        REQUIRE(e >= 0 && e < c->d.n_experts, "expert id %d out of range", e);
        const int s = c->slot_of[e];
        if (slots_out) slots_out[i] = s;
        miss += s < 0;
    }
    if (n_miss) *n_miss = miss;
    return MOE_OK;
}

static int stage_impl(moe_expcache *c, const int32_t *ids_host, int n, const void *const *src_host,
                      moe_stream_t compute, int32_t *hit_out, int32_t *slot_out, int32_t *victim_out) {
    REQUIRE(c && (n == 0 || ids_host), "cache/ids are NULL");
    REQUIRE(n >= 0 && n <= 32, "n must be in [0, 32]");
    if (n > c->d.capacity) {
        set_error("step needs %d experts but the cache holds %d", n, c->d.capacity);
        return MOE_EBUSY;
    }
    for (int i = 0; i < n; ++i) {
        REQUIRE(ids_host[i] >= 0 && ids_host[i] < c->d.n_experts, "expert id %d out of range", ids_host[i]);
        for (int j = 0; j < i; ++j) REQUIRE(ids_host[j] != ids_host[i], "expert id %d repeated in a step", ids_host[i]);
    }
    int n_miss = 0;
    for (int i = 0; i < n; ++i) n_miss += c->slot_of[ids_host[i]] < 0;
    if (src_host) {
        REQUIRE(!c->d.use_staging, "expcache_stage_from does not take a staging cache");
        for (int i = 0; i < n; ++i)
            REQUIRE(c->slot_of[ids_host[i]] >= 0 || src_host[i], "no source for missed expert %d", ids_host[i]);
    }
    if (n_miss > 0 && c->inject_fail > 0) {   // test hook: fail before any state changes
        c->inject_fail--;
        set_error("injected staging-copy failure");
        return MOE_EIO;
    }
    DeviceGuard guard(c->device);
    const int64_t s = c->step;
    // halving decay at the start of every decay_period-th step
    if (c->d.decay_period > 0 && s > 0 && s % c->d.decay_period == 0) {
        for (auto &v : c->cnt) v /= 2;
        c->order.clear();
        for (int e = 0; e < c->d.n_experts; ++e)
            if (c->slot_of[e] >= 0) c->order.emplace(c->cnt[e], c->last[e], e);
    }
    TablePatch patch{};
    PendingCopy copies[32];
    int nc = 0;
    for (int i = 0; i < n; ++i) {
        const int e = ids_host[i];
        const bool resident = c->slot_of[e] >= 0;
        if (resident) c->order.erase(std::make_tuple(c->cnt[e], c->last[e], e));
        c->cnt[e] += 1;
        c->last[e] = s;
        int victim = -1;
        if (resident) {
            c->order.emplace(c->cnt[e], c->last[e], e);
            c->st.hits++;
        } else {
            int slot;
            if (!c->free_slots.empty()) {
                slot = *c->free_slots.begin();
                c->free_slots.erase(c->free_slots.begin());
            } else {
                auto it = c->order.begin();
                for (; it != c->order.end(); ++it) {
                    const int v = std::get<2>(*it);
                    bool in_step = false;
                    for (int j = 0; j < n; ++j) in_step |= ids_host[j] == v;
                    if (!in_step) break;
                }
                victim = std::get<2>(*it);   // exists: capacity >= n and e is not resident
                c->order.erase(it);
                slot = c->slot_of[victim];
                c->slot_of[victim] = -1;
                c->inflight[victim] = 0;
                c->st.evictions++;
                patch.ids[patch.n] = victim;
                patch.ptrs[patch.n] = nullptr;
                patch.n++;
            }
            c->slot_of[e] = slot;
            c->expert_in[slot] = e;
            c->order.emplace(c->cnt[e], c->last[e], e);
            copies[nc++] = PendingCopy{e, slot, src_host ? static_cast<const uint8_t *>(src_host[i]) : nullptr};
            c->st.misses++;
        }
        if (hit_out) hit_out[i] = resident ? (c->inflight[e] ? 2 : 1) : 0;
        if (slot_out) slot_out[i] = c->slot_of[e];
        if (victim_out) victim_out[i] = victim;
    }
    c->step++;
    c->st.steps++;
    c->step_ids.assign(ids_host, ids_host + n);
    return issue_copies(c, copies, nc, patch, compute);
}

int expcache_stage(moe_expcache *c, const int32_t *ids_host, int n, moe_stream_t compute, int32_t *hit_out,
                   int32_t *slot_out, int32_t *victim_out) {
    moe::NvtxRange nvtx_range("expcache_stage");
    return stage_impl(c, ids_host, n, nullptr, compute, hit_out, slot_out, victim_out);
}

int expcache_stage_from(moe_expcache *c, const int32_t *ids_host, int n, const void *const *src_host,
                        moe_stream_t compute, int32_t *hit_out, int32_t *slot_out, int32_t *victim_out) {
    moe::NvtxRange nvtx_range("expcache_stage_from");
    REQUIRE(src_host || n == 0, "src_host is NULL");
    return stage_impl(c, ids_host, n, src_host, compute, hit_out, slot_out, victim_out);
}

int expcache_prefetch(moe_expcache *c, const int32_t *ids_host, int n, moe_stream_t compute, int32_t *slot_out,
                      int32_t *victim_out, int *n_admitted) {
    moe::NvtxRange nvtx_range("expcache_prefetch");
    REQUIRE(c && (n == 0 || ids_host), "cache/ids are NULL");
    REQUIRE(n >= 0 && n <= 32, "n must be in [0, 32]");
    for (int i = 0; i < n; ++i)
        REQUIRE(ids_host[i] >= -1 && ids_host[i] < c->d.n_experts, "expert id %d out of range", ids_host[i]);
    DeviceGuard guard(c->device);
    // protected: the last step's ids and every id on this list
    auto protected_id = [&](int v) {
        for (int32_t q : c->step_ids)
            if (q == v) return true;
        for (int i = 0; i < n; ++i)
            if (ids_host[i] == v) return true;
        return false;
    };
    TablePatch patch{};
    PendingCopy copies[32];
    int nc = 0;
    for (int i = 0; i < n; ++i) {
        const int e = ids_host[i];
        if (slot_out) slot_out[i] = -1;
        if (victim_out) victim_out[i] = -1;
        if (e < 0 || c->slot_of[e] >= 0) continue;
        int slot = -1, victim = -1;
        if (!c->free_slots.empty()) {
            slot = *c->free_slots.begin();
            c->free_slots.erase(c->free_slots.begin());
        } else {
            auto it = c->order.begin();
            while (it != c->order.end() && protected_id(std::get<2>(*it))) ++it;
            if (it == c->order.end()) continue;        // everything resident is protected
            victim = std::get<2>(*it);
            c->order.erase(it);
            slot = c->slot_of[victim];
            c->slot_of[victim] = -1;
            c->inflight[victim] = 0;
            c->st.evictions++;
            patch.ids[patch.n] = victim;
            patch.ptrs[patch.n] = nullptr;
            patch.n++;
        }
        // a prefetch is not a use: the counter and last use stay as they are
        c->slot_of[e] = slot;
        c->expert_in[slot] = e;
        c->order.emplace(c->cnt[e], c->last[e], e);
        c->inflight[e] = 1;
        copies[nc++] = PendingCopy{e, slot, nullptr};
        if (slot_out) slot_out[i] = slot;
        if (victim_out) victim_out[i] = victim;
    }
    c->st.prefetched += nc;
    if (n_admitted) *n_admitted = nc;
    return issue_copies(c, copies, nc, patch, compute);
}

int expcache_copy_times(moe_expcache *c, const void *ref_event, float *start_ms, float *end_ms) {
    REQUIRE(c && ref_event && start_ms && end_ms, "cache/ref_event/start_ms/end_ms are NULL");
    REQUIRE(c->timed, "no step has staged copies yet");
    DeviceGuard guard(c->device);
    cudaEvent_t ref = static_cast<cudaEvent_t>(const_cast<void *>(ref_event));
    int rc = cuda_status(cudaEventElapsedTime(start_ms, ref, c->ev_t0), "elapsed time");
    if (!rc) rc = cuda_status(cudaEventElapsedTime(end_ms, ref, c->ev_t1), "elapsed time");
    return rc;
}

int expcache_copy_histogram(moe_expcache *c, int64_t *bins_out, int64_t *steps_out) {
    REQUIRE(c && bins_out, "cache/bins_out are NULL");
    DeviceGuard guard(c->device);
    int rc = harvest_copy_times(c, false);
    if (rc) return rc;
    int64_t n = 0;
    for (int b = 0; b < MOE_COPY_HIST_BINS; ++b) {
        bins_out[b] = c->hist[b];
        n += c->hist[b];
    }
    if (steps_out) *steps_out = n;
    return MOE_OK;
}

int expcache_join(moe_expcache *c, moe_stream_t s) {
    REQUIRE(c != nullptr, "cache is NULL");
    const int rc = cuda_status(cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(s), c->ev_done, 0), "stream wait");
    if (!rc) std::fill(c->inflight.begin(), c->inflight.end(), 0);   // every copy so far is ordered before `s`
    return rc;
}

int expcache_wait(moe_expcache *c, int64_t timeout_us) {
    moe::NvtxRange nvtx_range("expcache_wait");
    REQUIRE(c != nullptr, "cache is NULL");
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t e = cudaEventQuery(c->ev_done);
        if (e == cudaSuccess) {
            std::fill(c->inflight.begin(), c->inflight.end(), 0);   // every copy so far has landed
            return MOE_OK;
        }
        if (e != cudaErrorNotReady) return cuda_status(e, "event query");
        const auto us =
            std::chrono::duration_cast<std::chrono::microseconds>(std::chrono::steady_clock::now() - t0).count();
        if (us >= timeout_us) {
            set_error("staged copies not done after %lld us", static_cast<long long>(timeout_us));
            return MOE_ETIMEDOUT;
        }
        std::this_thread::sleep_for(std::chrono::microseconds(20));
    }
}

int expcache_evict(moe_expcache *c, const int32_t *ids_host, int n) {
    REQUIRE(c && (n == 0 || ids_host), "cache/ids are NULL");
    REQUIRE(n >= 0 && n <= 64, "n must be in [0, 64]");
    TablePatch patch{};
    for (int i = 0; i < n; ++i) {
        const int e = ids_host[i];
        REQUIRE(e >= 0 && e < c->d.n_experts, "expert id %d out of range", e);
        const int s = c->slot_of[e];
        if (s < 0) continue;
        c->order.erase(std::make_tuple(c->cnt[e], c->last[e], e));
        c->slot_of[e] = -1;
        c->inflight[e] = 0;
        c->expert_in[s] = -1;
        c->free_slots.insert(s);
        c->st.evictions++;
        patch.ids[patch.n] = e;
        patch.ptrs[patch.n] = nullptr;
        patch.n++;
    }
    if (patch.n == 0) return MOE_OK;
    DeviceGuard guard(c->device);
    int rc = launch_table_patch(reinterpret_cast<const void **>(c->d.dev_table), patch, c->copy);
    if (!rc) rc = cuda_status(cudaEventRecord(c->ev_done, c->copy), "event record");
    return rc;
}

const void *const *expcache_device_table(moe_expcache *c) {
    return c ? static_cast<const void *const *>(c->d.dev_table) : nullptr;
}

int expcache_stats(moe_expcache *c, moe_expcache_stats *out) {
    REQUIRE(c && out, "cache/out are NULL");
    *out = c->st;
    out->resident = c->d.capacity - static_cast<int32_t>(c->free_slots.size());
    return MOE_OK;
}

int expcache_snapshot(moe_expcache *c, int64_t *counts_out, int32_t *slot_of_out) {
    REQUIRE(c != nullptr, "cache is NULL");
    if (counts_out) std::memcpy(counts_out, c->cnt.data(), sizeof(int64_t) * c->cnt.size());
    if (slot_of_out) std::memcpy(slot_of_out, c->slot_of.data(), sizeof(int32_t) * c->slot_of.size());
    return MOE_OK;
}

int expcache_inject_copy_failures(moe_expcache *c, int n) {
    REQUIRE(c && n >= 0, "bad arguments");
    c->inject_fail = n;
    return MOE_OK;
}

}  // extern "C"
