// The third tier: expert blobs in a file (an NVMe drive), read on demand into
// a page-locked RAM tier from which the expert cache copies them to HBM.
//
// Strata article, section 2 item 2 and its summary of the three tiers: hot
// experts in VRAM, the rest in RAM, the remainder on SSD; Janas-LLM page:
// experts read from NVMe per token with O_DIRECT into a RAM cache whose size
// is capped.  Host code only: a fixed pool of I/O threads issues pread()s
// (O_DIRECT when asked, so reads bypass the kernel's page cache and land
// straight in the page-locked slots), and the RAM tier keeps the least
// recently fetched slot as the next victim.
#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <algorithm>
#include <atomic>
#include <cerrno>
#include <chrono>
#include <condition_variable>
#include <cstring>
#include <exception>
#include <list>
#include <mutex>
#include <thread>
#include <unordered_map>
#include <vector>

#include "common.cuh"
#include "kernels.h"

using namespace moe;

namespace {

constexpr int kMaxFetch = 32;
constexpr size_t kDirectAlign = 4096;

struct ReadJob {
    int fd;
    uint8_t *dst;
    off_t off;
    size_t bytes;
    int err;                                        // errno of a failed read, 0 on success
};

// A fixed set of threads that run one batch of reads at a time.
class IoPool {
public:
    explicit IoPool(int n) {
        for (int i = 0; i < n; ++i) th_.emplace_back([this] { loop(); });
    }
    ~IoPool() {
        {
            std::lock_guard<std::mutex> g(m_);
            stop_ = true;
        }
        cv_.notify_all();
        for (auto &t : th_) t.join();
    }
    // Runs every job; returns when all have finished.
    void run(std::vector<ReadJob> &jobs) {
        if (jobs.empty()) return;
        {
            std::lock_guard<std::mutex> g(m_);
            jobs_ = &jobs;
            next_ = 0;
            left_ = jobs.size();
        }
        cv_.notify_all();
        std::unique_lock<std::mutex> g(m_);
        done_.wait(g, [this] { return left_ == 0; });
        jobs_ = nullptr;
    }

private:
    void loop() {
        for (;;) {
            ReadJob *job = nullptr;
            {
                std::unique_lock<std::mutex> g(m_);
                cv_.wait(g, [this] { return stop_ || (jobs_ && next_ < jobs_->size()); });
                if (stop_) return;
                job = &(*jobs_)[next_++];
            }
            size_t got = 0;
            job->err = 0;
            while (got < job->bytes) {
                const ssize_t r = pread(job->fd, job->dst + got, job->bytes - got, job->off + static_cast<off_t>(got));
                if (r < 0 && errno == EINTR) continue;
                if (r <= 0) {
                    job->err = r < 0 ? errno : EIO;     // a short file reads as EIO
                    break;
                }
                got += static_cast<size_t>(r);
            }
            std::lock_guard<std::mutex> g(m_);
            if (--left_ == 0) done_.notify_all();
        }
    }
    std::vector<std::thread> th_;
    std::mutex m_;
    std::condition_variable cv_, done_;
    std::vector<ReadJob> *jobs_ = nullptr;
    size_t next_ = 0, left_ = 0;
    bool stop_ = false;
};

}  // namespace

struct moe_expstore {
    moe_expstore_desc d{};
    int fd = -1;
    size_t read_bytes = 0;                          // bytes read per blob (rounded up for O_DIRECT)
    std::vector<int32_t> slot_of;                   // expert -> RAM slot or -1
    std::vector<int32_t> expert_in;                 // RAM slot -> expert or -1
    std::list<int32_t> lru;                         // RAM slots, least recently fetched first
    std::vector<std::list<int32_t>::iterator> pos;  // slot -> its place in lru
    IoPool *io = nullptr;
    moe_expstore_stats st{};
};

int expstore_create(const moe_expstore_desc *d, moe_expstore **out) {
    moe::NvtxRange nvtx_range("expstore_create");
    REQUIRE(d && out && d->path, "desc/out/path are NULL");
    *out = nullptr;
    REQUIRE(d->n_experts > 0 && d->ram_slots > 0, "n_experts and ram_slots must be positive");
    REQUIRE(d->blob_bytes > 0 && d->slot_stride >= d->blob_bytes && d->slot_stride % 256 == 0,
            "need 0 < blob_bytes <= slot_stride, slot_stride a multiple of 256");
    REQUIRE(d->ram_buffer, "ram_buffer is NULL");
    REQUIRE(d->io_threads >= 1 && d->io_threads <= 64, "io_threads must be in [1, 64]");
    size_t rb = static_cast<size_t>(d->blob_bytes);
    if (d->use_direct) {
        REQUIRE(d->slot_stride % kDirectAlign == 0 && reinterpret_cast<uintptr_t>(d->ram_buffer) % kDirectAlign == 0,
                "O_DIRECT needs slot_stride and ram_buffer aligned to 4096 bytes");
        rb = (rb + kDirectAlign - 1) / kDirectAlign * kDirectAlign;   // whole blocks; the slot holds them
    }
    const int fd = open(d->path, O_RDONLY | (d->use_direct ? O_DIRECT : 0));
    if (fd < 0) {
        set_error("cannot open %s%s: %s", d->path, d->use_direct ? " with O_DIRECT" : "", strerror(errno));
        return MOE_EIO;
    }
    struct stat sb{};
    const off_t need = static_cast<off_t>(d->n_experts - 1) * d->slot_stride + static_cast<off_t>(rb);
    if (fstat(fd, &sb) != 0 || sb.st_size < need) {
        close(fd);
        set_error("%s holds %lld bytes; %d experts need %lld", d->path, static_cast<long long>(sb.st_size),
                  d->n_experts, static_cast<long long>(need));
        return MOE_EINVAL;
    }
    moe_expstore *s = nullptr;
    try {
        s = new moe_expstore();
        s->d = *d;
        s->fd = fd;
        s->read_bytes = rb;
        s->slot_of.assign(d->n_experts, -1);
        s->expert_in.assign(d->ram_slots, -1);
        s->pos.resize(d->ram_slots);
        for (int i = 0; i < d->ram_slots; ++i) s->pos[i] = s->lru.insert(s->lru.end(), i);
        s->io = new IoPool(d->io_threads);
    } catch (const std::exception &ex) {          // out of memory, or threads that could not start
        if (s) {
            s->fd = -1;
            expstore_destroy(s);
        }
        close(fd);
        set_error("expert store: %s", ex.what());
        return MOE_ENOMEM;
    }
    *out = s;
    return MOE_OK;
}

void expstore_destroy(moe_expstore *s) {
    if (!s) return;
    delete s->io;
    if (s->fd >= 0) close(s->fd);
    delete s;
}

int expstore_fetch(moe_expstore *s, const int32_t *ids, int n, void **ram_ptrs_out, int8_t *hit_out) {
    moe::NvtxRange nvtx_range("expstore_fetch");
    REQUIRE(s && (n == 0 || ids), "store/ids are NULL");
    REQUIRE(n >= 0 && n <= kMaxFetch, "n must be in [0, 32]");
    if (n > s->d.ram_slots) {
        set_error("fetch needs %d experts but the RAM tier holds %d", n, s->d.ram_slots);
        return MOE_EBUSY;
    }
    for (int i = 0; i < n; ++i) {
        REQUIRE(ids[i] >= 0 && ids[i] < s->d.n_experts, "expert id %d out of range", ids[i]);
        for (int j = 0; j < i; ++j) REQUIRE(ids[j] != ids[i], "expert id %d repeated in a fetch", ids[i]);
    }
    const size_t S = static_cast<size_t>(s->d.slot_stride);
    auto *ram = static_cast<uint8_t *>(s->d.ram_buffer);
    std::vector<ReadJob> jobs;
    std::vector<int> job_slot, job_id;
    // every id of the call is touched first, so none can be a victim
    bool resident[kMaxFetch];
    for (int i = 0; i < n; ++i) {
        const int sl = s->slot_of[ids[i]];
        resident[i] = sl >= 0;
        if (resident[i]) s->lru.splice(s->lru.end(), s->lru, s->pos[sl]);
    }
    for (int i = 0; i < n; ++i) {
        if (resident[i]) continue;
        const int sl = s->lru.front();                  // least recently fetched, not one of this call's
        const int old = s->expert_in[sl];
        if (old >= 0) {
            s->slot_of[old] = -1;
            s->st.evictions++;
        }
        s->expert_in[sl] = ids[i];
        s->slot_of[ids[i]] = sl;
        s->lru.splice(s->lru.end(), s->lru, s->pos[sl]);
        jobs.push_back(ReadJob{s->fd, ram + static_cast<size_t>(sl) * S, static_cast<off_t>(ids[i]) * s->d.slot_stride,
                               s->read_bytes, 0});
        job_slot.push_back(sl);
        job_id.push_back(ids[i]);
    }
    const auto t0 = std::chrono::steady_clock::now();
    s->io->run(jobs);
    s->st.read_seconds += std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
    int bad = 0;
    for (size_t q = 0; q < jobs.size(); ++q) {
        if (jobs[q].err == 0) {
            s->st.reads++;
            s->st.bytes_read += static_cast<int64_t>(jobs[q].bytes);
            continue;
        }
        if (!bad) set_error("reading expert %d: %s", job_id[q], strerror(jobs[q].err));
        bad = 1;
        s->slot_of[job_id[q]] = -1;                     // a failed read leaves the expert out of RAM
        s->expert_in[job_slot[q]] = -1;
        s->lru.splice(s->lru.begin(), s->lru, s->pos[job_slot[q]]);
    }
    s->st.fetches++;
    for (int i = 0; i < n; ++i) {
        if (resident[i]) s->st.hits++;
        if (hit_out) hit_out[i] = resident[i] ? 1 : 0;
        const int sl = s->slot_of[ids[i]];
        if (ram_ptrs_out) ram_ptrs_out[i] = sl >= 0 ? ram + static_cast<size_t>(sl) * S : nullptr;
    }
    return bad ? MOE_EIO : MOE_OK;
}

int expstore_stats(moe_expstore *s, moe_expstore_stats *out) {
    REQUIRE(s && out, "store/out are NULL");
    *out = s->st;
    return MOE_OK;
}

int expstore_snapshot(moe_expstore *s, int32_t *slot_of_out) {
    REQUIRE(s && slot_of_out, "store/out are NULL");
    std::copy(s->slot_of.begin(), s->slot_of.end(), slot_of_out);
    return MOE_OK;
}
