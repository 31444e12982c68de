// Host-memory tier: tables too large for HBM stay in host DRAM, and each
// batch brings over PCIe only the rows its n-grams activate.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram" (system efficiency),
// and the Synced repost, section "System efficiency: decoupling compute and
// storage": the retrieval indices depend only on the token ids, so they are
// known before the layer runs; the activated rows can be fetched from host
// memory while the preceding layers compute, and with Zipf-distributed
// n-grams a batch touches far fewer distinct rows than it makes lookups.
// (QbitAI repost: a 100B-parameter table in host memory costs under 3 % of
// throughput.)
//
// One batch takes three steps:
//   engram_host_dedupe   (GPU, stream s)  the n_tok x J lookups go into a
//                        device hash set keyed by global row; each distinct
//                        row gets a slot, every lookup its row's slot; the
//                        distinct rows and their count are copied to pinned
//                        host memory.
//   engram_host_fetch    (host threads + side stream)  worker threads copy
//                        the distinct rows from the host tables into a pinned
//                        staging buffer in chunks; each packed chunk goes to
//                        the device with one cudaMemcpyAsync on the side
//                        stream while the next chunks are packed.
//   engram_gather_staged (GPU, stream s)  the gather kernel reads row
//                        slot[t][j] of the staged rows into e_cat[t][j].
// Between dedupe and gather_staged the caller's stream is free for other
// work (the preceding layers), which the fetch overlaps.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <condition_variable>
#include <cstring>
#include <mutex>
#include <new>
#include <thread>
#include <vector>

#if defined(__SSE2__)
#include <emmintrin.h>
#endif

#include "ctx.cuh"

namespace engram {
namespace {

constexpr uint64_t kEmpty = 0;               // hash-set key of an empty slot (keys are row + 1)
constexpr int64_t kPackChunkRows = 4096;     // rows per packing chunk (1 MB at 256-byte rows)
constexpr size_t kMinCopyBytes = 4u << 20;   // smallest row copy but the last: PCIe copies of a few MB
                                             // run faster than 1 MB or 100 MB ones
constexpr double kHostWaitSeconds = 20.0;    // bound on every host-side wait

// Murmur3's 64-bit finaliser (Appleby), to spread row numbers over the set.
__device__ __forceinline__ uint64_t mix64(uint64_t k) {
    k ^= k >> 33;
    k *= 0xff51afd7ed558ccdull;
    k ^= k >> 33;
    k *= 0xc4ceb9fe1a85ec53ull;
    k ^= k >> 33;
    return k;
}

struct TierParams {
    int64_t row_off[kMaxTables];   // first global row of table j
    uint32_t rows[kMaxTables];
    int32_t J;
};

// Insert every valid lookup's global row (+1) into the open-addressing set;
// the thread whose CAS claims an empty slot assigns the row the next unique
// id and records it.  Probing is bounded by the set size (half empty at most
// load), so a full set flags ERR_INDEX instead of looping.
__global__ void dedupe_insert_kernel(const uint32_t* __restrict__ idx, int64_t n_lookups, TierParams tp,
                                     unsigned long long* set_keys, uint32_t* set_vals, uint32_t mask,
                                     unsigned long long* ukeys, uint32_t* count, uint32_t* status) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_lookups;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int j = (int)(i % tp.J);
        const uint32_t r = __ldg(idx + i);
        if (r >= tp.rows[j]) continue;               // invalid token: zero row, no fetch
        const unsigned long long key = (unsigned long long)(tp.row_off[j] + r) + 1ull;
        uint32_t h = (uint32_t)mix64(key) & mask;
        bool placed = false;
        for (uint32_t probe = 0; probe <= mask; ++probe) {
            const unsigned long long prev = atomicCAS(set_keys + h, (unsigned long long)kEmpty, key);
            if (prev == kEmpty) {
                const uint32_t id = atomicAdd(count, 1u);
                set_vals[h] = id;
                ukeys[id] = key - 1ull;
                placed = true;
                break;
            }
            if (prev == key) {
                placed = true;
                break;
            }
            h = (h + 1u) & mask;
        }
        if (!placed) flag(status, ENGRAM_ERR_INDEX);
    }
}

// Slot of every lookup (a separate launch, so every insert and id is visible).
__global__ void dedupe_slot_kernel(const uint32_t* __restrict__ idx, int64_t n_lookups, TierParams tp,
                                   const unsigned long long* __restrict__ set_keys,
                                   const uint32_t* __restrict__ set_vals, uint32_t mask, uint32_t* __restrict__ slot) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_lookups;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int j = (int)(i % tp.J);
        const uint32_t r = __ldg(idx + i);
        uint32_t out = ENGRAM_INVALID_INDEX;
        if (r < tp.rows[j]) {
            const unsigned long long key = (unsigned long long)(tp.row_off[j] + r) + 1ull;
            uint32_t h = (uint32_t)mix64(key) & mask;
            for (uint32_t probe = 0; probe <= mask; ++probe) {
                const unsigned long long k = __ldg(set_keys + h);
                if (k == key) {
                    out = __ldg(set_vals + h);
                    break;
                }
                if (k == kEmpty) break;
                h = (h + 1u) & mask;
            }
        }
        slot[i] = out;
    }
}

// Copy rows [r0, r1) of the distinct-row list from the host tables into the
// staging buffer, prefetching a few rows ahead.  A row number outside the
// tables (impossible for lists the dedupe kernel wrote) gives a zero row.
// On x86 the staging writes are non-temporal (streaming) stores: the staging
// buffer is read next by the copy engine, not by this core, and skipping the
// read-for-ownership of each line leaves more host memory bandwidth to the
// PCIe copies running at the same time.  A store fence ends the range, so
// the rows are in memory before the chunk is marked packed.
void pack_range(const uint8_t* tables, int64_t total_rows, size_t row_bytes, const uint64_t* rows, int64_t r0,
                int64_t r1, uint8_t* dst) {
    constexpr int kAhead = 8;
#if defined(__SSE2__)
    const bool stream = (row_bytes % 16) == 0 && (reinterpret_cast<uintptr_t>(dst) % 16) == 0;
#else
    const bool stream = false;
#endif
    for (int64_t r = r0; r < r1; ++r) {
        if (r + kAhead < r1 && rows[r + kAhead] < (uint64_t)total_rows) {
            const uint8_t* pf = tables + rows[r + kAhead] * row_bytes;
            for (size_t o = 0; o < row_bytes; o += 64) __builtin_prefetch(pf + o);
        }
        uint8_t* out = dst + (size_t)r * row_bytes;
        if (rows[r] >= (uint64_t)total_rows) {
            std::memset(out, 0, row_bytes);
            continue;
        }
        const uint8_t* in = tables + rows[r] * row_bytes;
#if defined(__SSE2__)
        if (stream) {
            for (size_t o = 0; o < row_bytes; o += 16)
                _mm_stream_si128(reinterpret_cast<__m128i*>(out + o),
                                 _mm_loadu_si128(reinterpret_cast<const __m128i*>(in + o)));
            continue;
        }
#endif
        std::memcpy(out, in, row_bytes);
    }
#if defined(__SSE2__)
    if (stream) _mm_sfence();
#endif
}

}  // namespace
}  // namespace engram

using namespace engram;

// A pool of packing threads that sleep between batches.
struct engram_host_tier {
    engram_ctx* c;
    const uint8_t* host_tables;
    int64_t total_rows;
    size_t row_bytes;
    int64_t max_lookups;
    TierParams tp;
    // device
    unsigned long long* d_set_keys;
    uint32_t* d_set_vals;
    uint32_t set_mask;
    unsigned long long* d_ukeys;
    uint32_t* d_count;
    uint32_t* d_slot;
    uint8_t* d_rows;
    // pinned host
    unsigned long long* h_ukeys;
    uint32_t* h_count;
    uint8_t* h_stage;
    cudaEvent_t ev_keys, ev_ready, ev_consumed;
    cudaEvent_t ev_copy0, ev_copy1;   // timing: first row copy enqueued, last one done
    bool have_keys, fetched, consumed_recorded;
    int64_t pending_lookups;
    // packing pool
    std::vector<std::thread> workers;
    std::mutex mu;
    std::condition_variable cv;
    uint64_t job_gen;
    bool stop;
    const uint64_t* job_rows;
    int64_t job_n;
    int64_t job_chunks;
    std::atomic<int64_t> next_chunk;
    std::vector<std::atomic<uint8_t>>* chunk_done;
    // statistics of the last fetch
    int64_t last_unique;
    double last_wait_ms;
    double last_pack_ms;
    int64_t last_copies;
};

namespace {

void worker_main(engram_host_tier* t) {
    uint64_t seen = 0;
    for (;;) {
        {
            std::unique_lock<std::mutex> lock(t->mu);
            t->cv.wait(lock, [&] { return t->stop || t->job_gen != seen; });
            if (t->stop) return;
            seen = t->job_gen;
        }
        for (;;) {
            const int64_t k = t->next_chunk.fetch_add(1);
            if (k >= t->job_chunks) break;
            const int64_t r0 = k * kPackChunkRows;
            const int64_t r1 = std::min(t->job_n, r0 + kPackChunkRows);
            pack_range(t->host_tables, t->total_rows, t->row_bytes, t->job_rows, r0, r1, t->h_stage);
            (*t->chunk_done)[k].store(1, std::memory_order_release);
        }
    }
}

// Host wait on an event, bounded: ENGRAM_E_TIMEOUT if it does not complete.
engram_status wait_event_bounded(cudaEvent_t ev, const char* what) {
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t e = cudaEventQuery(ev);
        if (e == cudaSuccess) return ENGRAM_OK;
        if (e != cudaErrorNotReady) return cuda_fail(what, e);
        if (std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count() > kHostWaitSeconds) {
            set_error(what);
            return ENGRAM_E_TIMEOUT;
        }
        std::this_thread::sleep_for(std::chrono::microseconds(20));
    }
}

void tier_free(engram_host_tier* t) {
    if (!t) return;
    {
        std::lock_guard<std::mutex> lock(t->mu);
        t->stop = true;
    }
    t->cv.notify_all();
    for (auto& w : t->workers) w.join();
    if (t->ev_keys) cudaEventDestroy(t->ev_keys);
    if (t->ev_ready) cudaEventDestroy(t->ev_ready);
    if (t->ev_consumed) cudaEventDestroy(t->ev_consumed);
    if (t->ev_copy0) cudaEventDestroy(t->ev_copy0);
    if (t->ev_copy1) cudaEventDestroy(t->ev_copy1);
    cudaFree(t->d_set_keys);
    cudaFree(t->d_set_vals);
    cudaFree(t->d_ukeys);
    cudaFree(t->d_count);
    cudaFree(t->d_slot);
    cudaFree(t->d_rows);
    cudaFreeHost(t->h_ukeys);
    cudaFreeHost(t->h_count);
    cudaFreeHost(t->h_stage);
    delete t->chunk_done;
    delete t;
}

}  // namespace

extern "C" {

engram_status engram_pack_rows(const void* host_tables, int64_t total_rows, size_t row_bytes, const uint64_t* rows,
                               int64_t n, void* dst, int32_t n_threads) {
    if (n < 0 || row_bytes == 0 || total_rows < 0) return inval("need n >= 0, total_rows >= 0 and row_bytes > 0");
    if (n == 0) return ENGRAM_OK;
    if (!host_tables || !rows || !dst) return inval("null pointer");
    for (int64_t r = 0; r < n; ++r)
        if (rows[r] >= (uint64_t)total_rows) return inval("a row number lies outside the tables");
    const int nt = std::max(1, std::min<int>(n_threads, 256));
    const uint8_t* tb = static_cast<const uint8_t*>(host_tables);
    uint8_t* out = static_cast<uint8_t*>(dst);
    std::vector<std::thread> th;
    const int64_t per = (n + nt - 1) / nt;
    for (int i = 0; i < nt; ++i) {
        const int64_t r0 = i * per, r1 = std::min(n, r0 + per);
        if (r0 >= r1) break;
        th.emplace_back([=] { pack_range(tb, total_rows, row_bytes, rows, r0, r1, out); });
    }
    for (auto& x : th) x.join();
    return ENGRAM_OK;
}

engram_status engram_host_tier_create(engram_ctx* c, const void* host_tables, int64_t max_lookups, int32_t n_threads,
                                      engram_host_tier** out) {
    if (!c || !out) return inval("null context or output pointer");
    *out = nullptr;
    if (!host_tables) return inval("null host tables");
    if (max_lookups < 1 || max_lookups > ((int64_t)1 << 30)) return inval("max_lookups must be in [1, 2^30]");
    if (n_threads < 1 || n_threads > 256) return inval("n_threads must be in [1, 256]");
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    engram_host_tier* t = new (std::nothrow) engram_host_tier();
    if (!t) return ENGRAM_E_NOMEM;
    t->c = c;
    t->host_tables = static_cast<const uint8_t*>(host_tables);
    t->row_bytes = (size_t)c->cfg.row_dim * c->es;
    t->max_lookups = max_lookups;
    t->tp.J = c->J;
    int64_t off = 0;
    for (int j = 0; j < c->J; ++j) {
        t->tp.row_off[j] = off;
        t->tp.rows[j] = c->cfg.rows[j];
        off += c->cfg.rows[j];
    }
    t->total_rows = off;
    uint32_t cap = 1;
    while ((int64_t)cap < 2 * max_lookups) cap <<= 1;   // load factor <= 1/2
    t->set_mask = cap - 1;
    t->chunk_done = new (std::nothrow) std::vector<std::atomic<uint8_t>>(
        (size_t)((max_lookups + kPackChunkRows - 1) / kPackChunkRows));
    cudaError_t e = t->chunk_done ? cudaSuccess : cudaErrorMemoryAllocation;
    if (e == cudaSuccess) e = cudaMalloc(&t->d_set_keys, (size_t)cap * sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMalloc(&t->d_set_vals, (size_t)cap * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMalloc(&t->d_ukeys, (size_t)max_lookups * sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMalloc(&t->d_count, 256);
    if (e == cudaSuccess) e = cudaMalloc(&t->d_slot, (size_t)max_lookups * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMalloc(&t->d_rows, (size_t)max_lookups * t->row_bytes);
    if (e == cudaSuccess) e = cudaHostAlloc(&t->h_ukeys, (size_t)max_lookups * sizeof(unsigned long long), 0);
    if (e == cudaSuccess) e = cudaHostAlloc(&t->h_count, 256, 0);
    if (e == cudaSuccess) e = cudaHostAlloc(&t->h_stage, (size_t)max_lookups * t->row_bytes, 0);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t->ev_keys, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t->ev_ready, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t->ev_consumed, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreate(&t->ev_copy0);
    if (e == cudaSuccess) e = cudaEventCreate(&t->ev_copy1);
    if (e != cudaSuccess) {
        tier_free(t);
        if (e == cudaErrorMemoryAllocation) {
            set_error("host tier: device or pinned host allocation failed");
            return ENGRAM_E_NOMEM;
        }
        return cuda_fail("host tier set-up", e);
    }
    try {
        for (int i = 0; i < n_threads; ++i) t->workers.emplace_back(worker_main, t);
    } catch (...) {
        tier_free(t);
        set_error("host tier: could not start the packing threads");
        return ENGRAM_E_HOST;
    }
    *out = t;
    return ENGRAM_OK;
}

void engram_host_tier_destroy(engram_host_tier* t) {
    if (!t) return;
    // copies of the last batch may still be in flight into the pinned buffers
    if (t->fetched) wait_event_bounded(t->ev_ready, "host tier: draining the last fetch");
    if (t->have_keys) wait_event_bounded(t->ev_keys, "host tier: draining the last dedupe");
    tier_free(t);
}

engram_status engram_host_dedupe(engram_host_tier* t, const uint32_t* idx, int64_t n_tok, cudaStream_t s) {
    if (!t) return inval("null host tier");
    engram_ctx* c = t->c;
    if (n_tok < 0 || n_tok * c->J > t->max_lookups) return inval("n_tok * J exceeds the tier's max_lookups");
    if (n_tok > 0 && !idx) return inval("null index pointer");
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    // the pinned key list may still be read by a fetch of the previous batch:
    // fetches run on the caller's thread, so by now that fetch has returned
    const int64_t n = n_tok * c->J;
    cudaError_t e = cudaMemsetAsync(t->d_set_keys, 0, (size_t)(t->set_mask + 1) * sizeof(unsigned long long), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(t->d_count, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return cuda_fail("host tier: clearing the set", e);
    if (n > 0) {
        const int threads = 256;
        const int64_t want = (n + threads - 1) / threads;
        const int blocks = (int)std::min<int64_t>(want, (int64_t)c->num_sms * 8);
        dedupe_insert_kernel<<<blocks, threads, 0, s>>>(idx, n, t->tp, t->d_set_keys, t->d_set_vals, t->set_mask,
                                                        t->d_ukeys, t->d_count, c->d_status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("dedupe insert launch", e);
        dedupe_slot_kernel<<<blocks, threads, 0, s>>>(idx, n, t->tp, t->d_set_keys, t->d_set_vals, t->set_mask,
                                                      t->d_slot);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("dedupe slot launch", e);
    }
    // distinct-row count and list to pinned host memory (the list at its
    // largest possible length: one copy, no round trip for the count)
    e = cudaMemcpyAsync(t->h_count, t->d_count, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess && n > 0)
        e = cudaMemcpyAsync(t->h_ukeys, t->d_ukeys, (size_t)n * sizeof(unsigned long long), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaEventRecord(t->ev_keys, s);
    if (e != cudaSuccess) return cuda_fail("host tier: copying the row list out", e);
    t->have_keys = true;
    t->pending_lookups = n;
    return ENGRAM_OK;
}

engram_status engram_host_fetch(engram_host_tier* t, cudaStream_t side, int64_t* n_unique) {
    if (!t) return inval("null host tier");
    if (!t->have_keys) return inval("engram_host_fetch needs a preceding engram_host_dedupe");
    engram_status st = check_device(t->c);
    if (st != ENGRAM_OK) return st;
    const auto tw = std::chrono::steady_clock::now();
    st = wait_event_bounded(t->ev_keys, "host tier: waiting for the row list");
    if (st != ENGRAM_OK) return st;
    // the staging buffer and the device rows may still serve the previous batch
    if (t->fetched) {
        st = wait_event_bounded(t->ev_ready, "host tier: waiting for the previous copies");
        if (st != ENGRAM_OK) return st;
    }
    cudaError_t e = cudaSuccess;
    if (t->consumed_recorded) e = cudaStreamWaitEvent(side, t->ev_consumed, 0);
    if (e != cudaSuccess) return cuda_fail("host tier: ordering the copies after the last gather", e);
    const int64_t U = (int64_t)*t->h_count;
    if (U > t->pending_lookups) {
        set_error("host tier: distinct-row count exceeds the lookups");
        return ENGRAM_E_DEVICE;
    }
    const auto t0 = std::chrono::steady_clock::now();
    const int64_t n_chunks = (U + kPackChunkRows - 1) / kPackChunkRows;
    for (int64_t k = 0; k < n_chunks; ++k) (*t->chunk_done)[k].store(0, std::memory_order_relaxed);
    {
        std::lock_guard<std::mutex> lock(t->mu);
        t->job_rows = reinterpret_cast<const uint64_t*>(t->h_ukeys);
        t->job_n = U;
        t->job_chunks = n_chunks;
        t->next_chunk.store(0);
        ++t->job_gen;
    }
    t->cv.notify_all();
    // hand the packed chunks to the copy engine in order, several chunks per
    // copy (at least kMinCopyBytes but the last)
    const int64_t min_chunks =
        std::max<int64_t>(1, (int64_t)((kMinCopyBytes + kPackChunkRows * t->row_bytes - 1) / (kPackChunkRows * t->row_bytes)));
    auto wait_chunk = [&](int64_t k) -> bool {
        const auto w0 = std::chrono::steady_clock::now();
        while (!(*t->chunk_done)[k].load(std::memory_order_acquire)) {
            if (std::chrono::duration<double>(std::chrono::steady_clock::now() - w0).count() > kHostWaitSeconds)
                return false;
            std::this_thread::yield();
        }
        return true;
    };
    engram_status result = ENGRAM_OK;
    int64_t copies = 0;
    int64_t k = 0;
    while (k < n_chunks && result == ENGRAM_OK) {
        int64_t k1 = k;
        // the next min_chunks chunks (fewer at the end), then any later ones already packed
        while (k1 < n_chunks && (k1 - k < min_chunks || (*t->chunk_done)[k1].load(std::memory_order_acquire))) {
            if (!wait_chunk(k1)) {
                set_error("host tier: a packing thread did not finish its chunk");
                result = ENGRAM_E_HOST;
                break;
            }
            ++k1;
        }
        if (result != ENGRAM_OK) break;
        const int64_t r0 = k * kPackChunkRows;
        const int64_t rn = std::min(U, k1 * kPackChunkRows) - r0;
        if (copies == 0) e = cudaEventRecord(t->ev_copy0, side);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(t->d_rows + (size_t)r0 * t->row_bytes, t->h_stage + (size_t)r0 * t->row_bytes,
                                (size_t)rn * t->row_bytes, cudaMemcpyHostToDevice, side);
        if (e != cudaSuccess) result = cuda_fail("host tier: row copy", e);
        ++copies;
        k = k1;
    }
    if (result != ENGRAM_OK) {
        // let the workers run out of chunks before anyone reuses the job
        const auto w0 = std::chrono::steady_clock::now();
        for (int64_t q = 0; q < n_chunks; ++q)
            while (!(*t->chunk_done)[q].load(std::memory_order_acquire) &&
                   std::chrono::duration<double>(std::chrono::steady_clock::now() - w0).count() < kHostWaitSeconds)
                std::this_thread::yield();
        return result;
    }
    const auto t1 = std::chrono::steady_clock::now();
    if (copies > 0) e = cudaEventRecord(t->ev_copy1, side);
    if (e == cudaSuccess) e = cudaEventRecord(t->ev_ready, side);
    if (e != cudaSuccess) return cuda_fail("host tier: recording the ready event", e);
    t->fetched = true;
    t->have_keys = false;
    t->last_unique = U;
    t->last_copies = copies;
    t->last_wait_ms = std::chrono::duration<double, std::milli>(t0 - tw).count();
    t->last_pack_ms = std::chrono::duration<double, std::milli>(t1 - t0).count();
    if (n_unique) *n_unique = U;
    return ENGRAM_OK;
}

engram_status engram_gather_staged(engram_host_tier* t, int64_t n_tok, void* e_cat, cudaStream_t s) {
    if (!t) return inval("null host tier");
    engram_ctx* c = t->c;
    if (!t->fetched) return inval("engram_gather_staged needs a preceding engram_host_fetch");
    if (n_tok < 0 || n_tok * c->J > t->pending_lookups) return inval("n_tok differs from the deduplicated batch");
    if (n_tok == 0) return ENGRAM_OK;
    if (!e_cat || !aligned16(e_cat)) return inval("e_cat must be a 16-byte aligned device pointer");
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    cudaError_t e = cudaStreamWaitEvent(s, t->ev_ready, 0);
    if (e != cudaSuccess) return cuda_fail("host tier: waiting for the rows", e);
    GatherParams gp = c->gp;
    for (int j = 0; j < c->J; ++j) {
        gp.row_off[j] = 0;
        gp.rows[j] = (uint32_t)std::min<int64_t>(t->max_lookups, 0xFFFFFFFEll);
    }
    prof_reset(c);
    prof_begin(c, s, "gather_staged");
    e = launch_gather(t->d_slot, n_tok, t->d_rows, gp, e_cat, c->d_status, c->num_sms, s);
    prof_end(c, s);
    if (e != cudaSuccess) return cuda_fail("staged gather launch", e);
    e = cudaEventRecord(t->ev_consumed, s);
    if (e != cudaSuccess) return cuda_fail("host tier: recording the consumed event", e);
    t->consumed_recorded = true;
    return ENGRAM_OK;
}

engram_status engram_host_tier_stats(const engram_host_tier* t, engram_host_tier_stats_t* out) {
    if (!t || !out) return inval("null host tier or output");
    out->n_unique = t->last_unique;
    out->n_copies = t->last_copies;
    out->wait_ms = t->last_wait_ms;
    out->pack_ms = t->last_pack_ms;
    out->copy_ms = -1.0;
    if (t->fetched && t->last_copies > 0 && cudaEventQuery(t->ev_copy1) == cudaSuccess) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, t->ev_copy0, t->ev_copy1) == cudaSuccess) out->copy_ms = ms;
    }
    return ENGRAM_OK;
}

}  // extern "C"
