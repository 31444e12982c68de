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
//
// Hot-row cache (engram_host_cache_enable): the same sections, and the
// Synced repost's last paragraph of "System efficiency", keep the frequent
// n-grams' rows in a faster tier, because a few patterns take most of the
// accesses.  Here C rows of HBM in front of the host tables: a device hash
// set maps (table, row) to a cache slot.  The dedupe kernel resolves each
// distinct row of the batch against it; a resident row is read from its
// slot and is not fetched.  After the staged gather, the rows that this
// batch fetched and looked up at least min_count times are admitted into
// free slots (device-to-device, from the staged copy) until the cache is
// full.  Slots and staged rows share one device buffer (slots first), so
// the gather reads both through one slot map.
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
constexpr double kHostWaitSeconds = 20.0;    // default bound on every host-side wait

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

// Cache lookup: slot of global row key-1 in the hot-row set, or -1.
__device__ __forceinline__ int64_t cache_find(const unsigned long long* __restrict__ ckeys,
                                              const uint32_t* __restrict__ cvals, uint32_t cmask,
                                              unsigned long long key) {
    uint32_t h = (uint32_t)mix64(key) & cmask;
    for (uint32_t probe = 0; probe <= cmask; ++probe) {
        const unsigned long long k = ckeys[h];
        if (k == key) return (int64_t)cvals[h];
        if (k == kEmpty) return -1;
        h = (h + 1u) & cmask;
    }
    return -1;
}

struct CacheParams {
    const unsigned long long* keys;   // hot-row set (null: no cache)
    const uint32_t* vals;             // its slots
    uint32_t mask;
    uint32_t capacity;                // C: staged rows start at slot C
};

// Insert every valid lookup's global row (+1) into the open-addressing set
// and count the lookups per entry; the thread whose CAS claims an empty slot
// resolves the row once: a row resident in the hot-row cache gets its cache
// slot (counted in count[1]), any other row the next fetch id (count[0]),
// recorded in the fetch list, and slot C + id.  Probing is bounded by the
// set size (half empty at most load), so a full set flags ERR_INDEX instead
// of looping.
__global__ void dedupe_insert_kernel(const uint32_t* __restrict__ idx, int64_t n_lookups, TierParams tp,
                                     unsigned long long* set_keys, uint32_t* set_vals, uint32_t* set_cnt,
                                     uint32_t mask, CacheParams cp, unsigned long long* ukeys, uint32_t* count,
                                     uint32_t* status) {
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
                const int64_t cs = cp.keys ? cache_find(cp.keys, cp.vals, cp.mask, key) : -1;
                if (cs >= 0) {
                    set_vals[h] = (uint32_t)cs;
                    atomicAdd(count + 1, 1u);
                } else {
                    const uint32_t id = atomicAdd(count, 1u);
                    set_vals[h] = cp.capacity + id;
                    ukeys[id] = key - 1ull;
                }
                atomicAdd(set_cnt + h, 1u);
                placed = true;
                break;
            }
            if (prev == key) {
                atomicAdd(set_cnt + h, 1u);
                placed = true;
                break;
            }
            h = (h + 1u) & mask;
        }
        if (!placed) flag(status, ENGRAM_ERR_INDEX);
    }
}

// Admission into the hot-row cache, after the staged gather: every entry of
// the batch set that was fetched (slot >= C) and looked up at least
// min_count times takes the next free cache slot, while any is left; its row
// is copied from the staged rows (16-byte chunks, one warp per row) and its
// key enters the cache set.  count[2] is the number of slots in use.
__global__ void cache_admit_kernel(const unsigned long long* __restrict__ set_keys,
                                   const uint32_t* __restrict__ set_vals, const uint32_t* __restrict__ set_cnt,
                                   uint32_t set_slots, uint32_t min_count, unsigned long long* ckeys, uint32_t* cvals,
                                   uint32_t cmask, uint32_t capacity, uint4* rows, int chunks_per_row, uint32_t* count,
                                   uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = warp0 * 32; base < set_slots; base += nwarps * 32) {
        // each lane inspects one set entry; admitted entries are then copied by the whole warp
        const int64_t h = base + lane;
        bool want = false;
        unsigned long long key = kEmpty;
        uint32_t src = 0;
        if (h < set_slots) {
            key = set_keys[h];
            src = set_vals[h];
            want = key != kEmpty && src >= capacity && set_cnt[h] >= min_count;
        }
        uint32_t slot = 0xFFFFFFFFu;
        if (want) {
            const uint32_t s = atomicAdd(count + 2, 1u);
            if (s < capacity) {
                slot = s;
            } else {
                atomicSub(count + 2, 1u);    // full: the count stays at capacity
            }
        }
        if (slot != 0xFFFFFFFFu) {
            uint32_t hh = (uint32_t)mix64(key) & cmask;
            bool placed = false;
            for (uint32_t probe = 0; probe <= cmask; ++probe) {
                const unsigned long long prev = atomicCAS(ckeys + hh, (unsigned long long)kEmpty, key);
                if (prev == kEmpty) {
                    cvals[hh] = slot;
                    placed = true;
                    break;
                }
                hh = (hh + 1u) & cmask;
            }
            if (!placed) flag(status, ENGRAM_ERR_INDEX);
        }
        uint32_t todo = __ballot_sync(0xffffffffu, slot != 0xFFFFFFFFu);
        while (todo) {
            const int l = __ffs(todo) - 1;
            todo &= todo - 1;
            const uint32_t dst = __shfl_sync(0xffffffffu, slot, l);
            const uint32_t from = __shfl_sync(0xffffffffu, src, l);
            for (int c = lane; c < chunks_per_row; c += 32)
                rows[(int64_t)dst * chunks_per_row + c] = rows[(int64_t)from * chunks_per_row + c];
        }
    }
}

// Slot of every lookup (a separate launch, so every insert and slot is
// visible): a cache slot, C + fetch id, or ENGRAM_INVALID_INDEX.
__global__ void dedupe_slot_kernel(const uint32_t* __restrict__ idx, int64_t n_lookups, TierParams tp,
                                   const unsigned long long* __restrict__ set_keys,
                                   const uint32_t* __restrict__ set_vals, uint32_t mask, uint32_t capacity,
                                   uint32_t* __restrict__ slot, uint32_t* count) {
    // every thread of the grid runs the same number of iterations (the bound
    // is rounded up to the grid), so the warp-wide vote below is uniform
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t n_iter = (n_lookups + stride - 1) / stride * stride;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_iter; i += stride) {
        if (i >= n_lookups) {
            __ballot_sync(0xffffffffu, false);
            continue;
        }
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
        // lookups served from the hot-row cache, one atomic per warp
        const uint32_t hits = __ballot_sync(0xffffffffu, out < capacity);
        if ((threadIdx.x & 31) == 0 && hits) atomicAdd(count + 3, (uint32_t)__popc(hits));
    }
}

// Mapped fetch (engram_host_tier_map): the distinct rows come straight from
// the host tables, which are mapped into the device's address space, into
// the staged rows [C + id]: every load crosses PCIe as a read request of the
// GPU, issued by many warps at once, and no host thread packs anything.  The
// row list and its length are read on the device.  Each thread issues
// kBatchMapped independent 16-byte loads before its stores.
constexpr int kBatchMapped = 4;
__global__ void __launch_bounds__(256) mapped_fetch_kernel(const uint4* __restrict__ host_rows,
                                                          const unsigned long long* __restrict__ ukeys,
                                                          const uint32_t* __restrict__ count, int chunks_per_row,
                                                          uint64_t total_rows, uint4* __restrict__ staged,
                                                          uint32_t* status) {
    const int64_t n = (int64_t)__ldg(count) * chunks_per_row;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t f0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; f0 < n; f0 += stride * kBatchMapped) {
        uint4 v[kBatchMapped];
#pragma unroll
        for (int u = 0; u < kBatchMapped; ++u) {
            const int64_t f = f0 + u * stride;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (f < n) {
                const int64_t r = f / chunks_per_row, c = f - r * chunks_per_row;
                const uint64_t row = __ldg(ukeys + r);
                if (row < total_rows) v[u] = host_rows[row * chunks_per_row + c];
                else flag(status, ENGRAM_ERR_INDEX);
            }
        }
#pragma unroll
        for (int u = 0; u < kBatchMapped; ++u) {
            const int64_t f = f0 + u * stride;
            if (f < n) staged[f] = v[u];
        }
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
    uint32_t* d_set_cnt;    // lookups per set entry in this batch
    uint32_t* d_count;      // [0] rows to fetch, [1] distinct rows found in the cache, [2] cache slots in use,
                            // [3] lookups served from the cache
    uint32_t* d_slot;
    uint8_t* d_rows;        // cache slots [0, C) then the staged rows [C, C + max_lookups)
    // mapped mode (engram_host_tier_map): the host tables as device-visible memory
    const uint4* d_host_tables;
    bool mapped_registered;   // this tier registered the host range (and unregisters it)
    // hot-row cache (capacity 0: none)
    uint32_t cache_cap;
    uint32_t cache_min_count;
    unsigned long long* d_ckeys;
    uint32_t* d_cvals;
    uint32_t cache_mask;
    // pinned host
    unsigned long long* h_ukeys;
    uint32_t* h_count;
    uint8_t* h_stage;
    cudaEvent_t ev_keys, ev_ready, ev_consumed;
    cudaEvent_t ev_copy0, ev_copy1;   // timing: first row copy enqueued, last one done
    bool have_keys, fetched, consumed_recorded;
    bool copies_recorded;   // ev_ready marks the end of every copy enqueued so far (success or failure)
    // failure injection (engram_host_tier_debug): one-shot faults made on the host
    std::atomic<uint32_t> inject;
    double wait_limit_s;    // bound on every host-side wait
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
            if (k == t->job_chunks - 1 &&
                (t->inject.fetch_and(~ENGRAM_INJECT_PACK_ABANDON) & ENGRAM_INJECT_PACK_ABANDON))
                continue;   // injected: this thread gives up its chunk without packing or marking it
            const int64_t r0 = k * kPackChunkRows;
            const int64_t r1 = std::min(t->job_n, r0 + kPackChunkRows);
            pack_range(t->host_tables, t->total_rows, t->row_bytes, t->job_rows, r0, r1, t->h_stage);
            (*t->chunk_done)[k].store(1, std::memory_order_release);
        }
    }
}

// Host wait on an event, bounded by `limit` seconds: ENGRAM_E_TIMEOUT if it
// does not complete.  `never` fakes an event that never completes (the
// injected list-wait failure): the query's answer is replaced, nothing else.
engram_status wait_event_bounded(cudaEvent_t ev, const char* what, double limit = kHostWaitSeconds,
                                 bool never = false) {
    const auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        const cudaError_t e = never ? cudaErrorNotReady : cudaEventQuery(ev);
        if (e == cudaSuccess) return ENGRAM_OK;
        if (e != cudaErrorNotReady) return cuda_fail(what, e);
        if (std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count() > limit) {
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
    cudaFree(t->d_set_cnt);
    cudaFree(t->d_ckeys);
    cudaFree(t->d_cvals);
    cudaFree(t->d_slot);
    cudaFree(t->d_rows);
    cudaFreeHost(t->h_ukeys);
    cudaFreeHost(t->h_count);
    cudaFreeHost(t->h_stage);
    if (t->mapped_registered) cudaHostUnregister(const_cast<uint8_t*>(t->host_tables));
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
    t->wait_limit_s = kHostWaitSeconds;
    t->inject.store(0);
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
    if (e == cudaSuccess) e = cudaMalloc(&t->d_set_cnt, (size_t)cap * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMalloc(&t->d_ukeys, (size_t)max_lookups * sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMalloc(&t->d_count, 256);
    if (e == cudaSuccess) e = cudaMemset(t->d_count, 0, 256);
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
    if (t->copies_recorded) wait_event_bounded(t->ev_ready, "host tier: draining the last fetch");
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
    if (e == cudaSuccess) e = cudaMemsetAsync(t->d_set_cnt, 0, (size_t)(t->set_mask + 1) * sizeof(uint32_t), s);
    // the batch's counters; count[2] (cache slots in use) carries over
    if (e == cudaSuccess) e = cudaMemsetAsync(t->d_count, 0, 2 * sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(t->d_count + 3, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return cuda_fail("host tier: clearing the set", e);
    if (n > 0) {
        const int threads = 256;
        const int64_t want = (n + threads - 1) / threads;
        const int blocks = (int)std::min<int64_t>(want, (int64_t)c->num_sms * 8);
        CacheParams cp{t->cache_cap ? t->d_ckeys : nullptr, t->d_cvals, t->cache_mask, t->cache_cap};
        dedupe_insert_kernel<<<blocks, threads, 0, s>>>(idx, n, t->tp, t->d_set_keys, t->d_set_vals, t->d_set_cnt,
                                                        t->set_mask, cp, t->d_ukeys, t->d_count, c->d_status);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("dedupe insert launch", e);
        dedupe_slot_kernel<<<blocks, threads, 0, s>>>(idx, n, t->tp, t->d_set_keys, t->d_set_vals, t->set_mask,
                                                      t->cache_cap, t->d_slot, t->d_count);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("dedupe slot launch", e);
    }
    // distinct-row count and list to pinned host memory (the list at its
    // largest possible length: one copy, no round trip for the count)
    e = cudaMemcpyAsync(t->h_count, t->d_count, 4 * sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
    // the mapped fetch reads the list on the device: only the copy path needs it on the host
    if (e == cudaSuccess && n > 0 && !t->d_host_tables)
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
    if (t->d_host_tables) {
        // mapped: everything stays on the GPU's queues; the side stream waits
        // for the dedupe and for the previous staged gather, then one kernel
        // pulls the distinct rows over PCIe.  The count is not known here.
        t->fetched = false;
        cudaError_t e = cudaStreamWaitEvent(side, t->ev_keys, 0);
        if (e == cudaSuccess && t->consumed_recorded) e = cudaStreamWaitEvent(side, t->ev_consumed, 0);
        if (e == cudaSuccess) e = cudaEventRecord(t->ev_copy0, side);
        if (e != cudaSuccess) return cuda_fail("host tier: ordering the mapped fetch", e);
        const int cpr = (int)(t->row_bytes / 16);
        const int blocks = t->c->num_sms * 8;
        mapped_fetch_kernel<<<blocks, 256, 0, side>>>(t->d_host_tables, t->d_ukeys, t->d_count, cpr,
                                                      (uint64_t)t->total_rows,
                                                      reinterpret_cast<uint4*>(t->d_rows) + (size_t)t->cache_cap * cpr,
                                                      t->c->d_status);
        e = cudaGetLastError();
        if (e == cudaSuccess) e = cudaEventRecord(t->ev_copy1, side);
        if (e == cudaSuccess) e = cudaEventRecord(t->ev_ready, side);
        if (e != cudaSuccess) return cuda_fail("host tier: mapped fetch launch", e);
        t->fetched = true;
        t->copies_recorded = true;
        t->have_keys = false;
        t->last_unique = -1;
        t->last_copies = 0;
        t->last_wait_ms = 0.0;
        t->last_pack_ms = 0.0;
        if (n_unique) *n_unique = -1;
        return ENGRAM_OK;
    }
    // until this fetch succeeds, gather_staged must not read the staged rows
    t->fetched = false;
    const auto tw = std::chrono::steady_clock::now();
    const bool fake_list = (t->inject.fetch_and(~ENGRAM_INJECT_LIST_WAIT) & ENGRAM_INJECT_LIST_WAIT) != 0;
    st = wait_event_bounded(t->ev_keys, "host tier: waiting for the row list", t->wait_limit_s, fake_list);
    if (st != ENGRAM_OK) return st;
    // the staging buffer and the device rows may still serve the previous
    // batch, or hold copies that a failed fetch left in flight
    if (t->copies_recorded) {
        st = wait_event_bounded(t->ev_ready, "host tier: waiting for the previous copies", t->wait_limit_s);
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
            if (std::chrono::duration<double>(std::chrono::steady_clock::now() - w0).count() > t->wait_limit_s)
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
            e = cudaMemcpyAsync(t->d_rows + ((size_t)t->cache_cap + r0) * t->row_bytes,
                                t->h_stage + (size_t)r0 * t->row_bytes,
                                (size_t)rn * t->row_bytes, cudaMemcpyHostToDevice, side);
        if (e != cudaSuccess) result = cuda_fail("host tier: row copy", e);
        ++copies;
        k = k1;
    }
    if (result != ENGRAM_OK) {
        // copies already enqueued still read the pinned staging: the next
        // fetch (and destroy) must wait for them before the staging is
        // packed again, so their end is recorded like a successful fetch's
        if (copies > 0) {
            if (cudaEventRecord(t->ev_ready, side) == cudaSuccess) {
                t->copies_recorded = true;
            } else {
                cudaStreamSynchronize(side);
                t->copies_recorded = false;
            }
        }
        // let the workers run out of chunks before anyone reuses the job
        const auto w0 = std::chrono::steady_clock::now();
        for (int64_t q = 0; q < n_chunks; ++q)
            while (!(*t->chunk_done)[q].load(std::memory_order_acquire) &&
                   std::chrono::duration<double>(std::chrono::steady_clock::now() - w0).count() < t->wait_limit_s)
                std::this_thread::yield();
        return result;
    }
    const auto t1 = std::chrono::steady_clock::now();
    if (copies > 0) e = cudaEventRecord(t->ev_copy1, side);
    if (e == cudaSuccess) e = cudaEventRecord(t->ev_ready, side);
    if (e != cudaSuccess) return cuda_fail("host tier: recording the ready event", e);
    t->fetched = true;
    t->copies_recorded = true;
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
    if (!t->fetched) return inval("engram_gather_staged needs a preceding successful engram_host_fetch");
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
        gp.rows[j] = (uint32_t)std::min<int64_t>((int64_t)t->cache_cap + t->max_lookups, 0xFFFFFFFEll);
    }
    prof_reset(c);
    prof_begin(c, s, "gather_staged");
    e = launch_gather(t->d_slot, n_tok, t->d_rows, gp, e_cat, c->d_status, c->num_sms, s);
    prof_end(c, s);
    if (e != cudaSuccess) return cuda_fail("staged gather launch", e);
    if (t->cache_cap) {
        // admission reads the staged rows, so it runs before the next fetch may overwrite them
        const uint32_t slots = t->set_mask + 1;
        const int blocks = (int)std::min<int64_t>((slots + 255) / 256, (int64_t)c->num_sms * 8);
        prof_begin(c, s, "cache_admit");
        cache_admit_kernel<<<blocks, 256, 0, s>>>(t->d_set_keys, t->d_set_vals, t->d_set_cnt, slots,
                                                  t->cache_min_count, t->d_ckeys, t->d_cvals, t->cache_mask,
                                                  t->cache_cap, reinterpret_cast<uint4*>(t->d_rows),
                                                  (int)(t->row_bytes / 16), t->d_count, c->d_status);
        prof_end(c, s);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("cache admission launch", e);
    }
    e = cudaEventRecord(t->ev_consumed, s);
    if (e != cudaSuccess) return cuda_fail("host tier: recording the consumed event", e);
    t->consumed_recorded = true;
    return ENGRAM_OK;
}

engram_status engram_host_tier_map(engram_host_tier* t) {
    if (!t) return inval("null host tier");
    if (t->d_host_tables) return ENGRAM_OK;
    if (t->have_keys || t->fetched) return inval("map the host tables before the first batch");
    engram_status st = check_device(t->c);
    if (st != ENGRAM_OK) return st;
    const size_t bytes = (size_t)t->total_rows * t->row_bytes;
    void* host = const_cast<uint8_t*>(t->host_tables);
    cudaError_t e = cudaHostRegister(host, bytes, cudaHostRegisterMapped | cudaHostRegisterReadOnly);
    if (e == cudaErrorHostMemoryAlreadyRegistered) {
        cudaGetLastError();
        e = cudaSuccess;       // the caller's registration (it must be mapped)
    } else if (e == cudaSuccess) {
        t->mapped_registered = true;
    }
    void* dev = nullptr;
    if (e == cudaSuccess) e = cudaHostGetDevicePointer(&dev, host, 0);
    if (e != cudaSuccess) {
        if (t->mapped_registered) cudaHostUnregister(host);
        t->mapped_registered = false;
        return cuda_fail("host tier: mapping the host tables", e);
    }
    if ((reinterpret_cast<uintptr_t>(dev) & 15u) != 0) {
        if (t->mapped_registered) cudaHostUnregister(host);
        t->mapped_registered = false;
        return inval("the mapped host tables are not 16-byte aligned");
    }
    t->d_host_tables = static_cast<const uint4*>(dev);
    return ENGRAM_OK;
}

engram_status engram_host_cache_enable(engram_host_tier* t, int64_t capacity_rows, int32_t min_count) {
    if (!t) return inval("null host tier");
    if (capacity_rows < 1 || capacity_rows > ((int64_t)1 << 30)) return inval("capacity_rows must be in [1, 2^30]");
    if (min_count < 1) return inval("min_count must be >= 1");
    if (t->cache_cap) return inval("the hot-row cache is already enabled");
    if (t->have_keys || t->fetched) return inval("enable the hot-row cache before the first batch");
    engram_status st = check_device(t->c);
    if (st != ENGRAM_OK) return st;
    if (t->copies_recorded) {
        st = wait_event_bounded(t->ev_ready, "host tier: draining copies before the cache is set up", t->wait_limit_s);
        if (st != ENGRAM_OK) return st;
    }
    uint32_t cap = 1;
    while ((int64_t)cap < 2 * capacity_rows) cap <<= 1;   // load factor <= 1/2
    uint8_t* rows = nullptr;
    unsigned long long* ckeys = nullptr;
    uint32_t* cvals = nullptr;
    cudaError_t e = cudaMalloc(&rows, ((size_t)capacity_rows + (size_t)t->max_lookups) * t->row_bytes);
    if (e == cudaSuccess) e = cudaMalloc(&ckeys, (size_t)cap * sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMalloc(&cvals, (size_t)cap * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemset(ckeys, 0, (size_t)cap * sizeof(unsigned long long));
    if (e == cudaSuccess) e = cudaMemset(t->d_count + 2, 0, sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaFree(rows);
        cudaFree(ckeys);
        cudaFree(cvals);
        if (e == cudaErrorMemoryAllocation) {
            set_error("host tier: the hot-row cache does not fit in device memory");
            return ENGRAM_E_NOMEM;
        }
        return cuda_fail("host tier: hot-row cache set-up", e);
    }
    cudaFree(t->d_rows);
    t->d_rows = rows;
    t->d_ckeys = ckeys;
    t->d_cvals = cvals;
    t->cache_mask = cap - 1;
    t->cache_cap = (uint32_t)capacity_rows;
    t->cache_min_count = (uint32_t)min_count;
    return ENGRAM_OK;
}

engram_status engram_host_cache_reset(engram_host_tier* t, cudaStream_t s) {
    if (!t) return inval("null host tier");
    if (!t->cache_cap) return inval("the hot-row cache is not enabled");
    engram_status st = check_device(t->c);
    if (st != ENGRAM_OK) return st;
    cudaError_t e = cudaMemsetAsync(t->d_ckeys, 0, (size_t)(t->cache_mask + 1) * sizeof(unsigned long long), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(t->d_count + 2, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return cuda_fail("host tier: clearing the hot-row cache", e);
    return ENGRAM_OK;
}

engram_status engram_host_cache_stats(const engram_host_tier* t, engram_host_cache_stats_t* out) {
    if (!t || !out) return inval("null host tier or output");
    out->capacity = t->cache_cap;
    out->lookups = t->have_keys || t->fetched ? t->pending_lookups : 0;
    out->resident = t->h_count ? t->h_count[2] : 0;
    out->cached_rows = t->h_count ? t->h_count[1] : 0;
    out->fetched_rows = t->h_count ? t->h_count[0] : 0;
    out->cached_lookups = t->h_count ? t->h_count[3] : 0;
    return ENGRAM_OK;
}

engram_status engram_host_tier_debug(engram_host_tier* t, uint32_t inject, double wait_limit_s) {
    if (!t) return inval("null host tier");
    if (inject & ~(uint32_t)(ENGRAM_INJECT_LIST_WAIT | ENGRAM_INJECT_PACK_ABANDON)) return inval("unknown injection bit");
    if (!(wait_limit_s > 0.0) || wait_limit_s > 3600.0) return inval("wait_limit_s must be in (0, 3600]");
    t->wait_limit_s = wait_limit_s;
    t->inject.fetch_or(inject);
    return ENGRAM_OK;
}

engram_status engram_host_tier_stats(const engram_host_tier* t, engram_host_tier_stats_t* out) {
    if (!t || !out) return inval("null host tier or output");
    // mapped fetches learn the count from the dedupe's copy of it, once the batch is done
    out->n_unique = t->last_unique >= 0 ? t->last_unique : (int64_t)(t->h_count ? t->h_count[0] : 0);
    out->n_copies = t->last_copies;
    out->wait_ms = t->last_wait_ms;
    out->pack_ms = t->last_pack_ms;
    out->copy_ms = -1.0;
    if (t->fetched && (t->last_copies > 0 || t->d_host_tables) && cudaEventQuery(t->ev_copy1) == cudaSuccess) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, t->ev_copy0, t->ev_copy1) == cudaSuccess) out->copy_ms = ms;
    }
    return ENGRAM_OK;
}

}  // extern "C"
