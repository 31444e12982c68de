// Training backward for the tables: the gradient of every table row that a
// batch looked up, as a sparse list of (row, summed gradient).
//
// "DeepSeek AI II" digest, section "DeepSeek Engram", the training
// paragraph (and the Synced repost, "System efficiency"): the embedding
// tables are trained with the model; the backward sends each accessed row's
// gradient to the shard that stores it.  Since e_t is the concatenation of
// the rows E_j[idx_j(t)], the gradient of row r of table j is the sum, over
// the lookups (t, j) with idx_j(t) = r, of the slice j of dL/de_t.
//
// Deterministic: the sum of every row runs in an order fixed by the row's
// lookups alone, whatever order the atomics gave the work: increasing lookup
// order (t * J + j) for a row looked up at most 32 times; for a longer row,
// running sums over every slots-th lookup in increasing order, added in a
// fixed order (grad_reduce_heavy_kernel).
//   1. dedupe: every valid lookup's global row (row_off[j] + idx) goes into an
//      open-addressing set; the thread that claims a row gives it the next id
//      and records the row; every lookup then learns its row's id and counts
//      itself into its id's bucket.
//   2. scan: exclusive prefix sum of the bucket sizes (three levels of
//      4096-element blocks), the start of every row's segment.
//   3. place: every lookup writes its position into its row's segment (in
//      the order the atomics give).
//   4. reduce: a group of lanes per row (as many as the row has 16-byte
//      chunks, rounded up to a power of two) orders its segment by position
//      (each lookup's rank is the number of smaller positions in the segment)
//      and sums the slices of dL/de in that order, in fp32; a row looked up
//      once skips the ordering.  Rows looked up more than 32 times are only
//      listed by that launch; a second launch orders and sums each with a CTA.
// Ordering a row's segment costs k^2 comparisons for k lookups, spread over
// a lane group (k <= 32) or a CTA of 256 threads (longer rows): negligible
// for Zipf batches, whose longest segments hold a few hundred lookups, but
// a degenerate batch in which one n-gram fills a table of a million-token
// batch costs about 4e9 comparisons per thread of that row's CTA.
#include <algorithm>

#include "ctx.cuh"

namespace engram {
namespace {

constexpr uint64_t kEmptyKey = 0;   // set key of an empty slot (keys are row + 1)
constexpr int kScanThreads = 1024;
constexpr int kScanPer = 4;         // elements per thread
constexpr int kScanBlock = kScanThreads * kScanPer;

__device__ __forceinline__ uint64_t mix64(uint64_t k) {
    // Murmur3's 64-bit finaliser (Appleby), to spread row numbers over the set
    k ^= k >> 33;
    k *= 0xff51afd7ed558ccdull;
    k ^= k >> 33;
    k *= 0xc4ceb9fe1a85ec53ull;
    k ^= k >> 33;
    return k;
}

struct GradGeo {
    int64_t row_off[kMaxTables];
    uint32_t rows[kMaxTables];
    int32_t J;
};

__device__ __forceinline__ int64_t find_slot(const unsigned long long* keys, uint32_t mask, unsigned long long key) {
    uint32_t h = (uint32_t)mix64(key) & mask;
    for (uint32_t probe = 0; probe <= mask; ++probe) {
        const unsigned long long k = keys[h];
        if (k == key) return h;
        if (k == kEmptyKey) return -1;
        h = (h + 1u) & mask;
    }
    return -1;
}

// Where a lookup's key (global row + 1) comes from.  LookupKeys: the
// lookups (t, j) of a batch, global row row_off[j] + idx (an invalid n-gram
// has no row and no gradient).  PairKeys: (row, gradient) pairs sent by the
// ranks to the shard that owns rows [lo, hi); a row outside it is an error.
struct LookupKeys {
    const uint32_t* idx;
    GradGeo g;
    __device__ __forceinline__ bool key(int64_t i, unsigned long long& k, uint32_t*) const {
        const int j = (int)(i % g.J);
        const uint32_t r = __ldg(idx + i);
        if (r >= g.rows[j]) return false;
        k = (unsigned long long)(g.row_off[j] + r) + 1ull;
        return true;
    }
};

struct PairKeys {
    const uint64_t* rows;
    uint64_t lo, hi;
    __device__ __forceinline__ bool key(int64_t i, unsigned long long& k, uint32_t* status) const {
        const uint64_t r = __ldg(reinterpret_cast<const unsigned long long*>(rows) + i);
        if (r < lo || r >= hi) {
            if (status) flag(status, ENGRAM_ERR_INDEX);
            return false;
        }
        k = (unsigned long long)r + 1ull;
        return true;
    }
};

template <typename Keys>
__global__ void grad_insert_kernel(Keys src, int64_t n_lookups, unsigned long long* keys, uint32_t* vals,
                                   uint32_t mask, uint64_t* rows_out, unsigned long long* count, uint32_t* status) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_lookups;
         i += (int64_t)gridDim.x * blockDim.x) {
        unsigned long long key;
        if (!src.key(i, key, status)) continue;
        uint32_t h = (uint32_t)mix64(key) & mask;
        bool placed = false;
        for (uint32_t probe = 0; probe <= mask; ++probe) {
            const unsigned long long prev = atomicCAS(keys + h, kEmptyKey, key);
            if (prev == kEmptyKey) {
                const unsigned long long id = atomicAdd(count, 1ull);
                vals[h] = (uint32_t)id;
                rows_out[id] = key - 1ull;
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

// each valid lookup's row id (or 0xFFFFFFFF), and the size of every id's bucket
template <typename Keys>
__global__ void grad_id_kernel(Keys src, int64_t n_lookups, const unsigned long long* __restrict__ keys,
                               const uint32_t* __restrict__ vals, uint32_t mask, uint32_t* __restrict__ lid,
                               uint32_t* bucket) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_lookups;
         i += (int64_t)gridDim.x * blockDim.x) {
        uint32_t id = 0xFFFFFFFFu;
        unsigned long long key;
        if (src.key(i, key, nullptr)) {
            const int64_t h = find_slot(keys, mask, key);
            if (h >= 0) {
                id = vals[h];
                atomicAdd(bucket + id, 1u);
            }
        }
        lid[i] = id;
    }
}

// Exclusive scan of x[0, n) in blocks of kScanBlock: out gets the in-block
// prefix, block_sum[b] the block's total.
__global__ void __launch_bounds__(kScanThreads) scan_block_kernel(const uint32_t* __restrict__ x, int64_t n,
                                                                  uint32_t* __restrict__ out,
                                                                  uint32_t* __restrict__ block_sum) {
    __shared__ uint32_t s_warp[kScanThreads / 32];
    const int64_t base = (int64_t)blockIdx.x * kScanBlock + (int64_t)threadIdx.x * kScanPer;
    uint32_t v[kScanPer];
    uint32_t tsum = 0;
#pragma unroll
    for (int k = 0; k < kScanPer; ++k) {
        v[k] = base + k < n ? x[base + k] : 0u;
        tsum += v[k];
    }
    // inclusive scan of the thread sums within the warp, then across warps
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    uint32_t run = inc - tsum + (warp > 0 ? s_warp[warp - 1] : 0u);
#pragma unroll
    for (int k = 0; k < kScanPer; ++k) {
        if (base + k < n) out[base + k] = run;
        run += v[k];
    }
    if (threadIdx.x == kScanThreads - 1) block_sum[blockIdx.x] = run;
}

__global__ void scan_add_kernel(uint32_t* __restrict__ out, int64_t n, const uint32_t* __restrict__ block_off) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] += block_off[i / kScanBlock];
}

// every lookup's position into its row's segment (order within a segment:
// whatever the atomics give; the reduction orders it)
__global__ void grad_place_kernel(const uint32_t* __restrict__ lid, int64_t n_lookups,
                                  const uint32_t* __restrict__ start, uint32_t* cursor, uint32_t* __restrict__ seg) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_lookups;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t id = lid[i];
        if (id == 0xFFFFFFFFu) continue;
        seg[start[id] + atomicAdd(cursor + id, 1u)] = (uint32_t)i;
    }
}

// Where lookup `pos`'s gradient slice starts.  LookupSlices: slice j of
// dL/de_t for pos = t * J + j.  PairSlices: the pos-th received gradient row.
template <typename T>
struct LookupSlices {
    using Elem = T;
    const T* de;
    int J, D;
    __device__ __forceinline__ const T* at(uint32_t pos) const {
        const int64_t t = pos / J, j = pos - t * J;
        return de + t * ((int64_t)J * D) + j * D;
    }
};

struct PairSlices {
    using Elem = float;
    const float* g;
    int D;
    __device__ __forceinline__ const float* at(uint32_t pos) const { return g + (int64_t)pos * D; }
};

constexpr uint32_t kSmallSeg = 32;   // the longest segment a lane group orders by itself
constexpr int kTile = 2048;          // segment positions staged in shared memory at a time for ranking
constexpr int kPosCap = 4096;        // longest segment whose ordered positions stay in shared memory
constexpr int kStage = 1024;         // 16-byte words of shared memory for the long-segment partial sums
constexpr int kHeavyThreads = 256;

// One group of `gs` lanes per distinct row: gs is a power of two, at least
// the row's count of 16-byte chunks (D*elem/16) and at most 32, so a warp
// takes 32 / gs rows at a time and no lane idles for 128-wide bf16 rows.
// Lane l of a group owns its row's chunks l, l + gs, ...  A row looked up
// once (most rows of a Zipf batch) is its one slice, added to zero in fp32;
// a row looked up k > 1 times has its segment ordered by position (into
// `sorted`, each element's rank = the count of smaller positions) and its
// slices summed in that order, in fp32.  A row looked up more than kSmallSeg
// times (a Zipf-frequent n-gram) is only listed in `heavy`: ordering it
// costs k^2 comparisons, which one CTA does far faster than one lane group.
// Every lane of a group takes the same branches (they share the row), so the
// group's own mask serves its barrier.
template <typename Slices>
__global__ void grad_reduce_kernel(const uint32_t* __restrict__ seg, const uint32_t* __restrict__ start,
                                   const uint32_t* __restrict__ bucket, const unsigned long long* __restrict__ count,
                                   uint32_t* __restrict__ sorted, Slices src, int D, int gs,
                                   float* __restrict__ grad, uint32_t* __restrict__ heavy,
                                   unsigned long long* n_heavy) {
    using T = typename Slices::Elem;
    constexpr int EPC = 16 / sizeof(T);   // elements per 16-byte chunk
    const int lane = threadIdx.x & 31;
    const int grp = lane / gs, gl = lane - grp * gs;
    const unsigned gmask = gs == 32 ? 0xffffffffu : ((1u << gs) - 1u) << (grp * gs);
    const int rpw = 32 / gs;
    const int64_t U = (int64_t)*count;
    const int64_t groups = (((int64_t)gridDim.x * blockDim.x) >> 5) * rpw;
    const int chunks = D / EPC;
    for (int64_t id = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * rpw + grp; id < U; id += groups) {
        const uint32_t s0 = start[id], k = bucket[id];
        float* out = grad + id * D;
        if (k > kSmallSeg) {             // a long segment: a whole CTA orders it (grad_reduce_heavy_kernel)
            if (gl == 0) heavy[atomicAdd(n_heavy, 1ull)] = (uint32_t)id;
            continue;
        }
        if (k == 1) {
            const T* slice = src.at(seg[s0]);
            for (int c = gl; c < chunks; c += gs) {
                float f[EPC];
                Vec<T>::load(slice + c * EPC, f);
                float* o = out + c * EPC;
#pragma unroll
                for (int e = 0; e < EPC; e += 4)
                    *reinterpret_cast<float4*>(o + e) =
                        make_float4(0.f + f[e], 0.f + f[e + 1], 0.f + f[e + 2], 0.f + f[e + 3]);
            }
            continue;
        }
        const uint32_t* in = seg + s0;
        uint32_t* srt = sorted + s0;
        for (uint32_t a = gl; a < k; a += gs) {
            const uint32_t x = in[a];
            uint32_t rank = 0;
            for (uint32_t b = 0; b < k; ++b) rank += in[b] < x;
            srt[rank] = x;
        }
        __syncwarp(gmask);
        for (int c = gl; c < chunks; c += gs) {
            float acc[EPC];
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
            for (uint32_t a = 0; a < k; ++a) {
                float f[EPC];
                Vec<T>::load(src.at(srt[a]) + c * EPC, f);
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[e] += f[e];
            }
            float* o = out + c * EPC;
#pragma unroll
            for (int e = 0; e < EPC; e += 4) *reinterpret_cast<float4*>(o + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
        }
    }
}

// One CTA per listed long segment.  Ordering: every thread ranks its
// positions (the count of smaller positions in the segment, read from
// shared-memory tiles of kTile positions, so any length works); the ordered
// positions go to shared memory when the segment fits (kPosCap), else to
// `sorted`.  Summing, for rows of at most 256 chunks: the CTA's threads are
// `slots` = 256 / chunks running sums per chunk; slot p adds the slices at
// ordered positions p, p + slots, p + 2 slots, ... in that order, in fp32,
// and the slots' sums are then added in slot order (0 + s_0 + s_1 + ...).
// The order is fixed by the row alone, so the result is the same on every
// run; every thread has several loads in flight instead of one thread per
// chunk walking the whole segment.  Wider rows are summed in position order
// straight from memory, one thread per chunk.  All threads of the CTA share
// the row and its length, so every barrier is reached by all of them.
template <typename Slices>
__global__ void __launch_bounds__(kHeavyThreads)
    grad_reduce_heavy_kernel(const uint32_t* __restrict__ seg, const uint32_t* __restrict__ start,
                             const uint32_t* __restrict__ bucket, const uint32_t* __restrict__ heavy,
                             const unsigned long long* __restrict__ n_heavy, uint32_t* sorted, Slices src, int D,
                             float* __restrict__ grad) {
    using T = typename Slices::Elem;
    constexpr int EPC = 16 / sizeof(T);
    __shared__ uint32_t tile[kTile];
    __shared__ uint32_t s_pos[kPosCap];
    __shared__ uint4 stage[kStage];
    const int64_t H = (int64_t)*n_heavy;
    const int chunks = D / EPC;
    const bool staged = chunks <= kHeavyThreads;
    for (int64_t hh = blockIdx.x; hh < H; hh += gridDim.x) {
        const uint32_t id = heavy[hh];
        const uint32_t s0 = start[id], k = bucket[id];
        const uint32_t* in = seg + s0;
        uint32_t* srt = sorted + s0;
        const bool local = k <= (uint32_t)kPosCap;
        for (uint32_t a0 = 0; a0 < k; a0 += blockDim.x) {
            const uint32_t a = a0 + threadIdx.x;
            const uint32_t x = a < k ? in[a] : 0u;
            uint32_t rank = 0;
            for (uint32_t t0 = 0; t0 < k; t0 += kTile) {
                const uint32_t m = min((uint32_t)kTile, k - t0);
                __syncthreads();
                for (uint32_t b = threadIdx.x; b < m; b += blockDim.x) tile[b] = in[t0 + b];
                __syncthreads();
                if (a < k)
                    for (uint32_t b = 0; b < m; ++b) rank += tile[b] < x;
            }
            if (a < k) {
                if (local) s_pos[rank] = x;
                else srt[rank] = x;
            }
        }
        __syncthreads();   // the ordered positions (shared or global) are visible to the block
        float* out = grad + (int64_t)id * D;
        if (staged) {
            // thread (slot p, chunk c) keeps a running sum of chunk c over the
            // positions a = p, p + slots, ... in increasing order; the slots'
            // sums are then added in slot order
            const int slots = (int)blockDim.x / chunks;
            const int p = (int)threadIdx.x / chunks, c = (int)threadIdx.x - p * chunks;
            float acc[EPC];
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
            if (p < slots) {
#pragma unroll 4
                for (uint32_t a = (uint32_t)p; a < k; a += (uint32_t)slots) {
                    float f[EPC];
                    Vec<T>::load(src.at(local ? s_pos[a] : srt[a]) + c * EPC, f);
#pragma unroll
                    for (int e = 0; e < EPC; ++e) acc[e] += f[e];
                }
            }
            float* part = reinterpret_cast<float*>(stage);   // slots x chunks x EPC floats
            if (p < slots) {
#pragma unroll
                for (int e = 0; e < EPC; ++e) part[(p * chunks + c) * EPC + e] = acc[e];
            }
            __syncthreads();
            if ((int)threadIdx.x < chunks) {
                const int cc = (int)threadIdx.x;
                float tot[EPC];
#pragma unroll
                for (int e = 0; e < EPC; ++e) tot[e] = 0.f;
                for (int q = 0; q < slots; ++q) {
#pragma unroll
                    for (int e = 0; e < EPC; ++e) tot[e] += part[(q * chunks + cc) * EPC + e];
                }
#pragma unroll
                for (int e = 0; e < EPC; e += 4)
                    *reinterpret_cast<float4*>(out + cc * EPC + e) = make_float4(tot[e], tot[e + 1], tot[e + 2], tot[e + 3]);
            }
        } else {
            for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
                float acc[EPC];
#pragma unroll
                for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
                for (uint32_t a = 0; a < k; ++a) {
                    float f[EPC];
                    Vec<T>::load(src.at(local ? s_pos[a] : srt[a]) + c * EPC, f);
#pragma unroll
                    for (int e = 0; e < EPC; ++e) acc[e] += f[e];
                }
#pragma unroll
                for (int e = 0; e < EPC; e += 4)
                    *reinterpret_cast<float4*>(out + c * EPC + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
            }
        }
        __syncthreads();
    }
}

// tables[row - first] -= lr * grad for rows in [first, first + n_rows), in
// the tables' dtype (fp32 arithmetic, one rounding to the storage type).  The
// whole table is first = 0, n_rows = sum of M_j; a shard is its own range.
// A group of `gs` lanes per row (the row's 16-byte table chunks rounded up to
// a power of two, at most 32), each lane updating whole 16-byte chunks of the
// row (and reading the matching fp32 gradients as 16-byte vectors).
template <typename T>
__global__ void table_sgd_kernel(const uint64_t* __restrict__ rows, const float* __restrict__ grad,
                                 const unsigned long long* __restrict__ count, int64_t max_rows, uint64_t first,
                                 uint64_t n_rows, int D, int gs, float lr, T* tables, uint32_t* status) {
    constexpr int EPC = 16 / sizeof(T);   // table elements per 16-byte chunk
    const int lane = threadIdx.x & 31;
    const int grp = lane / gs, gl = lane - grp * gs;
    const int rpw = 32 / gs;
    const int64_t U = min((int64_t)*count, max_rows);
    const int64_t groups = (((int64_t)gridDim.x * blockDim.x) >> 5) * rpw;
    const int chunks = D / EPC;
    for (int64_t u = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * rpw + grp; u < U; u += groups) {
        const uint64_t r = rows[u];
        if (r < first || r - first >= n_rows) {
            if (gl == 0) flag(status, ENGRAM_ERR_INDEX);
            continue;
        }
        T* row = tables + (r - first) * D;
        const float* g = grad + u * D;
        for (int c = gl; c < chunks; c += gs) {
            float x[EPC], gv[EPC];
            Vec<T>::load(row + c * EPC, x);
#pragma unroll
            for (int e = 0; e < EPC; e += 4) Vec<float>::load(g + c * EPC + e, gv + e);
#pragma unroll
            for (int e = 0; e < EPC; ++e) x[e] = fmaf(-lr, gv[e], x[e]);
            Vec<T>::store(row + c * EPC, x);
        }
    }
}

// Routing of a rank's (row, gradient) pairs to the shards that own the rows
// (shard g holds global rows [g * per, (g + 1) * per)).  First the count of
// pairs for every shard, then every pair copied into its shard's segment of
// the send buffers (segments in shard order; within a segment, in the order
// the atomics give: the owner's sum does not depend on it, because a rank
// sends every row at most once).
__global__ void route_count_kernel(const uint64_t* __restrict__ rows, const unsigned long long* __restrict__ n_pairs,
                                   int64_t max_rows, uint64_t per, uint64_t total, int n_shards,
                                   unsigned long long* counts, uint32_t* status) {
    __shared__ unsigned int s_cnt[kMaxShards];
    if (threadIdx.x < kMaxShards) s_cnt[threadIdx.x] = 0u;
    __syncthreads();
    const int64_t U = min((int64_t)*n_pairs, max_rows);
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < U; u += (int64_t)gridDim.x * blockDim.x) {
        const uint64_t r = rows[u];
        if (r >= total) {
            flag(status, ENGRAM_ERR_INDEX);
            continue;
        }
        atomicAdd(&s_cnt[(int)(r / per)], 1u);
    }
    __syncthreads();
    if ((int)threadIdx.x < n_shards && s_cnt[threadIdx.x])
        atomicAdd(counts + threadIdx.x, (unsigned long long)s_cnt[threadIdx.x]);
}

// one warp per pair: lane 0 takes the slot, the warp copies the D floats
__global__ void route_place_kernel(const uint64_t* __restrict__ rows, const float* __restrict__ grad,
                                   const unsigned long long* __restrict__ n_pairs, int64_t max_rows, uint64_t per,
                                   uint64_t total, const unsigned long long* __restrict__ counts,
                                   unsigned long long* cursor, int D, uint64_t* __restrict__ send_rows,
                                   float* __restrict__ send_grad) {
    const int lane = threadIdx.x & 31;
    const int64_t U = min((int64_t)*n_pairs, max_rows);
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; u < U; u += warps) {
        const uint64_t r = rows[u];
        if (r >= total) continue;
        const int o = (int)(r / per);
        unsigned long long slot = 0ull;
        if (lane == 0) {
            unsigned long long base = 0ull;
            for (int g = 0; g < o; ++g) base += counts[g];
            slot = base + atomicAdd(cursor + o, 1ull);
            send_rows[slot] = r;
        }
        slot = __shfl_sync(0xffffffffu, slot, 0);
        const float4* in = reinterpret_cast<const float4*>(grad + u * D);
        float4* out = reinterpret_cast<float4*>(send_grad + (int64_t)slot * D);
        for (int q = lane; q < D / 4; q += 32) out[q] = in[q];
    }
}

size_t set_slots(int64_t n_lookups) {
    size_t cap = 1;
    while ((int64_t)cap < 2 * n_lookups) cap <<= 1;
    return cap;
}

struct GradWs {
    unsigned long long* keys;
    uint32_t* vals;
    unsigned long long* count;
    unsigned long long* n_heavy;   // rows handed to grad_reduce_heavy_kernel (their ids go into lid)
    uint32_t* lid;
    uint32_t* bucket;
    uint32_t* start;
    uint32_t* cursor;
    uint32_t* seg;
    uint32_t* sorted;
    uint32_t* bsum1;
    uint32_t* bsum2;
    uint32_t* bsum3;
    size_t bytes;
};

GradWs grad_carve(void* base, int64_t n) {
    GradWs w{};
    char* p = static_cast<char*>(base);
    const size_t cap = set_slots(n);
    const int64_t nb1 = (n + kScanBlock - 1) / kScanBlock;
    const int64_t nb2 = (nb1 + kScanBlock - 1) / kScanBlock;
    auto take = [&](size_t bytes) {
        char* q = p;
        p += align256(bytes);
        return q;
    };
    w.keys = reinterpret_cast<unsigned long long*>(take(cap * 8));
    w.vals = reinterpret_cast<uint32_t*>(take(cap * 4));
    w.count = reinterpret_cast<unsigned long long*>(take(8));
    w.n_heavy = reinterpret_cast<unsigned long long*>(take(8));
    w.lid = reinterpret_cast<uint32_t*>(take((size_t)n * 4));
    w.bucket = reinterpret_cast<uint32_t*>(take((size_t)n * 4));
    w.start = reinterpret_cast<uint32_t*>(take((size_t)n * 4));
    w.cursor = reinterpret_cast<uint32_t*>(take((size_t)n * 4));
    w.seg = reinterpret_cast<uint32_t*>(take((size_t)n * 4));
    w.sorted = reinterpret_cast<uint32_t*>(take((size_t)n * 4));
    w.bsum1 = reinterpret_cast<uint32_t*>(take((size_t)nb1 * 4));
    w.bsum2 = reinterpret_cast<uint32_t*>(take((size_t)nb2 * 4));
    w.bsum3 = reinterpret_cast<uint32_t*>(take(4));
    w.bytes = (size_t)(p - static_cast<char*>(base));
    return w;
}

constexpr int64_t kMaxGradLookups = (int64_t)kScanBlock * kScanBlock;   // two scan levels of 4096

// Clear the scratch, then steps 1-4 over n keyed gradient slices: the
// distinct rows into rows_out, their ordered sums into grad_out, the count
// into *n_unique.  `what` names the caller in errors.
template <typename Keys, typename Slices>
engram_status dedupe_and_sum(engram_ctx* c, const GradWs& w, int64_t n, Keys keys, Slices slices, int D,
                             uint64_t* rows_out, float* grad_out, uint64_t* n_unique, const char* what,
                             cudaStream_t s) {
    const size_t cap = set_slots(std::max<int64_t>(1, n));
    cudaError_t e = cudaMemsetAsync(w.keys, 0, cap * 8, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(w.count, 0, 8, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(w.n_heavy, 0, 8, s);
    if (e == cudaSuccess && n > 0) e = cudaMemsetAsync(w.bucket, 0, (size_t)n * 4, s);
    if (e == cudaSuccess && n > 0) e = cudaMemsetAsync(w.cursor, 0, (size_t)n * 4, s);
    if (e != cudaSuccess) return cuda_fail(what, e);
    if (n > 0) {
        const int threads = 256;
        const int blocks = (int)std::min<int64_t>((n + threads - 1) / threads, (int64_t)c->num_sms * 8);
        const uint32_t mask = (uint32_t)(cap - 1);
        prof_begin(c, s, "grad_dedupe");
        grad_insert_kernel<<<blocks, threads, 0, s>>>(keys, n, w.keys, w.vals, mask, rows_out, w.count, c->d_status);
        grad_id_kernel<<<blocks, threads, 0, s>>>(keys, n, w.keys, w.vals, mask, w.lid, w.bucket);
        prof_end(c, s);
        // segment starts: scan of the bucket sizes (ids >= U have empty buckets)
        const int64_t nb1 = (n + kScanBlock - 1) / kScanBlock;
        const int64_t nb2 = (nb1 + kScanBlock - 1) / kScanBlock;
        prof_begin(c, s, "grad_scan");
        scan_block_kernel<<<(unsigned)nb1, kScanThreads, 0, s>>>(w.bucket, n, w.start, w.bsum1);
        scan_block_kernel<<<(unsigned)nb2, kScanThreads, 0, s>>>(w.bsum1, nb1, w.bsum1, w.bsum2);
        scan_block_kernel<<<1, kScanThreads, 0, s>>>(w.bsum2, nb2, w.bsum2, w.bsum3);
        if (nb2 > 1) scan_add_kernel<<<(unsigned)((nb1 + 255) / 256), 256, 0, s>>>(w.bsum1, nb1, w.bsum2);
        if (nb1 > 1) scan_add_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(w.start, n, w.bsum1);
        prof_end(c, s);
        prof_begin(c, s, "grad_place");
        grad_place_kernel<<<blocks, threads, 0, s>>>(w.lid, n, w.start, w.cursor, w.seg);
        prof_end(c, s);
        prof_begin(c, s, "grad_reduce");
        // lanes per row: the row's 16-byte chunks rounded up to a power of two, at most a warp
        const int chunks = D / (16 / (int)sizeof(typename Slices::Elem));
        int gs = 1;
        while (gs < chunks && gs < 32) gs <<= 1;
        const int rblocks = (int)std::min<int64_t>((n + 7) / 8, (int64_t)c->num_sms * 16);
        // lid (one entry per lookup, free once the lookups are placed) lists the long segments
        grad_reduce_kernel<<<rblocks, 256, 0, s>>>(w.seg, w.start, w.bucket, w.count, w.sorted, slices, D, gs,
                                                   grad_out, w.lid, w.n_heavy);
        prof_end(c, s);
        prof_begin(c, s, "grad_reduce_long");
        grad_reduce_heavy_kernel<<<c->num_sms * 4, kHeavyThreads, 0, s>>>(w.seg, w.start, w.bucket, w.lid,
                                                                         w.n_heavy, w.sorted, slices, D, grad_out);
        prof_end(c, s);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(n_unique, w.count, 8, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(what, e);
    return ENGRAM_OK;
}

uint64_t total_rows(const engram_ctx* c) {
    uint64_t total = 0;
    for (int j = 0; j < c->J; ++j) total += c->cfg.rows[j];
    return total;
}

template <typename T>
void launch_sgd(engram_ctx* c, const uint64_t* rows, const float* grad, const uint64_t* n_unique, int64_t max_rows,
                uint64_t first, uint64_t n_rows, void* tables, float lr, cudaStream_t s) {
    const int chunks = c->cfg.row_dim / (16 / (int)sizeof(T));
    int gs = 1;   // lanes per row: the row's 16-byte chunks rounded up to a power of two, at most a warp
    while (gs < chunks && gs < 32) gs <<= 1;
    const int blocks = (int)std::min<int64_t>((max_rows + 7) / 8, (int64_t)c->num_sms * 16);
    table_sgd_kernel<T><<<blocks, 256, 0, s>>>(rows, grad, reinterpret_cast<const unsigned long long*>(n_unique),
                                               max_rows, first, n_rows, c->cfg.row_dim, gs, lr,
                                               static_cast<T*>(tables), c->d_status);
}

}  // namespace
}  // namespace engram

using namespace engram;

extern "C" {

size_t engram_table_grad_workspace_bytes(const engram_ctx* c, int64_t n_tok) {
    if (!c || n_tok < 0) return 0;
    return grad_carve(nullptr, std::max<int64_t>(1, n_tok * c->J)).bytes;
}

engram_status engram_table_grad(engram_ctx* c, const uint32_t* idx, int64_t n_tok, const void* d_e,
                                uint64_t* rows_out, float* grad_out, uint64_t* n_unique, void* workspace,
                                size_t workspace_bytes, cudaStream_t s) {
    if (!c) return inval("null context");
    if (n_tok < 0) return inval("n_tok must be >= 0");
    const int64_t n = n_tok * c->J;
    if (n > kMaxGradLookups) return inval("n_tok * J must be at most 2^24 lookups");
    if (c->cfg.dtype == ENGRAM_FP8) {
        set_error("engram_table_grad: FP8 tables are not trained here");
        return ENGRAM_E_UNSUPPORTED;
    }
    if (!n_unique) return inval("null n_unique pointer");
    if (n > 0 && (!idx || !d_e || !rows_out || !grad_out || !workspace)) return inval("null tensor pointer");
    if (!aligned16(d_e) || !aligned16(grad_out)) return inval("d_e and grad_out must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return inval("workspace must be 256-byte aligned");
    GradWs w = grad_carve(workspace, std::max<int64_t>(1, n));
    if (workspace_bytes < w.bytes) return ENGRAM_E_NOMEM;
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    GradGeo g{};
    for (int j = 0; j < c->J; ++j) {
        g.row_off[j] = c->gp.row_off[j];
        g.rows[j] = c->gp.rows[j];
    }
    g.J = c->J;
    const int D = c->cfg.row_dim;
    if (c->cfg.dtype == ENGRAM_BF16)
        return dedupe_and_sum(c, w, n, LookupKeys{idx, g},
                              LookupSlices<__nv_bfloat16>{static_cast<const __nv_bfloat16*>(d_e), c->J, D}, D,
                              rows_out, grad_out, n_unique, "table gradient", s);
    return dedupe_and_sum(c, w, n, LookupKeys{idx, g}, LookupSlices<float>{static_cast<const float*>(d_e), c->J, D},
                          D, rows_out, grad_out, n_unique, "table gradient", s);
}

engram_status engram_table_sgd(engram_ctx* c, const uint64_t* rows, const float* grad, const uint64_t* n_unique,
                               int64_t max_rows, void* tables, float lr, cudaStream_t s) {
    if (!c) return inval("null context");
    if (max_rows < 0) return inval("max_rows must be >= 0");
    if (max_rows == 0) return ENGRAM_OK;
    if (!rows || !grad || !n_unique || !tables) return inval("null tensor pointer");
    if (!aligned16(tables) || !aligned16(grad)) return inval("tables and grad must be 16-byte aligned");
    if (c->cfg.dtype == ENGRAM_FP8) {
        set_error("engram_table_sgd: FP8 tables are not trained here");
        return ENGRAM_E_UNSUPPORTED;
    }
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    prof_begin(c, s, "table_sgd");
    if (c->cfg.dtype == ENGRAM_BF16)
        launch_sgd<__nv_bfloat16>(c, rows, grad, n_unique, max_rows, 0, total_rows(c), tables, lr, s);
    else
        launch_sgd<float>(c, rows, grad, n_unique, max_rows, 0, total_rows(c), tables, lr, s);
    prof_end(c, s);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ENGRAM_OK : cuda_fail("table update launch", e);
}

size_t engram_grad_route_workspace_bytes(const engram_ctx* c) {
    return c ? (size_t)256 : 0;
}

engram_status engram_grad_route(engram_ctx* c, int32_t n_shards, const uint64_t* rows, const float* grad,
                                const uint64_t* n_pairs, int64_t max_rows, uint64_t* send_rows, float* send_grad,
                                int64_t* send_counts, void* workspace, size_t workspace_bytes, cudaStream_t s) {
    if (!c) return inval("null context");
    if (n_shards < 1 || n_shards > kMaxShards) return inval("n_shards must be in 1..16");
    if (max_rows < 0) return inval("max_rows must be >= 0");
    if (max_rows > kMaxGradLookups) return inval("max_rows must be at most 2^24 pairs");
    if (!n_pairs || !send_counts || !workspace) return inval("null count, send_counts or workspace pointer");
    if (max_rows > 0 && (!rows || !grad || !send_rows || !send_grad)) return inval("null tensor pointer");
    if (!aligned16(grad) || !aligned16(send_grad)) return inval("grad and send_grad must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return inval("workspace must be 256-byte aligned");
    if (workspace_bytes < engram_grad_route_workspace_bytes(c)) return ENGRAM_E_NOMEM;
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    const uint64_t total = total_rows(c);
    const uint64_t per = (total + (uint64_t)n_shards - 1) / (uint64_t)n_shards;
    unsigned long long* counts = reinterpret_cast<unsigned long long*>(send_counts);
    unsigned long long* cursor = static_cast<unsigned long long*>(workspace);
    prof_reset(c);
    cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)n_shards * 8, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(cursor, 0, (size_t)n_shards * 8, s);
    if (e != cudaSuccess) return cuda_fail("gradient routing: clearing the counts", e);
    if (max_rows == 0) return ENGRAM_OK;
    const int D = c->cfg.row_dim;
    prof_begin(c, s, "grad_route");
    const int cblocks = (int)std::min<int64_t>((max_rows + 255) / 256, (int64_t)c->num_sms * 4);
    route_count_kernel<<<cblocks, 256, 0, s>>>(rows, reinterpret_cast<const unsigned long long*>(n_pairs), max_rows,
                                               per, total, n_shards, counts, c->d_status);
    const int pblocks = (int)std::min<int64_t>((max_rows + 7) / 8, (int64_t)c->num_sms * 16);
    route_place_kernel<<<pblocks, 256, 0, s>>>(rows, grad, reinterpret_cast<const unsigned long long*>(n_pairs),
                                               max_rows, per, total, counts, cursor, D, send_rows, send_grad);
    prof_end(c, s);
    e = cudaGetLastError();
    return e == cudaSuccess ? ENGRAM_OK : cuda_fail("gradient routing launches", e);
}

size_t engram_grad_combine_workspace_bytes(const engram_ctx* c, int64_t n_pairs) {
    if (!c || n_pairs < 0) return 0;
    return grad_carve(nullptr, std::max<int64_t>(1, n_pairs)).bytes;
}

engram_status engram_grad_combine(engram_ctx* c, int32_t n_shards, int32_t shard, const uint64_t* pair_rows,
                                  const float* pair_grad, int64_t n_pairs, uint64_t* rows_out, float* grad_out,
                                  uint64_t* n_unique, void* workspace, size_t workspace_bytes, cudaStream_t s) {
    if (!c) return inval("null context");
    int64_t lo = 0, cnt = 0;
    engram_status st = engram_shard_range(c, n_shards, shard, &lo, &cnt);
    if (st != ENGRAM_OK) return st;
    if (n_pairs < 0) return inval("n_pairs must be >= 0");
    if (n_pairs > kMaxGradLookups) return inval("n_pairs must be at most 2^24");
    if (!n_unique || !workspace) return inval("null n_unique or workspace pointer");
    if (n_pairs > 0 && (!pair_rows || !pair_grad || !rows_out || !grad_out)) return inval("null tensor pointer");
    if (!aligned16(pair_grad) || !aligned16(grad_out)) return inval("pair_grad and grad_out must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return inval("workspace must be 256-byte aligned");
    GradWs w = grad_carve(workspace, std::max<int64_t>(1, n_pairs));
    if (workspace_bytes < w.bytes) return ENGRAM_E_NOMEM;
    st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    const int D = c->cfg.row_dim;
    return dedupe_and_sum(c, w, n_pairs, PairKeys{pair_rows, (uint64_t)lo, (uint64_t)(lo + cnt)},
                          PairSlices{pair_grad, D}, D, rows_out, grad_out, n_unique, "gradient combine", s);
}

engram_status engram_shard_sgd(engram_ctx* c, int32_t n_shards, int32_t shard, const uint64_t* rows,
                               const float* grad, const uint64_t* n_unique, int64_t max_rows, void* shard_table,
                               float lr, cudaStream_t s) {
    if (!c) return inval("null context");
    int64_t lo = 0, cnt = 0;
    engram_status st = engram_shard_range(c, n_shards, shard, &lo, &cnt);
    if (st != ENGRAM_OK) return st;
    if (max_rows < 0) return inval("max_rows must be >= 0");
    if (max_rows == 0) return ENGRAM_OK;
    if (!rows || !grad || !n_unique || (cnt > 0 && !shard_table)) return inval("null tensor pointer");
    if (!aligned16(shard_table) || !aligned16(grad)) return inval("shard_table and grad must be 16-byte aligned");
    if (c->cfg.dtype == ENGRAM_FP8) {
        set_error("engram_shard_sgd: FP8 tables are not trained here");
        return ENGRAM_E_UNSUPPORTED;
    }
    st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    prof_begin(c, s, "table_sgd");
    if (c->cfg.dtype == ENGRAM_BF16)
        launch_sgd<__nv_bfloat16>(c, rows, grad, n_unique, max_rows, (uint64_t)lo, (uint64_t)cnt, shard_table, lr, s);
    else
        launch_sgd<float>(c, rows, grad, n_unique, max_rows, (uint64_t)lo, (uint64_t)cnt, shard_table, lr, s);
    prof_end(c, s);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ENGRAM_OK : cuda_fail("shard update launch", e);
}

}  // extern "C"
