// Retrieval in one kernel: remap, suffix n-grams, the J hash heads and the
// gather of the J table rows into e_t, for the forward.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": x'_t = P(x_t); suffix
// n-grams g_{t,n}; K heads phi_{n,k} per order index prime-sized tables;
// the retrieved rows are concatenated into e_t (QbitAI repost: all orders and
// all heads).  The hash form is the one of hash.cu; this kernel fuses it with
// the gather of gather.cu so the indices never leave the SM before use (they
// are still written out, for inspection through the workspace).
//
// A CTA of 256 threads takes R = 256 / J rows: it stages their windows of
// canonical ids, hashes one (row, table) pair per thread into shared memory,
// then copies the R x J table rows as 16-byte chunks, each thread issuing a
// batch of independent loads before its stores, consecutive threads on
// consecutive chunks of e_cat (coalesced stores).
//
// Sharded tables (the pages' training layout, "DeepSeek AI II" digest,
// section "DeepSeek Engram", and the Synced repost, "System efficiency":
// the tables are split over the GPUs and the accessed rows are brought to
// the GPU that needs them).  The SHARDED variant resolves, in the hash
// phase, each (row, table) pair to the shard that owns the row and to the
// row's address there; the gather phase then reads every row straight from
// its owner's memory (over NVLink for another GPU's shard) into this GPU's
// e_cat.  The all-to-all of indices and rows becomes one-sided reads inside
// the kernel that needs them, and every remote row lands in local HBM
// before the projections use it.
#include "common.cuh"

namespace engram {

namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 4;   // 16-byte loads in flight per thread

__device__ __forceinline__ int32_t canon_id(const int32_t* ids, const int32_t* P, int64_t pos, int32_t V, int32_t Vc,
                                            uint32_t* status) {
    int32_t x = ids[pos];
    if (P) {
        if (x < 0 || x >= V) {
            flag(status, ENGRAM_ERR_TOKEN);
            return -1;
        }
        x = __ldg(P + x);
    }
    if (x < 0 || x >= Vc) {
        flag(status, ENGRAM_ERR_CANON);
        return -1;
    }
    return x;
}

template <bool SHARDED>
__global__ void __launch_bounds__(kThreads, 8)
retrieve_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ P, int32_t B, int32_t T, int64_t stride,
                int32_t t_begin, const HashParams hp, const GatherParams gp, const uint4* __restrict__ tables,
                const ShardParams sp, uint32_t* __restrict__ idx, uint4* __restrict__ e_cat, int rows_per_cta,
                int cpr_shift, int pr_shift, uint32_t* status) {
    __shared__ int32_t s_win[kThreads][4];
    __shared__ uint32_t s_idx[kThreads];
    // SHARDED: the first chunk of each (row, table) pair's table row, or null
    __shared__ const uint4* s_src[SHARDED ? kThreads : 1];
    __shared__ const uint4* s_base[SHARDED ? kMaxShards : 1];
    __shared__ int64_t s_bound[SHARDED ? kMaxShards + 1 : 1];
    // per-table constants in shared memory: lanes index them by table, and
    // divergent indexing of kernel parameters would serialise on the
    // constant cache
    __shared__ uint64_t s_mult[kMaxTables][4];
    __shared__ uint64_t s_recip[kMaxTables];
    __shared__ int64_t s_off[kMaxTables];
    __shared__ uint32_t s_rows[kMaxTables];
    __shared__ int32_t s_order[kMaxTables];
    // the key pass that follows may launch now: its CTAs take SMs as these
    // leave and wait for this grid's completion before they read e_cat
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t L = (int64_t)T - t_begin;
    const int64_t n = (int64_t)B * L;
    const int64_t row0 = (int64_t)blockIdx.x * rows_per_cta;
    const int R = (int)min((int64_t)rows_per_cta, n - row0);
    const int W = hp.max_order;
    const int J = hp.J;
    for (int k = threadIdx.x; k < J * 4; k += kThreads) s_mult[k >> 2][k & 3] = hp.mult[k >> 2][k & 3];
    for (int k = threadIdx.x; k < J; k += kThreads) {
        s_recip[k] = hp.recip[k];
        s_off[k] = gp.row_off[k];
        s_rows[k] = hp.rows[k];
        s_order[k] = hp.orders[k / hp.K];
    }
    if constexpr (SHARDED) {
        for (int k = threadIdx.x; k < sp.n; k += kThreads) s_base[k] = sp.base[k];
        for (int k = threadIdx.x; k <= sp.n; k += kThreads) s_bound[k] = sp.bound[k];
    }

    // 1. n-gram windows (PAD before the sequence start)
    for (int k = threadIdx.x; k < R * W; k += kThreads) {
        const int rr = k / W, j = k - rr * W;
        const int64_t row = row0 + rr;
        const int64_t b = row / L;
        const int64_t t = t_begin + (row - b * L);
        s_win[rr][j] = (t - j >= 0) ? canon_id(ids, P, b * stride + t - j, hp.V, hp.Vc, status) : hp.Vc;
    }
    __syncthreads();

    // 2. hash heads, one (row, table) pair per thread
    for (int k = threadIdx.x; k < R * J; k += kThreads) {
        const int rr = k / J, jt = k - rr * J;
        const int n_o = s_order[jt];
        bool invalid = false;
        uint64_t x = 0;
        for (int j = 0; j < n_o; ++j) {
            const int32_t sj = s_win[rr][j];
            invalid |= (sj < 0);
            x ^= (uint64_t)(uint32_t)(sj + 1) * s_mult[jt][j];
        }
        const uint32_t v = invalid ? ENGRAM_INVALID_INDEX : mod_u64(x, s_rows[jt], s_recip[jt]);
        s_idx[k] = v;
        idx[(row0 + rr) * J + jt] = v;
        if constexpr (SHARDED) {
            const uint4* src = nullptr;
            if (v < s_rows[jt]) {
                const int64_t g_row = s_off[jt] + v;
                int g = 0;
                while (g + 1 < sp.n && g_row >= s_bound[g + 1]) ++g;
                if (g_row >= s_bound[g] && g_row < s_bound[g + 1])
                    src = s_base[g] + (g_row - s_bound[g]) * gp.chunks_per_row;
            }
            s_src[k] = src;
        }
    }
    __syncthreads();

    // 3. gather: chunk f = (row, table, chunk) in e_cat order
    const int cpr = gp.chunks_per_row;
    const int per_row = J * cpr;
    const int total = R * per_row;
    uint4* out = e_cat + row0 * per_row;
    for (int f0 = threadIdx.x; f0 < total; f0 += kThreads * kBatch) {
        uint4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int f = f0 + u * kThreads;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (f < total) {
                // shifts when the row and table widths in chunks are powers of two
                const int rr = pr_shift >= 0 ? f >> pr_shift : f / per_row;
                const int rem = f - rr * per_row;
                const int jt = cpr_shift >= 0 ? rem >> cpr_shift : rem / cpr;
                const int c = rem - jt * cpr;
                const uint32_t r = s_idx[rr * J + jt];
                if constexpr (SHARDED) {
                    const uint4* src = s_src[rr * J + jt];
                    if (src) v[u] = __ldcg(src + c);
                    else if (r != ENGRAM_INVALID_INDEX) flag(status, ENGRAM_ERR_INDEX);
                } else {
                    if (r < s_rows[jt]) v[u] = __ldg(tables + (s_off[jt] + r) * cpr + c);
                    else if (r != ENGRAM_INVALID_INDEX) flag(status, ENGRAM_ERR_INDEX);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int f = f0 + u * kThreads;
            if (f < total) out[f] = v[u];
        }
    }
}

}  // namespace

namespace {

int log2_or_neg(int v) {
    if (v <= 0 || (v & (v - 1))) return -1;
    int k = 0;
    while ((1 << k) < v) ++k;
    return k;
}

template <bool SHARDED>
cudaError_t launch_retrieve_impl(const int32_t* ids, const int32_t* P, int32_t B, int32_t T, int64_t stride,
                                 int32_t t_begin, const HashParams& hp, const GatherParams& gp, const void* tables,
                                 const ShardParams& sp, uint32_t* idx, void* e_cat, uint32_t* status, int num_sms,
                                 cudaStream_t s) {
    const int64_t n = (int64_t)B * (T - t_begin);
    if (n == 0) return cudaSuccess;
    // 256 / J rows per CTA, or fewer when the batch is small (decode: a few
    // hundred rows), so that the grid still spreads over every SM: the
    // kernel is a chain of dependent loads, and a CTA's rows run one batch
    // of loads after another
    int rows_per_cta = kThreads / hp.J;
    const int64_t spread = (n + 2 * (int64_t)num_sms - 1) / (2 * (int64_t)num_sms);
    if (spread < rows_per_cta) rows_per_cta = (int)(spread < 1 ? 1 : spread);
    const int64_t blocks = (n + rows_per_cta - 1) / rows_per_cta;
    const int cpr_shift = log2_or_neg(gp.chunks_per_row);
    const int pr_shift = log2_or_neg(hp.J * gp.chunks_per_row);
    retrieve_kernel<SHARDED><<<(unsigned)blocks, kThreads, 0, s>>>(
        ids, P, B, T, stride, t_begin, hp, gp, static_cast<const uint4*>(tables), sp, idx, static_cast<uint4*>(e_cat),
        rows_per_cta, cpr_shift, pr_shift, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_retrieve(const int32_t* ids, const int32_t* P, int32_t B, int32_t T, int64_t stride,
                            int32_t t_begin, const HashParams& hp, const GatherParams& gp, const void* tables,
                            uint32_t* idx, void* e_cat, uint32_t* status, int num_sms, cudaStream_t s) {
    ShardParams none{};
    return launch_retrieve_impl<false>(ids, P, B, T, stride, t_begin, hp, gp, tables, none, idx, e_cat, status,
                                       num_sms, s);
}

cudaError_t launch_retrieve_sharded(const int32_t* ids, const int32_t* P, int32_t B, int32_t T, int64_t stride,
                                    int32_t t_begin, const HashParams& hp, const GatherParams& gp,
                                    const ShardParams& sp, uint32_t* idx, void* e_cat, uint32_t* status, int num_sms,
                                    cudaStream_t s) {
    return launch_retrieve_impl<true>(ids, P, B, T, stride, t_begin, hp, gp, nullptr, sp, idx, e_cat, status,
                                      num_sms, s);
}

}  // namespace engram
