// Gather and concatenation of the retrieved table rows into e_t.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": all retrieved
// embeddings are concatenated into the memory vector e_t (QbitAI repost: all
// orders and all heads).  A copy: e_cat[t][j*D:(j+1)*D] = E_j[idx[t][j]].
//
// HBM-bound.  The output row of a token is J*D elements written as 16-byte
// chunks by consecutive threads (fully coalesced stores); each thread owns
// one chunk position (table j, chunk c) and walks a batch of tokens, issuing
// all of its batch's table loads before any store so that several
// independent 16-byte loads per thread are in flight.  A table row is
// D*elem bytes (128 B or 256 B here), read by cpr consecutive lanes.
#include "common.cuh"

namespace engram {

namespace {

constexpr int kTokBatch = 4;

__global__ void __launch_bounds__(256)
gather_kernel(const uint32_t* __restrict__ idx, int64_t n_tok, const uint4* __restrict__ tables,
              const GatherParams gp, uint4* __restrict__ e_cat, uint32_t* status) {
    const int J = gp.J;
    const int cpr = gp.chunks_per_row;
    const int per_tok = J * cpr;
    for (int ch = threadIdx.x; ch < per_tok; ch += blockDim.x) {
        const int j = ch / cpr;
        const int c = ch - j * cpr;
        const uint4* tb = tables + gp.row_off[j] * cpr + c;
        const uint32_t M = gp.rows[j];
        for (int64_t t0 = (int64_t)blockIdx.x * kTokBatch; t0 < n_tok; t0 += (int64_t)gridDim.x * kTokBatch) {
            uint32_t r[kTokBatch];
#pragma unroll
            for (int u = 0; u < kTokBatch; ++u) {
                const int64_t t = t0 + u;
                r[u] = t < n_tok ? __ldg(idx + t * J + j) : ENGRAM_INVALID_INDEX;
            }
            uint4 val[kTokBatch];
#pragma unroll
            for (int u = 0; u < kTokBatch; ++u) {
                if (r[u] < M) {
                    val[u] = __ldg(tb + (int64_t)r[u] * cpr);
                } else {
                    val[u] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int u = 0; u < kTokBatch; ++u) {
                const int64_t t = t0 + u;
                if (t < n_tok) {
                    if (r[u] >= M && r[u] != ENGRAM_INVALID_INDEX) flag(status, ENGRAM_ERR_INDEX);
                    e_cat[t * per_tok + ch] = val[u];
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_gather(const uint32_t* idx, int64_t n_tok, const void* tables, const GatherParams& gp,
                          void* e_cat, uint32_t* status, int num_sms, cudaStream_t s) {
    if (n_tok == 0) return cudaSuccess;
    const int per_tok = gp.J * gp.chunks_per_row;
    const int threads = per_tok >= 256 ? 256 : ((per_tok + 31) / 32) * 32;
    const int64_t want = (n_tok + kTokBatch - 1) / kTokBatch;
    const int64_t cap = (int64_t)num_sms * (4096 / threads);
    const int64_t blocks = want < cap ? want : cap;
    gather_kernel<<<(unsigned)blocks, threads, 0, s>>>(idx, n_tok, static_cast<const uint4*>(tables), gp,
                                                       static_cast<uint4*>(e_cat), status);
    return cudaGetLastError();
}

}  // namespace engram
