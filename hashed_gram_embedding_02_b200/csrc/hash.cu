// Tokenizer compression and multi-head n-gram hashing.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": x'_t = P(x_t), suffix
// n-grams g_{t,n} = (x'_{t-n+1}, ..., x'_t), K hash heads phi_{n,k} per order
// mapping g_{t,n} to an index of table E_{n,k} whose size M_{n,k} is prime;
// phi is a lightweight multiplicative-XOR hash.  The exact form used here:
//   phi_{n,k}(g) = (XOR_{j<n} (s_j + 1) * a_{n,k,j} mod 2^64) mod M_{n,k},
// s_j = x'_{t-j}, s_j = V' (PAD) before the sequence start.
//
// A CTA takes 256/J consecutive output rows (b, t).  It first stages each
// row's window of canonical ids (x'_t, x'_{t-1}, ..., PAD before the start;
// reading into [0, t_begin) for decode) in shared memory, one (row, j) pair
// per thread, then hashes one (row, table) pair per thread, so consecutive
// threads write consecutive indices.
#include "common.cuh"

namespace engram {

namespace {

constexpr int kHashThreads = 256;

__device__ __forceinline__ int32_t canon_at(const int32_t* ids, const int32_t* P, int64_t pos,
                                            int32_t V, int32_t Vc, uint32_t* status) {
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

__global__ void __launch_bounds__(kHashThreads)
hash_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ P, int32_t B, int32_t T,
            int64_t stride, int32_t t_begin, uint32_t* __restrict__ idx, const HashParams hp, int rows_per_cta,
            uint32_t* status) {
    __shared__ int32_t s_win[kHashThreads][4];   // [row][j]: canonical id at t - j (PAD before the start)
    // per-table constants in shared memory (lanes index them by table; divergent
    // indexing of kernel parameters would serialise on the constant cache)
    __shared__ uint64_t s_mult[kMaxTables][4];
    __shared__ uint64_t s_recip[kMaxTables];
    __shared__ uint32_t s_rows[kMaxTables];
    __shared__ int32_t s_order[kMaxTables];
    for (int k = threadIdx.x; k < hp.J * 4; k += kHashThreads) s_mult[k >> 2][k & 3] = hp.mult[k >> 2][k & 3];
    for (int k = threadIdx.x; k < hp.J; k += kHashThreads) {
        s_recip[k] = hp.recip[k];
        s_rows[k] = hp.rows[k];
        s_order[k] = hp.orders[k / hp.K];
    }
    const int64_t L = (int64_t)T - t_begin;
    const int64_t n = (int64_t)B * L;
    const int64_t row0 = (int64_t)blockIdx.x * rows_per_cta;
    const int R = (int)min((int64_t)rows_per_cta, n - row0);
    const int W = hp.max_order;

    // 1. the n-gram windows of this CTA's rows, one (row, j) pair per thread
    for (int k = threadIdx.x; k < R * W; k += kHashThreads) {
        const int rr = k / W, j = k - rr * W;
        const int64_t row = row0 + rr;
        const int64_t b = row / L;
        const int64_t t = t_begin + (row - b * L);
        s_win[rr][j] = (t - j >= 0) ? canon_at(ids, P, b * stride + t - j, hp.V, hp.Vc, status) : hp.Vc;
    }
    __syncthreads();

    // 2. one (row, table) pair per thread; consecutive threads write
    //    consecutive words of idx
    const int J = hp.J;
    for (int k = threadIdx.x; k < R * J; k += kHashThreads) {
        const int rr = k / J, jt = k - rr * J;
        const int n_o = s_order[jt];
        bool invalid = false;
        uint64_t x = 0;
        for (int j = 0; j < n_o; ++j) {
            const int32_t sj = s_win[rr][j];
            invalid |= (sj < 0);
            x ^= (uint64_t)(uint32_t)(sj + 1) * s_mult[jt][j];
        }
        idx[(row0 + rr) * J + jt] = invalid ? ENGRAM_INVALID_INDEX : mod_u64(x, s_rows[jt], s_recip[jt]);
    }
}

__global__ void remap_kernel(const int32_t* __restrict__ tok, int64_t n, const int32_t* __restrict__ P,
                             int32_t V, int32_t* __restrict__ canon, uint32_t* status) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t x = tok[i];
        int32_t c = -1;
        if (x < 0 || x >= V) {
            flag(status, ENGRAM_ERR_TOKEN);
        } else {
            c = __ldg(P + x);
        }
        canon[i] = c;
    }
}

}  // namespace

cudaError_t launch_remap(const int32_t* tok, int64_t n, const int32_t* P, int32_t V, int32_t* canon,
                         uint32_t* status, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (n + threads - 1) / threads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    remap_kernel<<<(unsigned)blocks, threads, 0, s>>>(tok, n, P, V, canon, status);
    return cudaGetLastError();
}

cudaError_t launch_hash(const int32_t* ids, const int32_t* P, int32_t B, int32_t T, int64_t stride,
                        int32_t t_begin, uint32_t* idx, const HashParams& hp, uint32_t* status,
                        cudaStream_t s) {
    const int64_t n = (int64_t)B * (T - t_begin);
    if (n == 0) return cudaSuccess;
    const int rows_per_cta = kHashThreads / hp.J;          // J <= 32, so at least 8
    const int64_t blocks = (n + rows_per_cta - 1) / rows_per_cta;
    hash_kernel<<<(unsigned)blocks, kHashThreads, 0, s>>>(ids, P, B, T, stride, t_begin, idx, hp, rows_per_cta,
                                                          status);
    return cudaGetLastError();
}

}  // namespace engram
