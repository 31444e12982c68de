// Tokenizer compression and multi-head n-gram hashing.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": x'_t = P(x_t), suffix
// n-grams g_{t,n} = (x'_{t-n+1}, ..., x'_t), K hash heads phi_{n,k} per order
// mapping g_{t,n} to an index of table E_{n,k} whose size M_{n,k} is prime;
// phi is a lightweight multiplicative-XOR hash.  The exact form used here:
//   phi_{n,k}(g) = (XOR_{j<n} (s_j + 1) * a_{n,k,j} mod 2^64) mod M_{n,k},
// s_j = x'_{t-j}, s_j = V' (PAD) before the sequence start.
//
// One thread per output row (b, t).  A warp covers consecutive positions of a
// sequence, so the ids of the n-1 predecessors come from neighbouring lanes
// by __shfl_up_sync; only lanes whose predecessor belongs to another warp (or
// to the context before t_begin) read it from memory.  Indices are staged in
// shared memory and written out as one contiguous block per CTA.
#include "common.cuh"

namespace engram {

namespace {

constexpr int kHashThreads = 128;

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
            int64_t stride, int32_t t_begin, uint32_t* __restrict__ idx, const HashParams hp,
            uint32_t* status) {
    extern __shared__ uint32_t s_idx[];  // [kHashThreads][J]
    const int64_t L = (int64_t)T - t_begin;
    const int64_t n = (int64_t)B * L;
    const int64_t row0 = (int64_t)blockIdx.x * kHashThreads;
    const int64_t row = row0 + threadIdx.x;
    const bool active = row < n;
    const int lane = threadIdx.x & 31;
    int64_t b = 0, tl = 0;
    if (active) {
        b = row / L;
        tl = row - b * L;
    }
    const int64_t t = t_begin + tl;
    const int64_t base = b * stride;

    const int32_t mine = active ? canon_at(ids, P, base + t, hp.V, hp.Vc, status) : -1;
    int32_t s[4];
    s[0] = mine;
#pragma unroll
    for (int j = 1; j < 4; ++j) {
        const int32_t nb = __shfl_up_sync(0xffffffffu, mine, j);
        if (j < hp.max_order) {
            if (lane >= j && tl >= j) {
                s[j] = nb;                       // row - j: same sequence, previous lane
            } else if (t - j >= 0) {
                s[j] = active ? canon_at(ids, P, base + t - j, hp.V, hp.Vc, status) : -1;
            } else {
                s[j] = hp.Vc;                    // PAD before the sequence start
            }
        } else {
            s[j] = 0;
        }
    }

    if (active) {
        uint32_t* out = s_idx + threadIdx.x * hp.J;
        for (int o = 0; o < hp.n_orders; ++o) {
            const int n_o = hp.orders[o];
            bool invalid = false;
            for (int j = 0; j < n_o; ++j) invalid |= (s[j] < 0);
            for (int k = 0; k < hp.K; ++k) {
                const int jt = o * hp.K + k;
                uint32_t r = ENGRAM_INVALID_INDEX;
                if (!invalid) {
                    uint64_t x = 0;
                    for (int j = 0; j < n_o; ++j) x ^= (uint64_t)(uint32_t)(s[j] + 1) * hp.mult[jt][j];
                    r = (uint32_t)(x % (uint64_t)hp.rows[jt]);
                }
                out[jt] = r;
            }
        }
    }
    __syncthreads();
    // coalesced write of this CTA's rows (contiguous in idx)
    const int64_t rows_here = min((int64_t)kHashThreads, n - row0);
    const int64_t words = rows_here * hp.J;
    uint32_t* dst = idx + row0 * hp.J;
    for (int64_t i = threadIdx.x; i < words; i += kHashThreads) dst[i] = s_idx[i];
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
    const int64_t blocks = (n + kHashThreads - 1) / kHashThreads;
    const size_t smem = (size_t)kHashThreads * hp.J * sizeof(uint32_t);
    hash_kernel<<<(unsigned)blocks, kHashThreads, smem, s>>>(ids, P, B, T, stride, t_begin, idx, hp, status);
    return cudaGetLastError();
}

}  // namespace engram
