// Internal declarations shared by the Engram CUDA kernels and the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "engram.h"

namespace engram {

constexpr int kMaxTables = ENGRAM_MAX_TABLES;
constexpr int kGroup = ENGRAM_PART_GROUP;   // channels per gate-partial group
constexpr int kMaxConv = 8;

// Hash configuration passed by value to the hash kernel (about 1.2 KB of
// kernel parameters; dynamic indexing reads the constant bank).
struct HashParams {
    uint64_t mult[kMaxTables][4];
    uint64_t recip[kMaxTables];   // floor((2^64 - 1) / rows[j]) for the Barrett reduction
    uint32_t rows[kMaxTables];
    int32_t orders[4];
    int32_t n_orders;
    int32_t K;
    int32_t J;
    int32_t max_order;
    int32_t V;
    int32_t Vc;
};

// Table geometry passed by value to the gather kernel.
struct GatherParams {
    int64_t row_off[kMaxTables];   // first row of table j in the back-to-back table buffer
    uint32_t rows[kMaxTables];
    int32_t J;
    int32_t chunks_per_row;        // 16-byte chunks per table row
};

// Tables split across GPUs by global row (table j's row r is global row
// row_off[j] + r): shard g holds global rows [bound[g], bound[g + 1]) at
// base[g], a device pointer valid on the launching GPU (its own memory, or
// another GPU's mapped into this one's address space).
constexpr int kMaxShards = 16;
struct ShardParams {
    const uint4* base[kMaxShards];
    int64_t bound[kMaxShards + 1];
    int32_t n;
};

// x mod m for a 64-bit x and a 32-bit m, by Barrett's reduction (P. Barrett,
// CRYPTO '86) with recip = floor((2^64 - 1) / m): q = floor(x * recip / 2^64)
// undershoots floor(x / m) by at most 2, so at most two subtractions follow.
__device__ __forceinline__ uint32_t mod_u64(uint64_t x, uint32_t m, uint64_t recip) {
    const uint64_t q = __umul64hi(x, recip);
    uint64_t r = x - q * (uint64_t)m;
    if (r >= m) r -= m;
    if (r >= m) r -= m;
    return (uint32_t)r;
}

// Decode (one new position per sequence, at most 256 sequences, bf16, one
// branch): both projections in one kernel, K split over clusters of four
// CTAs, partials added through distributed shared memory, the rows' gate
// partials and v [n][d] fp32 to the workspace; then the gate and conv
// kernel, a programmatic dependent, which writes alpha and Y and updates the
// conv state in place.
bool decode_tc_supported(int64_t n, int32_t L, int32_t d_mem, int32_t d, int32_t M, bool f8);
int32_t decode_tc_max_tiles(int32_t d);   // channel tiles per row at most (the gate partials' width)
cudaError_t launch_decode_kv(const void* e, int32_t n, int32_t d_mem, const void* h, const void* Wk, const void* Wv,
                             const float* gq, const float* gk, int32_t d, float* part, float* v, uint32_t* status,
                             int num_sms, int stall, bool pdl, cudaStream_t s);
cudaError_t launch_decode_conv(const float* v, const float* part, int32_t n, const void* h, const float* conv_w,
                               int32_t d, float eps, float* alpha, float* alpha_out, float* state, void* y,
                               int32_t add_residual, int num_sms, bool pdl, cudaStream_t s);

// ---------------------------------------------------------------- launches
// Each returns cudaGetLastError() of its launch.
cudaError_t launch_remap(const int32_t* tok, int64_t n, const int32_t* P, int32_t V, int32_t* canon,
                         uint32_t* status, cudaStream_t s);
cudaError_t launch_hash(const int32_t* ids, const int32_t* P, int32_t B, int32_t T, int64_t stride,
                        int32_t t_begin, uint32_t* idx, const HashParams& hp, uint32_t* status,
                        cudaStream_t s);
cudaError_t launch_gather(const uint32_t* idx, int64_t n_tok, const void* tables, const GatherParams& gp,
                          void* e_cat, uint32_t* status, int num_sms, cudaStream_t s);
// launch_hash followed by launch_gather in one kernel (indices still written to idx)
cudaError_t launch_retrieve(const int32_t* ids, const int32_t* P, int32_t B, int32_t T, int64_t stride,
                            int32_t t_begin, const HashParams& hp, const GatherParams& gp, const void* tables,
                            uint32_t* idx, void* e_cat, uint32_t* status, int num_sms, cudaStream_t s);
// the same with the table rows read from the shards of sp (plain, L2-only
// loads, which reach peer memory over NVLink)
cudaError_t launch_retrieve_sharded(const int32_t* ids, const int32_t* P, int32_t B, int32_t T, int64_t stride,
                                    int32_t t_begin, const HashParams& hp, const GatherParams& gp,
                                    const ShardParams& sp, uint32_t* idx, void* e_cat, uint32_t* status,
                                    int num_sms, cudaStream_t s);
// CUDA-core projection (fp32 or bf16 operands, fp32 accumulation); v in fp32
cudaError_t launch_project_simt(bool bf16, const void* e, int64_t n_tok, int32_t d_mem, const void* h,
                                const void* Wk, const void* Wv, const float* gq, const float* gk, int32_t d,
                                float* v, float* part, cudaStream_t s);
// tcgen05 kernels (bf16 operands, fp32 accumulation in tensor memory); both
// return cudaErrorNotSupported when the shape does not fit their tiling.
// f8: e and W in FP8 E4M3 (kind::f8f6f4), else bf16
bool project_tc_supported(int64_t n_tok, int32_t d_mem, int32_t d, bool f8 = false);
cudaError_t launch_project_tc(const void* e, int64_t n_tok, int32_t d_mem, const void* h, const void* Wk,
                              const void* Wv, const float* gq, const float* gk, int32_t d, float* v,
                              float* part, uint32_t* status, int num_sms, cudaStream_t s);
// Multi-branch (M in 1..4): Wk is the M branches' W_K stacked [M*d][d_mem];
// h, gq, gk, alpha, Y, the conv history and its scratch are [M][...] of the
// single-branch shapes; e and W_V are shared.
// Pass 1: k -> gate partials [n_tok][G][4] and alpha [n_tok] (reduced by the
// CTA that completes each 128-row band; band_count holds ceil(n_tok/128)
// counters that must be zero on entry and are zero again on exit).
// pdl: launched as a programmatic dependent of the kernel just before it on
// the stream (which produced e); every thread waits for that kernel's
// completion before any global access, then lets the next pass launch.
cudaError_t launch_gate_k_tc(const void* e, int64_t n_tok, int32_t d_mem, const void* h, const void* Wk,
                             const float* gq, const float* gk, int32_t d, float eps, float* part, int* band_count,
                             float* alpha, float* alpha_out, uint32_t* status, int num_sms, int stall, bool pdl,
                             cudaStream_t s, int32_t M = 1, bool f8 = false, const float* kscale = nullptr);
// Pass 2: v -> gate (alpha from pass 1), causal conv, residual, Y (fused
// epilogue, conv width 4).  When state is non-null the new history goes to
// state_next ([B][w-1][d] fp32 scratch) and launch_state_merge folds it into
// state afterwards.  pdl: launched as a programmatic dependent of pass 1,
// which must be the kernel just before it on the stream; the operand loads
// and MMAs start on SMs as pass 1's CTAs leave, and the epilogue waits for
// pass 1's completion before it reads alpha.
cudaError_t launch_vconv_tc(const void* e, int32_t B, int32_t L, int32_t d_mem, const void* h, const void* Wv,
                            const float* conv_w, int32_t d, int32_t w, const float* alpha, const float* state,
                            float* state_next, int32_t state_tr, void* y, int32_t add_residual, uint32_t* status,
                            int num_sms, bool pdl, cudaStream_t s, int32_t M = 1, bool f8 = false,
                            const float* vscale = nullptr);
// conv history [B][w-1][d] -> the sequence-minor [w-1][d][B] that decode-shaped
// value passes read (state_tr), and the merge of such a pass's new history
// back into the caller's [B][w-1][d]
cudaError_t launch_state_to_tr(const float* state, float* state_t, int32_t B, int32_t w, int32_t d, cudaStream_t s);
cudaError_t launch_state_merge_tr(float* state, const float* state_next_t, int32_t B, int32_t L, int32_t w, int32_t d,
                                  cudaStream_t s);
cudaError_t launch_state_merge(float* state, const float* state_next, int32_t B, int32_t L, int32_t w, int32_t d,
                               int num_sms, cudaStream_t s);
// gate + conv from an fp32 v (CUDA cores)
cudaError_t launch_gate_conv(bool bf16, const float* v, const float* part, const void* h, const float* conv_w,
                             int32_t B, int32_t L, int32_t d, int32_t w, float eps, float* state, void* y,
                             float* alpha_out, int32_t add_residual, uint32_t* status, cudaStream_t s);

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ void flag(uint32_t* status, uint32_t bit) {
    if (status) atomicOr(status, bit);
}

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// fp32 -> bf16 round-to-nearest-even (cuda_bf16 intrinsic), two values packed
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

// 16-byte vector <-> floats
template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void load(const float* p, float* out) {
        float4 q = *reinterpret_cast<const float4*>(p);
        out[0] = q.x; out[1] = q.y; out[2] = q.z; out[3] = q.w;
    }
    __device__ __forceinline__ static void store(float* p, const float* in) {
        *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out) {
        uint4 q = *reinterpret_cast<const uint4*>(p);
        out[0] = bf16_lo(q.x); out[1] = bf16_hi(q.x);
        out[2] = bf16_lo(q.y); out[3] = bf16_hi(q.y);
        out[4] = bf16_lo(q.z); out[5] = bf16_hi(q.z);
        out[6] = bf16_lo(q.w); out[7] = bf16_hi(q.w);
    }
    __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* in) {
        uint4 q;
        q.x = pack_bf16x2(in[0], in[1]);
        q.y = pack_bf16x2(in[2], in[3]);
        q.z = pack_bf16x2(in[4], in[5]);
        q.w = pack_bf16x2(in[6], in[7]);
        *reinterpret_cast<uint4*>(p) = q;
    }
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float& dst, float x) { dst = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16& dst, float x) { dst = __float2bfloat16_rn(x); }

}  // namespace engram
