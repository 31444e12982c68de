// Decode passes: the key and value projections with the gate and the conv,
// for a call that computes one new position per sequence (L = 1) for at most
// 256 sequences.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": k_t = W_K e_t and
// v_t = W_V e_t; the scalar gate alpha_t from the RMS-normalised h_t and k_t;
// v~_t = alpha_t v_t; the short causal depthwise conv over v~ whose three
// earlier inputs of each sequence come from the caller's conv state; the
// output v~ + SiLU(conv), plus h when the residual is added.
//
// At decode the projections are 256-row GEMMs.  The 128-row tiles of the
// prefill passes give 40-60 CTAs there, each streaming a full K extent of
// operands (about 1 MB) through its ring, and the passes are bound by that
// per-SM stream.  Here each pass spreads the work over the SMs three ways:
//
//   - a cluster of kSplit = 4 CTAs splits K (d_mem): CTA r of the cluster
//     multiplies its quarter of the 64-wide k-blocks, for every row (up to
//     256, in two TMEM accumulators of 128 rows) and the cluster's BN
//     channels, so a CTA streams a quarter of the K extent;
//   - the four partial sums are added through distributed shared memory:
//     each CTA stores every accumulator row into the shared memory of the CTA
//     that owns the row (rows r*RP .. r*RP+RP-1 belong to CTA r, RP = rows/4),
//     and the owner adds the four partials in rank order, so the sum does
//     not depend on timing;
//   - the owner finishes its RP rows x BN channels with threads running along
//     the channels: the h, conv-state and output accesses are row pieces, and
//     the conv state is updated in place (one thread per (sequence, channel)).
//
// The grid is d / BN clusters (BN = 64, 80 or 128, the narrowest that still
// lets every cluster be resident at once).  The key pass reduces each row's
// gate partials across its clusters through a per-row-block counter, the
// last cluster to finish a block computing alpha.  Both passes issue their W
// loads before waiting for the kernel they depend on (the retrieval, the key
// pass), so the weight stream overlaps it.
//
// Every mbarrier wait is bounded.  A CTA whose wait runs out flags
// ENGRAM_ERR_TIMEOUT and votes to abort; after the first cluster barrier every
// CTA of the cluster reads the votes, and on any abort the cluster stores no
// partials and writes no output.  The CTA drains its own copies and MMAs
// (bounded) before it frees its TMEM and leaves.
#include "tc.cuh"

namespace engram {

namespace {

constexpr int DEC_K = 0;
constexpr int DEC_V = 1;
constexpr int kSplit = 4;             // CTAs per cluster (K split)
constexpr int kDecThreads = 256;
constexpr int kDecStages = 4;
constexpr int kDecRows = 256;         // rows per call (two 128-row accumulators)
constexpr int kDecRp = kDecRows / kSplit;   // rows owned by a CTA at most
constexpr int kAccStride = 128;       // TMEM column of the second accumulator
constexpr int kTmemCols = 256;
constexpr int kABytes = 128 * 128;    // one 128-row x 64-element bf16 box

template <int BN>
struct DecGeo {
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = 2 * kABytes + B_BYTES;
    static constexpr int RING = kDecStages * STAGE_BYTES;
    static constexpr int RS = BN + 4;   // floats per staged row (16-byte pad: conflict-free row-per-lane stores)
    // after the MMAs the ring holds this CTA's partial sums, [256][RS], and
    // the three peers' partials of the rows it owns, [3][64][RS]
    static constexpr int STAGE_OFF = 0;
    static constexpr int RECV_OFF = kDecRows * RS * 4;
    static constexpr int EXCH_BYTES = RECV_OFF + (kSplit - 1) * kDecRp * RS * 4;
    static constexpr int CONST_BYTES = BN * 16;   // conv taps (value pass) or gains (key pass)
    static constexpr int SMEM_BYTES = RING + 1024 + CONST_BYTES + 1024;
    static constexpr int ITEMS = kDecRp * (BN / 4) / kDecThreads;   // value items per thread at most
    static_assert(EXCH_BYTES <= RING, "the partials reuse the operand ring");
    static_assert(BN % 16 == 0 && BN <= kAccStride, "UMMA N and the accumulator spacing");
    static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
    static_assert(kDecRp * (BN / 4) % kDecThreads == 0, "whole value items per thread");
};

struct __align__(8) DecBarriers {
    uint64_t full[kDecStages];
    uint64_t empty[kDecStages];
    uint64_t tfull;
    uint64_t rfull;   // the peers' partials of this CTA's rows have landed
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;   // this CTA's vote (read by the cluster after the first barrier)
    int issued;       // k-block stages whose loads were issued
    int consumed;     // stages the MMAs have taken
    int last;         // key pass: this CTA completed its row block's partials
};

struct DecParams {
    const __nv_bfloat16* w;        // this pass's weights [d][d_mem]
    const __nv_bfloat16* w_next;   // key pass: W_V, brought into L2 for the value pass; else null
    const __nv_bfloat16* h;        // [n][d]
    const float* gq;               // [d] or null
    const float* gk;               // [d] or null
    const float* conv_w;           // [d][4]
    float* state;                  // [n][3][d] conv history, updated in place, or null (zero history)
    const float* alpha;            // value pass: [n]
    float* alpha_w;                // key pass: [n]
    float* alpha_out;              // key pass: caller's copy, or null
    float4* part;                  // key pass: [n][n_ct] (sum g h k, sum k^2, sum h^2, 0)
    int* band_count;               // key pass: [kSplit] per row block (zero on entry, zero on exit)
    __nv_bfloat16* y;              // value pass: [n][d]
    uint32_t* status;
    int n, d, d_mem, n_ct;
    int add_residual;
    float eps;
    int stall;                     // test hook: CTA 0 announces its first stage and never loads it
};

__device__ __forceinline__ bool dec_wait(uint64_t* bar, uint32_t parity, DecBarriers* sb, uint32_t* status) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(a, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&sb->abort_flag)) return false;
        if (clock64() - t0 > kWaitCycles) {
            flag(status, ENGRAM_ERR_TIMEOUT);
            *reinterpret_cast<volatile int*>(&sb->abort_flag) = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void dec_wait_drain(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(smem_u32(bar), parity) && clock64() - t0 < kWaitCycles) {
    }
}

__device__ __forceinline__ int dec_atomic_add_acq_rel(int* addr, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ float dec_tanh(float x) {
    float r;
    asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// bytes from this CTA's shared memory to another CTA of the cluster, counted
// on a barrier of that CTA (both addresses and the size multiples of 16)
__device__ __forceinline__ void bulk_s2cluster(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                               uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst_cluster),
        "r"(src), "r"(bytes), "r"(bar_cluster)
        : "memory");
}

__device__ __forceinline__ int owned_rows(int n, int rank, int rp) {
    const int r = n - rank * rp;
    return r < 0 ? 0 : (r < rp ? r : rp);
}

// While the MMAs run, warps 2-7 stage the per-channel constants in shared
// memory (g_q g_k for the key pass, the four conv taps for the value pass)
// and bring into L2 the k-blocks of the CTA's W slice that the first round of
// stages does not hold and (key pass) the same slice of W_V, which the value
// pass CTA with the same cluster rank and channel tile will read.  Offsets
// and lengths are multiples of 16 bytes (d_mem a multiple of 64).
template <int MODE, int BN>
__device__ __forceinline__ void dec_prefetch(const DecParams& p, int rank, int rp, int ct, int kb0, int nkb,
                                             float* s_const, int t, int nt) {
    const int c0 = ct * BN;
    if (MODE == DEC_K) {
        for (int c = t; c < BN; c += nt)
            s_const[c] = (p.gq ? __ldg(p.gq + c0 + c) : 1.f) * (p.gk ? __ldg(p.gk + c0 + c) : 1.f);
    } else {
        for (int c = t; c < BN; c += nt)
            reinterpret_cast<float4*>(s_const)[c] = __ldg(reinterpret_cast<const float4*>(p.conv_w) + c0 + c);
    }
    for (int c = t; c < BN; c += nt) {
        const int64_t wrow = (int64_t)(c0 + c) * p.d_mem + (int64_t)kb0 * 64;
        if (nkb > kDecStages) prefetch_l2(p.w + wrow + kDecStages * 64, (uint32_t)(nkb - kDecStages) * 128u);
        if (p.w_next) prefetch_l2(p.w_next + wrow, (uint32_t)nkb * 128u);
    }
}

// The four partial sums of an owned row, in rank order: this CTA's own from
// its staging rows, the peers' from the receive slots.
template <int BN>
struct PartRows {
    const float* stage;
    const float* recv;
    int rank, rp;
    __device__ __forceinline__ const float* row(int src, int lr) const {
        constexpr int RS = DecGeo<BN>::RS;
        if (src == rank) return stage + (rank * rp + lr) * RS;
        const int slot = src < rank ? src : src - 1;
        return recv + (slot * rp + lr) * RS;
    }
};

// The epilogues' global inputs, loaded into registers before the
// accumulators complete, so their latency hides behind the MMAs and the
// exchange.  Key pass: warp w holds h of rows w, w + 8, .. of the CTA's
// block, lane l channels l, l + 32, ..
template <int BN>
struct KIn {
    static constexpr int NJ = (BN + 31) / 32;
    static constexpr int NW = kDecThreads / 32;
    static constexpr int RPW = kDecRp / NW;   // rows per warp at most (8)
    float hv[RPW][NJ];
    __device__ __forceinline__ void load(const DecParams& p, int rank, int rp, int ct) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int lr = warp + NW * i, row = rank * rp + lr;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int c = lane + 32 * j;
                hv[i][j] = (lr < rp && row < p.n && c < BN)
                               ? __bfloat162float(p.h[(int64_t)row * p.d + ct * BN + c])
                               : 0.f;
            }
        }
    }
};

// Value pass: the thread's items (four channels of a row each): history and h.
template <int BN>
struct VIn {
    static constexpr int NQ = BN / 4;
    static constexpr int NI = DecGeo<BN>::ITEMS;
    float4 h0[NI], h1[NI], h2[NI];
    uint2 hq[NI];
    __device__ __forceinline__ void load(const DecParams& p, int rank, int rp, int ct) {
        const int items = rp * NQ;
#pragma unroll
        for (int b = 0; b < NI; ++b) {
            const int it = b * kDecThreads + threadIdx.x;
            const int lr = it / NQ, q4 = it - lr * NQ;
            const int row = rank * rp + lr;
            h0[b] = h1[b] = h2[b] = make_float4(0.f, 0.f, 0.f, 0.f);
            hq[b] = make_uint2(0u, 0u);
            if (it < items && row < p.n) {
                const int64_t c = ct * BN + 4 * q4;
                if (p.state) {
                    const float4* st = reinterpret_cast<const float4*>(p.state + (int64_t)row * 3 * p.d + c);
                    h0[b] = __ldcs(st);
                    h1[b] = __ldcs(st + p.d / 4);
                    h2[b] = __ldcs(st + p.d / 2);
                }
                if (p.add_residual) hq[b] = __ldcs(reinterpret_cast<const uint2*>(p.h + (int64_t)row * p.d + c));
            }
        }
    }
};

// Gate partials of the CTA's rows over its BN channels, then the row block's
// alpha by the last of the n_ct clusters to finish the block.
template <int BN>
__device__ __forceinline__ void dec_epilogue_k(const DecParams& p, const PartRows<BN>& pr, const KIn<BN>& in,
                                               const float* s_g, int rank, int rp, int ct, DecBarriers* sb) {
    constexpr int NJ = KIn<BN>::NJ;
    constexpr int NW = KIn<BN>::NW;
    constexpr int RPW = KIn<BN>::RPW;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const auto& hv = in.hv;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int lr = warp + NW * i, row = rank * rp + lr;
        if (lr >= rp || row >= p.n) break;
        float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int c = lane + 32 * j;
            if (c < BN) {
                float k = pr.row(0, lr)[c];
#pragma unroll
                for (int src = 1; src < kSplit; ++src) k += pr.row(src, lr)[c];
                s_qk = fmaf(s_g[c] * hv[i][j], k, s_qk);
                s_kk = fmaf(k, k, s_kk);
                s_hh = fmaf(hv[i][j], hv[i][j], s_hh);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s_qk += __shfl_xor_sync(0xffffffffu, s_qk, o);
            s_kk += __shfl_xor_sync(0xffffffffu, s_kk, o);
            s_hh += __shfl_xor_sync(0xffffffffu, s_hh, o);
        }
        if (lane == 0) p.part[(int64_t)row * p.n_ct + ct] = make_float4(s_qk, s_kk, s_hh, 0.f);
    }
    // the CTA barrier orders every thread's partials before thread 0's
    // release at device scope (the count), and its acquire before every
    // thread's reads of the other clusters' partials
    __syncthreads();
    if (threadIdx.x == 0) sb->last = dec_atomic_add_acq_rel(p.band_count + rank, 1) == p.n_ct - 1;
    __syncthreads();
    if (!sb->last) return;
    // every cluster's partials of this row block are visible: four threads
    // per row reduce a quarter of the channel tiles each, then combine
    const int lr = threadIdx.x >> 2, qq = threadIdx.x & 3;
    const int row = rank * rp + lr;
    const bool live = lr < rp && row < p.n;
    float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
    if (live) {
        const float4* src = p.part + (int64_t)row * p.n_ct;
#pragma unroll 8
        for (int t = qq; t < p.n_ct; t += 4) {
            const float4 v = __ldcg(src + t);
            s_qk += v.x;
            s_kk += v.y;
            s_hh += v.z;
        }
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
        s_qk += __shfl_xor_sync(0xffffffffu, s_qk, o);
        s_kk += __shfl_xor_sync(0xffffffffu, s_kk, o);
        s_hh += __shfl_xor_sync(0xffffffffu, s_hh, o);
    }
    if (live && qq == 0) {
        const float inv_d = 1.f / (float)p.d;
        const float rh = sqrtf(s_hh * inv_d + p.eps);
        const float rk = sqrtf(s_kk * inv_d + p.eps);
        const float a = 1.f / (1.f + expf(-(s_qk / (rh * rk)) * rsqrtf((float)p.d)));
        p.alpha_w[row] = a;
        if (p.alpha_out) p.alpha_out[row] = a;
    }
    if (threadIdx.x == 0) p.band_count[rank] = 0;
}

// Gate, conv over the history in the caller's state, SiLU, residual; four
// channels per item, consecutive threads on consecutive channels of a row.
template <int BN>
__device__ __forceinline__ void dec_epilogue_v(const DecParams& p, const PartRows<BN>& pr, const VIn<BN>& in,
                                               const float4* s_w, int rank, int rp, int ct) {
    constexpr int NQ = VIn<BN>::NQ;
    constexpr int NI = VIn<BN>::NI;
    const int c0 = ct * BN;
    const int items = rp * NQ;
    const int dq = p.d / 4;
    const auto &h0 = in.h0, &h1 = in.h1, &h2 = in.h2;
    const auto& hq = in.hq;
    float a[NI];
#pragma unroll
    for (int b = 0; b < NI; ++b) {
        const int it = b * kDecThreads + threadIdx.x;
        const int row = rank * rp + it / NQ;
        a[b] = (it < items && row < p.n) ? __ldg(p.alpha + row) : 0.f;
    }
#pragma unroll
    for (int b = 0; b < NI; ++b) {
        const int it = b * kDecThreads + threadIdx.x;
        const int lr = it / NQ, q4 = it - lr * NQ;
        const int row = rank * rp + lr;
        if (it >= items || row >= p.n) continue;
        const int64_t c = c0 + 4 * q4;
        float4 v = *reinterpret_cast<const float4*>(pr.row(0, lr) + 4 * q4);
#pragma unroll
        for (int src = 1; src < kSplit; ++src) {
            const float4 u = *reinterpret_cast<const float4*>(pr.row(src, lr) + 4 * q4);
            v.x += u.x;
            v.y += u.y;
            v.z += u.z;
            v.w += u.w;
        }
        const float x[4] = {a[b] * v.x, a[b] * v.y, a[b] * v.z, a[b] * v.w};
        const float s0[4] = {h0[b].x, h0[b].y, h0[b].z, h0[b].w};
        const float s1[4] = {h1[b].x, h1[b].y, h1[b].z, h1[b].w};
        const float s2[4] = {h2[b].x, h2[b].y, h2[b].z, h2[b].w};
        const float hv[4] = {bf16_lo(hq[b].x), bf16_hi(hq[b].x), bf16_lo(hq[b].y), bf16_hi(hq[b].y)};
        float yv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            // tap j multiplies the input j positions back: x_t, then the
            // history rows 2, 1, 0 (oldest last)
            const float4 w = s_w[4 * q4 + e];
            float u = w.x * x[e];
            u = fmaf(w.y, s2[e], u);
            u = fmaf(w.z, s1[e], u);
            u = fmaf(w.w, s0[e], u);
            const float hu = 0.5f * u;
            yv[e] = x[e] + fmaf(hu, dec_tanh(hu), hu) + hv[e];
        }
        *reinterpret_cast<uint2*>(p.y + (int64_t)row * p.d + c) =
            make_uint2(pack_bf16x2(yv[0], yv[1]), pack_bf16x2(yv[2], yv[3]));
        if (p.state) {
            float4* st = reinterpret_cast<float4*>(p.state + (int64_t)row * 3 * p.d + c);
            st[0] = h1[b];
            st[dq] = h2[b];
            st[2 * dq] = make_float4(x[0], x[1], x[2], x[3]);
        }
    }
}

template <int MODE, int BN>
__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(kDecThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const DecParams p) {
    using GE = DecGeo<BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024 - (raw & 1023)) & 1023);   // 1024-byte aligned ring
    const uint32_t ring = smem_u32(smem);
    DecBarriers* sb = reinterpret_cast<DecBarriers*>(smem + GE::RING);
    float* s_const = reinterpret_cast<float*>(smem + GE::RING + 1024);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_rank();
    const int ct = (int)blockIdx.x / kSplit;   // channel tile of the cluster
    const int nr = p.n > 128 ? 2 : 1;          // 128-row accumulators in use
    const int rp = nr * 128 / kSplit;          // rows owned by each CTA of the cluster
    // this CTA's k-blocks (64 elements each)
    const int kb_total = p.d_mem / 64;
    const int kb0 = rank * kb_total / kSplit, kb1 = (rank + 1) * kb_total / kSplit;
    const int nkb = kb1 - kb0;
    const uint32_t stage_tx = (uint32_t)(nr * kABytes + GE::B_BYTES);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&sb->full[s], 1);
            mbar_init(&sb->empty[s], 1);
        }
        mbar_init(&sb->tfull, 1);
        mbar_init(&sb->rfull, 1);
        mbar_init(&sb->drain, 1);
        sb->abort_flag = 0;
        sb->issued = 0;
        sb->consumed = 0;
        sb->last = 0;
        mbar_fence_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sb->tmem_base)),
                     "n"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sb->tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            const int pre = nkb < kDecStages ? nkb : kDecStages;
            auto load_b = [&](int j) {
                const int s = j % kDecStages;
                mbar_arrive_expect_tx(&sb->full[s], stage_tx);
                if (p.stall && j == 0 && blockIdx.x == 0) return;   // bounded-wait test: never loaded
                tma_load_2d(&map_b, ring + s * GE::STAGE_BYTES + 2 * kABytes, &sb->full[s], (kb0 + j) * 64, ct * BN);
            };
            auto load_a = [&](int j) {
                const int s = j % kDecStages;
                if (p.stall && j == 0 && blockIdx.x == 0) return;
                for (int rt = 0; rt < nr; ++rt)
                    tma_load_2d(&map_a, ring + s * GE::STAGE_BYTES + rt * kABytes, &sb->full[s], (kb0 + j) * 64,
                                rt * 128);
            };
            // the weights do not depend on the kernel before this one: their
            // first stages stream while it finishes.  The key pass reads e,
            // which the retrieval before it writes; the value pass reads e
            // only after the key pass, which waited for the retrieval, let
            // it launch
            for (int j = 0; j < pre; ++j) load_b(j);
            if (MODE == DEC_K) grid_dep_wait();
            for (int j = 0; j < pre; ++j) load_a(j);
            sb->issued = pre;
            for (int j = pre; j < nkb; ++j) {
                const int s = j % kDecStages;
                if (!dec_wait(&sb->empty[s], ((uint32_t)(j / kDecStages) & 1u) ^ 1u, sb, p.status)) break;
                load_b(j);
                load_a(j);
                sb->issued = j + 1;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            bool ok = true;
            for (int j = 0; j < nkb; ++j) {
                const int s = j % kDecStages;
                if (!dec_wait(&sb->full[s], (uint32_t)(j / kDecStages) & 1u, sb, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = ring + s * GE::STAGE_BYTES;
                const uint64_t db = smem_desc_sw128(a_addr + 2 * kABytes);
                for (int rt = 0; rt < nr; ++rt) {
                    const uint64_t da = smem_desc_sw128(a_addr + rt * kABytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16<BN>(tmem_base + (uint32_t)(rt * kAccStride), da + (uint64_t)(kk * 2),
                                      db + (uint64_t)(kk * 2), (j | kk) != 0);
                }
                umma_commit(&sb->empty[s]);
                sb->consumed = j + 1;
            }
            if (ok) umma_commit(&sb->tfull);
        }
        __syncwarp();
    } else {
        dec_prefetch<MODE, BN>(p, rank, rp, ct, kb0, nkb, s_const, threadIdx.x - 64, kDecThreads - 64);
    }
    // key pass: the value pass may launch once every thread of every CTA is
    // past the retrieval (warp 0 follows its lane 0, which waited above)
    if (MODE == DEC_K) {
        if (warp != 0) grid_dep_wait();
        grid_dep_launch_dependents();
    }

    // ---------------- accumulators complete: stage them in this CTA's ring
    const bool ok = nkb > 0 && dec_wait(&sb->tfull, 0, sb, p.status);
    const int cta_abort = __syncthreads_or(!ok || sb->abort_flag);
    tc_fence_after();
    float* stage = reinterpret_cast<float*>(smem + GE::STAGE_OFF);
    float* recv = reinterpret_cast<float*>(smem + GE::RECV_OFF);
    if (!cta_abort) {
        // warp w reads TMEM lanes 32 (w % 4) .. +31 and channel half w / 4;
        // one row per lane, padded rows: the stores hit distinct banks
        constexpr int HALF = BN / 2;
        constexpr int NCH = HALF / 8;
        const int q = warp & 3, col0 = (warp >> 2) * HALF;
        for (int rt = 0; rt < nr; ++rt) {
            const int row = rt * 128 + q * 32 + lane;
            uint32_t v[NCH][8];
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch)
                tmem_ld8(tmem_base + (uint32_t)(rt * kAccStride + col0 + ch * 8) + ((uint32_t)(q * 32) << 16), v[ch]);
            tmem_wait_ld();
            uint4* dst = reinterpret_cast<uint4*>(stage + row * GE::RS + col0);
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                dst[2 * ch] = make_uint4(v[ch][0], v[ch][1], v[ch][2], v[ch][3]);
                dst[2 * ch + 1] = make_uint4(v[ch][4], v[ch][5], v[ch][6], v[ch][7]);
            }
        }
        // the bulk copies below read the staged rows through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // the epilogue's global inputs, in flight during the exchange (issued
    // after the proxy fence, which would otherwise wait for them)
    KIn<BN> kin;
    VIn<BN> vin;
    if (MODE == DEC_K) kin.load(p, rank, rp, ct);
    else vin.load(p, rank, rp, ct);
    if (threadIdx.x == 0) {
        sb->abort_flag = cta_abort;
        // the three peers' copies of the rows this CTA owns (padded rows)
        mbar_arrive_expect_tx(&sb->rfull, (uint32_t)((kSplit - 1) * owned_rows(p.n, rank, rp) * GE::RS * 4));
    }
    tc_fence_before();
    // barrier 1: every CTA's MMAs have finished reading its ring, which now
    // receives the peers' partials; the abort votes are visible cluster-wide
    __syncwarp();
    cluster_sync_all();
    int any_abort = 0;
#pragma unroll
    for (int r = 0; r < kSplit; ++r) any_abort |= ld_remote_s32(peer_addr(&sb->abort_flag, (uint32_t)r));

    bool have = false;
    if (!any_abort) {
        // one bulk copy per peer: the staged rows the peer owns (contiguous,
        // padded) into its receive slot for this rank
        const int t = threadIdx.x;
        if (t < kSplit - 1) {
            const int o = t < rank ? t : t + 1;
            const int rows = owned_rows(p.n, o, rp);
            if (rows > 0) {
                const int slot = rank < o ? rank : rank - 1;
                bulk_s2cluster(peer_addr(recv + slot * rp * GE::RS, (uint32_t)o), smem_u32(stage + o * rp * GE::RS),
                               (uint32_t)(rows * GE::RS * 4), peer_addr(&sb->rfull, (uint32_t)o));
            }
        }
        have = dec_wait(&sb->rfull, 0, sb, p.status);
    }
    // barrier 2: every copy has landed, so no CTA's staged rows are read any more
    __syncwarp();
    cluster_sync_all();

    if (!any_abort && __syncthreads_and(have)) {
        const PartRows<BN> pr{stage, recv, rank, rp};
        if (MODE == DEC_K) {
            dec_epilogue_k<BN>(p, pr, kin, s_const, rank, rp, ct, sb);
        } else {
            grid_dep_wait();   // alpha comes from the key pass
            dec_epilogue_v<BN>(p, pr, vin, reinterpret_cast<const float4*>(s_const), rank, rp, ct);
        }
    } else if (cta_abort) {
        // this CTA stopped early: wait out the copies and MMAs it issued
        if (warp == 0 && lane == 0)
            for (int j = sb->consumed; j < sb->issued; ++j)
                dec_wait_drain(&sb->full[j % kDecStages], (uint32_t)(j / kDecStages) & 1u);
        if (warp == 1 && lane == 0) {
            umma_commit(&sb->drain);
            dec_wait_drain(&sb->drain, 0);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "n"(kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------- host side

// clusters of kSplit CTAs of the largest decode kernel that the device holds at once
int resident_clusters(int num_sms) {
    static int cached[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    auto kernel = decode_tc_kernel<DEC_V, 80>;
    int mc = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DecGeo<80>::SMEM_BYTES) ==
        cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(num_sms / kSplit * kSplit), 1, 1);
        cfg.blockDim = dim3(kDecThreads, 1, 1);
        cfg.dynamicSmemBytes = DecGeo<80>::SMEM_BYTES;
        if (cudaOccupancyMaxActiveClusters(&mc, kernel, &cfg) != cudaSuccess) mc = 0;
    }
    cudaGetLastError();
    if (mc < 1) mc = num_sms / kSplit;
    if (dev < 64) cached[dev] = mc;
    return mc;
}

// 64-channel tiles when all their clusters are resident at once, else
// 80-channel tiles where d allows them (fewer clusters), else 64 in several
// waves (clusters never wait on one another)
int pick_dec_bn(int32_t d, int num_sms) {
    const int cap = resident_clusters(num_sms);
    if (d / 64 <= cap || d % 80 != 0) return 64;
    return 80;
}

template <int MODE, int BN>
cudaError_t launch_dec(const CUtensorMap& ma, const CUtensorMap& mb, DecParams p, bool pdl, cudaStream_t s) {
    auto kernel = decode_tc_kernel<MODE, BN>;
    static unsigned long long attr_set = 0;   // one bit per device ordinal
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !(attr_set >> dev & 1ull)) {
        const cudaError_t err =
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DecGeo<BN>::SMEM_BYTES);
        if (err != cudaSuccess) return err;
        attr_set |= 1ull << dev;
    }
    p.n_ct = p.d / BN;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.n_ct * kSplit), 1, 1);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = DecGeo<BN>::SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kernel, ma, mb, p);
}

template <int MODE>
cudaError_t launch_dec_bn(int bn, const CUtensorMap& ma, const CUtensorMap& mb, const DecParams& p, bool pdl,
                          cudaStream_t s) {
    return bn == 80 ? launch_dec<MODE, 80>(ma, mb, p, pdl, s) : launch_dec<MODE, 64>(ma, mb, p, pdl, s);
}

}  // namespace

bool decode_tc_supported(int64_t n, int32_t L, int32_t d_mem, int32_t d, int32_t M, bool f8) {
    return L == 1 && n >= 1 && n <= kDecRows && M == 1 && !f8 && d % 64 == 0 && d_mem % 64 == 0 &&
           d_mem / 64 >= kSplit && encode_fn() != nullptr;
}

int32_t decode_tc_max_tiles(int32_t d) { return d / 64; }

cudaError_t launch_decode_k(const void* e, int32_t n, int32_t d_mem, const void* h, const void* Wk, const void* Wv,
                            const float* gq, const float* gk, int32_t d, float eps, float* part, int* band_count,
                            float* alpha, float* alpha_out, uint32_t* status, int num_sms, int stall, bool pdl,
                            cudaStream_t s) {
    if (!decode_tc_supported(n, 1, d_mem, d, 1, false)) return cudaErrorNotSupported;
    const int bn = pick_dec_bn(d, num_sms);
    CUtensorMap ma, mb;
    if (!make_map(&ma, e, (uint64_t)n, (uint64_t)d_mem, 128) || !make_map(&mb, Wk, (uint64_t)d, (uint64_t)d_mem, bn))
        return cudaErrorInvalidValue;
    DecParams p{};
    p.w = static_cast<const __nv_bfloat16*>(Wk);
    p.w_next = static_cast<const __nv_bfloat16*>(Wv);
    p.h = static_cast<const __nv_bfloat16*>(h);
    p.gq = gq;
    p.gk = gk;
    p.alpha_w = alpha;
    p.alpha_out = alpha_out;
    p.part = reinterpret_cast<float4*>(part);
    p.band_count = band_count;
    p.status = status;
    p.n = n;
    p.d = d;
    p.d_mem = d_mem;
    p.eps = eps;
    p.stall = stall;
    return launch_dec_bn<DEC_K>(bn, ma, mb, p, pdl, s);
}

cudaError_t launch_decode_v(const void* e, int32_t n, int32_t d_mem, const void* h, const void* Wv,
                            const float* conv_w, int32_t d, const float* alpha, float* state, void* y,
                            int32_t add_residual, uint32_t* status, int num_sms, bool pdl, cudaStream_t s) {
    if (!decode_tc_supported(n, 1, d_mem, d, 1, false)) return cudaErrorNotSupported;
    const int bn = pick_dec_bn(d, num_sms);
    CUtensorMap ma, mb;
    if (!make_map(&ma, e, (uint64_t)n, (uint64_t)d_mem, 128) || !make_map(&mb, Wv, (uint64_t)d, (uint64_t)d_mem, bn))
        return cudaErrorInvalidValue;
    DecParams p{};
    p.w = static_cast<const __nv_bfloat16*>(Wv);
    p.h = static_cast<const __nv_bfloat16*>(h);
    p.conv_w = conv_w;
    p.state = state;
    p.alpha = alpha;
    p.y = static_cast<__nv_bfloat16*>(y);
    p.status = status;
    p.n = n;
    p.d = d;
    p.d_mem = d_mem;
    p.add_residual = add_residual;
    return launch_dec_bn<DEC_V>(bn, ma, mb, p, pdl, s);
}

}  // namespace engram
