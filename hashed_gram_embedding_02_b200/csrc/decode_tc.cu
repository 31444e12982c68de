// Decode: the key and value projections with the gate and the conv, for a
// call that computes one new position per sequence (L = 1) for at most 256
// sequences.
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
// per-SM stream.  Here two kernels do the work:
//
// decode_kv_kernel (both projections, the gate partials): a cluster of 4
// CTAs per channel tile of BN channels, as two CTA pairs.
//   - each pair multiplies one half of K (d_mem) with M = 256 tcgen05 MMAs
//     (cta_group::2): each CTA of the pair stages its 128 rows of e and half
//     of the tile's W_K and W_V rows, and its TMEM receives its 128 rows of
//     k and v over all BN channels; each A stage of e feeds both products, so
//     e streams once for the two projections;
//   - the two halves of K are added through distributed shared memory: each
//     CTA stages its k and v rows in its own ring and sends, in two bulk
//     copies that complete on the receiver's mbarrier, the 64 rows that the
//     CTA holding the same rows from the other half of K owns; the owner adds
//     the two partials in K-half order, so the sums do not depend on timing;
//   - the owner finishes its 64 rows x BN channels with threads running
//     along channels: the rows' gate partials for the channel tile
//     (sum g_q g_k h k, sum k^2, sum h^2), and v, written to the workspace.
// decode_conv_kernel (the gate, the conv, SiLU and residual): each CTA
// reduces the gate partials of the rows it covers into alpha (one warp per
// row, in channel-tile order), then one thread per four channels of a row
// reads v, the history and h, writes Y and rewrites the history in place
// ([v~_{t-2}, v~_{t-1}, v~_t]; each (sequence, channel) belongs to one
// thread).  It is a programmatic dependent of the first kernel: its CTAs take
// the SMs' spare slots early and load the history, h and the taps before
// they wait for v and the partials.
//
// The grid of the first kernel is d / BN clusters (BN = 64 or 80, the
// narrowest whose clusters are all resident at once).  It issues its first W
// stages before waiting for the retrieval.  Each cluster walks its k-blocks
// from a different starting block (rotated by its channel tile): every
// cluster reads the same half of e, and the rotation spreads those reads
// over L2 instead of every cluster asking for the same lines at once.
//
// Every mbarrier wait is bounded.  A CTA whose wait runs out flags
// ENGRAM_ERR_TIMEOUT and votes to abort; after the first cluster barrier every
// CTA of the cluster reads the votes, and on any abort the cluster exchanges
// nothing and writes nothing.  The CTA drains its own copies and MMAs
// (bounded) before it frees its TMEM and leaves.
#include "tc.cuh"

namespace engram {

namespace {

constexpr int kCluster = 4;           // CTAs per cluster: two CTA pairs, one per half of K
constexpr int kDecThreads = 256;
constexpr int kDecStages = 8;
constexpr int kDecRows = 256;         // rows per call: one M = 256 pair accumulator
constexpr int kOwnRows = 64;          // rows a CTA finishes (half of its 128 accumulator rows)
constexpr int kAccK = 0;              // TMEM columns of the key accumulator
constexpr int kAccV = 128;            // and of the value accumulator
constexpr int kTmemCols = 256;
constexpr int kABytes = 128 * 128;    // one 128-row x 64-element bf16 box
constexpr int kConvThreads = 256;

template <int BN>
struct DecGeo {
    static constexpr int B_ROWS = BN / 2;                     // W rows (channels) this CTA of a pair stages
    static constexpr int B_BYTES = B_ROWS * 128;
    static constexpr int STAGE_BYTES = kABytes + 2 * B_BYTES;   // A (this CTA's 128 rows) | W_K half | W_V half
    static constexpr int RING = kDecStages * STAGE_BYTES;
    static constexpr int RS = BN + 4;   // floats per staged row (16-byte pad: conflict-free row-per-lane stores)
    // after the MMAs the ring holds, for k and then for v, this CTA's
    // partial sums [128][RS] and the partner's partials of the rows it owns
    // [64][RS]
    static constexpr int PART_BYTES = 128 * RS * 4;
    static constexpr int RECV_BYTES = kOwnRows * RS * 4;
    static constexpr int STAGE_K = 0;
    static constexpr int RECV_K = STAGE_K + PART_BYTES;
    static constexpr int STAGE_V = RECV_K + RECV_BYTES;
    static constexpr int RECV_V = STAGE_V + PART_BYTES;
    static constexpr int EXCH_BYTES = RECV_V + RECV_BYTES;
    static constexpr int CONST_BYTES = BN * 4;   // g_q g_k of the tile's channels
    static constexpr int SMEM_BYTES = RING + 1024 + CONST_BYTES + 1024;
    static_assert(EXCH_BYTES <= RING, "the partials reuse the operand ring");
    static_assert(BN % 16 == 0 && BN <= kAccV, "UMMA N and the accumulator spacing");
    static_assert(B_ROWS % 8 == 0, "whole 8-row swizzle atoms per W half");
    static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
};

struct __align__(8) DecBarriers {
    uint64_t full[kDecStages];
    uint64_t empty[kDecStages];
    uint64_t pfull[kDecStages];   // leader: the partner CTA's half of the stage is full
    uint64_t tfull;
    uint64_t rfull;   // the other half of K's partials (k and v) of this CTA's rows have landed
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;   // this CTA's vote (read by the cluster after the first barrier)
    int issued;       // k-block stages whose loads were issued
    int consumed;     // stages the MMAs have taken
};

struct DecParams {
    const __nv_bfloat16* wk;       // [d][d_mem]
    const __nv_bfloat16* wv;       // [d][d_mem]
    const __nv_bfloat16* h;        // [n][d]
    const float* gq;               // [d] or null
    const float* gk;               // [d] or null
    float4* part;                  // [n][n_ct] (sum g h k, sum k^2, sum h^2, 0)
    float* v;                      // [n][d] fp32, for the conv kernel
    uint32_t* status;
    int n, d, d_mem, n_ct;
    int stall;                     // test hook: CTA 0 announces its first stage and never loads it
};

struct ConvParams {
    const float* v;                // [n][d]
    const float4* part;            // [n][n_ct] gate partials
    float* alpha_w;                // [n] gate values (written)
    float* alpha_out;              // caller's copy, or null
    const __nv_bfloat16* h;        // [n][d]
    const float* conv_w;           // [d][4]
    float* state;                  // [n][3][d] conv history, updated in place, or null (zero history)
    __nv_bfloat16* y;              // [n][d]
    int n, d, n_ct;
    int add_residual;
    float eps;
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

// rows of [first, first + kOwnRows) below n
__device__ __forceinline__ int live_rows(int n, int first) {
    const int r = n - first;
    return r < 0 ? 0 : (r < kOwnRows ? r : kOwnRows);
}

// While the MMAs run, warps 2-7 stage g_q g_k of the tile's channels in
// shared memory and bring this CTA's halves of the W_K and W_V slices into
// L2, so the stages after the first round find them there.  Offsets and
// lengths are multiples of 16 bytes (d_mem a multiple of 64).
template <int BN>
__device__ __forceinline__ void dec_prefetch(const DecParams& p, int ct, int w_row0, int kb0, int nkb, float* s_g,
                                             int t, int nt) {
    const int c0 = ct * BN;
    for (int c = t; c < BN; c += nt)
        s_g[c] = (p.gq ? __ldg(p.gq + c0 + c) : 1.f) * (p.gk ? __ldg(p.gk + c0 + c) : 1.f);
    if (nkb <= kDecStages) return;
    for (int c = t; c < DecGeo<BN>::B_ROWS; c += nt) {
        const int64_t wrow = (int64_t)(w_row0 + c) * p.d_mem + (int64_t)kb0 * 64;
        prefetch_l2(p.wk + wrow, (uint32_t)nkb * 128u);
        prefetch_l2(p.wv + wrow, (uint32_t)nkb * 128u);
    }
}

// The two partial sums of an owned row, in K-half order: this CTA's own from
// its staging rows, the partner's from the receive rows.
template <int BN>
struct PartRows {
    const float* stage;   // this CTA's 128 accumulator rows
    const float* recv;    // the partner's partials of the owned rows
    int own0;             // first owned row within the CTA's 128
    int half;             // this CTA's half of K
    __device__ __forceinline__ const float* row(int src, int lr) const {
        constexpr int RS = DecGeo<BN>::RS;
        return src == half ? stage + (own0 + lr) * RS : recv + lr * RS;
    }
};

// h of the CTA's owned rows, in registers during the key exchange, so its
// latency hides behind it: warp w holds rows w, w + 8, .., lane l channels
// l, l + 32, ..
template <int BN>
struct KIn {
    static constexpr int NJ = (BN + 31) / 32;
    static constexpr int NW = kDecThreads / 32;
    static constexpr int RPW = kOwnRows / NW;   // rows per warp (8)
    float hv[RPW][NJ];
    __device__ __forceinline__ void load(const DecParams& p, int row0, int ct) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
            const int row = row0 + warp + NW * i;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const int c = lane + 32 * j;
                hv[i][j] = (row < p.n && c < BN) ? __bfloat162float(p.h[(int64_t)row * p.d + ct * BN + c]) : 0.f;
            }
        }
    }
};

// Gate partials of the CTA's owned rows over its BN channels.
template <int BN>
__device__ __forceinline__ void dec_epilogue_k(const DecParams& p, const PartRows<BN>& pr, const KIn<BN>& in,
                                               const float* s_g, int row0, int ct) {
    constexpr int NJ = KIn<BN>::NJ;
    constexpr int NW = KIn<BN>::NW;
    constexpr int RPW = KIn<BN>::RPW;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const auto& hv = in.hv;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int lr = warp + NW * i, row = row0 + lr;
        if (row >= p.n) break;
        float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int c = lane + 32 * j;
            if (c < BN) {
                const float k = pr.row(0, lr)[c] + pr.row(1, lr)[c];
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
}

// v of the CTA's owned rows over its BN channels: the two partials in K-half
// order, four channels per item, consecutive threads on consecutive channels
template <int BN>
__device__ __forceinline__ void dec_write_v(const DecParams& p, const PartRows<BN>& pr, int row0, int ct) {
    constexpr int NQ = BN / 4;
    for (int it = threadIdx.x; it < kOwnRows * NQ; it += kDecThreads) {
        const int lr = it / NQ, q4 = it - lr * NQ;
        const int row = row0 + lr;
        if (row >= p.n) break;
        const float4 a = *reinterpret_cast<const float4*>(pr.row(0, lr) + 4 * q4);
        const float4 b = *reinterpret_cast<const float4*>(pr.row(1, lr) + 4 * q4);
        *reinterpret_cast<float4*>(p.v + (int64_t)row * p.d + ct * BN + 4 * q4) =
            make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
    }
}

// One accumulator (this CTA's 128 rows) into its staging rows: warp w reads
// TMEM lanes 32 (w % 4) .. +31 and channel half w / 4, one row per lane;
// the padded rows put the lanes' stores in distinct banks
template <int BN>
__device__ __forceinline__ void stage_acc(uint32_t tmem, float* stage) {
    constexpr int HALF = BN / 2;
    constexpr int NCH = HALF / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = warp & 3, col0 = (warp >> 2) * HALF;
    const int row = q * 32 + lane;
    uint32_t v[NCH][8];
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch)
        tmem_ld8(tmem + (uint32_t)(col0 + ch * 8) + ((uint32_t)(q * 32) << 16), v[ch]);
    tmem_wait_ld();
    uint4* dst = reinterpret_cast<uint4*>(stage + row * DecGeo<BN>::RS + col0);
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
        dst[2 * ch] = make_uint4(v[ch][0], v[ch][1], v[ch][2], v[ch][3]);
        dst[2 * ch + 1] = make_uint4(v[ch][4], v[ch][5], v[ch][6], v[ch][7]);
    }
    // the bulk copy reads the staged rows through the async proxy
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// one bulk copy: the staged rows the partner owns (contiguous, padded) into
// its receive rows (thread 0)
template <int BN>
__device__ __forceinline__ void send_partials(DecBarriers* sb, float* stage, float* recv, int partner,
                                              int partner_own0, int rows) {
    constexpr int RS = DecGeo<BN>::RS;
    if (threadIdx.x != 0 || rows <= 0) return;
    bulk_s2cluster(peer_addr(recv, (uint32_t)partner), smem_u32(stage + partner_own0 * RS), (uint32_t)(rows * RS * 4),
                   peer_addr(&sb->rfull, (uint32_t)partner));
}

// Cluster of 4: rank 2h + m.  The pair {2h, 2h+1} multiplies the h-th half
// of K with M = 256 tcgen05 MMAs issued by its leader (m = 0): CTA m stages
// rows 128m .. 128m+127 of e and channels m BN/2 .. (m+1) BN/2 - 1 of the
// tile's W_K and W_V, and its TMEM receives its 128 rows of k and v over all
// BN channels.  CTA (h, m) owns rows 128m + 64h .. +63 and exchanges its
// other 64 rows (k and v) with CTA (1-h, m), which holds the same rows from
// the other half of K; two cluster barriers bracket the exchange.
template <int BN>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kDecThreads, 1)
decode_kv_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_bk,
                 const __grid_constant__ CUtensorMap map_bv, const DecParams p) {
    using GE = DecGeo<BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024 - (raw & 1023)) & 1023);   // 1024-byte aligned ring
    const uint32_t ring = smem_u32(smem);
    DecBarriers* sb = reinterpret_cast<DecBarriers*>(smem + GE::RING);
    float* s_g = reinterpret_cast<float*>(smem + GE::RING + 1024);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_rank();
    const int half = rank >> 1, m = rank & 1;
    const bool leader = m == 0;
    const int lead_rank = rank & ~1;            // the pair's leader
    const uint16_t pair_mask = (uint16_t)(3u << lead_rank);
    const int partner = rank ^ 2;               // same rows, other half of K
    const int ct = (int)blockIdx.x / kCluster;  // channel tile of the cluster
    const int own0 = half * kOwnRows;           // first owned row within the CTA's 128
    const int row0 = m * 128 + own0;            // first owned row
    // this pair's k-blocks (64 elements each)
    const int kb_total = p.d_mem / 64;
    const int kb0 = half * kb_total / 2, kb1 = (half + 1) * kb_total / 2;
    const int nkb = kb1 - kb0;
    const int rot = nkb > 0 ? ct % nkb : 0;     // this cluster's first k-block (see the header)
    const int w_row0 = ct * BN + m * GE::B_ROWS;   // this CTA's W rows

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&sb->full[s], 1);
            mbar_init(&sb->empty[s], 1);
            mbar_init(&sb->pfull[s], 1);
        }
        mbar_init(&sb->tfull, 1);
        mbar_init(&sb->rfull, 1);
        mbar_init(&sb->drain, 1);
        sb->abort_flag = 0;
        sb->issued = 0;
        sb->consumed = 0;
        mbar_fence_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_bk);
        tma_prefetch_desc(&map_bv);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sb->tmem_base)),
                     "n"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();   // every CTA's barriers are initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = sb->tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer (each CTA loads its own rows and W half;
        // the partner of a pair counts its stages on the leader's pfull)
        if (lane == 0) {
            const int pre = nkb < kDecStages ? nkb : kDecStages;
            auto kcol = [&](int j) { return (kb0 + (j + rot) % nkb) * 64; };
            auto bar_of = [&](int s) {
                return leader ? smem_u32(&sb->full[s]) : peer_addr(&sb->pfull[s], (uint32_t)lead_rank);
            };
            auto load = [&](const CUtensorMap* map, uint32_t dst, int s, int x, int y) {
                if (leader) tma_load_2d(map, dst, &sb->full[s], x, y);
                else tma_load_2d_peer_bar(map, dst, bar_of(s), x, y);
            };
            auto load_w = [&](int j) {
                const int s = j % kDecStages;
                if (leader) mbar_arrive_expect_tx(&sb->full[s], GE::STAGE_BYTES);
                else mbar_arrive_expect_tx_remote(bar_of(s), GE::STAGE_BYTES);
                if (p.stall && j == 0 && blockIdx.x == 0) return;   // bounded-wait test: never loaded
                const uint32_t b = ring + s * GE::STAGE_BYTES + kABytes;
                load(&map_bk, b, s, kcol(j), w_row0);
                load(&map_bv, b + GE::B_BYTES, s, kcol(j), w_row0);
            };
            auto load_a = [&](int j) {
                const int s = j % kDecStages;
                if (p.stall && j == 0 && blockIdx.x == 0) return;
                load(&map_a, ring + s * GE::STAGE_BYTES, s, kcol(j), m * 128);
            };
            // the weights do not depend on the retrieval: their first stages
            // stream while it finishes; e is read after it completes
            for (int j = 0; j < pre; ++j) load_w(j);
            grid_dep_wait();
            for (int j = 0; j < pre; ++j) load_a(j);
            sb->issued = pre;
            for (int j = pre; j < nkb; ++j) {
                const int s = j % kDecStages;
                if (!dec_wait(&sb->empty[s], ((uint32_t)(j / kDecStages) & 1u) ^ 1u, sb, p.status)) break;
                load_w(j);
                load_a(j);
                sb->issued = j + 1;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (the pair's leader): each stage feeds k and v
        if (lane == 0 && leader) {
            bool ok = true;
            for (int j = 0; j < nkb; ++j) {
                const int s = j % kDecStages;
                const uint32_t ph = (uint32_t)(j / kDecStages) & 1u;
                if (!dec_wait(&sb->full[s], ph, sb, p.status) || !dec_wait(&sb->pfull[s], ph, sb, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = ring + s * GE::STAGE_BYTES;
                const uint64_t da = smem_desc_sw128(a_addr);
                const uint64_t dbk = smem_desc_sw128(a_addr + kABytes);
                const uint64_t dbv = smem_desc_sw128(a_addr + kABytes + GE::B_BYTES);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    umma_bf16_pair<BN>(tmem_base + kAccK, da + (uint64_t)(kk * 2), dbk + (uint64_t)(kk * 2),
                                       (j | kk) != 0);
                    umma_bf16_pair<BN>(tmem_base + kAccV, da + (uint64_t)(kk * 2), dbv + (uint64_t)(kk * 2),
                                       (j | kk) != 0);
                }
                umma_commit_pair_mask(&sb->empty[s], pair_mask);
                sb->consumed = j + 1;
            }
            if (ok) umma_commit_pair_mask(&sb->tfull, pair_mask);
        }
        __syncwarp();
    } else {
        dec_prefetch<BN>(p, ct, w_row0, kb0, nkb, s_g, threadIdx.x - 64, kDecThreads - 64);
    }
    // the conv kernel may launch once every thread of every CTA is past the
    // retrieval (warp 0 follows its lane 0, which waited above); its CTAs
    // load the history and h while this grid runs
    if (warp != 0) grid_dep_wait();
    grid_dep_launch_dependents();

    // ---------------- accumulators complete (the leader's commits arrive in both CTAs)
    const bool ok = nkb > 0 && dec_wait(&sb->tfull, 0, sb, p.status);
    const int cta_abort = __syncthreads_or(!ok || sb->abort_flag);
    tc_fence_after();
    float* stage_k = reinterpret_cast<float*>(smem + GE::STAGE_K);
    float* recv_k = reinterpret_cast<float*>(smem + GE::RECV_K);
    float* stage_v = reinterpret_cast<float*>(smem + GE::STAGE_V);
    float* recv_v = reinterpret_cast<float*>(smem + GE::RECV_V);
    const PartRows<BN> pk{stage_k, recv_k, own0, half}, pv{stage_v, recv_v, own0, half};
    const int partner_own0 = (1 - half) * kOwnRows;
    const int send_rows = live_rows(p.n, m * 128 + partner_own0);
    const uint32_t rbytes = (uint32_t)(live_rows(p.n, row0) * GE::RS * 4);

    // ---- k and v: stage both, one exchange
    if (!cta_abort) {
        stage_acc<BN>(tmem_base + kAccK, stage_k);
        stage_acc<BN>(tmem_base + kAccV, stage_v);
    }
    if (threadIdx.x == 0) {
        sb->abort_flag = cta_abort;
        mbar_arrive_expect_tx(&sb->rfull, 2 * rbytes);   // the partner's k and v rows
    }
    tc_fence_before();
    // barrier 1: every CTA's MMAs have finished reading its ring, which now
    // receives the partner's partials; the abort votes are visible cluster-wide
    __syncwarp();
    cluster_sync_all();
    int any_abort = 0;
#pragma unroll
    for (int r = 0; r < kCluster; ++r) any_abort |= ld_remote_s32(peer_addr(&sb->abort_flag, (uint32_t)r));
    if (!any_abort) {
        send_partials<BN>(sb, stage_k, recv_k, partner, partner_own0, send_rows);
        send_partials<BN>(sb, stage_v, recv_v, partner, partner_own0, send_rows);
    }
    // h of the owned rows, in flight during the exchange (issued after the
    // barrier, whose release would otherwise wait for the loads)
    KIn<BN> kin;
    kin.load(p, row0, ct);
    const bool have = !any_abort && dec_wait(&sb->rfull, 0, sb, p.status);
    // barrier 2: every copy has landed, so no CTA's staged rows are read any more
    __syncwarp();
    cluster_sync_all();
    if (!any_abort && __syncthreads_and(have)) {
        dec_epilogue_k<BN>(p, pk, kin, s_g, row0, ct);
        dec_write_v<BN>(p, pv, row0, ct);
    } else if (any_abort && leader) {
        // the pair stopped early: the leader waits out every stage either CTA
        // of the pair issued (the partner's complete on its pfull), then its MMAs
        if (warp == 0 && lane == 0) {
            for (int j = sb->consumed; j < sb->issued; ++j)
                dec_wait_drain(&sb->full[j % kDecStages], (uint32_t)(j / kDecStages) & 1u);
            const int peer_issued = ld_remote_s32(peer_addr(&sb->issued, (uint32_t)(rank + 1)));
            for (int j = sb->consumed; j < peer_issued; ++j)
                dec_wait_drain(&sb->pfull[j % kDecStages], (uint32_t)(j / kDecStages) & 1u);
        }
        if (warp == 1 && lane == 0) {
            umma_commit_pair_local(&sb->drain);
            dec_wait_drain(&sb->drain, 0);
        }
    }
    __syncthreads();
    // the cluster leaves together: no copy or MMA of a pair is in flight
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "n"(kTmemCols)
                     : "memory");
    }
}

// Gate, conv over the history in the caller's state, SiLU, residual; one
// thread per four channels of a row.  The history, h and the taps are read
// before the wait for the kernel that writes v and the gate partials; then
// warp w reduces the partials of the CTA's w-th row into alpha (a CTA covers
// at most 8 rows: d is a multiple of 128, so a row is at least 32 items).
constexpr int kConvRows = kConvThreads / 32;

__global__ void __launch_bounds__(kConvThreads) decode_conv_kernel(const ConvParams q) {
    __shared__ float s_alpha[kConvRows];
    const int dq = q.d / 4;
    const int64_t it0 = (int64_t)blockIdx.x * kConvThreads;
    const int64_t it = it0 + threadIdx.x;
    const bool live = it < (int64_t)q.n * dq;
    const int64_t row = live ? it / dq : 0;
    const int c = live ? (int)(it - row * dq) * 4 : 0;
    float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0, s2 = s0;
    uint2 hq = make_uint2(0u, 0u);
    float4 w[4];
    float4* st = nullptr;
    if (live) {
        if (q.state) {
            st = reinterpret_cast<float4*>(q.state + row * 3 * q.d + c);
            s0 = __ldcs(st);
            s1 = __ldcs(st + dq);
            s2 = __ldcs(st + 2 * dq);
        }
        if (q.add_residual) hq = __ldcs(reinterpret_cast<const uint2*>(q.h + row * q.d + c));
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = __ldg(reinterpret_cast<const float4*>(q.conv_w) + c + e);
    }
    grid_dep_wait();   // v and the gate partials come from the projection kernel

    // alpha of the rows this CTA covers, each reduced in channel-tile order
    const int64_t row0 = it0 / dq;
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t r = row0 + wid;
    if (r < q.n && r * dq < it0 + kConvThreads) {
        float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
        for (int t = lane; t < q.n_ct; t += 32) {
            const float4 v = __ldcg(q.part + r * q.n_ct + t);
            s_qk += v.x;
            s_kk += v.y;
            s_hh += v.z;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s_qk += __shfl_xor_sync(0xffffffffu, s_qk, o);
            s_kk += __shfl_xor_sync(0xffffffffu, s_kk, o);
            s_hh += __shfl_xor_sync(0xffffffffu, s_hh, o);
        }
        if (lane == 0) {
            const float inv_d = 1.f / (float)q.d;
            const float rh = sqrtf(s_hh * inv_d + q.eps);
            const float rk = sqrtf(s_kk * inv_d + q.eps);
            const float a = 1.f / (1.f + expf(-(s_qk / (rh * rk)) * rsqrtf((float)q.d)));
            s_alpha[wid] = a;
            // the CTA that holds the row's first channels publishes it
            if (r * dq >= it0) {
                q.alpha_w[r] = a;
                if (q.alpha_out) q.alpha_out[r] = a;
            }
        }
    }
    __syncthreads();
    if (!live) return;
    const float4 v = __ldcg(reinterpret_cast<const float4*>(q.v + row * q.d + c));
    const float a = s_alpha[row - row0];
    const float x[4] = {a * v.x, a * v.y, a * v.z, a * v.w};
    const float h0[4] = {s0.x, s0.y, s0.z, s0.w}, h1[4] = {s1.x, s1.y, s1.z, s1.w}, h2[4] = {s2.x, s2.y, s2.z, s2.w};
    const float hv[4] = {bf16_lo(hq.x), bf16_hi(hq.x), bf16_lo(hq.y), bf16_hi(hq.y)};
    float yv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        // tap j multiplies the input j positions back: x_t, then the history
        // rows 2, 1, 0 (oldest last)
        float u = w[e].x * x[e];
        u = fmaf(w[e].y, h2[e], u);
        u = fmaf(w[e].z, h1[e], u);
        u = fmaf(w[e].w, h0[e], u);
        const float hu = 0.5f * u;
        yv[e] = x[e] + fmaf(hu, dec_tanh(hu), hu) + hv[e];
    }
    *reinterpret_cast<uint2*>(q.y + row * q.d + c) = make_uint2(pack_bf16x2(yv[0], yv[1]), pack_bf16x2(yv[2], yv[3]));
    if (st) {
        st[0] = s1;
        st[dq] = s2;
        st[2 * dq] = make_float4(x[0], x[1], x[2], x[3]);
    }
}

// ---------------------------------------------------------------- host side

// clusters of kCluster CTAs of the decode kernel that the device holds at once
int resident_clusters(int num_sms) {
    static int cached[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    auto kernel = decode_kv_kernel<80>;
    int mc = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DecGeo<80>::SMEM_BYTES) ==
        cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(num_sms / kCluster * kCluster), 1, 1);
        cfg.blockDim = dim3(kDecThreads, 1, 1);
        cfg.dynamicSmemBytes = DecGeo<80>::SMEM_BYTES;
        if (cudaOccupancyMaxActiveClusters(&mc, kernel, &cfg) != cudaSuccess) mc = 0;
    }
    cudaGetLastError();
    if (mc < 1) mc = num_sms / kCluster;
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

template <int BN>
cudaError_t launch_kv(const CUtensorMap& ma, const CUtensorMap& mk, const CUtensorMap& mv, DecParams p, bool pdl,
                      cudaStream_t s) {
    auto kernel = decode_kv_kernel<BN>;
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
    cfg.gridDim = dim3((unsigned)(p.n_ct * kCluster), 1, 1);
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
    return cudaLaunchKernelEx(&cfg, kernel, ma, mk, mv, p);
}

}  // namespace

bool decode_tc_supported(int64_t n, int32_t L, int32_t d_mem, int32_t d, int32_t M, bool f8) {
    return L == 1 && n >= 1 && n <= kDecRows && M == 1 && !f8 && d % 64 == 0 && d_mem % 64 == 0 &&
           d_mem / 64 >= 2 && encode_fn() != nullptr;
}

int32_t decode_tc_max_tiles(int32_t d) { return d / 64; }

cudaError_t launch_decode_kv(const void* e, int32_t n, int32_t d_mem, const void* h, const void* Wk, const void* Wv,
                             const float* gq, const float* gk, int32_t d, float* part, float* v, uint32_t* status,
                             int num_sms, int stall, bool pdl, cudaStream_t s) {
    if (!decode_tc_supported(n, 1, d_mem, d, 1, false)) return cudaErrorNotSupported;
    const int bn = pick_dec_bn(d, num_sms);
    CUtensorMap ma, mk, mv;
    // each CTA of a pair stages half of the tile's W rows
    if (!make_map(&ma, e, (uint64_t)n, (uint64_t)d_mem, 128) ||
        !make_map(&mk, Wk, (uint64_t)d, (uint64_t)d_mem, bn / 2) ||
        !make_map(&mv, Wv, (uint64_t)d, (uint64_t)d_mem, bn / 2))
        return cudaErrorInvalidValue;
    DecParams p{};
    p.wk = static_cast<const __nv_bfloat16*>(Wk);
    p.wv = static_cast<const __nv_bfloat16*>(Wv);
    p.h = static_cast<const __nv_bfloat16*>(h);
    p.gq = gq;
    p.gk = gk;
    p.part = reinterpret_cast<float4*>(part);
    p.v = v;
    p.status = status;
    p.n = n;
    p.d = d;
    p.d_mem = d_mem;
    p.stall = stall;
    return bn == 80 ? launch_kv<80>(ma, mk, mv, p, pdl, s) : launch_kv<64>(ma, mk, mv, p, pdl, s);
}

cudaError_t launch_decode_conv(const float* v, const float* part, int32_t n, const void* h, const float* conv_w,
                               int32_t d, float eps, float* alpha, float* alpha_out, float* state, void* y,
                               int32_t add_residual, int num_sms, bool pdl, cudaStream_t s) {
    ConvParams q{};
    q.v = v;
    q.part = reinterpret_cast<const float4*>(part);
    q.alpha_w = alpha;
    q.alpha_out = alpha_out;
    q.h = static_cast<const __nv_bfloat16*>(h);
    q.conv_w = conv_w;
    q.state = state;
    q.y = static_cast<__nv_bfloat16*>(y);
    q.n = n;
    q.d = d;
    q.n_ct = d / pick_dec_bn(d, num_sms);   // the projection kernel's channel tiles
    q.add_residual = add_residual;
    q.eps = eps;
    const int64_t items = (int64_t)n * (d / 4);
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((items + kConvThreads - 1) / kConvThreads), 1, 1);
    cfg.blockDim = dim3(kConvThreads, 1, 1);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, decode_conv_kernel, q);
}

}  // namespace engram
