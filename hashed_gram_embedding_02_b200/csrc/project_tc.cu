// Key/value projections on the 5th-generation tensor cores (tcgen05), with
// the gate and the causal convolution fused into the GEMM epilogues.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": k_t = W_K e_t and
// v_t = W_V e_t; RMSNorm on the query h_t and on the key; a scalar gate
// alpha_t in (0,1); v~_t = alpha_t v_t; a short-kernel per-channel causal
// convolution; Y added to the residual stream.  (The multi-branch variant of
// the same section fuses the projections into one dense GEMM to keep the GPU
// busy.)  One kernel template, three epilogues:
//
//   MODE_KV    tile = 128 rows x (128 k-channels | the same 128 v-channels):
//              writes v (fp32) and the group's gate partials; the standalone
//              engram_project.
//   MODE_K     tile = 128 rows x BN k-channels: writes the gate partials
//              (sum g_q g_k h k, sum k^2, sum h^2) of its BN/128 channel
//              groups; k never leaves the SM.
//   MODE_VCONV tile = 128 rows x BN v-channels, row tiles overlapping by the
//              conv history (w-1 rows): each thread owns one TMEM lane (one
//              row), reduces its row's partials into alpha, forms v~ = alpha v,
//              takes v~ of the w-1 previous rows from the neighbouring lanes
//              (warp shuffles, plus a shared-memory hand-over between the four
//              epilogue warps), applies the conv taps, SiLU, the residual, and
//              writes Y.  v itself never reaches global memory.
//
// Persistent kernel, one CTA per SM, warp-specialised:
//   warp 0     TMA producer: 2-D tiled loads (128-byte swizzle) of the A
//              (e) tile and the W tile(s) into a shared-memory ring
//   warp 1     allocates TMEM (two fp32 accumulators) and issues
//              tcgen05.mma kind::f16 (M=128, N=BN, K=16) from one thread
//   warps 4-7  epilogue: tcgen05.ld of the accumulator; warp w reads TMEM
//              lanes 32(w-4) .. 32(w-4)+31
// The double-buffered accumulator lets the epilogue of tile i overlap the
// MMAs of tile i+1.  Tiles run channel-fastest so consecutive tiles share the
// A block in L2; W stays L2-resident.
//
// Every mbarrier wait is bounded (about 2 s of clock64 time).  A wait that runs
// out sets ENGRAM_ERR_TIMEOUT, raises a CTA-wide abort flag that makes the
// other roles leave their loops, drains the copies and MMAs this CTA issued
// (bounded again), frees the TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace engram {

namespace {

constexpr int MODE_KV = 0;
constexpr int MODE_K = 1;
constexpr int MODE_VCONV = 2;

constexpr int BM = 128;                 // rows per tile (UMMA M)
constexpr int BK = 64;                  // K per stage: 64 bf16 = 128 bytes = one swizzle row
constexpr int UK = 16;                  // K per tcgen05.mma kind::f16
constexpr int A_BYTES = BM * BK * 2;    // 16 KB
constexpr int THREADS = 256;
constexpr int kMaxHist = kMaxConv - 1;

template <int BN>
struct Geo {
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (192 * 1024) / STAGE_BYTES;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int SMEM_TILES = STAGES * STAGE_BYTES;
    // tiles | barriers (1 KB) | conv taps [2][BN * 8] fp32 | hand-over [2][4][kMaxHist][32] fp32 | slack
    static constexpr int CW_BYTES = 2 * BN * kMaxConv * 4;
    static constexpr int XB_BYTES = 2 * 4 * kMaxHist * 32 * 4;
    static constexpr int SMEM_BYTES = SMEM_TILES + 1024 + CW_BYTES + XB_BYTES + 1024;
};

struct __align__(8) Barriers {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort_flag;
    int issued;       // k-block loads issued by the producer
    int consumed;     // k-block stages consumed by the MMA issuer
};

struct EpiParams {
    const __nv_bfloat16* h;     // [n_tok][d]
    const float* gq;            // [d] or null
    const float* gk;            // [d] or null
    float* v;                   // MODE_KV: [n_tok][d] fp32
    float4* part;               // [n_tok][G]: written (KV, K), read (VCONV)
    const float* conv_w;        // [d][w]
    const float* state;         // [B][w-1][d] history, or null (zero history)
    float* state_next;          // [B][w-1][d] new history (merged by a second kernel), or null
    __nv_bfloat16* y;           // [n_tok][d]
    float* alpha_out;           // [n_tok] or null
    uint32_t* status;
    int n_tok, d_mem, d, G;
    int n_groups;               // tiles along the channel dimension
    int num_tiles;
    int m_stride;               // rows advanced per row tile (128, or 128 - (w-1) in MODE_VCONV)
    int halo;                   // leading rows of a tile that are history only (MODE_VCONV)
    int L;                      // rows per sequence
    int w;                      // conv width
    int add_residual;
    float eps;
};

// Bounded wait: true when the phase with `parity` completed, false when the
// CTA aborted or the wait ran out (then the status bit and abort flag are set).
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, Barriers* sb, uint32_t* status) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(a, parity)) return true;
        if (sb->abort_flag) return false;
        if (clock64() - t0 > kWaitCycles) {
            flag(status, ENGRAM_ERR_TIMEOUT);
            sb->abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint32_t dst, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row core groups 1024 bytes apart (SBO), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFF) >> 4);          // start address [0,14)
    d |= (uint64_t)1 << 16;                          // leading byte offset (unused for SW128 K-major)
    d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset [32,46)
    d |= (uint64_t)1 << 46;                          // version [46,48) = 1
    d |= (uint64_t)2 << 61;                          // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = BN, M = 128.
template <int BN>
struct Idesc {
    static constexpr uint32_t value =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
};

template <int BN>
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(tmem_d), "l"(da), "l"(db), "n"(Idesc<BN>::value), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// named barrier among the four epilogue warps (id 1; id 0 is __syncthreads)
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// the same barrier as a vote: true on every epilogue thread when any passed true
__device__ __forceinline__ bool epi_any(bool x) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)x)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float silu_bf16out(float x) {
    // x * sigmoid(x) = hx + hx * tanh(hx), hx = x/2; hardware tanh approximation
    // (relative error about 2^-11, below the bf16 rounding of Y)
    const float hx = 0.5f * x;
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hx));
    return fmaf(hx, t, hx);
}

// ---------------------------------------------------------------- epilogues

// gate partials of one 128-channel group from 128 k columns at taddr
__device__ __forceinline__ void partials_128(uint32_t taddr, const EpiParams& p, int64_t row, bool valid, int c0,
                                             float& s_qk, float& s_kk, float& s_hh) {
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t kr[32];
        tmem_ld32(taddr + ch * 32, kr);
        tmem_wait_ld();
        if (valid) {
            const uint4* hp = reinterpret_cast<const uint4*>(p.h + row * p.d + c0 + ch * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint4 hv = __ldg(hp + u);
                const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const int i = u * 8 + q * 2 + half;
                        const int c = c0 + ch * 32 + i;
                        const float hf = half ? bf16_hi(hw[q]) : bf16_lo(hw[q]);
                        const float kf = __uint_as_float(kr[i]);
                        const float gg = (p.gq ? __ldg(p.gq + c) : 1.f) * (p.gk ? __ldg(p.gk + c) : 1.f);
                        s_qk = fmaf(gg * hf, kf, s_qk);
                        s_kk = fmaf(kf, kf, s_kk);
                        s_hh = fmaf(hf, hf, s_hh);
                    }
                }
            }
        }
    }
}

__device__ __forceinline__ void epilogue_kv(uint32_t taddr, const EpiParams& p, int m0, int nt, int q, int lane) {
    const int64_t row = (int64_t)m0 + q * 32 + lane;
    const bool valid = row < p.n_tok;
    const int c0 = nt * 128;
    float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
    partials_128(taddr, p, row, valid, c0, s_qk, s_kk, s_hh);
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
        uint32_t vr[32];
        tmem_ld32(taddr + 128 + ch * 32, vr);
        tmem_wait_ld();
        if (valid) {
            float4* vp = reinterpret_cast<float4*>(p.v + row * p.d + c0 + ch * 32);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                vp[u] = make_float4(__uint_as_float(vr[4 * u]), __uint_as_float(vr[4 * u + 1]),
                                    __uint_as_float(vr[4 * u + 2]), __uint_as_float(vr[4 * u + 3]));
        }
    }
    if (valid) p.part[row * p.G + nt] = make_float4(s_qk, s_kk, s_hh, 0.f);
}

template <int BN>
__device__ __forceinline__ void epilogue_k(uint32_t taddr, const EpiParams& p, int m0, int nt, int q, int lane) {
    const int64_t row = (int64_t)m0 + q * 32 + lane;
    const bool valid = row < p.n_tok;
#pragma unroll 1
    for (int gi = 0; gi < BN / 128; ++gi) {
        const int g = nt * (BN / 128) + gi;
        float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
        partials_128(taddr + gi * 128, p, row, valid, g * 128, s_qk, s_kk, s_hh);
        if (valid) p.part[row * p.G + g] = make_float4(s_qk, s_kk, s_hh, 0.f);
    }
}

// Gate + causal depthwise conv + residual on a v tile.  TMEM lane i holds flat
// row m0 + i; lanes below `halo` are history rows of the previous tile.
template <int BN>
__device__ __forceinline__ void epilogue_vconv(uint32_t taddr, const EpiParams& p, int m0, int nt, int q, int lane,
                                               int tcount, uint32_t& xcount, float* s_cw, float* s_xb) {
    const int i = q * 32 + lane;
    const int64_t r = (int64_t)m0 + i;
    const bool in_range = r >= 0 && r < p.n_tok;
    const bool out_row = in_range && i >= p.halo;
    const int W = p.w, H = W - 1;
    int64_t b = 0;
    int t = 0;
    if (in_range) {
        b = r / p.L;
        t = (int)(r - b * p.L);
    }
    // alpha of this row: fixed-order sum of its G partials
    float a = 0.f;
    if (in_range) {
        float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
        const float4* pp = p.part + r * p.G;
        for (int g = 0; g < p.G; ++g) {
            const float4 v4 = pp[g];
            s_qk += v4.x;
            s_kk += v4.y;
            s_hh += v4.z;
        }
        const float inv_d = 1.f / (float)p.d;
        const float rh = sqrtf(s_hh * inv_d + p.eps);
        const float rk = sqrtf(s_kk * inv_d + p.eps);
        a = 1.f / (1.f + expf(-(s_qk / (rh * rk)) * rsqrtf((float)p.d)));
    }
    if (out_row && nt == 0 && p.alpha_out) p.alpha_out[r] = a;

    // conv taps of this tile's channels into shared memory (double-buffered by tile)
    const int n0 = nt * BN;
    float* cw = s_cw + (tcount & 1) * (BN * kMaxConv);
    for (int k = i; k < BN * W; k += 128) cw[k] = __ldg(p.conv_w + (int64_t)n0 * W + k);
    epi_sync();

    const bool has_state = p.state != nullptr;
#pragma unroll 1
    for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t vr[32];
        tmem_ld32(taddr + ch * 32, vr);
        tmem_wait_ld();
        float vt[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) vt[c] = a * __uint_as_float(vr[c]);
        // hand the last H lanes' values to the next warp
        float* xb = s_xb + (xcount & 1) * (4 * kMaxHist * 32);
        if (lane >= 32 - H) {
#pragma unroll
            for (int c = 0; c < 32; ++c) xb[(q * kMaxHist + (lane - (32 - H))) * 32 + c] = vt[c];
        }
        epi_sync();
        ++xcount;
        const int cbase = n0 + ch * 32;
        float yv[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) yv[c] = 0.f;
#pragma unroll 1
        for (int j = 1; j < W; ++j) {
            const bool from_prev = lane < j;
            const bool before_seq = t < j;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                float pv = __shfl_up_sync(0xffffffffu, vt[c], j);
                if (from_prev) pv = q > 0 ? xb[((q - 1) * kMaxHist + (H - j + lane)) * 32 + c] : 0.f;
                if (before_seq) pv = has_state ? p.state[(b * H + (H + t - j)) * p.d + cbase + c] : 0.f;
                yv[c] = fmaf(cw[(ch * 32 + c) * W + j], pv, yv[c]);
            }
        }
        if (out_row) {
            float hv[32];
            if (p.add_residual) {
                const uint4* hp = reinterpret_cast<const uint4*>(p.h + r * p.d + cbase);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint4 q4 = __ldg(hp + u);
                    hv[8 * u + 0] = bf16_lo(q4.x); hv[8 * u + 1] = bf16_hi(q4.x);
                    hv[8 * u + 2] = bf16_lo(q4.y); hv[8 * u + 3] = bf16_hi(q4.y);
                    hv[8 * u + 4] = bf16_lo(q4.z); hv[8 * u + 5] = bf16_hi(q4.z);
                    hv[8 * u + 6] = bf16_lo(q4.w); hv[8 * u + 7] = bf16_hi(q4.w);
                }
            }
            uint4* yp = reinterpret_cast<uint4*>(p.y + r * p.d + cbase);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int c = 8 * u + e;
                    const float uu = fmaf(cw[(ch * 32 + c) * W], vt[c], yv[c]);
                    float res = vt[c] + silu_bf16out(uu);
                    if (p.add_residual) res += hv[c];
                    o[e] = res;
                }
                yp[u] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                   pack_bf16x2(o[6], o[7]));
            }
            // the last H rows of a sequence become its next conv history
            if (p.state_next && t >= p.L - H) {
                float* sp = p.state_next + (b * H + (t - (p.L - H))) * p.d + cbase;
#pragma unroll
                for (int c = 0; c < 32; ++c) sp[c] = vt[c];
            }
        }
    }
}

// ---------------------------------------------------------------- kernel

template <int MODE, int BN>
__global__ void __launch_bounds__(THREADS, 1)
project_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b0,
                  const __grid_constant__ CUtensorMap map_b1, const EpiParams p) {
    using GE = Geo<BN>;
    constexpr int STAGES = GE::STAGES;
    constexpr int STAGE_BYTES = GE::STAGE_BYTES;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024 - (raw & 1023)) & 1023);   // 1024-byte aligned tile base
    const uint32_t tiles_u32 = smem_u32(smem);
    Barriers* sb = reinterpret_cast<Barriers*>(smem + GE::SMEM_TILES);
    float* s_cw = reinterpret_cast<float*>(smem + GE::SMEM_TILES + 1024);
    float* s_xb = reinterpret_cast<float*>(smem + GE::SMEM_TILES + 1024 + GE::CW_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int KB = p.d_mem / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sb->full[s], 1);
            mbar_init(&sb->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sb->tfull[a], 1);
            mbar_init(&sb->tempty[a], 4);
        }
        mbar_init(&sb->drain, 1);
        sb->abort_flag = 0;
        sb->issued = 0;
        sb->consumed = 0;
        mbar_fence_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b0);
        if (MODE == MODE_KV) tma_prefetch_desc(&map_b1);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sb->tmem_base)),
                     "r"(GE::TMEM_COLS)
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
            int it = 0;
            for (int tile = blockIdx.x; tile < p.num_tiles && !sb->abort_flag; tile += gridDim.x) {
                const int mt = tile / p.n_groups, nt = tile % p.n_groups;
                const int m0 = mt * p.m_stride - p.halo;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!wait_bounded(&sb->empty[s], ph ^ 1u, sb, p.status)) break;
                    const uint32_t a_dst = tiles_u32 + s * STAGE_BYTES;
                    const uint32_t b_dst = a_dst + A_BYTES;
                    mbar_arrive_expect_tx(&sb->full[s], STAGE_BYTES);
                    tma_load_2d(&map_a, a_dst, &sb->full[s], kb * BK, m0);
                    if (MODE == MODE_KV) {
                        tma_load_2d(&map_b0, b_dst, &sb->full[s], kb * BK, nt * 128);
                        tma_load_2d(&map_b1, b_dst + 128 * BK * 2, &sb->full[s], kb * BK, nt * 128);
                    } else {
                        tma_load_2d(&map_b0, b_dst, &sb->full[s], kb * BK, nt * BN);
                    }
                    sb->issued = it + 1;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            int it = 0, tc = 0;
            for (int tile = blockIdx.x; tile < p.num_tiles && !sb->abort_flag; tile += gridDim.x, ++tc) {
                const int acc = tc & 1;
                const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
                if (!wait_bounded(&sb->tempty[acc], aph ^ 1u, sb, p.status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!wait_bounded(&sb->full[s], ph, sb, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = tiles_u32 + s * STAGE_BYTES;
                    const uint64_t da = smem_desc_sw128(a_addr);
                    const uint64_t db = smem_desc_sw128(a_addr + A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk) {
                        // +32 bytes along K inside the swizzled 128-byte row
                        umma_bf16<BN>(d_tmem, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), (kb | kk) != 0);
                    }
                    umma_commit(&sb->empty[s]);
                    sb->consumed = it + 1;
                }
                if (!ok) break;
                umma_commit(&sb->tfull[acc]);
            }
        }
    } else if (warp >= 4) {
        // ---------------- epilogue
        const int q = warp - 4;
        int tc = 0;
        uint32_t xcount = 0;
        for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tc) {
            const int acc = tc & 1;
            const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
            const bool ok = wait_bounded(&sb->tfull[acc], aph, sb, p.status);
            if (epi_any(!ok)) break;          // one decision for all four warps
            tc_fence_after();
            const int mt = tile / p.n_groups, nt = tile % p.n_groups;
            const int m0 = mt * p.m_stride - p.halo;
            const uint32_t taddr = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
            if (MODE == MODE_KV) epilogue_kv(taddr, p, m0, nt, q, lane);
            if (MODE == MODE_K) epilogue_k<BN>(taddr, p, m0, nt, q, lane);
            if (MODE == MODE_VCONV) epilogue_vconv<BN>(taddr, p, m0, nt, q, lane, tc, xcount, s_cw, s_xb);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb->tempty[acc]);
        }
    }

    __syncthreads();
    if (sb->abort_flag) {
        // drain: copies this CTA issued but the MMA never consumed, then the MMAs
        if (warp == 0 && lane == 0) {
            for (int it = sb->consumed; it < sb->issued; ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                const long long t0 = clock64();
                while (!mbar_try_wait(smem_u32(&sb->full[s]), ph) && clock64() - t0 < kWaitCycles) {
                }
            }
        }
        if (warp == 1 && lane == 0) {
            umma_commit(&sb->drain);
            const long long t0 = clock64();
            while (!mbar_try_wait(smem_u32(&sb->drain), 0) && clock64() - t0 < kWaitCycles) {
            }
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(GE::TMEM_COLS)
                     : "memory");
    }
}

// merge the new conv history: rows of the old history that are still inside
// the window (L < w-1) shift down; the rest come from state_next.  In order
// of increasing row, so the update is in place.
__global__ void state_merge_kernel(float* state, const float* state_next, int B, int L, int H, int d) {
    const int64_t n = (int64_t)B * d;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += (int64_t)gridDim.x * blockDim.x) {
        const int64_t b = k / d, c = k - b * d;
        for (int i = 0; i < H; ++i) {
            const int p = L - H + i;
            const float val = p >= 0 ? state_next[(b * H + i) * d + c] : state[(b * H + (L + i)) * d + c];
            state[(b * H + i) * d + c] = val;
        }
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* q = nullptr;
        cudaDriverEntryPointQueryResult res;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &res) == cudaSuccess &&
            res == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(q);
    }
    return fn;
}

// 2-D bf16 row-major [rows][cols] map with a box of box_rows x 64 columns
// (128 bytes, 128-byte swizzle); rows outside [0, rows) read as zero.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int BN>
cudaError_t launch_mode(const CUtensorMap& ma, const CUtensorMap& mb0, const CUtensorMap& mb1, EpiParams p,
                        int64_t m_tiles, int num_sms, cudaStream_t s) {
    using GE = Geo<BN>;
    static unsigned long long attr_set = 0;   // one bit per device ordinal
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !(attr_set >> dev & 1ull)) {
        cudaError_t err = cudaFuncSetAttribute(project_tc_kernel<MODE, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               GE::SMEM_BYTES);
        if (err != cudaSuccess) return err;
        attr_set |= 1ull << dev;
    }
    const int64_t tiles = m_tiles * p.n_groups;
    if (tiles >= (int64_t)1 << 31) return cudaErrorInvalidValue;
    p.num_tiles = (int)tiles;
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    project_tc_kernel<MODE, BN><<<grid, THREADS, GE::SMEM_BYTES, s>>>(ma, mb0, mb1, p);
    return cudaGetLastError();
}

int pick_bn(int32_t d) { return d % 256 == 0 ? 256 : 128; }

}  // namespace

bool project_tc_supported(int64_t n_tok, int32_t d_mem, int32_t d) {
    return n_tok > 0 && n_tok < (int64_t)1 << 30 && d_mem % BK == 0 && d_mem >= BK && d % 128 == 0 &&
           encode_fn() != nullptr;
}

cudaError_t launch_project_tc(const void* e, int64_t n_tok, int32_t d_mem, const void* h, const void* Wk,
                              const void* Wv, const float* gq, const float* gk, int32_t d, float* v, float* part,
                              uint32_t* status, int num_sms, cudaStream_t s) {
    if (!project_tc_supported(n_tok, d_mem, d)) return cudaErrorNotSupported;
    CUtensorMap ma, mk, mv;
    if (!make_map(&ma, e, (uint64_t)n_tok, (uint64_t)d_mem, BM) || !make_map(&mk, Wk, (uint64_t)d, (uint64_t)d_mem, 128) ||
        !make_map(&mv, Wv, (uint64_t)d, (uint64_t)d_mem, 128))
        return cudaErrorInvalidValue;
    EpiParams p{};
    p.h = static_cast<const __nv_bfloat16*>(h);
    p.gq = gq;
    p.gk = gk;
    p.v = v;
    p.part = reinterpret_cast<float4*>(part);
    p.status = status;
    p.n_tok = (int)n_tok;
    p.d_mem = d_mem;
    p.d = d;
    p.G = d / 128;
    p.n_groups = d / 128;
    p.m_stride = BM;
    p.halo = 0;
    return launch_mode<MODE_KV, 256>(ma, mk, mv, p, (n_tok + BM - 1) / BM, num_sms, s);
}

cudaError_t launch_gate_k_tc(const void* e, int64_t n_tok, int32_t d_mem, const void* h, const void* Wk,
                             const float* gq, const float* gk, int32_t d, float* part, uint32_t* status, int num_sms,
                             cudaStream_t s) {
    if (!project_tc_supported(n_tok, d_mem, d)) return cudaErrorNotSupported;
    const int bn = pick_bn(d);
    CUtensorMap ma, mk;
    if (!make_map(&ma, e, (uint64_t)n_tok, (uint64_t)d_mem, BM) || !make_map(&mk, Wk, (uint64_t)d, (uint64_t)d_mem, bn))
        return cudaErrorInvalidValue;
    EpiParams p{};
    p.h = static_cast<const __nv_bfloat16*>(h);
    p.gq = gq;
    p.gk = gk;
    p.part = reinterpret_cast<float4*>(part);
    p.status = status;
    p.n_tok = (int)n_tok;
    p.d_mem = d_mem;
    p.d = d;
    p.G = d / 128;
    p.n_groups = d / bn;
    p.m_stride = BM;
    p.halo = 0;
    const int64_t mt = (n_tok + BM - 1) / BM;
    return bn == 256 ? launch_mode<MODE_K, 256>(ma, mk, mk, p, mt, num_sms, s)
                     : launch_mode<MODE_K, 128>(ma, mk, mk, p, mt, num_sms, s);
}

cudaError_t launch_vconv_tc(const void* e, int32_t B, int32_t L, int32_t d_mem, const void* h, const void* Wv,
                            const float* conv_w, int32_t d, int32_t w, float eps, const float* part,
                            const float* state, float* state_next, void* y, float* alpha_out, int32_t add_residual,
                            uint32_t* status, int num_sms, cudaStream_t s) {
    const int64_t n_tok = (int64_t)B * L;
    if (!project_tc_supported(n_tok, d_mem, d) || w < 1 || w > kMaxConv) return cudaErrorNotSupported;
    const int bn = pick_bn(d);
    const int H = w - 1;
    CUtensorMap ma, mv;
    if (!make_map(&ma, e, (uint64_t)n_tok, (uint64_t)d_mem, BM) || !make_map(&mv, Wv, (uint64_t)d, (uint64_t)d_mem, bn))
        return cudaErrorInvalidValue;
    EpiParams p{};
    p.h = static_cast<const __nv_bfloat16*>(h);
    p.part = const_cast<float4*>(reinterpret_cast<const float4*>(part));
    p.conv_w = conv_w;
    p.state = state;
    p.state_next = state ? state_next : nullptr;
    p.y = static_cast<__nv_bfloat16*>(y);
    p.alpha_out = alpha_out;
    p.status = status;
    p.n_tok = (int)n_tok;
    p.d_mem = d_mem;
    p.d = d;
    p.G = d / 128;
    p.n_groups = d / bn;
    p.L = L;
    p.w = w;
    p.add_residual = add_residual;
    p.eps = eps;
    // row tiles overlap by the H history rows
    p.m_stride = BM - H;
    p.halo = H;
    const int64_t mt = (n_tok + p.m_stride - 1) / p.m_stride;
    return bn == 256 ? launch_mode<MODE_VCONV, 256>(ma, mv, mv, p, mt, num_sms, s)
                     : launch_mode<MODE_VCONV, 128>(ma, mv, mv, p, mt, num_sms, s);
}

cudaError_t launch_state_merge(float* state, const float* state_next, int32_t B, int32_t L, int32_t w, int32_t d,
                               int num_sms, cudaStream_t s) {
    const int H = w - 1;
    if (H <= 0 || B == 0) return cudaSuccess;
    const int64_t n = (int64_t)B * d;
    int64_t blocks = (n + 255) / 256;
    if (blocks > num_sms * 8) blocks = num_sms * 8;
    state_merge_kernel<<<(unsigned)blocks, 256, 0, s>>>(state, state_next, B, L, H, d);
    return cudaGetLastError();
}

}  // namespace engram
