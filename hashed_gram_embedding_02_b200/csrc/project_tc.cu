// Key/value projections on the 5th-generation tensor cores (tcgen05), with
// the gate's partial sums in the epilogue.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": k_t = W_K e_t and
// v_t = W_V e_t feed an RMSNorm'd dot product with the query h_t (the
// multi-branch variant fuses all projections into one dense GEMM "to maximise
// GPU utilisation").  Here one GEMM computes [k | v] = e [W_K; W_V]^T:
//
//   A = e      [n_tok][d_mem] bf16, K-major
//   B = W_K, W_V [d][d_mem]   bf16, K-major (nn.Linear layout)
//   CTA tile   128 rows x (128 k-channels + the same 128 v-channels), K step 64
//
// Persistent kernel, one CTA per SM, warp-specialised:
//   warp 0     TMA producer: 2-D tiled loads (128-byte swizzle) of the A tile
//              and of the W_K and W_V tiles into a 4-stage shared-memory ring
//   warp 1     allocates 512 TMEM columns (two 128x256 fp32 accumulators) and
//              issues tcgen05.mma kind::f16 (M=128, N=256, K=16) from one thread
//   warps 4-7  epilogue: tcgen05.ld of the accumulator rows (warp w reads TMEM
//              lanes 32(w-4)..32(w-4)+31), store v as bf16, and reduce the
//              group's gate partials (sum g_q g_k h k, sum k^2, sum h^2); the
//              key k never leaves the SM
// The double-buffered accumulator lets the epilogue of tile i overlap the
// MMAs of tile i+1.  Tiles run channel-group-fastest so that consecutive tiles
// share the A block in L2; all of W stays L2-resident.
//
// Every mbarrier wait is bounded (about 2 s of clock64 time).  A wait that runs
// out sets ENGRAM_ERR_TIMEOUT, raises a CTA-wide abort flag that makes the
// other roles leave their loops, drains the copies and MMAs this CTA issued
// (bounded again), frees the TMEM and returns.
#include <cuda.h>

#include "common.cuh"

namespace engram {

namespace {

constexpr int BM = 128;                 // rows per tile (UMMA M)
constexpr int BNH = 128;                // channels per tile (k and v halves)
constexpr int BN = 2 * BNH;             // UMMA N
constexpr int BK = 64;                  // K per stage: 64 bf16 = 128 bytes = one swizzle row
constexpr int UK = 16;                  // K per tcgen05.mma kind::f16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;    // 16 KB
constexpr int B_BYTES = BN * BK * 2;    // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;       // two accumulators
constexpr int THREADS = 256;
constexpr int SMEM_TILES = STAGES * STAGE_BYTES;
constexpr int SMEM_BYTES = SMEM_TILES + 1024 /* barriers */ + 1024 /* alignment slack */;
constexpr long long WAIT_CYCLES = 4000000000LL;   // ~2 s at 1.9 GHz

struct __align__(8) Barriers {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort_flag;
    int issued;       // k-block loads issued by the producer
    int consumed;     // k-block stages consumed by the MMA issuer
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: true when the phase with `parity` completed, false when the
// CTA aborted or the wait ran out (then the status bit and abort flag are set).
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, Barriers* sb, uint32_t* status) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(a, parity)) return true;
        if (sb->abort_flag) return false;
        if (clock64() - t0 > WAIT_CYCLES) {
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
// K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n"
        ::"r"(tmem_d), "l"(da), "l"(db), "r"(kIdesc), "r"(accumulate));
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

__global__ void __launch_bounds__(THREADS, 1)
project_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_wk,
                  const __grid_constant__ CUtensorMap map_wv, const __nv_bfloat16* __restrict__ h,
                  const float* __restrict__ gq, const float* __restrict__ gk, __nv_bfloat16* __restrict__ v,
                  float4* __restrict__ part, uint32_t* status, int n_tok, int d_mem, int d, int G, int num_tiles) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024 - (raw & 1023)) & 1023);   // 1024-byte aligned tile base
    const uint32_t tiles_u32 = smem_u32(smem);
    Barriers* sb = reinterpret_cast<Barriers*>(smem + SMEM_TILES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int KB = d_mem / BK;

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
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_wk);
        tma_prefetch_desc(&map_wv);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sb->tmem_base)),
                     "r"(TMEM_COLS)
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
            for (int tile = blockIdx.x; tile < num_tiles && !sb->abort_flag; tile += gridDim.x) {
                const int m0 = (tile / G) * BM;
                const int c0 = (tile % G) * BNH;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!wait_bounded(&sb->empty[s], ph ^ 1u, sb, status)) break;
                    const uint32_t a_dst = tiles_u32 + s * STAGE_BYTES;
                    const uint32_t b_dst = a_dst + A_BYTES;
                    mbar_arrive_expect_tx(&sb->full[s], STAGE_BYTES);
                    tma_load_2d(&map_a, a_dst, &sb->full[s], kb * BK, m0);
                    tma_load_2d(&map_wk, b_dst, &sb->full[s], kb * BK, c0);
                    tma_load_2d(&map_wv, b_dst + BNH * BK * 2, &sb->full[s], kb * BK, c0);
                    sb->issued = it + 1;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            int it = 0, tc = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !sb->abort_flag; tile += gridDim.x, ++tc) {
                const int acc = tc & 1;
                const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
                if (!wait_bounded(&sb->tempty[acc], aph ^ 1u, sb, status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!wait_bounded(&sb->full[s], ph, sb, status)) {
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
                        umma_bf16(d_tmem, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), (kb | kk) != 0);
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
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tc) {
            const int acc = tc & 1;
            const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
            if (!wait_bounded(&sb->tfull[acc], aph, sb, status)) break;
            tc_fence_after();
            const int g = tile % G;
            const int c0 = g * BNH;
            const int64_t row = (int64_t)(tile / G) * BM + q * 32 + lane;
            const bool valid = row < n_tok;
            const uint32_t taddr = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
            float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
#pragma unroll 1
            for (int ch = 0; ch < BNH / 32; ++ch) {
                uint32_t kr[32];
                tmem_ld32(taddr + ch * 32, kr);
                tmem_wait_ld();
                if (valid) {
                    const uint4* hp = reinterpret_cast<const uint4*>(h + row * d + c0 + ch * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint4 hv = __ldg(hp + u);
                        const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
#pragma unroll
                            for (int half = 0; half < 2; ++half) {
                                const int i = u * 8 + p * 2 + half;
                                const int c = c0 + ch * 32 + i;
                                const float hf = half ? bf16_hi(hw[p]) : bf16_lo(hw[p]);
                                const float kf = __uint_as_float(kr[i]);
                                const float gg = (gq ? __ldg(gq + c) : 1.f) * (gk ? __ldg(gk + c) : 1.f);
                                s_qk = fmaf(gg * hf, kf, s_qk);
                                s_kk = fmaf(kf, kf, s_kk);
                                s_hh = fmaf(hf, hf, s_hh);
                            }
                        }
                    }
                }
            }
#pragma unroll 1
            for (int ch = 0; ch < BNH / 32; ++ch) {
                uint32_t vr[32];
                tmem_ld32(taddr + BNH + ch * 32, vr);
                tmem_wait_ld();
                if (valid) {
                    uint4* vp = reinterpret_cast<uint4*>(v + row * d + c0 + ch * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint4 o;
                        o.x = pack_bf16x2(__uint_as_float(vr[u * 8 + 0]), __uint_as_float(vr[u * 8 + 1]));
                        o.y = pack_bf16x2(__uint_as_float(vr[u * 8 + 2]), __uint_as_float(vr[u * 8 + 3]));
                        o.z = pack_bf16x2(__uint_as_float(vr[u * 8 + 4]), __uint_as_float(vr[u * 8 + 5]));
                        o.w = pack_bf16x2(__uint_as_float(vr[u * 8 + 6]), __uint_as_float(vr[u * 8 + 7]));
                        vp[u] = o;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb->tempty[acc]);
            if (valid) part[row * G + g] = make_float4(s_qk, s_kk, s_hh, 0.f);
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
                while (!mbar_try_wait(smem_u32(&sb->full[s]), ph) && clock64() - t0 < WAIT_CYCLES) {
                }
            }
        }
        if (warp == 1 && lane == 0) {
            umma_commit(&sb->drain);
            const long long t0 = clock64();
            while (!mbar_try_wait(smem_u32(&sb->drain), 0) && clock64() - t0 < WAIT_CYCLES) {
            }
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
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
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D bf16 row-major [rows][cols] map with a box of box_rows x 64 columns
// (128 bytes, 128-byte swizzle); rows beyond `rows` read as zero.
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

}  // namespace

bool project_tc_supported(int64_t n_tok, int32_t d_mem, int32_t d) {
    return n_tok > 0 && n_tok < (int64_t)1 << 31 && d_mem % BK == 0 && d_mem >= BK && d % BNH == 0 &&
           encode_fn() != nullptr;
}

cudaError_t launch_project_tc(const void* e, int64_t n_tok, int32_t d_mem, const void* h, const void* Wk,
                              const void* Wv, const float* gq, const float* gk, int32_t d, void* v, float* part,
                              uint32_t* status, int num_sms, cudaStream_t s) {
    if (!project_tc_supported(n_tok, d_mem, d)) return cudaErrorNotSupported;
    CUtensorMap ma, mk, mv;
    if (!make_map(&ma, e, (uint64_t)n_tok, (uint64_t)d_mem, BM) || !make_map(&mk, Wk, (uint64_t)d, (uint64_t)d_mem, BNH) ||
        !make_map(&mv, Wv, (uint64_t)d, (uint64_t)d_mem, BNH))
        return cudaErrorInvalidValue;
    static unsigned long long attr_set = 0;   // one bit per device ordinal
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !(attr_set >> dev & 1ull)) {
        cudaError_t err = cudaFuncSetAttribute(project_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (err != cudaSuccess) return err;
        attr_set |= 1ull << dev;
    }
    const int G = d / BNH;
    const int64_t m_blocks = (n_tok + BM - 1) / BM;
    const int64_t tiles = m_blocks * G;
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    project_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(ma, mk, mv, static_cast<const __nv_bfloat16*>(h), gq, gk,
                                                        static_cast<__nv_bfloat16*>(v), reinterpret_cast<float4*>(part),
                                                        status, (int)n_tok, d_mem, d, G, (int)tiles);
    return cudaGetLastError();
}

}  // namespace engram
