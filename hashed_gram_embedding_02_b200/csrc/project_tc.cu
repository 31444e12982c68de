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
//              (sum g_q g_k h k, sum k^2, sum h^2) of its channel groups;
//              k never leaves the SM.
//   MODE_VCONV tile = 4 row segments x BN v-channels.  Each epilogue warp owns
//              32 TMEM lanes = 3 history rows + 29 output rows, so a row's
//              conv history (rows t-1..t-3) sits in the same warp: v~ =
//              alpha v is formed per lane and the history arrives by warp
//              shuffles.  Taps, SiLU and the residual follow (all fp32) and
//              Y is written;
//              v never reaches global memory.  Consecutive segments overlap
//              by 3 rows (116 output rows per 128-row MMA tile).  On CTA
//              pairs (bf16, K >= 2048) the tile is instead 128 contiguous
//              rows per CTA (3 history rows, then 125 output rows): the
//              first three rows of warps 1-3 take their history from the
//              previous warp's last three through shared-memory halo slots.
//
// Persistent kernel, one CTA per SM, warp-specialised (640 threads):
//   warp 0     TMA producer: 2-D tiled loads (128-byte swizzle) of A (e) and
//              W into a shared-memory ring; in MODE_K/MODE_KV also the tile's
//              h slice into a shared buffer the epilogue reads (issued after
//              the tile's k-blocks, so it never holds back the MMA)
//   warp 1     allocates TMEM (two fp32 accumulators) and issues
//              tcgen05.mma kind::f16 (M=128, N=BN, K=16) from one thread
//   warp 2     MODE_VCONV: loads each channel half of the tile's h slice as
//              soon as the epilogue has released it
//   warps 4-19 epilogue: warp w reads TMEM lanes 32(w%4) .. 32(w%4)+31;
//              the four groups of four warps take four column parts of
//              the tile's channels
// The double-buffered accumulator lets the epilogue of tile i overlap the
// MMAs of tile i+1.  Tiles run channel-fastest so consecutive tiles share the
// A block in L2; W stays L2-resident, and h, read once per pass, is loaded
// with an evict-first hint.  In engram_forward the key pass is a
// programmatic dependent of the retrieval and the value pass one of the key
// pass: only the value epilogue's read of alpha waits for the key pass.
//
// Every mbarrier wait is bounded (about 2 s of clock64 time).  A wait that runs
// out sets ENGRAM_ERR_TIMEOUT, raises a CTA-wide abort flag that makes the
// other roles leave their loops, drains the copies and MMAs this CTA issued
// (bounded again), frees the TMEM and returns.
#include "tc.cuh"

namespace engram {

namespace {

constexpr int MODE_KV = 0;
constexpr int MODE_K = 1;
constexpr int MODE_VCONV = 2;

constexpr int BM = 128;                 // rows per tile (UMMA M)
constexpr int BK = 64;                  // K per stage: 64 bf16 = 128 bytes = one swizzle row
constexpr int UK = 16;                  // K per tcgen05.mma kind::f16
// FP8 (E4M3) operands: the same 128-byte swizzle rows hold 128 elements, and
// one tcgen05.mma kind::f8f6f4 covers K = 32 (32 bytes, like 16 bf16)
template <bool F8> struct Elt {
    static constexpr int BKE = F8 ? 128 : 64;   // K elements per stage
};
constexpr int A_BYTES = BM * BK * 2;    // 16 KB
constexpr int THREADS = 640;            // warps 0-3 producer / MMA / idle, warps 4-19 epilogue
constexpr int EPI_WARPS = 16;           // four per TMEM lane quarter
constexpr int EPI_THREADS = EPI_WARPS * 32;
constexpr int NPART = EPI_WARPS / 4;    // column parts per tile
constexpr int CONV_W = 4;               // conv width of the fused epilogue
constexpr int SEG = 32;                 // rows per epilogue warp
constexpr int SEG_OUT = SEG - (CONV_W - 1);   // output rows per warp segment (29)
constexpr int TILE_OUT = 4 * SEG_OUT;         // output rows per value tile (116)
// The value pass on CTA pairs reads each CTA's 128 rows as one contiguous
// block (3 history rows, then 125 output rows); a warp's first three rows
// take their conv history from the previous warp's last three (halo slots
// in shared memory)
constexpr int TILE_OUT_C = BM - (CONV_W - 1);   // output rows per contiguous value tile (125)
constexpr int HALO_SLOTS = 4;                   // (tile parity, channel half)

// PAIR: a cluster of two CTAs runs one M = 256 tcgen05 MMA (cta_group::2);
// each CTA stages its own 128 rows of A and half of the BN columns of W, so a
// stage costs each CTA 32 KB instead of 48 KB and four stages fit.
template <int MODE, int BN, bool PAIR = false>
struct Geo {
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;          // W rows (channels) this CTA stages
    static constexpr int B_BYTES = B_ROWS * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = PAIR ? 4 : (BN == 256 ? 3 : 4);
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int SMEM_TILES = STAGES * STAGE_BYTES;
    static constexpr int HC = MODE == MODE_KV ? 128 : BN;      // h channels per tile
    static constexpr int H_BYTES = BM * HC * 2;                // h tile, [HC/64][128 rows][128 B] swizzled
    // tiles | h tile | barriers (1 KB) | per-tile gains [HC] fp32 or taps |
    // partial hand-over [NPART][128] float4 | slack
    // MODE_VCONV: the gains area and the partial hand-over together hold the
    // epilogue warps' fp32 taps, 16 warps x 2 phases x BN/16 pairs x 32 bytes
    // MODE_VCONV on pairs (contiguous tiles): the warps stage the taps of one
    // phase at a time (16 warps x BN/16 pairs x 32 bytes, the gains area
    // alone), and the halo slots follow:
    // [slot][warp q < 3][part][3 rows][BN/8 channels] fp32
    static constexpr bool CONTIG = MODE == MODE_VCONV && PAIR;
    static constexpr int GG_BYTES = MODE == MODE_VCONV ? BN * 32 : BN * 16;
    static constexpr int RED_BYTES = CONTIG ? 0 : NPART * BM * 16;
    static constexpr int HALO_PW = BN / (2 * NPART);   // channels of one part in one phase
    static constexpr int HALO_BYTES = CONTIG ? HALO_SLOTS * 3 * NPART * 3 * HALO_PW * 4 : 0;
    static constexpr int SMEM_BYTES = SMEM_TILES + H_BYTES + 1024 + GG_BYTES + RED_BYTES + HALO_BYTES + 1024;
};

struct __align__(8) Barriers {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t pfull[8];    // PAIR, leader: the peer's stage is full (one remote arrival)
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t hfull;
    uint64_t hempty;
    uint64_t hfull_v[2];    // MODE_VCONV: the two channel halves of the tile's h slice
    uint64_t hempty_v[2];
    uint64_t drain;
    uint64_t hx[HALO_SLOTS][3][NPART];   // contiguous value tiles: warp q's halo rows are in the slot
    uint32_t tmem_base;
    volatile int abort_flag;
    int issued;       // k-block loads issued by the producer
    int consumed;     // k-block stages consumed by the MMA issuer
    int h_issued;     // h tiles issued
    int h_consumed;   // h tiles released by the epilogue
    int band_last;    // this CTA completed a row band's partials (MODE_K)
    int h_issued_v[2];      // MODE_VCONV: h halves issued / released, per half
    int h_consumed_v[2];
    uint32_t peer_abort;   // PAIR: cluster address of the other CTA's abort_flag, else 0
};

struct EpiParams {
    const float* gq;            // [d] or null
    const float* gk;            // [d] or null
    float* v;                   // MODE_KV: [n_tok][d] fp32
    float4* part;               // [n_tok][G]: written (KV, K)
    const float* alpha;         // MODE_VCONV: [n_tok] gate values
    const float* conv_w;        // [d][4]
    const float* state;         // history, or null (zero history): [B][3][d], or [3][d][B] with state_tr
    float* state_next;          // new history (merged by a second kernel), or null; same layout as state
    int state_tr;               // history in the sequence-minor layout [3][d][B] (decode: lanes = sequences)
    int B;
    __nv_bfloat16* y;           // [n_tok][d]
    uint32_t* status;
    int n_tok, d_mem, d, G;
    int n_groups;               // tiles along the channel dimension
    int num_tiles;
    int L;                      // rows per sequence
    int add_residual;
    int* band_count;            // MODE_K: per row band, channel tiles done (zero on entry, zero on exit)
    int stall;                  // test hook: CTA 0 announces its first stage but never loads it
    float* alpha_w;             // MODE_K: [n_tok] gate values written by each band's last CTA
    float* alpha_out;           // MODE_K: caller's copy of alpha, or null
    float eps;
    // multi-branch: M residual branches share e and W_V and have their own
    // W_K (stacked [M*d][d_mem]), h, gains, gate, conv history and Y, each
    // [M][...] with the single-branch layout per branch
    int M;
    int Gb;                     // 128-channel groups per branch (d / 128); G = M * Gb in MODE_K
    // per output channel dequantisation of the accumulators (null: none):
    // k = kscale[c] * acc over the stacked [M*d] key channels, v = vscale[c] * acc
    const float* kscale;
    const float* vscale;
    // tile order: 0 = channel-fastest (a row band's tiles run together, A is
    // read once); rb > 0 = groups of rb row units per channel tile, so that a
    // W slice is reused by rb bands in a row (wide N: the stacked W_K of
    // several branches does not stay in L2 under channel-fastest order)
    int raster_rb;
};

constexpr int kMaxBranches = ENGRAM_MAX_BRANCHES;

// Bounded wait: true when the phase with `parity` completed, false when the
// CTA aborted or the wait ran out (then the status bit and abort flag are set).
// CLUSTER: the barrier also receives arrivals from the other CTA of a pair
// (acquire at cluster scope).  A timeout also raises the peer's abort flag.
template <bool CLUSTER = false>
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, Barriers* sb, uint32_t* status) {
    const uint32_t a = smem_u32(bar);
    auto try_wait = [&]() { return CLUSTER ? mbar_try_wait_cluster(a, parity) : mbar_try_wait(a, parity); };
    if (try_wait()) return true;
    const long long t0 = clock64();
    while (true) {
        if (try_wait()) return true;
        if (sb->abort_flag) return false;
        if (clock64() - t0 > kWaitCycles) {
            flag(status, ENGRAM_ERR_TIMEOUT);
            sb->abort_flag = 1;
            if (sb->peer_abort) st_remote_s32(sb->peer_abort, 1);
            return false;
        }
    }
}

// named barrier among the epilogue warps (id 1; id 0 is __syncthreads)
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory"); }

// the same barrier as a vote: true on every epilogue thread when any passed true
__device__ __forceinline__ bool epi_any(bool x) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)x), "n"(EPI_THREADS)
        : "memory");
    return r != 0;
}

// 8 channels (16 bytes) of row i at tile-local channel cl (cl % 8 == 0) from
// the h tile: boxes of 64 channels x 128 rows, 128-byte rows, 16-byte chunks
// XOR-swizzled by the row index (the TMA 128-byte swizzle pattern)
__device__ __forceinline__ uint4 h_chunk(const uint8_t* hs, int i, int cl) {
    const int cb = cl >> 6;
    const int ck = (cl & 63) >> 3;
    return *reinterpret_cast<const uint4*>(hs + cb * (BM * 128) + i * 128 + ((ck ^ (i & 7)) << 4));
}

__device__ __forceinline__ uint4* h_chunk_ptr(uint8_t* hs, int i, int cl) {
    const int cb = cl >> 6;
    const int ck = (cl & 63) >> 3;
    return reinterpret_cast<uint4*>(hs + cb * (BM * 128) + i * 128 + ((ck ^ (i & 7)) << 4));
}

__device__ __forceinline__ void unpack8(const uint4& q, float* f) {
    f[0] = bf16_lo(q.x); f[1] = bf16_hi(q.x);
    f[2] = bf16_lo(q.y); f[3] = bf16_hi(q.y);
    f[4] = bf16_lo(q.z); f[5] = bf16_hi(q.z);
    f[6] = bf16_lo(q.w); f[7] = bf16_hi(q.w);
}

// ---------------------------------------------------------------- epilogues

// Gate partials of row i over `ncols` k columns (multiple of 32) starting at
// TMEM column taddr and tile-local channel cl; gains s_gg and the key
// channels' dequantisation scales s_ks indexed tile-locally.  TMEM loads run
// one 16-column chunk ahead of the math.
template <bool SCALED>
__device__ __forceinline__ void partials_cols(uint32_t taddr, const uint8_t* hs, int i, bool valid, int cl,
                                              int ncols, const float* s_gg, const float* s_ks, float& s_qk,
                                              float& s_kk, float& s_hh) {
    uint32_t ka[16], kb[16];
    const int nch = ncols / 16;
    tmem_ld16(taddr, ka);
#pragma unroll 1
    for (int ch = 0; ch < nch; ch += 2) {
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
            uint32_t(&cur)[16] = sub ? kb : ka;
            uint32_t(&nxt)[16] = sub ? ka : kb;
            const int c = ch + sub;
            tmem_wait_ld(cur);
            if (c + 1 < nch) tmem_ld16(taddr + (c + 1) * 16, nxt);
            if (valid) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c8 = cl + c * 16 + u * 8;
                    float hf[8];
                    unpack8(h_chunk(hs, i, c8), hf);
                    const float4 g0 = *reinterpret_cast<const float4*>(s_gg + c8);
                    const float4 g1 = *reinterpret_cast<const float4*>(s_gg + c8 + 4);
                    const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                    float ks[8] = {1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f, 1.f};
                    if constexpr (SCALED) {
                        const float4 k0 = *reinterpret_cast<const float4*>(s_ks + c8);
                        const float4 k1 = *reinterpret_cast<const float4*>(s_ks + c8 + 4);
                        ks[0] = k0.x; ks[1] = k0.y; ks[2] = k0.z; ks[3] = k0.w;
                        ks[4] = k1.x; ks[5] = k1.y; ks[6] = k1.z; ks[7] = k1.w;
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float kf = SCALED ? __uint_as_float(cur[u * 8 + e]) * ks[e] : __uint_as_float(cur[u * 8 + e]);
                        s_qk = fmaf(gg[e] * hf[e], kf, s_qk);
                        s_kk = fmaf(kf, kf, s_kk);
                        s_hh = fmaf(hf[e], hf[e], s_hh);
                    }
                }
            }
        }
    }
}

// g_q * g_k of channels [c0, c0 + n) into s_gg (all epilogue threads)
__device__ __forceinline__ void load_gains(const EpiParams& p, int c0, int n, float* s_gg, int et) {
    for (int k = et; k < n; k += EPI_THREADS) {
        const int c = c0 + k;
        s_gg[k] = (p.gq ? __ldg(p.gq + c) : 1.f) * (p.gk ? __ldg(p.gk + c) : 1.f);
    }
}

// Partials over the channel slice [cl0, cl0 + ncols) of this warp's part,
// added across the parts of each 128-channel group in a fixed order through
// s_red, written by the group's first part.
template <bool SCALED>
__device__ __forceinline__ void group_partials(uint32_t taddr, const uint8_t* hs, const EpiParams& p, int64_t row,
                                               int i, bool valid, int part, int cl0, int ncols, int parts_per_group,
                                               int g, const float* s_gg, const float* s_ks, float4* s_red) {
    float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
    partials_cols<SCALED>(taddr, hs, i, valid, cl0, ncols, s_gg, s_ks, s_qk, s_kk, s_hh);
    s_red[part * BM + i] = make_float4(s_qk, s_kk, s_hh, 0.f);
    epi_sync();
    if (part % parts_per_group == 0 && valid) {
        float4 o = s_red[part * BM + i];
        for (int k = 1; k < parts_per_group; ++k) {
            const float4 x = s_red[(part + k) * BM + i];
            o.x += x.x;
            o.y += x.y;
            o.z += x.z;
        }
        p.part[row * p.G + g] = o;
    }
}

// [k | v] tile: parts 0-1 reduce the k half (128 channels, one group) into
// the group's partials, parts 2-3 store the v half (fp32).
__device__ __forceinline__ void epilogue_kv(uint32_t taddr, const uint8_t* hs, const EpiParams& p, int m0, int nt,
                                            int q, int part, int lane, int et, float* s_gg, float4* s_red) {
    const int i = q * 32 + lane;
    const int64_t row = (int64_t)m0 + i;
    const bool valid = row < p.n_tok;
    const int c0 = nt * 128;
    epi_sync();                       // previous tile's readers are done with s_gg and s_red
    load_gains(p, c0, 128, s_gg, et);
    epi_sync();
    if (part < 2) {
        float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
        partials_cols<false>(taddr + part * 64, hs, i, valid, part * 64, 64, s_gg, nullptr, s_qk, s_kk, s_hh);
        s_red[part * BM + i] = make_float4(s_qk, s_kk, s_hh, 0.f);
    } else {
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
            const int cl = (part - 2) * 64 + ch * 32;
            uint32_t vr[32];
            tmem_ld32(taddr + 128 + cl, vr);
            tmem_wait_ld();
            if (valid) {
                float4* vp = reinterpret_cast<float4*>(p.v + row * p.d + c0 + cl);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    vp[u] = make_float4(__uint_as_float(vr[4 * u]), __uint_as_float(vr[4 * u + 1]),
                                        __uint_as_float(vr[4 * u + 2]), __uint_as_float(vr[4 * u + 3]));
            }
        }
    }
    epi_sync();
    if (part == 0 && valid) {
        const float4 a = s_red[i], b = s_red[BM + i];
        p.part[row * p.G + nt] = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, 0.f);
    }
}

// Per-tile values the epilogue reads from global memory (the conv taps or the
// RMSNorm gains of the tile's channels, the gate of the thread's row), loaded
// one tile ahead so their latency hides behind the current tile's epilogue.
struct TilePre {
    float4 w0, w1;   // MODE_VCONV: taps of this lane's channel pair of its warp's part (see vconv_pair)
    float g;         // MODE_K: g_q * g_k of channel et
    float ks;        // MODE_K: dequantisation scale of key channel et
    float a;         // MODE_VCONV: alpha of this thread's row (branch 0; other branches load theirs in turn)
};

// The value epilogue's warp (q, part) uses, per phase, BN/(2 NPART) channels =
// VPP channel pairs; lane l of the warp loads pair l % 16 of phase l / 16
// (when it exists), so a warp stages its own taps and needs no barrier with
// the other warps.  Tile-local pair index of that lane, or -1.
template <int BN>
__device__ __forceinline__ int vconv_pair(int part, int lane) {
    constexpr int VPP = BN / (4 * NPART);
    const int ph = lane >> 4, k = lane & 15;
    return k < VPP ? ph * (BN / 4) + part * VPP + k : -1;
}

// first row of a value tile's lane quarter q (its lane 0), both layouts
template <bool CONTIG>
__device__ __forceinline__ int64_t vrow0(int mt, int q) {
    return CONTIG ? (int64_t)mt * TILE_OUT_C + q * 32 - (CONV_W - 1)
                  : (int64_t)mt * TILE_OUT + q * SEG_OUT - (CONV_W - 1);
}

template <int MODE, int BN, bool CONTIG = false>
__device__ __forceinline__ TilePre tile_pre_load(const EpiParams& p, int mt, int nt, int q, int lane, int et) {
    TilePre t{};
    const int n0 = nt * BN;
    if (MODE == MODE_VCONV) {
        const int pr = vconv_pair<BN>((et >> 5) >> 2, lane);
        if (pr >= 0) {
            t.w0 = __ldg(reinterpret_cast<const float4*>(p.conv_w) + n0 + 2 * pr);
            t.w1 = __ldg(reinterpret_cast<const float4*>(p.conv_w) + n0 + 2 * pr + 1);
        }
        const int64_t r = vrow0<CONTIG>(mt, q) + lane;
        t.a = (r >= 0 && r < p.n_tok) ? __ldg(p.alpha + r) : 0.f;
    } else if (MODE == MODE_K) {
        if (et < BN) {
            t.g = (p.gq ? __ldg(p.gq + n0 + et) : 1.f) * (p.gk ? __ldg(p.gk + n0 + et) : 1.f);
            t.ks = p.kscale ? __ldg(p.kscale + n0 + et) : 1.f;
        }
    }
    return t;
}

// k tile of BN channels: each of the NPART parts reduces BN/NPART columns,
// the parts of one 128-channel group are then added in order.
template <int BN, bool SCALED>
__device__ __forceinline__ void epilogue_k(uint32_t taddr, const uint8_t* hs, const EpiParams& p, int m0, int nt,
                                           int q, int part, int lane, int et, float* s_gg, float4* s_red,
                                           TilePre& pre, bool has_next, int mt_next, int nt_next) {
    constexpr int PW = BN / NPART;                    // columns per part
    constexpr int PPG = 128 / PW;                     // parts per 128-channel group
    const int i = q * 32 + lane;
    const int64_t row = (int64_t)m0 + i;
    const bool valid = row < p.n_tok;
    const int n0 = nt * BN;
    epi_sync();
    if (et < BN) {
        s_gg[et] = pre.g;
        if (SCALED) s_gg[BN + et] = pre.ks;
    }
    epi_sync();
    if (has_next) pre = tile_pre_load<MODE_K, BN>(p, mt_next, nt_next, q, lane, et);
    group_partials<SCALED>(taddr + part * PW, hs, p, row, i, valid, part, part * PW, PW, PPG, (n0 + part * PW) / 128, s_gg,
                   s_gg + BN, s_red);
}

// Gate + causal depthwise conv (width 4) + residual on a value tile of BN
// channels.  Lane l of warp segment q holds row r0q + l; lanes 0..2 are the
// history rows of the segment's first output row.  Each of the NPART parts
// handles BN/NPART channels, 16 at a time, TMEM loads one chunk ahead.
// Everything is fp32: v~ = alpha v per lane, the history rows t-1..t-3 by
// warp shuffles, the tap sum by fused multiply-adds in tap order, and
// SiLU(x) = x/2 + x/2 tanh(x/2) with the hardware tanh approximation
// (relative error about 2^-11, below the bf16 rounding of Y).  The taps
// arrive pre-halved, so the tap sum is already x/2.  Only Y is rounded, once,
// to bf16.
__device__ __forceinline__ float tanh_f32(float x) {
    float r;
    asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float mask_f(float x, uint32_t m) { return __uint_as_float(__float_as_uint(x) & m); }

// CONTIG: halo_r is the previous warp's slot (its last three rows' v~ over
// this part's channels of the phase, [3][NCH * 16]; null for the first
// warp, whose first three rows are history only).  MASK: some row of the
// warp is among its sequence's first three (the fast path then zeroes the
// history before the start; without such a row the masks are all ones and
// are skipped)
template <int NCH, bool SLOW, bool RES, bool SCALED, bool CONTIG = false, bool MASK = true>
__device__ __forceinline__ void vconv_chunks(uint32_t taddr, uint8_t* hs, const EpiParams& p, int i, int64_t r,
                                             int64_t b, int t, float a, bool out_row, int n0, int cbeg,
                                             const float4* s_cw, uint32_t m1, uint32_t m2, uint32_t m3, int br,
                                             const float* halo_r = nullptr) {
    constexpr int H = CONV_W - 1;
    // this branch's history and new history (the same size in both layouts)
    const int64_t hist_off = (int64_t)br * p.B * H * p.d;
    const float* state = p.state ? p.state + hist_off : nullptr;
    float* state_next = p.state_next ? p.state_next + hist_off : nullptr;
    const bool write_state = SLOW && state_next && out_row && t >= p.L - H;
    const bool from_state = SLOW && t < H && state;
    uint32_t va[16], vb[16];
    tmem_ld16(taddr + cbeg, va);
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
        uint32_t(&cur)[16] = (ch & 1) ? vb : va;
        uint32_t(&nxt)[16] = (ch & 1) ? va : vb;
        const int cl = cbeg + ch * 16;
        float hv[16];
        if (RES) {
            unpack8(h_chunk(hs, i, cl), hv);
            unpack8(h_chunk(hs, i, cl + 8), hv + 8);
        }
        tmem_wait_ld(cur);
        if (ch + 1 < NCH) tmem_ld16(taddr + cl + 16, nxt);
        float o[16];
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
            float v0 = a * __uint_as_float(cur[c]), v1 = a * __uint_as_float(cur[c + 1]);
            if constexpr (SCALED) {
                // warp-uniform address: one broadcast load per channel pair
                const float2 vs = __ldg(reinterpret_cast<const float2*>(p.vscale + n0 + cl + c));
                v0 *= vs.x;
                v1 *= vs.y;
            }
            float s1a = __shfl_up_sync(0xffffffffu, v0, 1), s1b = __shfl_up_sync(0xffffffffu, v1, 1);
            float s2a = __shfl_up_sync(0xffffffffu, v0, 2), s2b = __shfl_up_sync(0xffffffffu, v1, 2);
            float s3a = __shfl_up_sync(0xffffffffu, v0, 3), s3b = __shfl_up_sync(0xffffffffu, v1, 3);
            if (CONTIG && halo_r != nullptr && (i & 31) < 3) {
                // rows t-k before this warp's first row: slot row 3-k+lane
                // holds the previous warp's lane 29+(3-k+lane)
                const int ln = i & 31;
                const float* hr = halo_r + (cl + c - cbeg);
                constexpr int PWC = NCH * 16;
                if (ln < 1) {
                    s1a = hr[2 * PWC];
                    s1b = hr[2 * PWC + 1];
                }
                if (ln < 2) {
                    s2a = hr[(1 + ln) * PWC];
                    s2b = hr[(1 + ln) * PWC + 1];
                }
                s3a = hr[ln * PWC];
                s3b = hr[ln * PWC + 1];
            }
            if (!SLOW && MASK) {
                // rows before the sequence start (no conv_state): zero history
                s1a = mask_f(s1a, m1);
                s1b = mask_f(s1b, m1);
                s2a = mask_f(s2a, m2);
                s2b = mask_f(s2b, m2);
                s3a = mask_f(s3a, m3);
                s3b = mask_f(s3b, m3);
            }
            if (SLOW && t < H) {
                // history before the slab start: conv_state (zero without one);
                // the row t-k comes from state row H-k+t
                float2 ps[H] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                if (from_state) {
                    const int chn = n0 + cl + c;
#pragma unroll
                    for (int k = 1; k <= H; ++k)
                        if (t < k) {
                            const int hr = H - k + t;            // history row holding v~_{t-k}
                            if (p.state_tr) {                     // [3][d][B]: consecutive lanes, consecutive b
                                const float* st = state + ((int64_t)hr * p.d + chn) * p.B + b;
                                ps[k - 1] = make_float2(__ldg(st), __ldg(st + p.B));
                            } else {
                                ps[k - 1] = __ldg(reinterpret_cast<const float2*>(state + (b * H + hr) * p.d + chn));
                            }
                        }
                }
                if (t < 1) {
                    s1a = ps[0].x;
                    s1b = ps[0].y;
                }
                if (t < 2) {
                    s2a = ps[1].x;
                    s2b = ps[1].y;
                }
                s3a = ps[2].x;
                s3b = ps[2].y;
            }
            if (write_state) {
                const int hr = t - (p.L - H);
                const int chn = n0 + cl + c;
                if (p.state_tr) {
                    float* sn = state_next + ((int64_t)hr * p.d + chn) * p.B + b;
                    sn[0] = v0;
                    sn[p.B] = v1;
                } else {
                    *reinterpret_cast<float2*>(state_next + (b * H + hr) * p.d + chn) = make_float2(v0, v1);
                }
            }
            // halved taps of the channel pair: (c_0 ch0, c_0 ch1, c_1 ch0, c_1 ch1), (c_2 .., c_3 ..)
            const float4 wa = s_cw[(cl + c)], wb = s_cw[(cl + c) + 1];
            float hx0 = wa.x * v0, hx1 = wa.y * v1;
            hx0 = fmaf(wa.z, s1a, hx0);
            hx1 = fmaf(wa.w, s1b, hx1);
            hx0 = fmaf(wb.x, s2a, hx0);
            hx1 = fmaf(wb.y, s2b, hx1);
            hx0 = fmaf(wb.z, s3a, hx0);
            hx1 = fmaf(wb.w, s3b, hx1);
            const float sl0 = fmaf(hx0, tanh_f32(hx0), hx0);
            const float sl1 = fmaf(hx1, tanh_f32(hx1), hx1);
            o[c] = (RES ? v0 + hv[c] : v0) + sl0;
            o[c + 1] = (RES ? v1 + hv[c + 1] : v1) + sl1;
        }
        // Y replaces this row's h in the staged tile (each element of the tile
        // is read and written by one lane only); the warp stores its block
        // with row-contiguous lanes afterwards
        *h_chunk_ptr(hs, i, cl) = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                             pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
        *h_chunk_ptr(hs, i, cl + 8) = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]),
                                                 pack_bf16x2(o[12], o[13]), pack_bf16x2(o[14], o[15]));
    }
}

// The value tile's epilogue runs in two phases over the two channel halves of
// the tile, so that the h half of phase 0 can be refilled for the next tile
// while phase 1 runs; with M branches, 2M phases: both halves for branch 0,
// then for branch 1, ... (the accumulator holds v for all of them).  In each
// phase part `part` takes BN/8 channels.
//
// CONTIG (contiguous tiles, one branch): warp q < 3 first publishes the
// gated values of its last three rows over the part's channels in the
// phase's halo slot, and warp q > 0 waits for warp q-1's slot before its
// first three rows read their history from it.  Slots rotate over (tile
// parity, phase): a warp is never more than one tile ahead of another (the
// accumulator it needs next is released only by all of them), so a slot is
// rewritten only after its reader has finished that tile.  False when a
// wait ran out.
template <int BN, bool SCALED, bool CONTIG = false>
__device__ __forceinline__ bool epilogue_vconv(uint32_t taddr, uint8_t* hs, const EpiParams& p, int mt, int nt,
                                               int q, int part, int lane, int et, float* s_taps, int phase,
                                               float a, const TilePre& pre, int br, Barriers* sb = nullptr,
                                               float* s_halo = nullptr, int tc = 0) {
    constexpr int H = CONV_W - 1;
    const int i = q * 32 + lane;
    const int64_t r = vrow0<CONTIG>(mt, q) + lane;
    const bool in_range = r >= 0 && r < p.n_tok;
    const bool out_row = in_range && (lane >= H || (CONTIG && q > 0));
    int64_t b = 0;
    int t = 0;
    if (in_range) {
        b = r / p.L;
        t = (int)(r - b * p.L);
    }
    const int n0 = nt * BN;
    // the warp's own taps (both phases), halved, fp32: slot [warp][phase][pair]
    // holds two float4, (c_0, c_0', c_1, c_1') and (c_2, c_2', c_3, c_3') of
    // channels (2m, 2m+1); staged in phase 0 from the values loaded a tile
    // ahead, read by this warp only.  CONTIG stages one phase at a time
    // (slot [warp][pair]).
    constexpr int VPP = BN / (4 * NPART);
    float4* s_tw = reinterpret_cast<float4*>(s_taps) + (size_t)(q * NPART + part) * (CONTIG ? 1 : 2) * VPP * 2;
    if (CONTIG || (phase == 0 && br == 0)) {
        const int k = lane & 15, ph = lane >> 4;
        if (k < VPP && (!CONTIG || ph == phase)) {
            const float4 w0 = pre.w0, w1 = pre.w1;
            // (CONTIG: the previous phase's reads of the slot ended at its
            // __syncwarp before the Y stores)
            const int at = CONTIG ? k : ph * VPP + k;
            s_tw[at * 2] = make_float4(0.5f * w0.x, 0.5f * w1.x, 0.5f * w0.y, 0.5f * w1.y);
            s_tw[at * 2 + 1] = make_float4(0.5f * w0.z, 0.5f * w1.z, 0.5f * w0.w, 0.5f * w1.w);
        }
        __syncwarp();
    }
    constexpr int PW = BN / (2 * NPART);     // channels of this part in this phase
    constexpr int NCHK = PW / 16;
    const int cbeg = phase * (BN / 2) + part * PW;
    const float* halo_r = nullptr;
    if constexpr (CONTIG) {
        static_assert(PW == 32, "halo rows hold one 32-channel part");
        const int slot = (tc & 1) * 2 + phase;
        float* slot_base = s_halo + (size_t)slot * 3 * NPART * 3 * PW;
        if (q < 3) {
            // this warp's last three rows (lanes 29-31), gated as in the
            // chunk loop, into its slot; each writer arrives on the slot
            uint32_t va[16], vb[16];
            tmem_ld16(taddr + cbeg, va);
            tmem_ld16(taddr + cbeg + 16, vb);
            tmem_wait_ld(va);
            tmem_wait_ld(vb);
            if (lane >= 32 - H) {
                float* w = slot_base + ((size_t)(q * NPART + part) * 3 + (lane - (32 - H))) * PW;
#pragma unroll
                for (int c = 0; c < PW; ++c) {
                    float v = a * __uint_as_float(c < 16 ? va[c] : vb[c - 16]);
                    if constexpr (SCALED) v *= __ldg(p.vscale + n0 + cbeg + c);
                    w[c] = v;
                }
                mbar_arrive(&sb->hx[slot][q][part]);
            }
        }
        if (q > 0) {
            const bool ok = wait_bounded(&sb->hx[slot][q - 1][part], (uint32_t)(tc >> 1) & 1u, sb, p.status);
            if (!__all_sync(0xffffffffu, ok)) return false;
            halo_r = slot_base + (size_t)((q - 1) * NPART + part) * 3 * PW;
        }
    }
    // Rows whose history reaches back into conv_state, and rows among a
    // sequence's last H when the new history is written, take the slow path
    // (only warps holding such rows).  Without conv_state the history before
    // a sequence start is zero, which the fast path applies through per-lane
    // masks: a separate path that one warp in a few tiles runs stalled that
    // warp, and with it the CTA's next tiles, for about 15 us.
    const bool slow_row = out_row && ((t < H && p.state) || (p.state_next && t >= p.L - H));
    const uint32_t m1 = t >= 1 ? ~0u : 0u, m2 = t >= 2 ? ~0u : 0u, m3 = t >= 3 ? ~0u : 0u;
    // indexed by tile-local channel (even): this warp's slot, shifted to the phase's first pair
    const float4* cw = s_tw + (CONTIG ? 0 : phase * VPP * 2) - cbeg;
    const bool slow = __any_sync(0xffffffffu, slow_row);
    const bool masked = __any_sync(0xffffffffu, t < H);
    if (p.add_residual) {
        if (slow)
            vconv_chunks<NCHK, true, true, SCALED, CONTIG>(taddr, hs, p, i, r, b, t, a, out_row, n0, cbeg, cw, m1, m2,
                                                           m3, br, halo_r);
        else if (masked)
            vconv_chunks<NCHK, false, true, SCALED, CONTIG>(taddr, hs, p, i, r, b, t, a, out_row, n0, cbeg, cw, m1, m2,
                                                            m3, br, halo_r);
        else
            vconv_chunks<NCHK, false, true, SCALED, CONTIG, false>(taddr, hs, p, i, r, b, t, a, out_row, n0, cbeg, cw,
                                                                   m1, m2, m3, br, halo_r);
    } else {
        if (slow)
            vconv_chunks<NCHK, true, false, SCALED, CONTIG>(taddr, hs, p, i, r, b, t, a, out_row, n0, cbeg, cw, m1,
                                                            m2, m3, br, halo_r);
        else
            vconv_chunks<NCHK, false, false, SCALED, CONTIG>(taddr, hs, p, i, r, b, t, a, out_row, n0, cbeg, cw, m1,
                                                             m2, m3, br, halo_r);
    }
    // the warp's Y block (its 32 rows x PW channels, in place of h) to global
    // memory: LPR lanes cover one row's contiguous bytes, so each store
    // instruction writes whole row pieces; history-only rows are skipped
    __syncwarp();
    constexpr int LPR = PW * 2 / 16;
    constexpr int RPI = 32 / LPR;
    const int cb = cbeg >> 6;
    const int j = ((cbeg & 63) >> 3) + lane % LPR;
    const int64_t seg0 = vrow0<CONTIG>(mt, q);   // global row of the warp's lane 0
    __nv_bfloat16* y = p.y + (int64_t)br * p.n_tok * p.d;
#pragma unroll
    for (int k = 0; k < 32 / RPI; ++k) {
        const int rr = k * RPI + lane / LPR;
        const int ii = q * 32 + rr;
        const uint4 v = *reinterpret_cast<const uint4*>(hs + cb * (BM * 128) + ii * 128 + ((j ^ (ii & 7)) << 4));
        const int64_t rg = seg0 + rr;
        if ((rr >= H || (CONTIG && q > 0)) && rg < p.n_tok)
            __stcs(reinterpret_cast<uint4*>(y + rg * p.d + n0 + cb * 64 + j * 8), v);
    }
    return true;
}

// After a key tile's partials are written: the CTA that completes a row band
// (the last of its n_groups channel tiles) reduces the band's G partials per
// row into alpha, in the same fixed order as any other reduction of them,
// and re-arms the counter.  One thread counts with a release/acquire atomic
// at device scope after the CTA barrier; the band's partials (written by
// other CTAs, read through L2) are staged in one pass into the h buffer,
// which this tile no longer needs and the producer refills only after the
// epilogue releases it.
__device__ __forceinline__ int atomic_add_acq_rel(int* addr, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void band_alpha(const EpiParams& p, int mt, int et, Barriers* sb, float4* s_stage,
                                           int stage_bytes) {
    epi_sync();
    if (et == 0) sb->band_last = (atomic_add_acq_rel(p.band_count + mt, 1) == p.n_groups - 1);
    epi_sync();
    if (!sb->band_last) return;
    const int64_t row0 = (int64_t)mt * BM;
    const int rows = (int)min((int64_t)BM, (int64_t)p.n_tok - row0);
    const float4* src = p.part + row0 * p.G;
    // wide hidden sizes whose band does not fit the buffer read L2 directly
    const bool staged = rows * p.G * 16 <= stage_bytes;
    if (staged)
        for (int k = et; k < rows * p.G; k += EPI_THREADS) s_stage[k] = __ldcg(src + k);
    epi_sync();
    // one (row, branch) per thread: branch m's gate reduces its Gb groups
    for (int k = et; k < rows * p.M; k += EPI_THREADS) {
        const int m = k / rows, rr = k - m * rows;
        float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
        for (int g = m * p.Gb; g < (m + 1) * p.Gb; ++g) {
            const float4 v4 = staged ? s_stage[rr * p.G + g] : __ldcg(src + rr * p.G + g);
            s_qk += v4.x;
            s_kk += v4.y;
            s_hh += v4.z;
        }
        const float inv_d = 1.f / (float)p.d;
        const float rh = sqrtf(s_hh * inv_d + p.eps);
        const float rk = sqrtf(s_kk * inv_d + p.eps);
        const float a = 1.f / (1.f + expf(-(s_qk / (rh * rk)) * rsqrtf((float)p.d)));
        const int64_t o = (int64_t)m * p.n_tok + row0 + rr;
        p.alpha_w[o] = a;
        if (p.alpha_out) p.alpha_out[o] = a;
    }
    if (et == 0) p.band_count[mt] = 0;
}

// ---------------------------------------------------------------- kernel

// PAIR (cluster of two CTAs, MODE_K / MODE_VCONV): both CTAs walk the same
// pair tiles; CTA r takes row tile 2 * mt2 + r and W channels
// [n0 + r * BN/2, n0 + (r + 1) * BN/2).  The leader's TMA loads complete on
// its full barrier; the peer announces its bytes on the leader's pfull
// barrier and its TMA loads (cta_group::2 form) complete there too, so the
// leader's warp 1 issues the M = 256 MMAs once both barriers flip and commits
// the stage's empty barrier (and the accumulator's full barrier) in both
// CTAs.  Each CTA's epilogue reads its own TMEM rows; the accumulator is free
// once the 32 epilogue warps of both CTAs have arrived on the leader's tempty.
// On an abort both CTAs stop issuing, meet at a cluster barrier, and the
// leader drains every stage either CTA issued before both leave together.
template <int MODE, int BN, bool PAIR, bool F8>
__global__ void __launch_bounds__(THREADS, 1)
project_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b0,
                  const __grid_constant__ CUtensorMap map_b1, const __grid_constant__ CUtensorMap map_h,
                  const EpiParams p) {
    static_assert(!PAIR || MODE != MODE_KV, "the KV tile runs on one CTA");
    static_assert(sizeof(Barriers) <= 1024, "the barrier block");
    using GE = Geo<MODE, BN, PAIR>;
    static_assert(!GE::CONTIG || GE::GG_BYTES >= EPI_WARPS * (BN / (4 * NPART)) * 32, "one phase of taps per warp");
    static_assert(GE::SMEM_BYTES <= 232448, "shared memory per CTA");
    constexpr bool CONTIG = GE::CONTIG;
    constexpr int STAGES = GE::STAGES;
    constexpr int STAGE_BYTES = GE::STAGE_BYTES;
    constexpr int NCTA = PAIR ? 2 : 1;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024 - (raw & 1023)) & 1023);   // 1024-byte aligned tile base
    const uint32_t tiles_u32 = smem_u32(smem);
    uint8_t* s_h = smem + GE::SMEM_TILES;
    Barriers* sb = reinterpret_cast<Barriers*>(smem + GE::SMEM_TILES + GE::H_BYTES);
    float* s_gg = reinterpret_cast<float*>(smem + GE::SMEM_TILES + GE::H_BYTES + 1024);
    float4* s_red = reinterpret_cast<float4*>(smem + GE::SMEM_TILES + GE::H_BYTES + 1024 + GE::GG_BYTES);
    float* s_halo = reinterpret_cast<float*>(smem + GE::SMEM_TILES + GE::H_BYTES + 1024 + GE::GG_BYTES + GE::RED_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr int BKE = Elt<F8>::BKE;
    const int KB = p.d_mem / BKE;
    const uint32_t rank = PAIR ? cluster_rank() : 0u;
    const bool leader = rank == 0;
    // work units: single tiles, or pair tiles shared by the two CTAs of a cluster
    const int unit0 = (int)blockIdx.x / NCTA;
    const int units_step = (int)gridDim.x / NCTA;
    const int num_units = p.num_tiles;   // pair tiles when PAIR

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sb->full[s], 1);
            mbar_init(&sb->empty[s], 1);
            mbar_init(&sb->pfull[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&sb->tfull[a], 1);
            mbar_init(&sb->tempty[a], NCTA * EPI_WARPS);
        }
        mbar_init(&sb->hfull, 1);
        mbar_init(&sb->hempty, EPI_WARPS);
        for (int hf = 0; hf < 2; ++hf) {
            mbar_init(&sb->hfull_v[hf], 1);
            mbar_init(&sb->hempty_v[hf], EPI_WARPS);
            sb->h_issued_v[hf] = 0;
            sb->h_consumed_v[hf] = 0;
        }
        mbar_init(&sb->drain, 1);
        for (int k = 0; k < HALO_SLOTS * 3 * NPART; ++k) mbar_init(&sb->hx[0][0][0] + k, CONV_W - 1);
        sb->abort_flag = 0;
        sb->issued = 0;
        sb->consumed = 0;
        sb->h_issued = 0;
        sb->h_consumed = 0;
        sb->peer_abort = PAIR ? peer_addr(const_cast<const int*>(&sb->abort_flag), rank ^ 1u) : 0u;
        mbar_fence_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tma_prefetch_desc(&map_a);
        tma_prefetch_desc(&map_b0);
        tma_prefetch_desc(&map_h);
        if (MODE == MODE_KV) tma_prefetch_desc(&map_b1);
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(&sb->tmem_base)),
                         "r"(GE::TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(&sb->tmem_base)),
                         "r"(GE::TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    if constexpr (PAIR) cluster_sync_all();   // barriers of both CTAs initialised before any remote arrival
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sb->tmem_base;
    if (MODE != MODE_VCONV) {
        // e comes from the kernel before this one: wait for it, then let the
        // value pass launch (its CTAs take SMs as this pass's CTAs leave)
        grid_dep_wait();
        grid_dep_launch_dependents();
    }

    // row tile of this CTA for unit u; channel tile
    const int m_units = num_units / p.n_groups;
    auto unit_row = [&](int u) {
        if (p.raster_rb <= 0) return u / p.n_groups;
        const int per = p.raster_rb * p.n_groups;
        const int g = u / per, local = u - g * per;
        const int rows_g = min(p.raster_rb, m_units - g * p.raster_rb);
        return g * p.raster_rb + local % rows_g;
    };
    auto unit_nt = [&](int u) {
        if (p.raster_rb <= 0) return u % p.n_groups;
        const int per = p.raster_rb * p.n_groups;
        const int g = u / per, local = u - g * per;
        const int rows_g = min(p.raster_rb, m_units - g * p.raster_rb);
        return local / rows_g;
    };
    auto unit_mt = [&](int u) { return PAIR ? 2 * unit_row(u) + (int)rank : unit_row(u); };

    if (warp == 0) {
        // ---------------- TMA producer (each CTA loads its own rows and W half)
        if (lane == 0) {
            int it = 0, tc = 0;
            const uint32_t h_dst = smem_u32(s_h);
            const uint64_t h_pol = l2_policy_evict_first();
            for (int u = unit0; u < num_units && !sb->abort_flag; u += units_step, ++tc) {
                const int mt = unit_mt(u), nt = unit_nt(u);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!wait_bounded(&sb->empty[s], ph ^ 1u, sb, p.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = tiles_u32 + s * STAGE_BYTES;
                    const uint32_t b_dst = a_dst + A_BYTES;
                    // the leader counts its stage on full[s]; the peer on the leader's pfull[s]
                    const bool remote = PAIR && !leader;
                    const uint32_t bar = remote ? peer_addr(&sb->pfull[s], 0u) : smem_u32(&sb->full[s]);
                    auto load = [&](const CUtensorMap* m, uint32_t dst, int x, int y) {
                        if (remote) tma_load_2d_peer_bar(m, dst, bar, x, y);
                        else tma_load_2d(m, dst, &sb->full[s], x, y);
                    };
                    if (remote) mbar_arrive_expect_tx_remote(bar, STAGE_BYTES);
                    else mbar_arrive_expect_tx(&sb->full[s], STAGE_BYTES);
                    if (p.stall && it == 0 && blockIdx.x == 0) {
                        // bounded-wait test: the stage's bytes are announced
                        // and never arrive, so the MMA's wait on it runs out
                        sb->issued = it + 1;
                        continue;
                    }
                    if (MODE == MODE_VCONV && CONTIG) {
                        // one 128-row block, starting 3 rows before its outputs
                        load(&map_a, a_dst, kb * BKE, (int)vrow0<true>(mt, 0));
                    } else if (MODE == MODE_VCONV) {
                        // four 32-row segments, each starting 3 rows before its outputs
#pragma unroll
                        for (int sg = 0; sg < 4; ++sg)
                            load(&map_a, a_dst + sg * (SEG * 128), kb * BKE, mt * TILE_OUT + sg * SEG_OUT - (CONV_W - 1));
                    } else {
                        load(&map_a, a_dst, kb * BKE, mt * BM);
                    }
                    if (MODE == MODE_KV) {
                        load(&map_b0, b_dst, kb * BKE, nt * 128);
                        load(&map_b1, b_dst + 128 * 128, kb * BKE, nt * 128);
                    } else {
                        load(&map_b0, b_dst, kb * BKE, nt * BN + (int)rank * GE::B_ROWS);
                    }
                    sb->issued = it + 1;
                }
                if (!ok) break;
                if (MODE == MODE_VCONV) continue;   // warp 2 loads the value tile's h
                // the tile's h slice, once the epilogue has released the previous one
                if (!wait_bounded(&sb->hempty, ((uint32_t)tc & 1u) ^ 1u, sb, p.status)) break;
                mbar_arrive_expect_tx(&sb->hfull, GE::H_BYTES);
                // the tile's channels in the stacked [M*d] key space: branch m, channel hc0 within
                // it; branch m's rows start at row m * n_tok of the stacked [M * n_tok][d] h
                const int ck = MODE == MODE_KV ? nt * 128 : nt * BN;
                const int hm = ck / p.d, hc0 = ck - hm * p.d;
#pragma unroll 1
                for (int cb = 0; cb < GE::HC / 64; ++cb)
                    tma_load_2d_hint(&map_h, h_dst + cb * (BM * 128), &sb->hfull, hc0 + cb * 64, hm * p.n_tok + mt * BM,
                                     h_pol);
                sb->h_issued = tc + 1;
            }
        }
    } else if (warp == 1 && (!PAIR || leader)) {
        // ---------------- MMA issuer (the leader of a pair)
        if (lane == 0) {
            int it = 0, tc = 0;
            for (int u = unit0; u < num_units && !sb->abort_flag; u += units_step, ++tc) {
                const int acc = tc & 1;
                const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
                if (!wait_bounded(&sb->tempty[acc], aph ^ 1u, sb, p.status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    if (!wait_bounded(&sb->full[s], ph, sb, p.status) ||
                        (PAIR && !wait_bounded(&sb->pfull[s], ph, sb, p.status))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = tiles_u32 + s * STAGE_BYTES;
                    const uint64_t da = smem_desc_sw128(a_addr);
                    const uint64_t db = smem_desc_sw128(a_addr + A_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / UK; ++kk) {
                        // +32 bytes along K inside the swizzled 128-byte row (16 bf16 or 32 FP8)
                        if constexpr (PAIR)
                            umma_bf16_pair<BN, F8>(d_tmem, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2),
                                                   (kb | kk) != 0);
                        else
                            umma_bf16<BN, F8>(d_tmem, da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), (kb | kk) != 0);
                    }
                    if constexpr (PAIR) umma_commit_pair_both(&sb->empty[s]);
                    else umma_commit(&sb->empty[s]);
                    sb->consumed = it + 1;
                }
                if (!ok) break;
                if constexpr (PAIR) umma_commit_pair_both(&sb->tfull[acc]);
                else umma_commit(&sb->tfull[acc]);
            }
        }
    } else if (warp == 2 && MODE == MODE_VCONV) {
        // ---------------- h loader of the value pass: the two channel halves of
        // each tile's h slice, each as soon as the epilogue has released it, so
        // neither the operand stream nor the next tile waits on an h load
        if (lane == 0) {
            const uint32_t h_dst = smem_u32(s_h);
            const uint64_t h_pol = l2_policy_evict_first();
            constexpr int CB_HALF = GE::HC / 128;   // 64-channel blocks per half
            int tc = 0;
            for (int u = unit0; u < num_units && !sb->abort_flag; u += units_step, ++tc) {
                const int mt = unit_mt(u), nt = unit_nt(u);
                bool ok = true;
                // each half is filled once per branch: use k = tc * M + m
                for (int m = 0; m < p.M && ok; ++m) {
                    const int k = tc * p.M + m;
                    for (int hf = 0; hf < 2; ++hf) {
                        if (!wait_bounded(&sb->hempty_v[hf], ((uint32_t)k & 1u) ^ 1u, sb, p.status)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&sb->hfull_v[hf], GE::H_BYTES / 2);
                        for (int cb = hf * CB_HALF; cb < (hf + 1) * CB_HALF; ++cb) {
#pragma unroll
                            for (int sg = 0; sg < 4; ++sg)
                                tma_load_2d_hint(&map_h, h_dst + cb * (BM * 128) + sg * (SEG * 128), &sb->hfull_v[hf],
                                                 nt * BN + cb * 64, m * p.n_tok + (int)vrow0<CONTIG>(mt, sg), h_pol);
                        }
                        sb->h_issued_v[hf] = k + 1;
                    }
                }
                if (!ok) break;
            }
        }
    } else if (warp >= 4) {
        // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) ..; the
        // four warps of each lane quarter take the four column parts
        const int q = warp & 3;
        const int part = (warp - 4) >> 2;
        const int et = threadIdx.x - 128;    // 0 .. EPI_THREADS-1
        const uint32_t tempty_leader0 = PAIR ? peer_addr(&sb->tempty[0], 0u) : 0u;
        const uint32_t tempty_leader1 = PAIR ? peer_addr(&sb->tempty[1], 0u) : 0u;
        int tc = 0;
        TilePre pre{};
        // alpha comes from the key pass, which may still be running when this
        // grid was launched as its programmatic dependent
        if (MODE == MODE_VCONV) grid_dep_wait();
        if (unit0 < num_units) pre = tile_pre_load<MODE, BN, CONTIG>(p, unit_mt(unit0), unit_nt(unit0), q, lane, et);
        for (int u = unit0; u < num_units; u += units_step, ++tc) {
            const int acc = tc & 1;
            const uint32_t aph = (uint32_t)(tc >> 1) & 1u;
            const int mt = unit_mt(u), nt = unit_nt(u);
            const uint32_t taddr = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
            const int un = u + units_step;
            const bool has_next = un < num_units;
            if (MODE == MODE_VCONV) {
                // phase 0 on the first channel half, release its h, phase 1;
                // each warp decides alone: the value epilogue has no barrier
                // across warps, so a warp that stops cannot strand the others.
                // Both phases run one copy of the code (not unrolled), so the
                // first tile fetches the epilogue's instructions once.
                bool ok = wait_bounded(&sb->tfull[acc], aph, sb, p.status);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after();
                const float a0 = pre.a;
                const int64_t r_lane = vrow0<CONTIG>(mt, q) + lane;
                const bool r_ok = r_lane >= 0 && r_lane < p.n_tok;
                float a_br = a0;
                const int n_ph = 2 * p.M;
#pragma unroll 1
                for (int ph = 0; ph < n_ph; ++ph) {
                    const int phase = ph & 1, br = ph >> 1;
                    const int k = tc * p.M + br;
                    ok = wait_bounded(&sb->hfull_v[phase], (uint32_t)k & 1u, sb, p.status);
                    if (!__all_sync(0xffffffffu, ok)) break;
                    if (br > 0 && phase == 0) a_br = r_ok ? __ldg(p.alpha + (int64_t)br * p.n_tok + r_lane) : 0.f;
                    ok = epilogue_vconv<BN, F8, CONTIG>(taddr, s_h, p, mt, nt, q, part, lane, et, s_gg, phase, a_br,
                                                        pre, br, sb, s_halo, tc);
                    if (!ok) break;
                    // the next tile's taps and gates, once this tile's last use of
                    // them is staged (contiguous tiles stage the taps phase by phase)
                    if (ph == (CONTIG ? n_ph - 1 : 0) && has_next)
                        pre = tile_pre_load<MODE, BN, CONTIG>(p, unit_mt(un), unit_nt(un), q, lane, et);
                    const bool last = ph == n_ph - 1;
                    if (last) tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (last) {
                            if (PAIR && !leader) mbar_arrive_remote(acc ? tempty_leader1 : tempty_leader0);
                            else mbar_arrive(&sb->tempty[acc]);
                        }
                        mbar_arrive(&sb->hempty_v[phase]);
                    }
                    if (threadIdx.x == 128) sb->h_consumed_v[phase] = k + 1;
                }
                if (!__all_sync(0xffffffffu, ok)) break;
                continue;
            }
            bool ok = wait_bounded(&sb->tfull[acc], aph, sb, p.status);
            ok = ok && wait_bounded(&sb->hfull, (uint32_t)tc & 1u, sb, p.status);
            if (epi_any(!ok)) break;          // one decision for all epilogue warps
            tc_fence_after();
            // the odd CTA of the last pair may hold a row tile past the end
            const bool rows_live = MODE == MODE_VCONV ? (int64_t)mt * TILE_OUT < p.n_tok : (int64_t)mt * BM < p.n_tok;
            if (MODE == MODE_KV) epilogue_kv(taddr, s_h, p, mt * BM, nt, q, part, lane, et, s_gg, s_red);
            if (MODE == MODE_K && rows_live) {
                epilogue_k<BN, F8>(taddr, s_h, p, mt * BM, nt, q, part, lane, et, s_gg, s_red, pre, has_next,
                               unit_mt(un), unit_nt(un));
                band_alpha(p, mt, et, sb, reinterpret_cast<float4*>(s_h), GE::H_BYTES);
            } else if (MODE == MODE_K && has_next) {
                pre = tile_pre_load<MODE, BN>(p, unit_mt(un), unit_nt(un), q, lane, et);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR && !leader) mbar_arrive_remote(acc ? tempty_leader1 : tempty_leader0);
                else mbar_arrive(&sb->tempty[acc]);
                mbar_arrive(&sb->hempty);
            }
            if (threadIdx.x == 128) sb->h_consumed = tc + 1;
        }
    }

    __syncthreads();
    // a pair decides together: both CTAs have stopped issuing once they meet here
    bool aborted = sb->abort_flag != 0;
    if constexpr (PAIR) {
        cluster_sync_all();
        aborted = aborted || ld_remote_s32(sb->peer_abort) != 0;
    }
    if (aborted) {
        // drain: copies issued but not consumed (for a pair, the leader also
        // waits out the peer's stages, which complete on its pfull), the h
        // tiles, then the MMAs
        if (warp == 0 && lane == 0) {
            if (!PAIR || leader) {
                for (int it = sb->consumed; it < sb->issued; ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    const long long t0 = clock64();
                    while (!mbar_try_wait(smem_u32(&sb->full[s]), ph) && clock64() - t0 < kWaitCycles) {
                    }
                }
            }
            if (PAIR && leader) {
                const int peer_issued = ld_remote_s32(peer_addr(&sb->issued, 1u));
                for (int it = sb->consumed; it < peer_issued; ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                    const long long t0 = clock64();
                    while (!mbar_try_wait(smem_u32(&sb->pfull[s]), ph) && clock64() - t0 < kWaitCycles) {
                    }
                }
            }
            for (int k = sb->h_consumed; k < sb->h_issued; ++k) {
                const long long t0 = clock64();
                while (!mbar_try_wait(smem_u32(&sb->hfull), (uint32_t)k & 1u) && clock64() - t0 < kWaitCycles) {
                }
            }
            for (int hf = 0; hf < 2; ++hf) {
                for (int k = sb->h_consumed_v[hf]; k < sb->h_issued_v[hf]; ++k) {
                    const long long t0 = clock64();
                    while (!mbar_try_wait(smem_u32(&sb->hfull_v[hf]), (uint32_t)k & 1u) &&
                           clock64() - t0 < kWaitCycles) {
                    }
                }
            }
        }
        if (warp == 1 && lane == 0 && (!PAIR || leader)) {
            if constexpr (PAIR) umma_commit_pair_local(&sb->drain);
            else umma_commit(&sb->drain);
            const long long t0 = clock64();
            while (!mbar_try_wait(smem_u32(&sb->drain), 0) && clock64() - t0 < kWaitCycles) {
            }
        }
        __syncthreads();
    }
    // a pair leaves together: no remote arrival may reach a CTA that has exited
    if constexpr (PAIR) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        if constexpr (PAIR)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(GE::TMEM_COLS)
                         : "memory");
        else
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

// The history in the sequence-minor layout for decode-shaped calls: tiles of
// 32 sequences x 32 channels go through shared memory so that both the read
// and the write are coalesced.  state [B][H][d] -> state_t [H][d][B].
__global__ void state_to_tr_kernel(const float* __restrict__ state, float* __restrict__ state_t, int B, int H, int d) {
    __shared__ float tile[32][33];
    const int c0 = blockIdx.x * 32, b0 = blockIdx.y * 32, i = blockIdx.z;
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const int b = b0 + r, c = c0 + threadIdx.x;
        tile[r][threadIdx.x] = (b < B && c < d) ? state[((int64_t)b * H + i) * d + c] : 0.f;
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        const int c = c0 + r, b = b0 + threadIdx.x;
        if (b < B && c < d) state_t[((int64_t)i * d + c) * B + b] = tile[threadIdx.x][r];
    }
}

// merge for the sequence-minor layout: new history row i of sequence b is
// state_next_t[i][c][b] when position L - H + i was computed, else the old
// row L + i (L < H); each block walks i upwards, so the in-place shift reads
// a row before the block overwrites it.
__global__ void state_merge_tr_kernel(float* __restrict__ state, const float* __restrict__ state_next_t, int B, int L,
                                      int H, int d) {
    __shared__ float tile[32][33];
    const int c0 = blockIdx.x * 32, b0 = blockIdx.y * 32;
    for (int i = 0; i < H; ++i) {
        const bool fresh = L - H + i >= 0;
        if (fresh) {
            for (int r = threadIdx.y; r < 32; r += blockDim.y) {
                const int c = c0 + r, b = b0 + threadIdx.x;
                tile[r][threadIdx.x] = (b < B && c < d) ? state_next_t[((int64_t)i * d + c) * B + b] : 0.f;
            }
        }
        __syncthreads();
        for (int r = threadIdx.y; r < 32; r += blockDim.y) {
            const int b = b0 + r, c = c0 + threadIdx.x;
            if (b < B && c < d) {
                const float v = fresh ? tile[threadIdx.x][r] : state[((int64_t)b * H + (L + i)) * d + c];
                state[((int64_t)b * H + i) * d + c] = v;
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------- host side

// h of M branches stacked as a 2-D bf16 [M * rows][cols] map (box_rows x 64
// columns, 128-byte swizzle).  A tile's rows before its branch's row 0 or
// past its last row read the neighbouring branch (or zeros at the ends);
// those rows are never used: they are conv history rows, whose h the value
// epilogue does not read, or rows past n_tok, which neither epilogue keeps.
bool make_map_h(CUtensorMap* m, const void* base, uint64_t branches, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    return make_map(m, base, branches * rows, cols, box_rows);
}

template <int MODE, int BN, bool PAIR, bool F8 = false>
cudaError_t launch_mode(const CUtensorMap& ma, const CUtensorMap& mb0, const CUtensorMap& mb1, const CUtensorMap& mh,
                        EpiParams p, int64_t m_tiles, int num_sms, cudaStream_t s, bool pdl = false) {
    using GE = Geo<MODE, BN, PAIR>;
    auto kernel = project_tc_kernel<MODE, BN, PAIR, F8>;
    static unsigned long long attr_set = 0;   // one bit per device ordinal
    static int max_clusters[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !(attr_set >> dev & 1ull)) {
        cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GE::SMEM_BYTES);
        if (err != cudaSuccess) return err;
        if (PAIR) {
            err = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
            (void)err;
        }
        attr_set |= 1ull << dev;
    }
    const int64_t units = (PAIR ? (m_tiles + 1) / 2 : m_tiles) * p.n_groups;
    if (units >= (int64_t)1 << 31) return cudaErrorInvalidValue;
    p.num_tiles = (int)units;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = GE::SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (pdl) {
        attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
        ++cfg.numAttrs;
    }
    if (!PAIR) {
        const int grid = (int)(units < num_sms ? units : num_sms);
        if (!pdl) {
            kernel<<<grid, THREADS, GE::SMEM_BYTES, s>>>(ma, mb0, mb1, mh, p);
            return cudaGetLastError();
        }
        cfg.gridDim = dim3((unsigned)grid, 1, 1);
        return cudaLaunchKernelEx(&cfg, kernel, ma, mb0, mb1, mh, p);
    }
    attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
    attr[cfg.numAttrs].val.clusterDim.x = 2;
    attr[cfg.numAttrs].val.clusterDim.y = 1;
    attr[cfg.numAttrs].val.clusterDim.z = 1;
    ++cfg.numAttrs;
    if (dev < 64 && max_clusters[dev] == 0) {
        cfg.gridDim = dim3((unsigned)(num_sms & ~1), 1, 1);
        int mc = 0;
        cudaLaunchConfig_t qcfg = cfg;                 // the cluster shape alone
        qcfg.attrs = &attr[cfg.numAttrs - 1];
        qcfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&mc, kernel, &qcfg) != cudaSuccess || mc < 1) {
            cudaGetLastError();
            mc = num_sms / 2;
        }
        max_clusters[dev] = mc;
    }
    const int64_t cap = dev < 64 ? max_clusters[dev] : num_sms / 2;
    const int64_t clusters = units < cap ? units : cap;
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    return cudaLaunchKernelEx(&cfg, kernel, ma, mb0, mb1, mh, p);
}

// 256-channel tiles where d allows them, except for decode-sized calls (a few
// hundred rows) where they would leave most SMs idle: 128-channel tiles
// double the CTAs there
int pick_bn(int32_t d, int64_t n_tok, int64_t m_tiles, int num_sms) {
    if (d % 256 != 0) return 128;
    return (n_tok <= 1024 && m_tiles * (d / 256) < num_sms / 2) ? 128 : 256;
}

// CTA pairs once there are enough row tiles to give every SM pair work
bool use_pair(int64_t m_tiles, int n_groups, int num_sms) { return m_tiles * n_groups >= 2 * (int64_t)num_sms; }

// Row units per group of the grouped tile order of a wide key pass (stacked
// W_K of several branches): a group's rows of e and the whole stacked W_K
// stay in L2 together, in 70 % of it (the rest holds the streaming h and the
// gate partials).  Measured at c3 with four bf16 branches (row units of 256
// rows, W_K 42 MB): 8 / 16 / 32 / 48 / 64 / 128 units per group gave a key
// pass of 1780 / 1437 / 1200 / 1157 / 1235 / 1308 us; this rule gives 44.
int raster_group(int32_t M, int32_t d, int32_t d_mem, bool f8, bool pair) {
    static int64_t l2_bytes[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    int64_t l2 = dev < 64 ? l2_bytes[dev] : 0;
    if (l2 == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev) != cudaSuccess || v <= 0) v = 96 << 20;
        cudaGetLastError();
        l2 = v;
        if (dev < 64) l2_bytes[dev] = l2;
    }
    const double es = f8 ? 1.0 : 2.0;
    const double w_bytes = (double)M * d * d_mem * es;
    const double unit_bytes = (double)(pair ? 2 * BM : BM) * d_mem * es;
    const double rb = (0.7 * (double)l2 - w_bytes) / unit_bytes;
    return rb < 8.0 ? 8 : (rb > 4096.0 ? 4096 : (int)rb);
}

// The value pass runs on CTA pairs with contiguous 128-row tiles (one A box
// per CTA and stage, 125 output rows) for one bf16 branch, 256-channel tiles
// and K >= 2048: there a tile's MMAs outlast the epilogue's halo exchange
// between warps (about 2.5 us a tile), which at K = 1024 sits on the
// critical path (B200, c2: 131 against 108 us single; c3: 323-331 against
// 351-376 us).  On pairs the layout of four overlapping 32-row boxes per
// stage starves the MMAs (124 against 101 us on single CTAs at c2, 399
// against 322 us at c3), so that layout stays on single CTAs.
bool use_contig_pair(int bn, int32_t M, bool f8, int32_t d_mem, int64_t m_tiles_c, int n_groups, int num_sms) {
    return bn == 256 && M == 1 && !f8 && d_mem >= 2048 && use_pair(m_tiles_c, n_groups, num_sms);
}

}  // namespace

bool project_tc_supported(int64_t n_tok, int32_t d_mem, int32_t d, bool f8) {
    const int bke = f8 ? Elt<true>::BKE : Elt<false>::BKE;
    return n_tok > 0 && n_tok < (int64_t)1 << 30 && d_mem % bke == 0 && d_mem >= bke && d % 128 == 0 &&
           encode_fn() != nullptr;
}

cudaError_t launch_project_tc(const void* e, int64_t n_tok, int32_t d_mem, const void* h, const void* Wk,
                              const void* Wv, const float* gq, const float* gk, int32_t d, float* v, float* part,
                              uint32_t* status, int num_sms, cudaStream_t s) {
    if (!project_tc_supported(n_tok, d_mem, d, false)) return cudaErrorNotSupported;
    CUtensorMap ma, mk, mv, mh;
    if (!make_map(&ma, e, (uint64_t)n_tok, (uint64_t)d_mem, BM) || !make_map(&mk, Wk, (uint64_t)d, (uint64_t)d_mem, 128) ||
        !make_map(&mv, Wv, (uint64_t)d, (uint64_t)d_mem, 128) || !make_map_h(&mh, h, 1, (uint64_t)n_tok, (uint64_t)d, BM))
        return cudaErrorInvalidValue;
    EpiParams p{};
    p.M = 1;
    p.Gb = d / 128;
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
    return launch_mode<MODE_KV, 256, false>(ma, mk, mv, mh, p, (n_tok + BM - 1) / BM, num_sms, s);
}

cudaError_t launch_gate_k_tc(const void* e, int64_t n_tok, int32_t d_mem, const void* h, const void* Wk,
                             const float* gq, const float* gk, int32_t d, float eps, float* part, int* band_count,
                             float* alpha, float* alpha_out, uint32_t* status, int num_sms, int stall, bool pdl,
                             cudaStream_t s, int32_t M, bool f8, const float* kscale) {
    if (!project_tc_supported(n_tok, d_mem, d, f8) || M < 1 || M > kMaxBranches || (int64_t)M * n_tok >= (1ll << 31))
        return cudaErrorNotSupported;
    const int bn = pick_bn(d, n_tok, (n_tok + BM - 1) / BM, num_sms);
    CUtensorMap ma, mk, mh;
    if (!make_map(&ma, e, (uint64_t)n_tok, (uint64_t)d_mem, BM, f8) ||
        !make_map(&mk, Wk, (uint64_t)M * d, (uint64_t)d_mem, bn, f8) ||
        !make_map_h(&mh, h, (uint64_t)M, (uint64_t)n_tok, (uint64_t)d, BM))
        return cudaErrorInvalidValue;
    EpiParams p{};
    p.M = M;
    p.Gb = d / 128;
    p.kscale = kscale;
    p.gq = gq;
    p.gk = gk;
    p.part = reinterpret_cast<float4*>(part);
    p.band_count = band_count;
    p.stall = stall;
    p.alpha_w = alpha;
    p.alpha_out = alpha_out;
    p.eps = eps;
    p.status = status;
    p.n_tok = (int)n_tok;
    p.d_mem = d_mem;
    p.d = d;
    p.G = M * (d / 128);
    p.n_groups = M * (d / bn);
    const int64_t mt = (n_tok + BM - 1) / BM;
    const bool pair = bn == 256 && use_pair(mt, p.n_groups, num_sms);
    p.raster_rb = p.n_groups > 16 ? raster_group(M, d, d_mem, f8, pair) : 0;
    if (pair) {
        CUtensorMap mk2;
        if (!make_map(&mk2, Wk, (uint64_t)M * d, (uint64_t)d_mem, 128, f8)) return cudaErrorInvalidValue;
        return f8 ? launch_mode<MODE_K, 256, true, true>(ma, mk2, mk2, mh, p, mt, num_sms, s, pdl)
                  : launch_mode<MODE_K, 256, true, false>(ma, mk2, mk2, mh, p, mt, num_sms, s, pdl);
    }
    if (f8)
        return bn == 256 ? launch_mode<MODE_K, 256, false, true>(ma, mk, mk, mh, p, mt, num_sms, s, pdl)
                         : launch_mode<MODE_K, 128, false, true>(ma, mk, mk, mh, p, mt, num_sms, s, pdl);
    return bn == 256 ? launch_mode<MODE_K, 256, false>(ma, mk, mk, mh, p, mt, num_sms, s, pdl)
                     : launch_mode<MODE_K, 128, false>(ma, mk, mk, mh, p, mt, num_sms, s, pdl);
}

cudaError_t launch_vconv_tc(const void* e, int32_t B, int32_t L, int32_t d_mem, const void* h, const void* Wv,
                            const float* conv_w, int32_t d, int32_t w, const float* alpha, const float* state,
                            float* state_next, int32_t state_tr, void* y, int32_t add_residual, uint32_t* status,
                            int num_sms, bool pdl, cudaStream_t s, int32_t M, bool f8, const float* vscale) {
    const int64_t n_tok = (int64_t)B * L;
    if (!project_tc_supported(n_tok, d_mem, d, f8) || w != CONV_W || M < 1 || M > kMaxBranches ||
        (int64_t)M * n_tok >= (1ll << 31))
        return cudaErrorNotSupported;
    const int bn = pick_bn(d, n_tok, (n_tok + TILE_OUT - 1) / TILE_OUT, num_sms);
    CUtensorMap ma, mv, mh;
    if (!make_map(&ma, e, (uint64_t)n_tok, (uint64_t)d_mem, SEG, f8) ||
        !make_map(&mv, Wv, (uint64_t)d, (uint64_t)d_mem, bn, f8) ||
        !make_map_h(&mh, h, (uint64_t)M, (uint64_t)n_tok, (uint64_t)d, SEG))
        return cudaErrorInvalidValue;
    EpiParams p{};
    p.M = M;
    p.Gb = d / 128;
    p.vscale = vscale;
    p.alpha = alpha;
    p.conv_w = conv_w;
    p.state = state;
    p.state_next = state ? state_next : nullptr;
    p.state_tr = state_tr;
    p.B = B;
    p.y = static_cast<__nv_bfloat16*>(y);
    p.status = status;
    p.n_tok = (int)n_tok;
    p.d_mem = d_mem;
    p.d = d;
    p.G = d / 128;
    p.n_groups = d / bn;
    p.L = L;
    p.add_residual = add_residual;
    const int64_t mt = (n_tok + TILE_OUT - 1) / TILE_OUT;
    const int64_t mt_c = (n_tok + TILE_OUT_C - 1) / TILE_OUT_C;
    if (use_contig_pair(bn, M, f8, d_mem, mt_c, p.n_groups, num_sms)) {
        // contiguous tiles on CTA pairs: each CTA's A block is 128 rows, its
        // half of the W_V tile 128 channels
        CUtensorMap ma_c, mv_c;
        if (!make_map(&ma_c, e, (uint64_t)n_tok, (uint64_t)d_mem, BM) ||
            !make_map(&mv_c, Wv, (uint64_t)d, (uint64_t)d_mem, 128))
            return cudaErrorInvalidValue;
        return launch_mode<MODE_VCONV, 256, true, false>(ma_c, mv_c, mv_c, mh, p, mt_c, num_sms, s, pdl);
    }
    if (f8)
        return bn == 256 ? launch_mode<MODE_VCONV, 256, false, true>(ma, mv, mv, mh, p, mt, num_sms, s, pdl)
                         : launch_mode<MODE_VCONV, 128, false, true>(ma, mv, mv, mh, p, mt, num_sms, s, pdl);
    return bn == 256 ? launch_mode<MODE_VCONV, 256, false>(ma, mv, mv, mh, p, mt, num_sms, s, pdl)
                     : launch_mode<MODE_VCONV, 128, false>(ma, mv, mv, mh, p, mt, num_sms, s, pdl);
}

cudaError_t launch_state_to_tr(const float* state, float* state_t, int32_t B, int32_t w, int32_t d, cudaStream_t s) {
    const int H = w - 1;
    if (H <= 0 || B == 0) return cudaSuccess;
    const dim3 grid((unsigned)((d + 31) / 32), (unsigned)((B + 31) / 32), (unsigned)H);
    state_to_tr_kernel<<<grid, dim3(32, 8), 0, s>>>(state, state_t, B, H, d);
    return cudaGetLastError();
}

cudaError_t launch_state_merge_tr(float* state, const float* state_next_t, int32_t B, int32_t L, int32_t w, int32_t d,
                                  cudaStream_t s) {
    const int H = w - 1;
    if (H <= 0 || B == 0) return cudaSuccess;
    const dim3 grid((unsigned)((d + 31) / 32), (unsigned)((B + 31) / 32), 1);
    state_merge_tr_kernel<<<grid, dim3(32, 8), 0, s>>>(state, state_next_t, B, L, H, d);
    return cudaGetLastError();
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
