// C ABI of the Engram forward path: argument checks, workspace layout and
// kernel sequencing.  Every entry point validates on the host and launches
// nothing on error; kernels report data errors through the context's device
// status word instead of trapping.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>

#include <cuda.h>
#include <nvtx3/nvToolsExt.h>

#include "ctx.cuh"

namespace engram {

thread_local char g_last_error[256] = "";

void set_error(const char* what, cudaError_t e) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
}

void set_error(const char* what) { std::snprintf(g_last_error, sizeof(g_last_error), "%s", what); }

engram_status inval(const char* what) {
    set_error(what);
    return ENGRAM_E_INVAL;
}

engram_status cuda_fail(const char* what, cudaError_t e) {
    set_error(what, e);
    return ENGRAM_E_CUDA;
}

int n_tables_of(const engram_config& k) { return k.n_orders * k.heads; }

bool is_prime_u32(uint32_t n) {
    if (n < 2) return false;
    if (n % 2 == 0) return n == 2;
    for (uint32_t f = 3; (uint64_t)f * f <= n; f += 2)
        if (n % f == 0) return false;
    return true;
}

// ---------------------------------------------------------------- profiling

void prof_reset(engram_ctx* c) { c->prof_n = 0; }

// Every launch is also an NVTX range named for the kernel's role, so a
// profiler timeline of a step shows which launch is which (NVTX costs a
// pointer test when no tool is attached).
// Under stream capture a plain event record only orders work inside the
// graph; the external form makes it a record node that each replay records,
// so a captured forward can be timed kernel by kernel.
static void prof_record(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, s);
}

void prof_begin(engram_ctx* c, cudaStream_t s, const char* name) {
    nvtxRangePushA(name);
    if (!c->prof || c->prof_n >= kMaxProf) return;
    c->prof_name[c->prof_n] = name;
    prof_record(c->ev[2 * c->prof_n], s);
}

void prof_end(engram_ctx* c, cudaStream_t s) {
    nvtxRangePop();
    if (!c->prof || c->prof_n >= kMaxProf) return;
    prof_record(c->ev[2 * c->prof_n + 1], s);
    ++c->prof_n;
}

// ---------------------------------------------------------------- workspace

bool tc_path(const engram_ctx* c, int64_t n) {
    return (c->cfg.dtype == ENGRAM_BF16 || c->cfg.dtype == ENGRAM_FP8) && c->sm100 &&
           project_tc_supported(n, c->d_mem, c->cfg.hidden, c->cfg.dtype == ENGRAM_FP8);
}

// projections with the gate and the conv fused into the epilogue (conv width 4)
bool fused_path(const engram_ctx* c, int64_t n) { return tc_path(c, n) && c->cfg.conv_width == 4; }

// Decode-shaped calls (a few positions per sequence) hand the fused value pass
// the conv history in the sequence-minor layout [w-1][d][B]: consecutive lanes
// then read consecutive sequences' history instead of rows d floats apart.
constexpr int32_t kDecodeRows = 8;
bool decode_shaped(const engram_ctx* c, int64_t n, int64_t L) { return fused_path(c, n) && L <= kDecodeRows; }

// One new position per sequence for at most 256 sequences (bf16, one branch):
// the decode passes, which read and update the caller's conv state in place.
bool decode_kernels(const engram_ctx* c, int64_t n, int64_t L, int M) {
    return fused_path(c, n) && decode_tc_supported(n, (int32_t)L, c->d_mem, c->cfg.hidden, M,
                                                   c->cfg.dtype == ENGRAM_FP8);
}

// per-128-row-band counters of the key pass (at least 8: the decode key pass
// counts four row blocks)
size_t band_bytes(int64_t n) {
    const int64_t k = (n + 127) / 128;
    return (size_t)(k < 8 ? 8 : k) * sizeof(int);
}

Workspace carve(const engram_ctx* c, void* base, int64_t B, int64_t L, bool with_idx_e, int M) {
    const int64_t n = B * L;
    Workspace w{};
    char* p = static_cast<char*>(base);
    if (with_idx_e) {
        w.idx = reinterpret_cast<uint32_t*>(p);
        p += align256((size_t)n * c->J * sizeof(uint32_t));
        w.e = p;
        p += align256((size_t)n * c->d_mem * c->es);
    }
    const bool dec = decode_kernels(c, n, L, M);
    w.part = reinterpret_cast<float*>(p);
    const int64_t groups = dec ? decode_tc_max_tiles(c->cfg.hidden) : c->G;
    p += align256((size_t)n * M * groups * 4 * sizeof(float));
    w.alpha = reinterpret_cast<float*>(p);
    p += align256((size_t)M * n * sizeof(float));
    w.band = reinterpret_cast<int*>(p);
    w.counter_bytes = band_bytes(n);
    p += align256(band_bytes(n));
    const size_t hist_bytes =
        align256((size_t)M * B * (c->cfg.conv_width - 1) * c->cfg.hidden * sizeof(float));
    w.state_next = reinterpret_cast<float*>(p);
    p += hist_bytes;
    if (decode_shaped(c, n, L) && !dec) {
        w.state_t = reinterpret_cast<float*>(p);
        p += hist_bytes;
    }
    if (!fused_path(c, n) || dec) {
        w.v = reinterpret_cast<float*>(p);
        p += align256((size_t)n * c->cfg.hidden * sizeof(float));
    }
    w.bytes = (size_t)(p - static_cast<char*>(base));
    return w;
}

engram_status check_device(const engram_ctx* c) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev != c->device) return inval("the current device is not the context's device");
    return ENGRAM_OK;
}

engram_status launched(const char* what, cudaError_t e) {
    if (e != cudaSuccess) return cuda_fail(what, e);
    return ENGRAM_OK;
}

engram_status project_impl(engram_ctx* c, const void* e_cat, int64_t n, const void* h, const void* Wk,
                           const void* Wv, const float* gq, const float* gk, float* v, float* part,
                           cudaStream_t s) {
    const bool bf16 = c->cfg.dtype == ENGRAM_BF16;
    if (tc_path(c, n)) {
        prof_begin(c, s, "project_kv_tc");
        cudaError_t e = launch_project_tc(e_cat, n, c->d_mem, h, Wk, Wv, gq, gk, c->cfg.hidden, v, part, c->d_status,
                                          c->num_sms, s);
        prof_end(c, s);
        return launched("tcgen05 projection launch", e);
    }
    prof_begin(c, s, "project_simt");
    cudaError_t e = launch_project_simt(bf16, e_cat, n, c->d_mem, h, Wk, Wv, gq, gk, c->cfg.hidden, v, part, s);
    prof_end(c, s);
    return launched("projection launch", e);
}

engram_status conv_impl(engram_ctx* c, const float* v, const float* part, const void* h, const float* conv_w,
                        int32_t B, int32_t L, float* state, void* y, float* alpha_out, int32_t add_residual,
                        cudaStream_t s) {
    prof_begin(c, s, "gate_conv");
    cudaError_t e = launch_gate_conv(c->cfg.dtype == ENGRAM_BF16, v, part, h, conv_w, B, L, c->cfg.hidden,
                                     c->cfg.conv_width, c->cfg.eps, state, y, alpha_out, add_residual, c->d_status,
                                     s);
    prof_end(c, s);
    return launched("gate/conv launch", e);
}

// Decode-shaped fused calls read the conv history from a sequence-minor copy
// [w-1][d][B]: the transpose runs on the side stream (it needs only the
// caller's conv_state), and the value pass waits for aux_ev[1].
engram_status launch_history_transpose(engram_ctx* c, float* state, const Workspace& w, int32_t B, int M,
                                       cudaStream_t s) {
    const size_t hist_elems = (size_t)B * (c->cfg.conv_width - 1) * c->cfg.hidden;
    cudaError_t e = cudaEventRecord(c->aux_ev[0], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(c->aux, c->aux_ev[0], 0);
    if (e != cudaSuccess) return cuda_fail("ordering the history transpose", e);
    prof_begin(c, c->aux, "state_to_tr");
    for (int m = 0; m < M && e == cudaSuccess; ++m)
        e = launch_state_to_tr(state + m * hist_elems, w.state_t + m * hist_elems, B, c->cfg.conv_width,
                               c->cfg.hidden, c->aux);
    prof_end(c, c->aux);
    if (e == cudaSuccess) e = cudaEventRecord(c->aux_ev[1], c->aux);
    if (e != cudaSuccess) return cuda_fail("conv-state transpose launch", e);
    return ENGRAM_OK;
}

// projections + gate + conv; on the fused path two tcgen05 GEMM passes with
// the gate and the conv in the second one's epilogue, otherwise the
// projection (tcgen05 or CUDA cores) followed by the CUDA-core gate/conv.
// after_retrieve: the band counters are already cleared and the kernel just
// before on the stream is the retrieval that wrote e_cat, so the key pass
// can be its programmatic dependent (unless the decode history transpose
// records an event in between).  Timed runs (engram_profile_enable) put
// events between the kernels and launch them plainly.
engram_status gate_conv_impl(engram_ctx* c, const void* e_cat, const void* h, const void* Wk, const void* Wv,
                             const float* gq, const float* gk, const float* conv_w, int32_t B, int32_t L,
                             float* state, void* y, float* alpha_out, int32_t add_residual, const Workspace& w,
                             cudaStream_t s, bool after_retrieve = false, int M = 1, const float* kscale = nullptr,
                             const float* vscale = nullptr) {
    const bool f8 = c->cfg.dtype == ENGRAM_FP8;
    const int64_t n = (int64_t)B * L;
    const size_t hist_elems = (size_t)B * (c->cfg.conv_width - 1) * c->cfg.hidden;   // one branch's history
    if (decode_kernels(c, n, L, M)) {
        cudaError_t e = cudaSuccess;
        prof_begin(c, s, "gate_kv_decode");
        e = launch_decode_kv(e_cat, (int32_t)n, c->d_mem, h, Wk, Wv, gq, gk, c->cfg.hidden, w.part, w.v, c->d_status,
                             c->num_sms, c->debug_stall, after_retrieve && !c->prof, s);
        c->debug_stall = 0;
        prof_end(c, s);
        if (e != cudaSuccess) return cuda_fail("tcgen05 decode projections launch", e);
        prof_begin(c, s, "conv_decode");
        e = launch_decode_conv(w.v, w.part, (int32_t)n, h, conv_w, c->cfg.hidden, c->cfg.eps, w.alpha, alpha_out,
                               state, y, add_residual, c->num_sms, !c->prof, s);
        prof_end(c, s);
        if (e != cudaSuccess) return cuda_fail("decode conv launch", e);
        return ENGRAM_OK;
    }
    if (fused_path(c, n)) {
        const bool tr = state && decode_shaped(c, n, L);
        cudaError_t e = cudaSuccess;
        // after_retrieve: the forward launched the transpose ahead of the
        // retrieval, so nothing stands between the retrieval and the key pass
        if (tr && !after_retrieve) {
            engram_status st = launch_history_transpose(c, state, w, B, M, s);
            if (st != ENGRAM_OK) return st;
        }
        if (!after_retrieve) {
            e = cudaMemsetAsync(w.band, 0, w.counter_bytes, s);
            if (e != cudaSuccess) return cuda_fail("clearing the band counters", e);
        }
        prof_begin(c, s, "gate_k_tc");
        e = launch_gate_k_tc(e_cat, n, c->d_mem, h, Wk, gq, gk, c->cfg.hidden, c->cfg.eps, w.part, w.band, w.alpha,
                             alpha_out, c->d_status, c->num_sms, c->debug_stall, after_retrieve && !c->prof,
                             s, M, f8, kscale);
        c->debug_stall = 0;
        prof_end(c, s);
        if (e != cudaSuccess) return cuda_fail("tcgen05 key/gate launch", e);
        if (tr) {
            e = cudaStreamWaitEvent(s, c->aux_ev[1], 0);
            if (e != cudaSuccess) return cuda_fail("joining the history transpose", e);
        }
        prof_begin(c, s, "vconv_tc");
        e = launch_vconv_tc(e_cat, B, L, c->d_mem, h, Wv, conv_w, c->cfg.hidden, c->cfg.conv_width, w.alpha,
                            tr ? w.state_t : state, w.state_next, tr ? 1 : 0, y, add_residual, c->d_status,
                            c->num_sms, !tr && !c->prof, s, M, f8, vscale);
        prof_end(c, s);
        if (e != cudaSuccess) return cuda_fail("tcgen05 value/conv launch", e);
        if (state) {
            prof_begin(c, s, "state_merge");
            for (int m = 0; m < M && e == cudaSuccess; ++m)
                e = tr ? launch_state_merge_tr(state + m * hist_elems, w.state_next + m * hist_elems, B, L,
                                               c->cfg.conv_width, c->cfg.hidden, s)
                       : launch_state_merge(state + m * hist_elems, w.state_next + m * hist_elems, B, L,
                                            c->cfg.conv_width, c->cfg.hidden, c->num_sms, s);
            prof_end(c, s);
            if (e != cudaSuccess) return cuda_fail("conv-state merge launch", e);
        }
        return ENGRAM_OK;
    }
    if (M != 1 || f8 || kscale || vscale) {
        set_error("multi-branch, FP8 and scaled projections run on the fused tensor-core path only");
        return ENGRAM_E_UNSUPPORTED;
    }
    engram_status st = project_impl(c, e_cat, n, h, Wk, Wv, gq, gk, w.v, w.part, s);
    if (st != ENGRAM_OK) return st;
    return conv_impl(c, w.v, w.part, h, conv_w, B, L, state, y, alpha_out, add_residual, s);
}

engram_status check_forward_args(const engram_ctx* c, int32_t B, int32_t T, int64_t tok_stride, int32_t t_begin) {
    if (!c) return inval("null context");
    if (B < 0 || T < 0 || t_begin < 0 || t_begin > T) return inval("need B >= 0 and 0 <= t_begin <= T");
    if (tok_stride < T) return inval("tok_stride must be >= T");
    return ENGRAM_OK;
}

engram_status forward_impl(engram_ctx* c, const int32_t* tok, int32_t B, int32_t T, int64_t tok_stride,
                           int32_t t_begin, const int32_t* P, const void* tables, const void* h, const void* Wk,
                           const void* Wv, const float* gq, const float* gk, const float* conv_w, float* conv_state,
                           void* y, float* alpha_out, int32_t add_residual, const Workspace& w, cudaStream_t s,
                           const ShardParams* shards, int M, const float* kscale, const float* vscale) {
    const int32_t L = T - t_begin;
    const bool fused = fused_path(c, (int64_t)B * L);
    if (fused && conv_state && decode_shaped(c, (int64_t)B * L, L) && !decode_kernels(c, (int64_t)B * L, L, M)) {
        engram_status st = launch_history_transpose(c, conv_state, w, B, M, s);
        if (st != ENGRAM_OK) return st;
    }
    if (fused && !decode_kernels(c, (int64_t)B * L, L, M)) {
        // cleared ahead of the retrieval, so that the key pass directly follows it
        cudaError_t e = cudaMemsetAsync(w.band, 0, w.counter_bytes, s);
        if (e != cudaSuccess) return cuda_fail("clearing the band counters", e);
    }
    prof_begin(c, s, shards ? "retrieve_sharded" : "retrieve");
    cudaError_t e = shards ? launch_retrieve_sharded(tok, P, B, T, tok_stride, t_begin, c->hp, c->gp, *shards, w.idx,
                                                     w.e, c->d_status, c->num_sms, s)
                           : launch_retrieve(tok, P, B, T, tok_stride, t_begin, c->hp, c->gp, tables, w.idx, w.e,
                                             c->d_status, c->num_sms, s);
    prof_end(c, s);
    if (e != cudaSuccess) return cuda_fail("retrieve (hash + gather) launch", e);
    return gate_conv_impl(c, w.e, h, Wk, Wv, gq, gk, conv_w, B, L, conv_state, y, alpha_out, add_residual, w, s,
                          fused, M, kscale, vscale);
}

}  // namespace engram

using namespace engram;

extern "C" {

const char* engram_last_error(void) { return g_last_error; }

const char* engram_strerror(engram_status s) {
    switch (s) {
        case ENGRAM_OK: return "ok";
        case ENGRAM_E_INVAL: return "invalid argument";
        case ENGRAM_E_CUDA: return "CUDA runtime error";
        case ENGRAM_E_NOMEM: return "out of memory or workspace too small";
        case ENGRAM_E_UNSUPPORTED: return "unsupported";
        case ENGRAM_E_TIMEOUT: return "device wait timed out";
        case ENGRAM_E_HOST: return "host-tier failure";
        case ENGRAM_E_DEVICE: return "device reported a data error";
    }
    return "unknown status";
}

engram_status engram_create(const engram_config* cfg, engram_ctx** out) {
    if (!cfg || !out) return inval("null config or output pointer");
    *out = nullptr;
    const engram_config& k = *cfg;
    if (k.n_orders < 1 || k.n_orders > 4) return inval("n_orders must be in 1..4");
    int max_order = 0;
    for (int o = 0; o < k.n_orders; ++o) {
        if (k.orders[o] < 1 || k.orders[o] > 4) return inval("each order must be in 1..4");
        if (o > 0 && k.orders[o] <= k.orders[o - 1]) return inval("orders must be strictly ascending");
        if (k.orders[o] > max_order) max_order = k.orders[o];
    }
    if (k.heads < 1) return inval("heads must be >= 1");
    const int J = k.n_orders * k.heads;
    if (J > ENGRAM_MAX_TABLES) return inval("n_orders * heads must be <= 32");
    for (int j = 0; j < J; ++j) {
        if (k.rows[j] >= 0x80000000u || !is_prime_u32(k.rows[j])) return inval("every table size must be a prime < 2^31");
    }
    if (k.dtype != ENGRAM_F32 && k.dtype != ENGRAM_BF16 && k.dtype != ENGRAM_FP8) return inval("unknown dtype");
    const int es = k.dtype == ENGRAM_F32 ? 4 : (k.dtype == ENGRAM_BF16 ? 2 : 1);
    if (k.dtype == ENGRAM_FP8 &&
        (k.hidden % 128 != 0 || ((int64_t)n_tables_of(k) * k.row_dim) % 128 != 0 || k.conv_width != 4))
        return inval("FP8 needs hidden and J*row_dim multiples of 128 and conv width 4 (the fused path)");
    if (k.row_dim < 1 || ((int64_t)k.row_dim * es) % 16 != 0) return inval("row_dim * element size must be a multiple of 16 bytes");
    if (k.hidden < 8 || k.hidden % 8 != 0) return inval("hidden must be a positive multiple of 8");
    if (k.conv_width < 1 || k.conv_width > kMaxConv) return inval("conv_width must be in 1..8");
    if (k.vocab < 1) return inval("vocab must be >= 1");
    if (k.canon_vocab < 1 || k.canon_vocab >= 0x7FFFFFFF) return inval("canon_vocab must be in [1, 2^31 - 1)");
    if (!(k.eps >= 0.f) || !std::isfinite(k.eps)) return inval("eps must be finite and >= 0");

    engram_ctx* c = new (std::nothrow) engram_ctx();
    if (!c) return ENGRAM_E_NOMEM;
    c->cfg = k;
    c->J = J;
    c->es = es;
    c->hs = k.dtype == ENGRAM_F32 ? 4 : 2;
    c->d_mem = J * k.row_dim;
    c->G = (k.hidden + kGroup - 1) / kGroup;
    cudaError_t e = cudaGetDevice(&c->device);
    if (e != cudaSuccess) {
        delete c;
        return cuda_fail("cudaGetDevice", e);
    }
    int major = 0;
    cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, c->device);
    c->sm100 = (major == 10);

    std::memset(&c->hp, 0, sizeof(c->hp));
    for (int j = 0; j < J; ++j) {
        for (int q = 0; q < 4; ++q) c->hp.mult[j][q] = k.mult[j][q];
        c->hp.rows[j] = k.rows[j];
        c->hp.recip[j] = ~(uint64_t)0 / k.rows[j];
    }
    for (int o = 0; o < 4; ++o) c->hp.orders[o] = o < k.n_orders ? k.orders[o] : 0;
    c->hp.n_orders = k.n_orders;
    c->hp.K = k.heads;
    c->hp.J = J;
    c->hp.max_order = max_order;
    c->hp.V = k.vocab;
    c->hp.Vc = k.canon_vocab;

    std::memset(&c->gp, 0, sizeof(c->gp));
    int64_t off = 0;
    for (int j = 0; j < J; ++j) {
        c->gp.row_off[j] = off;
        c->gp.rows[j] = k.rows[j];
        off += k.rows[j];
    }
    c->gp.J = J;
    c->gp.chunks_per_row = k.row_dim * es / 16;

    e = cudaMalloc(&c->d_status, 256);
    if (e != cudaSuccess) {
        delete c;
        return e == cudaErrorMemoryAllocation ? ENGRAM_E_NOMEM : cuda_fail("cudaMalloc status", e);
    }
    e = cudaMemset(c->d_status, 0, 256);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->io_h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->io_d2h, cudaStreamNonBlocking);
    for (int i = 0; i < kIoEvents && e == cudaSuccess; ++i)
        e = cudaEventCreateWithFlags(&c->io_ev[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c->aux, cudaStreamNonBlocking);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&c->aux_ev[i], cudaEventDisableTiming);
    if (e != cudaSuccess) {
        engram_destroy(c);
        return cuda_fail("context set-up (status word, copy streams, events)", e);
    }
    *out = c;
    return ENGRAM_OK;
}

void engram_destroy(engram_ctx* c) {
    if (!c) return;
    if (c->prof)
        for (int i = 0; i < 2 * kMaxProf; ++i) cudaEventDestroy(c->ev[i]);
    for (int i = 0; i < kIoEvents; ++i)
        if (c->io_ev[i]) cudaEventDestroy(c->io_ev[i]);
    for (int i = 0; i < 2; ++i)
        if (c->aux_ev[i]) cudaEventDestroy(c->aux_ev[i]);
    if (c->aux) cudaStreamDestroy(c->aux);
    if (c->io_h2d) cudaStreamDestroy(c->io_h2d);
    if (c->io_d2h) cudaStreamDestroy(c->io_d2h);
    if (c->d_status) cudaFree(c->d_status);
    delete c;
}

size_t engram_workspace_bytes(const engram_ctx* c, int32_t B, int32_t L) {
    if (!c || B < 0 || L < 0) return 0;
    return carve(c, nullptr, B, L, true).bytes;
}

engram_status engram_debug_stall_next(engram_ctx* c) {
    if (!c) return inval("null context");
    c->debug_stall = 1;
    return ENGRAM_OK;
}

engram_status engram_profile_enable(engram_ctx* c, int32_t enable) {
    if (!c) return inval("null context");
    if (enable && !c->prof) {
        for (int i = 0; i < 2 * kMaxProf; ++i) {
            cudaError_t e = cudaEventCreate(&c->ev[i]);
            if (e != cudaSuccess) {
                for (int k = 0; k < i; ++k) cudaEventDestroy(c->ev[k]);
                return cuda_fail("cudaEventCreate", e);
            }
        }
        c->prof = true;
    } else if (!enable && c->prof) {
        for (int i = 0; i < 2 * kMaxProf; ++i) cudaEventDestroy(c->ev[i]);
        c->prof = false;
    }
    c->prof_n = 0;
    return ENGRAM_OK;
}

int32_t engram_profile_read(engram_ctx* c, float* ms, const char** names, int32_t max) {
    if (!c || !c->prof) return 0;
    int n = c->prof_n < max ? c->prof_n : max;
    for (int i = 0; i < n; ++i) {
        float t = -1.f;
        if (cudaEventSynchronize(c->ev[2 * i + 1]) != cudaSuccess ||
            cudaEventElapsedTime(&t, c->ev[2 * i], c->ev[2 * i + 1]) != cudaSuccess) {
            t = -1.f;
            cudaGetLastError();   // a failed query must not surface at the next launch
        }
        if (ms) ms[i] = t;
        if (names) names[i] = c->prof_name[i];
    }
    return n;
}

engram_status engram_device_status(engram_ctx* c, cudaStream_t s, uint32_t* flags) {
    if (!c) return inval("null context");
    uint32_t h = 0;
    cudaError_t e = cudaMemcpyAsync(&h, c->d_status, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail("reading the device status word", e);
    if (h) {
        e = cudaMemsetAsync(c->d_status, 0, sizeof(uint32_t), s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_fail("clearing the device status word", e);
    }
    if (flags) *flags = h;
    if (h & ENGRAM_ERR_TIMEOUT) return ENGRAM_E_TIMEOUT;
    return h ? ENGRAM_E_DEVICE : ENGRAM_OK;
}

engram_status engram_remap(engram_ctx* c, const int32_t* tok, int64_t n, const int32_t* P, int32_t* canon,
                           cudaStream_t s) {
    if (!c) return inval("null context");
    if (n < 0) return inval("n must be >= 0");
    if (n > 0 && (!tok || !P || !canon)) return inval("null tensor pointer");
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    prof_begin(c, s, "remap");
    cudaError_t e = launch_remap(tok, n, P, c->cfg.vocab, canon, c->d_status, s);
    prof_end(c, s);
    return launched("remap launch", e);
}

engram_status engram_hash(engram_ctx* c, const int32_t* ids, const int32_t* P, int32_t B, int32_t T,
                          int64_t stride, int32_t t_begin, uint32_t* idx, cudaStream_t s) {
    if (!c) return inval("null context");
    if (B < 0 || T < 0 || t_begin < 0 || t_begin > T) return inval("need B >= 0 and 0 <= t_begin <= T");
    if (stride < T) return inval("stride must be >= T");
    if ((int64_t)B * (T - t_begin) == 0) return ENGRAM_OK;
    if (!ids || !idx) return inval("null tensor pointer");
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    prof_begin(c, s, "hash");
    cudaError_t e = launch_hash(ids, P, B, T, stride, t_begin, idx, c->hp, c->d_status, s);
    prof_end(c, s);
    return launched("hash launch", e);
}

engram_status engram_gather(engram_ctx* c, const uint32_t* idx, int64_t n_tok, const void* tables,
                            void* e_cat, cudaStream_t s) {
    if (!c) return inval("null context");
    if (n_tok < 0) return inval("n_tok must be >= 0");
    if (n_tok == 0) return ENGRAM_OK;
    if (!idx || !tables || !e_cat) return inval("null tensor pointer");
    if (!aligned16(tables) || !aligned16(e_cat)) return inval("tables and e_cat must be 16-byte aligned");
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    prof_begin(c, s, "gather");
    cudaError_t e = launch_gather(idx, n_tok, tables, c->gp, e_cat, c->d_status, c->num_sms, s);
    prof_end(c, s);
    return launched("gather launch", e);
}

engram_status engram_project(engram_ctx* c, const void* e_cat, int64_t n_tok, const void* h, const void* Wk,
                             const void* Wv, const float* gq, const float* gk, float* v, float* part,
                             cudaStream_t s) {
    if (!c) return inval("null context");
    if (n_tok < 0) return inval("n_tok must be >= 0");
    if (n_tok == 0) return ENGRAM_OK;
    if (!e_cat || !h || !Wk || !Wv || !v || !part) return inval("null tensor pointer");
    if (c->cfg.dtype == ENGRAM_FP8) {
        set_error("engram_project: FP8 runs on the fused forward only");
        return ENGRAM_E_UNSUPPORTED;
    }
    if (!aligned16(e_cat) || !aligned16(h) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(v) || !aligned16(part))
        return inval("e_cat, h, Wk, Wv, v and part must be 16-byte aligned");
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    return project_impl(c, e_cat, n_tok, h, Wk, Wv, gq, gk, v, part, s);
}

engram_status engram_conv(engram_ctx* c, const float* v, const float* part, const void* h, const float* conv_w,
                          int32_t B, int32_t L, float* conv_state, void* y, float* alpha_out,
                          int32_t add_residual, cudaStream_t s) {
    if (!c) return inval("null context");
    if (B < 0 || L < 0) return inval("B and L must be >= 0");
    if ((int64_t)B * L == 0) return ENGRAM_OK;
    if (!v || !part || !conv_w || !y || (add_residual && !h)) return inval("null tensor pointer");
    if (c->cfg.dtype == ENGRAM_FP8) {
        set_error("engram_conv: FP8 runs on the fused forward only");
        return ENGRAM_E_UNSUPPORTED;
    }
    if (!aligned16(v) || !aligned16(part) || !aligned16(y) || (add_residual && !aligned16(h)) ||
        (conv_state && !aligned16(conv_state)) || !aligned16(conv_w))
        return inval("v, part, y, h, conv_w and conv_state must be 16-byte aligned");
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    return conv_impl(c, v, part, h, conv_w, B, L, conv_state, y, alpha_out, add_residual, s);
}

engram_status engram_gate_conv(engram_ctx* c, const void* e_cat, const void* h, const void* Wk, const void* Wv,
                               const float* gq, const float* gk, const float* conv_w, int32_t B, int32_t L,
                               float* conv_state, void* y, float* alpha_out, int32_t add_residual,
                               void* workspace, size_t workspace_bytes, cudaStream_t s) {
    if (!c) return inval("null context");
    if (B < 0 || L < 0) return inval("B and L must be >= 0");
    const int64_t n = (int64_t)B * L;
    if (n == 0) return ENGRAM_OK;
    if (!e_cat || !h || !Wk || !Wv || !conv_w || !y || !workspace) return inval("null tensor pointer");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return inval("workspace must be 256-byte aligned");
    Workspace w = carve(c, workspace, B, L, false);
    if (workspace_bytes < w.bytes) return ENGRAM_E_NOMEM;
    if (!aligned16(e_cat) || !aligned16(h) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(y) ||
        (conv_state && !aligned16(conv_state)) || !aligned16(conv_w))
        return inval("e_cat, h, Wk, Wv, y, conv_w and conv_state must be 16-byte aligned");
    engram_status st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    return gate_conv_impl(c, e_cat, h, Wk, Wv, gq, gk, conv_w, B, L, conv_state, y, alpha_out, add_residual, w, s);
}

engram_status engram_forward(engram_ctx* c, const int32_t* tok, int32_t B, int32_t T, int64_t tok_stride,
                             int32_t t_begin, const int32_t* P, const void* tables, const void* h, const void* Wk,
                             const void* Wv, const float* gq, const float* gk, const float* conv_w,
                             float* conv_state, void* y, float* alpha_out, int32_t add_residual, void* workspace,
                             size_t workspace_bytes, cudaStream_t s) {
    engram_status st = check_forward_args(c, B, T, tok_stride, t_begin);
    if (st != ENGRAM_OK) return st;
    const int32_t L = T - t_begin;
    const int64_t n = (int64_t)B * L;
    if (n == 0) return ENGRAM_OK;
    if (!tok || !P || !tables || !h || !Wk || !Wv || !conv_w || !y || !workspace) return inval("null tensor pointer");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return inval("workspace must be 256-byte aligned");
    Workspace w = carve(c, workspace, B, L, true);
    if (workspace_bytes < w.bytes) return ENGRAM_E_NOMEM;
    if (!aligned16(tables) || !aligned16(h) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(y) ||
        (conv_state && !aligned16(conv_state)) || !aligned16(conv_w))
        return inval("tables, h, Wk, Wv, y, conv_w and conv_state must be 16-byte aligned");
    st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    return forward_impl(c, tok, B, T, tok_stride, t_begin, P, tables, h, Wk, Wv, gq, gk, conv_w, conv_state, y,
                        alpha_out, add_residual, w, s);
}

// ---------------------------------------------------------------- multi-branch

size_t engram_multibranch_workspace_bytes(const engram_ctx* c, int32_t M, int32_t B, int32_t L) {
    if (!c || M < 1 || M > ENGRAM_MAX_BRANCHES || B < 0 || L < 0) return 0;
    return carve(c, nullptr, B, L, true, M).bytes;
}

engram_status engram_forward_multibranch(engram_ctx* c, int32_t M, const int32_t* tok, int32_t B, int32_t T,
                                         int64_t tok_stride, int32_t t_begin, const int32_t* P, const void* tables,
                                         const void* h, const void* Wk, const void* Wv, const float* gq,
                                         const float* gk, const float* k_scale, const float* v_scale,
                                         const float* conv_w, float* conv_state, void* y, float* alpha_out,
                                         int32_t add_residual, void* workspace, size_t workspace_bytes,
                                         cudaStream_t s) {
    engram_status st = check_forward_args(c, B, T, tok_stride, t_begin);
    if (st != ENGRAM_OK) return st;
    if (M < 1 || M > ENGRAM_MAX_BRANCHES) return inval("M must be in 1..4");
    const int32_t L = T - t_begin;
    const int64_t n = (int64_t)B * L;
    if (n == 0) return ENGRAM_OK;
    if (!fused_path(c, n)) {
        set_error("the multi-branch forward runs on the fused tensor-core path only (bf16 or FP8, conv width 4, d "
                  "a multiple of 128, J*D a multiple of 64 (128 for FP8))");
        return ENGRAM_E_UNSUPPORTED;
    }
    if (c->cfg.dtype == ENGRAM_FP8) {
        if (!k_scale || !v_scale) return inval("FP8 needs k_scale and v_scale (the dequantisation scales)");
        if (!aligned16(k_scale) || !aligned16(v_scale)) return inval("k_scale and v_scale must be 16-byte aligned");
    } else if (k_scale || v_scale) {
        return inval("k_scale and v_scale dequantise FP8 operands: pass null for other dtypes");
    }
    if (!tok || !P || !tables || !h || !Wk || !Wv || !conv_w || !y || !workspace) return inval("null tensor pointer");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return inval("workspace must be 256-byte aligned");
    Workspace w = carve(c, workspace, B, L, true, M);
    if (workspace_bytes < w.bytes) return ENGRAM_E_NOMEM;
    if (!aligned16(tables) || !aligned16(h) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(y) ||
        (conv_state && !aligned16(conv_state)) || !aligned16(conv_w))
        return inval("tables, h, Wk, Wv, y, conv_w and conv_state must be 16-byte aligned");
    st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    return forward_impl(c, tok, B, T, tok_stride, t_begin, P, tables, h, Wk, Wv, gq, gk, conv_w, conv_state, y,
                        alpha_out, add_residual, w, s, nullptr, M, k_scale, v_scale);
}

// ---------------------------------------------------------------- tables sharded across GPUs

engram_status engram_shard_range(const engram_ctx* c, int32_t n_shards, int32_t shard, int64_t* first_row,
                                 int64_t* n_rows) {
    if (!c || !first_row || !n_rows) return inval("null context or output pointer");
    if (n_shards < 1 || n_shards > kMaxShards) return inval("n_shards must be in 1..16");
    if (shard < 0 || shard >= n_shards) return inval("shard must be in [0, n_shards)");
    int64_t total = 0;
    for (int j = 0; j < c->J; ++j) total += c->cfg.rows[j];
    const int64_t per = (total + n_shards - 1) / n_shards;
    const int64_t lo = std::min<int64_t>(total, (int64_t)shard * per);
    const int64_t hi = std::min<int64_t>(total, lo + per);
    *first_row = lo;
    *n_rows = hi - lo;
    return ENGRAM_OK;
}

engram_status engram_forward_sharded(engram_ctx* c, const int32_t* tok, int32_t B, int32_t T, int64_t tok_stride,
                                     int32_t t_begin, const int32_t* P, const void* const* shard_tables,
                                     int32_t n_shards, const void* h, const void* Wk, const void* Wv, const float* gq,
                                     const float* gk, const float* conv_w, float* conv_state, void* y,
                                     float* alpha_out, int32_t add_residual, void* workspace, size_t workspace_bytes,
                                     cudaStream_t s) {
    engram_status st = check_forward_args(c, B, T, tok_stride, t_begin);
    if (st != ENGRAM_OK) return st;
    if (n_shards < 1 || n_shards > kMaxShards) return inval("n_shards must be in 1..16");
    if (!shard_tables) return inval("null shard table list");
    ShardParams sp{};
    sp.n = n_shards;
    for (int g = 0; g < n_shards; ++g) {
        int64_t lo = 0, cnt = 0;
        engram_shard_range(c, n_shards, g, &lo, &cnt);
        if (cnt > 0 && !shard_tables[g]) return inval("null shard pointer");
        if (!aligned16(shard_tables[g])) return inval("every shard must be 16-byte aligned");
        sp.base[g] = static_cast<const uint4*>(shard_tables[g]);
        sp.bound[g] = lo;
        sp.bound[g + 1] = lo + cnt;
    }
    const int32_t L = T - t_begin;
    const int64_t n = (int64_t)B * L;
    if (n == 0) return ENGRAM_OK;
    if (!tok || !P || !h || !Wk || !Wv || !conv_w || !y || !workspace) return inval("null tensor pointer");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return inval("workspace must be 256-byte aligned");
    Workspace w = carve(c, workspace, B, L, true);
    if (workspace_bytes < w.bytes) return ENGRAM_E_NOMEM;
    if (!aligned16(h) || !aligned16(Wk) || !aligned16(Wv) || !aligned16(y) ||
        (conv_state && !aligned16(conv_state)) || !aligned16(conv_w))
        return inval("h, Wk, Wv, y, conv_w and conv_state must be 16-byte aligned");
    st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);
    return forward_impl(c, tok, B, T, tok_stride, t_begin, P, nullptr, h, Wk, Wv, gq, gk, conv_w, conv_state, y,
                        alpha_out, add_residual, w, s, &sp);
}

// Cross-process mapping of a shard: the allocation that holds `ptr` is
// exported as a CUDA IPC handle plus the offset of `ptr` inside it.
engram_status engram_ipc_export(const void* ptr, void* handle_out, uint64_t* offset_out) {
    if (!ptr || !handle_out || !offset_out) return inval("null pointer");
    static CUresult (*get_range)(CUdeviceptr*, size_t*, CUdeviceptr) = nullptr;
    if (!get_range) {
        void* q = nullptr;
        cudaDriverEntryPointQueryResult res;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &q, cudaEnableDefault, &res) != cudaSuccess ||
            res != cudaDriverEntryPointSuccess)
            return cuda_fail("cuMemGetAddressRange entry point", cudaErrorNotSupported);
        get_range = reinterpret_cast<CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr)>(q);
    }
    CUdeviceptr base = 0;
    size_t size = 0;
    if (get_range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
        return inval("the pointer is not inside a device allocation");
    cudaIpcMemHandle_t hd;
    cudaError_t e = cudaIpcGetMemHandle(&hd, reinterpret_cast<void*>(base));
    if (e != cudaSuccess) return cuda_fail("cudaIpcGetMemHandle", e);
    std::memcpy(handle_out, &hd, sizeof(hd));
    *offset_out = reinterpret_cast<uint64_t>(ptr) - (uint64_t)base;
    return ENGRAM_OK;
}

engram_status engram_ipc_open(const void* handle, uint64_t offset, void** ptr_out, void** base_out) {
    if (!handle || !ptr_out || !base_out) return inval("null pointer");
    cudaIpcMemHandle_t hd;
    std::memcpy(&hd, handle, sizeof(hd));
    void* base = nullptr;
    cudaError_t e = cudaIpcOpenMemHandle(&base, hd, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return cuda_fail("cudaIpcOpenMemHandle", e);
    *base_out = base;
    *ptr_out = static_cast<char*>(base) + offset;
    return ENGRAM_OK;
}

engram_status engram_ipc_close(void* base) {
    if (!base) return inval("null pointer");
    cudaError_t e = cudaIpcCloseMemHandle(base);
    if (e != cudaSuccess) return cuda_fail("cudaIpcCloseMemHandle", e);
    return ENGRAM_OK;
}

// ---------------------------------------------------------------- forward without allocation
//
// For callers that cannot allocate device memory at all: an inference
// engine's execution callback that forbids allocation, a process whose device
// memory is already handed to another allocator, or a latency-critical loop
// that must avoid cudaMalloc's implicit synchronisation.  They get the forward
// with its scratch in this file-scope device array instead of a caller
// workspace.  Every GPU that loads the library holds the array until exit.

}  // extern "C"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ENGRAM_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64];   // device address of g_noalloc_scratch per device ordinal, from the last lookup

// Device address of the static scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with that device current.  The lookup is repeated on every call whose
// stream is not capturing (a cheap table lookup once the module is loaded),
// so a device reset or a new primary context never leaves a stale address;
// a capturing stream uses the address of the last uncaptured call, so the
// first call on a device must come before any stream capture.
engram_status noalloc_scratch(cudaStream_t s, void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= 64) return inval("device ordinal out of range for the static scratch");
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(s, &cap);
    if (e != cudaSuccess) return cuda_fail("cudaStreamIsCapturing", e);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress of the static scratch", e);
        g_noalloc_ptr[dev] = p;
    } else if (!g_noalloc_ptr[dev]) {
        return inval("engram_forward_noalloc: the first call on a device must come before any stream capture");
    }
    *out = g_noalloc_ptr[dev];
    return ENGRAM_OK;
}

}  // namespace

extern "C" {

engram_status engram_forward_noalloc(engram_ctx* c, const int32_t* tok, int32_t B, int32_t T, int64_t tok_stride,
                                     int32_t t_begin, const int32_t* P, const void* tables, const void* h,
                                     const void* Wk, const void* Wv, const float* gq, const float* gk,
                                     const float* conv_w, float* conv_state, void* y, float* alpha_out,
                                     int32_t add_residual, cudaStream_t s) {
    engram_status st = check_forward_args(c, B, T, tok_stride, t_begin);
    if (st != ENGRAM_OK) return st;
    // on the wrong device nothing (not even the scratch lookup) touches it
    st = check_device(c);
    if (st != ENGRAM_OK) return st;
    const size_t need = carve(c, nullptr, B, T - t_begin, true).bytes;
    if (need > (size_t)ENGRAM_NOALLOC_SCRATCH_BYTES) {
        std::snprintf(g_last_error, sizeof(g_last_error),
                      "engram_forward_noalloc: %zu bytes of scratch needed, the static scratch holds %zu; "
                      "use engram_forward with a workspace or split the batch",
                      need, (size_t)ENGRAM_NOALLOC_SCRATCH_BYTES);
        return ENGRAM_E_NOMEM;
    }
    void* scratch = nullptr;
    st = noalloc_scratch(s, &scratch);
    if (st != ENGRAM_OK) return st;
    return engram_forward(c, tok, B, T, tok_stride, t_begin, P, tables, h, Wk, Wv, gq, gk, conv_w, conv_state, y,
                          alpha_out, add_residual, scratch, (size_t)ENGRAM_NOALLOC_SCRATCH_BYTES, s);
}

}  // extern "C"
