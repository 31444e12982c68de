// The context behind the opaque engram_ctx handle and the host-side helpers
// that the C ABI's source files share (argument errors, workspace layout,
// kernel sequencing).  Internal: nothing here is exported.
#pragma once

#include <cstddef>

#include "common.cuh"

namespace engram {
constexpr int kMaxProf = 16;
constexpr int kIoEvents = 8;   // events of the host-buffer pipeline (engram_forward_host)
}  // namespace engram

struct engram_ctx {
    engram_config cfg;
    int device;
    int num_sms;
    bool sm100;
    int J;
    int d_mem;
    int G;
    int es;                 // element size of the tables, e and W (4, 2, or 1 for FP8)
    int hs;                 // element size of h and Y (4 for fp32, else 2: bf16)
    engram::HashParams hp;
    engram::GatherParams gp;
    uint32_t* d_status;     // device status word (256-byte block)
    // per-kernel timing (engram_profile_enable)
    bool prof;
    cudaEvent_t ev[2 * engram::kMaxProf];
    const char* prof_name[engram::kMaxProf];
    int prof_n;
    int debug_stall;        // engram_debug_stall_next: the next fused key pass stalls (one shot)
    // copy streams and events of the host-buffer pipeline, made at create time
    cudaStream_t io_h2d;
    cudaStream_t io_d2h;
    cudaEvent_t io_ev[engram::kIoEvents];
    // side stream for work that overlaps the key pass (the decode history transpose)
    cudaStream_t aux;
    cudaEvent_t aux_ev[2];
};

namespace engram {

extern thread_local char g_last_error[256];

void set_error(const char* what, cudaError_t e);
void set_error(const char* what);
engram_status inval(const char* what);
engram_status cuda_fail(const char* what, cudaError_t e);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

void prof_reset(engram_ctx* c);
void prof_begin(engram_ctx* c, cudaStream_t s, const char* name);
void prof_end(engram_ctx* c, cudaStream_t s);

engram_status check_device(const engram_ctx* c);

// Scratch of one forward over B sequences of L computed rows:
// idx [n][J] u32 | e [n][J*D] | part [n][G][4] f32 | alpha [n] f32 | band
// counters | state_next [B][w-1][d] f32 | state_t [w-1][d][B] f32 (fused
// decode-shaped calls, L <= 8) | v [n][d] f32 (unfused paths only), each
// 256-byte aligned.  With base == nullptr only `bytes` is meaningful.
struct Workspace {
    uint32_t* idx;
    void* e;
    float* part;
    float* alpha;
    int* band;
    float* state_next;
    float* state_t;     // decode-shaped fused calls: the history, sequence-minor
    float* v;
    size_t counter_bytes;   // band counters: cleared before every fused call
    size_t bytes;
};
// M > 1 (multi-branch, fused path only): part [n][M*G][4], alpha [M][n],
// state_next / state_t [M][...].
Workspace carve(const engram_ctx* c, void* base, int64_t B, int64_t L, bool with_idx_e, int M = 1);

// Argument checks shared by the forward entry points (device pointers).
engram_status check_forward_args(const engram_ctx* c, int32_t B, int32_t T, int64_t tok_stride, int32_t t_begin);

// hash -> gather -> projections + gate + conv on stream s, into workspace w
// (arguments already checked; no profiling reset).
engram_status forward_impl(engram_ctx* c, const int32_t* tok, int32_t B, int32_t T, int64_t tok_stride,
                           int32_t t_begin, const int32_t* P, const void* tables, const void* h, const void* Wk,
                           const void* Wv, const float* gq, const float* gk, const float* conv_w, float* conv_state,
                           void* y, float* alpha_out, int32_t add_residual, const Workspace& w, cudaStream_t s,
                           const ShardParams* shards = nullptr, int M = 1, const float* kscale = nullptr,
                           const float* vscale = nullptr);

}  // namespace engram
