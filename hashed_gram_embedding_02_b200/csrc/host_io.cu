// engram_forward_host: the forward with its per-token tensors (ids, hidden
// states, output) in host memory.
//
// The retrieval depends only on token ids (Synced repost of the Engram
// announcement, section "System efficiency: decoupling compute and
// storage"), and every row's output depends only on its own row of h plus a
// three-row conv history, so the batch splits into chunks of positions that
// pipeline over PCIe: while chunk i computes on the caller's stream, the h of
// chunk i+1 comes in on one copy stream and the Y of chunk i-1 goes out on
// the other.  Two device buffers per direction; events order each reuse.
// The conv history crosses chunk boundaries through conv_state (the caller's,
// or a zeroed one in the workspace), exactly as a decode step continues a
// prefill.
//
// Chunk sizes (chunk_rows = 0): a long batch runs 16 MiB chunks of h, whose
// compute is short next to their copies, so the copies run back to back;
// the first three chunks grow from 2 to 8 MiB and the last three shrink
// again, so that the first compute starts early and the last copy out is
// short.  A batch under four 16 MiB chunks runs uniform chunks of about
// 4 MiB.  chunk_rows > 0 fixes uniform chunks of that many positions.
#include <algorithm>

#include "ctx.cuh"

namespace engram {
namespace {

constexpr size_t kShortChunkBytes = 4u << 20;   // h bytes per uniform chunk when chunk_rows = 0 (short batches)
constexpr size_t kLongChunkBytes = 16u << 20;   // h bytes per middle chunk of a long batch
constexpr int kRamp = 3;                        // chunks of 1/8, 1/4, 1/2 the middle size at each end

enum IoEvent { EV_START = 0, EV_H_READY = 1, EV_COMPUTED = 3, EV_DRAINED = 5, EV_DONE = 7 };
static_assert(EV_DONE < kIoEvents, "event slots");

struct HostPlan {
    int32_t lo;          // first id position copied per sequence
    int32_t Tw;          // ids copied per sequence (T - lo)
    int32_t R;           // positions per chunk at most (the buffers' size)
    int32_t n_ramp;      // ramp chunks at each end (0: uniform chunks of R)
    int32_t ramp_rows;   // positions in the chunks of one ramp
    int32_t n_mid;       // middle chunks, each of R positions but the last
    int32_t mid_rows;    // positions in the middle chunks
    int32_t n_chunks;
    size_t row_bytes;    // one position of h or Y
    size_t tok_off, state_off, h_off[2], y_off[2], fwd_off;
    size_t bytes;
};

HostPlan make_plan(const engram_ctx* c, int32_t B, int32_t T, int32_t t_begin, int32_t chunk_rows) {
    HostPlan p{};
    const int32_t L = T - t_begin;
    p.lo = std::max(0, t_begin - (c->hp.max_order - 1));
    p.Tw = T - p.lo;
    p.row_bytes = (size_t)c->cfg.hidden * c->hs;
    const size_t seq_row = std::max<size_t>(1, (size_t)B * p.row_bytes);   // one position of every sequence
    int64_t R = chunk_rows;
    const int64_t R_long = (int64_t)std::max<size_t>(1, kLongChunkBytes / seq_row);
    if (R <= 0 && R_long >= 8 && (int64_t)L >= 4 * R_long) {
        // ramp up, 16 MiB chunks, ramp down
        R = R_long;
        p.n_ramp = kRamp;
        for (int i = 0; i < kRamp; ++i) p.ramp_rows += (int32_t)(R >> (kRamp - i));
    } else if (R <= 0) {
        R = (int64_t)std::max<size_t>(1, kShortChunkBytes / seq_row);
    }
    R = std::min<int64_t>(R, std::max(L, 1));
    p.R = (int32_t)R;
    p.mid_rows = L - 2 * p.ramp_rows;
    p.n_mid = p.mid_rows > 0 ? (int32_t)((p.mid_rows + R - 1) / R) : 0;
    p.n_chunks = L > 0 ? p.n_mid + 2 * p.n_ramp : 0;
    const size_t chunk_bytes = (size_t)B * R * p.row_bytes;
    size_t off = 0;
    p.tok_off = off;
    off += align256((size_t)B * p.Tw * sizeof(int32_t));
    // carried conv history for callers without conv_state (several chunks only)
    p.state_off = off;
    if (p.n_chunks > 1) off += align256((size_t)B * (c->cfg.conv_width - 1) * c->cfg.hidden * sizeof(float));
    for (int i = 0; i < 2; ++i) {
        p.h_off[i] = off;
        off += align256(chunk_bytes);
    }
    for (int i = 0; i < 2; ++i) {
        p.y_off[i] = off;
        off += align256(chunk_bytes);
    }
    p.fwd_off = off;
    off += carve(c, nullptr, B, R, true).bytes;
    p.bytes = off;
    return p;
}

// positions [*r0, *r0 + *rc) of chunk ci
void chunk_of(const HostPlan& p, int32_t ci, int32_t* r0, int32_t* rc) {
    if (ci < p.n_ramp) {   // growing: R/8, R/4, R/2
        int32_t o = 0;
        for (int i = 0; i < ci; ++i) o += p.R >> (p.n_ramp - i);
        *r0 = o;
        *rc = p.R >> (p.n_ramp - ci);
        return;
    }
    const int32_t j = ci - p.n_ramp;
    if (j < p.n_mid) {
        *r0 = p.ramp_rows + j * p.R;
        *rc = std::min(p.R, p.mid_rows - j * p.R);
        return;
    }
    const int32_t k = j - p.n_mid;   // shrinking: R/2, R/4, R/8
    int32_t o = p.ramp_rows + p.mid_rows;
    for (int i = 0; i < k; ++i) o += p.R >> (i + 1);
    *r0 = o;
    *rc = p.R >> (k + 1);
}

}  // namespace
}  // namespace engram

using namespace engram;

extern "C" {

size_t engram_host_workspace_bytes(const engram_ctx* c, int32_t B, int32_t T, int32_t t_begin, int32_t chunk_rows) {
    if (!c || B < 0 || T < 0 || t_begin < 0 || t_begin > T) return 0;
    return make_plan(c, B, T, t_begin, chunk_rows).bytes;
}

engram_status engram_forward_host(engram_ctx* c, const int32_t* tok_host, int32_t B, int32_t T, int64_t tok_stride,
                                  int32_t t_begin, const int32_t* P, const void* tables, const void* h_host,
                                  const void* Wk, const void* Wv, const float* gq, const float* gk,
                                  const float* conv_w, float* conv_state, void* y_host, int32_t add_residual,
                                  int32_t chunk_rows, void* workspace, size_t workspace_bytes, cudaStream_t s) {
    engram_status st = check_forward_args(c, B, T, tok_stride, t_begin);
    if (st != ENGRAM_OK) return st;
    const int32_t L = T - t_begin;
    if ((int64_t)B * L == 0) return ENGRAM_OK;
    if (!tok_host || !P || !tables || !h_host || !Wk || !Wv || !conv_w || !y_host || !workspace)
        return inval("null pointer");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return inval("workspace must be 256-byte aligned");
    const HostPlan p = make_plan(c, B, T, t_begin, chunk_rows);
    if (workspace_bytes < p.bytes) return ENGRAM_E_NOMEM;
    if (!aligned16(tables) || !aligned16(Wk) || !aligned16(Wv) || (conv_state && !aligned16(conv_state)) ||
        !aligned16(conv_w))
        return inval("tables, Wk, Wv, conv_w and conv_state must be 16-byte aligned");
    st = check_device(c);
    if (st != ENGRAM_OK) return st;
    prof_reset(c);

    char* base = static_cast<char*>(workspace);
    int32_t* tok_d = reinterpret_cast<int32_t*>(base + p.tok_off);
    // one chunk with no caller history needs no carried state (zero history)
    float* state = conv_state ? conv_state
                              : (p.n_chunks > 1 ? reinterpret_cast<float*>(base + p.state_off) : nullptr);
    cudaEvent_t* ev = c->io_ev;
    const char* h_src = static_cast<const char*>(h_host);
    char* y_dst = static_cast<char*>(y_host);
    const size_t seq_bytes = (size_t)L * p.row_bytes;   // one sequence of h or Y on the host

#define IO_TRY(call, what)                                \
    do {                                                  \
        cudaError_t e_ = (call);                          \
        if (e_ != cudaSuccess) return cuda_fail(what, e_); \
    } while (0)

    // the copies follow the caller's earlier work on `s` (a previous call may
    // still be reading the buffers they overwrite)
    IO_TRY(cudaEventRecord(ev[EV_START], s), "recording the start event");
    IO_TRY(cudaStreamWaitEvent(c->io_h2d, ev[EV_START], 0), "ordering the input copies");
    IO_TRY(cudaStreamWaitEvent(c->io_d2h, ev[EV_START], 0), "ordering the output copies");
    if (state && !conv_state)
        IO_TRY(cudaMemsetAsync(state, 0, (size_t)B * (c->cfg.conv_width - 1) * c->cfg.hidden * sizeof(float), s),
               "clearing the carried conv history");
    // ids of every sequence from position lo (the n-gram context of t_begin)
    IO_TRY(cudaMemcpy2DAsync(tok_d, (size_t)p.Tw * sizeof(int32_t), tok_host + p.lo,
                             (size_t)tok_stride * sizeof(int32_t), (size_t)p.Tw * sizeof(int32_t), B,
                             cudaMemcpyHostToDevice, c->io_h2d),
           "copying the ids in");

    for (int32_t ci = 0; ci < p.n_chunks; ++ci) {
        const int b = ci & 1;
        int32_t r0 = 0, rc = 0;
        chunk_of(p, ci, &r0, &rc);
        const size_t width = (size_t)rc * p.row_bytes;
        char* h_d = base + p.h_off[b];
        char* y_d = base + p.y_off[b];
        // h of this chunk in, once chunk ci-2 has finished reading the buffer
        if (ci >= 2) IO_TRY(cudaStreamWaitEvent(c->io_h2d, ev[EV_COMPUTED + b], 0), "ordering an input copy");
        IO_TRY(cudaMemcpy2DAsync(h_d, width, h_src + (size_t)r0 * p.row_bytes, seq_bytes, width, B,
                                 cudaMemcpyHostToDevice, c->io_h2d),
               "copying h in");
        IO_TRY(cudaEventRecord(ev[EV_H_READY + b], c->io_h2d), "recording an input event");
        // compute, once h is in and chunk ci-2's Y has left the buffer
        IO_TRY(cudaStreamWaitEvent(s, ev[EV_H_READY + b], 0), "ordering a chunk");
        if (ci >= 2) IO_TRY(cudaStreamWaitEvent(s, ev[EV_DRAINED + b], 0), "ordering a chunk");
        const Workspace w = carve(c, base + p.fwd_off, B, rc, true);
        st = forward_impl(c, tok_d, B, t_begin - p.lo + r0 + rc, p.Tw, t_begin - p.lo + r0, P, tables, h_d, Wk, Wv,
                          gq, gk, conv_w, state, y_d, nullptr, add_residual, w, s);
        if (st != ENGRAM_OK) return st;
        IO_TRY(cudaEventRecord(ev[EV_COMPUTED + b], s), "recording a compute event");
        // Y of this chunk out
        IO_TRY(cudaStreamWaitEvent(c->io_d2h, ev[EV_COMPUTED + b], 0), "ordering an output copy");
        IO_TRY(cudaMemcpy2DAsync(y_dst + (size_t)r0 * p.row_bytes, seq_bytes, y_d, width, width, B,
                                 cudaMemcpyDeviceToHost, c->io_d2h),
               "copying Y out");
        IO_TRY(cudaEventRecord(ev[EV_DRAINED + b], c->io_d2h), "recording an output event");
    }
    // the caller's stream completes when the last Y has landed
    IO_TRY(cudaEventRecord(ev[EV_DONE], c->io_d2h), "recording the done event");
    IO_TRY(cudaStreamWaitEvent(s, ev[EV_DONE], 0), "joining the caller's stream");
#undef IO_TRY
    return ENGRAM_OK;
}

}  // extern "C"
