/*
 * engram.h - C ABI of the Engram conditional-memory forward path on NVIDIA
 * B200 (sm_100a).
 *
 * The method (DeepSeek Engram; "DeepSeek AI II" digest, section "DeepSeek
 * Engram", and the Synced repost, sections "hashed N-gram sparse retrieval"
 * and "context-aware gating") processes every position t of a token sequence
 * in two stages:
 *   retrieval: x'_t = P(x_t) (tokenizer compression), suffix n-grams
 *              g_{t,n} = (x'_{t-n+1}, ..., x'_t) for each order n, K hash
 *              heads per order indexing tables E_{n,k} of prime size M_{n,k},
 *              the rows concatenated into e_t;
 *   fusion:    k_t = W_K e_t, v_t = W_V e_t, a scalar gate
 *              alpha_t = sigmoid(<RMSNorm(h_t), RMSNorm(k_t)> / sqrt(d)),
 *              v~_t = alpha_t v_t, and a short causal depthwise convolution
 *              over time giving Y_t (added to the residual stream by the
 *              caller, or here when add_residual is set).
 *
 * Readings fixed by this library where the pages give no formula:
 *   hash      phi_{n,k}(g) = (XOR_{j<n} (s_j + 1) * a_{n,k,j} mod 2^64) mod M,
 *             s_j = x'_{t-j}; s_j = PAD = V' before the sequence start;
 *             the odd 64-bit multipliers a are configuration (engram_config).
 *   concat    table order: order ascending, then head ascending;
 *             table j = o*K + k for order index o and head k.
 *   gate      q^ = g_q * h / rms(h), k^ = g_k * k / rms(k),
 *             rms(x) = sqrt(mean(x^2) + eps), alpha = sigmoid(<q^,k^>/sqrt(d)).
 *   conv      u_t = sum_{j<w} c[ch][j] * v~_{t-j} (per channel, causal;
 *             history before the first computed position from conv_state,
 *             else zero), Y_t = v~_t + SiLU(u_t) (+ h_t with add_residual).
 *   storage   bf16 configurations store e and Y as bf16; k, v, alpha and
 *             the conv history stay fp32 (v is stored, in fp32, only where
 *             the gate and conv are not fused into the projection).  The
 *             gate, the tap sum, SiLU and the residual add are fp32
 *             arithmetic on every path; Y is rounded once, when stored.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are caller-owned DEVICE memory unless stated; the
 *     library never allocates per call.  engram_create allocates one small
 *     device status block (freed by engram_destroy).
 *   - Every call is asynchronous on the given stream and launches nothing
 *     when it returns an error.  Host-side checks (null pointers, sizes,
 *     16-byte alignment) return synchronously.
 *   - Device-side data errors (an id outside [0, V), a canonical id outside
 *     [0, V'), a gather index >= M, a pipeline wait that ran out) never trap:
 *     the kernel records a bit in the context's device status word and keeps
 *     going with zero rows for the affected position.  engram_device_status
 *     reads and clears that word.
 *   - Matrices are row-major.  A "row" is one computed token position; rows
 *     are ordered sequence-major: row = b * L + (t - t_begin), L = T - t_begin.
 *   - One context per stream at a time (the status word is shared).
 */
#ifndef ENGRAM_H_
#define ENGRAM_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define ENGRAM_API __attribute__((visibility("default")))
#else
#define ENGRAM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum engram_status {
    ENGRAM_OK = 0,
    ENGRAM_E_INVAL = 1,        /* bad argument: null pointer, size, alignment, non-prime M */
    ENGRAM_E_CUDA = 2,         /* a CUDA runtime call failed */
    ENGRAM_E_NOMEM = 3,        /* workspace too small, or allocation in engram_create failed */
    ENGRAM_E_UNSUPPORTED = 4,  /* valid but not implemented (e.g. device is not sm_100) */
    ENGRAM_E_TIMEOUT = 5,      /* a bounded device wait ran out (device status bit) */
    ENGRAM_E_HOST = 6,         /* host-tier worker failure */
    ENGRAM_E_DEVICE = 7        /* device status word reports a data error */
} engram_status;

typedef enum engram_dtype {
    ENGRAM_F32 = 0,   /* tables, e, W, h, v, Y in fp32; projections on CUDA cores */
    ENGRAM_BF16 = 1,  /* tables, e, W, h, v, Y in bf16; projections on tcgen05 tensor cores */
    ENGRAM_FP8 = 2    /* tables, e, W_K, W_V in FP8 E4M3 (1 byte: sign, 4 exponent bits with bias 7, 3
                         mantissa bits; no infinities); h and Y in bf16; the projections as FP8 tcgen05
                         GEMMs (kind::f8f6f4) with fp32 accumulation, dequantised per output channel by
                         the k_scale / v_scale arguments of engram_forward_multibranch.  Needs d and J*D
                         multiples of 128 and conv width 4 (the fused path); only the forward entry
                         points take it ("DeepSeek AI II" digest, section "DeepSeek Engram": the
                         multi-branch projections fuse into one dense FP8 GEMM) */
} engram_dtype;

/* device status word bits (engram_device_status) */
#define ENGRAM_ERR_TOKEN   0x1u   /* raw id outside [0, V) */
#define ENGRAM_ERR_CANON   0x2u   /* canonical id outside [0, V') */
#define ENGRAM_ERR_INDEX   0x4u   /* gather index >= M (other than the invalid marker) */
#define ENGRAM_ERR_TIMEOUT 0x8u   /* a bounded device wait ran out */

#define ENGRAM_INVALID_INDEX 0xFFFFFFFFu  /* index of an n-gram that holds an invalid id */
#define ENGRAM_MAX_TABLES 32
#define ENGRAM_PART_GROUP 128             /* channels per gate-partial group */

typedef struct engram_config {
    int32_t n_orders;                        /* number of n-gram orders, 1..4 */
    int32_t orders[4];                       /* the orders, ascending, each in 1..4 (pages: {2,3}) */
    int32_t heads;                           /* K hash heads per order; J = n_orders*heads <= 32 */
    uint32_t rows[ENGRAM_MAX_TABLES];        /* M_j for table j = o*K + k; each prime, < 2^31 */
    uint64_t mult[ENGRAM_MAX_TABLES][4];     /* a_{n,k,j}: multiplier of s_j for table j (j < n) */
    int32_t row_dim;                         /* D, elements per table row */
    int32_t hidden;                          /* d, hidden width (query, k, v, Y) */
    int32_t conv_width;                      /* w, causal conv taps, 1..8 */
    int32_t vocab;                           /* V, raw vocabulary */
    int32_t canon_vocab;                     /* V', canonical vocabulary; PAD id = V' */
    engram_dtype dtype;
    float eps;                               /* RMSNorm epsilon (1e-6) */
} engram_config;

typedef struct engram_ctx engram_ctx;

/* Validate cfg (orders ascending in 1..4, J <= 32, every M prime and < 2^31,
 * D*elem a multiple of 16 bytes, d a multiple of 8, V' < 2^31 - 1; for
 * ENGRAM_FP8 also d and J*D multiples of 128 and conv width 4) and bind a
 * context to the CURRENT device.  Allocates a 256-byte device status block.
 * Returns ENGRAM_E_INVAL for a bad config, ENGRAM_E_CUDA/NOMEM on failure. */
ENGRAM_API engram_status engram_create(const engram_config* cfg, engram_ctx** out);
ENGRAM_API void engram_destroy(engram_ctx* ctx);
ENGRAM_API const char* engram_strerror(engram_status s);
/* Text of the last host-side failure on the calling thread (argument check
 * or CUDA error with its call site); empty when none.  Owned by the library. */
ENGRAM_API const char* engram_last_error(void);

/* Bytes of scratch that engram_forward / engram_gate_conv need for B
 * sequences of L computed rows (n_tok = B*L): indices [n_tok][J] u32,
 * e [n_tok][J*D], gate partials [n_tok][G][4] f32 with G = ceil(d / 128)
 * (d / 64 for the decode passes of one-position bf16 calls), the gate values
 * [n_tok] f32, max(ceil(n_tok/128), 8) int32 counters, the next conv history
 * [B][w-1][d] f32, for other fused calls with L <= 8 a second history buffer
 * (the history in the sequence-minor layout [w-1][d][B] that the value pass
 * reads coalesced across sequences) and, where the gate and conv are not
 * fused into the projection (see engram_gate_conv) or for the decode
 * kernels, v [n_tok][d] f32; each part 256-byte aligned.  0 for a null
 * context. */
ENGRAM_API size_t engram_workspace_bytes(const engram_ctx* ctx, int32_t B, int32_t L);

/* Per-kernel timing for benchmarks.  While enabled, every entry point records
 * a pair of CUDA events (created here, on the context's device) around each
 * kernel it launches on the caller's stream; engram_profile_read waits for
 * the events of the most recent call and writes up to `max` durations in
 * milliseconds and kernel names (library-owned strings) in launch order,
 * returning how many; a duration that could not be measured reads -1.
 * Under stream capture the events become record nodes of the graph, so
 * after a replay engram_profile_read returns that replay's durations.  Not
 * thread-safe; disable to free the events. */
ENGRAM_API engram_status engram_profile_enable(engram_ctx* ctx, int32_t enable);
ENGRAM_API int32_t engram_profile_read(engram_ctx* ctx, float* ms, const char** names, int32_t max);

/* Test hook for the bounded device waits (failure detection without a
 * fault): the next fused key pass (tcgen05 path) of this context announces
 * the bytes of its first operand stage in CTA 0 but never loads them, so the
 * MMA warp's wait on that stage runs out after about 2 s.  The kernel then
 * sets ENGRAM_ERR_TIMEOUT, raises its abort flag, drains the copies and MMAs
 * it issued (bounded again), frees its tensor memory and returns; the
 * following kernels run to completion.  engram_device_status then reports
 * ENGRAM_E_TIMEOUT, and the context and its workspace stay usable for the
 * next call.  The outputs of the stalled call are undefined.  One shot. */
ENGRAM_API engram_status engram_debug_stall_next(engram_ctx* ctx);

/* Synchronise `stream`, return the device status word in *flags (nullable)
 * and clear it.  ENGRAM_OK when it was zero, ENGRAM_E_TIMEOUT when the
 * timeout bit was set, else ENGRAM_E_DEVICE. */
ENGRAM_API engram_status engram_device_status(engram_ctx* ctx, cudaStream_t stream, uint32_t* flags);

/* Tokenizer compression ("DeepSeek AI II" digest, section "DeepSeek Engram":
 * the surjection P: V -> V').  canon[i] = P[tok[i]] for i < n; P is [V] int32.
 * An id outside [0, V) gives canon = -1 and sets ENGRAM_ERR_TOKEN. */
ENGRAM_API engram_status engram_remap(engram_ctx* ctx, const int32_t* tok, int64_t n, const int32_t* P,
                           int32_t* canon, cudaStream_t stream);

/* Suffix n-grams and multi-head hashing (same section: g_{t,n}, phi_{n,k},
 * prime table sizes; Synced repost, "hashed N-gram sparse retrieval": K
 * independent heads per order).  ids is [B] sequences of `stride` int32
 * (positions 0..T-1 valid); rows t in [t_begin, T) are computed and the
 * n-gram windows reach back into [0, t_begin).  When P is non-null, ids are
 * raw token ids remapped on the fly; otherwise they are canonical ids.
 * idx is [B*(T-t_begin)][J] uint32; an n-gram holding an invalid id gives
 * ENGRAM_INVALID_INDEX for its order's K tables. */
ENGRAM_API engram_status engram_hash(engram_ctx* ctx, const int32_t* ids, const int32_t* P, int32_t B, int32_t T,
                          int64_t stride, int32_t t_begin, uint32_t* idx, cudaStream_t stream);

/* Gather and concatenation (same section: e_t = concat of E_{n,k}[phi]).
 * tables holds the J tables back to back (table j starts at row
 * sum_{i<j} M_i; each row D elements of the context dtype); e_cat is
 * [n_tok][J*D].  An index >= M_j writes a zero row (ENGRAM_ERR_INDEX unless
 * it is ENGRAM_INVALID_INDEX).  tables and e_cat 16-byte aligned. */
ENGRAM_API engram_status engram_gather(engram_ctx* ctx, const uint32_t* idx, int64_t n_tok, const void* tables,
                            void* e_cat, cudaStream_t stream);

/* Key/value projections with the gate's partial sums (same section: k = W_K e,
 * v = W_V e; RMSNorm on query and key).  Wk and Wv are [d][J*D] (nn.Linear
 * layout), h is [n_tok][d], gq/gk are [d] fp32 RMSNorm gains (null = ones).
 * Writes v [n_tok][d] in fp32 and part [n_tok][G][4] fp32, G = ceil(d/128):
 * for channel group g, part = (sum g_q g_k h k, sum k^2, sum h^2, 0) over the
 * group's channels.  k itself is never stored. */
ENGRAM_API engram_status engram_project(engram_ctx* ctx, const void* e_cat, int64_t n_tok, const void* h,
                             const void* Wk, const void* Wv, const float* gq, const float* gk,
                             float* v, float* part, cudaStream_t stream);

/* Gate and causal depthwise convolution (same section: alpha_t in (0,1),
 * v~ = alpha v, short-kernel per-channel causal conv; residual H <- H + Y).
 * v (fp32) and part as written by engram_project for B sequences of L rows
 * each; conv_w is [d][w] fp32 (tap j multiplies v~_{t-j}); conv_state
 * (nullable) is [B][w-1][d] fp32 holding v~ of the w-1 positions before the
 * first row (row w-2 most recent): read as history and overwritten with the
 * last w-1 v~ rows of the extended sequence (in place is safe).  Null: zero
 * history.  h is read only when add_residual != 0.  y is [B*L][d] (context
 * dtype); alpha_out (nullable) [B*L] fp32. */
ENGRAM_API engram_status engram_conv(engram_ctx* ctx, const float* v, const float* part, const void* h,
                          const float* conv_w, int32_t B, int32_t L, float* conv_state, void* y,
                          float* alpha_out, int32_t add_residual, cudaStream_t stream);

/* Projections, gate and conv from e ("DeepSeek AI II" digest, section
 * "DeepSeek Engram": k = W_K e and v = W_V e, RMSNorm on the query h and the
 * key, a scalar gate alpha in (0,1), v~ = alpha v, a short-kernel per-channel
 * causal convolution, the residual H <- H + Y; Synced repost, section
 * "context-aware gating").  On bf16 tensor-core shapes (d a
 * multiple of 128, J*D a multiple of 64) with conv width 4, two tcgen05 GEMM
 * passes, the first producing the gate partials from k, the second v with
 * the gate, the conv and the residual applied in its epilogue (v is never
 * stored); otherwise engram_project followed by engram_conv.  Scratch in `workspace`
 * (engram_workspace_bytes(ctx, B, L); the index and e parts are unused). */
ENGRAM_API engram_status engram_gate_conv(engram_ctx* ctx, const void* e_cat, const void* h, const void* Wk,
                               const void* Wv, const float* gq, const float* gk, const float* conv_w,
                               int32_t B, int32_t L, float* conv_state, void* y, float* alpha_out,
                               int32_t add_residual, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/* The whole forward ("DeepSeek AI II" digest, section "DeepSeek Engram": the
 * module takes the token ids and the hidden states of a layer and returns Y,
 * through retrieval (tokenizer compression, suffix n-grams, multi-head
 * hashing into prime-sized tables, concatenation) and fusion (the gate and
 * the causal convolution)): what engram_hash (with remap), engram_gather and
 * engram_gate_conv compute, with the first two fused into one retrieval
 * kernel; intermediates in `workspace` (engram_workspace_bytes(ctx, B,
 * T-t_begin) bytes, 256-byte aligned).  tok is [B] rows of `tok_stride` raw
 * ids; prefill uses t_begin = 0, a decode step for the last position uses
 * t_begin = T-1 with conv_state.  On the tensor-core path the two GEMM passes
 * are launched as programmatic dependents of the kernel before each (they
 * overlap its last CTAs and wait for its results on the device); seen from
 * the stream, the call is ordered like any other work on `stream`.  A decode
 * step (T - t_begin = 1) for at most 256 sequences of a bf16 context runs
 * the decode passes: K split over clusters of four CTAs, and conv_state
 * rewritten in place by the value pass (same result as above).  The call
 * only enqueues work on `stream`, so it can be captured into a CUDA graph;
 * a replay recomputes from the pointers given at capture, whose contents
 * may change between replays. */
ENGRAM_API engram_status engram_forward(engram_ctx* ctx, const int32_t* tok, int32_t B, int32_t T,
                             int64_t tok_stride, int32_t t_begin, const int32_t* P,
                             const void* tables, const void* h, const void* Wk, const void* Wv,
                             const float* gq, const float* gk, const float* conv_w,
                             float* conv_state, void* y, float* alpha_out, int32_t add_residual,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------ multi-branch
 *
 * The pages ("DeepSeek AI II" digest, section "DeepSeek Engram", the
 * multi-branch paragraphs; the Synced repost, "context-aware gating") use a
 * backbone whose residual stream has M parallel branches.  All branches share
 * the sparse tables and the value projection W_V; branch m has its own key
 * projection W_K^(m) and hidden state h^(m), hence its own gate
 *   alpha^(m)_t = sigmoid(<RMSNorm(h^(m)_t), RMSNorm(W_K^(m) e_t)> / sqrt(d)),
 * applied to the shared value: u^(m)_t = alpha^(m)_t * (W_V e_t).  The
 * projections fuse into dense GEMMs over [W_V; W_K^(1..M)]: here one key pass
 * over the stacked W_K^(1..M) (N = M*d) yields the M gates per token, and one
 * value pass computes v once and, in its epilogue, applies each branch's
 * gate, the causal depthwise conv, SiLU and the residual, writing M outputs.
 * Readings (the pages stop at u^(m)): each branch's u^(m) goes through the
 * same conv as the single-branch module (shared conv_w, a history per
 * branch), and the RMSNorm gains are per branch.
 *   h          [M][B*L][d] (model dtype), branch-major;
 *   Wk         [M][d][J*D]: W_K^(m) stacked;       Wv [d][J*D], shared;
 *   gq, gk     [M][d] fp32 or null (ones);           conv_w [d][w], shared;
 *   conv_state [M][B][w-1][d] fp32 or null;          y [M][B*L][d];
 *   alpha_out  [M][B*L] fp32 or null;
 *   k_scale    [M][d] fp32, v_scale [d] fp32 (16-byte aligned): with
 *              ENGRAM_FP8, the per output channel dequantisation of the GEMM
 *              accumulators, k^(m)_c = k_scale[m][c] * (W_K^(m) e)_c and
 *              v_c = v_scale[c] * (W_V e)_c (the tables' scale times the weight
 *              row's scale); required there, and null for the other dtypes
 *              (ENGRAM_E_INVAL otherwise).
 * M in 1..ENGRAM_MAX_BRANCHES.  With ENGRAM_FP8 tables, e, W_K and W_V are
 * E4M3 bytes and the fused GEMM over [W_V; W_K^(1..M)] runs as FP8 MMAs, as
 * the pages describe.  Runs on the fused tensor-core path only
 * (bf16, conv width 4, d a multiple of 128, J*D a multiple of 64);
 * otherwise ENGRAM_E_UNSUPPORTED.  Scratch: engram_multibranch_workspace_bytes
 * (M = 1 gives engram_workspace_bytes). */
#define ENGRAM_MAX_BRANCHES 4
ENGRAM_API size_t engram_multibranch_workspace_bytes(const engram_ctx* ctx, int32_t M, int32_t B, int32_t L);
ENGRAM_API engram_status engram_forward_multibranch(engram_ctx* ctx, int32_t M, const int32_t* tok, int32_t B,
                                                    int32_t T, int64_t tok_stride, int32_t t_begin, const int32_t* P,
                                                    const void* tables, const void* h, const void* Wk, const void* Wv,
                                                    const float* gq, const float* gk, const float* k_scale,
                                                    const float* v_scale, const float* conv_w, float* conv_state,
                                                    void* y, float* alpha_out, int32_t add_residual,
                                                    void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------ sharded tables
 *
 * Tables split across GPUs.  The pages ("DeepSeek AI II" digest, section
 * "DeepSeek Engram", the training paragraph; the Synced repost, section
 * "System efficiency: decoupling compute and storage") shard the embedding
 * tables over the available GPUs so that capacity grows with their number,
 * and bring the accessed rows to each GPU in the forward (an all-to-all).
 * Here the rows of all J tables, numbered globally (table j's row r is global
 * row sum_{i<j} M_i + r), are split into n_shards contiguous ranges of
 * ceil(R / n_shards) rows (R = sum of M_j; the last range may be shorter or
 * empty); engram_shard_range gives the range of shard g.  Shard g stores its
 * rows back to back, D elements of the model dtype per row.  The forward's
 * retrieval kernel reads every row directly from the shard that owns it:
 * shard_tables[g] is a device pointer valid on THIS GPU, to this GPU's own
 * memory or to another GPU's memory mapped here (engram_ipc_open, or peer
 * access).  Remote rows cross NVLink once, with plain loads, and land in
 * this GPU's e_cat before the projections read them: the all-to-all of
 * indices and rows is one-sided reads inside the retrieval. */
ENGRAM_API engram_status engram_shard_range(const engram_ctx* ctx, int32_t n_shards, int32_t shard,
                                            int64_t* first_row, int64_t* n_rows);
/* engram_forward with the tables given as n_shards (1..16) shards instead of
 * one array: shard_tables is a HOST array of n_shards device pointers (16-byte
 * aligned; null only for an empty shard).  Every other argument and the
 * result are engram_forward's; an index whose row no shard covers gathers a
 * zero row and sets ENGRAM_ERR_INDEX.  The shards must stay mapped until the
 * call completes on `stream`; nothing is exchanged between GPUs except these
 * reads, so the caller's only ordering duty is that the shards hold their
 * rows before the call (they are read-only here). */
ENGRAM_API engram_status engram_forward_sharded(engram_ctx* ctx, const int32_t* tok, int32_t B, int32_t T,
                                                int64_t tok_stride, int32_t t_begin, const int32_t* P,
                                                const void* const* shard_tables, int32_t n_shards, const void* h,
                                                const void* Wk, const void* Wv, const float* gq, const float* gk,
                                                const float* conv_w, float* conv_state, void* y, float* alpha_out,
                                                int32_t add_residual, void* workspace, size_t workspace_bytes,
                                                cudaStream_t stream);
/* Cross-process mapping of a shard (plumbing for one process per GPU).
 * engram_ipc_export: the cudaMalloc allocation that contains the device
 * pointer `ptr`, as a 64-byte CUDA IPC handle (handle_out) plus the offset of
 * `ptr` in it.  engram_ipc_open (in another process, any GPU with peer
 * access to the owner): maps that allocation into the calling process on the
 * current device and returns the pointer at the offset (*ptr_out) and the
 * mapping's base (*base_out, for engram_ipc_close).  Memory from a
 * virtual-memory (cuMemMap) allocator cannot be exported: ENGRAM_E_CUDA. */
#define ENGRAM_IPC_HANDLE_BYTES 64
ENGRAM_API engram_status engram_ipc_export(const void* ptr, void* handle_out, uint64_t* offset_out);
ENGRAM_API engram_status engram_ipc_open(const void* handle, uint64_t offset, void** ptr_out, void** base_out);
ENGRAM_API engram_status engram_ipc_close(void* base);

/* ------------------------------------------------------------ table backward
 *
 * The tables are trained with the model ("DeepSeek AI II" digest, section
 * "DeepSeek Engram", the training paragraph: the backward sends each
 * accessed row's gradient to the shard that holds it).  e_t concatenates
 * the rows E_j[idx_j(t)], so the gradient of table j's row r is the sum of
 * slice j of dL/de_t over the lookups (t, j) with idx_j(t) = r; rows no
 * lookup touched have zero gradient and are not listed.
 *
 * engram_table_grad: idx [n_tok][J] (engram_hash's output), d_e
 * [n_tok][J*D] in the context dtype (16-byte aligned).  Writes, for the U
 * distinct rows the valid lookups touched: rows_out[u] = the global row
 * (sum_{i<j} M_i + r) and grad_out[u][D] (fp32, 16-byte aligned) its
 * summed gradient, u < U; *n_unique (DEVICE uint64) = U.  Capacity: n_tok*J
 * rows in rows_out and grad_out.  Invalid indices (an n-gram with an
 * invalid id) contribute nothing.  Each row's sum runs in fp32 in an order
 * fixed by its lookups alone: increasing lookup order (t * J + j) for a row
 * looked up at most 32 times; for a longer row, S = 256 / (D*elem/16)
 * running sums, the p-th over the row's lookups p, p + S, p + 2S, ... in
 * increasing order, then added in order of p.  So the (row, gradient) pairs
 * are the same on every run; which u a row lands at depends on the device's
 * atomics.
 * n_tok * J <= 2^24.  Scratch: engram_table_grad_workspace_bytes(ctx, n_tok)
 * bytes, 256-byte aligned.
 *
 * engram_table_sgd: tables[rows[u]] -= lr * grad[u] for u < min(*n_unique,
 * max_rows), in fp32 arithmetic with one rounding to the tables' dtype;
 * tables as in engram_gather (16-byte aligned, as is grad).  A row outside
 * the tables sets ENGRAM_ERR_INDEX and is skipped. */
ENGRAM_API size_t engram_table_grad_workspace_bytes(const engram_ctx* ctx, int64_t n_tok);
ENGRAM_API engram_status engram_table_grad(engram_ctx* ctx, const uint32_t* idx, int64_t n_tok, const void* d_e,
                                           uint64_t* rows_out, float* grad_out, uint64_t* n_unique, void* workspace,
                                           size_t workspace_bytes, cudaStream_t stream);
ENGRAM_API engram_status engram_table_sgd(engram_ctx* ctx, const uint64_t* rows, const float* grad,
                                          const uint64_t* n_unique, int64_t max_rows, void* tables, float lr,
                                          cudaStream_t stream);

/* ------------------------------------------------------------ table backward across shards
 *
 * With the tables sharded (shard g holds the global rows engram_shard_range
 * gives it, one shard per rank), the backward sends every accessed row's
 * gradient to the shard that stores it ("DeepSeek AI II" digest, section
 * "DeepSeek Engram", the training paragraph; the Synced repost, section
 * "System efficiency: decoupling compute and storage": the rows are gathered
 * to each GPU by an all-to-all in the forward and their gradients are
 * scattered back to the owners in the backward).  Three steps per rank:
 *
 * engram_grad_route: this rank's (row, gradient) pairs (engram_table_grad's
 * rows_out, grad_out and DEVICE *n_pairs; pairs beyond max_rows are ignored)
 * split by owner.  Writes send_counts[g] (DEVICE int64, n_shards entries) =
 * the number of pairs for shard g, and the pairs themselves into send_rows
 * (uint64 global rows) and send_grad ([.][D] fp32, 16-byte aligned), shard
 * 0's segment first, then shard 1's, and so on (capacity max_rows each).
 * Within a segment the order is whatever the device's atomics give.  A row
 * beyond the tables sets ENGRAM_ERR_INDEX and is not sent.  Scratch:
 * engram_grad_route_workspace_bytes(ctx) bytes, 256-byte aligned.
 *
 * The exchange itself is the caller's: an all-to-all (NCCL's, through
 * torch.distributed.all_to_all_single) of send_counts, then of the segments,
 * which leaves on every rank the pairs for its shard from rank 0, then rank
 * 1, and so on.
 *
 * engram_grad_combine: the pairs received by shard `shard` of n_shards
 * (pair_rows uint64 [n_pairs], pair_grad [n_pairs][D] fp32, 16-byte aligned;
 * n_pairs <= 2^24 is a HOST count).  Writes the distinct rows into rows_out
 * (global rows), their summed gradients into grad_out ([.][D] fp32, 16-byte
 * aligned; capacity n_pairs each) and their number into DEVICE *n_unique.
 * Each row's sum runs in increasing pair order, i.e. in rank order when the
 * pairs arrive in rank order, in fp32; since every rank sends a row at most
 * once, the result does not depend on the order within a rank's segment.
 * (A row received more than 32 times, which at most 16 ranks sending it once
 * each never produce, is summed in engram_table_grad's order for long
 * rows.)  A
 * pair whose row the shard does not hold sets ENGRAM_ERR_INDEX and is
 * dropped.  Scratch: engram_grad_combine_workspace_bytes(ctx, n_pairs) bytes,
 * 256-byte aligned.
 *
 * engram_shard_sgd: engram_table_sgd on one shard: shard_table holds the
 * shard's rows back to back ([n_rows][D], the model dtype), rows are global;
 * shard_table[row - first_row] -= lr * grad for u < min(*n_unique,
 * max_rows).  A row outside the shard sets ENGRAM_ERR_INDEX and is skipped. */
ENGRAM_API size_t engram_grad_route_workspace_bytes(const engram_ctx* ctx);
ENGRAM_API engram_status engram_grad_route(engram_ctx* ctx, int32_t n_shards, const uint64_t* rows,
                                           const float* grad, const uint64_t* n_pairs, int64_t max_rows,
                                           uint64_t* send_rows, float* send_grad, int64_t* send_counts,
                                           void* workspace, size_t workspace_bytes, cudaStream_t stream);
ENGRAM_API size_t engram_grad_combine_workspace_bytes(const engram_ctx* ctx, int64_t n_pairs);
ENGRAM_API engram_status engram_grad_combine(engram_ctx* ctx, int32_t n_shards, int32_t shard,
                                             const uint64_t* pair_rows, const float* pair_grad, int64_t n_pairs,
                                             uint64_t* rows_out, float* grad_out, uint64_t* n_unique,
                                             void* workspace, size_t workspace_bytes, cudaStream_t stream);
ENGRAM_API engram_status engram_shard_sgd(engram_ctx* ctx, int32_t n_shards, int32_t shard, const uint64_t* rows,
                                          const float* grad, const uint64_t* n_unique, int64_t max_rows,
                                          void* shard_table, float lr, cudaStream_t stream);

/* engram_forward for callers that cannot allocate device memory (an engine
 * callback where allocation is forbidden, a process whose device memory is
 * all owned by another allocator, a loop that cannot afford cudaMalloc's
 * implicit synchronisation).  The pages have no counterpart: this is an
 * interface of this library only.  Same arguments as engram_forward without
 * the workspace: the scratch lives in a static device array of
 * ENGRAM_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until
 * the process exits.  Every call whose stream is not capturing looks up that
 * array's device address on the current device (cudaGetSymbolAddress); a
 * call on a capturing stream reuses the last address looked up, so the first
 * call on a device must come before any stream capture.  The context's device
 * must be current (ENGRAM_E_INVAL otherwise, before anything is looked up).  Calls needing more than the array (engram_workspace_bytes(ctx,
 * B, T - t_begin)) return ENGRAM_E_NOMEM with an explanation in
 * engram_last_error and launch nothing.  No cudaMalloc or cudaFree is called.
 * All calls share the one array, which keeps the last call's contents (the
 * forward clears the counters it needs zeroed and writes every other
 * scratch byte before reading it): calls that may
 * overlap on the GPU (other streams, other host threads) race on it and must
 * be serialised by the caller. */
#define ENGRAM_NOALLOC_SCRATCH_BYTES (32u << 20)
ENGRAM_API engram_status engram_forward_noalloc(engram_ctx* ctx, const int32_t* tok, int32_t B, int32_t T,
                                     int64_t tok_stride, int32_t t_begin, const int32_t* P,
                                     const void* tables, const void* h, const void* Wk, const void* Wv,
                                     const float* gq, const float* gk, const float* conv_w,
                                     float* conv_state, void* y, float* alpha_out, int32_t add_residual,
                                     cudaStream_t stream);

/* The whole forward from and to HOST memory: the end-to-end call of a caller
 * whose hidden states live on the host.  The pages (the Synced repost,
 * section "System efficiency: decoupling compute and storage") describe the
 * retrieval as depending only on token ids, which is what lets transfers
 * overlap compute; this entry point applies that to the per-token tensors.
 *   tok_host  int32 [B][tok_stride] raw ids, host memory;
 *   h_host    [B][L][d] hidden states (model dtype), host memory;
 *   y_host    [B][L][d] output (model dtype), host memory, L = T - t_begin;
 *   P, tables, Wk, Wv, gq, gk, conv_w, conv_state: device memory, as in
 *             engram_forward (conv_state nullable: zero history).
 * The rows are processed in chunks of `chunk_rows` positions of every
 * sequence.  With chunk_rows = 0, a batch of at least four 16 MiB chunks of
 * h runs 16 MiB chunks, entered and left through chunks of 2, 4 and 8 MiB
 * (the first compute starts early, the last copy out is short); a shorter
 * batch runs chunks of about 4 MiB.  While chunk i computes on
 * `stream`, the h of chunk i+1 is copied in on one of the context's copy
 * streams and the Y of chunk i-1 is copied out on the other
 * (cudaMemcpy2DAsync).  The conv history passes from chunk to chunk through
 * conv_state, or through a zeroed copy in the workspace when conv_state is
 * null, so the result equals engram_forward's.  Only the id window each
 * sequence needs (from t_begin - (max order - 1)) is copied in.
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister); with
 * pageable memory the copies are correct but do not overlap.
 * Device scratch: `workspace`, engram_host_workspace_bytes(ctx, B, T,
 * t_begin, chunk_rows) bytes, 256-byte aligned.
 * Returns once everything is enqueued; y_host (and conv_state) are complete
 * when `stream` completes.  Host buffers must stay valid until then.  Errors
 * are as engram_forward's, checked before anything is enqueued. */
ENGRAM_API size_t engram_host_workspace_bytes(const engram_ctx* ctx, int32_t B, int32_t T, int32_t t_begin,
                                              int32_t chunk_rows);
ENGRAM_API engram_status engram_forward_host(engram_ctx* ctx, const int32_t* tok_host, int32_t B, int32_t T,
                                             int64_t tok_stride, int32_t t_begin, const int32_t* P,
                                             const void* tables, const void* h_host, const void* Wk,
                                             const void* Wv, const float* gq, const float* gk,
                                             const float* conv_w, float* conv_state, void* y_host,
                                             int32_t add_residual, int32_t chunk_rows, void* workspace,
                                             size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------- host tier
 *
 * Tables too large for HBM stay in host memory; each batch fetches over PCIe
 * only the rows its n-grams activate.  The pages (the "DeepSeek AI II"
 * digest, section "DeepSeek Engram", system efficiency; the Synced repost,
 * section "System efficiency: decoupling compute and storage"; the QbitAI
 * repost on the 100B-parameter table held in host memory) base this on the
 * indices depending only on token ids: they are computed ahead of the layer,
 * the distinct rows are copied while the preceding layers run, and the
 * Zipf-skewed n-gram distribution keeps the distinct rows far fewer than the
 * lookups.  A batch is three calls, in this order, with dedupe and
 * gather_staged on the same stream:
 *   engram_hash(...)                     indices [n_tok][J] on the device
 *   engram_host_dedupe(tier, idx, n_tok, s)
 *   ... other work on s (the preceding layers) ...
 *   engram_host_fetch(tier, side, &n_unique)     blocks the calling thread
 *                                                 while the rows are packed
 *   engram_gather_staged(tier, n_tok, e_cat, s)  then engram_gate_conv.
 */
typedef struct engram_host_tier engram_host_tier;

/* host_tables: [J][M_j][D] rows (model dtype) in host memory, back to back
 * in table order; pageable memory is fine (it is only read by the packing
 * threads).  max_lookups: the largest n_tok * J of any batch.  The tier
 * allocates, once: a device hash set of 2^ceil(log2(2 max_lookups)) keys,
 * the distinct-row list, the slot map and the staged rows on the device
 * (max_lookups * D * elem bytes), and pinned host buffers for the list and
 * the staging; it starts n_threads packing threads.  Returns
 * ENGRAM_E_NOMEM when an allocation fails, ENGRAM_E_HOST when the threads
 * cannot start.  The host tables must outlive the tier. */
ENGRAM_API engram_status engram_host_tier_create(engram_ctx* ctx, const void* host_tables, int64_t max_lookups,
                                                 int32_t n_threads, engram_host_tier** out);
/* Waits (bounded) for copies in flight into the tier's pinned buffers, stops
 * the threads and frees everything the tier allocated. */
ENGRAM_API void engram_host_tier_destroy(engram_host_tier* tier);

/* Enqueue on `stream`: clear the set; one kernel inserts every valid lookup's
 * global row (row_off[j] + idx) and gives each distinct row the next slot;
 * a second kernel writes each lookup's slot (invalid indices keep
 * ENGRAM_INVALID_INDEX and later gather a zero row); the count and the
 * distinct-row list are copied to pinned host memory.  Slot order depends
 * on the atomics' timing; the gathered rows do not.  A set that overflows
 * (impossible at its load factor of 1/2) sets ENGRAM_ERR_INDEX. */
ENGRAM_API engram_status engram_host_dedupe(engram_host_tier* tier, const uint32_t* idx, int64_t n_tok,
                                            cudaStream_t stream);
/* Host side: waits (bounded, 20 s) for the distinct-row list, then the
 * packing threads copy the rows from the host tables into pinned staging in
 * chunks of 4096 rows; this thread hands the finished chunks, in order and
 * at least 4 MB at a time (but the last), to cudaMemcpyAsync calls on
 * `side_stream`.  Returns once every copy is
 * enqueued, with the number of distinct rows in *n_unique (nullable).
 * ENGRAM_E_TIMEOUT / ENGRAM_E_HOST when a wait or a packing thread runs out
 * of time. */
ENGRAM_API engram_status engram_host_fetch(engram_host_tier* tier, cudaStream_t side_stream, int64_t* n_unique);
/* Enqueue on `stream`: wait for the fetched rows, then gather
 * e_cat [n_tok][J*D] (device, 16-byte aligned) from the staged rows through
 * the slot map: the same kernel and layout as engram_gather. */
ENGRAM_API engram_status engram_gather_staged(engram_host_tier* tier, int64_t n_tok, void* e_cat,
                                              cudaStream_t stream);
/* Mapped fetch: registers the host tables as mapped page-locked memory
 * (cudaHostRegister, read-only; already registered memory must be mapped)
 * and switches the tier to fetching the distinct rows with a GPU kernel that
 * reads them straight from host memory over PCIe into the staged rows.  No
 * packing thread runs and the host never waits for the row list:
 * engram_host_fetch only enqueues, on side_stream, a wait for the dedupe and
 * the fetch kernel, and reports *n_unique = -1 (the count is in
 * engram_host_tier_stats / engram_host_cache_stats once the batch is done).
 * Pinning a large table takes time once.  Call before the first batch; the
 * tier unregisters what it registered when destroyed.  ENGRAM_E_CUDA when
 * the memory cannot be registered or mapped.  Measured on B200 with 256-byte
 * rows: about 12 GB/s, against about 26 GB/s for the packing threads and
 * copies (the GPU keeps too few PCIe reads in flight), so the copy path
 * stays the default; this mode frees the host's cores and memory bandwidth. */
ENGRAM_API engram_status engram_host_tier_map(engram_host_tier* tier);

/* Hot-row cache in HBM in front of the host tables.  The pages (the
 * "DeepSeek AI II" digest, section "DeepSeek Engram", last paragraph; the
 * Synced repost, section "System efficiency: decoupling compute and
 * storage", last paragraph) keep the frequently accessed n-gram rows in a
 * faster tier, since a few patterns take most accesses under the Zipf law.
 * capacity_rows rows of device memory (plus a hash set of 2^ceil(log2(2 C))
 * 12-byte entries) are allocated once, here; the tier's staged-row buffer
 * is re-allocated to hold the cache slots in front of the staged rows.
 * From the next batch on, engram_host_dedupe resolves every distinct row
 * against the cache: resident rows are gathered from HBM and not fetched.
 * engram_gather_staged then admits the rows this batch fetched and looked up
 * at least min_count times (2 keeps the one-off tail out) into free slots
 * until the cache is full; nothing is evicted (engram_host_cache_reset
 * empties it).  Which rows win the last free slots depends on the device's
 * atomics; the gathered e_cat never does.  Call before the first batch.
 * ENGRAM_E_NOMEM when the device memory is short. */
ENGRAM_API engram_status engram_host_cache_enable(engram_host_tier* tier, int64_t capacity_rows, int32_t min_count);
/* Enqueue on `stream`: empty the hot-row cache. */
ENGRAM_API engram_status engram_host_cache_reset(engram_host_tier* tier, cudaStream_t stream);
/* Figures of the last batch (valid once its fetch has returned). */
typedef struct {
    int64_t capacity;        /* cache slots */
    int64_t resident;        /* slots in use when the batch was deduplicated */
    int64_t lookups;         /* the batch's lookups (n_tok * J) */
    int64_t cached_lookups;  /* lookups served from the cache */
    int64_t cached_rows;     /* distinct rows served from the cache (not fetched) */
    int64_t fetched_rows;    /* distinct rows fetched over PCIe */
} engram_host_cache_stats_t;
ENGRAM_API engram_status engram_host_cache_stats(const engram_host_tier* tier, engram_host_cache_stats_t* out);

/* Test hook for the host-side failure paths (failure detection without a
 * GPU fault; every failure is made on the host).  `inject` arms one-shot
 * faults for the next fetch:
 *   ENGRAM_INJECT_LIST_WAIT     the wait for the distinct-row list is told the
 *                               list never arrives (the event query's answer
 *                               is replaced), so the fetch returns
 *                               ENGRAM_E_TIMEOUT after the wait limit;
 *   ENGRAM_INJECT_PACK_ABANDON  the packing thread that takes the last chunk
 *                               of the batch gives it up without packing or
 *                               marking it, so the fetch returns ENGRAM_E_HOST
 *                               after the wait limit; the copies of the
 *                               earlier chunks, already enqueued, are
 *                               recorded, and the next fetch waits for them.
 * wait_limit_s replaces the 20 s bound of every host-side wait of the tier
 * (list, previous copies, packed chunks) from now on.  After either failure
 * the tier stays usable: the next dedupe + fetch + gather_staged is correct;
 * engram_gather_staged refuses to run on the failed batch. */
#define ENGRAM_INJECT_LIST_WAIT 0x1u
#define ENGRAM_INJECT_PACK_ABANDON 0x2u
ENGRAM_API engram_status engram_host_tier_debug(engram_host_tier* tier, uint32_t inject, double wait_limit_s);

/* Figures of the last fetch. */
typedef struct {
    int64_t n_unique;   /* distinct rows fetched */
    int64_t n_copies;   /* cudaMemcpyAsync calls that carried them */
    double wait_ms;     /* host wait for the distinct-row list (and the previous batch's copies) */
    double pack_ms;     /* host: packing start to the last copy enqueued */
    double copy_ms;     /* device: first row copy enqueued to the last one done; -1 while in flight */
} engram_host_tier_stats_t;
ENGRAM_API engram_status engram_host_tier_stats(const engram_host_tier* tier, engram_host_tier_stats_t* out);
/* The packing step alone, on the host (no device involved): rows[i] of the
 * [total_rows][row_bytes] host tables into dst[i], split over n_threads
 * threads.  Every row number is checked (< total_rows) before any copy. */
ENGRAM_API engram_status engram_pack_rows(const void* host_tables, int64_t total_rows, size_t row_bytes,
                                          const uint64_t* rows, int64_t n, void* dst, int32_t n_threads);

#ifdef __cplusplus
}
#endif

#endif /* ENGRAM_H_ */
