// Engram forward oracle: plain, single-threaded, fp64 reference.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
// benchmark's CPU-baseline leg may load this library.  It shares no code,
// header, table or constant with the CUDA library; it follows the method as
// the pages state it, one step after the other, with no blocking or fusion.
//
// Sources (page title, section):
//   [P1] "Conditional Memory via Scalable Lookup: DeepSeek Engram" digest
//        (taking-lying-flat blog, DeepSeek AI II), section "DeepSeek Engram":
//        tokenizer compression P: V -> V', suffix n-gram g_{t,n}, K hash heads
//        per order into prime-sized tables E_{n,k}, concatenation into e_t,
//        k = W_K e_t and v = W_V e_t, RMSNorm on query h_t and key, scalar
//        gate alpha_t in (0,1), v~_t = alpha_t * v_t, short causal depthwise
//        convolution, residual H <- H + Y.
//   [P2] "DeepSeek open-sources the memory module" (Synced repost), section
//        "hashed N-gram sparse retrieval": vocabulary projection, K
//        independent heads per order.
//   [P5] QbitAI repost: table size is prime; all orders and heads are
//        concatenated into e_t.
//
// Readings where the pages are silent (each listed in the design notes):
//   * positions with fewer than n-1 predecessors pad with PAD = V';
//   * phi_{n,k}(g) = (XOR_j (s_j + 1) * a_{n,k,j} mod 2^64) mod M_{n,k},
//     s_j = x'_{t-j}, multipliers supplied by the caller;
//   * concatenation order: order ascending, then head ascending;
//   * alpha = sigmoid(<q^, k^> / sqrt(d)), q^ = g_q * h / rms(h),
//     k^ = g_k * k / rms(k), rms(x) = sqrt(mean(x^2) + eps);
//   * u_t = sum_{j<w} c_{.,j} v~_{t-j} (zero or caller-given history),
//     Y = v~ + SiLU(u) (+ h when the residual is requested);
//   * invalid ids: a raw id outside [0, V) (or a canonical id outside
//     [0, V')) makes every n-gram that contains it produce index 0xFFFFFFFF,
//     and an index >= M gathers a zero row.
#include <cmath>
#include <cstdint>
#include <cstring>

extern "C" {

// Step 1 [P1]: x'_t = P(x_t).  Returns the number of ids outside [0, V);
// those positions get canonical id -1.
int64_t orc_remap(const int32_t* tok, int64_t n, const int32_t* P, int32_t V, int32_t* canon) {
    int64_t bad = 0;
    for (int64_t i = 0; i < n; ++i) {
        int32_t x = tok[i];
        if (x < 0 || x >= V) {
            canon[i] = -1;
            ++bad;
        } else {
            canon[i] = P[x];
        }
    }
    return bad;
}

// Steps 2-3 [P1]: for each sequence b and position t in [t_begin, T), for
// each order n = orders[o] and head k, the suffix n-gram s_j = x'_{t-j}
// (j = 0..n-1, PAD = Vc before the sequence start) is hashed into table
// J-index o*K + k.  idx is [B*(T-t_begin)][J], rows b-major.
// Returns the number of n-grams that contained an invalid id.
int64_t orc_hash(const int32_t* canon, int32_t B, int32_t T, int64_t stride, int32_t t_begin,
                 int32_t Vc, int32_t n_orders, const int32_t* orders, int32_t K,
                 const uint64_t* mult /* [J][4] */, const uint32_t* M /* [J] */,
                 uint32_t* idx) {
    const int32_t J = n_orders * K;
    int64_t bad = 0;
    int64_t row = 0;
    for (int32_t b = 0; b < B; ++b) {
        for (int32_t t = t_begin; t < T; ++t, ++row) {
            for (int32_t o = 0; o < n_orders; ++o) {
                const int32_t n = orders[o];
                uint64_t s[4];
                bool invalid = false;
                for (int32_t j = 0; j < n; ++j) {
                    const int64_t tt = (int64_t)t - j;
                    if (tt < 0) {
                        s[j] = (uint64_t)Vc;  // PAD
                    } else {
                        const int32_t c = canon[(int64_t)b * stride + tt];
                        if (c < 0 || c >= Vc) invalid = true;
                        s[j] = (uint64_t)(uint32_t)c;
                    }
                }
                if (invalid) ++bad;
                for (int32_t k = 0; k < K; ++k) {
                    const int32_t jt = o * K + k;
                    uint32_t out;
                    if (invalid) {
                        out = 0xFFFFFFFFu;
                    } else {
                        uint64_t x = 0;
                        for (int32_t j = 0; j < n; ++j) x ^= (s[j] + 1u) * mult[jt * 4 + j];
                        out = (uint32_t)(x % (uint64_t)M[jt]);
                    }
                    idx[row * J + jt] = out;
                }
            }
        }
    }
    return bad;
}

// Step 4 [P1][P5]: e_t = concat_j E_j[idx_{t,j}].  The J tables are stored
// back to back (table j starts at row sum_{i<j} M_i) with row_bytes per row;
// e_cat is [n][J*row_bytes] bytes.  An index >= M_j yields a zero row.
void orc_gather(const uint32_t* idx, int64_t n, int32_t J, const uint32_t* M,
                const void* tables, int64_t row_bytes, void* e_cat) {
    const unsigned char* tb = (const unsigned char*)tables;
    unsigned char* out = (unsigned char*)e_cat;
    for (int64_t i = 0; i < n; ++i) {
        int64_t off = 0;
        for (int32_t j = 0; j < J; ++j) {
            unsigned char* dst = out + (i * J + j) * row_bytes;
            const uint32_t r = idx[i * J + j];
            if (r < M[j]) {
                std::memcpy(dst, tb + (off + (int64_t)r) * row_bytes, (size_t)row_bytes);
            } else {
                std::memset(dst, 0, (size_t)row_bytes);
            }
            off += M[j];
        }
    }
}

// Step 5 [P1]: out[i][c] = sum_q W[c][q] e[i][q]  (W stored [d][d_mem]).
void orc_project(const double* e, int64_t n, int32_t d_mem, const double* W, int32_t d, double* out) {
    for (int64_t i = 0; i < n; ++i) {
        for (int32_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int32_t q = 0; q < d_mem; ++q) acc += W[(int64_t)c * d_mem + q] * e[i * d_mem + q];
            out[i * d + c] = acc;
        }
    }
}

// Step 6 [P1]: alpha_i = sigmoid(<q^_i, k^_i> / sqrt(d)).
void orc_gate(const double* h, const double* k, int64_t n, int32_t d, const double* gq,
              const double* gk, double eps, double* alpha) {
    for (int64_t i = 0; i < n; ++i) {
        const double* hi = h + i * d;
        const double* ki = k + i * d;
        double sh = 0.0, sk = 0.0;
        for (int32_t c = 0; c < d; ++c) {
            sh += hi[c] * hi[c];
            sk += ki[c] * ki[c];
        }
        const double rh = std::sqrt(sh / d + eps);
        const double rk = std::sqrt(sk / d + eps);
        double dot = 0.0;
        for (int32_t c = 0; c < d; ++c) dot += (gq[c] * hi[c] / rh) * (gk[c] * ki[c] / rk);
        alpha[i] = 1.0 / (1.0 + std::exp(-dot / std::sqrt((double)d)));
    }
}

// Step 8 [P1]: causal depthwise convolution over one sequence segment of L
// rows, u[t][c] = sum_{j<w} cw[c][j] * vt[t-j][c]; rows before the segment
// come from hist ([w-1][d], row w-2 most recent) or are zero when hist is null.
void orc_conv(const double* vt, int32_t L, int32_t d, const double* cw, int32_t w,
              const double* hist, double* u) {
    for (int32_t t = 0; t < L; ++t) {
        for (int32_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int32_t j = 0; j < w; ++j) {
                const int32_t tt = t - j;
                double x;
                if (tt >= 0) {
                    x = vt[(int64_t)tt * d + c];
                } else {
                    x = hist ? hist[(int64_t)(w - 1 + tt) * d + c] : 0.0;
                }
                acc += cw[(int64_t)c * w + j] * x;
            }
            u[(int64_t)t * d + c] = acc;
        }
    }
}

double orc_silu(double x) { return x / (1.0 + std::exp(-x)); }

// Y = v~ + SiLU(u), plus h when add_residual is non-zero.
void orc_output(const double* vt, const double* u, const double* h, int64_t n, int32_t d,
                int32_t add_residual, double* y) {
    for (int64_t i = 0; i < n * d; ++i) {
        double r = vt[i] + orc_silu(u[i]);
        if (add_residual) r += h[i];
        y[i] = r;
    }
}

}  // extern "C"
