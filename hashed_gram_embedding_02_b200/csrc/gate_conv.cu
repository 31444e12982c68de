// Scalar gate and short causal depthwise convolution.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": the current hidden state
// h_t is the query, the retrieved memory feeds the key and value projections,
// RMSNorm is applied to query and key, and a scalar gate alpha_t in (0, 1)
// scales the value: v~_t = alpha_t v_t.  A short-kernel, per-channel causal
// convolution follows to widen the receptive field and add non-linearity.
// Readings: alpha_t = sigmoid(<q^, k^> / sqrt(d)) with q^ = g_q h / rms(h),
// k^ = g_k k / rms(k); u_t = sum_{j<w} c[j] v~_{t-j}; Y_t = v~_t + SiLU(u_t).
//
// HBM-bound: per row it reads v (d elements) and the G gate partials and
// writes Y (d elements).  A CTA owns TT consecutive rows of one sequence and
// all d channels: its warps first reduce the partials of its TT rows plus the
// w-1 rows before them into alpha (fixed lane order, deterministic), then each
// thread walks its 16-byte channel chunk down the rows, keeping the last w-1
// gated values in registers.  The CTA holding a sequence's first rows also
// reads the conv history and writes the new history (the last w-1 gated rows),
// so updating conv_state in place is race-free.
#include "common.cuh"

namespace engram {

namespace {

constexpr int kTT = 16;   // rows per CTA (>= kMaxConv - 1)

__device__ __forceinline__ float row_alpha(const float4* __restrict__ part, int64_t row, int G, float inv_d,
                                           float eps, float inv_sqrt_d, int lane) {
    float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
    for (int g = lane; g < G; g += 32) {
        const float4 p = part[row * G + g];
        s_qk += p.x;
        s_kk += p.y;
        s_hh += p.z;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        s_qk += __shfl_xor_sync(0xffffffffu, s_qk, off);
        s_kk += __shfl_xor_sync(0xffffffffu, s_kk, off);
        s_hh += __shfl_xor_sync(0xffffffffu, s_hh, off);
    }
    const float rh = sqrtf(s_hh * inv_d + eps);
    const float rk = sqrtf(s_kk * inv_d + eps);
    const float logit = s_qk / (rh * rk) * inv_sqrt_d;
    return 1.f / (1.f + expf(-logit));
}

__device__ __forceinline__ float silu(float x) { return x / (1.f + expf(-x)); }

template <typename T, int W>
__global__ void gate_conv_kernel(const T* __restrict__ v, const float4* __restrict__ part, const T* __restrict__ h,
                                 const float* __restrict__ conv_w, int32_t L, int32_t d, float eps,
                                 float* state, T* __restrict__ y, float* __restrict__ alpha_out,
                                 int32_t add_residual) {
    constexpr int VN = Vec<T>::N;
    constexpr int H = W - 1;                 // history rows
    __shared__ float s_alpha[kTT + kMaxConv];
    __shared__ float s_tail[kMaxConv];        // alpha of the sequence's last H rows

    const int b = blockIdx.y;
    const int t0 = blockIdx.x * kTT;
    const int t1 = min(t0 + kTT, L);
    const int G = (d + kGroup - 1) / kGroup;
    const float inv_d = 1.f / (float)d;
    const float inv_sqrt_d = rsqrtf((float)d);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    const int64_t seq0 = (int64_t)b * L;
    const bool first = (blockIdx.x == 0);

    // alpha for rows [t0 - H, t1) of this sequence (and the last H rows when
    // this CTA maintains the conv history)
    const int lo = t0 - H;
    for (int r = lo + warp; r < t1; r += nwarp) {
        float a = 0.f;
        if (r >= 0) a = row_alpha(part, seq0 + r, G, inv_d, eps, inv_sqrt_d, lane);
        if (lane == 0) {
            s_alpha[r - lo] = a;
            if (r >= t0 && alpha_out) alpha_out[seq0 + r] = a;
        }
    }
    if (first && state) {
        for (int i = warp; i < H; i += nwarp) {
            const int r = L - H + i;
            float a = 0.f;
            if (r >= 0) a = row_alpha(part, seq0 + r, G, inv_d, eps, inv_sqrt_d, lane);
            if (lane == 0) s_tail[i] = a;
        }
    }
    __syncthreads();

    const int chunks = d / VN;
    for (int cc = threadIdx.x; cc < chunks; cc += blockDim.x) {
        const int c0 = cc * VN;
        float cw[VN][W];
#pragma unroll
        for (int e = 0; e < VN; ++e)
#pragma unroll
            for (int j = 0; j < W; ++j) cw[e][j] = __ldg(conv_w + (int64_t)(c0 + e) * W + j);

        // history: gated values of rows t0-H .. t0-1 (hist[H-1] most recent)
        float hist[H > 0 ? H : 1][VN];
#pragma unroll
        for (int i = 0; i < H; ++i) {
            const int p = t0 - H + i;
            if (p >= 0) {
                float vv[VN];
                Vec<T>::load(v + (seq0 + p) * d + c0, vv);
                const float a = s_alpha[p - lo];
#pragma unroll
                for (int e = 0; e < VN; ++e) hist[i][e] = a * vv[e];
            } else if (state) {
                const float* sp = state + ((int64_t)b * H + (H + p)) * d + c0;
#pragma unroll
                for (int e = 0; e < VN; ++e) hist[i][e] = sp[e];
            } else {
#pragma unroll
                for (int e = 0; e < VN; ++e) hist[i][e] = 0.f;
            }
        }

        for (int t = t0; t < t1; ++t) {
            const int64_t row = seq0 + t;
            float vv[VN];
            Vec<T>::load(v + row * d + c0, vv);
            const float a = s_alpha[t - lo];
            float out[VN];
            float hv[VN];
            if (add_residual) Vec<T>::load(h + row * d + c0, hv);
#pragma unroll
            for (int e = 0; e < VN; ++e) {
                const float vt = a * vv[e];
                float u = cw[e][0] * vt;
#pragma unroll
                for (int j = 1; j < W; ++j) u = fmaf(cw[e][j], hist[H - j][e], u);
                float r = vt + silu(u);
                if (add_residual) r += hv[e];
                out[e] = r;
#pragma unroll
                for (int i = 0; i + 1 < H; ++i) hist[i][e] = hist[i + 1][e];
                if (H > 0) hist[H > 0 ? H - 1 : 0][e] = vt;
            }
            Vec<T>::store(y + row * d + c0, out);
        }

        // new history: gated values of the sequence's last H rows.  Rows
        // before the sequence start come from the old history (row L + i of
        // the old buffer), read before row i is written.
        if (first && state) {
#pragma unroll
            for (int i = 0; i < H; ++i) {
                const int p = L - H + i;
                float nv[VN];
                if (p >= 0) {
                    float vv[VN];
                    Vec<T>::load(v + (seq0 + p) * d + c0, vv);
#pragma unroll
                    for (int e = 0; e < VN; ++e) nv[e] = s_tail[i] * vv[e];
                } else {
                    const float* sp = state + ((int64_t)b * H + (H + p)) * d + c0;
#pragma unroll
                    for (int e = 0; e < VN; ++e) nv[e] = sp[e];
                }
                float* dp = state + ((int64_t)b * H + i) * d + c0;
#pragma unroll
                for (int e = 0; e < VN; ++e) dp[e] = nv[e];
            }
        }
    }
}

template <typename T, int W>
void launch_w(const void* v, const float* part, const void* h, const float* conv_w, int32_t B, int32_t L,
              int32_t d, float eps, float* state, void* y, float* alpha_out, int32_t add_residual,
              cudaStream_t s) {
    const int chunks = d / Vec<T>::N;
    int threads = ((chunks + 31) / 32) * 32;
    if (threads > 512) threads = 512;
    dim3 grid((unsigned)((L + kTT - 1) / kTT), (unsigned)B);
    gate_conv_kernel<T, W><<<grid, threads, 0, s>>>(static_cast<const T*>(v), reinterpret_cast<const float4*>(part),
                                                    static_cast<const T*>(h), conv_w, L, d, eps, state,
                                                    static_cast<T*>(y), alpha_out, add_residual);
}

template <typename T>
void launch_t(int w, const void* v, const float* part, const void* h, const float* conv_w, int32_t B, int32_t L,
              int32_t d, float eps, float* state, void* y, float* alpha_out, int32_t add_residual, cudaStream_t s) {
    switch (w) {
        case 1: launch_w<T, 1>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s); break;
        case 2: launch_w<T, 2>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s); break;
        case 3: launch_w<T, 3>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s); break;
        case 4: launch_w<T, 4>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s); break;
        case 5: launch_w<T, 5>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s); break;
        case 6: launch_w<T, 6>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s); break;
        case 7: launch_w<T, 7>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s); break;
        default: launch_w<T, 8>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s); break;
    }
}

}  // namespace

cudaError_t launch_gate_conv(bool bf16, const void* v, const float* part, const void* h, const float* conv_w,
                             int32_t B, int32_t L, int32_t d, int32_t w, float eps, float* state, void* y,
                             float* alpha_out, int32_t add_residual, cudaStream_t s) {
    if ((int64_t)B * L == 0) return cudaSuccess;
    if (bf16) {
        launch_t<__nv_bfloat16>(w, v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
    } else {
        launch_t<float>(w, v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
    }
    return cudaGetLastError();
}

}  // namespace engram
