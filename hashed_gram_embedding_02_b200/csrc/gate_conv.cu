// Scalar gate and short causal depthwise convolution from a stored v (CUDA
// cores).  The tensor-core path fuses this step into the projection's
// epilogue; this kernel serves the standalone engram_conv and the shapes the
// tensor-core kernels do not tile.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": the current hidden state
// h_t is the query, the retrieved memory feeds the key and value projections,
// RMSNorm is applied to query and key, and a scalar gate alpha_t in (0, 1)
// scales the value: v~_t = alpha_t v_t.  A short-kernel, per-channel causal
// convolution follows to widen the receptive field and add non-linearity.
// Readings: alpha_t = sigmoid(<q^, k^> / sqrt(d)) with q^ = g_q h / rms(h),
// k^ = g_k k / rms(k); u_t = sum_{j<w} c[j] v~_{t-j}; Y_t = v~_t + SiLU(u_t).
//
// A CTA owns TT consecutive rows of one sequence and a slice of the channels:
//   1. the G partials of its rows and of the w-1 rows before them are staged
//      in shared memory in one pass, then each warp reduces whole rows into
//      alpha (fixed order: deterministic);
//   2. each thread walks a chunk of channels down the rows in groups of RG
//      rows (all loads of a group issued before use), keeping the last w-1
//      gated values in registers.
// The CTAs holding a sequence's first rows also read the conv history and
// write the new one (the last w-1 gated rows, their alpha reduced separately),
// all for their own channels, so updating conv_state in place is race-free.
#include "common.cuh"

namespace engram {

namespace {

constexpr int kTT = 32;   // rows per CTA (>= kMaxConv - 1)
constexpr int kRG = 4;    // rows per load group

__device__ __forceinline__ float alpha_from(float s_qk, float s_kk, float s_hh, float inv_d, float eps,
                                            float inv_sqrt_d) {
    const float rh = sqrtf(s_hh * inv_d + eps);
    const float rk = sqrtf(s_kk * inv_d + eps);
    const float logit = s_qk / (rh * rk) * inv_sqrt_d;
    return 1.f / (1.f + expf(-logit));
}

// alpha of one row from global partials, by one warp
__device__ __forceinline__ float row_alpha_global(const float4* __restrict__ part, int64_t row, int G, float inv_d,
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
    return alpha_from(s_qk, s_kk, s_hh, inv_d, eps, inv_sqrt_d);
}

// SiLU(x) = x * sigmoid(x).  fp32 output: the fast exponential and divide
// intrinsics (a few ulp, far below the 1e-5 bar).  bf16 output: sigmoid(x) =
// (1 + tanh(x/2)) / 2 with the hardware tanh approximation (tanh.approx.f32,
// relative error about 2^-11), below the output's bf16 rounding.
template <typename T>
__device__ __forceinline__ float silu(float x);
template <>
__device__ __forceinline__ float silu<float>(float x) { return __fdividef(x, 1.f + __expf(-x)); }
template <>
__device__ __forceinline__ float silu<__nv_bfloat16>(float x) {
    const float hx = 0.5f * x;
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hx));
    return fmaf(hx, t, hx);
}

// per-thread channel chunk: 8 bytes of output (4 bf16 or 2 fp32 channels);
// v is fp32, so its chunk is 16 or 8 bytes
template <typename T> struct Chunk;
template <> struct Chunk<__nv_bfloat16> {
    static constexpr int N = 4;
    using VT = float4;
    __device__ __forceinline__ static void unpack_v(const float4& q, float* out) {
        out[0] = q.x; out[1] = q.y; out[2] = q.z; out[3] = q.w;
    }
    __device__ __forceinline__ static void unpack(const uint2& q, float* out) {
        out[0] = bf16_lo(q.x); out[1] = bf16_hi(q.x);
        out[2] = bf16_lo(q.y); out[3] = bf16_hi(q.y);
    }
    __device__ __forceinline__ static uint2 pack(const float* in) {
        return make_uint2(pack_bf16x2(in[0], in[1]), pack_bf16x2(in[2], in[3]));
    }
};
template <> struct Chunk<float> {
    static constexpr int N = 2;
    using VT = float2;
    __device__ __forceinline__ static void unpack_v(const float2& q, float* out) {
        out[0] = q.x; out[1] = q.y;
    }
    __device__ __forceinline__ static void unpack(const uint2& q, float* out) {
        out[0] = __uint_as_float(q.x); out[1] = __uint_as_float(q.y);
    }
    __device__ __forceinline__ static uint2 pack(const float* in) {
        return make_uint2(__float_as_uint(in[0]), __float_as_uint(in[1]));
    }
};

template <typename T, int W>
__global__ void __launch_bounds__(160, 4)
gate_conv_kernel(const float* __restrict__ v, const float4* __restrict__ part, const T* __restrict__ h,
                 const float* __restrict__ conv_w, int32_t L, int32_t d, float eps, float* state,
                 T* __restrict__ y, float* __restrict__ alpha_out, int32_t add_residual) {
    using C = Chunk<T>;
    using VT = typename C::VT;
    constexpr int VN = C::N;
    constexpr int H = W - 1;                 // history rows
    extern __shared__ float4 s_part[];       // [(kTT + H) * G]
    __shared__ float s_alpha[kTT + kMaxConv];
    __shared__ float s_tail[kMaxConv];        // alpha of the sequence's last H rows

    const int b = blockIdx.z;
    const int t0 = blockIdx.x * kTT;
    const int t1 = min(t0 + kTT, L);
    const int G = (d + kGroup - 1) / kGroup;
    const float inv_d = 1.f / (float)d;
    const float inv_sqrt_d = rsqrtf((float)d);
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5, nwarp = blockDim.x >> 5;
    const int64_t seq0 = (int64_t)b * L;
    const bool first = (blockIdx.x == 0);
    const int chunks = d / VN;
    const int cc = blockIdx.y * blockDim.x + tid;    // this thread's channel chunk
    const bool has_chunk = cc < chunks;
    const int c0 = cc * VN;

    // ---- 1. gate: partials of rows [lo, t1) into shared memory, then alpha
    const int lo = t0 - H;
    const int R = t1 - lo;
    for (int i = tid; i < R * G; i += blockDim.x) {
        const int r = lo + i / G;
        s_part[i] = r >= 0 ? part[(seq0 + r) * G + (i % G)] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    for (int r = warp; r < R; r += nwarp) {
        float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
        for (int g = lane; g < G; g += 32) {
            const float4 p = s_part[r * G + g];
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
        if (lane == 0) {
            const int row = lo + r;
            const float a = row >= 0 ? alpha_from(s_qk, s_kk, s_hh, inv_d, eps, inv_sqrt_d) : 0.f;
            s_alpha[r] = a;
            if (row >= t0 && alpha_out && blockIdx.y == 0) alpha_out[seq0 + row] = a;
        }
    }
    if (first && state) {
        for (int i = warp; i < H; i += nwarp) {
            const int r = L - H + i;
            float a = 0.f;
            if (r >= 0) a = row_alpha_global(part, seq0 + r, G, inv_d, eps, inv_sqrt_d, lane);
            if (lane == 0) s_tail[i] = a;
        }
    }
    __syncthreads();
    if (!has_chunk) return;

    // ---- 2. convolution down the rows
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
            C::unpack_v(*reinterpret_cast<const VT*>(v + (seq0 + p) * d + c0), vv);
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

    const float* vp = v + (seq0 + t0) * d + c0;
    const T* hp = h + (seq0 + t0) * d + c0;
    T* yp = y + (seq0 + t0) * d + c0;
    const float* ap = s_alpha + (t0 - lo);
    for (int tb = t0; tb < t1; tb += kRG) {
        const int nr = min(kRG, t1 - tb);
        VT vq[kRG];
        uint2 hq[kRG];
#pragma unroll
        for (int r = 0; r < kRG; ++r) {
            if (r < nr) {
                vq[r] = *reinterpret_cast<const VT*>(vp + (int64_t)r * d);
                if (add_residual) hq[r] = *reinterpret_cast<const uint2*>(hp + (int64_t)r * d);
            }
        }
#pragma unroll
        for (int r = 0; r < kRG; ++r) {
            if (r < nr) {
                float vv[VN], hv[VN], out[VN];
                C::unpack_v(vq[r], vv);
                if (add_residual) C::unpack(hq[r], hv);
                const float a = ap[r];
#pragma unroll
                for (int e = 0; e < VN; ++e) {
                    const float vt = a * vv[e];
                    float u = cw[e][0] * vt;
#pragma unroll
                    for (int j = 1; j < W; ++j) u = fmaf(cw[e][j], hist[H - j][e], u);
                    float res = vt + silu<T>(u);
                    if (add_residual) res += hv[e];
                    out[e] = res;
#pragma unroll
                    for (int i = 0; i + 1 < H; ++i) hist[i][e] = hist[i + 1][e];
                    if (H > 0) hist[H > 0 ? H - 1 : 0][e] = vt;
                }
                *reinterpret_cast<uint2*>(yp + (int64_t)r * d) = C::pack(out);
            }
        }
        vp += (int64_t)kRG * d;
        hp += (int64_t)kRG * d;
        yp += (int64_t)kRG * d;
        ap += kRG;
    }

    // new history: gated values of the sequence's last H rows.  Rows before the
    // sequence start come from the old history (row L + i of the old buffer),
    // read before row i is written.
    if (first && state) {
#pragma unroll
        for (int i = 0; i < H; ++i) {
            const int p = L - H + i;
            float nv[VN];
            if (p >= 0) {
                float vv[VN];
                C::unpack_v(*reinterpret_cast<const VT*>(v + (seq0 + p) * d + c0), vv);
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

template <typename T, int W>
cudaError_t launch_w(const float* v, const float* part, const void* h, const float* conv_w, int32_t B, int32_t L,
                     int32_t d, float eps, float* state, void* y, float* alpha_out, int32_t add_residual,
                     cudaStream_t s) {
    const int chunks = d / Chunk<T>::N;
    int slices = (chunks + 80) / 160;            // about 160 chunks per CTA
    if (slices < 1) slices = 1;
    int threads = (chunks + slices - 1) / slices;
    threads = ((threads + 31) / 32) * 32;
    if (threads > 160) {
        threads = 160;
        slices = (chunks + 159) / 160;
    }
    const int G = (d + kGroup - 1) / kGroup;
    const size_t smem = (size_t)(kTT + W - 1) * G * sizeof(float4);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(gate_conv_kernel<T, W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((unsigned)((L + kTT - 1) / kTT), (unsigned)slices, (unsigned)B);
    gate_conv_kernel<T, W><<<grid, threads, smem, s>>>(v, reinterpret_cast<const float4*>(part),
                                                       static_cast<const T*>(h), conv_w, L, d, eps, state,
                                                       static_cast<T*>(y), alpha_out, add_residual);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(int w, const float* v, const float* part, const void* h, const float* conv_w, int32_t B,
                     int32_t L, int32_t d, float eps, float* state, void* y, float* alpha_out, int32_t add_residual,
                     cudaStream_t s) {
    switch (w) {
        case 1: return launch_w<T, 1>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
        case 2: return launch_w<T, 2>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
        case 3: return launch_w<T, 3>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
        case 4: return launch_w<T, 4>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
        case 5: return launch_w<T, 5>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
        case 6: return launch_w<T, 6>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
        case 7: return launch_w<T, 7>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
        default: return launch_w<T, 8>(v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
    }
}

}  // namespace

cudaError_t launch_gate_conv(bool bf16, const float* v, const float* part, const void* h, const float* conv_w,
                             int32_t B, int32_t L, int32_t d, int32_t w, float eps, float* state, void* y,
                             float* alpha_out, int32_t add_residual, uint32_t* status, cudaStream_t s) {
    (void)status;
    if ((int64_t)B * L == 0) return cudaSuccess;
    if (bf16) return launch_t<__nv_bfloat16>(w, v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
    return launch_t<float>(w, v, part, h, conv_w, B, L, d, eps, state, y, alpha_out, add_residual, s);
}

}  // namespace engram
