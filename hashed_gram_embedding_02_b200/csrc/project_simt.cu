// Key/value projections on CUDA cores, with the gate's partial sums.
//
// "DeepSeek AI II" digest, section "DeepSeek Engram": k_t = W_K e_t and
// v_t = W_V e_t; RMSNorm is applied to the query h_t and to the key before
// the scalar gate.  This kernel computes, for a tile of 32 rows and one
// group of 128 channels, both k and v (fp32 accumulation in a fixed order),
// writes v in fp32 and reduces the group's gate partials
//   (sum g_q g_k h k, sum k^2, sum h^2)
// so that k is never written to memory.  It serves the fp32 configuration
// and bf16 shapes that the tensor-core kernels do not tile.
#include "common.cuh"

namespace engram {

namespace {

constexpr int kRows = 32;     // rows per CTA
constexpr int kKc = 32;       // reduction chunk
constexpr int kThreads = 256; // channel c = tid % 128, row half = tid / 128

template <typename T>
__global__ void __launch_bounds__(kThreads)
project_simt_kernel(const T* __restrict__ e, int64_t n_tok, int32_t d_mem, const T* __restrict__ h,
                    const T* __restrict__ Wk, const T* __restrict__ Wv, const float* __restrict__ gq,
                    const float* __restrict__ gk, int32_t d, float* __restrict__ v, float* __restrict__ part) {
    __shared__ float e_s[kRows][kKc + 1];
    __shared__ float wk_s[kGroup][kKc + 1];
    __shared__ float wv_s[kGroup][kKc + 1];
    __shared__ float red[3][kRows][4];

    const int tid = threadIdx.x;
    const int c_loc = tid & (kGroup - 1);
    const int half = tid >> 7;
    const int g = blockIdx.y;
    const int c = g * kGroup + c_loc;
    const int64_t r0 = (int64_t)blockIdx.x * kRows;

    float acc_k[16], acc_v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        acc_k[i] = 0.f;
        acc_v[i] = 0.f;
    }

    for (int q0 = 0; q0 < d_mem; q0 += kKc) {
        // e tile: 32 x 32
        for (int i = tid; i < kRows * kKc; i += kThreads) {
            const int rr = i / kKc, qq = i % kKc;
            const int64_t row = r0 + rr;
            const int q = q0 + qq;
            e_s[rr][qq] = (row < n_tok && q < d_mem) ? to_f(e[row * d_mem + q]) : 0.f;
        }
        // W tiles: 128 channels x 32
        for (int i = tid; i < kGroup * kKc; i += kThreads) {
            const int cc = i / kKc, qq = i % kKc;
            const int ch = g * kGroup + cc;
            const int q = q0 + qq;
            const bool ok = ch < d && q < d_mem;
            wk_s[cc][qq] = ok ? to_f(Wk[(int64_t)ch * d_mem + q]) : 0.f;
            wv_s[cc][qq] = ok ? to_f(Wv[(int64_t)ch * d_mem + q]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int qq = 0; qq < kKc; ++qq) {
            const float wk = wk_s[c_loc][qq];
            const float wv = wv_s[c_loc][qq];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float a = e_s[half * 16 + i][qq];
                acc_k[i] = fmaf(a, wk, acc_k[i]);
                acc_v[i] = fmaf(a, wv, acc_v[i]);
            }
        }
        __syncthreads();
    }

    // epilogue: v store, gate partials reduced over the group's channels
    const float gg = (c < d) ? (gq ? gq[c] : 1.f) * (gk ? gk[c] : 1.f) : 0.f;
    const int warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3;  // warp index within the row half
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int rr = half * 16 + i;
        const int64_t row = r0 + rr;
        float s_qk = 0.f, s_kk = 0.f, s_hh = 0.f;
        if (row < n_tok && c < d) {
            v[row * d + c] = acc_v[i];
            const float hv = to_f(h[row * d + c]);
            s_qk = gg * hv * acc_k[i];
            s_kk = acc_k[i] * acc_k[i];
            s_hh = hv * hv;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            s_qk += __shfl_xor_sync(0xffffffffu, s_qk, off);
            s_kk += __shfl_xor_sync(0xffffffffu, s_kk, off);
            s_hh += __shfl_xor_sync(0xffffffffu, s_hh, off);
        }
        if (lane == 0) {
            red[0][rr][wq] = s_qk;
            red[1][rr][wq] = s_kk;
            red[2][rr][wq] = s_hh;
        }
    }
    __syncthreads();
    const int G = (d + kGroup - 1) / kGroup;
    if (tid < kRows) {
        const int64_t row = r0 + tid;
        if (row < n_tok) {
            float4 o;
            o.x = (red[0][tid][0] + red[0][tid][1]) + (red[0][tid][2] + red[0][tid][3]);
            o.y = (red[1][tid][0] + red[1][tid][1]) + (red[1][tid][2] + red[1][tid][3]);
            o.z = (red[2][tid][0] + red[2][tid][1]) + (red[2][tid][2] + red[2][tid][3]);
            o.w = 0.f;
            reinterpret_cast<float4*>(part)[row * G + g] = o;
        }
    }
}

}  // namespace

cudaError_t launch_project_simt(bool bf16, const void* e, int64_t n_tok, int32_t d_mem, const void* h,
                                const void* Wk, const void* Wv, const float* gq, const float* gk, int32_t d,
                                float* v, float* part, cudaStream_t s) {
    if (n_tok == 0) return cudaSuccess;
    dim3 grid((unsigned)((n_tok + kRows - 1) / kRows), (unsigned)((d + kGroup - 1) / kGroup));
    if (bf16) {
        using T = __nv_bfloat16;
        project_simt_kernel<T><<<grid, kThreads, 0, s>>>(
            static_cast<const T*>(e), n_tok, d_mem, static_cast<const T*>(h), static_cast<const T*>(Wk),
            static_cast<const T*>(Wv), gq, gk, d, v, part);
    } else {
        project_simt_kernel<float><<<grid, kThreads, 0, s>>>(
            static_cast<const float*>(e), n_tok, d_mem, static_cast<const float*>(h),
            static_cast<const float*>(Wk), static_cast<const float*>(Wv), gq, gk, d, v, part);
    }
    return cudaGetLastError();
}

}  // namespace engram
