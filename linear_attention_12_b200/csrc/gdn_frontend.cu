// gdn_frontend.cu -- the GDN front end (sm_100a): short causal convolution of
// the q, k, v channels, L2 normalisation of q and k, gate activations.
//
// What it computes (the jianying88.com article "Qwen3.8-Flash-Next混合注意力
// 深度解析…", section 三: the GDN layer stacks a short convolution of kernel
// width 4, config linear_conv_kernel_dim 4; the pages print no formula):
//
//   y[t, c] = sum_{i=0..3} w[c, i] x[t - 3 + i, c]    (x = 0 before the sequence start)
//   y = act(y)                                        (none, or SiLU y sigmoid(y))
//   q, k = y / sqrt(sum_head y^2 + eps)               (per token and head)
//   log_alpha = -softplus(a),  beta = sigmoid(b)
//
// The normalisation and the gate activations follow the recipes of the
// workloads the layer is measured on.  Channels are ordered q (head-major),
// k, v; the weight is [(2 H_qk + H_v) d, 4] fp32.
//
// The work is HBM-bound: one warp streams 16 consecutive tokens of one head,
// each lane holding 4 channels, with the three previous rows of the causal
// window kept in registers; rows load and store as one coalesced 256-byte
// (bf16) or 512-byte (fp32) segment per warp.
#include <cuda_bf16.h>

#include "../../include/gdn.h"
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int FD = 128;      // head dim
constexpr int FE_TOK = 16;   // tokens per warp
constexpr int FE_WARPS = 4;  // warps per CTA: 64 consecutive tokens

template <typename IO>
struct Vec4;
template <>
struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 load(const __nv_bfloat16* p) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float4 v) {
        uint2 u;
        u.x = pack_bf16x2(v.x, v.y);
        u.y = pack_bf16x2(v.z, v.w);
        *reinterpret_cast<uint2*>(p) = u;
    }
};
template <>
struct Vec4<float> {
    static __device__ __forceinline__ float4 load(const float* p) {
        return *reinterpret_cast<const float4*>(p);
    }
    static __device__ __forceinline__ void store(float* p, float4 v) {
        *reinterpret_cast<float4*>(p) = v;
    }
};

__device__ __forceinline__ float silu(float y) { return y / (1.f + expf(-y)); }

__device__ __forceinline__ float4 act4(float4 y, int act) {
    if (act == GDN_ACT_SILU) return make_float4(silu(y.x), silu(y.y), silu(y.z), silu(y.w));
    return y;
}

// y = w0 x_{t-3} + w1 x_{t-2} + w2 x_{t-1} + w3 x_t for 4 channels
__device__ __forceinline__ float4 conv4(const float4 (&w)[4], float4 x3, float4 x2, float4 x1,
                                        float4 x0) {
    float4 y;
    y.x = fmaf(w[0].x, x3.x, fmaf(w[1].x, x2.x, fmaf(w[2].x, x1.x, w[3].x * x0.x)));
    y.y = fmaf(w[0].y, x3.y, fmaf(w[1].y, x2.y, fmaf(w[2].y, x1.y, w[3].y * x0.y)));
    y.z = fmaf(w[0].z, x3.z, fmaf(w[1].z, x2.z, fmaf(w[2].z, x1.z, w[3].z * x0.z)));
    y.w = fmaf(w[0].w, x3.w, fmaf(w[1].w, x2.w, fmaf(w[2].w, x1.w, w[3].w * x0.w)));
    return y;
}

// Scale 4 channels of a head row to unit L2 norm over the head (the warp holds
// the whole 128-channel row).
__device__ __forceinline__ float4 l2norm_row(float4 y, float eps) {
    float ss = y.x * y.x + y.y * y.y + y.z * y.z + y.w * y.w;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float r = rsqrtf(ss + eps);
    return make_float4(y.x * r, y.y * r, y.z * r, y.w * r);
}

// softplus(a) = max(a, 0) + log(1 + e^{-|a|}), without overflow
__device__ __forceinline__ float softplus(float a) { return fmaxf(a, 0.f) + log1pf(expf(-fabsf(a))); }
__device__ __forceinline__ float sigmoidf(float b) { return 1.f / (1.f + expf(-b)); }

// Start of the sequence that holds token t (the last cu[n] <= t).
__device__ __forceinline__ int seq_start(const int32_t* cu, int N, int t) {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return cu[lo];
}

// The first sequence start after token t (cu[N] = T closes the last sequence).
__device__ __forceinline__ int next_start(const int32_t* cu, int N, int t) {
    int lo = 0, hi = N;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] > t) hi = mid; else lo = mid + 1;
    }
    return cu[lo];
}

struct FrontendParams {
    const void* x[3];      // q_raw, k_raw, v_raw
    void* y[3];            // q, k, v
    const float* w;        // [(2 H_qk + H_v) d, 4]
    const float* a;        // [T, H_v]
    const float* b;
    float* log_alpha;
    float* beta;
    const int32_t* cu_seqlens;
    int N, T, H_qk, H_v;
    int act;
    float eps;
};

// Grid (ceil(T / 64), 2 H_qk + H_v): warp w of CTA (bx, hid) handles tokens
// 64 bx + 16 w .. +15 of head hid (q heads first, then k, then v).
template <typename IO>
__global__ void __launch_bounds__(FE_WARPS * 32)
    frontend_kernel(const FrontendParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hid = blockIdx.y;
    const int kind = hid < p.H_qk ? 0 : (hid < 2 * p.H_qk ? 1 : 2);  // q, k, v
    const int head = kind == 0 ? hid : (kind == 1 ? hid - p.H_qk : hid - 2 * p.H_qk);
    const int H = kind == 2 ? p.H_v : p.H_qk;
    const int t0 = blockIdx.x * (FE_WARPS * FE_TOK) + warp * FE_TOK;
    if (t0 >= p.T) return;  // warp-uniform
    const int t1 = min(t0 + FE_TOK, p.T);
    // (the pointers are picked without indexing the parameter arrays at run time)
    const void* xk = kind == 0 ? p.x[0] : (kind == 1 ? p.x[1] : p.x[2]);
    void* yk = kind == 0 ? p.y[0] : (kind == 1 ? p.y[1] : p.y[2]);
    const IO* x = static_cast<const IO*>(xk) + (size_t)head * FD + 4 * lane;
    IO* y = static_cast<IO*>(yk) + (size_t)head * FD + 4 * lane;
    const size_t rs = (size_t)H * FD;  // row stride in elements

    float4 w[4];
    {
        const float4* wp = reinterpret_cast<const float4*>(p.w + ((size_t)hid * FD + 4 * lane) * 4);
        // 4 channels x 4 taps, channel-major -> per-tap float4 over the channels
        const float4 c0 = wp[0], c1 = wp[1], c2 = wp[2], c3 = wp[3];
        w[0] = make_float4(c0.x, c1.x, c2.x, c3.x);
        w[1] = make_float4(c0.y, c1.y, c2.y, c3.y);
        w[2] = make_float4(c0.z, c1.z, c2.z, c3.z);
        w[3] = make_float4(c0.w, c1.w, c2.w, c3.w);
    }
    // causal window: x_{t-3}, x_{t-2}, x_{t-1} (zero before the sequence start)
    const int s = seq_start(p.cu_seqlens, p.N, t0);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 x3 = (t0 - 3 >= s) ? Vec4<IO>::load(x + (size_t)(t0 - 3) * rs) : z;
    float4 x2 = (t0 - 2 >= s) ? Vec4<IO>::load(x + (size_t)(t0 - 2) * rs) : z;
    float4 x1 = (t0 - 1 >= s) ? Vec4<IO>::load(x + (size_t)(t0 - 1) * rs) : z;
    int nxt = next_start(p.cu_seqlens, p.N, t0);  // the next sequence start after t0
    for (int t = t0; t < t1; ++t) {
        if (t == nxt) {  // a sequence starts at t: its window starts empty
            x3 = x2 = x1 = z;
            nxt = next_start(p.cu_seqlens, p.N, t);
        }
        const float4 x0 = Vec4<IO>::load(x + (size_t)t * rs);
        float4 v = act4(conv4(w, x3, x2, x1, x0), p.act);
        if (kind < 2) v = l2norm_row(v, p.eps);
        Vec4<IO>::store(y + (size_t)t * rs, v);
        x3 = x2;
        x2 = x1;
        x1 = x0;
    }
    // gates, once per (token, value head): lanes 0-15 log_alpha, 16-31 beta
    if (kind == 2) {
        const int t = t0 + (lane & 15);
        if (t < t1) {
            const size_t gi = (size_t)t * p.H_v + head;
            if (lane < 16) p.log_alpha[gi] = -softplus(p.a[gi]);
            else p.beta[gi] = sigmoidf(p.b[gi]);
        }
    }
}

// Grid (B, 2 H_qk + H_v), one warp: one decode step of one head of one sequence.
// state [B, 3, C] (io dtype) holds the last three raw input rows, oldest first;
// it is shifted in place.
template <typename IO>
__global__ void __launch_bounds__(32)
    frontend_decode_kernel(const FrontendParams p, IO* state, int C) {
    const int lane = threadIdx.x;
    const int bi = blockIdx.x, hid = blockIdx.y;
    const int kind = hid < p.H_qk ? 0 : (hid < 2 * p.H_qk ? 1 : 2);
    const int head = kind == 0 ? hid : (kind == 1 ? hid - p.H_qk : hid - 2 * p.H_qk);
    const int H = kind == 2 ? p.H_v : p.H_qk;
    const size_t off = ((size_t)bi * H + head) * FD + 4 * lane;
    float4 w[4];
    {
        const float4* wp = reinterpret_cast<const float4*>(p.w + ((size_t)hid * FD + 4 * lane) * 4);
        const float4 c0 = wp[0], c1 = wp[1], c2 = wp[2], c3 = wp[3];
        w[0] = make_float4(c0.x, c1.x, c2.x, c3.x);
        w[1] = make_float4(c0.y, c1.y, c2.y, c3.y);
        w[2] = make_float4(c0.z, c1.z, c2.z, c3.z);
        w[3] = make_float4(c0.w, c1.w, c2.w, c3.w);
    }
    IO* sp = state + (size_t)bi * 3 * C + (size_t)hid * FD + 4 * lane;
    const float4 x3 = Vec4<IO>::load(sp), x2 = Vec4<IO>::load(sp + C),
                 x1 = Vec4<IO>::load(sp + 2 * C);
    const void* xk = kind == 0 ? p.x[0] : (kind == 1 ? p.x[1] : p.x[2]);
    void* yk = kind == 0 ? p.y[0] : (kind == 1 ? p.y[1] : p.y[2]);
    const float4 x0 = Vec4<IO>::load(static_cast<const IO*>(xk) + off);
    float4 v = act4(conv4(w, x3, x2, x1, x0), p.act);
    if (kind < 2) v = l2norm_row(v, p.eps);
    Vec4<IO>::store(static_cast<IO*>(yk) + off, v);
    // the raw rows are stored as given (exact in the io dtype)
    Vec4<IO>::store(sp, x2);
    Vec4<IO>::store(sp + C, x1);
    Vec4<IO>::store(sp + 2 * C, x0);
    if (kind == 2 && lane < 2) {
        const size_t gi = (size_t)bi * p.H_v + head;
        if (lane == 0) p.log_alpha[gi] = -softplus(p.a[gi]);
        else p.beta[gi] = sigmoidf(p.b[gi]);
    }
}

}  // namespace

cudaError_t launch_frontend(const void* q_raw, const void* k_raw, const void* v_raw,
                            const float* conv_w, const float* a, const float* b,
                            const int32_t* cu_seqlens, int N, int T, int H_qk, int H_v,
                            bool bf16, int act, float eps, void* q, void* k, void* v,
                            float* log_alpha, float* beta, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    FrontendParams prm{{q_raw, k_raw, v_raw}, {q, k, v}, conv_w, a, b, log_alpha, beta,
                       cu_seqlens, N, T, H_qk, H_v, act, eps};
    dim3 grid((T + FE_WARPS * FE_TOK - 1) / (FE_WARPS * FE_TOK), 2 * H_qk + H_v);
    if (bf16)
        frontend_kernel<__nv_bfloat16><<<grid, FE_WARPS * 32, 0, stream>>>(prm);
    else
        frontend_kernel<float><<<grid, FE_WARPS * 32, 0, stream>>>(prm);
    return cudaGetLastError();
}

cudaError_t launch_frontend_decode(const void* q_raw, const void* k_raw, const void* v_raw,
                                   const float* conv_w, const float* a, const float* b,
                                   void* conv_state, int B, int H_qk, int H_v, bool bf16, int act,
                                   float eps, void* q, void* k, void* v, float* log_alpha,
                                   float* beta, cudaStream_t stream) {
    if (B == 0) return cudaSuccess;
    FrontendParams prm{{q_raw, k_raw, v_raw}, {q, k, v}, conv_w, a, b, log_alpha, beta,
                       nullptr, 0, 0, H_qk, H_v, act, eps};
    const int C = (2 * H_qk + H_v) * FD;
    dim3 grid(B, 2 * H_qk + H_v);
    if (bf16)
        frontend_decode_kernel<__nv_bfloat16><<<grid, 32, 0, stream>>>(
            prm, static_cast<__nv_bfloat16*>(conv_state), C);
    else
        frontend_decode_kernel<float><<<grid, 32, 0, stream>>>(prm, static_cast<float*>(conv_state),
                                                               C);
    return cudaGetLastError();
}

}  // namespace gdn
