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
// The work is HBM-bound.  The prefill form stages each block's rows in shared
// memory with bulk copies (up to 35 KB in flight per block, six blocks per
// SM), then one warp per head convolves them with a rolling window, each lane
// holding 4 channels; outputs leave as one coalesced 256-byte (bf16) or
// 512-byte (fp32) row segment per warp.
#include <cuda_bf16.h>

#include "../../include/gdn.h"
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int FD = 128;      // head dim

template <typename IO>
struct Vec4;
template <>
struct Vec4<__nv_bfloat16> {
    using Raw = uint2;  // 4 channels as stored
    static __device__ __forceinline__ Raw load_raw(const __nv_bfloat16* p) {
        return *reinterpret_cast<const uint2*>(p);
    }
    static __device__ __forceinline__ Raw zero() { return make_uint2(0u, 0u); }
    static __device__ __forceinline__ float4 widen(Raw u) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
    static __device__ __forceinline__ float4 load(const __nv_bfloat16* p) {
        return widen(load_raw(p));
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
    using Raw = float4;
    static __device__ __forceinline__ Raw load_raw(const float* p) {
        return *reinterpret_cast<const float4*>(p);
    }
    static __device__ __forceinline__ Raw zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
    static __device__ __forceinline__ float4 widen(Raw u) { return u; }
    static __device__ __forceinline__ float4 load(const float* p) { return load_raw(p); }
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

// ---- prefill front end: rows staged in shared memory by bulk copies ----
//
// A block handles FE_TC consecutive tokens of a group of HG heads of one
// kind (HG = 4 for bf16, 2 for fp32: 1 KB of each token row).  One thread
// issues one bulk copy per token row -- the three rows of history before the
// tile and its FE_TC tokens -- so that the whole tile (up to 35 KB) is in
// flight at once; warp w then convolves head w of the group from shared
// memory with a rolling window, each lane holding 4 channels.
constexpr int FE_TC = 32;                         // tokens per block
constexpr int FE_ROWS = FE_TC + 3;                // staged rows: history + tile
constexpr uint32_t FE_ROWB = 1024;                // shared-memory bytes of one staged row
constexpr uint32_t FE_SMEM = FE_ROWS * FE_ROWB + 16;  // + mbarrier and abort flag
static_assert(FE_TC <= 32, "lane j handles token j of a tile (gates, sequence starts)");

template <typename IO>
__host__ __device__ constexpr int fe_heads() { return FE_ROWB / (FD * sizeof(IO)); }

// Grid: token tiles x head groups (q groups, then k, then v), the group index
// varying fastest so that the blocks resident at one time read whole token rows.
template <typename IO, int ACT>
__global__ void __launch_bounds__(fe_heads<IO>() * 32)
    frontend_kernel(const FrontendParams p) {
    constexpr int HG = fe_heads<IO>();
    extern __shared__ __align__(128) uint8_t fe_sm[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(fe_sm + FE_ROWS * FE_ROWB);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(fe_sm + FE_ROWS * FE_ROWB + 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int gq = (p.H_qk + HG - 1) / HG, gv = (p.H_v + HG - 1) / HG;
    const int NG = 2 * gq + gv;
    const int grp = blockIdx.x % NG, tile = blockIdx.x / NG;
    const int kind = grp < gq ? 0 : (grp < 2 * gq ? 1 : 2);  // q, k, v
    const int head0 = HG * (kind == 0 ? grp : (kind == 1 ? grp - gq : grp - 2 * gq));
    const int H = kind == 2 ? p.H_v : p.H_qk;
    const int nh = min(HG, H - head0);
    const int t0 = tile * FE_TC;  // < T: the grid holds exactly the tiles that start inside
    const int t1 = min(t0 + FE_TC, p.T);
    const size_t rs = (size_t)H * FD;  // row stride in elements
    // (the pointers are picked without indexing the parameter arrays at run time)
    const IO* x = static_cast<const IO*>(kind == 0 ? p.x[0] : (kind == 1 ? p.x[1] : p.x[2]));
    IO* y = static_cast<IO*>(kind == 0 ? p.y[0] : (kind == 1 ? p.y[1] : p.y[2]));

    // staged row i holds token t0 - 3 + i; rows before token 0 are not loaded
    const int r_lo = max(0, t0 - 3);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        const uint32_t row_bytes = (uint32_t)nh * FD * sizeof(IO);
        mbar_arrive_expect_tx(bar, (uint32_t)(t1 - r_lo) * row_bytes);
        for (int t = r_lo; t < t1; ++t)
            bulk_load(fe_sm + (t - (t0 - 3)) * FE_ROWB, x + (size_t)t * rs + (size_t)head0 * FD,
                      row_bytes, bar);
    }

    // while the rows land: weights, gate inputs, sequence starts
    const bool active = warp < nh;
    const int head = head0 + min(warp, nh - 1);
    const int hid = (kind == 0 ? 0 : (kind == 1 ? p.H_qk : 2 * p.H_qk)) + head;
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
    const int tg = t0 + lane;  // lane <-> token for the gates and the sequence starts
    float ga = 0.f, gb = 0.f;
    const bool gate = kind == 2 && active && tg < t1;
    if (gate) {
        ga = p.a[(size_t)tg * p.H_v + head];
        gb = p.b[(size_t)tg * p.H_v + head];
    }
    const int s_mine = seq_start(p.cu_seqlens, p.N, min(tg, t1 - 1));
    const bool one_seq = __all_sync(0xffffffffu, s_mine <= t0 - 3);

    __syncthreads();  // the barrier is initialised before anyone waits on it
    const bool ok = mbar_wait(bar, 0, abort_flag);
    if (!__syncthreads_and(ok)) {
        // the copies may still land: wait for them (bounded) before the block exits
        if (threadIdx.x == 0) {
            const unsigned long long ts = globaltimer();
            while (!mbar_try_wait(smem_u32(bar), 0) && globaltimer() - ts < kWaitLimitNs) {
            }
        }
        __syncthreads();
        return;
    }

    if (active) {
        const uint8_t* rp = fe_sm + (warp * FD + 4 * lane) * sizeof(IO);
        float4 x3 = Vec4<IO>::widen(*reinterpret_cast<const typename Vec4<IO>::Raw*>(rp));
        float4 x2 = Vec4<IO>::widen(*reinterpret_cast<const typename Vec4<IO>::Raw*>(rp + FE_ROWB));
        float4 x1 =
            Vec4<IO>::widen(*reinterpret_cast<const typename Vec4<IO>::Raw*>(rp + 2 * FE_ROWB));
        IO* yt = y + (size_t)t0 * rs + (size_t)head * FD + 4 * lane;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int j = 0; j < FE_TC; ++j) {
            const float4 x0 = Vec4<IO>::widen(
                *reinterpret_cast<const typename Vec4<IO>::Raw*>(rp + (j + 3) * FE_ROWB));
            float4 a3 = x3, a2 = x2, a1 = x1;
            if (!one_seq) {  // taps before the start of token t's sequence are zero
                const int t = t0 + j, s = __shfl_sync(0xffffffffu, s_mine, j);
                a3 = (t - 3 >= s) ? a3 : z;
                a2 = (t - 2 >= s) ? a2 : z;
                a1 = (t - 1 >= s) ? a1 : z;
            }
            float4 v = act4(conv4(w, a3, a2, a1, x0), ACT);
            if (kind < 2) v = l2norm_row(v, p.eps);
            if (t0 + j < t1) Vec4<IO>::store(yt, v);
            yt += rs;
            x3 = x2;
            x2 = x1;
            x1 = x0;
        }
    }
    if (gate) {
        p.log_alpha[(size_t)tg * p.H_v + head] = -softplus(ga);
        p.beta[(size_t)tg * p.H_v + head] = sigmoidf(gb);
    }
}

template <typename IO, int ACT>
cudaError_t launch_frontend_t(const FrontendParams& prm, int T, int H_qk, int H_v,
                              cudaStream_t stream) {
    constexpr int HG = fe_heads<IO>();
    const cudaError_t attr = cudaFuncSetAttribute(
        frontend_kernel<IO, ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize, FE_SMEM);
    if (attr != cudaSuccess) return attr;
    const long long groups = 2LL * ((H_qk + HG - 1) / HG) + (H_v + HG - 1) / HG;
    const long long blocks = ((long long)T + FE_TC - 1) / FE_TC * groups;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    frontend_kernel<IO, ACT><<<(unsigned)blocks, HG * 32, FE_SMEM, stream>>>(prm);
    return cudaGetLastError();
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
    if (bf16)
        return act == GDN_ACT_SILU
                   ? launch_frontend_t<__nv_bfloat16, GDN_ACT_SILU>(prm, T, H_qk, H_v, stream)
                   : launch_frontend_t<__nv_bfloat16, GDN_ACT_NONE>(prm, T, H_qk, H_v, stream);
    return act == GDN_ACT_SILU ? launch_frontend_t<float, GDN_ACT_SILU>(prm, T, H_qk, H_v, stream)
                               : launch_frontend_t<float, GDN_ACT_NONE>(prm, T, H_qk, H_v, stream);
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
