// gdn_decode.cu -- one decode step of the gated delta rule, HBM-bound.
//
// For each (sequence b, value head h), with k, q from query/key head
// h / (H_v / H_qk) and alpha = exp(log_alpha), the state-update formula of
// the bjdmk.com.cn article (section 2.1) is evaluated in one pass over S:
//
//     a = S^T k,  b = S^T q                  (column reductions over d_k)
//     w = beta (v - alpha a)                 (the corrected write vector)
//     o = alpha b + (k . q) w                (= S_new^T q)
//     S_new = alpha S + k w^T                (written back in place)
//
// which equals alpha (I - beta k k^T) S + beta k v^T and o = S_new^T q.
//
// Work split: one CTA of 256 threads per (b, h).  Thread (warp w, lane l)
// owns columns [4l, 4l+4) of rows w, w+8, ..., w+120 -- 16 float4 = 64 fp32
// registers -- so every warp load/store is one contiguous 512-byte row.  The
// whole 64 KiB state is loaded before any reduction, giving 64 KiB in flight
// per CTA; loads and stores use the streaming (evict-first) cache policy
// because each state is touched exactly once per step.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kD = 128;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerThread = kD / kWarps;  // 16

template <typename IO>
__device__ __forceinline__ float io_load(const IO* p);
template <>
__device__ __forceinline__ float io_load<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float io_load<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(__ldg(p));
}

template <typename IO>
__device__ __forceinline__ void io_store4(IO* p, float4 v);
template <>
__device__ __forceinline__ void io_store4<float>(float* p, float4 v) {
    *reinterpret_cast<float4*>(p) = v;
}
template <>
__device__ __forceinline__ void io_store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
    uint2 u;
    u.x = pack_bf16x2(v.x, v.y);
    u.y = pack_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2*>(p) = u;
}

template <typename IO>
__global__ void __launch_bounds__(kThreads, 2)
    decode_step_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                       const IO* __restrict__ v, const float* __restrict__ log_alpha,
                       const float* __restrict__ beta, float* __restrict__ S, int H_qk, int H_v,
                       IO* __restrict__ o) {
    __shared__ float s_k[kD];
    __shared__ float s_q[kD];
    __shared__ float4 s_part[2][kWarps][32];

    const int unit = blockIdx.x;  // b * H_v + h
    const int b = unit / H_v;
    const int h = unit - b * H_v;
    const int hq = h / (H_v / H_qk);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    float* Sg = S + (size_t)unit * (kD * kD);

    // Issue all state loads first: 16 x 16 B per thread.
    float4 s[kRowsPerThread];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i)
        s[i] = __ldcs(reinterpret_cast<const float4*>(Sg + (size_t)(warp + kWarps * i) * kD) +
                      lane);

    const size_t qk_off = ((size_t)b * H_qk + hq) * kD;
    if (tid < kD)
        s_k[tid] = io_load(k + qk_off + tid);
    else
        s_q[tid - kD] = io_load(q + qk_off + (tid - kD));
    const float alpha = expf(log_alpha[unit]);
    const float bet = beta[unit];
    const size_t v_off = (size_t)unit * kD + 4 * lane;
    float4 vv;
    vv.x = io_load(v + v_off + 0);
    vv.y = io_load(v + v_off + 1);
    vv.z = io_load(v + v_off + 2);
    vv.w = io_load(v + v_off + 3);
    __syncthreads();

    // Partial column sums over this thread's 16 rows.
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), bq = a;
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = warp + kWarps * i;
        const float kr = s_k[r], qr = s_q[r];
        a.x = fmaf(s[i].x, kr, a.x); a.y = fmaf(s[i].y, kr, a.y);
        a.z = fmaf(s[i].z, kr, a.z); a.w = fmaf(s[i].w, kr, a.w);
        bq.x = fmaf(s[i].x, qr, bq.x); bq.y = fmaf(s[i].y, qr, bq.y);
        bq.z = fmaf(s[i].z, qr, bq.z); bq.w = fmaf(s[i].w, qr, bq.w);
    }
    s_part[0][warp][lane] = a;
    s_part[1][warp][lane] = bq;
    // k . q, reduced within each warp (every warp computes it; no extra sync).
    float kq = 0.f;
#pragma unroll
    for (int i = 0; i < kD / 32; ++i) kq = fmaf(s_k[lane + 32 * i], s_q[lane + 32 * i], kq);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    __syncthreads();

    a = make_float4(0.f, 0.f, 0.f, 0.f);
    bq = a;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const float4 pa = s_part[0][w][lane], pb = s_part[1][w][lane];
        a.x += pa.x; a.y += pa.y; a.z += pa.z; a.w += pa.w;
        bq.x += pb.x; bq.y += pb.y; bq.z += pb.z; bq.w += pb.w;
    }
    float4 w4;
    w4.x = bet * (vv.x - alpha * a.x);
    w4.y = bet * (vv.y - alpha * a.y);
    w4.z = bet * (vv.z - alpha * a.z);
    w4.w = bet * (vv.w - alpha * a.w);
    if (warp == 0) {
        float4 ov;
        ov.x = fmaf(alpha, bq.x, kq * w4.x);
        ov.y = fmaf(alpha, bq.y, kq * w4.y);
        ov.z = fmaf(alpha, bq.z, kq * w4.z);
        ov.w = fmaf(alpha, bq.w, kq * w4.w);
        io_store4(o + v_off, ov);
    }
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = warp + kWarps * i;
        const float kr = s_k[r];
        float4 n;
        n.x = fmaf(alpha, s[i].x, kr * w4.x);
        n.y = fmaf(alpha, s[i].y, kr * w4.y);
        n.z = fmaf(alpha, s[i].z, kr * w4.z);
        n.w = fmaf(alpha, s[i].w, kr * w4.w);
        __stcs(reinterpret_cast<float4*>(Sg + (size_t)r * kD) + lane, n);
    }
}

// M tokens per (sequence b, value head h) in one pass over the state (speculative
// verification of drafted tokens).  Same thread layout as decode_step_kernel:
// the state is read once into registers, then token j = 0 .. M-1 is applied
// to it in order, writing o for that token and the state after it to
// S_steps[b, j].  The k/q staging and the cross-warp partial sums are double-
// buffered by token parity, so each token needs the same two barriers as a
// single step.  Layouts: q, k [B, M, H_qk, 128]; v, o [B, M, H_v, 128];
// gates [B, M, H_v]; S_in [B, H_v, 128, 128]; S_steps [B, M, H_v, 128, 128].
template <typename IO>
__global__ void __launch_bounds__(kThreads, 2)
    decode_multi_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                        const IO* __restrict__ v, const float* __restrict__ log_alpha,
                        const float* __restrict__ beta, const float* __restrict__ S_in,
                        float* __restrict__ S_steps, int M, int H_qk, int H_v,
                        IO* __restrict__ o) {
    __shared__ float s_k[2][kD];
    __shared__ float s_q[2][kD];
    __shared__ float4 s_part[2][2][kWarps][32];  // [token parity][S^T k, S^T q][warp][lane]

    const int unit = blockIdx.x;  // b * H_v + h
    const int b = unit / H_v;
    const int h = unit - b * H_v;
    const int hq = h / (H_v / H_qk);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    const float* Sg = S_in + (size_t)unit * (kD * kD);
    float4 s[kRowsPerThread];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i)
        s[i] = __ldcs(reinterpret_cast<const float4*>(Sg + (size_t)(warp + kWarps * i) * kD) +
                      lane);

    for (int j = 0; j < M; ++j) {
        const int par = j & 1;
        const size_t tok = (size_t)b * M + j;  // token row of the [B, M, ...] layouts
        const size_t qk_off = (tok * H_qk + hq) * kD;
        if (tid < kD)
            s_k[par][tid] = io_load(k + qk_off + tid);
        else
            s_q[par][tid - kD] = io_load(q + qk_off + (tid - kD));
        const size_t gi = tok * H_v + h;
        const float alpha = expf(log_alpha[gi]);
        const float bet = beta[gi];
        const size_t v_off = gi * kD + 4 * lane;
        float4 vv;
        vv.x = io_load(v + v_off + 0);
        vv.y = io_load(v + v_off + 1);
        vv.z = io_load(v + v_off + 2);
        vv.w = io_load(v + v_off + 3);
        __syncthreads();

        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), bq = a;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
            const int r = warp + kWarps * i;
            const float kr = s_k[par][r], qr = s_q[par][r];
            a.x = fmaf(s[i].x, kr, a.x); a.y = fmaf(s[i].y, kr, a.y);
            a.z = fmaf(s[i].z, kr, a.z); a.w = fmaf(s[i].w, kr, a.w);
            bq.x = fmaf(s[i].x, qr, bq.x); bq.y = fmaf(s[i].y, qr, bq.y);
            bq.z = fmaf(s[i].z, qr, bq.z); bq.w = fmaf(s[i].w, qr, bq.w);
        }
        s_part[par][0][warp][lane] = a;
        s_part[par][1][warp][lane] = bq;
        float kq = 0.f;
#pragma unroll
        for (int i = 0; i < kD / 32; ++i)
            kq = fmaf(s_k[par][lane + 32 * i], s_q[par][lane + 32 * i], kq);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        __syncthreads();

        a = make_float4(0.f, 0.f, 0.f, 0.f);
        bq = a;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float4 pa = s_part[par][0][w][lane], pb = s_part[par][1][w][lane];
            a.x += pa.x; a.y += pa.y; a.z += pa.z; a.w += pa.w;
            bq.x += pb.x; bq.y += pb.y; bq.z += pb.z; bq.w += pb.w;
        }
        float4 w4;
        w4.x = bet * (vv.x - alpha * a.x);
        w4.y = bet * (vv.y - alpha * a.y);
        w4.z = bet * (vv.z - alpha * a.z);
        w4.w = bet * (vv.w - alpha * a.w);
        if (warp == 0) {
            float4 ov;
            ov.x = fmaf(alpha, bq.x, kq * w4.x);
            ov.y = fmaf(alpha, bq.y, kq * w4.y);
            ov.z = fmaf(alpha, bq.z, kq * w4.z);
            ov.w = fmaf(alpha, bq.w, kq * w4.w);
            io_store4(o + v_off, ov);
        }
        float* Sj = S_steps + (tok * H_v + h) * (size_t)(kD * kD);
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
            const int r = warp + kWarps * i;
            const float kr = s_k[par][r];
            s[i].x = fmaf(alpha, s[i].x, kr * w4.x);
            s[i].y = fmaf(alpha, s[i].y, kr * w4.y);
            s[i].z = fmaf(alpha, s[i].z, kr * w4.z);
            s[i].w = fmaf(alpha, s[i].w, kr * w4.w);
            __stcs(reinterpret_cast<float4*>(Sj + (size_t)r * kD) + lane, s[i]);
        }
    }
}

}  // namespace

cudaError_t launch_decode_multi(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta, const float* S_in,
                                float* S_steps, int B, int M, int H_qk, int H_v, bool bf16,
                                void* o, cudaStream_t stream) {
    const long long units = (long long)B * H_v;
    if (units == 0) return cudaSuccess;
    if (M == 1 && S_in == S_steps)  // one token in place: the single-step kernel
        return launch_decode_step(q, k, v, log_alpha, beta, S_steps, B, H_qk, H_v, bf16, o,
                                  stream);
    dim3 grid((unsigned)units), block(kThreads);
    if (bf16)
        decode_multi_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
            static_cast<const __nv_bfloat16*>(v), log_alpha, beta, S_in, S_steps, M, H_qk, H_v,
            static_cast<__nv_bfloat16*>(o));
    else
        decode_multi_kernel<float><<<grid, block, 0, stream>>>(
            static_cast<const float*>(q), static_cast<const float*>(k),
            static_cast<const float*>(v), log_alpha, beta, S_in, S_steps, M, H_qk, H_v,
            static_cast<float*>(o));
    return cudaGetLastError();
}

cudaError_t launch_decode_step(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta, float* S, int B,
                               int H_qk, int H_v, bool bf16, void* o, cudaStream_t stream) {
    const long long units = (long long)B * H_v;
    if (units == 0) return cudaSuccess;
    dim3 grid((unsigned)units), block(kThreads);
    if (bf16)
        decode_step_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
            static_cast<const __nv_bfloat16*>(v), log_alpha, beta, S, H_qk, H_v,
            static_cast<__nv_bfloat16*>(o));
    else
        decode_step_kernel<float><<<grid, block, 0, stream>>>(
            static_cast<const float*>(q), static_cast<const float*>(k),
            static_cast<const float*>(v), log_alpha, beta, S, H_qk, H_v, static_cast<float*>(o));
    return cudaGetLastError();
}

}  // namespace gdn
