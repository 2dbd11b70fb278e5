// gdn_api.cu -- the C ABI of libgdn.so (declared in include/gdn.h).
//
// Host-side argument validation, capability check, dispatch to the kernel
// launchers, and the device status word.  Every argument error is detected
// here, before any CUDA call, so invalid calls neither launch nor touch
// outputs (and can be tested on a machine without a GPU).
#include <cuda_runtime.h>

#include "../../include/gdn.h"
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

__device__ unsigned int g_status = 0u;

cudaError_t read_and_clear_status(unsigned int* status, cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbolAsync(status, g_status, sizeof(unsigned int), 0,
                                  cudaMemcpyDeviceToHost, stream);
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0u;
    e = cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(unsigned int), 0,
                                cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(stream);
}

// Waits (bounded) on an mbarrier that nothing arrives at: the wait gives up,
// records the timeout in the status word, and every thread returns.
__global__ void selftest_bounded_wait_kernel() {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    mbar_wait(&bar, 0, &abort_flag);
    __syncthreads();
}

}  // namespace gdn

namespace {

constexpr int kHeadDim = 128;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 0 = OK, otherwise a gdn_status.
gdn_status check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return GDN_ERR_CUDA;
    if (major != 10 || minor != 0) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

gdn_status check_heads(int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv, gdn_dtype dt) {
    if (H_qk <= 0 || H_v <= 0 || H_v % H_qk != 0) return GDN_ERR_INVALID_ARG;
    if (dt != GDN_BF16 && dt != GDN_F32) return GDN_ERR_INVALID_ARG;
    if (dk != kHeadDim || dv != kHeadDim) return GDN_ERR_UNSUPPORTED;
    return GDN_OK;
}

}  // namespace

extern "C" {

const char* gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE";
    }
    return "GDN_ERR_UNKNOWN";
}

int32_t gdn_version(void) { return 100; }

int32_t gdn_prefill_auto_segments(int32_t N, int32_t T, int32_t H_qk, int32_t H_v) {
    if (N <= 0 || T < 0 || H_qk <= 0 || H_v <= 0 || H_v % H_qk != 0) return 1;
    return gdn::choose_segments(N, T, H_v, gdn::device_sms());
}

size_t gdn_prefill_segmented_workspace_size(int32_t N, int32_t T, int32_t H_qk, int32_t H_v,
                                            int32_t dk, int32_t dv, gdn_dtype io_dtype,
                                            int32_t segments) {
    if (N <= 0 || T < 0 || segments < 0 || segments > GDN_MAX_PREFILL_SEGMENTS ||
        check_heads(H_qk, H_v, dk, dv, io_dtype) != GDN_OK)
        return 0;
    if ((long long)N * (segments > 0 ? segments : 1) >= (1ll << 30)) return 0;
    const int P = segments > 0 ? segments : gdn_prefill_auto_segments(N, T, H_qk, H_v);
    return gdn::prefill_workspace_bytes(N, T, H_qk, H_v, io_dtype == GDN_BF16, P);
}

size_t gdn_prefill_workspace_size(int32_t N, int32_t T, int32_t H_qk, int32_t H_v, int32_t dk,
                                  int32_t dv, gdn_dtype io_dtype) {
    return gdn_prefill_segmented_workspace_size(N, T, H_qk, H_v, dk, dv, io_dtype, 0);
}

}  // extern "C"

namespace {

// Every host-side check of a prefill call except the workspace.
gdn_status check_prefill_args(const void* q, const void* k, const void* v, const float* log_alpha,
                              const float* beta, const float* S0, const int32_t* cu_seqlens,
                              int32_t N, int32_t T, int32_t H_qk, int32_t H_v, int32_t dk,
                              int32_t dv, gdn_dtype io_dtype, const void* o,
                              const float* S_final) {
    gdn_status st = check_heads(H_qk, H_v, dk, dv, io_dtype);
    if (st != GDN_OK) return st;
    if (N <= 0 || T < 0) return GDN_ERR_INVALID_ARG;
    // Every element index must fit in 64-bit arithmetic and every token
    // coordinate in the int32 coordinates of the tensor maps.
    if ((long long)T * H_v * kHeadDim >= (1ll << 40)) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens || !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
    if (T > 0) {
        if (!q || !k || !v || !log_alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
            !aligned(log_alpha, 4) || !aligned(beta, 4))
            return GDN_ERR_INVALID_ARG;
    }
    if ((S0 && !aligned(S0, 16)) || (S_final && !aligned(S_final, 16))) return GDN_ERR_INVALID_ARG;
    return GDN_OK;
}

gdn_status prefill_call(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* S0, const int32_t* cu_seqlens, int32_t N,
                        int32_t T, int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                        gdn_dtype io_dtype, void* o, float* S_final, int32_t segments,
                        void* workspace, size_t workspace_bytes, int state_pass, void* stream);

}  // namespace

extern "C" {

gdn_status gdn_prefill_segmented(const void* q, const void* k, const void* v,
                                 const float* log_alpha, const float* beta, const float* S0,
                                 const int32_t* cu_seqlens, int32_t N, int32_t T, int32_t H_qk,
                                 int32_t H_v, int32_t dk, int32_t dv, gdn_dtype io_dtype, void* o,
                                 float* S_final, int32_t segments, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    return prefill_call(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v, dk, dv,
                        io_dtype, o, S_final, segments, workspace, workspace_bytes,
                        gdn::STATE_PASS_AUTO, stream);
}

gdn_status gdn_prefill_mma(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* S0, const int32_t* cu_seqlens, int32_t N,
                           int32_t T, int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                           gdn_dtype io_dtype, void* o, float* S_final, void* workspace,
                           size_t workspace_bytes, void* stream) {
    return prefill_call(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v, dk, dv,
                        io_dtype, o, S_final, 0, workspace, workspace_bytes, gdn::STATE_PASS_MMA,
                        stream);
}

gdn_status gdn_prefill_tc(const void* q, const void* k, const void* v, const float* log_alpha,
                          const float* beta, const float* S0, const int32_t* cu_seqlens, int32_t N,
                          int32_t T, int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                          gdn_dtype io_dtype, void* o, float* S_final, void* workspace,
                          size_t workspace_bytes, void* stream) {
    return prefill_call(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v, dk, dv,
                        io_dtype, o, S_final, 0, workspace, workspace_bytes, gdn::STATE_PASS_TC,
                        stream);
}

}  // extern "C"

namespace {

gdn_status backward_call(const void* q, const void* k, const void* v,
                         const float* log_alpha, const float* beta, const float* S0,
                         const int32_t* cu_seqlens, const void* dO, const float* dS_final,
                         int32_t N, int32_t T, int32_t H_qk, int32_t H_v, int32_t dk,
                         int32_t dv, gdn_dtype io_dtype, void* dq, void* dk_out,
                         void* dv_out, float* dlog_alpha, float* dbeta, float* dS0,
                         void* workspace, size_t workspace_bytes, bool recompute,
                         void* stream) {
    gdn_status st = check_prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v,
                                       dk, dv, io_dtype, dq, nullptr);
    if (st != GDN_OK) return st;
    if (T > 0) {
        const void* p16[] = {dO, dk_out, dv_out};
        for (const void* ptr : p16)
            if (!ptr || !aligned(ptr, 16)) return GDN_ERR_INVALID_ARG;
        if (!dlog_alpha || !dbeta || !aligned(dlog_alpha, 4) || !aligned(dbeta, 4))
            return GDN_ERR_INVALID_ARG;
    }
    if ((dS_final && !aligned(dS_final, 16)) || (dS0 && !aligned(dS0, 16)))
        return GDN_ERR_INVALID_ARG;
    const size_t need = gdn::prefill_backward_workspace_bytes(N, T, H_qk, H_v, io_dtype == GDN_BF16);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256)))
        return GDN_ERR_WORKSPACE;
    st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = gdn::launch_prefill_backward(q, k, v, log_alpha, beta, S0, cu_seqlens, dO,
                                                 dS_final, N, T, H_qk, H_v,
                                                 io_dtype == GDN_BF16, dq, dk_out, dv_out,
                                                 dlog_alpha, dbeta, dS0, workspace, recompute,
                                                 static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}


gdn_status prefill_call(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* S0, const int32_t* cu_seqlens, int32_t N,
                        int32_t T, int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                        gdn_dtype io_dtype, void* o, float* S_final, int32_t segments,
                        void* workspace, size_t workspace_bytes, int state_pass, void* stream) {
    gdn_status st = check_prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v,
                                       dk, dv, io_dtype, o, S_final);
    if (st != GDN_OK) return st;
    if (segments < 0 || segments > GDN_MAX_PREFILL_SEGMENTS) return GDN_ERR_INVALID_ARG;
    if ((long long)N * (segments > 0 ? segments : 1) >= (1ll << 30)) return GDN_ERR_INVALID_ARG;
    const bool bf16 = io_dtype == GDN_BF16;
    const int P = segments > 0 ? segments : gdn_prefill_auto_segments(N, T, H_qk, H_v);
    const size_t need = gdn::prefill_workspace_bytes(N, T, H_qk, H_v, bf16, P);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256)))
        return GDN_ERR_WORKSPACE;
    st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = gdn::launch_prefill(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk,
                                        H_v, bf16, o, S_final, workspace, P, state_pass,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

extern "C" {

gdn_status gdn_prefill(const void* q, const void* k, const void* v, const float* log_alpha,
                       const float* beta, const float* S0, const int32_t* cu_seqlens, int32_t N,
                       int32_t T, int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                       gdn_dtype io_dtype, void* o, float* S_final, void* workspace,
                       size_t workspace_bytes, void* stream) {
    return gdn_prefill_segmented(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v, dk,
                                 dv, io_dtype, o, S_final, 0, workspace, workspace_bytes, stream);
}

gdn_status gdn_prefill_noalloc(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta, const float* S0,
                               const int32_t* cu_seqlens, int32_t N, int32_t T, int32_t H_qk,
                               int32_t H_v, int32_t dk, int32_t dv, gdn_dtype io_dtype, void* o,
                               float* S_final, void* stream) {
    gdn_status st = check_prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v,
                                       dk, dv, io_dtype, o, S_final);
    if (st != GDN_OK) return st;
    // The scratch this call needs is the workspace gdn_prefill would take; it
    // comes from the library's fixed device array instead of the caller.  When
    // the automatic split of the sequences needs more than the array holds, the
    // unsplit prefill (one piece per sequence, the least scratch) runs instead.
    const size_t cap = gdn::noalloc_scratch_bytes();
    int32_t segments = 0;
    size_t need = gdn_prefill_workspace_size(N, T, H_qk, H_v, dk, dv, io_dtype);
    if (need > cap) {
        segments = 1;
        need = gdn_prefill_segmented_workspace_size(N, T, H_qk, H_v, dk, dv, io_dtype, 1);
        if (need > cap) return GDN_ERR_WORKSPACE;
    }
    void* scratch = nullptr;
    if (need > 0 && gdn::noalloc_scratch_address(&scratch) != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_prefill_segmented(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v, dk,
                                 dv, io_dtype, o, S_final, segments, scratch,
                                 need > 0 ? cap : 0, stream);
}

size_t gdn_prefill_noalloc_max_scratch_bytes(void) { return gdn::noalloc_scratch_bytes(); }

gdn_status gdn_decode_step(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, float* S_inout, int32_t B, int32_t H_qk,
                           int32_t H_v, int32_t dk, int32_t dv, gdn_dtype io_dtype, void* o,
                           void* stream) {
    gdn_status st = check_heads(H_qk, H_v, dk, dv, io_dtype);
    if (st != GDN_OK) return st;
    if (B < 0) return GDN_ERR_INVALID_ARG;
    if ((long long)B * H_v >= (1ll << 31)) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S_inout || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(S_inout, 16) || !aligned(log_alpha, 4) || !aligned(beta, 4))
        return GDN_ERR_INVALID_ARG;
    st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = gdn::launch_decode_step(q, k, v, log_alpha, beta, S_inout, B, H_qk, H_v,
                                            io_dtype == GDN_BF16, o,
                                            static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

size_t gdn_prefill_backward_workspace_size(int32_t N, int32_t T, int32_t H_qk, int32_t H_v,
                                           int32_t dk, int32_t dv, gdn_dtype io_dtype) {
    if (N <= 0 || T < 0 || check_heads(H_qk, H_v, dk, dv, io_dtype) != GDN_OK) return 0;
    return gdn::prefill_backward_workspace_bytes(N, T, H_qk, H_v, io_dtype == GDN_BF16);
}

gdn_status gdn_prefill_backward(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta, const float* S0,
                                const int32_t* cu_seqlens, const void* dO, const float* dS_final,
                                int32_t N, int32_t T, int32_t H_qk, int32_t H_v, int32_t dk,
                                int32_t dv, gdn_dtype io_dtype, void* dq, void* dk_out,
                                void* dv_out, float* dlog_alpha, float* dbeta, float* dS0,
                                void* workspace, size_t workspace_bytes, void* stream) {
    return backward_call(q, k, v, log_alpha, beta, S0, cu_seqlens, dO, dS_final, N, T, H_qk, H_v,
                         dk, dv, io_dtype, dq, dk_out, dv_out, dlog_alpha, dbeta, dS0, workspace,
                         workspace_bytes, true, stream);
}

gdn_status gdn_prefill_backward_saved(const void* q, const void* k, const void* v,
                                      const float* log_alpha, const float* beta, const float* S0,
                                      const int32_t* cu_seqlens, const void* dO,
                                      const float* dS_final, int32_t N, int32_t T, int32_t H_qk,
                                      int32_t H_v, int32_t dk, int32_t dv, gdn_dtype io_dtype,
                                      void* dq, void* dk_out, void* dv_out, float* dlog_alpha,
                                      float* dbeta, float* dS0, void* workspace,
                                      size_t workspace_bytes, void* stream) {
    return backward_call(q, k, v, log_alpha, beta, S0, cu_seqlens, dO, dS_final, N, T, H_qk, H_v,
                         dk, dv, io_dtype, dq, dk_out, dv_out, dlog_alpha, dbeta, dS0, workspace,
                         workspace_bytes, false, stream);
}

gdn_status gdn_prefill_train(const void* q, const void* k, const void* v, const float* log_alpha,
                             const float* beta, const float* S0, const int32_t* cu_seqlens,
                             int32_t N, int32_t T, int32_t H_qk, int32_t H_v, int32_t dk,
                             int32_t dv, gdn_dtype io_dtype, void* o, float* S_final,
                             void* workspace, size_t workspace_bytes, void* stream) {
    gdn_status st = check_prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v,
                                       dk, dv, io_dtype, o, S_final);
    if (st != GDN_OK) return st;
    const size_t need =
        gdn::prefill_backward_workspace_bytes(N, T, H_qk, H_v, io_dtype == GDN_BF16);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 256)))
        return GDN_ERR_WORKSPACE;
    st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = gdn::launch_prefill_train(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T,
                                              H_qk, H_v, io_dtype == GDN_BF16, o, S_final,
                                              workspace, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_decode_multi(const void* q, const void* k, const void* v, const float* log_alpha,
                            const float* beta, const float* S_in, int32_t B, int32_t M,
                            int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                            gdn_dtype io_dtype, void* o, float* S_steps, void* stream) {
    gdn_status st = check_heads(H_qk, H_v, dk, dv, io_dtype);
    if (st != GDN_OK) return st;
    if (B < 0 || M < 1 || M > GDN_MAX_DECODE_TOKENS) return GDN_ERR_INVALID_ARG;
    if ((long long)B * M * H_v >= (1ll << 31)) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !log_alpha || !beta || !S_in || !o || !S_steps)
        return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(S_in, 16) || !aligned(S_steps, 16) || !aligned(log_alpha, 4) ||
        !aligned(beta, 4))
        return GDN_ERR_INVALID_ARG;
    // the kernel reads S_in while other blocks write S_steps: no overlap, except
    // the in-place single step
    const uintptr_t in0 = reinterpret_cast<uintptr_t>(S_in);
    const uintptr_t in1 = in0 + (uintptr_t)B * H_v * dk * dv * sizeof(float);
    const uintptr_t out0 = reinterpret_cast<uintptr_t>(S_steps);
    const uintptr_t out1 = out0 + (uintptr_t)B * M * H_v * dk * dv * sizeof(float);
    if (in0 < out1 && out0 < in1 && !(M == 1 && in0 == out0)) return GDN_ERR_INVALID_ARG;
    st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = gdn::launch_decode_multi(q, k, v, log_alpha, beta, S_in, S_steps, B, M, H_qk,
                                             H_v, io_dtype == GDN_BF16, o,
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_frontend(const void* q_raw, const void* k_raw, const void* v_raw,
                        const float* conv_w, const float* a, const float* b,
                        const int32_t* cu_seqlens, int32_t N, int32_t T, int32_t H_qk,
                        int32_t H_v, int32_t dk, int32_t dv, gdn_dtype io_dtype,
                        gdn_activation act, float eps, void* q, void* k, void* v,
                        float* log_alpha, float* beta, void* stream) {
    gdn_status st = check_heads(H_qk, H_v, dk, dv, io_dtype);
    if (st != GDN_OK) return st;
    if (N <= 0 || T < 0 || (act != GDN_ACT_NONE && act != GDN_ACT_SILU) || !(eps >= 0.f))
        return GDN_ERR_INVALID_ARG;
    if ((long long)T * H_v * kHeadDim >= (1ll << 40)) return GDN_ERR_INVALID_ARG;
    if (!cu_seqlens || !aligned(cu_seqlens, 4)) return GDN_ERR_INVALID_ARG;
    if (T > 0) {
        const void* p16[] = {q_raw, k_raw, v_raw, conv_w, q, k, v};
        for (const void* ptr : p16)
            if (!ptr || !aligned(ptr, 16)) return GDN_ERR_INVALID_ARG;
        const void* p4[] = {a, b, log_alpha, beta};
        for (const void* ptr : p4)
            if (!ptr || !aligned(ptr, 4)) return GDN_ERR_INVALID_ARG;
    }
    st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = gdn::launch_frontend(q_raw, k_raw, v_raw, conv_w, a, b, cu_seqlens, N, T, H_qk,
                                         H_v, io_dtype == GDN_BF16, (int)act, eps, q, k, v,
                                         log_alpha, beta, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_frontend_decode_step(const void* q_raw, const void* k_raw, const void* v_raw,
                                    const float* conv_w, const float* a, const float* b,
                                    void* conv_state, int32_t B, int32_t H_qk, int32_t H_v,
                                    int32_t dk, int32_t dv, gdn_dtype io_dtype,
                                    gdn_activation act, float eps, void* q, void* k, void* v,
                                    float* log_alpha, float* beta, void* stream) {
    gdn_status st = check_heads(H_qk, H_v, dk, dv, io_dtype);
    if (st != GDN_OK) return st;
    if (B < 0 || (act != GDN_ACT_NONE && act != GDN_ACT_SILU) || !(eps >= 0.f))
        return GDN_ERR_INVALID_ARG;
    if ((long long)B * (2 * H_qk + H_v) >= (1ll << 31)) return GDN_ERR_INVALID_ARG;
    if (B == 0) return GDN_OK;
    const void* p16[] = {q_raw, k_raw, v_raw, conv_w, conv_state, q, k, v};
    for (const void* ptr : p16)
        if (!ptr || !aligned(ptr, 16)) return GDN_ERR_INVALID_ARG;
    const void* p4[] = {a, b, log_alpha, beta};
    for (const void* ptr : p4)
        if (!ptr || !aligned(ptr, 4)) return GDN_ERR_INVALID_ARG;
    st = check_device();
    if (st != GDN_OK) return st;
    cudaError_t e = gdn::launch_frontend_decode(q_raw, k_raw, v_raw, conv_w, a, b, conv_state, B,
                                                H_qk, H_v, io_dtype == GDN_BF16, (int)act, eps,
                                                q, k, v, log_alpha, beta,
                                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_selftest_bounded_wait(void* stream) {
    gdn_status st = check_device();
    if (st != GDN_OK) return st;
    gdn::selftest_bounded_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>();
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

gdn_status gdn_get_last_device_error(void* stream) {
    unsigned int status = 0u;
    if (gdn::read_and_clear_status(&status, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return GDN_ERR_CUDA;
    return status == GDN_DEV_OK ? GDN_OK : GDN_ERR_TIMEOUT;
}

}  // extern "C"
