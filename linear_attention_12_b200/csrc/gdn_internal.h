// gdn_internal.h -- launchers behind the C ABI (not part of the public header).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn {

cudaError_t launch_decode_step(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta, float* S, int B,
                               int H_qk, int H_v, bool bf16, void* o, cudaStream_t stream);
cudaError_t launch_decode_multi(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta, const float* S_in,
                                float* S_steps, int B, int M, int H_qk, int H_v, bool bf16,
                                void* o, cudaStream_t stream);

// Workspace bytes the prefill needs with P segments per sequence (fp32 I/O
// also stages bf16 copies of q, k, v).
size_t prefill_workspace_bytes(int N, int T, int H_qk, int H_v, bool bf16, int P);

// SM count of the current device (148 when there is none).
int device_sms();

// Segments per sequence the prefill uses when the caller leaves it to the
// library: 1 unless splitting the sequences fills more of the SMs.
int choose_segments(int N, int T, int H_v, int sms);

// Which implementation runs the state pass that writes the prefill's outputs.
constexpr int STATE_PASS_AUTO = 0;  // the faster one for the slice width
constexpr int STATE_PASS_TC = 1;    // tcgen05, accumulators in tensor memory
constexpr int STATE_PASS_MMA = 2;   // warp-level mma.sync, accumulators in registers

// P segments per sequence (P <= 0: choose_segments).
cudaError_t launch_prefill(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* S0, const int32_t* cu_seqlens, int N,
                           int T, int H_qk, int H_v, bool bf16, void* o, float* S_final,
                           void* workspace, int P, int state_pass, cudaStream_t stream);

// Records and chunk-entering states (bf16 images) of a prefill with bf16
// q, k, v, for its gradients; with o non-null also its outputs (bf16 or fp32)
// and final states.
cudaError_t launch_prefill_save(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta, const float* S0,
                                const int32_t* cu_seqlens, int N, int T, int H_qk, int H_v,
                                uint8_t* records, uint8_t* S_saved, void* o, float* S_final,
                                bool out_bf16, cudaStream_t stream);
size_t prefill_record_bytes(int N, int T, int H_v);

// Gradients of a bf16 prefill: workspace bytes, and the launches (the forward
// pass saving every chunk's state, the reverse chain, the per-chunk gradients).
size_t prefill_backward_workspace_bytes(int N, int T, int H_qk, int H_v, bool bf16);
cudaError_t launch_prefill_backward(const void* q, const void* k, const void* v,
                                    const float* log_alpha, const float* beta, const float* S0,
                                    const int32_t* cu_seqlens, const void* dO,
                                    const float* dS_final, int N, int T, int H_qk, int H_v,
                                    bool bf16, void* dq, void* dk, void* dv, float* dlog_alpha,
                                    float* dbeta, float* dS0, void* workspace, bool recompute,
                                    cudaStream_t stream);
// The prefill (outputs, final states) that also leaves in `workspace` (laid
// out as launch_prefill_backward's) the records and entering states its
// gradients read; launch_prefill_backward with recompute = false then skips
// the forward re-run.
cudaError_t launch_prefill_train(const void* q, const void* k, const void* v,
                                 const float* log_alpha, const float* beta, const float* S0,
                                 const int32_t* cu_seqlens, int N, int T, int H_qk, int H_v,
                                 bool bf16, void* o, float* S_final, void* workspace,
                                 cudaStream_t stream);

cudaError_t launch_frontend(const void* q_raw, const void* k_raw, const void* v_raw,
                            const float* conv_w, const float* a, const float* b,
                            const int32_t* cu_seqlens, int N, int T, int H_qk, int H_v,
                            bool bf16, int act, float eps, void* q, void* k, void* v,
                            float* log_alpha, float* beta, cudaStream_t stream);

cudaError_t launch_frontend_decode(const void* q_raw, const void* k_raw, const void* v_raw,
                                   const float* conv_w, const float* a, const float* b,
                                   void* conv_state, int B, int H_qk, int H_v, bool bf16, int act,
                                   float eps, void* q, void* k, void* v, float* log_alpha,
                                   float* beta, cudaStream_t stream);

cudaError_t read_and_clear_status(unsigned int* status, cudaStream_t stream);

// Fixed-size device scratch used by gdn_prefill_noalloc (bytes, and its address
// on the current device; the address is looked up once per device).
size_t noalloc_scratch_bytes();
cudaError_t noalloc_scratch_address(void** out);

}  // namespace gdn
