/*
 * gdn.h -- C ABI of libgdn.so, a B200 (sm_100a) implementation of the Gated
 * DeltaNet (GDN) token mixer.
 *
 * The operation (bjdmk.com.cn article "为什么 Qwen3.8-Flash-Next 值得单独跑一遍",
 * section 2.1 "Gated DeltaNet 负责廉价压缩历史", state-update formula):
 *
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t            (post-update state, no scale factor)
 *
 * S_t is a d_k x d_v fp32 matrix per (sequence, value head); alpha_t =
 * exp(log_alpha[t,h]) is the forget gate and beta_t = beta[t,h] the write
 * strength, one scalar each per (token, value head).  H_v value heads share
 * H_qk query/key heads: value head h reads q/k head h / (H_v / H_qk)
 * (section 2.1 of the same article and the jianying88.com article
 * "Qwen3.8-Flash-Next混合注意力深度解析", section 三: 48 V heads, 16 QK heads,
 * head dim 128).  The readout is not printed on the pages; o_t = S_t^T q_t
 * is the reading this library implements.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory and keeps no per-call state.  The only
 *     library-global state is a per-device status word in a static
 *     __device__ variable (see gdn_get_last_device_error).
 *   - Layouts are dense, row-major, packed token-major ("varlen" packing):
 *       q, k      [T, H_qk, dk]      io_dtype
 *       v, o      [T, H_v,  dv]      io_dtype
 *       log_alpha [T, H_v]           fp32  (log of the forget gate, <= 0 in normal use)
 *       beta      [T, H_v]           fp32
 *       S0/S_final/S_inout [N, H_v, dk, dv] fp32 (row i = key dim, column j = value dim)
 *   - dk = dv = 128 is the only supported head size; H_v % H_qk == 0.
 *   - q, k, v, o and the state pointers must be 16-byte aligned; log_alpha,
 *     beta and cu_seqlens 4-byte aligned; the workspace 256-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and return GDN_OK once the work is
 *     enqueued.  Argument errors are detected on the host before anything is
 *     launched and leave every output untouched.
 *   - Inputs are used as given: no normalisation of q/k, no gate activation,
 *     no scaling.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, H_v % H_qk != 0, ... */
    GDN_ERR_UNSUPPORTED = 2,  /* dk/dv != 128, or the device is not compute capability 10.0 */
    GDN_ERR_CUDA = 3,         /* a CUDA runtime/driver call or a kernel launch failed */
    GDN_ERR_TIMEOUT = 4,      /* a device-side bounded wait gave up (see gdn_get_last_device_error) */
    GDN_ERR_WORKSPACE = 5     /* workspace pointer/size too small for this call */
} gdn_status;

typedef enum {
    GDN_BF16 = 1,  /* q, k, v and o are bfloat16 */
    GDN_F32 = 2    /* q, k, v and o are float32 (computed through bf16 tensor-core operands) */
} gdn_dtype;

typedef enum {
    GDN_ACT_NONE = 0,  /* no activation after the short convolution */
    GDN_ACT_SILU = 1   /* y * sigmoid(y) after the short convolution */
} gdn_activation;

/*
 * gdn_prefill -- run the recurrence over N packed sequences (chunked prefill).
 *
 *   q, k, v, log_alpha, beta : inputs, layouts above, T tokens in total.
 *   S0        : initial state per (sequence, value head), or NULL for zeros.
 *   cu_seqlens: device int32 [N+1], cu[0] = 0, non-decreasing, cu[N] = T;
 *               sequence n is tokens [cu[n], cu[n+1]).  Its contents are not
 *               read on the host; malformed contents are undefined behaviour.
 *               Zero-length sequences are allowed (their S_final = S0).
 *   o         : output [T, H_v, dv] in io_dtype (every row is written).
 *   S_final   : final state per (sequence, value head), or NULL to skip it.
 *               May alias S0 exactly (in-place state update); no other overlap
 *               between outputs and inputs is allowed.
 *   workspace : device scratch of at least gdn_prefill_workspace_size(...)
 *               bytes (may be NULL when that size is 0), owned by the caller
 *               and not used after the work on `stream` completes.  It holds
 *               one 16,912-byte "chunk operator" record per (chunk slot, value
 *               head) -- N + ceil(T / 64) slots; about 416 MB for T = 32,768
 *               and 48 value heads -- written by the first of the two passes
 *               of the prefill and read by the second, plus bf16 copies of
 *               q, k, v when io_dtype is GDN_F32.  When few sequences x value
 *               heads would leave SMs idle, gdn_prefill splits the sequences
 *               (gdn_prefill_segmented with segments = 0) and the workspace
 *               also holds that split's states.
 *
 * Arithmetic: tensor-core products with 16-bit operands and fp32 accumulators;
 * the state is carried in fp32.  The state S and d o Delta enter the products
 * as bf16 (they meet the bf16 K and Q tiles).  Unless the sequences are split,
 * the chunk operators T diag(beta) and M o Q K^T and the intermediates
 * X = V - diag(gamma) K S and Delta enter as fp16 (11 significant bits); their
 * entries must stay below 65,504 in magnitude, which unit-norm q, k and
 * unit-scale v satisfy.  The split prefill keeps them in bf16.
 *
 * Returns GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE
 * or GDN_ERR_CUDA.
 */
GDN_API gdn_status gdn_prefill(const void *q, const void *k, const void *v,
                       const float *log_alpha, const float *beta,
                       const float *S0, const int32_t *cu_seqlens,
                       int32_t N, int32_t T, int32_t H_qk, int32_t H_v,
                       int32_t dk, int32_t dv, gdn_dtype io_dtype,
                       void *o, float *S_final,
                       void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of device workspace gdn_prefill needs for these sizes (0 when T == 0
 * or the arguments are invalid).  Includes what the automatic sequence split
 * (gdn_prefill_segmented) needs on the current device. */
GDN_API size_t gdn_prefill_workspace_size(int32_t N, int32_t T, int32_t H_qk, int32_t H_v,
                                  int32_t dk, int32_t dv, gdn_dtype io_dtype);

/* Most segments per sequence gdn_prefill_segmented takes. */
#define GDN_MAX_PREFILL_SEGMENTS 64

/*
 * gdn_prefill_segmented -- gdn_prefill with each sequence split into `segments`
 * pieces that run side by side on one GPU (sequence parallelism within the
 * card, for inputs with too few sequences x value heads to fill the SMs: long
 * contexts, or the few heads a tensor-parallel shard holds).
 *
 * The Qwen3.8-Flash-Next article of alwayszhang ("GDN+QSA、门控残差与 N-gram
 * Embedding…", section 九) names intra-card context parallelism among the
 * FlashQLA kernel techniques and gives no formulas.  The split done here is
 * exact, not a truncation of the decay:
 *   1. The state after a segment is affine in the state before it,
 *      S_end = P_s S_start + R_s.
 *   2. Every segment runs twice side by side: from S = 0, which gives R_s, and
 *      from S = I with v = 0, which gives the d_k x d_k propagator P_s.
 *   3. A scan over the segments gives each entering state.
 *   4. Every segment then runs again from that state and writes its outputs.
 * Segments are whole 64-token chunks: sequence n is cut into `segments`
 * pieces of ceil(ceil(len_n / 64) / segments) chunks, and trailing pieces may
 * be empty.  The cost is about 2.5 times the state-carrying work, spread over
 * `segments` times more blocks; it pays when those blocks would otherwise
 * leave SMs idle.
 *
 *   segments : 0 = choose automatically (what gdn_prefill does; see
 *              gdn_prefill_auto_segments), 1 = no split, 2 ..
 *              GDN_MAX_PREFILL_SEGMENTS = that many pieces per sequence.
 *   workspace: at least gdn_prefill_segmented_workspace_size(..., segments)
 *              bytes, 256-byte aligned.  A split adds (N x segments) record
 *              slots, N x segments + 1 int32 segment starts and three
 *              fp32 states per (piece, value head).
 * Other arguments, results and errors as gdn_prefill; GDN_ERR_INVALID_ARG also
 * for `segments` out of range.
 */
GDN_API gdn_status gdn_prefill_segmented(const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta,
                                 const float *S0, const int32_t *cu_seqlens,
                                 int32_t N, int32_t T, int32_t H_qk, int32_t H_v,
                                 int32_t dk, int32_t dv, gdn_dtype io_dtype,
                                 void *o, float *S_final, int32_t segments,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_prefill_tc / gdn_prefill_mma -- gdn_prefill with the implementation of
 * the state pass that writes the outputs fixed.
 *
 * There are two, of the same chunk form of the bjdmk.com.cn article's
 * recurrence, section 2.1:
 *   - gdn_prefill_tc: the fifth-generation tensor cores (tcgen05.mma,
 *     accumulators in tensor memory);
 *   - gdn_prefill_mma: warp-level mma.sync with the state in registers.
 *
 * gdn_prefill picks per d_v slice width.  It takes tcgen05 for the 48-column
 * slices it uses at 38-49 (sequence, value head) units, e.g. 16/48 heads and
 * one sequence: 1.31-1.32 against 1.32-1.34 ms at 32,768 tokens.  It takes
 * mma.sync otherwise (at 32-column slices mma.sync measured faster).
 *
 * Same arguments, layouts, workspace (gdn_prefill_workspace_size), results
 * within rounding, and errors as gdn_prefill; the automatic segment choice
 * applies as there.
 */
GDN_API gdn_status gdn_prefill_tc(const void *q, const void *k, const void *v,
                                  const float *log_alpha, const float *beta, const float *S0,
                                  const int32_t *cu_seqlens, int32_t N, int32_t T, int32_t H_qk,
                                  int32_t H_v, int32_t dk, int32_t dv, gdn_dtype io_dtype,
                                  void *o, float *S_final, void *workspace,
                                  size_t workspace_bytes, void *stream);
GDN_API gdn_status gdn_prefill_mma(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta, const float *S0,
                                   const int32_t *cu_seqlens, int32_t N, int32_t T, int32_t H_qk,
                                   int32_t H_v, int32_t dk, int32_t dv, gdn_dtype io_dtype,
                                   void *o, float *S_final, void *workspace,
                                   size_t workspace_bytes, void *stream);

/* Workspace bytes of gdn_prefill_segmented with these arguments (0 when T == 0
 * or the arguments are invalid). */
GDN_API size_t gdn_prefill_segmented_workspace_size(int32_t N, int32_t T, int32_t H_qk,
                                            int32_t H_v, int32_t dk, int32_t dv,
                                            gdn_dtype io_dtype, int32_t segments);

/* Segments per sequence gdn_prefill uses for these sizes on the current device:
 * 1 unless a split fills more SMs (a cost model over the SM count, the
 * sequences x value heads and the average sequence length; pieces of at least
 * 8 chunks, at most 16 pieces).  Returns 1 for invalid arguments. */
GDN_API int32_t gdn_prefill_auto_segments(int32_t N, int32_t T, int32_t H_qk, int32_t H_v);

/*
 * gdn_prefill_noalloc -- gdn_prefill for callers that cannot allocate device
 * memory.  (No counterpart in the paper: this is an interface convenience.)
 *
 * Some callers can't call cudaMalloc: plug-ins run inside a server or framework
 * that owns all device memory through its own pool and hands each operator only
 * its input and output tensors, or latency-critical loops where an allocation
 * (which may synchronise the device or fail on a fragmented heap) is not
 * allowed.  This entry point takes the same arguments as gdn_prefill minus the
 * workspace and allocates nothing: the scratch it needs (what
 * gdn_prefill_workspace_size reports for the same sizes: the chunk-operator
 * records, 16,912 bytes per chunk and value head, plus bf16 copies of fp32
 * q, k, v) lives in a fixed device array inside the library, of
 * gdn_prefill_noalloc_max_scratch_bytes() bytes (16 MiB), which every GPU that
 * loads the library holds until the process exits.  When the automatic split
 * of long sequences (gdn_prefill_auto_segments) would need more scratch than
 * that, the call runs the prefill unsplit (gdn_prefill_segmented with
 * segments = 1, the least scratch; same results, fewer SMs busy).  Calls whose
 * scratch would still exceed the array return GDN_ERR_WORKSPACE and launch
 * nothing; use gdn_prefill with a caller-owned workspace instead.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  All calls share the one array, which keeps the
 * last call's contents: calls that may overlap on the GPU (different streams
 * without ordering between them) race on it.  Results and errors are otherwise
 * those of gdn_prefill.
 */
GDN_API gdn_status gdn_prefill_noalloc(const void *q, const void *k, const void *v,
                               const float *log_alpha, const float *beta,
                               const float *S0, const int32_t *cu_seqlens,
                               int32_t N, int32_t T, int32_t H_qk, int32_t H_v,
                               int32_t dk, int32_t dv, gdn_dtype io_dtype,
                               void *o, float *S_final, void *stream);

/* Size in bytes of the fixed scratch array behind gdn_prefill_noalloc. */
GDN_API size_t gdn_prefill_noalloc_max_scratch_bytes(void);

/*
 * gdn_decode_step -- advance B independent sequences by one token each.
 *
 *   q, k [B, H_qk, dk], v [B, H_v, dv] (io_dtype); log_alpha, beta [B, H_v] fp32.
 *   S_inout [B, H_v, dk, dv] fp32: read, then overwritten in place with S_t.
 *   o [B, H_v, dv] (io_dtype): o = S_t^T q_t.
 *
 * One pass over the state: the kernel reads each 64 KiB state once, forms
 * S^T k and S^T q, and writes the updated state once.
 * Returns GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED or GDN_ERR_CUDA.
 */
GDN_API gdn_status gdn_decode_step(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           float *S_inout, int32_t B, int32_t H_qk, int32_t H_v,
                           int32_t dk, int32_t dv, gdn_dtype io_dtype,
                           void *o, void *stream);

/*
 * gdn_prefill_backward -- gradients of gdn_prefill for training.
 *
 * The Qwen3.8-Flash-Next article of alwayszhang (section 九) lists a chunked
 * prefill backward among the FlashQLA kernels and prints nothing about it.
 * This computes the gradients of
 *
 *     L = <dO, o> + <dS_final, S_final>
 *
 * by the chain rule of the state-update formula (bjdmk.com.cn article, section
 * 2.1), taken through the chunk form of the forward kernels:
 *   1. It reruns the forward pass, saving the state entering every chunk.
 *   2. It carries the state gradient backwards through the chunks (one block
 *      per sequence, value head and d_v slice).
 *   3. It computes every chunk's gradients in parallel.
 *
 *   q, k, v, log_alpha, beta, S0, cu_seqlens: the prefill's inputs, as for
 *              gdn_prefill (S0 may be NULL).
 *   dO       : [T, H_v, dv] in io_dtype, the gradient of o.
 *   dS_final : [N, H_v, dk, dv] fp32, the gradient of S_final, or NULL for zero.
 *   dq, dk   : [T, H_qk, dk] in io_dtype (written; the value heads of a
 *              query/key head are summed).
 *   dv       : [T, H_v, dv] in io_dtype (written).
 *   dlog_alpha, dbeta: [T, H_v] fp32 (written).
 *   dS0      : [N, H_v, dk, dv] fp32 (written), or NULL to skip it.
 *   workspace: at least gdn_prefill_backward_workspace_size(...) bytes,
 *              256-byte aligned.  It holds the chunk-operator records and two
 *              bf16 states per (chunk slot, value head) -- the state entering
 *              the chunk and the gradient of the state after it, each a 32 KB
 *              128B-swizzled tile image: about 2.0 GB for T = 32,768 and 48
 *              value heads.  For GDN_F32 it also
 *              holds bf16 copies of q, k, v and dO (the products read bf16
 *              operands, as in the forward pass).
 * Returns GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE
 * or GDN_ERR_CUDA.
 */
GDN_API gdn_status gdn_prefill_backward(const void *q, const void *k, const void *v,
                                const float *log_alpha, const float *beta,
                                const float *S0, const int32_t *cu_seqlens,
                                const void *dO, const float *dS_final,
                                int32_t N, int32_t T, int32_t H_qk, int32_t H_v,
                                int32_t dk, int32_t dv, gdn_dtype io_dtype,
                                void *dq, void *dk_out, void *dv_out,
                                float *dlog_alpha, float *dbeta, float *dS0,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_prefill_train -- gdn_prefill for a training step: the same outputs o
 * and S_final (same arguments, layouts and errors; no sequence split), and in
 * `workspace` -- at least gdn_prefill_backward_workspace_size(...) bytes,
 * 256-byte aligned, owned by the caller -- the chunk-operator records and
 * every chunk's entering state that the gradients read.  Pass the same
 * inputs and the untouched workspace to gdn_prefill_backward_saved, which
 * then skips re-running the forward pass.
 */
GDN_API gdn_status gdn_prefill_train(const void *q, const void *k, const void *v,
                                     const float *log_alpha, const float *beta, const float *S0,
                                     const int32_t *cu_seqlens, int32_t N, int32_t T,
                                     int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                                     gdn_dtype io_dtype, void *o, float *S_final,
                                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdn_prefill_backward_saved -- gdn_prefill_backward (same arguments, outputs
 * and errors) reading the records and entering states that gdn_prefill_train
 * left in `workspace` for the same q, k, v, gates, S0 and cu_seqlens, instead
 * of recomputing them.  Behaviour is undefined if the workspace was not filled
 * that way (the library cannot tell).
 */
GDN_API gdn_status gdn_prefill_backward_saved(
    const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
    const float *S0, const int32_t *cu_seqlens, const void *dO, const float *dS_final, int32_t N,
    int32_t T, int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv, gdn_dtype io_dtype, void *dq,
    void *dk_out, void *dv_out, float *dlog_alpha, float *dbeta, float *dS0, void *workspace,
    size_t workspace_bytes, void *stream);

/* Workspace bytes of gdn_prefill_backward (0 when T == 0 or the arguments are
 * invalid). */
GDN_API size_t gdn_prefill_backward_workspace_size(int32_t N, int32_t T, int32_t H_qk,
                                           int32_t H_v, int32_t dk, int32_t dv,
                                           gdn_dtype io_dtype);

/* Most tokens per sequence that one gdn_decode_multi call takes. */
#define GDN_MAX_DECODE_TOKENS 8

/*
 * gdn_decode_multi -- advance B independent sequences by M tokens each, keeping
 * the state after every token (speculative verification of drafted tokens).
 *
 * Defined by the same state-update formula as gdn_decode_step (bjdmk.com.cn
 * article "为什么 Qwen3.8-Flash-Next 值得单独跑一遍", section 2.1), applied to the
 * M tokens of each sequence in order; the pages' multi-token prediction runs
 * with num_speculative_tokens = 3, i.e. M = 4 tokens per verification step.
 *
 *   q, k [B, M, H_qk, dk], v [B, M, H_v, dv] (io_dtype), token-major within a
 *     sequence; log_alpha, beta [B, M, H_v] fp32.
 *   S_in [B, H_v, dk, dv] fp32: the state before the first token (read only).
 *   o [B, M, H_v, dv] (io_dtype): o[b, j] = S_{b,j}^T q[b, j].
 *   S_steps [B, M, H_v, dk, dv] fp32 (written): S_steps[b, j] is the state after
 *     token j -- the state to continue from when the first j + 1 tokens are
 *     accepted.
 *
 * 1 <= M <= GDN_MAX_DECODE_TOKENS.  S_steps must not overlap S_in, except that
 * M == 1 with S_steps == S_in updates the state in place (gdn_decode_step).
 * One pass over the state: each 64 KiB state is read once and written M times.
 * The caller owns every buffer.
 * Returns GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED or GDN_ERR_CUDA.
 */
GDN_API gdn_status gdn_decode_multi(const void *q, const void *k, const void *v,
                            const float *log_alpha, const float *beta,
                            const float *S_in, int32_t B, int32_t M, int32_t H_qk,
                            int32_t H_v, int32_t dk, int32_t dv, gdn_dtype io_dtype,
                            void *o, float *S_steps, void *stream);

/*
 * gdn_get_last_device_error -- synchronise `stream`, then read and clear the
 * current device's status word.  Returns GDN_ERR_TIMEOUT if a kernel gave up
 * on a bounded wait since the last call, GDN_ERR_CUDA if the synchronisation
 * failed, GDN_OK otherwise.
 */
GDN_API gdn_status gdn_get_last_device_error(void *stream);

/*
 * gdn_selftest_bounded_wait -- exercise the library's failure detection on
 * the device.  (No counterpart in the paper: a test hook for the bounded
 * waits every kernel of the library uses.)
 *
 * Enqueues on `stream` one small kernel whose threads wait, through the same
 * bounded mbarrier wait the prefill kernels use, on a barrier that nothing
 * ever arrives at.  The wait gives up after its time limit (about 2 s),
 * records GDN_ERR_TIMEOUT in the device status word and the kernel returns
 * normally: no fault, no trap, and the context stays usable.  The next
 * gdn_get_last_device_error(stream) returns GDN_ERR_TIMEOUT (and clears it).
 * Returns GDN_OK once enqueued, GDN_ERR_UNSUPPORTED on a device other than
 * compute capability 10.0, GDN_ERR_CUDA if the launch failed.
 */
GDN_API gdn_status gdn_selftest_bounded_wait(void *stream);

/*
 * gdn_frontend -- the step before the recurrence: turn a layer's raw q, k, v
 * projections and gate pre-activations into gdn_prefill's inputs.
 *
 * The jianying88.com article "Qwen3.8-Flash-Next混合注意力深度解析…",
 * section 三, gives the GDN layer a short convolution of kernel width 4
 * (config linear_conv_kernel_dim 4) and prints no formula.  This library
 * reads it as a causal depthwise convolution of every q, k and v channel
 * within its sequence, followed by an optional activation (the pages name
 * none), then normalises q and k per (token, head) and activates the gates as
 * the workloads' recipes do:
 *
 *     y[t, c]   = sum_{i=0..3} conv_w[c, i] x[t - 3 + i, c]   (x = 0 before the sequence start)
 *     y         = act(y)                                      (GDN_ACT_NONE or GDN_ACT_SILU)
 *     q, k      = y / sqrt(sum over the head's d channels of y^2 + eps)
 *     v         = y
 *     log_alpha = -softplus(a),  beta = sigmoid(b)
 *
 *   q_raw, k_raw [T, H_qk, dk], v_raw [T, H_v, dv] : io_dtype; a, b [T, H_v] fp32.
 *   conv_w    : fp32 [(2 H_qk + H_v) * 128, 4]: the q channels (head-major),
 *               then k, then v; tap 3 weighs the current token.
 *   cu_seqlens: as for gdn_prefill (the convolution restarts at each sequence).
 *   q, k, v   : outputs, shapes and dtype of the raw inputs (must not overlap them).
 *   log_alpha, beta : outputs [T, H_v] fp32.
 *   All tensor pointers 16-byte aligned; a, b, log_alpha, beta 4-byte aligned.
 *
 * Returns GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED or GDN_ERR_CUDA.
 */
GDN_API gdn_status gdn_frontend(const void *q_raw, const void *k_raw, const void *v_raw,
                        const float *conv_w, const float *a, const float *b,
                        const int32_t *cu_seqlens, int32_t N, int32_t T,
                        int32_t H_qk, int32_t H_v, int32_t dk, int32_t dv,
                        gdn_dtype io_dtype, gdn_activation act, float eps,
                        void *q, void *k, void *v, float *log_alpha, float *beta,
                        void *stream);

/*
 * gdn_frontend_decode_step -- gdn_frontend for one new token of each of B
 * sequences.  conv_state [B, 3, (2 H_qk + H_v) * 128] (io_dtype) holds each
 * sequence's last three raw input rows, oldest first (zeros at a sequence's
 * start); it is read, then shifted in place to end with this token's raw row.
 * Other arguments as for gdn_frontend with T = B rows and no cu_seqlens.
 */
GDN_API gdn_status gdn_frontend_decode_step(const void *q_raw, const void *k_raw,
                                    const void *v_raw, const float *conv_w,
                                    const float *a, const float *b, void *conv_state,
                                    int32_t B, int32_t H_qk, int32_t H_v, int32_t dk,
                                    int32_t dv, gdn_dtype io_dtype, gdn_activation act,
                                    float eps, void *q, void *k, void *v,
                                    float *log_alpha, float *beta, void *stream);

/* Static, human-readable name of a status code. */
GDN_API const char *gdn_status_string(gdn_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
GDN_API int32_t gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
