// gdn_prefill.cu -- chunked GDN prefill (sm_100a): TMA tile loads, warp-level
// bf16 tensor-core products (ldmatrix + mma.sync m16n8k16, fp32 accumulate),
// fp32 triangular solve on CUDA cores, state resident in registers.
//
// Operation: the gated delta rule of the bjdmk.com.cn article (section 2.1,
// state-update formula) over packed sequences, with readout o_t = S_t^T q_t.
// The article says the recurrence is made chunk-parallel with the WY
// representation but prints no formulas; the chunk algebra used here is
// derived from the recurrence itself.  For a chunk of C = 64 tokens with entry
// state S (d_k x d_v), cumulative log-gates g_r = sum_{i<=r} log alpha_i,
// gamma_r = exp(g_r):
//
//   A_rj  = beta_r exp(g_r - g_j) (k_r . k_j)  for j < r     (strictly lower)
//   T     = (I + A)^{-1}                                      (unit lower)
//   W     = T diag(beta gamma) K,   U = T diag(beta) V
//   Delta = U - W S                                           (true write vectors)
//   O     = diag(gamma) Q S + (M o Q K^T) Delta,  M_rj = exp(g_r - g_j), j <= r
//   S    <- gamma_C S + K^T diag(exp(g_C - g_j)) Delta
//
// Work split: one CTA per (sequence, value head, d_v slice of NS columns);
// the columns of S evolve independently, so slices need no communication.
// Each math warp keeps 16 rows x NS columns of S as fp32 mma accumulators for
// the whole sequence.
//
// Roles (288 threads): warps 0-7 are the math warps; warp 8 is the TMA
// producer, which streams K, Q (64 x 128 bf16 each) and the V slice (64 x 64
// bf16) of every chunk into a 2-stage ring of 128-byte-swizzled tiles.  Every
// operand tile in shared memory uses that swizzle (16-byte chunk c of row r
// stored at chunk c ^ (r % 8)), so ldmatrix reads are bank-conflict free.
//
// Every mbarrier wait is bounded (gdn_common.cuh); on a timeout the CTA
// records the error in the device status word, lets its copies land and exits.
#include <cudaTypedefs.h>

#include <mutex>

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int C = 64;           // chunk length
constexpr int D = 128;          // head dim (d_k = d_v)
constexpr int NSTAGE = 2;       // TMA ring depth
constexpr int kMathWarps = 8;
constexpr int kMathThreads = kMathWarps * 32;
constexpr int kThreads = kMathThreads + 32;

// ---- shared memory layout (byte offsets from a 1024-aligned base) ----
// ring stage: K (two 64-column halves, 8 KB each), Q (same), V slice (8 KB)
constexpr uint32_t HALF = 8192;                        // 64 rows x 128 B
constexpr uint32_t ST_K = 0, ST_Q = 2 * HALF, ST_V = 4 * HALF;
constexpr uint32_t STAGE_BYTES = 5 * HALF;
constexpr uint32_t OFF_RING = 0;
constexpr uint32_t OFF_TBG = OFF_RING + NSTAGE * STAGE_BYTES;  // T diag(beta gamma), 64x64
constexpr uint32_t OFF_TB = OFF_TBG + HALF;                    // T diag(beta), 64x64
constexpr uint32_t OFF_MQ = OFF_TB + HALF;                     // (M o Q K^T), 64x64
constexpr uint32_t OFF_W = OFF_MQ + HALF;                      // -W, 64x128 (two halves)
constexpr uint32_t OFF_SB = OFF_W + 2 * HALF;                  // S in bf16, 128 x 64
constexpr uint32_t OFF_DU = OFF_SB + 2 * HALF;                 // Delta, 64 x 64
constexpr uint32_t OFF_DD = OFF_DU + HALF;                     // d o Delta, 64 x 64
constexpr uint32_t OFF_AF = OFF_DD + HALF;                     // A in fp32, 64 x 68
constexpr int AF_LD = 68;
constexpr uint32_t OFF_TF = OFF_AF + 64 * AF_LD * 4;           // T in fp32, 64 x 68
constexpr uint32_t OFF_XS = OFF_TF + 64 * AF_LD * 4;           // 3 x 16 x 16 fp32 scratch
constexpr uint32_t OFF_VEC = OFF_XS + 3 * 256 * 4;             // g, beta, gamma, dscale, carry
constexpr uint32_t OFF_BAR = OFF_VEC + 5 * 64 * 4;
constexpr int NBAR = 2 * NSTAGE;                               // full[2], empty[2]
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;              // abort flag
constexpr uint32_t SMEM_USED = OFF_MISC + 16;
constexpr uint32_t SMEM_ALLOC = SMEM_USED + 1024;              // slack for 1024-byte alignment
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

enum Bar { B_FULL = 0, B_EMPTY = NSTAGE };

#ifdef GDN_DEBUG_TRACE
__device__ volatile int* g_trace = nullptr;
__device__ __forceinline__ void trace_mark(int role, int phase, int c) {
    volatile int* t = g_trace;
    if (t) {
        const int cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
        if (cta < 1024) t[cta * 4 + role] = (phase << 20) | (c & 0xFFFFF);
        __threadfence_system();
    }
}
#define TRACE_T(tid, role, phase, c) \
    do { if (threadIdx.x == (tid)) trace_mark(role, phase, c); } while (0)
#else
#define TRACE_T(tid, role, phase, c) ((void)0)
#endif

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void math_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(kMathThreads) : "memory");
}

// Address of element (row, col) of a 128B-swizzled tile whose 64-column
// halves lie `half` bytes apart; col is a multiple of 8.
__device__ __forceinline__ uint32_t taddr(uint32_t base, int row, int col, uint32_t half) {
    return base + (col >> 6) * half + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4);
}
__device__ __forceinline__ uint32_t taddr_e(uint32_t base, int row, int col, uint32_t half) {
    return taddr(base, row, col & ~7, half) + (col & 7) * 2;  // any column
}

__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t a, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment (16 x 16 at rows m0, cols k0) of a K-major tile (rows m, cols k).
__device__ __forceinline__ void lda_k(uint32_t base, uint32_t half, int m0, int k0, int lane,
                                      uint32_t* a) {
    ldsm_x4(taddr(base, m0 + (lane & 15), k0 + ((lane >> 4) << 3), half), a);
}
// A fragment of an MN-major tile (stored rows k, cols m).
__device__ __forceinline__ void lda_mn(uint32_t base, uint32_t half, int m0, int k0, int lane,
                                       uint32_t* a) {
    const int j = lane >> 3;
    ldsm_x4_t(taddr(base, k0 + (lane & 7) + ((j >> 1) << 3), m0 + ((j & 1) << 3), half), a);
}
// B fragments of two n-tiles (n0, n0+8) x (k0..k0+15) from a K-major tile (rows n, cols k).
__device__ __forceinline__ void ldb_k(uint32_t base, uint32_t half, int n0, int k0, int lane,
                                      uint32_t* b) {
    const int j = lane >> 3;
    ldsm_x4(taddr(base, n0 + (lane & 7) + ((j >> 1) << 3), k0 + ((j & 1) << 3), half), b);
}
// B fragments of two n-tiles from an MN-major tile (stored rows k, cols n).
__device__ __forceinline__ void ldb_mn(uint32_t base, uint32_t half, int n0, int k0, int lane,
                                       uint32_t* b) {
    const int j = lane >> 3;
    ldsm_x4_t(taddr(base, k0 + (lane & 7) + ((j & 1) << 3), n0 + ((j >> 1) << 3), half), b);
}

// acc[NT][4] += A(16 x 16*KS) * B(16*KS x 8*NT)
template <int NT, int KS, bool A_MN, bool B_MN>
__device__ __forceinline__ void warp_gemm(float (*acc)[4], uint32_t a_base, uint32_t a_half,
                                          int m0, uint32_t b_base, uint32_t b_half, int lane) {
    static_assert(NT % 2 == 0, "n-tiles come in pairs");
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        uint32_t a[4];
        if (A_MN)
            lda_mn(a_base, a_half, m0, 16 * ks, lane, a);
        else
            lda_k(a_base, a_half, m0, 16 * ks, lane, a);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
            uint32_t b[4];
            if (B_MN)
                ldb_mn(b_base, b_half, 16 * np, 16 * ks, lane, b);
            else
                ldb_k(b_base, b_half, 16 * np, 16 * ks, lane, b);
            mma16816(acc[2 * np], a, b[0], b[1]);
            mma16816(acc[2 * np + 1], a, b[2], b[3]);
        }
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16x2(lo, hi); }

// Store an accumulator tile (rows m0.., NT n-tiles) as bf16 into a swizzled tile
// (rows = accumulator rows), scaled per row by rs_lo (row g) and rs_hi (row g+8).
template <int NT>
__device__ __forceinline__ void store_acc_bf16(uint8_t* smem, uint32_t base_off, uint32_t half,
                                               int m0, const float (*acc)[4], int lane,
                                               float rs_lo, float rs_hi) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int col = 8 * nt + 2 * t;
        *reinterpret_cast<uint32_t*>(smem + taddr_e(base_off, m0 + g, col, half)) =
            pack2(acc[nt][0] * rs_lo, acc[nt][1] * rs_lo);
        *reinterpret_cast<uint32_t*>(smem + taddr_e(base_off, m0 + g + 8, col, half)) =
            pack2(acc[nt][2] * rs_hi, acc[nt][3] * rs_hi);
    }
}

struct PrefillParams {
    const float* log_alpha;
    const float* beta;
    const float* S0;
    const int32_t* cu_seqlens;
    void* o;
    float* S_final;
    int H_qk, H_v;
    int N, T;
};

template <typename IO>
__device__ __forceinline__ void store2(IO* p, float a, float b);
template <>
__device__ __forceinline__ void store2<float>(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
template <>
__device__ __forceinline__ void store2<__nv_bfloat16>(__nv_bfloat16* p, float a, float b) {
    *reinterpret_cast<uint32_t*>(p) = pack2(a, b);
}

template <int NS, typename IO>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const PrefillParams p) {
    static_assert(NS == 32 || NS == 64, "slice width");
    constexpr int NT = NS / 8;  // n-tiles of a slice
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC);
    float* s_g = reinterpret_cast<float*>(sm + OFF_VEC);  // g_r * log2(e)
    float* s_b = s_g + 64;                                // beta_r (0 past the end)
    float* s_gam = s_g + 128;                             // gamma_r
    float* s_ds = s_g + 192;                              // exp(g_C - g_r)
    float* s_carry = s_g + 256;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int n = blockIdx.z;
    const int hq = h / (p.H_v / p.H_qk);
    const int col0 = blockIdx.x * NS;
    const int t_beg = p.cu_seqlens[n];
    const int t_end = p.cu_seqlens[n + 1];
    const int nchunks = (t_end - t_beg + C - 1) / C;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kMathWarps) {
        // ------------------------------------------------------------ TMA producer
        int issued = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NSTAGE;
            if (c >= NSTAGE) {
                const bool ok = mbar_wait(&bars[B_EMPTY + s], ((c / NSTAGE) - 1) & 1, abort_flag);
                if (!__all_sync(0xffffffffu, ok)) break;
            }
            if (lane == 0) {
                uint8_t* st = sm + OFF_RING + s * STAGE_BYTES;
                const int y = t_beg + c * C;
                mbar_arrive_expect_tx(&bars[B_FULL + s], STAGE_BYTES);
                tma_load_2d(st + ST_K, &map_k, hq * D, y, &bars[B_FULL + s]);
                tma_load_2d(st + ST_K + HALF, &map_k, hq * D + 64, y, &bars[B_FULL + s]);
                tma_load_2d(st + ST_Q, &map_q, hq * D, y, &bars[B_FULL + s]);
                tma_load_2d(st + ST_Q + HALF, &map_q, hq * D + 64, y, &bars[B_FULL + s]);
                tma_load_2d(st + ST_V, &map_v, h * D + col0, y, &bars[B_FULL + s]);
            }
            __syncwarp();
            issued = c + 1;
        }
        // Drain: no copy may still be landing in shared memory when the CTA exits.
        for (int c = max(0, issued - NSTAGE); c < issued; ++c)
            mbar_wait(&bars[B_FULL + (c % NSTAGE)], (c / NSTAGE) & 1, abort_flag);
        __syncwarp();
        TRACE_T(kMathThreads, 0, 4, issued);
    } else {
        // ------------------------------------------------------------ math warps
        const int tid = threadIdx.x;
        const int g = lane >> 2, t4 = lane & 3;
        const int m0 = 16 * (warp & 3);       // this warp's 16-row block of 64-row products
        const bool upper = warp < 4;          // warps 0-3 vs 4-7
        float* Af = reinterpret_cast<float*>(sm + OFF_AF);
        float* Tf = reinterpret_cast<float*>(sm + OFF_TF);
        float* Xs = reinterpret_cast<float*>(sm + OFF_XS);
        const float LOG2E = 1.4426950408889634f;
        const int ncols = min(NS, D - col0);

        // S rows 16*warp + {g, g+8}, columns 8*nt + 2*t4 + {0,1}, as fp32 accumulators
        float Sacc[NT][4];
        {
            const float* s0 = p.S0 ? p.S0 + ((size_t)n * p.H_v + h) * D * D : nullptr;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int row = 16 * warp + g + ((e >> 1) << 3);
                    const int col = 8 * nt + 2 * t4 + (e & 1);
                    Sacc[nt][e] = (s0 && col < ncols) ? s0[(size_t)row * D + col0 + col] : 0.f;
                }
            store_acc_bf16<NT>(sm, OFF_SB, HALF, 16 * warp, Sacc, lane, 1.f, 1.f);
        }

        float keep[NT][4];  // warps 0-3: U then Delta; warps 4-7: gamma o (Q S), then O

        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NSTAGE;
            const int tc0 = t_beg + c * C;
            const int valid = min(C, t_end - tc0);
            const uint32_t st = sb + OFF_RING + s * STAGE_BYTES;
            uint8_t* stp = sm + OFF_RING + s * STAGE_BYTES;
            TRACE_T(0, 2, 20, c);

            // gates of this chunk (rows past the sequence end: log alpha = 0, beta = 0)
            float la = 0.f, be = 0.f;
            if (tid < C && tid < valid) {
                la = p.log_alpha[(size_t)(tc0 + tid) * p.H_v + h];
                be = p.beta[(size_t)(tc0 + tid) * p.H_v + h];
            }
            const bool ok = mbar_wait(&bars[B_FULL + s], (c / NSTAGE) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (valid < C) {  // zero K, Q, V rows past the end of the sequence
                for (int i = tid; i < 5 * 64 * 8; i += kMathThreads) {
                    const int tile = i / 512, row = (i >> 3) & 63, ch = i & 7;
                    if (row >= valid)
                        *reinterpret_cast<uint4*>(stp + tile * HALF + row * 128 + ch * 16) =
                            make_uint4(0, 0, 0, 0);
                }
            }
            // inclusive scan of log alpha (rows 0..63 live in warps 0 and 1)
            float gsum = la * LOG2E;
            if (tid < C) {
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, gsum, off);
                    if (lane >= off) gsum += y;
                }
                if (tid == 31) s_carry[0] = gsum;
            }
            math_bar();
            if (tid >= 32 && tid < C) gsum += s_carry[0];
            if (tid < C) {
                s_g[tid] = gsum;
                s_b[tid] = be;
            }
            math_bar();
            const float gC = s_g[C - 1];
            if (tid < C) {
                s_gam[tid] = ex2(gsum);
                s_ds[tid] = (tid < valid) ? ex2(gC - gsum) : 0.f;
            }

            // ---- grams: warps 0-3 rows of K K^T (-> A), warps 4-7 rows of Q K^T (-> M_Q)
            {
                float acc[8][4];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
                warp_gemm<8, 8, false, false>(acc, st + (upper ? ST_K : ST_Q), HALF, m0,
                                              st + ST_K, HALF, lane);
                const int r_lo = m0 + g, r_hi = m0 + g + 8;
                const float g_lo = s_g[r_lo], g_hi = s_g[r_hi];
                if (upper) {
                    const float b_lo = s_b[r_lo], b_hi = s_b[r_hi];
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt) {
                        const int j = 8 * nt + 2 * t4;
                        float2 lo, hi;
                        lo.x = (j < r_lo) ? b_lo * ex2(g_lo - s_g[j]) * acc[nt][0] : 0.f;
                        lo.y = (j + 1 < r_lo) ? b_lo * ex2(g_lo - s_g[j + 1]) * acc[nt][1] : 0.f;
                        hi.x = (j < r_hi) ? b_hi * ex2(g_hi - s_g[j]) * acc[nt][2] : 0.f;
                        hi.y = (j + 1 < r_hi) ? b_hi * ex2(g_hi - s_g[j + 1]) * acc[nt][3] : 0.f;
                        *reinterpret_cast<float2*>(Af + r_lo * AF_LD + j) = lo;
                        *reinterpret_cast<float2*>(Af + r_hi * AF_LD + j) = hi;
                    }
                } else {
                    const bool v_lo = r_lo < valid, v_hi = r_hi < valid;
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt) {
                        const int j = 8 * nt + 2 * t4;
                        const float m00 = (v_lo && j <= r_lo) ? ex2(g_lo - s_g[j]) * acc[nt][0] : 0.f;
                        const float m01 = (v_lo && j + 1 <= r_lo) ? ex2(g_lo - s_g[j + 1]) * acc[nt][1] : 0.f;
                        const float m10 = (v_hi && j <= r_hi) ? ex2(g_hi - s_g[j]) * acc[nt][2] : 0.f;
                        const float m11 = (v_hi && j + 1 <= r_hi) ? ex2(g_hi - s_g[j + 1]) * acc[nt][3] : 0.f;
                        *reinterpret_cast<uint32_t*>(sm + taddr_e(OFF_MQ, r_lo, j, HALF)) = pack2(m00, m01);
                        *reinterpret_cast<uint32_t*>(sm + taddr_e(OFF_MQ, r_hi, j, HALF)) = pack2(m10, m11);
                    }
                }
            }
            for (int i = tid; i < 64 * AF_LD / 4; i += kMathThreads)
                reinterpret_cast<float4*>(Tf)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            math_bar();
            TRACE_T(0, 2, 22, c);

            // ---- T = (I + A)^{-1}: diagonal 16x16 blocks by forward substitution
            if (tid < C) {
                const int b = tid >> 4, cc = tid & 15;
                const float* Ab = Af + (16 * b) * AF_LD + 16 * b;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float sacc = 0.f;
#pragma unroll
                    for (int j = 0; j < i; ++j) sacc = fmaf(-Ab[i * AF_LD + j], x[j], sacc);
                    x[i] = (i == cc) ? 1.f : ((i > cc) ? sacc : 0.f);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) Tf[(16 * b + i) * AF_LD + 16 * b + cc] = x[i];
            }
            math_bar();
            // off-diagonal blocks by distance l = i - j:  X = sum_{k=j}^{i-1} A_ik T_kj ; T_ij = -T_ii X
#pragma unroll 1
            for (int l = 1; l < 4; ++l) {
                const int nb = 4 - l;
                for (int e = tid; e < nb * 256; e += kMathThreads) {
                    const int blk = e >> 8, a = (e >> 4) & 15, bc = e & 15;
                    const int bi = blk + l, bj = blk;
                    float x = 0.f;
                    for (int kb = bj; kb < bi; ++kb) {
                        const float* ar = Af + (16 * bi + a) * AF_LD + 16 * kb;
                        const float* tcol = Tf + (16 * kb) * AF_LD + 16 * bj + bc;
#pragma unroll
                        for (int m = 0; m < 16; ++m) x = fmaf(ar[m], tcol[m * AF_LD], x);
                    }
                    Xs[e] = x;
                }
                math_bar();
                for (int e = tid; e < nb * 256; e += kMathThreads) {
                    const int blk = e >> 8, a = (e >> 4) & 15, bc = e & 15;
                    const int bi = blk + l, bj = blk;
                    const float* tr = Tf + (16 * bi + a) * AF_LD + 16 * bi;
                    const float* xc = Xs + blk * 256 + bc;
                    float y = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m) y = fmaf(tr[m], xc[m * 16], y);
                    Tf[(16 * bi + a) * AF_LD + 16 * bj + bc] = -y;
                }
                math_bar();
            }
            // T_bg = T diag(beta gamma), T_b = T diag(beta) -> bf16 K-major tiles;
            // thread (row, part): parts 0-1 fill T_bg, parts 2-3 fill T_b, 32 columns each
            {
                const int row = tid & 63, part = tid >> 6;
                const bool with_gamma = part < 2;
                const int cb = 32 * (part & 1);
                const uint32_t dst = with_gamma ? OFF_TBG : OFF_TB;
                const float* trow = Tf + row * AF_LD;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    float m[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = cb + 8 * ch + e;
                        m[e] = trow[j] * (with_gamma ? s_b[j] * s_gam[j] : s_b[j]);
                    }
                    uint4 u;
                    u.x = pack2(m[0], m[1]);
                    u.y = pack2(m[2], m[3]);
                    u.z = pack2(m[4], m[5]);
                    u.w = pack2(m[6], m[7]);
                    *reinterpret_cast<uint4*>(sm + taddr(dst, row, cb + 8 * ch, HALF)) = u;
                }
            }
            math_bar();
            TRACE_T(0, 2, 23, c);

            // ---- warps 4-7: W = T_bg K (-> -W tile);  warps 0-3: U = T_b V (registers)
            if (!upper) {
                float acc[16][4];
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
                warp_gemm<16, 4, false, true>(acc, sb + OFF_TBG, HALF, m0, st + ST_K, HALF, lane);
                store_acc_bf16<16>(sm, OFF_W, HALF, m0, acc, lane, -1.f, -1.f);
            } else {
#pragma unroll
                for (int i = 0; i < NT; ++i) keep[i][0] = keep[i][1] = keep[i][2] = keep[i][3] = 0.f;
                warp_gemm<NT, 4, false, true>(keep, sb + OFF_TB, HALF, m0, st + ST_V, HALF, lane);
            }
            math_bar();

            // ---- warps 0-3: Delta = U + (-W) S;  warps 4-7: Q S
            if (upper) {
                warp_gemm<NT, 8, false, true>(keep, sb + OFF_W, HALF, m0, sb + OFF_SB, HALF, lane);
                const float d_lo = s_ds[m0 + g], d_hi = s_ds[m0 + g + 8];
                store_acc_bf16<NT>(sm, OFF_DU, HALF, m0, keep, lane, 1.f, 1.f);
                store_acc_bf16<NT>(sm, OFF_DD, HALF, m0, keep, lane, d_lo, d_hi);
            } else {
#pragma unroll
                for (int i = 0; i < NT; ++i) keep[i][0] = keep[i][1] = keep[i][2] = keep[i][3] = 0.f;
                warp_gemm<NT, 8, false, true>(keep, st + ST_Q, HALF, m0, sb + OFF_SB, HALF, lane);
                const float gm_lo = s_gam[m0 + g], gm_hi = s_gam[m0 + g + 8];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    keep[nt][0] *= gm_lo;
                    keep[nt][1] *= gm_lo;
                    keep[nt][2] *= gm_hi;
                    keep[nt][3] *= gm_hi;
                }
            }
            math_bar();
            TRACE_T(0, 2, 25, c);

            // ---- warps 4-7: O = gamma (Q S) + (M o Q K^T) Delta, stored
            if (!upper) {
                warp_gemm<NT, 4, false, true>(keep, sb + OFF_MQ, HALF, m0, sb + OFF_DU, HALF, lane);
                IO* ob = static_cast<IO*>(p.o);
#pragma unroll
                for (int hl = 0; hl < 2; ++hl) {
                    const int r = m0 + g + 8 * hl;
                    if (r < valid) {
                        IO* orow = ob + ((size_t)(tc0 + r) * p.H_v + h) * D + col0;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const int col = 8 * nt + 2 * t4;
                            if (col < ncols)
                                store2<IO>(orow + col, keep[nt][2 * hl], keep[nt][2 * hl + 1]);
                        }
                    }
                }
            }
            // ---- all warps: S <- gamma_C S + K^T (d o Delta)  (rows 16*warp .. +15)
            {
                const float gamC = ex2(gC);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) Sacc[nt][e] *= gamC;
                warp_gemm<NT, 4, true, true>(Sacc, st + ST_K, HALF, 16 * warp, sb + OFF_DD, HALF,
                                            lane);
            }
            // Every read of this chunk's ring stage is done; generic writes to it (the
            // zeroed padding rows) are ordered before the next TMA refill.
            fence_proxy_async_smem();
            math_bar();
            if (tid == 0) mbar_arrive(&bars[B_EMPTY + s]);
            store_acc_bf16<NT>(sm, OFF_SB, HALF, 16 * warp, Sacc, lane, 1.f, 1.f);
            TRACE_T(0, 2, 27, c);
        }
        if (p.S_final && !*abort_flag) {
            float* sf = p.S_final + ((size_t)n * p.H_v + h) * D * D;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int hl = 0; hl < 2; ++hl) {
                    const int row = 16 * warp + g + 8 * hl;
                    const int col = 8 * nt + 2 * t4;
                    if (col < ncols)
                        *reinterpret_cast<float2*>(sf + (size_t)row * D + col0 + col) =
                            make_float2(Sacc[nt][2 * hl], Sacc[nt][2 * hl + 1]);
                }
        }
        TRACE_T(0, 2, 30, nchunks);
    }
    __syncthreads();
}

// fp32 -> bf16 staging of q, k, v for fp32 I/O.
__global__ void f32_to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                   size_t n4) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
         i += (size_t)gridDim.x * blockDim.x) {
        const float4 v = reinterpret_cast<const float4*>(src)[i];
        uint2 u;
        u.x = pack2(v.x, v.y);
        u.y = pack2(v.z, v.w);
        reinterpret_cast<uint2*>(dst)[i] = u;
    }
}

// S_final = S0, or zeros when S0 is NULL (used when no sequence has tokens).
__global__ void copy_state_kernel(const float* __restrict__ S0, float* __restrict__ S_final,
                                  size_t n4) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
         i += (size_t)gridDim.x * blockDim.x) {
        float4 v = S0 ? reinterpret_cast<const float4*>(S0)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        reinterpret_cast<float4*>(S_final)[i] = v;
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// 2-D bf16 tensor map over a [rows, cols] row-major matrix, 64 x 64 boxes, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows > 0 ? rows : 1};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int NS, typename IO>
cudaError_t launch_ns(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const PrefillParams& prm, int N, cudaStream_t stream) {
    auto kern = prefill_kernel<NS, IO>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    dim3 grid(D / NS, prm.H_v, N);
    kern<<<grid, kThreads, SMEM_ALLOC, stream>>>(mq, mk, mv, prm);
    return cudaGetLastError();
}

}  // namespace

// ---- scratch for gdn_prefill_noalloc -------------------------------------
// A file-scope device array that stands in for the caller's workspace (the bf16
// copies of fp32 q, k, v).  Every GPU that loads the library holds it until the
// process exits.  Its host-side name is not a device address: the address is
// obtained once per device with cudaGetSymbolAddress, with that device current.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t noalloc_scratch_address(void** out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void* addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

size_t prefill_workspace_bytes(int N, int T, int H_qk, int H_v, bool bf16) {
    (void)N;
    if (bf16) return 0;
    auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
    return up((size_t)T * H_qk * D * 2) * 2 + up((size_t)T * H_v * D * 2);
}

cudaError_t launch_prefill(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* S0, const int32_t* cu_seqlens, int N,
                           int T, int H_qk, int H_v, bool bf16, void* o, float* S_final,
                           void* workspace, cudaStream_t stream) {
    if (T == 0) {  // every sequence is empty: S_final = S0 (or zeros)
        if (!S_final) return cudaSuccess;
        copy_state_kernel<<<592, 256, 0, stream>>>(S0, S_final, (size_t)N * H_v * D * D / 4);
        return cudaGetLastError();
    }
    const void *qb = q, *kb = k, *vb = v;
    if (!bf16) {
        auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        const size_t nqk = (size_t)T * H_qk * D, nv = (size_t)T * H_v * D;
        __nv_bfloat16* q16 = reinterpret_cast<__nv_bfloat16*>(ws);
        __nv_bfloat16* k16 = reinterpret_cast<__nv_bfloat16*>(ws + up(nqk * 2));
        __nv_bfloat16* v16 = reinterpret_cast<__nv_bfloat16*>(ws + 2 * up(nqk * 2));
        f32_to_bf16_kernel<<<592, 256, 0, stream>>>(static_cast<const float*>(q), q16, nqk / 4);
        f32_to_bf16_kernel<<<592, 256, 0, stream>>>(static_cast<const float*>(k), k16, nqk / 4);
        f32_to_bf16_kernel<<<592, 256, 0, stream>>>(static_cast<const float*>(v), v16, nv / 4);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        qb = q16;
        kb = k16;
        vb = v16;
    }
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, qb, T, (uint64_t)H_qk * D) || !make_map(&mk, kb, T, (uint64_t)H_qk * D) ||
        !make_map(&mv, vb, T, (uint64_t)H_v * D))
        return cudaErrorInvalidValue;
    PrefillParams prm{log_alpha, beta, S0, cu_seqlens, o, S_final, H_qk, H_v, N, T};
    // Slice width: one CTA per SM at most (each holds ~190 KB of shared memory), so
    // split the head into four 32-column slices only when that still fits in one
    // wave; otherwise two 64-column slices (half the redundant per-chunk work).
    int num_sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    const bool narrow = (long long)N * H_v * 4 <= num_sms;
    if (bf16) {
        if (!narrow) return launch_ns<64, __nv_bfloat16>(mq, mk, mv, prm, N, stream);
        return launch_ns<32, __nv_bfloat16>(mq, mk, mv, prm, N, stream);
    }
    if (!narrow) return launch_ns<64, float>(mq, mk, mv, prm, N, stream);
    return launch_ns<32, float>(mq, mk, mv, prm, N, stream);
}

}  // namespace gdn

#ifdef GDN_DEBUG_TRACE
extern "C" __attribute__((visibility("default"))) int gdn_debug_set_trace(void* host_mapped) {
    volatile int* p = static_cast<volatile int*>(host_mapped);
    return (int)cudaMemcpyToSymbol(gdn::g_trace, &p, sizeof(p));
}
#endif
