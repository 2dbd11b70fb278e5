// gdn_backward.cu -- gradients of the chunked GDN prefill (sm_100a).
//
// The loss is L = <dO, o> + <dS_final, S_final>; the gradients are those of
// the state-update formula of the bjdmk.com.cn article (section 2.1) with
// readout o_t = S_t^T q_t, taken through the same chunk form the forward
// kernels use (T_b = T diag(beta), X = V - diag(gamma) K S, Delta = T_b X,
// O = diag(gamma) Q S + (M o Q K^T) Delta, S' = gamma_C S + K^T diag(d) Delta).
// Per chunk, with S its entering state and dS' the gradient of the state
// after it:
//
//   dDelta = (M o QK^T)^T dO + diag(d) K dS'        dX = T_b^T dDelta  (= dV)
//   dS     = gamma_C dS' + (diag(gamma) Q)^T dO - (diag(gamma) K)^T dX
//   dQ     = diag(gamma) dO S^T + P K,              P = M o (dO Delta^T)
//   dK     = P^T Q - diag(gamma) dX S^T + diag(d) Delta dS'^T + (E + E^T) K
//            E = strict_lower(-T_b^T dT_b T_b^T) o M,   dT_b = dDelta X^T
//   dbeta_j = (sum_r dT_b,rj T_b,rj + sum_i E_ji (K K^T)_ji) / beta_j
//
// and the gate gradient through the cumulative log gates g (gamma, d, M and
// gamma_C are exponentials of g and of its differences), reverse-summed within
// the chunk into dlog_alpha.
//
// Three launches after the forward pass (chunk operators, then the state pass
// saving every chunk's entering state):
//   grad_state_kernel  one CTA per (sequence, value head, d_v slice): the
//                      reverse chain over the chunks, carrying dS in registers;
//                      writes dV, dS0 and every chunk's dS'.
//   grad_chunk_kernel  one CTA per (chunk, query/key head), over the head's
//                      value heads: dQ, dK, dbeta, dlog_alpha of the chunk.
#include <cudaTypedefs.h>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_tiles.cuh"

namespace gdn {

namespace {

struct GradParams {
    const float* log_alpha;   // [T, H_v]
    const float* beta;        // [T, H_v]
    const int32_t* cu_seqlens;
    const uint8_t* records;   // chunk-operator records of the forward pass
    const uint8_t* S_saved;   // [slot, H_v] bf16 images: state entering each chunk
    uint8_t* dS_saved;        // [slot, H_v] bf16 images: gradient of the state after it
    const float* dS_final;    // [N, H_v, 128, 128] or null
    float* dS0;               // [N, H_v, 128, 128] or null
    void* dq;                 // [T, H_qk, 128]
    void* dk;                 // [T, H_qk, 128]
    void* dv;                 // [T, H_v, 128]
    float* dlog_alpha;        // [T, H_v]
    float* dbeta;             // [T, H_v]
    int H_qk, H_v, N, T;
};

// acc[2 NP n-tiles] += A (16 rows at m0; A_K: K-major tile, else MN-major) x B
// (n-tiles n0 .. n0 + 16 NP; B_K: K-major tile, else MN-major) over k-steps
// ks0 .. ks1 - 1 of 16.
template <int NP, bool A_K, bool B_K>
__device__ __forceinline__ void mma_rows(float (*acc)[4], uint32_t a, uint32_t ah, int m0, uint32_t b,
                                         uint32_t bh, int n0, int ks0, int ks1, int lane) {
    for (int ks = ks0; ks < ks1; ++ks) {
        uint32_t af[4];
        if (A_K) lda_k(a, ah, m0, 16 * ks, lane, af);
        else lda_mn(a, ah, m0, 16 * ks, lane, af);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
            uint32_t bf[4];
            if (B_K) ldb_k(b, bh, n0 + 16 * p, 16 * ks, lane, bf);
            else ldb_mn(b, bh, n0 + 16 * p, 16 * ks, lane, bf);
            mma16816(acc[2 * p], af, bf[0], bf[1]);
            mma16816(acc[2 * p + 1], af, bf[2], bf[3]);
        }
    }
}

// Accumulators (rows m0 + g (+8), columns c0 + 8 nt + 2 t (+1)) as bf16 into a
// swizzled 64-column tile.
template <int NT>
__device__ __forceinline__ void store_acc_cols(uint8_t* smem, uint32_t base_off, int m0, int c0,
                                               const float (*acc)[4], int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int col = c0 + 8 * nt + 2 * t;
        *reinterpret_cast<uint32_t*>(smem + taddr_e(base_off, m0 + g, col, 0)) =
            pack2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<uint32_t*>(smem + taddr_e(base_off, m0 + g + 8, col, 0)) =
            pack2(acc[nt][2], acc[nt][3]);
    }
}

template <int N>
__device__ __forceinline__ void zero_acc(float (*acc)[4]) {
#pragma unroll
    for (int i = 0; i < N; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
}

__device__ __forceinline__ float2 ld_bf16x2(const uint8_t* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

// ============================================================================
// Reverse chain.  Grid (d_v slices, H_v, N); 256 threads; ring of K, Q, the dO
// slice and the chunk's record, filled in reverse chunk order by one thread.
// ============================================================================
constexpr int GS_STAGES = 3;
constexpr int GS_LOADER = 128;
constexpr int GS_BAR_ID = 1;
constexpr uint32_t GS_K = 0, GS_Q = 2 * HALF, GS_O = 4 * HALF, GS_REC = 5 * HALF;
constexpr uint32_t GS_STAGE = ((GS_REC + REC_BYTES + 1023) / 1024) * 1024;
constexpr uint32_t GS_TX = 5 * HALF + REC_BYTES;
constexpr uint32_t GS_DSB = GS_STAGES * GS_STAGE;  // dS' in bf16, 128 x 64
constexpr uint32_t GS_DDEL = GS_DSB + 2 * HALF;    // dDelta, 64 x 64
constexpr uint32_t GS_GDO = GS_DDEL + HALF;        // gamma o dO
constexpr uint32_t GS_GDX = GS_GDO + HALF;         // -gamma o dX
constexpr uint32_t GS_BAR = GS_GDX + HALF;
constexpr uint32_t GS_MISC = GS_BAR + GS_STAGES * 8;
constexpr uint32_t GS_SMEM = GS_MISC + 16 + 1024;
static_assert(GS_SMEM <= 232448, "reverse chain shared memory budget");

// dX = T_b^T dDelta for rows 16 rb .. +15 and the n-tiles of column half H
// (T_b^T is upper triangular: key blocks rb .. 3); writes dV and -gamma o dX.
template <int NT, int H, typename IO>
__device__ __forceinline__ void dx_half(uint8_t* sm, uint32_t sb, uint32_t tb, int rb, int lane,
                                        const float* rv, int valid, const GradParams& p, int tc0,
                                        int h, int col0, int ncols) {
    constexpr int N0 = H * (NT / 2), N1 = (H + 1) * (NT / 2);
    float acc[N1 - N0][4];
    zero_acc<N1 - N0>(acc);
    for (int ks = rb; ks < 4; ++ks) {
        uint32_t a[4];
        lda_mn(tb, 0, 16 * rb, 16 * ks, lane, a);
#pragma unroll
        for (int nt = N0; nt < N1; nt += 2) {
            if (nt + 1 < N1) {
                uint32_t b[4];
                ldb_mn(sb + GS_DDEL, 0, 8 * nt, 16 * ks, lane, b);
                mma16816(acc[nt - N0], a, b[0], b[1]);
                mma16816(acc[nt - N0 + 1], a, b[2], b[3]);
            } else {
                uint32_t b[2];
                ldb_mn1(sb + GS_DDEL, 8 * nt, 16 * ks, lane, b);
                mma16816(acc[nt - N0], a, b[0], b[1]);
            }
        }
    }
    const int g = lane >> 2, t = lane & 3, r = 16 * rb + g;
    const float gm_lo = rv[r], gm_hi = rv[r + 8];
    IO* dv = static_cast<IO*>(p.dv);
#pragma unroll
    for (int i = 0; i < N1 - N0; ++i) {
        const int col = 8 * (N0 + i) + 2 * t;
        *reinterpret_cast<uint32_t*>(sm + taddr_e(GS_GDX, r, col, 0)) =
            pack2(-gm_lo * acc[i][0], -gm_lo * acc[i][1]);
        *reinterpret_cast<uint32_t*>(sm + taddr_e(GS_GDX, r + 8, col, 0)) =
            pack2(-gm_hi * acc[i][2], -gm_hi * acc[i][3]);
        if (col < ncols) {
            if (r < valid)
                store2<IO>(dv + ((size_t)(tc0 + r) * p.H_v + h) * D + col0 + col, acc[i][0], acc[i][1]);
            if (r + 8 < valid)
                store2<IO>(dv + ((size_t)(tc0 + r + 8) * p.H_v + h) * D + col0 + col, acc[i][2],
                           acc[i][3]);
        }
    }
}

template <int NS, typename IO>
__global__ void __launch_bounds__(256, 1)
    grad_state_kernel(const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_do, const GradParams p) {
    static_assert(NS == 32 || NS == 48 || NS == 64, "slice width");
    constexpr int NT = NS / 8, NP = NT / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + GS_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + GS_MISC);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
    const int h = blockIdx.y, n = blockIdx.z;
    const int hq = h / (p.H_v / p.H_qk);
    const int col0 = blockIdx.x * NS;
    const int ncols = min(NS, D - col0);
    const int t_beg = p.cu_seqlens[n], t_end = p.cu_seqlens[n + 1];
    const int nchunks = (t_end - t_beg + C - 1) / C;

    if (tid == 0) {
        for (int i = 0; i < GS_STAGES; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // iteration i handles chunk nchunks - 1 - i, in ring stage i % GS_STAGES
    auto issue = [&](int i) {
        const int c = nchunks - 1 - i, s = i % GS_STAGES;
        uint8_t* st = sm + s * GS_STAGE;
        const int y = t_beg + c * C;
        uint64_t* full = &bars[s];
        mbar_arrive_expect_tx(full, GS_TX);
        tma_load_2d(st + GS_K, &map_k, hq * D, y, full);
        tma_load_2d(st + GS_K + HALF, &map_k, hq * D + 64, y, full);
        tma_load_2d(st + GS_Q, &map_q, hq * D, y, full);
        tma_load_2d(st + GS_Q + HALF, &map_q, hq * D + 64, y, full);
        tma_load_2d(st + GS_O, &map_do, h * D + col0, y, full);
        bulk_load(st + GS_REC, p.records + (size_t)(record_slot(n, y) * p.H_v + h) * REC_BYTES,
                  REC_BYTES, full);
    };
    int issued = 0;
    if (tid == GS_LOADER)
        for (; issued < min(GS_STAGES, nchunks); ++issued) issue(issued);

    const bool mw = warp < 4;
    const int m0 = 16 * (warp & 3);
    const int r0 = 16 * warp;
    // G: gradient of the state after the chunk in flight, rows r0 + {g, g+8},
    // columns 8 nt + 2 t4 + {0, 1} of this slice
    float G[NT][4];
    {
        const float* s0 = p.dS_final ? p.dS_final + ((size_t)n * p.H_v + h) * D * D : nullptr;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int row = r0 + g + ((e >> 1) << 3), col = 8 * nt + 2 * t4 + (e & 1);
                G[nt][e] = (s0 && col < ncols) ? s0[(size_t)row * D + col0 + col] : 0.f;
            }
        store_acc_bf16<NT>(sm, GS_DSB, 0, r0, G, lane, 1.f, 1.f);
    }
    bar_sync<GS_BAR_ID, 256>();

    for (int i = 0; i < nchunks; ++i) {
        const int c = nchunks - 1 - i, s = i % GS_STAGES;
        const uint32_t st = sb + s * GS_STAGE;
        const uint8_t* stp = sm + s * GS_STAGE;
        const float* rv = reinterpret_cast<const float*>(stp + GS_REC + REC_VEC);
        const int tc0 = t_beg + c * C;
        const int valid = min(C, t_end - tc0);
        const bool ok = mbar_wait(&bars[s], (i / GS_STAGES) & 1, abort_flag);
        __syncwarp();
        {  // the gradient of the state after this chunk (bf16 image), for the per-chunk gradients
            uint8_t* sv = p.dS_saved + ((size_t)record_slot(n, tc0) * p.H_v + h) * STATE_IMAGE_BYTES;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int hl = 0; hl < 2; ++hl) {
                    const int row = r0 + g + 8 * hl, col = 8 * nt + 2 * t4;
                    if (col < ncols)
                        *reinterpret_cast<uint32_t*>(sv + taddr_e(0, row, col0 + col, 2 * HALF)) =
                            pack2(G[nt][2 * hl], G[nt][2 * hl + 1]);
                }
        }
        if (mw) {
            // dDelta = (M o QK^T)^T dO + d o (K dS')  (rows m0 .. m0+15); the masked
            // QK^T is lower triangular, so its transpose needs key blocks rb .. 3
            float accY[NT][4], accM[NT][4];
            zero_acc<NT>(accY);
            zero_acc<NT>(accM);
            mma_rows<NP, true, false>(accY, st + GS_K, HALF, m0, sb + GS_DSB, 0, 0, 0, 8, lane);
            mma_rows<NP, false, false>(accM, st + GS_REC + REC_MQ, 0, m0, st + GS_O, 0, 0, warp, 4,
                                       lane);
            const float d_lo = rv[64 + m0 + g], d_hi = rv[64 + m0 + g + 8];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                accM[nt][0] = fmaf(d_lo, accY[nt][0], accM[nt][0]);
                accM[nt][1] = fmaf(d_lo, accY[nt][1], accM[nt][1]);
                accM[nt][2] = fmaf(d_hi, accY[nt][2], accM[nt][2]);
                accM[nt][3] = fmaf(d_hi, accY[nt][3], accM[nt][3]);
            }
            store_acc_bf16<NT>(sm, GS_DDEL, 0, m0, accM, lane, 1.f, 1.f);
        } else {
            // gamma o dO, rows past the sequence end zero (they belong to the next one)
            const int ma = 16 * (warp - 4);
            for (int e = lane; e < 16 * (NS / 2); e += 32) {
                const int row = ma + e / (NS / 2), col = 2 * (e % (NS / 2));
                const float gm = row < valid ? rv[row] : 0.f;
                const float2 x = ld_bf16x2(stp + GS_O + taddr_e(0, row, col, 0));
                *reinterpret_cast<uint32_t*>(sm + taddr_e(GS_GDO, row, col, 0)) =
                    pack2(gm * x.x, gm * x.y);
            }
        }
        if (!bar_and<GS_BAR_ID, 256>(ok)) break;
        if (warp < 4)
            dx_half<NT, 0, IO>(sm, sb, st + GS_REC + REC_TB, warp & 3, lane, rv, valid, p, tc0, h,
                               col0, ncols);
        else
            dx_half<NT, 1, IO>(sm, sb, st + GS_REC + REC_TB, warp & 3, lane, rv, valid, p, tc0, h,
                               col0, ncols);
        if (!bar_and<GS_BAR_ID, 256>(ok)) break;
        {  // dS = gamma_C dS' + Q^T (gamma o dO) + K^T (-gamma o dX)   (rows r0 .. r0+15)
            const float gamC = rv[128];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) G[nt][e] *= gamC;
            mma_rows<NP, false, false>(G, st + GS_Q, HALF, r0, sb + GS_GDO, 0, 0, 0, 4, lane);
            mma_rows<NP, false, false>(G, st + GS_K, HALF, r0, sb + GS_GDX, 0, 0, 0, 4, lane);
        }
        store_acc_bf16<NT>(sm, GS_DSB, 0, r0, G, lane, 1.f, 1.f);
        if (!bar_and<GS_BAR_ID, 256>(ok)) break;
        if (tid == GS_LOADER && i + GS_STAGES < nchunks) issue(issued++);
    }
    if (p.dS0 && !*abort_flag) {
        float* d0 = p.dS0 + ((size_t)n * p.H_v + h) * D * D;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int hl = 0; hl < 2; ++hl) {
                const int row = r0 + g + 8 * hl, col = 8 * nt + 2 * t4;
                if (col < ncols)
                    *reinterpret_cast<float2*>(d0 + (size_t)row * D + col0 + col) =
                        make_float2(G[nt][2 * hl], G[nt][2 * hl + 1]);
            }
    }
    if (tid == GS_LOADER)
        for (int i = max(0, issued - GS_STAGES); i < issued; ++i)
            mbar_wait_drain(&bars[i % GS_STAGES], (i / GS_STAGES) & 1);
    __syncthreads();
}

// ============================================================================
// Per-chunk gradients.  Grid (record slots, H_qk); 256 threads, one CTA per SM.
// Warp w: rows 16 (w & 3) of the 64-row products; column half (w >> 2) of the
// 128-wide ones (64 columns) or of the 64-wide ones (32 columns).
// ============================================================================
constexpr uint32_t GC_K = 0;                    // K, 64 x 128 (two halves)
constexpr uint32_t GC_Q = 2 * HALF;             // Q
constexpr uint32_t GC_V = 4 * HALF;             // V, then X in place
constexpr uint32_t GC_O = 6 * HALF;             // dO
constexpr uint32_t SHALF = 16384;               // a 128-row half of a 128 x 128 tile
constexpr uint32_t GC_S = 8 * HALF;             // S (entering state), 128 x 128
constexpr uint32_t GC_DS = GC_S + 2 * SHALF;    // dS' (gradient of the state after)
constexpr uint32_t GC_REC = GC_DS + 2 * SHALF;  // the chunk's operator record
constexpr uint32_t GC_DEL = GC_REC + ((REC_BYTES + 1023) / 1024) * 1024;  // Delta
constexpr uint32_t GC_DDEL = GC_DEL + 2 * HALF;                          // dDelta
constexpr uint32_t GC_DX = GC_DDEL + 2 * HALF;                           // dX
constexpr uint32_t GC_PY = GC_DX + 2 * HALF;    // P (then Y), 64 x 64
constexpr uint32_t GC_TE = GC_PY + HALF;        // dT_b (then E), 64 x 64
constexpr uint32_t GC_F = GC_TE + HALF;         // fp32: g2[64], dg[64], dbeta[64], misc[64]
constexpr uint32_t GC_BAR = GC_F + 4 * 64 * 4;  // three mbarriers
constexpr uint32_t GC_MISC = GC_BAR + 24;
constexpr uint32_t GC_SMEM = GC_MISC + 16 + 1024;
static_assert(GC_SMEM <= 232448, "per-chunk gradient shared memory budget");

// This thread's part of sum(S o dS') over two bf16 state tiles of the same
// layout (each thread 128 bytes of each).
__device__ __forceinline__ float tile_dot(const uint8_t* a, const uint8_t* b, int tid) {
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t off = (uint32_t)(tid + 256 * i) * 16;
        const uint4 x = *reinterpret_cast<const uint4*>(a + off);
        const uint4 y = *reinterpret_cast<const uint4*>(b + off);
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 u = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[e]));
            const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[e]));
            dot = fmaf(u.x, v.x, fmaf(u.y, v.y, dot));
        }
    }
    return dot;
}

// Row sums (over the accumulator's columns) of acc o w, into dst[row] (smem,
// atomically): rows m0 + g and m0 + g + 8, scaled by s_lo and s_hi.
template <int NT>
__device__ __forceinline__ void add_row_sums(float* dst, int m0, const float (*v)[4], int lane,
                                             float s_lo, float s_hi) {
    float lo = 0.f, hi = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        lo += v[nt][0] + v[nt][1];
        hi += v[nt][2] + v[nt][3];
    }
    lo += __shfl_xor_sync(0xffffffffu, lo, 1);
    lo += __shfl_xor_sync(0xffffffffu, lo, 2);
    hi += __shfl_xor_sync(0xffffffffu, hi, 1);
    hi += __shfl_xor_sync(0xffffffffu, hi, 2);
    if ((lane & 3) == 0) {
        const int g = lane >> 2;
        atomicAdd(&dst[m0 + g], s_lo * lo);
        atomicAdd(&dst[m0 + g + 8], s_hi * hi);
    }
}
// Column sums (over the accumulator's 16 rows) of v, into dst[n0 + col] with
// factor s.
template <int NT>
__device__ __forceinline__ void add_col_sums(float* dst, int n0, const float (*v)[4], int lane,
                                             float s) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float c0 = v[nt][0] + v[nt][2], c1 = v[nt][1] + v[nt][3];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            c0 += __shfl_xor_sync(0xffffffffu, c0, off);
            c1 += __shfl_xor_sync(0xffffffffu, c1, off);
        }
        if (lane < 4) {
            atomicAdd(&dst[n0 + 8 * nt + 2 * lane], s * c0);
            atomicAdd(&dst[n0 + 8 * nt + 2 * lane + 1], s * c1);
        }
    }
}

template <typename IO>
__global__ void __launch_bounds__(256, 1)
    grad_chunk_kernel(const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v,
                      const __grid_constant__ CUtensorMap map_do, const GradParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + GC_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + GC_MISC);
    float* g2 = reinterpret_cast<float*>(sm + GC_F);  // cumulative log2 gates
    float* dg = g2 + 64;                              // gradient w.r.t. g (natural log)
    float* dbt = g2 + 128;                            // dbeta * beta
    float* misc = g2 + 192;                           // [0] sum ddv, [1] <dS', S>, [2..] beta
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
    const int rb = warp & 3, hh = warp >> 2;
    const int m0 = 16 * rb;
    int n, c;
    slot_owner(p.cu_seqlens, p.N, blockIdx.x, n, c);
    if (n < 0) return;  // uniform across the CTA
    const int hq = blockIdx.y;
    const int group = p.H_v / p.H_qk;
    const int t_end = p.cu_seqlens[n + 1];
    const int tc0 = p.cu_seqlens[n] + c * C;
    const int valid = min(C, t_end - tc0);
    const long long slot = record_slot(n, tc0);

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // value head vh's V, dO and saved states (bf16 images, straight into their
    // tiles) on bars[1]; its record on bars[2]
    auto issue_head = [&](int vh) {
        const int h = hq * group + vh;
        const size_t so = ((size_t)slot * p.H_v + h) * STATE_IMAGE_BYTES;
        mbar_arrive_expect_tx(&bars[1], 4 * HALF + 2 * STATE_IMAGE_BYTES);
        tma_load_2d(sm + GC_V, &map_v, h * D, tc0, &bars[1]);
        tma_load_2d(sm + GC_V + HALF, &map_v, h * D + 64, tc0, &bars[1]);
        tma_load_2d(sm + GC_O, &map_do, h * D, tc0, &bars[1]);
        tma_load_2d(sm + GC_O + HALF, &map_do, h * D + 64, tc0, &bars[1]);
        bulk_load(sm + GC_S, p.S_saved + so, STATE_IMAGE_BYTES, &bars[1]);
        bulk_load(sm + GC_DS, p.dS_saved + so, STATE_IMAGE_BYTES, &bars[1]);
    };
    auto issue_rec = [&](int vh) {
        const int h = hq * group + vh;
        mbar_arrive_expect_tx(&bars[2], REC_BYTES);
        bulk_load(sm + GC_REC, p.records + (size_t)(slot * p.H_v + h) * REC_BYTES, REC_BYTES,
                  &bars[2]);
    };
    int heads = 0, recs = 0;  // copies issued (thread 0)
    // after a failed wait: let every copy in flight land (bounded), then leave
    auto drain = [&]() {
        if (tid == 0) {
            mbar_wait_drain(&bars[0], 0);
            if (heads > 0) mbar_wait_drain(&bars[1], (heads - 1) & 1);
            if (recs > 0) mbar_wait_drain(&bars[2], (recs - 1) & 1);
        }
        __syncthreads();
    };
    if (tid == 0) {
        mbar_arrive_expect_tx(&bars[0], 4 * HALF);
        tma_load_2d(sm + GC_K, &map_k, hq * D, tc0, &bars[0]);
        tma_load_2d(sm + GC_K + HALF, &map_k, hq * D + 64, tc0, &bars[0]);
        tma_load_2d(sm + GC_Q, &map_q, hq * D, tc0, &bars[0]);
        tma_load_2d(sm + GC_Q + HALF, &map_q, hq * D + 64, tc0, &bars[0]);
        issue_head(0);
        issue_rec(0);
        heads = recs = 1;
    }
    bool ok = mbar_wait(&bars[0], 0, abort_flag);
    if (!__syncthreads_and(ok)) {
        drain();
        return;
    }
    if (valid < C) {  // rows past the sequence end belong to the next sequence: zero them
        for (int i = tid; i < 4 * 64 * 8; i += 256) {
            const int tile = i / 512, row = (i >> 3) & 63, ch = i & 7;
            if (row >= valid)
                *reinterpret_cast<uint4*>(sm + tile * HALF + row * 128 + ch * 16) =
                    make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();

    float dQ[8][4], dK[8][4];  // rows m0.., columns 64 hh .. 64 hh + 63
    zero_acc<8>(dQ);
    zero_acc<8>(dK);

    for (int vh = 0; vh < group; ++vh) {
        const int h = hq * group + vh;
        // the gates (while this head's copies land)
        if (tid < 64) {
            dg[tid] = 0.f;
            dbt[tid] = 0.f;
            misc[tid] = 0.f;
        }
        if (warp == 0) {  // inclusive scan of log alpha (log2 units); lane l: tokens 2l, 2l+1
            float la[2] = {0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 2; ++e)
                if (2 * lane + e < valid) la[e] = p.log_alpha[(size_t)(tc0 + 2 * lane + e) * p.H_v + h];
            const float x0 = la[0] * LOG2E, x1 = la[1] * LOG2E;
            float incl = x0 + x1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            g2[2 * lane] = incl - x1;
            g2[2 * lane + 1] = incl;
        }
        __syncthreads();
        ok = mbar_wait(&bars[1], vh & 1, abort_flag);
        ok = mbar_wait(&bars[2], vh & 1, abort_flag) && ok;
        if (!__syncthreads_and(ok)) {
            drain();
            return;
        }
        {  // <dS', S>, for the gate gradient of the chunk's last row
            float dot = tile_dot(sm + GC_S, sm + GC_DS, tid);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            if (lane == 0) atomicAdd(&misc[1], dot);
        }
        if (valid < C) {  // V and dO rows past the sequence end
            for (int i = tid; i < 4 * 64 * 8; i += 256) {
                const int tile = i / 512, row = (i >> 3) & 63, ch = i & 7;
                if (row >= valid)
                    *reinterpret_cast<uint4*>(sm + GC_V + tile * HALF + row * 128 + ch * 16) =
                        make_uint4(0, 0, 0, 0);
            }
            __syncthreads();
        }
        const float* rv = reinterpret_cast<const float*>(sm + GC_REC + REC_VEC);
        const uint32_t tb = sb + GC_REC + REC_TB, mq = sb + GC_REC + REC_MQ;
        const int n0 = 64 * hh;  // this warp's columns of the 128-wide products
        const float gm_lo = rv[m0 + g], gm_hi = rv[m0 + g + 8];
        const float d_lo = rv[64 + m0 + g], d_hi = rv[64 + m0 + g + 8];
        const float gam_C = rv[128];

        // 1. K S (kept for dg), Q S -> dg += gamma_r dO_r . (QS)_r; X = V - gamma o KS
        float KS[8][4];
        {
            zero_acc<8>(KS);
            mma_rows<4, true, false>(KS, sb + GC_K, HALF, m0, sb + GC_S, SHALF, n0, 0, 8, lane);
            float QS[8][4];
            zero_acc<8>(QS);
            mma_rows<4, true, false>(QS, sb + GC_Q, HALF, m0, sb + GC_S, SHALF, n0, 0, 8, lane);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int col = n0 + 8 * nt + 2 * t4;
                const float2 o_lo = ld_bf16x2(sm + taddr_e(GC_O, m0 + g, col, HALF));
                const float2 o_hi = ld_bf16x2(sm + taddr_e(GC_O, m0 + g + 8, col, HALF));
                QS[nt][0] *= o_lo.x;
                QS[nt][1] *= o_lo.y;
                QS[nt][2] *= o_hi.x;
                QS[nt][3] *= o_hi.y;
                const float2 v_lo = ld_bf16x2(sm + taddr_e(GC_V, m0 + g, col, HALF));
                const float2 v_hi = ld_bf16x2(sm + taddr_e(GC_V, m0 + g + 8, col, HALF));
                *reinterpret_cast<uint32_t*>(sm + taddr_e(GC_V, m0 + g, col, HALF)) =
                    pack2(v_lo.x - gm_lo * KS[nt][0], v_lo.y - gm_lo * KS[nt][1]);
                *reinterpret_cast<uint32_t*>(sm + taddr_e(GC_V, m0 + g + 8, col, HALF)) =
                    pack2(v_hi.x - gm_hi * KS[nt][2], v_hi.y - gm_hi * KS[nt][3]);
            }
            add_row_sums<8>(dg, m0, QS, lane, gm_lo, gm_hi);
        }
        __syncthreads();
        // 2. Delta = T_b X (T_b lower triangular: key blocks 0 .. rb)
        {
            float acc[8][4];
            zero_acc<8>(acc);
            mma_rows<4, true, false>(acc, tb, 0, m0, sb + GC_V, HALF, n0, 0, rb + 1, lane);
            store_acc_bf16<8>(sm, GC_DEL + (hh ? HALF : 0), 0, m0, acc, lane, 1.f, 1.f);
        }
        __syncthreads();
        // 3. dDelta = (M o QK^T)^T dO + d o (K dS');  ddv_r = d_r (K dS')_r . Delta_r
        {
            float KD[8][4], acc[8][4];
            zero_acc<8>(KD);
            zero_acc<8>(acc);
            mma_rows<4, true, false>(KD, sb + GC_K, HALF, m0, sb + GC_DS, SHALF, n0, 0, 8, lane);
            mma_rows<4, false, false>(acc, mq, 0, m0, sb + GC_O, HALF, n0, rb, 4, lane);
            float ddv[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int col = n0 + 8 * nt + 2 * t4;
                const float2 e_lo = ld_bf16x2(sm + taddr_e(GC_DEL, m0 + g, col, HALF));
                const float2 e_hi = ld_bf16x2(sm + taddr_e(GC_DEL, m0 + g + 8, col, HALF));
                ddv[nt][0] = KD[nt][0] * e_lo.x;
                ddv[nt][1] = KD[nt][1] * e_lo.y;
                ddv[nt][2] = KD[nt][2] * e_hi.x;
                ddv[nt][3] = KD[nt][3] * e_hi.y;
                acc[nt][0] = fmaf(d_lo, KD[nt][0], acc[nt][0]);
                acc[nt][1] = fmaf(d_lo, KD[nt][1], acc[nt][1]);
                acc[nt][2] = fmaf(d_hi, KD[nt][2], acc[nt][2]);
                acc[nt][3] = fmaf(d_hi, KD[nt][3], acc[nt][3]);
            }
            // -ddv_r into dg_r; their total goes to dg of the last row (misc[0])
            add_row_sums<8>(dg, m0, ddv, lane, -d_lo, -d_hi);
            float tot = 0.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
                tot += d_lo * (ddv[nt][0] + ddv[nt][1]) + d_hi * (ddv[nt][2] + ddv[nt][3]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
            if (lane == 0) atomicAdd(&misc[0], tot);
            store_acc_bf16<8>(sm, GC_DDEL + (hh ? HALF : 0), 0, m0, acc, lane, 1.f, 1.f);
        }
        __syncthreads();
        // 4. dX = T_b^T dDelta (upper triangular: key blocks rb .. 3); dg -= gamma_r dX_r . KS_r
        {
            float acc[8][4];
            zero_acc<8>(acc);
            mma_rows<4, false, false>(acc, tb, 0, m0, sb + GC_DDEL, HALF, n0, rb, 4, lane);
            store_acc_bf16<8>(sm, GC_DX + (hh ? HALF : 0), 0, m0, acc, lane, 1.f, 1.f);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) KS[nt][e] *= acc[nt][e];
            add_row_sums<8>(dg, m0, KS, lane, -gm_lo, -gm_hi);
        }
        __syncthreads();
        // 5. P = M o (dO Delta^T) (64 x 64: columns 32 hh ..); dg gets the rows and
        // columns of P o (M o QK^T)
        {
            const int p0 = 32 * hh;
            float acc[4][4];
            zero_acc<4>(acc);
            mma_rows<2, true, true>(acc, sb + GC_O, HALF, m0, sb + GC_DEL, HALF, p0, 0, 8, lane);
            float pm[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + ((e >> 1) << 3), j = p0 + 8 * nt + 2 * t4 + (e & 1);
                    const float mrj = j <= r ? ex2(g2[r] - g2[j]) : 0.f;
                    const float2 qk = ld_bf16x2(sm + taddr_e(GC_REC + REC_MQ, r, j & ~1, 0));
                    pm[nt][e] = acc[nt][e] * ((e & 1) ? qk.y : qk.x);  // P o (M o QK^T)
                    acc[nt][e] *= mrj;
                }
            store_acc_cols<4>(sm, GC_PY, m0, p0, acc, lane);
            add_row_sums<4>(dg, m0, pm, lane, 1.f, 1.f);
            add_col_sums<4>(dg, p0, pm, lane, -1.f);
        }
        __syncthreads();
        // 6. dQ += gamma o (dO S^T) + P K     7. dK += P^T Q - gamma o (dX S^T) + d o (Delta dS'^T)
        {
            float acc[8][4];
            zero_acc<8>(acc);
            mma_rows<4, true, true>(acc, sb + GC_O, HALF, m0, sb + GC_S, SHALF, n0, 0, 8, lane);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                dQ[nt][0] = fmaf(gm_lo, acc[nt][0], dQ[nt][0]);
                dQ[nt][1] = fmaf(gm_lo, acc[nt][1], dQ[nt][1]);
                dQ[nt][2] = fmaf(gm_hi, acc[nt][2], dQ[nt][2]);
                dQ[nt][3] = fmaf(gm_hi, acc[nt][3], dQ[nt][3]);
            }
            mma_rows<4, true, false>(dQ, sb + GC_PY, 0, m0, sb + GC_K, HALF, n0, 0, rb + 1, lane);
            mma_rows<4, false, false>(dK, sb + GC_PY, 0, m0, sb + GC_Q, HALF, n0, rb, 4, lane);
            zero_acc<8>(acc);
            mma_rows<4, true, true>(acc, sb + GC_DX, HALF, m0, sb + GC_S, SHALF, n0, 0, 8, lane);
            float acc2[8][4];
            zero_acc<8>(acc2);
            mma_rows<4, true, true>(acc2, sb + GC_DEL, HALF, m0, sb + GC_DS, SHALF, n0, 0, 8, lane);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                dK[nt][0] += d_lo * acc2[nt][0] - gm_lo * acc[nt][0];
                dK[nt][1] += d_lo * acc2[nt][1] - gm_lo * acc[nt][1];
                dK[nt][2] += d_hi * acc2[nt][2] - gm_hi * acc[nt][2];
                dK[nt][3] += d_hi * acc2[nt][3] - gm_hi * acc[nt][3];
            }
        }
        // 8. dT_b = dDelta X^T (64 x 64); dbeta * beta gets the columns of dT_b o T_b
        {
            const int p0 = 32 * hh;
            float acc[4][4];
            zero_acc<4>(acc);
            mma_rows<2, true, true>(acc, sb + GC_DDEL, HALF, m0, sb + GC_V, HALF, p0, 0, 8, lane);
            store_acc_cols<4>(sm, GC_TE, m0, p0, acc, lane);
            float tt[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + ((e >> 1) << 3), j = p0 + 8 * nt + 2 * t4 + (e & 1);
                    const float2 tv = ld_bf16x2(sm + taddr_e(GC_REC + REC_TB, r, j & ~1, 0));
                    tt[nt][e] = acc[nt][e] * ((e & 1) ? tv.y : tv.x);
                }
            add_col_sums<4>(dbt, p0, tt, lane, 1.f);
        }
        __syncthreads();
        // V (X), dO and both states are free: the next head's copies land during steps 9-12
        if (tid == 0 && vh + 1 < group) {
            issue_head(vh + 1);
            ++heads;
        }
        // 9. Y = dT_b T_b^T
        {
            const int p0 = 32 * hh;
            float acc[4][4];
            zero_acc<4>(acc);
            mma_rows<2, true, true>(acc, sb + GC_TE, 0, m0, tb, 0, p0, 0, 4, lane);
            store_acc_cols<4>(sm, GC_PY, m0, p0, acc, lane);
        }
        __syncthreads();
        // 10. E = strict_lower(-T_b^T Y) o M;  K K^T;  E o KK into dbeta * beta (rows)
        // and dg (rows +, columns -)
        {
            const int p0 = 32 * hh;
            float acc[4][4], kk[4][4];
            zero_acc<4>(acc);
            zero_acc<4>(kk);
            mma_rows<2, false, false>(acc, tb, 0, m0, sb + GC_PY, 0, p0, rb, 4, lane);
            mma_rows<2, true, true>(kk, sb + GC_K, HALF, m0, sb + GC_K, HALF, p0, 0, 8, lane);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + ((e >> 1) << 3), j = p0 + 8 * nt + 2 * t4 + (e & 1);
                    acc[nt][e] = j < r ? -acc[nt][e] * ex2(g2[r] - g2[j]) : 0.f;
                    kk[nt][e] *= acc[nt][e];
                }
            store_acc_cols<4>(sm, GC_TE, m0, p0, acc, lane);
            add_row_sums<4>(dbt, m0, kk, lane, 1.f, 1.f);
            add_row_sums<4>(dg, m0, kk, lane, 1.f, 1.f);
            add_col_sums<4>(dg, p0, kk, lane, -1.f);
        }
        __syncthreads();
        // the record is free too (gamma_C is in a register)
        if (tid == 0 && vh + 1 < group) {
            issue_rec(vh + 1);
            ++recs;
        }
        // 11. dK += E K + E^T K
        mma_rows<4, true, false>(dK, sb + GC_TE, 0, m0, sb + GC_K, HALF, n0, 0, rb + 1, lane);
        mma_rows<4, false, false>(dK, sb + GC_TE, 0, m0, sb + GC_K, HALF, n0, rb, 4, lane);
        // 12. the gates: dg of the last row gets sum ddv + gamma_C <dS', S>;
        // dlog_alpha_t = sum_{r >= t} dg_r (dg holds the gradient w.r.t. g in
        // natural-log units); dbeta_j = (dbeta * beta)_j / beta_j
        if (warp == 0) {
            const float last = misc[0] + gam_C * misc[1];
            // reverse inclusive scan of dg over 64 rows, 2 per lane (rows 2l, 2l+1)
            float d0 = dg[2 * lane], d1 = dg[2 * lane + 1];
            if (lane == 31) d1 += last;
            float s = d0 + d1;  // suffix sums from the top lane down
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, s, off);
                if (lane + off < 32) s += y;
            }
            // s = sum of rows >= 2 lane; row 2l+1's suffix is s - d0
            const float suf0 = s, suf1 = s - d0;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = 2 * lane + e;
                if (r < valid) {
                    const size_t gi = (size_t)(tc0 + r) * p.H_v + h;
                    p.dlog_alpha[gi] = e ? suf1 : suf0;
                    const float b = p.beta[gi];
                    p.dbeta[gi] = b != 0.f ? dbt[r] / b : 0.f;
                }
            }
        }
        __syncthreads();  // the next head's gates overwrite dg, dbt and misc
    }
    // dQ, dK of this chunk and query/key head (every value head of the group summed)
    IO* dq = static_cast<IO*>(p.dq);
    IO* dk = static_cast<IO*>(p.dk);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int hl = 0; hl < 2; ++hl) {
            const int r = m0 + g + 8 * hl, col = 64 * hh + 8 * nt + 2 * t4;
            if (r < valid) {
                const size_t o = ((size_t)(tc0 + r) * p.H_qk + hq) * D + col;
                store2<IO>(dq + o, dQ[nt][2 * hl], dQ[nt][2 * hl + 1]);
                store2<IO>(dk + o, dK[nt][2 * hl], dK[nt][2 * hl + 1]);
            }
        }
}

template <int NS, typename IO>
cudaError_t launch_grad_state(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mo,
                              const GradParams& prm, cudaStream_t stream) {
    auto kern = grad_state_kernel<NS, IO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GS_SMEM);
    if (e != cudaSuccess) return e;
    kern<<<dim3((D + NS - 1) / NS, prm.H_v, prm.N), 256, GS_SMEM, stream>>>(mq, mk, mo, prm);
    return cudaGetLastError();
}

// The reverse chain (as many d_v slices as fit in one wave of one block per
// SM), then the per-chunk gradients; IO is the type of dq, dk and dv.
template <typename IO>
cudaError_t launch_grads(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mo, const GradParams& prm, long long units, int sms,
                         size_t slots, cudaStream_t stream) {
    cudaError_t e = units * 4 <= sms ? launch_grad_state<32, IO>(mq, mk, mo, prm, stream)
                    : units * 3 <= sms ? launch_grad_state<48, IO>(mq, mk, mo, prm, stream)
                                       : launch_grad_state<64, IO>(mq, mk, mo, prm, stream);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(grad_chunk_kernel<IO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GC_SMEM);
    if (e != cudaSuccess) return e;
    grad_chunk_kernel<IO><<<dim3((unsigned)slots, prm.H_qk), 256, GC_SMEM, stream>>>(mq, mk, mv, mo,
                                                                                    prm);
    return cudaGetLastError();
}

}  // namespace

size_t prefill_backward_workspace_bytes(int N, int T, int H_qk, int H_v, bool bf16) {
    if (T == 0) return 0;
    const size_t slots = (size_t)N + ((size_t)T + C - 1) / C;
    const size_t states = up256(slots * H_v * STATE_IMAGE_BYTES);
    const size_t staging =
        bf16 ? 0 : 2 * up256((size_t)T * H_qk * D * 2) + 2 * up256((size_t)T * H_v * D * 2);
    return prefill_record_bytes(N, T, H_v) + 2 * states + staging;
}

cudaError_t launch_prefill_train(const void* q, const void* k, const void* v,
                                 const float* log_alpha, const float* beta, const float* S0,
                                 const int32_t* cu_seqlens, int N, int T, int H_qk, int H_v,
                                 bool bf16, void* o, float* S_final, void* workspace,
                                 cudaStream_t stream) {
    if (T == 0) return launch_prefill(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v,
                                      bf16, o, S_final, nullptr, 1, STATE_PASS_MMA, stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const size_t slots = (size_t)N + ((size_t)T + C - 1) / C;
    const size_t states = up256(slots * H_v * STATE_IMAGE_BYTES);
    uint8_t* records = ws;
    uint8_t* S_saved = ws + prefill_record_bytes(N, T, H_v);
    if (!bf16) {  // bf16 copies of q, k and v where the gradients stage them too
        uint8_t* st = S_saved + 2 * states;
        const size_t nqk = (size_t)T * H_qk * D, nv = (size_t)T * H_v * D;
        const void* src[3] = {q, k, v};
        const size_t cnt[3] = {nqk, nqk, nv};
        const void* dst[3];
        for (int i = 0; i < 3; ++i) {
            f32_to_bf16_kernel<<<592, 256, 0, stream>>>(static_cast<const float*>(src[i]),
                                                        reinterpret_cast<__nv_bfloat16*>(st),
                                                        cnt[i] / 4);
            dst[i] = st;
            st += up256(cnt[i] * 2);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        q = dst[0];
        k = dst[1];
        v = dst[2];
    }
    return launch_prefill_save(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v, records,
                               S_saved, o, S_final, bf16, stream);
}

cudaError_t launch_prefill_backward(const void* q, const void* k, const void* v,
                                    const float* log_alpha, const float* beta, const float* S0,
                                    const int32_t* cu_seqlens, const void* dO,
                                    const float* dS_final, int N, int T, int H_qk, int H_v,
                                    bool bf16, void* dq, void* dk, void* dv, float* dlog_alpha,
                                    float* dbeta, float* dS0, void* workspace, bool recompute,
                                    cudaStream_t stream) {
    if (T == 0) {  // nothing ran: dS0 = dS_final (or zero)
        if (dS0) {
            const size_t bytes = (size_t)N * H_v * D * D * sizeof(float);
            return dS_final ? cudaMemcpyAsync(dS0, dS_final, bytes, cudaMemcpyDeviceToDevice, stream)
                            : cudaMemsetAsync(dS0, 0, bytes, stream);
        }
        return cudaSuccess;
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const size_t slots = (size_t)N + ((size_t)T + C - 1) / C;
    const size_t states = up256(slots * H_v * STATE_IMAGE_BYTES);
    uint8_t* records = ws;
    uint8_t* S_saved = ws + prefill_record_bytes(N, T, H_v);  // bf16 state images
    uint8_t* dS_saved = S_saved + states;
    cudaError_t e;
    if (!bf16) {  // bf16 copies of q, k, v and dO after the states
        uint8_t* st = dS_saved + states;
        const size_t nqk = (size_t)T * H_qk * D, nv = (size_t)T * H_v * D;
        const void* src[4] = {q, k, v, dO};
        const size_t cnt[4] = {nqk, nqk, nv, nv};
        const void* dst[4];
        for (int i = 0; i < 4; ++i) {
            f32_to_bf16_kernel<<<592, 256, 0, stream>>>(static_cast<const float*>(src[i]),
                                                       reinterpret_cast<__nv_bfloat16*>(st),
                                                       cnt[i] / 4);
            dst[i] = st;
            st += up256(cnt[i] * 2);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        q = dst[0];
        k = dst[1];
        v = dst[2];
        dO = dst[3];
    }
    if (recompute) {  // the records and entering states, unless a training forward left them
        e = launch_prefill_save(q, k, v, log_alpha, beta, S0, cu_seqlens, N, T, H_qk, H_v, records,
                                S_saved, nullptr, nullptr, true, stream);
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, q, T, (uint64_t)H_qk * D) || !make_map(&mk, k, T, (uint64_t)H_qk * D) ||
        !make_map(&mv, v, T, (uint64_t)H_v * D) || !make_map(&mo, dO, T, (uint64_t)H_v * D))
        return cudaErrorInvalidValue;
    const GradParams prm{log_alpha, beta, cu_seqlens, records, S_saved, dS_saved, dS_final, dS0,
                         dq,        dk,   dv,         dlog_alpha, dbeta, H_qk, H_v, N, T};
    const long long units = (long long)N * H_v;
    const int sms = device_sms();
    return bf16 ? launch_grads<__nv_bfloat16>(mq, mk, mv, mo, prm, units, sms, slots, stream)
                : launch_grads<float>(mq, mk, mv, mo, prm, units, sms, slots, stream);
}

}  // namespace gdn
