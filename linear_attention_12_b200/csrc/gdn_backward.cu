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
//   grad_state_kernel     one CTA per (sequence, value head, d_v slice): the
//                         reverse chain over the chunks, carrying dS in
//                         registers; writes dV, dS0 and every chunk's dS'.
//   grad_chunk_tc_kernel  one CTA per (chunk, query/key head), over the head's
//                         value heads: dQ, dK, dbeta, dlog_alpha of the chunk,
//                         its products on the fifth-generation tensor cores
//                         with dQ and dK accumulated in tensor memory.
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
// HANDOFF (the tcgen05 reverse chain): once -gamma o dX is in shared memory,
// fence it for the tensor cores and arrive on that named barrier, then store dV.
template <int NT, int H, typename IO, int HANDOFF = 0, int HANDOFF_N = 0>
__device__ __forceinline__ void dx_half(uint8_t* sm, uint32_t sb, uint32_t tb, int rb, int lane,
                                        const float* rv, int valid, const GradParams& p, int tc0,
                                        int h, int col0, int ncols, uint32_t ddel = GS_DDEL,
                                        uint32_t gdx = GS_GDX) {
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
                ldb_mn(sb + ddel, 0, 8 * nt, 16 * ks, lane, b);
                mma16816(acc[nt - N0], a, b[0], b[1]);
                mma16816(acc[nt - N0 + 1], a, b[2], b[3]);
            } else {
                uint32_t b[2];
                ldb_mn1(sb + ddel, 8 * nt, 16 * ks, lane, b);
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
        *reinterpret_cast<uint32_t*>(sm + taddr_e(gdx, r, col, 0)) =
            pack2(-gm_lo * acc[i][0], -gm_lo * acc[i][1]);
        *reinterpret_cast<uint32_t*>(sm + taddr_e(gdx, r + 8, col, 0)) =
            pack2(-gm_hi * acc[i][2], -gm_hi * acc[i][3]);
    }
    if constexpr (HANDOFF != 0) {
        fence_proxy_async_smem();
        bar_arrive<HANDOFF, HANDOFF_N>();
    }
#pragma unroll
    for (int i = 0; i < N1 - N0; ++i) {
        const int col = 8 * (N0 + i) + 2 * t;
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

constexpr uint32_t SHALF = 16384;  // a 128-row half of a 128 x 128 state image

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

// ============================================================================
// Reverse chain on the fifth-generation tensor cores.  Grid (d_v slices, H_v,
// N); 288 threads (eight compute warps, one issuing warp); the chunks in
// reverse order through a 3-stage ring
// [Q h0 | K h0 | Q h1 | K h1 | dO slice | record], filled by warp 6's thread 0.
// Per chunk, with dS' the gradient of the state after it:
//   [Q; K] dS'                 tcgen05, M = 128: lanes 64-127 hold K dS'
//   [T_b^T; (M o QK^T)^T] dO   tcgen05, M = 128: lanes 64-127 hold (M o QK^T)^T dO
//   dDelta = (M o QK^T)^T dO + d o (K dS')     the warps on lanes 64-127
//   dX = T_b^T dDelta          warp-level mma.sync (T_b^T upper triangular);
//                              -gamma o dX to shared memory, then dV = dX out
//   dS = gamma_C dS' + Q^T (gamma o dO) + K^T (-gamma o dX)
//                              tcgen05, M = 128, both products into one
//                              accumulator (lane = d_k index)
// The products that read only dO (the second, and Q^T (gamma o dO)) are issued
// a chunk ahead: the second right behind [Q; K] dS', Q^T (gamma o dO) behind
// K^T (-gamma o dX) once the warps on lanes 0-63 have formed gamma o dO; only
// [Q; K] dS' and K^T (-gamma o dX) sit on the chain.  Every thread of the eight
// compute warps keeps half a row of dS in fp32, writes its bf16 copy (the next
// [Q; K] dS' operand) and, per chunk, its part of the bf16 image of dS' for the
// per-chunk gradients.  The ninth warp only issues the products (tcgen05.mma
// issue stalls while the pipe is busy, which held a compute warp back): the
// compute warps bar.arrive on a named barrier once an operand tile is written,
// and the issuer bar.syncs on it.  The compute warps leave the chunk loop only
// at its end, after their last arrive, so that the issuer's barriers always
// complete; the issuer reads the abort flag after the first barrier of each
// chunk (the previous chunk's last hand-off).
// ============================================================================
constexpr int GST_THREADS = 288;  // eight compute warps and the issuing warp
constexpr int GST_COMPUTE = 256;  // warps 0-7; warp 8's lane 0 issues
constexpr int GST_LOADER = 192;   // warp 6
// named barriers: the compute warps; -gamma o dX (and the next chunk's gamma o
// dO) ready; dS' ready (compute warps arrive, the issuer waits)
constexpr int GST_BAR = 1, GST_BAR_GDX = 2, GST_BAR_DSB = 3;
constexpr uint32_t GST_O = 4 * HALF, GST_REC = 5 * HALF;
constexpr uint32_t GST_STAGE = ((GST_REC + REC_BYTES + 1023) / 1024) * 1024;
constexpr uint32_t GST_TX = 5 * HALF + REC_BYTES;
constexpr uint32_t GST_DSB = GS_STAGES * GST_STAGE;  // dS' in bf16, 128 x 64, MN-major
constexpr uint32_t GST_DDEL = GST_DSB + 2 * HALF;    // dDelta, 64 x 64
constexpr uint32_t GST_GDX = GST_DDEL + HALF;        // -gamma o dX
constexpr uint32_t GST_GDO = GST_GDX + HALF;         // gamma o dO, two buffers
constexpr uint32_t GST_BARS = GST_GDO + 2 * HALF;    // full[3], a, o[2], u, drain
constexpr uint32_t GST_MISC = GST_BARS + 128;        // abort flag, TMEM base
constexpr uint32_t GST_SMEM = GST_MISC + 16 + 1024;
static_assert(GST_STAGE % 1024 == 0 && GST_DSB % 1024 == 0, "swizzled tiles sit on 1 KB");
static_assert(GST_SMEM <= 232448, "tcgen05 reverse chain shared memory budget");
// TMEM columns: K dS' (lanes 64-127 read), (M o QK^T)^T dO (two buffers), the
// dS increment (two buffers)
constexpr uint32_t GTM_A = 0, GTM_O = 64, GTM_U = 192, GTM_COLS = 512;

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* r) {
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]),
                   "=r"(u[6]), "=r"(u[7])
                 : "r"(taddr));
}
// N columns (a multiple of 8) of this thread's TMEM lane, pinned behind the wait.
template <int N>
__device__ __forceinline__ void tmem_row(uint32_t ta, float* v) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i) tmem_ld8(ta + 8 * i, v + 8 * i);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}
// Columns c0 .. c0 + N - 1 (multiples of 8) of row r of a 64-column MN-major
// 128B-swizzled bf16 tile, scaled by s.
template <int N>
__device__ __forceinline__ void put_row(uint8_t* sm, uint32_t tile, int r, int c0, const float* v,
                                        float s) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i)
        *reinterpret_cast<uint4*>(sm + taddr(tile, r, c0 + 8 * i, 0)) =
            make_uint4(pack2(s * v[8 * i], s * v[8 * i + 1]), pack2(s * v[8 * i + 2], s * v[8 * i + 3]),
                       pack2(s * v[8 * i + 4], s * v[8 * i + 5]),
                       pack2(s * v[8 * i + 6], s * v[8 * i + 7]));
}

template <int NS, typename IO>
__global__ void __launch_bounds__(GST_THREADS, 1)
    grad_state_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                         const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_do, const GradParams p) {
    static_assert(NS == 32 || NS == 48 || NS == 64, "slice width");
    constexpr int HN = NS / 2, NT = NS / 8;
    constexpr uint32_t ID_KM = idesc_bf16(128, NS, 0, 1);  // K-major A, MN-major B
    constexpr uint32_t ID_MM = idesc_bf16(128, NS, 1, 1);  // MN-major A and B
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + GST_BARS);
    uint64_t* bar_a = bars + GS_STAGES;
    uint64_t* bar_o = bars + GS_STAGES + 1;  // two: chunk index i commits to bar_o[i & 1]
    uint64_t* bar_u = bars + GS_STAGES + 3;
    uint64_t* drain_bar = bars + GS_STAGES + 4;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + GST_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + GST_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool issuer = tid >= GST_COMPUTE;  // warp 8
    const int quad = warp & 3;               // TMEM lanes 32 quad .. + 31
    const int c_lo = ((warp >> 2) & 1) * HN; // this warp's half of the slice's columns
    const int row = 32 * quad + lane;        // my row of an M = 128 product (a d_k index)
    const int h = blockIdx.y, n = blockIdx.z;
    const int hq = h / (p.H_v / p.H_qk);
    const int col0 = blockIdx.x * NS;
    const int ncols = min(NS, D - col0);
    const int t_beg = p.cu_seqlens[n], t_end = p.cu_seqlens[n + 1];
    const int nchunks = (t_end - t_beg + C - 1) / C;

    if (tid == 0) {
        for (int i = 0; i < GS_STAGES + 5; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, GTM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(32 * quad) << 16) + c_lo;  // my lanes, my columns

    // chunk index i is chunk nchunks - 1 - i, in ring stage i % GS_STAGES
    auto issue = [&](int i) {
        const int c = nchunks - 1 - i, s = i % GS_STAGES;
        uint8_t* st = sm + s * GST_STAGE;
        const int y = t_beg + c * C;
        uint64_t* full = &bars[s];
        mbar_arrive_expect_tx(full, GST_TX);
        tma_load_2d(st, &map_q, hq * D, y, full);
        tma_load_2d(st + HALF, &map_k, hq * D, y, full);
        tma_load_2d(st + 2 * HALF, &map_q, hq * D + 64, y, full);
        tma_load_2d(st + 3 * HALF, &map_k, hq * D + 64, y, full);
        tma_load_2d(st + GST_O, &map_do, h * D + col0, y, full);
        bulk_load(st + GST_REC, p.records + (size_t)(record_slot(n, y) * p.H_v + h) * REC_BYTES,
                  REC_BYTES, full);
    };
    int issued = 0;
    if (tid == GST_LOADER)
        for (; issued < min(GS_STAGES, nchunks); ++issued) issue(issued);

    // gamma o dO of chunk index i into GDO[i & 1] (warps on lanes 0-63: token row
    // `row`; zero past the sequence end, where the rows belong to the next one)
    auto gamma_do = [&](int i) -> bool {
        const int s = i % GS_STAGES;
        const bool landed = mbar_wait(&bars[s], (i / GS_STAGES) & 1, abort_flag);
        const uint8_t* stp = sm + s * GST_STAGE;
        const float* rv = reinterpret_cast<const float*>(stp + GST_REC + REC_VEC);
        const int valid = min(C, t_end - (t_beg + (nchunks - 1 - i) * C));
        const float gm = row < valid ? rv[row] : 0.f;
        float x[HN];
#pragma unroll
        for (int q = 0; q < HN / 8; ++q) {
            const uint4 u = *reinterpret_cast<const uint4*>(stp + taddr(GST_O, row, c_lo + 8 * q, 0));
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
                x[8 * q + 2 * e] = f.x;
                x[8 * q + 2 * e + 1] = f.y;
            }
        }
        put_row<HN>(sm, GST_GDO + (i & 1) * HALF, row, c_lo, x, gm);
        fence_proxy_async_smem();
        return landed;
    };

    if (issuer) {
        // ---- the issuing warp: lane 0 issues, the warp takes the barriers
        const bool lead = lane == 0;
        // (lead) the products of chunk index i that read only dO:
        // [T_b^T; (M o QK^T)^T] dO into O[i & 1], and Q^T (gamma o dO) into U[i & 1]
        auto issue_mdo = [&](int i) {
            const uint32_t st = sb + (i % GS_STAGES) * GST_STAGE;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GTM_O + 64 * (i & 1),
                            sdesc_sw128(st + GST_REC + ks * 2048, HALF, 1024),
                            sdesc_sw128(st + GST_O + ks * 2048, 8192, 1024), ID_MM, ks > 0);
            mma_commit(&bar_o[i & 1]);
        };
        auto issue_qdo = [&](int i) {
            const uint32_t st = sb + (i % GS_STAGES) * GST_STAGE;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GTM_U + 64 * (i & 1), sdesc_sw128(st + ks * 2048, 2 * HALF, 1024),
                            sdesc_sw128(sb + GST_GDO + (i & 1) * HALF + ks * 2048, 8192, 1024),
                            ID_MM, ks > 0);
        };
        __syncthreads();  // the first dS' tile and gamma o dO are written
        if (nchunks > 0 && lead) {
            tc_fence_after();
            issue_mdo(0);
            issue_qdo(0);
        }
        bool stopped = false;
        for (int i = 0; i < nchunks; ++i) {
            const int s = i % GS_STAGES;
            const uint32_t st = sb + s * GST_STAGE;
            const uint32_t par = i & 1;
            if (i > 0) {
                bar_sync<GST_BAR_DSB, GST_THREADS>();  // the compute warps wrote dS'
                if (*abort_flag) {  // they left the loop after that arrive
                    stopped = true;
                    break;
                }
            }
            const bool landed = mbar_wait(&bars[s], (i / GS_STAGES) & 1, abort_flag);
            if (lead && landed) {  // [Q; K] dS'
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16_ss(tmem + GTM_A,
                                sdesc_sw128(st + (ks >> 2) * 2 * HALF + (ks & 3) * 32, 16, 1024),
                                sdesc_sw128(sb + GST_DSB + ks * 2048, 8192, 1024), ID_KM, ks > 0);
                mma_commit(bar_a);
            }
            // the next chunk's (M o QK^T)^T dO right behind, so that it runs while
            // dDelta is formed, not beside dX's mma.sync products
            if (i + 1 < nchunks &&
                mbar_wait(&bars[(i + 1) % GS_STAGES], ((i + 1) / GS_STAGES) & 1, abort_flag) && lead) {
                tc_fence_after();
                issue_mdo(i + 1);
            }
            bar_sync<GST_BAR_GDX, GST_THREADS>();  // -gamma o dX is written
            if (lead) {  // K^T (-gamma o dX) on top of Q^T (gamma o dO), then the next Q^T (gamma o dO)
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tmem + GTM_U + 64 * par,
                                sdesc_sw128(st + HALF + ks * 2048, 2 * HALF, 1024),
                                sdesc_sw128(sb + GST_GDX + ks * 2048, 8192, 1024), ID_MM, true);
                mma_commit(bar_u);
                if (i + 1 < nchunks) issue_qdo(i + 1);
            }
        }
        // the compute warps' arrive after the last chunk
        if (nchunks > 0 && !stopped) bar_sync<GST_BAR_DSB, GST_THREADS>();
        if (lead) {  // no product may still run when TMEM is freed (bounded wait)
            mma_commit(drain_bar);
            mbar_wait_drain(drain_bar, 0);
        }
    } else {
        // ---- the compute warps
        // dS: row `row`, columns col0 + c_lo .. + HN - 1, fp32 (dS_final to start)
        float G[HN];
        {
            const float* s0 = p.dS_final
                                  ? p.dS_final + (((size_t)n * p.H_v + h) * D + row) * D + col0 + c_lo
                                  : nullptr;
#pragma unroll
            for (int j = 0; j < HN; ++j) G[j] = (s0 && c_lo + j < ncols) ? s0[j] : 0.f;
            put_row<HN>(sm, GST_DSB, row, c_lo, G, 1.f);
            fence_proxy_async_smem();
        }
        bool ok = true;
        if (quad < 2 && nchunks > 0) ok = gamma_do(0);
        tc_fence_before();
        __syncthreads();  // the issuer starts

        for (int i = 0; i < nchunks; ++i) {
            const int c = nchunks - 1 - i, s = i % GS_STAGES;
            const uint32_t st = sb + s * GST_STAGE;
            const uint8_t* stp = sm + s * GST_STAGE;
            const uint32_t par = i & 1;
            const float* rv = reinterpret_cast<const float*>(stp + GST_REC + REC_VEC);
            const int tc0 = t_beg + c * C;
            const int valid = min(C, t_end - tc0);
            ok = mbar_wait(&bars[s], (i / GS_STAGES) & 1, abort_flag) && ok;
            const float g_C = rv[128];
            {  // the gradient of the state after this chunk, as its bf16 image
                uint8_t* sv =
                    p.dS_saved + ((size_t)record_slot(n, tc0) * p.H_v + h) * STATE_IMAGE_BYTES;
#pragma unroll
                for (int q = 0; q < HN / 8; ++q)
                    if (c_lo + 8 * q < ncols)
                        *reinterpret_cast<uint4*>(sv + taddr(0, row, col0 + c_lo + 8 * q, 2 * HALF)) =
                            make_uint4(pack2(G[8 * q], G[8 * q + 1]), pack2(G[8 * q + 2], G[8 * q + 3]),
                                       pack2(G[8 * q + 4], G[8 * q + 5]),
                                       pack2(G[8 * q + 6], G[8 * q + 7]));
            }
            if (quad >= 2) {  // dDelta, token row row - 64
                ok = mbar_wait(&bar_o[par], (i >> 1) & 1, abort_flag) && ok;
                ok = mbar_wait(bar_a, par, abort_flag) && ok;
                tc_fence_after();
                float a[HN], o[HN];  // both reads behind one wait
#pragma unroll
                for (int i = 0; i < HN / 8; ++i) {
                    tmem_ld8(tl + GTM_A + 8 * i, a + 8 * i);
                    tmem_ld8(tl + GTM_O + 64 * par + 8 * i, o + 8 * i);
                }
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < HN; ++j) {
                    asm volatile("" : "+f"(a[j]));
                    asm volatile("" : "+f"(o[j]));
                }
                const float d = rv[64 + row - 64];  // zero past the sequence end
#pragma unroll
                for (int j = 0; j < HN; ++j) a[j] = fmaf(d, a[j], o[j]);
                put_row<HN>(sm, GST_DDEL, row - 64, c_lo, a, 1.f);  // read by ldmatrix only
                tc_fence_before();
            } else if (i + 1 < nchunks) {  // the next chunk's gamma o dO (read after the
                ok = gamma_do(i + 1) && ok;  // -gamma o dX hand-off)
            }
            bar_sync<GST_BAR, GST_COMPUTE>();  // dDelta is complete

            // dX = T_b^T dDelta: warp (quad, column half) takes rows 16 quad .. + 15
            // (-gamma o dX is handed to the issuing warp before dV goes out)
            if (warp < 4)
                dx_half<NT, 0, IO, GST_BAR_GDX, GST_THREADS>(sm, sb, st + GST_REC + REC_TB, quad, lane,
                                                             rv, valid, p, tc0, h, col0, ncols,
                                                             GST_DDEL, GST_GDX);
            else
                dx_half<NT, 1, IO, GST_BAR_GDX, GST_THREADS>(sm, sb, st + GST_REC + REC_TB, quad, lane,
                                                             rv, valid, p, tc0, h, col0, ncols,
                                                             GST_DDEL, GST_GDX);

            // dS = gamma_C dS' + Q^T (gamma o dO) + K^T (-gamma o dX)
            ok = mbar_wait(bar_u, par, abort_flag) && ok;
            tc_fence_after();
            {
                float u[HN];
                tmem_row<HN>(tl + GTM_U + 64 * par, u);
#pragma unroll
                for (int j = 0; j < HN; ++j) G[j] = fmaf(g_C, G[j], u[j]);
                put_row<HN>(sm, GST_DSB, row, c_lo, G, 1.f);
                fence_proxy_async_smem();
            }
            tc_fence_before();
            bar_arrive<GST_BAR_DSB, GST_THREADS>();
            // every product and read of this stage is done: it takes chunk index i + 3
            // (the compute warps leave the loop only here, after their last arrive)
            if (!bar_and<GST_BAR, GST_COMPUTE>(ok)) break;
            if (tid == GST_LOADER && i + GS_STAGES < nchunks) issue(issued++);
        }
        if (p.dS0 && !*abort_flag) {
            float* d0 = p.dS0 + (((size_t)n * p.H_v + h) * D + row) * D + col0 + c_lo;
#pragma unroll
            for (int j = 0; j < HN / 4; ++j)
                if (c_lo + 4 * j < ncols)
                    reinterpret_cast<float4*>(d0)[j] =
                        make_float4(G[4 * j], G[4 * j + 1], G[4 * j + 2], G[4 * j + 3]);
        }
        if (tid == GST_LOADER)
            for (int i = max(0, issued - GS_STAGES); i < issued; ++i)
                mbar_wait_drain(&bars[i % GS_STAGES], (i / GS_STAGES) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, GTM_COLS);
    }
}

template <int NS, typename IO>
cudaError_t launch_grad_state_tc(const CUtensorMap& mq, const CUtensorMap& mk,
                                 const CUtensorMap& mo, const GradParams& prm, cudaStream_t stream) {
    auto kern = grad_state_tc_kernel<NS, IO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GST_SMEM);
    if (e != cudaSuccess) return e;
    kern<<<dim3((D + NS - 1) / NS, prm.H_v, prm.N), GST_THREADS, GST_SMEM, stream>>>(mq, mk, mo, prm);
    return cudaGetLastError();
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

// ============================================================================
// Per-chunk gradients on the fifth-generation tensor cores.  Grid (record
// slots, H_qk); 256 threads; one CTA per SM (all 512 TMEM columns).  Per value
// head of the query/key head, twelve steps (numbered in the kernel) form
// K S and Q S, X, Delta, dDelta, dX, P, the dQ and dK terms, dT_b, Y and E,
// and the gate gradients, following the formulas at the top of this file.
// Each product is a tcgen05.mma group issued by thread 0, its accumulator in
// tensor memory:
//   columns   0-127  dQ, accumulated over the query/key head's value heads
//   columns 128-255  dK, likewise
//   columns 256-383  T1 and 384-511 T2: one step's products
// Warp w reads TMEM lanes 32 (w % 4) .. + 31 (an M = 128 product's rows, or,
// in its lanes 0-15, rows 16 (w % 4) .. + 15 of an M = 64 product) and the
// column half w / 4.  Every operand is one of the kernel's 128B-swizzled bf16
// tiles: a tile stored [rows][columns] is K-major for a product contracting
// over its columns and MN-major for one contracting over its rows, so the
// transposes of the chunk form (T_b^T, (M o QK^T)^T, P^T, E^T, S^T, dS'^T,
// X^T, Delta^T) are descriptors, not copies.
// ============================================================================
constexpr uint32_t GT_KQ = 0;                   // K h0 | Q h0 | K h1 | Q h1 (token rows)
constexpr uint32_t GT_V = 4 * HALF;             // V, then X in place (halves HALF apart)
constexpr uint32_t GT_O = 6 * HALF;             // dO, then gamma o dO in place
constexpr uint32_t GT_S = 8 * HALF;             // S image (halves SHALF apart)
constexpr uint32_t GT_DS = GT_S + 2 * SHALF;    // dS' image
constexpr uint32_t GT_REC = GT_DS + 2 * SHALF;  // the chunk's operator record (bf16 tiles)
constexpr uint32_t GT_DEL = GT_REC + ((REC_BYTES + 1023) / 1024) * 1024;  // Delta, then d o Delta
constexpr uint32_t GT_DDEL = GT_DEL + 2 * HALF;                          // dDelta
constexpr uint32_t GT_DX = GT_DDEL + 2 * HALF;  // K S in bf16, then -gamma o dX
constexpr uint32_t GT_PY = GT_DX + 2 * HALF;    // P, then Y (64 x 64)
constexpr uint32_t GT_TE = GT_PY + HALF;        // dT_b, then E (64 x 64)
constexpr uint32_t GT_F = GT_TE + HALF;         // fp32: g2[64], dg[64], dbt[64], misc[64]
constexpr uint32_t GT_BAR = GT_F + 4 * 64 * 4;  // K/Q copies, head copies, record copy,
                                                // products, drain
constexpr uint32_t GT_MISC = GT_BAR + 40;       // abort flag, TMEM base
constexpr uint32_t GT_SMEM = GT_MISC + 16 + 1024;
static_assert(GT_SMEM <= 232448, "tcgen05 per-chunk gradient shared memory budget");
static_assert(GT_DEL % 1024 == 0, "swizzled tiles sit on 1 KB");
constexpr uint32_t GT_DQ = 0, GT_DK = 128, GT_T1 = 256, GT_T2 = 384, GT_COLS = 512;

// K-major operand: tile rows index M (or N), tile columns the contraction, in
// 64-column halves hs bytes apart; k step ks covers columns 16 ks .. + 15.
__device__ __forceinline__ uint64_t kdesc(uint32_t tile, uint32_t hs, int ks) {
    return sdesc_sw128(tile + (uint32_t)(ks >> 2) * hs + (uint32_t)(ks & 3) * 32, 16, 1024);
}
// MN-major operand: tile rows index the contraction, tile columns M (or N), in
// 64-column blocks bs bytes apart; k step ks covers rows 16 ks .. + 15.
__device__ __forceinline__ uint64_t mdesc(uint32_t tile, uint32_t bs, int ks) {
    return sdesc_sw128(tile + (uint32_t)ks * 2048, bs, 1024);
}

// An M = 64 accumulator's rows 16 (w % 4) .. + 15 for warp w, in the m16n8
// fragment layout of mma.sync (thread t: rows t / 4 and t / 4 + 8, columns
// 2 (t % 4) and 2 (t % 4) + 1 of each 8-column group): NT groups from TMEM
// address ta, by tcgen05.ld.16x256b (layout checked by a probe on the B200).
__device__ __forceinline__ void tld_frag4(uint32_t ta, float (*acc)[4]) {
    uint32_t* u = reinterpret_cast<uint32_t*>(&acc[0][0]);
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]),
          "=r"(u[14]), "=r"(u[15])
        : "r"(ta));
}
// (The empty asm statements after each wait keep every use of the values read
// behind the tcgen05.wait::ld.)
template <int NT>
__device__ __forceinline__ void tld_frag(uint32_t ta, float (*acc)[4]) {
    static_assert(NT % 4 == 0, "groups of four 8-column groups");
#pragma unroll
    for (int i = 0; i < NT / 4; ++i) tld_frag4(ta + 32 * i, acc + 4 * i);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) asm volatile("" : "+f"(acc[i][e]));
}

// Two such reads (NT groups each) behind one wait.
template <int NT>
__device__ __forceinline__ void tld_frag2(uint32_t ta, float (*acc)[4], uint32_t tb,
                                          float (*bcc)[4]) {
    static_assert(NT % 4 == 0, "groups of four 8-column groups");
#pragma unroll
    for (int i = 0; i < NT / 4; ++i) tld_frag4(ta + 32 * i, acc + 4 * i);
#pragma unroll
    for (int i = 0; i < NT / 4; ++i) tld_frag4(tb + 32 * i, bcc + 4 * i);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            asm volatile("" : "+f"(acc[i][e]));
            asm volatile("" : "+f"(bcc[i][e]));
        }
}

// Row sums (over the fragment's columns) of v into dst[row] (shared memory,
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
// Column sums (over the fragment's 16 rows) of v into dst[n0 + column], scaled by s.
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
// A fragment as bf16 into a 64-column swizzled tile: rows m0 + g (+8), columns
// c0 + 8 nt + 2 t (+1).
template <int NT>
__device__ __forceinline__ void store_frag_cols(uint8_t* smem, uint32_t base_off, int m0, int c0,
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

// 16 bf16 values at row r, columns c .. c + 15 (c a multiple of 8) of a swizzled
// tile whose 64-column halves lie hs bytes apart.
__device__ __forceinline__ void ld16_bf16(const uint8_t* sm, uint32_t tile, uint32_t hs, int r,
                                          int c, float* v) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint4 u = *reinterpret_cast<const uint4*>(sm + taddr(tile, r, c + 8 * h, hs));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
            v[8 * h + 2 * e] = f.x;
            v[8 * h + 2 * e + 1] = f.y;
        }
    }
}
__device__ __forceinline__ void st16_bf16(uint8_t* sm, uint32_t tile, uint32_t hs, int r, int c,
                                          const float* v, float s) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
        *reinterpret_cast<uint4*>(sm + taddr(tile, r, c + 8 * h, hs)) =
            make_uint4(pack2(s * v[8 * h], s * v[8 * h + 1]), pack2(s * v[8 * h + 2], s * v[8 * h + 3]),
                       pack2(s * v[8 * h + 4], s * v[8 * h + 5]),
                       pack2(s * v[8 * h + 6], s * v[8 * h + 7]));
}
// 16 consecutive values to global memory in 16-byte stores (dst 16-byte aligned).
template <typename IO>
__device__ __forceinline__ void store16(IO* dst, const float* v);
template <>
__device__ __forceinline__ void store16<float>(float* dst, const float* v) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
template <>
__device__ __forceinline__ void store16<__nv_bfloat16>(__nv_bfloat16* dst, const float* v) {
#pragma unroll
    for (int i = 0; i < 2; ++i)
        reinterpret_cast<uint4*>(dst)[i] =
            make_uint4(pack2(v[8 * i], v[8 * i + 1]), pack2(v[8 * i + 2], v[8 * i + 3]),
                       pack2(v[8 * i + 4], v[8 * i + 5]), pack2(v[8 * i + 6], v[8 * i + 7]));
}
// Two 16-column TMEM reads of this warp's lanes, then the wait.
__device__ __forceinline__ void tld2x16(uint32_t a0, float* v0, uint32_t a1, float* v1) {
    tmem_ld16(a0, v0);
    tmem_ld16(a1, v1);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        asm volatile("" : "+f"(v0[i]));
        asm volatile("" : "+f"(v1[i]));
    }
}

template <typename IO>
__global__ void __launch_bounds__(256, 1)
    grad_chunk_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                         const __grid_constant__ CUtensorMap map_k,
                         const __grid_constant__ CUtensorMap map_v,
                         const __grid_constant__ CUtensorMap map_do, const GradParams p) {
    constexpr uint32_t ID_128_KM = idesc_bf16(128, 128, 0, 1);  // M = 128, N = 128, A K-major, B MN-major
    constexpr uint32_t ID_KM = idesc_bf16(64, 128, 0, 1);
    constexpr uint32_t ID_MM = idesc_bf16(64, 128, 1, 1);
    constexpr uint32_t ID_KK = idesc_bf16(64, 128, 0, 0);
    constexpr uint32_t ID64_KK = idesc_bf16(64, 64, 0, 0);      // N = 64
    constexpr uint32_t ID64_MM = idesc_bf16(64, 64, 1, 1);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + GT_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + GT_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + GT_MISC + 4);
    float* g2 = reinterpret_cast<float*>(sm + GT_F);  // cumulative log2 gates
    float* dg = g2 + 64;                              // gradient w.r.t. g (natural log)
    float* dbt = g2 + 128;                            // dbeta * beta
    float* misc = g2 + 192;                           // [0] sum ddv, [1] <dS', S>
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, chalf = warp >> 2;
    const bool lo16 = lane < 16;
    const int r64 = 16 * quad + (lane & 15);  // my row of an M = 64 product in lanes < 16
    const int m0 = 16 * quad, g = lane >> 2, t4 = lane & 3;  // the same product as fragments
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
        for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, GT_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tq = tmem + ((uint32_t)(32 * quad) << 16);  // my lane quadrant

    // value head vh's V, dO and saved states on bars[1]; its record on bars[2]
    auto issue_head = [&](int vh) {
        const int h = hq * group + vh;
        const size_t so = ((size_t)slot * p.H_v + h) * STATE_IMAGE_BYTES;
        mbar_arrive_expect_tx(&bars[1], 4 * HALF + 2 * STATE_IMAGE_BYTES);
        tma_load_2d(sm + GT_V, &map_v, h * D, tc0, &bars[1]);
        tma_load_2d(sm + GT_V + HALF, &map_v, h * D + 64, tc0, &bars[1]);
        tma_load_2d(sm + GT_O, &map_do, h * D, tc0, &bars[1]);
        tma_load_2d(sm + GT_O + HALF, &map_do, h * D + 64, tc0, &bars[1]);
        bulk_load(sm + GT_S, p.S_saved + so, STATE_IMAGE_BYTES, &bars[1]);
        bulk_load(sm + GT_DS, p.dS_saved + so, STATE_IMAGE_BYTES, &bars[1]);
    };
    auto issue_rec = [&](int vh) {
        const int h = hq * group + vh;
        mbar_arrive_expect_tx(&bars[2], REC_BYTES);
        bulk_load(sm + GT_REC, p.records + (size_t)(slot * p.H_v + h) * REC_BYTES, REC_BYTES,
                  &bars[2]);
    };
    int heads = 0, recs = 0;  // copies issued (thread 0)
    uint32_t groups = 0;      // product groups committed (every thread counts them)
    // After a failed wait: every copy and product in flight completes (bounded
    // waits), then the tensor memory is freed.
    auto leave = [&]() {
        if (tid == 0) {
            mbar_wait_drain(&bars[0], 0);
            if (heads > 0) mbar_wait_drain(&bars[1], (heads - 1) & 1);
            if (recs > 0) mbar_wait_drain(&bars[2], (recs - 1) & 1);
            mma_commit(&bars[4]);  // a barrier of its own: its first phase covers every product
            mbar_wait_drain(&bars[4], 0);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            tmem_dealloc(tmem, GT_COLS);
        }
    };
    // commit the products thread 0 issued since the last commit; every thread waits
    auto commit_wait = [&]() -> bool {
        if (tid == 0) mma_commit(&bars[3]);
        const bool ok = mbar_wait(&bars[3], groups & 1, abort_flag);
        ++groups;
        tc_fence_after();
        return ok;
    };
    // generic writes of operand tiles are made visible to the tensor cores, and
    // TMEM reads are ordered before the next products
    auto publish = [&](bool ok) -> bool {
        fence_proxy_async_smem();
        tc_fence_before();
        return __syncthreads_and(ok);
    };

    if (tid == 0) {
        mbar_arrive_expect_tx(&bars[0], 4 * HALF);
        tma_load_2d(sm + GT_KQ, &map_k, hq * D, tc0, &bars[0]);
        tma_load_2d(sm + GT_KQ + HALF, &map_q, hq * D, tc0, &bars[0]);
        tma_load_2d(sm + GT_KQ + 2 * HALF, &map_k, hq * D + 64, tc0, &bars[0]);
        tma_load_2d(sm + GT_KQ + 3 * HALF, &map_q, hq * D + 64, tc0, &bars[0]);
        issue_head(0);
        issue_rec(0);
        heads = recs = 1;
    }
    bool ok = mbar_wait(&bars[0], 0, abort_flag);
    if (!__syncthreads_and(ok)) {
        leave();
        return;
    }
    if (valid < C) {  // rows past the sequence end belong to the next sequence: zero them
        for (int i = tid; i < 4 * 64 * 8; i += 256) {
            const int tile = i / 512, row = (i >> 3) & 63, ch = i & 7;
            if (row >= valid)
                *reinterpret_cast<uint4*>(sm + GT_KQ + tile * HALF + row * 128 + ch * 16) =
                    make_uint4(0, 0, 0, 0);
        }
    }

    // warp 1 holds a value head's gates in registers, loaded one head ahead (lane l:
    // tokens 2l, 2l+1; zero past the sequence end).  (Not warp 0: its thread 0
    // issues the products, and tcgen05.mma issue stalls while the pipe is busy.)
    float la[2] = {0.f, 0.f}, be[2] = {0.f, 0.f};
    auto load_gates = [&](int vh) {
        const int h = hq * group + vh;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const bool in = 2 * lane + e < valid;
            la[e] = in ? p.log_alpha[(size_t)(tc0 + 2 * lane + e) * p.H_v + h] : 0.f;
            be[e] = in ? p.beta[(size_t)(tc0 + 2 * lane + e) * p.H_v + h] : 0.f;
        }
    };
    if (warp == 1) load_gates(0);

    for (int vh = 0; vh < group; ++vh) {
        const int h = hq * group + vh;
        if (tid < 64) {
            dg[tid] = 0.f;
            dbt[tid] = 0.f;
            misc[tid] = 0.f;
        }
        if (warp == 1) {  // inclusive scan of log alpha (log2 units)
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
            leave();
            return;
        }
        if (valid < C) {  // V and dO rows past the sequence end
            for (int i = tid; i < 4 * 64 * 8; i += 256) {
                const int tile = i / 512, row = (i >> 3) & 63, ch = i & 7;
                if (row >= valid)
                    *reinterpret_cast<uint4*>(sm + GT_V + tile * HALF + row * 128 + ch * 16) =
                        make_uint4(0, 0, 0, 0);
            }
        }
        const float* rv = reinterpret_cast<const float*>(sm + GT_REC + REC_VEC);
        const float gam_C = rv[128];
        const float gm_lo = rv[m0 + g], gm_hi = rv[m0 + g + 8];      // gamma of my fragment rows
        const float d_lo = rv[64 + m0 + g], d_hi = rv[64 + m0 + g + 8];  // d of my fragment rows
        const int c0 = 64 * chalf, p0 = 32 * chalf;  // my columns of the 128- and 64-wide products
        if (!publish(true)) {
            leave();
            return;
        }

        // 1. K S (kept for dg, as bf16 in the dX tile), Q S -> dg += gamma_r dO_r . (QS)_r;
        //    X = V - gamma o KS in place over V
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_ss(tmem + GT_T1, kdesc(sb + GT_KQ, 2 * HALF, ks), mdesc(sb + GT_S, SHALF, ks),
                            ID_128_KM, ks > 0);
        }
        {  // <dS', S>, for the gate gradient of the chunk's last row (while the product runs)
            float dot = tile_dot(sm + GT_S, sm + GT_DS, tid);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            if (lane == 0) atomicAdd(&misc[1], dot);
        }
        ok = commit_wait();
        {
            const int row = 32 * (quad & 1) + lane;  // token row
            const float gm = rv[row];
            float s = 0.f;
            float a4[4][16];  // the row's 64 columns, read with one wait
#pragma unroll
            for (int i = 0; i < 4; ++i) tmem_ld16(tq + GT_T1 + 64 * chalf + 16 * i, a4[i]);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int e = 0; e < 16; ++e) asm volatile("" : "+f"(a4[i][e]));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int col = 64 * chalf + 16 * i;
                float* a = a4[i];
                float b[16];
                if (quad < 2) {
                    ld16_bf16(sm, GT_V, HALF, row, col, b);
#pragma unroll
                    for (int e = 0; e < 16; ++e) b[e] -= gm * a[e];
                    st16_bf16(sm, GT_V, HALF, row, col, b, 1.f);
                    st16_bf16(sm, GT_DX, HALF, row, col, a, 1.f);
                } else {
                    ld16_bf16(sm, GT_O, HALF, row, col, b);
#pragma unroll
                    for (int e = 0; e < 16; ++e) s = fmaf(a[e], b[e], s);
                }
            }
            if (quad >= 2) atomicAdd(&dg[row], gm * s);
        }
        if (!publish(ok)) {
            leave();
            return;
        }

        // 2. Delta = T_b X
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GT_T2, kdesc(sb + GT_REC + REC_TB, HALF, ks),
                            mdesc(sb + GT_V, HALF, ks), ID_KM, ks > 0);
        }
        ok = commit_wait();
        {
            float acc[8][4];
            tld_frag<8>(tq + GT_T2 + c0, acc);
            store_acc_bf16<8>(sm, GT_DEL + chalf * HALF, 0, m0, acc, lane, 1.f, 1.f);
        }
        if (!publish(ok)) {
            leave();
            return;
        }

        // 3. dDelta = (M o QK^T)^T dO + d o (K dS');  ddv_r = d_r (K dS')_r . Delta_r
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_ss(tmem + GT_T1, kdesc(sb + GT_KQ, 2 * HALF, ks), mdesc(sb + GT_DS, SHALF, ks),
                            ID_KM, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GT_T2, mdesc(sb + GT_REC + REC_MQ, HALF, ks),
                            mdesc(sb + GT_O, HALF, ks), ID_MM, ks > 0);
        }
        ok = commit_wait();
        {
            float kd[8][4], acc[8][4], ddv[8][4];
            tld_frag2<8>(tq + GT_T1 + c0, kd, tq + GT_T2 + c0, acc);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int col = c0 + 8 * nt + 2 * t4;
                const float2 e_lo = ld_bf16x2(sm + taddr_e(GT_DEL, m0 + g, col, HALF));
                const float2 e_hi = ld_bf16x2(sm + taddr_e(GT_DEL, m0 + g + 8, col, HALF));
                ddv[nt][0] = kd[nt][0] * e_lo.x;
                ddv[nt][1] = kd[nt][1] * e_lo.y;
                ddv[nt][2] = kd[nt][2] * e_hi.x;
                ddv[nt][3] = kd[nt][3] * e_hi.y;
                acc[nt][0] = fmaf(d_lo, kd[nt][0], acc[nt][0]);
                acc[nt][1] = fmaf(d_lo, kd[nt][1], acc[nt][1]);
                acc[nt][2] = fmaf(d_hi, kd[nt][2], acc[nt][2]);
                acc[nt][3] = fmaf(d_hi, kd[nt][3], acc[nt][3]);
            }
            // -d_r ddv_r into dg_r; their total goes to dg of the last row (misc[0])
            add_row_sums<8>(dg, m0, ddv, lane, -d_lo, -d_hi);
            float tot = 0.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
                tot += d_lo * (ddv[nt][0] + ddv[nt][1]) + d_hi * (ddv[nt][2] + ddv[nt][3]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
            if (lane == 0) atomicAdd(&misc[0], tot);
            store_acc_bf16<8>(sm, GT_DDEL + chalf * HALF, 0, m0, acc, lane, 1.f, 1.f);
        }
        if (!publish(ok)) {
            leave();
            return;
        }

        // 4. dX = T_b^T dDelta;  dg -= gamma_r dX_r . KS_r;  the dX tile <- -gamma o dX
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GT_T1, mdesc(sb + GT_REC + REC_TB, HALF, ks),
                            mdesc(sb + GT_DDEL, HALF, ks), ID_MM, ks > 0);
        }
        ok = commit_wait();
        {
            float dx[8][4], w[8][4];
            tld_frag<8>(tq + GT_T1 + c0, dx);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int col = c0 + 8 * nt + 2 * t4;
                const float2 k_lo = ld_bf16x2(sm + taddr_e(GT_DX, m0 + g, col, HALF));
                const float2 k_hi = ld_bf16x2(sm + taddr_e(GT_DX, m0 + g + 8, col, HALF));
                w[nt][0] = dx[nt][0] * k_lo.x;
                w[nt][1] = dx[nt][1] * k_lo.y;
                w[nt][2] = dx[nt][2] * k_hi.x;
                w[nt][3] = dx[nt][3] * k_hi.y;
            }
            add_row_sums<8>(dg, m0, w, lane, -gm_lo, -gm_hi);
            store_acc_bf16<8>(sm, GT_DX + chalf * HALF, 0, m0, dx, lane, -gm_lo, -gm_hi);
        }
        if (!publish(ok)) {
            leave();
            return;
        }

        // 5. P = M o (dO Delta^T) (64 x 64); dg gets the rows and columns of
        //    P o (M o QK^T).  Then dO <- gamma o dO and Delta <- d o Delta in place
        //    (their last reads as they are were steps 3 and 5).
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_ss(tmem + GT_T2, kdesc(sb + GT_O, HALF, ks), kdesc(sb + GT_DEL, HALF, ks),
                            ID64_KK, ks > 0);
        }
        ok = commit_wait();
        {
            float acc[4][4], pm[4][4];
            tld_frag<4>(tq + GT_T2 + p0, acc);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + ((e >> 1) << 3), j = p0 + 8 * nt + 2 * t4 + (e & 1);
                    const float mrj = j <= r ? ex2(g2[r] - g2[j]) : 0.f;
                    const float2 qk = ld_bf16x2(sm + taddr_e(GT_REC + REC_MQ, r, j & ~1, 0));
                    pm[nt][e] = acc[nt][e] * ((e & 1) ? qk.y : qk.x);  // P o (M o QK^T)
                    acc[nt][e] *= mrj;
                }
            store_frag_cols<4>(sm, GT_PY, m0, p0, acc, lane);
            add_row_sums<4>(dg, m0, pm, lane, 1.f, 1.f);
            add_col_sums<4>(dg, p0, pm, lane, -1.f);
        }
        if (!publish(ok)) {
            leave();
            return;
        }

        // 6. dQ += P K + (gamma o dO) S^T
        // 7. dK += P^T Q + (-gamma o dX) S^T + (d o Delta) dS'^T
        // 8. dT_b = dDelta X^T (64 x 64)
        // The products that read neither dO nor Delta go first; the row scalings of
        // dO (by gamma) and Delta (by d) run meanwhile, then the rest follows.
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_ss(tmem + GT_T2, kdesc(sb + GT_DDEL, HALF, ks), kdesc(sb + GT_V, HALF, ks),
                            ID64_KK, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GT_DQ, kdesc(sb + GT_PY, HALF, ks),
                            mdesc(sb + GT_KQ, 2 * HALF, ks), ID_KM, vh > 0 || ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GT_DK, mdesc(sb + GT_PY, HALF, ks),
                            mdesc(sb + GT_KQ + HALF, 2 * HALF, ks), ID_MM, vh > 0 || ks > 0);
        }
        // (warps 1-7: warp 0's thread 0 is issuing the products above)
        for (int idx = tid - 32; warp > 0 && idx < 2 * 1024; idx += 224) {  // 16 bytes at a time
            const int t = idx >> 10, i = idx & 1023;
            const int row = (i >> 3) & 63;
            uint8_t* q = sm + (t ? GT_DEL : GT_O) + (i >> 9) * HALF + row * 128 + (i & 7) * 16;
            const float sc = t ? rv[64 + row] : rv[row];
            const uint4 u = *reinterpret_cast<const uint4*>(q);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
                o[e] = pack2(sc * f.x, sc * f.y);
            }
            *reinterpret_cast<uint4*>(q) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        if (!publish(true)) {
            leave();
            return;
        }
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_ss(tmem + GT_DQ, kdesc(sb + GT_O, HALF, ks), kdesc(sb + GT_S, SHALF, ks),
                            ID_KK, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_ss(tmem + GT_DK, kdesc(sb + GT_DX, HALF, ks), kdesc(sb + GT_S, SHALF, ks),
                            ID_KK, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_ss(tmem + GT_DK, kdesc(sb + GT_DEL, HALF, ks), kdesc(sb + GT_DS, SHALF, ks),
                            ID_KK, 1);
        }
        ok = commit_wait();
        // X, dO, both states and Delta are free: the next head's copies land during
        // steps 9-12
        if (tid == 0 && ok && vh + 1 < group) {
            issue_head(vh + 1);
            ++heads;
        }
        {  // dT_b to its tile; dbeta * beta gets the columns of dT_b o T_b
            float acc[4][4];
            tld_frag<4>(tq + GT_T2 + p0, acc);
            store_frag_cols<4>(sm, GT_TE, m0, p0, acc, lane);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + ((e >> 1) << 3), j = p0 + 8 * nt + 2 * t4 + (e & 1);
                    const float2 tv = ld_bf16x2(sm + taddr_e(GT_REC + REC_TB, r, j & ~1, 0));
                    acc[nt][e] *= (e & 1) ? tv.y : tv.x;
                }
            add_col_sums<4>(dbt, p0, acc, lane, 1.f);
        }
        if (!publish(ok)) {
            leave();
            return;
        }

        // 9. Y = dT_b T_b^T
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GT_T1, kdesc(sb + GT_TE, HALF, ks),
                            kdesc(sb + GT_REC + REC_TB, HALF, ks), ID64_KK, ks > 0);
        }
        ok = commit_wait();
        {
            float acc[4][4];
            tld_frag<4>(tq + GT_T1 + p0, acc);
            store_frag_cols<4>(sm, GT_PY, m0, p0, acc, lane);
        }
        if (!publish(ok)) {
            leave();
            return;
        }

        // 10. E = strict_lower(-T_b^T Y) o M;  K K^T;  E o KK into dbeta * beta (rows)
        //     and dg (rows +, columns -)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GT_T2, mdesc(sb + GT_REC + REC_TB, HALF, ks),
                            mdesc(sb + GT_PY, HALF, ks), ID64_MM, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_bf16_ss(tmem + GT_T2 + 64, kdesc(sb + GT_KQ, 2 * HALF, ks),
                            kdesc(sb + GT_KQ, 2 * HALF, ks), ID64_KK, ks > 0);
        }
        ok = commit_wait();
        // the record is free too (gamma_C is in a register)
        if (tid == 0 && ok && vh + 1 < group) {
            issue_rec(vh + 1);
            ++recs;
        }
        {
            float acc[4][4], kk[4][4];
            tld_frag2<4>(tq + GT_T2 + p0, acc, tq + GT_T2 + 64 + p0, kk);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = m0 + g + ((e >> 1) << 3), j = p0 + 8 * nt + 2 * t4 + (e & 1);
                    acc[nt][e] = j < r ? -acc[nt][e] * ex2(g2[r] - g2[j]) : 0.f;
                    kk[nt][e] *= acc[nt][e];
                }
            store_frag_cols<4>(sm, GT_TE, m0, p0, acc, lane);
            add_row_sums<4>(dbt, m0, kk, lane, 1.f, 1.f);
            add_row_sums<4>(dg, m0, kk, lane, 1.f, 1.f);
            add_col_sums<4>(dg, p0, kk, lane, -1.f);
        }
        if (!publish(ok)) {
            leave();
            return;
        }

        // 11. dK += E K + E^T K (committed with the next group)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GT_DK, kdesc(sb + GT_TE, HALF, ks),
                            mdesc(sb + GT_KQ, 2 * HALF, ks), ID_KM, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tmem + GT_DK, mdesc(sb + GT_TE, HALF, ks),
                            mdesc(sb + GT_KQ, 2 * HALF, ks), ID_MM, 1);
        }
        // 12. the gates: dg of the last row gets sum ddv + gamma_C <dS', S>;
        // dlog_alpha_t = sum_{r >= t} dg_r (dg holds the gradient w.r.t. g in
        // natural-log units); dbeta_j = (dbeta * beta)_j / beta_j
        if (warp == 1) {
            const float last = misc[0] + gam_C * misc[1];
            float d0 = dg[2 * lane], d1 = dg[2 * lane + 1];
            if (lane == 31) d1 += last;
            float s = d0 + d1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, s, off);
                if (lane + off < 32) s += y;
            }
            const float suf0 = s, suf1 = s - d0;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = 2 * lane + e;
                if (r < valid) {
                    const size_t gi = (size_t)(tc0 + r) * p.H_v + h;
                    p.dlog_alpha[gi] = e ? suf1 : suf0;
                    const float b = be[e];
                    p.dbeta[gi] = b != 0.f ? dbt[r] / b : 0.f;
                }
            }
            if (vh + 1 < group) load_gates(vh + 1);
        }
        __syncthreads();  // the next head's gates overwrite dg, dbt and misc
    }
    // dQ, dK of this chunk and query/key head (every value head of the group summed)
    ok = commit_wait();
    if (!__syncthreads_and(ok)) {
        leave();
        return;
    }
    IO* dq = static_cast<IO*>(p.dq);
    IO* dk = static_cast<IO*>(p.dk);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int col = 64 * chalf + 16 * i;
        float a[16], b[16];
        tld2x16(tq + GT_DQ + col, a, tq + GT_DK + col, b);
        if (lo16 && r64 < valid) {
            const size_t o = ((size_t)(tc0 + r64) * p.H_qk + hq) * D + col;
            store16<IO>(dq + o, a);
            store16<IO>(dk + o, b);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, GT_COLS);
    }
}

// The reverse chain (as many d_v slices as fit in one wave of one block per
// SM), then the per-chunk gradients; IO is the type of dq, dk and dv.
template <typename IO>
cudaError_t launch_grads(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mo, const GradParams& prm, long long units, int sms,
                         size_t slots, cudaStream_t stream) {
    // (at 48- and 64-column slices on tcgen05, as the forward chain)
    cudaError_t e = units * 4 <= sms ? launch_grad_state<32, IO>(mq, mk, mo, prm, stream)
                    : units * 3 <= sms ? launch_grad_state_tc<48, IO>(mq, mk, mo, prm, stream)
                                       : launch_grad_state_tc<64, IO>(mq, mk, mo, prm, stream);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(grad_chunk_tc_kernel<IO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GT_SMEM);
    if (e != cudaSuccess) return e;
    grad_chunk_tc_kernel<IO><<<dim3((unsigned)slots, prm.H_qk), 256, GT_SMEM, stream>>>(
        mq, mk, mv, mo, prm);
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
        F32ToBf16Batch cv{};  // the three copies in one launch
        for (int i = 0; i < 3; ++i) {
            cv.src[i] = static_cast<const float*>(src[i]);
            cv.dst[i] = reinterpret_cast<__nv_bfloat16*>(st);
            cv.n4[i] = cnt[i] / 4;
            dst[i] = st;
            st += up256(cnt[i] * 2);
        }
        f32_to_bf16_batch_kernel<<<592, 256, 0, stream>>>(cv);
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
        F32ToBf16Batch cv{};  // the four copies in one launch
        for (int i = 0; i < 4; ++i) {
            cv.src[i] = static_cast<const float*>(src[i]);
            cv.dst[i] = reinterpret_cast<__nv_bfloat16*>(st);
            cv.n4[i] = cnt[i] / 4;
            dst[i] = st;
            st += up256(cnt[i] * 2);
        }
        f32_to_bf16_batch_kernel<<<592, 256, 0, stream>>>(cv);
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
