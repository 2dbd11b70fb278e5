// gdn_prefill.cu -- chunked GDN prefill (sm_100a) in two kernels: a fully
// parallel pass over all chunks that computes each chunk's state-independent
// operators, and a sequential pass that carries the state through the chunks.
// Both stage their tiles with TMA / bulk copies into 128-byte-swizzled shared
// memory.
//
// Operation: the gated delta rule of the bjdmk.com.cn article (section 2.1,
// state-update formula) over packed sequences, with readout o_t = S_t^T q_t.
// The article says the recurrence is made chunk-parallel with the WY
// representation but prints no formulas; the chunk algebra used here is
// derived from the recurrence itself.  For a chunk of C = 64 tokens with entry
// state S (d_k x d_v), cumulative log-gates g_r = sum_{i<=r} log alpha_i,
// gamma_r = exp(g_r), d_r = exp(g_C - g_r) (zero past the sequence end):
//
//   A     = strict_lower( diag(beta) (M o K K^T) ),  M_rj = exp(g_r - g_j)
//   T     = (I + A)^{-1},   T_b = T diag(beta)                 (unit lower / lower)
//   X     = V - diag(gamma) K S
//   Delta = T_b X                                              (true write vectors)
//   O     = diag(gamma) Q S + (M o Q K^T) Delta
//   S    <- gamma_C S + K^T diag(d) Delta
//
// (Delta equals U - W S of the WY form with U = T_b V and W = T_b diag(gamma) K.)
//
// Pass 1, chunk_ops_kernel: one CTA per (chunk, query/key head).  Both grams
// K K^T and Q K^T come from one tcgen05 product [K; Q] K^T accumulated in
// tensor memory and are shared by the value heads of that query/key head.  Per
// value head two "solver" warps build A (the masks factor per 16-column block,
// so each entry left of the diagonal block costs two multiplies) and solve for
// T (fp32 forward substitution on the diagonal 16 x 16 blocks, tf32
// tensor-core block products for the rest), while two "writer" warps store
// M o Q K^T, then T diag(beta), as 128-byte-swizzled tiles of one "chunk
// operator" record together with gamma, d and gamma_C, straight from registers.
// The unsplit prefill writes the tiles in fp16, and its output pass then
// carries X and Delta in fp16 as well (11 significant bits against bf16's 8);
// the segmented prefill and the gradients' forward keep bf16.  The state S and
// d o Delta stay bf16 operands: they meet the bf16 K and Q tiles.
//
// Pass 2 (the prefill's outputs): one CTA per (sequence, value head, d_v slice
// of NS columns); the columns of S evolve independently, so slices need no
// communication.  state_tc_kernel runs the products on the fifth-generation
// tensor cores with the accumulators in tensor memory (the 48-column slices of
// the 16/48-head workload); state_pass_kernel runs them as warp-level mma.sync
// with the state in registers (other slice widths, the segmented prefill's
// first phase and the gradients' forward).
//
// Every mbarrier wait is bounded (gdn_common.cuh); every named barrier inside
// the chunk loop also votes on whether all of its threads are still healthy,
// so a timeout makes the CTA leave the loop together, drain its in-flight
// copies (bounded) and exit.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "gdn_common.cuh"
#include "gdn_internal.h"
#include "gdn_tiles.cuh"

namespace gdn {

namespace {

constexpr int kMaxSegments = 16;  // most segments per sequence the automatic choice takes
// ---- pass 1 ----
constexpr int P1_MAX_GROUP = 4;       // value heads per work item
constexpr int AF_LD = 68;             // fp32 row stride of A and T (conflict-free row writes)

// ---- pass 2 shared memory ----
constexpr int NSTAGE = 3;
constexpr int P2_CHAIN_WARPS = 8;
constexpr int P2_CHAIN_THREADS = P2_CHAIN_WARPS * 32;
constexpr int P2_THREADS = P2_CHAIN_THREADS;
constexpr int P2_LOADER = 128;                                 // thread that issues the copies
constexpr int BAR_CHAIN = 1;
// ring stage: K and Q (two 64-column halves each), V slice, operator record
constexpr uint32_t ST_K = 0, ST_Q = 2 * HALF, ST_V = 4 * HALF, ST_REC = 5 * HALF;
constexpr uint32_t STAGE_BYTES = ((ST_REC + REC_BYTES + 1023) / 1024) * 1024;
constexpr uint32_t STAGE_TX = 5 * HALF + REC_BYTES;           // bytes landing per stage
constexpr uint32_t P2_SB = NSTAGE * STAGE_BYTES;               // S in bf16, 128 x 64
constexpr uint32_t P2_X = P2_SB + 2 * HALF;                    // X, 64 x 64
constexpr uint32_t P2_DU = P2_X + HALF;                        // Delta
constexpr uint32_t P2_DD = P2_DU + HALF;                       // d o Delta
constexpr uint32_t P2_BAR = P2_DD + HALF;
enum Bar2 { B2_FULL = 0, NBAR2 = NSTAGE };
constexpr uint32_t P2_MISC = P2_BAR + NBAR2 * 8;
constexpr uint32_t P2_SMEM = P2_MISC + 16 + 1024;
static_assert(P2_SMEM <= 232448, "pass 2 shared memory budget");

struct PrefillParams {
    const float* log_alpha;
    const float* beta;
    const float* S0;
    const int32_t* cu_seqlens;
    void* o;
    float* S_final;
    uint8_t* records;  // chunk operator records, REC_BYTES each
    float* S_aux;      // P2_SEGMENT: the segment propagators; P2_SAVE: every
                       // chunk's entering state as a bf16 image [record slot, H_v]
    int H_qk, H_v;
    int N, T;
};

// ============================================================================
// Pass 1: chunk operators.  Grid (record slots, H_qk, batches of up to 4 value
// heads of that head); 128 threads, four CTAs per SM.  The grams come from one
// tcgen05 product [K; Q] K^T (M = 128, N = 64, K = 128) accumulated in tensor
// memory: TMEM lane r holds row r of K K^T (r < 64) or of Q K^T (r >= 64).
// Warps 0-1 (the
// solvers) read the K K^T rows, build A and solve for T = (I + A)^{-1} in fp32
// shared memory; warps 2-3 (the writers) read the Q K^T rows, store M o Q K^T
// and the gate vectors of the record, then store T diag(beta) once the solvers
// have finished T.  The solvers start the next value head's A while the
// writers store the previous head's T_b.  Records go to global memory straight
// from registers.  Once the grams are complete the K and Q tiles' shared memory
// holds A and T.
// ============================================================================
constexpr int CO_THREADS = 128;
constexpr uint32_t CO_KQ = 0;                       // [K h0 | Q h0 | K h1 | Q h1], 32 KB
constexpr uint32_t CO_AF = 0;                       // after the grams: A, fp32 64 x AF_LD
constexpr uint32_t CO_TF = 64 * AF_LD * 4;          //                  T, fp32 64 x AF_LD
constexpr uint32_t CO_XS = 2 * 64 * AF_LD * 4;      // block-product scratch per solver warp
constexpr int CO_XS_FLOATS = 16 * 36;
constexpr uint32_t CO_VEC = CO_XS + 2 * CO_XS_FLOATS * 4;  // per value head: g[64] (log2), beta[64],
                                                    // w[64] = exp2(g_{16J+15} - g_j), J = j / 16
constexpr int CO_VEC_FLOATS = 192;
constexpr uint32_t CO_BAR = CO_VEC + P1_MAX_GROUP * CO_VEC_FLOATS * 4;  // K/Q copies, grams
constexpr uint32_t CO_MISC = CO_BAR + 16;           // abort flag, TMEM base
constexpr uint32_t CO_SMEM = CO_MISC + 16 + 1024;
constexpr uint32_t CO_TM_COLS = 64;
static_assert(CO_XS >= 4 * HALF, "the K and Q tiles lie inside A and T");
static_assert(4 * (CO_SMEM + 1024) <= 233472, "four pass-1 CTAs per SM");
// named barriers of pass 1 (0 is __syncthreads)
constexpr int CO_BAR_SOLVE = 1;  // the two solver warps
constexpr int CO_BAR_TDONE = 2;  // solvers -> writers: T is complete
constexpr int CO_BAR_TFREE = 3;  // writers -> solvers: T has been read


// Two values as a packed pair of the chunk-operator records' tile type: fp16
// (F16) for the unsplit prefill's output passes, whose products T_b X and
// [T_b; M o Q K^T] Delta then take fp16 operands; bf16 for every other reader.
template <bool F16>
__device__ __forceinline__ uint32_t packr(float lo, float hi) {
    return F16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

// Values read from tensor memory stay behind the tcgen05.wait::ld that follows
// the reads: an empty asm on each makes every later use depend on it.
template <int N>
__device__ __forceinline__ void pin_after_wait(float* v) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}

// tf32 rounding of an fp32 value, kept as fp32 (the low mantissa bits cleared)
__device__ __forceinline__ float tf32r(float x) { return __uint_as_float(to_tf32(x)); }
// The decay mask M_rj = exp2(g_r - g_j) (j <= r, g in log2 units) of a row r in
// 16-row block R.  Left of the diagonal block (column block J < R) it factors as
// exp2(g_r - g_e) * w_j with g_e = g_{16J+15} and w_j = exp2(g_e - g_j): both
// factors are at most 1, so nothing overflows whatever the gates, and the row
// pays one exponential per block.  In the diagonal block each entry takes its
// own exponential of g_r - g_j <= 0.
//
// Row r = 32 W + lane of A = strict_lower(diag(beta) (M o K K^T)), rounded to
// tf32, into Af: the blocks left of the diagonal block and the diagonal block
// (zeros on and above the diagonal).  Blocks right of it are never read.
// tm_row addresses row r of K K^T in tensor memory, read one 16-column block at
// a time; lanes 16-31 lie in row block 2W + 1, lanes 0-15 in 2W.
__device__ __forceinline__ void build_a(float* Af, uint32_t tm_row, const float* s_g,
                                        const float* s_b, const float* s_w, int W, int lane) {
    const int r = 32 * W + lane;
    const bool hi = lane >= 16;
    const float g_r = s_g[r], b_r = s_b[r];
    float* arow = Af + r * AF_LD;
    float gA[16], gB[16];  // gram columns 16 J .. 16 J + 15 of row r
#pragma unroll 1
    for (int J = 0; J <= 2 * W; ++J) {
        tmem_ld16(tm_row + 16 * J, gA);
        if (J == 2 * W) tmem_ld16(tm_row + 16 * J + 16, gB);
        tmem_ld_wait();
        pin_after_wait<16>(gA);
        pin_after_wait<16>(gB);
        if (J < 2 * W || hi) {
            const float s = b_r * ex2(g_r - s_g[16 * J + 15]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 w4 = *reinterpret_cast<const float4*>(s_w + 16 * J + 4 * q);
                const float* gq = gA + 4 * q;
                *reinterpret_cast<float4*>(arow + 16 * J + 4 * q) =
                    make_float4(tf32r(gq[0] * w4.x * s), tf32r(gq[1] * w4.y * s),
                                tf32r(gq[2] * w4.z * s), tf32r(gq[3] * w4.w * s));
            }
        }
    }
    const int jb = 32 * W + (hi ? 16 : 0);  // the diagonal block's first column
    const int rr = lane & 15;                // r - jb
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 g4 = *reinterpret_cast<const float4*>(s_g + jb + 4 * q);
        const float gj[4] = {g4.x, g4.y, g4.z, g4.w};
        float a[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int c = 4 * q + e;
            const float gv = hi ? gB[c] : gA[c];
            a[e] = (c < rr) ? tf32r(gv * b_r * ex2(g_r - gj[e])) : 0.f;
        }
        *reinterpret_cast<float4*>(arow + jb + 4 * q) = make_float4(a[0], a[1], a[2], a[3]);
    }
}

// Row r = 32 W + lane of M o Q K^T (lower triangle with the diagonal; zero past
// the sequence end), as bf16 or fp16 straight into the record's swizzled tile in
// global memory; every byte of the row is written.  tm_row addresses row r of
// Q K^T.
template <bool F16>
__device__ __forceinline__ void build_mqk(uint8_t* rec, uint32_t tm_row, const float* s_g,
                                          const float* s_w, int W, int lane, int valid) {
    const int r = 32 * W + lane;
    const bool hi = lane >= 16;
    const bool live = r < valid;
    const float g_r = s_g[r];
    float gA[16], gB[16];
#pragma unroll 1
    for (int J = 0; J <= 2 * W; ++J) {
        tmem_ld16(tm_row + 16 * J, gA);
        if (J == 2 * W) tmem_ld16(tm_row + 16 * J + 16, gB);
        tmem_ld_wait();
        pin_after_wait<16>(gA);
        pin_after_wait<16>(gB);
        if (J < 2 * W || hi) {
            const float s = live ? ex2(g_r - s_g[16 * J + 15]) : 0.f;
            uint32_t w[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 w4 = *reinterpret_cast<const float4*>(s_w + 16 * J + 4 * q);
                const float* gq = gA + 4 * q;
                w[2 * q] = packr<F16>(gq[0] * w4.x * s, gq[1] * w4.y * s);
                w[2 * q + 1] = packr<F16>(gq[2] * w4.z * s, gq[3] * w4.w * s);
            }
            *reinterpret_cast<uint4*>(rec + taddr(0, r, 16 * J, 0)) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(rec + taddr(0, r, 16 * J + 8, 0)) =
                make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
    const int jb = 32 * W + (hi ? 16 : 0);
    const int rr = lane & 15;
    uint32_t w[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 g4 = *reinterpret_cast<const float4*>(s_g + jb + 4 * q);
        const float gj[4] = {g4.x, g4.y, g4.z, g4.w};
        float m[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int c = 4 * q + e;
            const float gv = hi ? gB[c] : gA[c];
            m[e] = (live && c <= rr) ? gv * ex2(g_r - gj[e]) : 0.f;
        }
        w[2 * q] = packr<F16>(m[0], m[1]);
        w[2 * q + 1] = packr<F16>(m[2], m[3]);
    }
    *reinterpret_cast<uint4*>(rec + taddr(0, r, jb, 0)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(rec + taddr(0, r, jb + 8, 0)) = make_uint4(w[4], w[5], w[6], w[7]);
#pragma unroll 1
    for (int J = 2 * W + 1; J < 4; ++J)
        if (J > 2 * W + (hi ? 1 : 0)) {
            *reinterpret_cast<uint4*>(rec + taddr(0, r, 16 * J, 0)) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(rec + taddr(0, r, 16 * J + 8, 0)) = make_uint4(0, 0, 0, 0);
        }
}

// Diagonal 16 x 16 blocks of T = (I + A)^{-1}: thread tid < 64 (block b = tid / 16,
// column cc = tid % 16) forward-substitutes column cc in fp32, row by row as dot
// products over the already solved entries (the A rows read four at a time), and
// stores it rounded to tf32 (zeros above the diagonal included).  Block b's rows
// of A were written by the same warp.
__device__ __forceinline__ void solve_diag_blocks(const float* Af, float* Tf, int tid) {
    const int b = tid >> 4, cc = tid & 15;
    const float* Ab = Af + (16 * b) * AF_LD + 16 * b;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float acc0 = (i == cc) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
        for (int j4 = 0; j4 < (i + 3) / 4; ++j4) {
            const float4 a = *reinterpret_cast<const float4*>(Ab + i * AF_LD + 4 * j4);
            if (4 * j4 + 0 < i) acc0 = fmaf(-a.x, x[4 * j4 + 0], acc0);
            if (4 * j4 + 1 < i) acc1 = fmaf(-a.y, x[4 * j4 + 1], acc1);
            if (4 * j4 + 2 < i) acc0 = fmaf(-a.z, x[4 * j4 + 2], acc0);
            if (4 * j4 + 3 < i) acc1 = fmaf(-a.w, x[4 * j4 + 3], acc1);
        }
        x[i] = acc0 + acc1;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) Tf[(16 * b + i) * AF_LD + 16 * b + cc] = tf32r(x[i]);
}

// m16n8k8 tf32 product on fragments already in registers
__device__ __forceinline__ void mma_tf32_frag(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// The A fragment of a 16 x 8 fp32 tile (rows of stride lda floats, 16-byte
// aligned) in one ldmatrix.x4: an 8 x 8 b16 matrix read as 8 rows of 4 fp32
// puts element (lane / 4, lane % 4) in the lane's register, and the four
// matrices are rows 0-7 / 8-15 by columns 0-3 / 4-7 -- the fragment's a0..a3.
__device__ __forceinline__ void lda_tf32(const float* A, int lda, int lane, uint32_t* a) {
    const int mat = lane >> 3;
    ldsm_x4(smem_u32(A + ((lane & 7) + 8 * (mat & 1)) * lda + 4 * (mat >> 1)), a);
}
// The B fragments of two n-tiles (n0 .. n0 + 15) at one k step from a tile held
// transposed, Bt[n][k] (rows of stride ldb floats): registers {b0, b1} of n-tile 0,
// then of n-tile 1.
__device__ __forceinline__ void ldb_tf32_t2(const float* Bt, int ldb, int lane, uint32_t* b) {
    const int mat = lane >> 3;
    ldsm_x4(smem_u32(Bt + ((lane & 7) + 8 * (mat >> 1)) * ldb + 4 * (mat & 1)), b);
}
// Store an m16n8 accumulator fragment (tf32-rounded) transposed: Xt[n][m], row
// stride ldx floats, at m-offset m0 and n-offset n0.
__device__ __forceinline__ void store_frag_t(float* Xt, int ldx, int m0, int n0, const float* d,
                                             int lane) {
    const int g = lane >> 2, t4 = lane & 3;
    float* x = Xt + (n0 + 2 * t4) * ldx + m0 + g;
    x[0] = tf32r(d[0]);
    x[ldx] = tf32r(d[1]);
    x[8] = tf32r(d[2]);
    x[ldx + 8] = tf32r(d[3]);
}

// The off-diagonal blocks of T from tf32 tensor-core block products, by the two
// solver warps (w = 0, 1; xw = CO_XS_FLOATS floats of scratch per warp):
//   level 1: T_10 = -T_11 (A_10 T_00) (warp 0),  T_32 = -T_33 (A_32 T_22) (warp 1);
//            each warp reads only the rows it built, so a warp barrier precedes it;
//   level 2: T_ba = -T_bb (A_ba T_aa)  (a = rows/columns 0..31, b = 32..63), warp w
//            taking columns 16 w .. 16 w + 15, after a barrier of both warps.
// The intermediate products go to the scratch transposed (the next product's B
// operand).  Level-1 blocks and the scratch hold tf32-rounded values; level 2 is
// final fp32.
constexpr int XT1_LD = 20;  // level-1 scratch: 16 n-rows x 16 m (+4 pad)
constexpr int XT2_LD = 36;  // level-2 scratch: 16 n-rows x 32 m (+4 pad)
__device__ __forceinline__ void solve_level1(const float* Af, float* Tf, float* xw, int w,
                                             int lane) {
    const int g = lane >> 2, t4 = lane & 3;
    const int bi = 2 * w + 1, bj = 2 * w;
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t a[4];
        lda_tf32(Af + (16 * bi) * AF_LD + 16 * bj + 8 * ks, AF_LD, lane, a);
        const float* B = Tf + (16 * bj + 8 * ks) * AF_LD + 16 * bj;
        mma_tf32_frag(d0, a, __float_as_uint(B[t4 * AF_LD + g]), __float_as_uint(B[(t4 + 4) * AF_LD + g]));
        mma_tf32_frag(d1, a, __float_as_uint(B[t4 * AF_LD + 8 + g]),
                      __float_as_uint(B[(t4 + 4) * AF_LD + 8 + g]));
    }
    store_frag_t(xw, XT1_LD, 0, 0, d0, lane);
    store_frag_t(xw, XT1_LD, 0, 8, d1, lane);
    __syncwarp();
    float e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t a[4], b[4];
        lda_tf32(Tf + (16 * bi) * AF_LD + 16 * bi + 8 * ks, AF_LD, lane, a);
        ldb_tf32_t2(xw + 8 * ks, XT1_LD, lane, b);
        mma_tf32_frag(e0, a, b[0], b[1]);
        mma_tf32_frag(e1, a, b[2], b[3]);
    }
    float* to = Tf + (16 * bi) * AF_LD + 16 * bj + 2 * t4;
    *reinterpret_cast<float2*>(to + g * AF_LD) = make_float2(tf32r(-e0[0]), tf32r(-e0[1]));
    *reinterpret_cast<float2*>(to + (g + 8) * AF_LD) = make_float2(tf32r(-e0[2]), tf32r(-e0[3]));
    *reinterpret_cast<float2*>(to + 8 + g * AF_LD) = make_float2(tf32r(-e1[0]), tf32r(-e1[1]));
    *reinterpret_cast<float2*>(to + 8 + (g + 8) * AF_LD) = make_float2(tf32r(-e1[2]), tf32r(-e1[3]));
}

__device__ __forceinline__ void solve_level2(const float* Af, float* Tf, float* xw, int w,
                                             int lane) {
    const int g = lane >> 2, t4 = lane & 3;
    const int c0 = 16 * w;
    // X = A_ba T_aa for columns c0 .. c0 + 15: T_aa's rows 0-15 are zero right of column 15
    float x[2][2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) x[mt][nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        if (w == 1 && ks < 2) continue;
        const float* B = Tf + (8 * ks) * AF_LD + c0;
        uint32_t b[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            b[nt][0] = __float_as_uint(B[t4 * AF_LD + 8 * nt + g]);
            b[nt][1] = __float_as_uint(B[(t4 + 4) * AF_LD + 8 * nt + g]);
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            uint32_t a[4];
            lda_tf32(Af + (32 + 16 * mt) * AF_LD + 8 * ks, AF_LD, lane, a);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) mma_tf32_frag(x[mt][nt], a, b[nt][0], b[nt][1]);
        }
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) store_frag_t(xw, XT2_LD, 16 * mt, 8 * nt, x[mt][nt], lane);
    __syncwarp();
    // T_ba = -T_bb X: rows 32-47 take T_22 (k = X rows 0-15), rows 48-63 take
    // [T_32 T_33] (k = X rows 0-31)
    {  // rows 32-47
        float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t b[4], a[4];
            ldb_tf32_t2(xw + 8 * ks, XT2_LD, lane, b);
            lda_tf32(Tf + 32 * AF_LD + 32 + 8 * ks, AF_LD, lane, a);
            mma_tf32_frag(y[0], a, b[0], b[1]);
            mma_tf32_frag(y[1], a, b[2], b[3]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float* to = Tf + (32 + g) * AF_LD + c0 + 8 * nt + 2 * t4;
            *reinterpret_cast<float2*>(to) = make_float2(-y[nt][0], -y[nt][1]);
            *reinterpret_cast<float2*>(to + 8 * AF_LD) = make_float2(-y[nt][2], -y[nt][3]);
        }
    }
    {  // rows 48-63
        float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t b[4], a[4];
            ldb_tf32_t2(xw + 8 * ks, XT2_LD, lane, b);
            lda_tf32(Tf + 48 * AF_LD + 32 + 8 * ks, AF_LD, lane, a);
            mma_tf32_frag(y[0], a, b[0], b[1]);
            mma_tf32_frag(y[1], a, b[2], b[3]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float* to = Tf + (48 + g) * AF_LD + c0 + 8 * nt + 2 * t4;
            *reinterpret_cast<float2*>(to) = make_float2(-y[nt][0], -y[nt][1]);
            *reinterpret_cast<float2*>(to + 8 * AF_LD) = make_float2(-y[nt][2], -y[nt][3]);
        }
    }
}

template <bool F16>
__global__ void __launch_bounds__(CO_THREADS, 4)
    chunk_ops_kernel(const __grid_constant__ CUtensorMap map_q,
                     const __grid_constant__ CUtensorMap map_k, const PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + CO_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + CO_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + CO_MISC + 4);
    float* Af = reinterpret_cast<float*>(sm + CO_AF);
    float* Tf = reinterpret_cast<float*>(sm + CO_TF);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int n, c;
    slot_owner(p.cu_seqlens, p.N, blockIdx.x, n, c);
    if (n < 0) return;  // uniform across the CTA
    const int hq = blockIdx.y;
    const int group = p.H_v / p.H_qk;
    const int hv0 = hq * group + blockIdx.z * P1_MAX_GROUP;
    const int nheads = min(P1_MAX_GROUP, group - blockIdx.z * P1_MAX_GROUP);
    const int t_end = p.cu_seqlens[n + 1];
    const int t0 = p.cu_seqlens[n] + c * C;
    const int valid = min(C, t_end - t0);
    const long long slot = record_slot(n, t0);

    // The copies are issued first (only thread 0 touches the barriers before the
    // CTA barrier), then the gates are loaded while the copies and the tensor
    // memory allocation proceed.
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
        mbar_arrive_expect_tx(&bars[0], 4 * HALF);
        tma_load_2d(sm + CO_KQ, &map_k, hq * D, t0, &bars[0]);
        tma_load_2d(sm + CO_KQ + HALF, &map_q, hq * D, t0, &bars[0]);
        tma_load_2d(sm + CO_KQ + 2 * HALF, &map_k, hq * D + 64, t0, &bars[0]);
        tma_load_2d(sm + CO_KQ + 3 * HALF, &map_q, hq * D + 64, t0, &bars[0]);
    }
    // gate scan per value head: warp w < nheads handles head hv0 + w (lane l:
    // tokens 2l, 2l+1, of block l / 8); gates past the sequence end are 0
    float la[2] = {0.f, 0.f}, be[2] = {0.f, 0.f};
    if (warp < nheads) {
        const int h = hv0 + warp;
#pragma unroll
        for (int e = 0; e < 2; ++e)
            if (2 * lane + e < valid) {
                la[e] = p.log_alpha[(size_t)(t0 + 2 * lane + e) * p.H_v + h];
                be[e] = p.beta[(size_t)(t0 + 2 * lane + e) * p.H_v + h];
            }
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, CO_TM_COLS);
        tmem_relinquish();
    }
    if (warp < nheads) {
        const float x0 = la[0] * LOG2E, x1 = la[1] * LOG2E;
        float incl = x0 + x1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const float g0 = incl - x1;
        const float g_e = __shfl_sync(0xffffffffu, incl, lane | 7);  // g at the block's last token
        float* v = reinterpret_cast<float*>(sm + CO_VEC) + warp * CO_VEC_FLOATS;
        *reinterpret_cast<float2*>(v + 2 * lane) = make_float2(g0, incl);
        *reinterpret_cast<float2*>(v + 64 + 2 * lane) = make_float2(be[0], be[1]);
        *reinterpret_cast<float2*>(v + 128 + 2 * lane) = make_float2(ex2(g_e - g0), ex2(g_e - incl));
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = mbar_wait(&bars[0], 0, abort_flag);
    if (!__syncthreads_and(ok)) {  // the copies may still land: wait (bounded), then leave
        if (tid == 0) mbar_wait_drain(&bars[0], 0);
        __syncthreads();
        if (warp == 0) tmem_dealloc(tmem, CO_TM_COLS);
        return;
    }
    // [K; Q] K^T: A = the 128 rows K h | Q h of each 64-column half (K-major),
    // B = K (K-major, N = 64 tokens); k step ks reads 16 columns of half ks / 4
    if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t ID_G = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint32_t a = sb + CO_KQ + (ks >> 2) * 2 * HALF + (ks & 3) * 32;
            mma_bf16_ss(tmem, sdesc_sw128(a, 16, 1024), sdesc_sw128(a, 16, 1024), ID_G, ks > 0);
        }
        mma_commit(&bars[1]);
    }
    ok = mbar_wait(&bars[1], 0, abort_flag);
    if (!__syncthreads_and(ok)) {
        if (tid == 0) mbar_wait_drain(&bars[1], 0);
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            tmem_dealloc(tmem, CO_TM_COLS);
        }
        return;
    }
    tc_fence_after();
    // The product is complete, so K and Q are no longer read: their bytes become A
    // and T.  The grams stay in tensor memory; each value head reads its row again.
    for (int vh = 0; vh < nheads; ++vh) {
        const int h = hv0 + vh;
        const float* s_g = reinterpret_cast<const float*>(sm + CO_VEC) + vh * CO_VEC_FLOATS;
        const float* s_b = s_g + 64;
        const float* s_w = s_g + 128;
        uint8_t* rec = p.records + (size_t)(slot * p.H_v + h) * REC_BYTES;
        const uint32_t tm_row = tmem + ((uint32_t)(32 * warp) << 16);  // row tid of [K K^T; Q K^T]
        if (warp < 2) {
            build_a(Af, tm_row, s_g, s_b, s_w, warp, lane);
            __syncwarp();
            if (vh > 0) bar_sync<CO_BAR_TFREE, CO_THREADS>();  // the previous T has been read
            solve_diag_blocks(Af, Tf, tid);
            __syncwarp();
            solve_level1(Af, Tf, reinterpret_cast<float*>(sm + CO_XS) + warp * CO_XS_FLOATS, warp, lane);
            bar_sync<CO_BAR_SOLVE, 64>();
            solve_level2(Af, Tf, reinterpret_cast<float*>(sm + CO_XS) + warp * CO_XS_FLOATS, warp, lane);
            bar_sync<CO_BAR_SOLVE, 64>();  // both solvers are done with this head's A
            bar_arrive<CO_BAR_TDONE, CO_THREADS>();
        } else {
            const int q = tid - 64;
            build_mqk<F16>(rec + REC_MQ, tm_row, s_g, s_w, warp - 2, lane, valid);
            // gamma_r, d_r (zero past the sequence end), gamma_C, zero padding
            float* rv = reinterpret_cast<float*>(rec + REC_VEC);
            const float gC = s_g[C - 1];
            rv[q] = ex2(s_g[q]);
            rv[64 + q] = (q < valid) ? ex2(gC - s_g[q]) : 0.f;
            if (q < REC_VEC_FLOATS - 128) rv[128 + q] = (q == 0) ? ex2(gC) : 0.f;
            bar_sync<CO_BAR_TDONE, CO_THREADS>();
            // T diag(beta) as a bf16 or fp16 tile; its 16 x 16 blocks above the diagonal are
            // written as zeros so that every byte of the record is defined
#pragma unroll 2
            for (int it = 0; it < 8; ++it) {
                const int idx = q + 64 * it;
                const int rr = idx >> 3, ch = idx & 7;
                uint4 w = make_uint4(0, 0, 0, 0);
                if ((ch >> 1) <= (rr >> 4)) {
                    const float4 ta = *reinterpret_cast<const float4*>(Tf + rr * AF_LD + 8 * ch);
                    const float4 tb = *reinterpret_cast<const float4*>(Tf + rr * AF_LD + 8 * ch + 4);
                    const float4 b0 = *reinterpret_cast<const float4*>(s_b + 8 * ch);
                    const float4 b1 = *reinterpret_cast<const float4*>(s_b + 8 * ch + 4);
                    w = make_uint4(packr<F16>(ta.x * b0.x, ta.y * b0.y),
                                   packr<F16>(ta.z * b0.z, ta.w * b0.w),
                                   packr<F16>(tb.x * b1.x, tb.y * b1.y),
                                   packr<F16>(tb.z * b1.z, tb.w * b1.w));
                }
                *reinterpret_cast<uint4*>(rec + REC_TB + taddr(0, rr, 8 * ch, 0)) = w;
            }
            if (vh + 1 < nheads) bar_arrive<CO_BAR_TFREE, CO_THREADS>();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, CO_TM_COLS);
    }
}



// D += A * B, m16n8k16, fp32 accumulate: fp16 inputs when F16, else bf16 (the
// products with a record tile as A when the records are fp16).
template <bool F16>
__device__ __forceinline__ void mma16816r(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    if constexpr (F16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        mma16816(d, a, b0, b1);
    }
}

// store_acc_bf16 in the records' tile type (fp16 when F16)
template <int NT, bool F16>
__device__ __forceinline__ void store_acc_r(uint8_t* smem, uint32_t base_off, int m0,
                                            const float (*acc)[4], int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int col = 8 * nt + 2 * t;
        *reinterpret_cast<uint32_t*>(smem + taddr_e(base_off, m0 + g, col, 0)) =
            packr<F16>(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<uint32_t*>(smem + taddr_e(base_off, m0 + g + 8, col, 0)) =
            packr<F16>(acc[nt][2], acc[nt][3]);
    }
}

// Delta = T_b X for row block rb (rows 16 rb .. +15) and n-tiles of column half H
// of an NT-tile slice, stored as Delta (in the records' tile type: X is in it
// too) at shared offset DU and d o Delta (bf16: it meets the bf16 K tile) at DD.
// T_b is lower triangular, so row block rb takes k-steps 0 .. rb only.
template <int NT, int H, bool F16, uint32_t DU, uint32_t DD>
__device__ __forceinline__ void delta_half(uint8_t* sm, uint32_t tb, uint32_t xt, int rb,
                                           int lane, float d_lo, float d_hi) {
    constexpr int N0 = H * (NT / 2), N1 = (H + 1) * (NT / 2);
    float acc[N1 - N0][4];
#pragma unroll
    for (int i = 0; i < N1 - N0; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        if (ks <= rb) {
            uint32_t a[4];
            lda_k(tb, 0, 16 * rb, 16 * ks, lane, a);
#pragma unroll
            for (int nt = N0; nt < N1; nt += 2) {
                if (nt + 1 < N1) {
                    uint32_t b[4];
                    ldb_mn(xt, 0, 8 * nt, 16 * ks, lane, b);
                    mma16816r<F16>(acc[nt - N0], a, b[0], b[1]);
                    mma16816r<F16>(acc[nt - N0 + 1], a, b[2], b[3]);
                } else {
                    uint32_t b[2];
                    ldb_mn1(xt, 8 * nt, 16 * ks, lane, b);
                    mma16816r<F16>(acc[nt - N0], a, b[0], b[1]);
                }
            }
        }
    }
    const int g = lane >> 2, t = lane & 3, r = 16 * rb + g;
#pragma unroll
    for (int i = 0; i < N1 - N0; ++i) {
        const int col = 8 * (N0 + i) + 2 * t;
        *reinterpret_cast<uint32_t*>(sm + taddr_e(DU, r, col, 0)) =
            packr<F16>(acc[i][0], acc[i][1]);
        *reinterpret_cast<uint32_t*>(sm + taddr_e(DU, r + 8, col, 0)) =
            packr<F16>(acc[i][2], acc[i][3]);
        *reinterpret_cast<uint32_t*>(sm + taddr_e(DD, r, col, 0)) =
            pack2(acc[i][0] * d_lo, acc[i][1] * d_lo);
        *reinterpret_cast<uint32_t*>(sm + taddr_e(DD, r + 8, col, 0)) =
            pack2(acc[i][2] * d_hi, acc[i][3] * d_hi);
    }
}

// ============================================================================
// Pass 2: state pass.  Grid (d_v slices, H_v, N).
// ============================================================================
// MODE P2_OUT: the prefill proper (outputs, final states).  MODE P2_SEGMENT:
// phase A of the segmented prefill -- no outputs; blocks x < slices carry the
// state from zero (final state to S_final), blocks x >= slices carry the
// identity with V taken as zero, so that their final state is the segment's
// propagator P (to S_aux): S_end = P S_start + (state from zero).  MODE
// P2_SAVE: no outputs; every chunk's entering state is stored to S_aux (for
// the gradients).
// MODE P2_OUT_SAVE: the outputs and final states of P2_OUT, and the entering
// states of P2_SAVE (a training forward whose gradients follow).
constexpr int P2_OUT = 0, P2_SEGMENT = 1, P2_SAVE = 2, P2_OUT_SAVE = 3;

template <int NS, typename IO, int MODE, bool F16>
__global__ void __launch_bounds__(P2_THREADS, 1)
    state_pass_kernel(const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v, const PrefillParams p) {
    static_assert(NS == 32 || NS == 48 || NS == 64, "slice width");
    constexpr int NT = NS / 8;  // n-tiles of a slice
    constexpr int NP = NT / 2;  // n-tile pairs
    constexpr int NSL = (D + NS - 1) / NS;  // slices of a head
    constexpr bool OUTS = MODE == P2_OUT || MODE == P2_OUT_SAVE;  // writes the outputs
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P2_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + P2_MISC);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int h = blockIdx.y;
    const int n = blockIdx.z;
    const int hq = h / (p.H_v / p.H_qk);
    const bool prop = MODE == P2_SEGMENT && blockIdx.x >= NSL;  // propagator block
    const int col0 = (blockIdx.x - (prop ? NSL : 0)) * NS;
    const int ncols = min(NS, D - col0);
    const int t_beg = p.cu_seqlens[n];
    const int t_end = p.cu_seqlens[n + 1];
    const int nchunks = (t_end - t_beg + C - 1) / C;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR2; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // Copies of chunk c into ring stage c % NSTAGE: K, Q (both halves), the V slice
    // and the chunk's operator record.  Issued by one thread; a stage is refilled
    // only after every chain warp has finished with it.
    auto issue_chunk = [&](int c) {
        const int s = c % NSTAGE;
        uint8_t* st = sm + s * STAGE_BYTES;
        const int y = t_beg + c * C;
        uint64_t* full = &bars[B2_FULL + s];
        mbar_arrive_expect_tx(full, prop ? STAGE_TX - HALF : STAGE_TX);
        tma_load_2d(st + ST_K, &map_k, hq * D, y, full);
        tma_load_2d(st + ST_K + HALF, &map_k, hq * D + 64, y, full);
        tma_load_2d(st + ST_Q, &map_q, hq * D, y, full);
        tma_load_2d(st + ST_Q + HALF, &map_q, hq * D + 64, y, full);
        if (!prop) tma_load_2d(st + ST_V, &map_v, h * D + col0, y, full);
        bulk_load(st + ST_REC, p.records + (size_t)(record_slot(n, y) * p.H_v + h) * REC_BYTES,
                  REC_BYTES, full);
    };
    int issued = 0;
    if (threadIdx.x == P2_LOADER)
        for (; issued < min(NSTAGE, nchunks); ++issued) issue_chunk(issued);
    {
        // ------------------------------------------------------------ chain warps
        const int tid = threadIdx.x;
        const bool mw = warp < 4;        // warps 0-3 also compute K S, Q S and the output
        const int m0 = 16 * (warp & 3);  // this warp's 16 rows of the 64-row products
        const int r0 = 16 * warp;        // this warp's 16 rows of S

        // S rows r0 + {g, g+8}, columns 8 nt + 2 t4 + {0, 1}
        float Sacc[NT][4];
        {
            const float* s0 = p.S0 ? p.S0 + ((size_t)n * p.H_v + h) * D * D : nullptr;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int row = r0 + g + ((e >> 1) << 3);
                    const int col = 8 * nt + 2 * t4 + (e & 1);
                    if (prop)  // the identity's columns col0 .. col0 + NS - 1
                        Sacc[nt][e] = (col < ncols && row == col0 + col) ? 1.f : 0.f;
                    else
                        Sacc[nt][e] = (s0 && col < ncols) ? s0[(size_t)row * D + col0 + col] : 0.f;
                }
            store_acc_bf16<NT>(sm, P2_SB, 0, r0, Sacc, lane, 1.f, 1.f);
        }
        bar_sync<BAR_CHAIN, P2_CHAIN_THREADS>();

        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NSTAGE;
            const uint32_t st = sb + s * STAGE_BYTES;
            const uint8_t* stp = sm + s * STAGE_BYTES;
            const float* rv = reinterpret_cast<const float*>(stp + ST_REC + REC_VEC);
            const int tc0 = t_beg + c * C;
            const int valid = min(C, t_end - tc0);
            const bool ok = mbar_wait(&bars[B2_FULL + s], (c / NSTAGE) & 1, abort_flag);
            __syncwarp();
            if constexpr (MODE == P2_SAVE || MODE == P2_OUT_SAVE) {  // the entering state, bf16 image
                uint8_t* sv = reinterpret_cast<uint8_t*>(p.S_aux) +
                              ((size_t)record_slot(n, tc0) * p.H_v + h) * STATE_IMAGE_BYTES;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int hl = 0; hl < 2; ++hl) {
                        const int row = r0 + g + 8 * hl;
                        const int col = 8 * nt + 2 * t4;
                        if (col < ncols)
                            *reinterpret_cast<uint32_t*>(sv + taddr_e(0, row, col0 + col, 2 * HALF)) =
                                pack2(Sacc[nt][2 * hl], Sacc[nt][2 * hl + 1]);
                    }
            }

            // ---- warps 0-3: K S and Q S for rows m0 .. m0+15 (one pass over S)
            float accK[NT][4], accQ[NT][4];
            if (mw) {
#pragma unroll
                for (int i = 0; i < NT; ++i)
#pragma unroll
                    for (int e = 0; e < 4; ++e) accK[i][e] = accQ[i][e] = 0.f;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    uint32_t ak[4], aq[4];
                    lda_k(st + ST_K, HALF, m0, 16 * ks, lane, ak);
                    if constexpr (OUTS) lda_k(st + ST_Q, HALF, m0, 16 * ks, lane, aq);
#pragma unroll
                    for (int np = 0; np < NP; ++np) {
                        uint32_t b[4];
                        ldb_mn(sb + P2_SB, 0, 16 * np, 16 * ks, lane, b);
                        mma16816(accK[2 * np], ak, b[0], b[1]);
                        mma16816(accK[2 * np + 1], ak, b[2], b[3]);
                        if constexpr (OUTS) {
                            mma16816(accQ[2 * np], aq, b[0], b[1]);
                            mma16816(accQ[2 * np + 1], aq, b[2], b[3]);
                        }
                    }
                }
                // X = V - gamma o (K S)   (rows past the sequence end are zero: V and K are);
                // gamma o (Q S) is kept for the output
                const float gm_lo = rv[m0 + g], gm_hi = rv[m0 + g + 8];
                const uint8_t* vt = stp + ST_V;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int col = 8 * nt + 2 * t4;
                    float2 v_lo = make_float2(0.f, 0.f), v_hi = v_lo;
                    if (!prop) {
                        v_lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
                            vt + taddr_e(0, m0 + g, col, 0)));
                        v_hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(
                            vt + taddr_e(0, m0 + g + 8, col, 0)));
                    }
                    accK[nt][0] = v_lo.x - gm_lo * accK[nt][0];
                    accK[nt][1] = v_lo.y - gm_lo * accK[nt][1];
                    accK[nt][2] = v_hi.x - gm_hi * accK[nt][2];
                    accK[nt][3] = v_hi.y - gm_hi * accK[nt][3];
                    accQ[nt][0] *= gm_lo;
                    accQ[nt][1] *= gm_lo;
                    accQ[nt][2] *= gm_hi;
                    accQ[nt][3] *= gm_hi;
                }
                store_acc_r<NT, F16>(sm, P2_X, m0, accK, lane);
            }
            if (!bar_and<BAR_CHAIN, P2_CHAIN_THREADS>(ok)) break;

            // ---- Delta = T_b X: all eight warps, warp = (row block m0 / 16, column half);
            // T_b is lower triangular, so row block rb needs key blocks 0..rb only
            {
                const int rb = warp & 3;
                const float d_lo = rv[64 + m0 + g], d_hi = rv[64 + m0 + g + 8];
                if (warp < 4)
                    delta_half<NT, 0, F16, P2_DU, P2_DD>(sm, st + ST_REC + REC_TB, sb + P2_X, rb, lane,
                                                         d_lo, d_hi);
                else
                    delta_half<NT, 1, F16, P2_DU, P2_DD>(sm, st + ST_REC + REC_TB, sb + P2_X, rb, lane,
                                                         d_lo, d_hi);
            }
            if (!bar_and<BAR_CHAIN, P2_CHAIN_THREADS>(ok)) break;

            // ---- S <- gamma_C S + K^T (d o Delta)   (rows r0 .. r0+15)
            {
                const float gamC = rv[128];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) Sacc[nt][e] *= gamC;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    uint32_t a[4];
                    lda_mn(st + ST_K, HALF, r0, 16 * ks, lane, a);
#pragma unroll
                    for (int np = 0; np < NP; ++np) {
                        uint32_t b[4];
                        ldb_mn(sb + P2_DD, 0, 16 * np, 16 * ks, lane, b);
                        mma16816(Sacc[2 * np], a, b[0], b[1]);
                        mma16816(Sacc[2 * np + 1], a, b[2], b[3]);
                    }
                }
            }
            // ---- O = gamma o (Q S) + (M o Q K^T) Delta   (warps 0-3), stored
            if (OUTS && mw) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    if (ks <= warp) {
                        uint32_t a[4];
                        lda_k(st + ST_REC + REC_MQ, 0, m0, 16 * ks, lane, a);
#pragma unroll
                        for (int np = 0; np < NP; ++np) {
                            uint32_t b[4];
                            ldb_mn(sb + P2_DU, 0, 16 * np, 16 * ks, lane, b);
                            mma16816r<F16>(accQ[2 * np], a, b[0], b[1]);
                            mma16816r<F16>(accQ[2 * np + 1], a, b[2], b[3]);
                        }
                    }
                }
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
                                store2<IO>(orow + col, accQ[nt][2 * hl], accQ[nt][2 * hl + 1]);
                        }
                    }
                }
            }
            store_acc_bf16<NT>(sm, P2_SB, 0, r0, Sacc, lane, 1.f, 1.f);
            if (!bar_and<BAR_CHAIN, P2_CHAIN_THREADS>(ok)) break;
            // this ring stage is free again: refill it with the chunk NSTAGE ahead
            if (tid == P2_LOADER && c + NSTAGE < nchunks) issue_chunk(issued++);
        }
        float* const s_out = prop ? p.S_aux : p.S_final;
        if (s_out && !*abort_flag) {
            float* sf = s_out + ((size_t)n * p.H_v + h) * D * D;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int hl = 0; hl < 2; ++hl) {
                    const int row = r0 + g + 8 * hl;
                    const int col = 8 * nt + 2 * t4;
                    if (col < ncols)
                        *reinterpret_cast<float2*>(sf + (size_t)row * D + col0 + col) =
                            make_float2(Sacc[nt][2 * hl], Sacc[nt][2 * hl + 1]);
                }
        }
    }
    // Drain: no copy may still be landing in shared memory when the CTA exits.
    if (threadIdx.x == P2_LOADER)
        for (int c = max(0, issued - NSTAGE); c < issued; ++c)
            mbar_wait_drain(&bars[B2_FULL + (c % NSTAGE)], (c / NSTAGE) & 1);
    __syncthreads();
}

// ============================================================================
// Pass 2 on the fifth-generation tensor cores: the prefill's outputs and final
// states (and, in the save modes, every chunk's entering state).  Grid (d_v
// slices, H_v, N); 288 threads: eight compute warps and one issuing warp whose
// lane 0 issues every tcgen05.mma; accumulators live in tensor memory.  Per
// chunk:
//   [K; Q] S             M = 128: lanes 0-63 K S, lanes 64-127 Q S
//   Delta = T_b X        warp-level mma.sync (64 x NS, K = 64, T_b lower triangular)
//   K^T (d o Delta)      M = 128: the state increment, lane = d_k index
//   [T_b; M_Q] Delta     M = 128: lanes 64-127 (M o Q K^T) Delta, beside Q S
// (M_Q = M o Q K^T; the record stores T_b and M_Q as adjacent 64-row K-major
// tiles, so [T_b; M_Q] is one 128-row operand.)  Between the products every
// warp reads its TMEM lanes and half of the slice's columns (warps w and w + 4
// share lane quadrant w): X goes to shared memory as the B operand of T_b X,
// Delta as that of the next products (MN-major); each thread keeps half a row
// of the fp32 state and writes its bf16 copy, the next [K; Q] S's B operand.
// The output rows O = gamma o (Q S) + (M o Q K^T) Delta of a chunk are formed by
// the warps on lanes 64-127 while the next chunk's [K; Q] S runs ([K; Q] S
// and [T_b; M_Q] Delta are double-buffered in TMEM).  Every product commits
// to an mbarrier of its own, once per chunk.  Warp 6's thread 0 streams K, Q,
// the V slice and the record into a 3-stage ring; it refills the previous
// chunk's stage while X is formed.  The issuing warp does nothing else
// (tcgen05.mma issue stalls while the pipe is busy, which held a compute warp
// back): it waits on named barriers that the compute warps bar.arrive on once
// d o Delta and the bf16 S are written.  The compute warps leave the chunk loop
// only at its end, after their last arrive, and the issuer reads the abort flag
// after each chunk's first wait, so that every barrier completes.
// ============================================================================
constexpr int TC_THREADS = 288;  // eight compute warps and the issuing warp
constexpr int TC_COMPUTE = 256;  // warps 0-7; warp 8's lane 0 issues every product
constexpr int TC_LOADER = 192;   // warp 6: idle while warps 0, 1, 4, 5 form X
// named barriers: the compute warps; Delta and d o Delta written, S written
// (compute warps arrive, the issuing warp waits)
constexpr int BAR_TC = 1, BAR_TC_DD = 2, BAR_TC_SB = 3;
// ring stage: K h0 | Q h0 | K h1 | Q h1 -- [K; Q] is one 128-row K-major tile
// per 64-column half, and K alone an MN-major one with its halves 16 KB apart --
// then the V slice and the record (T_b, then M o Q K^T)
constexpr uint32_t TS_KQ = 0, TS_V = 4 * HALF, TS_REC = 5 * HALF;
constexpr uint32_t TS_STAGE = ((TS_REC + REC_BYTES + 1023) / 1024) * 1024;
constexpr uint32_t TS_TX = 5 * HALF + REC_BYTES;
constexpr uint32_t TC_SB = NSTAGE * TS_STAGE;  // S in bf16: 128 k-rows x 64 columns, MN-major
constexpr uint32_t TC_X = TC_SB + 2 * HALF;    // X, 64 token rows x 64 columns, MN-major
constexpr uint32_t TC_DU = TC_X + HALF;        // Delta
constexpr uint32_t TC_DD = TC_DU + HALF;       // d o Delta
constexpr uint32_t TC_BAR = TC_DD + HALF;      // full[NSTAGE], ks, u, o, drain
constexpr uint32_t TC_MISC = TC_BAR + 128;     // abort flag, TMEM base
constexpr uint32_t TC_SMEM = TC_MISC + 16 + 1024;
static_assert(TS_STAGE % 1024 == 0 && TC_SB % 1024 == 0, "swizzled tiles sit on 1 KB");
static_assert(TC_SMEM <= 232448, "tcgen05 state pass shared memory budget");
// TMEM columns (512 allocated): [K; Q] S (two buffers), the state increment,
// [T_b; M_Q] Delta (two buffers)
constexpr uint32_t TM_KQ = 0, TM_U = 192, TM_O = 256, TM_COLS = 512;

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* r) {
    uint32_t* u = reinterpret_cast<uint32_t*>(r);
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]),
                   "=r"(u[6]), "=r"(u[7])
                 : "r"(taddr));
}

// N columns (a multiple of 8) of this thread's TMEM lane, fp32.  The values are
// pinned behind the wait so that no use moves above it.
template <int N>
__device__ __forceinline__ void tmem_cols(uint32_t ta, float* v) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i) tmem_ld8(ta + 8 * i, v + 8 * i);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}

// Columns c0 .. c0 + N - 1 (c0, N multiples of 8) of row r of an MN-major
// 128B-swizzled bf16 (or fp16) tile (one 64-column block), scaled by s.
template <int N, bool F16 = false>
__device__ __forceinline__ void put_cols(uint8_t* sm, uint32_t tile, int r, int c0, const float* v,
                                         float s) {
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
        const int j = c0 / 8 + i;
        *reinterpret_cast<uint4*>(sm + tile + r * 128 + ((j ^ (r & 7)) << 4)) =
            make_uint4(packr<F16>(s * v[8 * i], s * v[8 * i + 1]),
                       packr<F16>(s * v[8 * i + 2], s * v[8 * i + 3]),
                       packr<F16>(s * v[8 * i + 4], s * v[8 * i + 5]),
                       packr<F16>(s * v[8 * i + 6], s * v[8 * i + 7]));
    }
}

template <typename IO>
__device__ __forceinline__ void store8(IO* p, const float* v);
template <>
__device__ __forceinline__ void store8<float>(float* p, const float* v) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float* v) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]),
                                              pack2(v[4], v[5]), pack2(v[6], v[7]));
}

// MODE P2_OUT: outputs and final states.  P2_SAVE: no outputs; every chunk's
// entering state goes to S_aux as a bf16 image (for the gradients).
// P2_OUT_SAVE: both.
template <int NS, typename IO, bool F16, int MODE>
__global__ void __launch_bounds__(TC_THREADS, 1)
    state_tc_kernel(const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const PrefillParams p) {
    static_assert(NS == 32 || NS == 48 || NS == 64, "slice width");
    static_assert(MODE == P2_OUT || MODE == P2_SAVE || MODE == P2_OUT_SAVE, "modes");
    constexpr bool OUTS = MODE != P2_SAVE;  // writes the outputs
    constexpr bool SAVE = MODE != P2_OUT;   // saves every chunk's entering state
    constexpr int HN = NS / 2;                              // columns per half
    constexpr uint32_t ID_128 = idesc_bf16(128, NS, 0, 1);  // K-major A, MN-major B
    constexpr uint32_t ID_KT = idesc_bf16(128, NS, 1, 1);   // MN-major A (K^T), MN-major B
    // the products with a record tile as A (T_b X, [T_b; M o Q K^T] Delta): fp16
    // when the records are fp16, and then X and Delta are written as fp16 too
    constexpr uint32_t ID_R128 = F16 ? idesc_f16(128, NS, 0, 1) : idesc_bf16(128, NS, 0, 1);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_u32(sm);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + TC_BAR);
    uint64_t* bar_ks = bars + NSTAGE;
    uint64_t* bar_u = bars + NSTAGE + 1;
    uint64_t* bar_o = bars + NSTAGE + 2;
    uint64_t* drain_bar = bars + NSTAGE + 3;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + TC_MISC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + TC_MISC + 4);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3;          // TMEM lanes 32 quad .. 32 quad + 31
    const bool issuer = tid >= TC_COMPUTE;       // warp 8
    const int c_lo = ((warp >> 2) & 1) * HN;  // this warp's half of the slice's columns
    const int row = 32 * quad + lane;   // my row of an M = 128 product (a state row)
    const int h = blockIdx.y, n = blockIdx.z;
    const int hq = h / (p.H_v / p.H_qk);
    const int col0 = blockIdx.x * NS;
    const int ncols = min(NS, D - col0);
    const int t_beg = p.cu_seqlens[n];
    const int t_end = p.cu_seqlens[n + 1];
    const int nchunks = (t_end - t_beg + C - 1) / C;

    if (tid == 0) {
        for (int i = 0; i < NSTAGE + 4; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(32 * quad) << 16) + c_lo;  // my lanes, my columns

    auto issue_chunk = [&](int c) {
        const int s = c % NSTAGE;
        uint8_t* st = sm + s * TS_STAGE;
        const int y = t_beg + c * C;
        uint64_t* full = &bars[s];
        mbar_arrive_expect_tx(full, TS_TX);
        tma_load_2d(st + TS_KQ, &map_k, hq * D, y, full);
        tma_load_2d(st + TS_KQ + HALF, &map_q, hq * D, y, full);
        tma_load_2d(st + TS_KQ + 2 * HALF, &map_k, hq * D + 64, y, full);
        tma_load_2d(st + TS_KQ + 3 * HALF, &map_q, hq * D + 64, y, full);
        tma_load_2d(st + TS_V, &map_v, h * D + col0, y, full);
        bulk_load(st + TS_REC, p.records + (size_t)(record_slot(n, y) * p.H_v + h) * REC_BYTES,
                  REC_BYTES, full);
    };
    int issued = 0;
    if (tid == TC_LOADER)
        for (; issued < min(NSTAGE, nchunks); ++issued) issue_chunk(issued);

    // row `row` of the state, columns col0 + c_lo .. + HN - 1, fp32
    float Sr[HN];
    // the state entering chunk cc into its bf16 image (16 bytes per 8 columns)
    auto save_image = [&](int cc) {
        if (!SAVE || cc >= nchunks) return;
        uint8_t* sv = reinterpret_cast<uint8_t*>(p.S_aux) +
                      ((size_t)record_slot(n, t_beg + cc * C) * p.H_v + h) * STATE_IMAGE_BYTES;
#pragma unroll
        for (int i = 0; i < HN / 8; ++i)
            if (c_lo + 8 * i < ncols)
                *reinterpret_cast<uint4*>(sv + taddr(0, row, col0 + c_lo + 8 * i, 2 * HALF)) =
                    make_uint4(pack2(Sr[8 * i], Sr[8 * i + 1]), pack2(Sr[8 * i + 2], Sr[8 * i + 3]),
                               pack2(Sr[8 * i + 4], Sr[8 * i + 5]),
                               pack2(Sr[8 * i + 6], Sr[8 * i + 7]));
    };
    if (!issuer) {
        const float* s0 =
            p.S0 ? p.S0 + (((size_t)n * p.H_v + h) * D + row) * D + col0 + c_lo : nullptr;
#pragma unroll
        for (int j = 0; j < HN; ++j) Sr[j] = (s0 && c_lo + j < ncols) ? s0[j] : 0.f;
        put_cols<HN>(sm, TC_SB, row, c_lo, Sr, 1.f);
        fence_proxy_async_smem();
        save_image(0);
    }
    __syncthreads();  // the first K S reads the whole tile

    // O rows of chunk c (warps on lanes 64-127: token row row - 64), once
    // (M o Q K^T) Delta is done
    auto output = [&](int c, float g_o) -> bool {
        const bool ok = mbar_wait(bar_o, c & 1, abort_flag);
        tc_fence_after();
        float qs[HN], oi[HN];  // both reads behind one wait
#pragma unroll
        for (int i = 0; i < HN / 8; ++i) {
            tmem_ld8(tl + TM_KQ + 64 * (c & 1) + 8 * i, qs + 8 * i);
            tmem_ld8(tl + TM_O + 64 * (c & 1) + 8 * i, oi + 8 * i);
        }
        tmem_ld_wait();
        pin_after_wait<HN>(qs);
        pin_after_wait<HN>(oi);
        const int tc0 = t_beg + c * C, i = row - 64;
        if (ok && i < t_end - tc0) {
            IO* orow = static_cast<IO*>(p.o) + ((size_t)(tc0 + i) * p.H_v + h) * D + col0 + c_lo;
#pragma unroll
            for (int j = 0; j < HN / 8; ++j) {
                if (c_lo + 8 * j < ncols) {
                    float ov[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) ov[e] = fmaf(g_o, qs[8 * j + e], oi[8 * j + e]);
                    store8<IO>(orow + 8 * j, ov);
                }
            }
        }
        return ok;
    };

    if (issuer) {
        // ---- the issuing warp: lane 0 issues, the warp takes the barriers
        const bool lead = lane == 0;
        bool stopped = false;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NSTAGE;
            const uint32_t st = sb + s * TS_STAGE;
            const uint32_t par = c & 1;
            if (c > 0) {
                bar_sync<BAR_TC_SB, TC_THREADS>();  // the previous chunk's S is written
                if (*abort_flag) {  // the compute warps left the loop after that arrive
                    stopped = true;
                    break;
                }
            }
            const bool landed = mbar_wait(&bars[s], (c / NSTAGE) & 1, abort_flag);
            if (lead && landed) {  // [K; Q] S
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16_ss(tmem + TM_KQ + 64 * par,
                                sdesc_sw128(st + TS_KQ + (ks >> 2) * 2 * HALF + (ks & 3) * 32, 16, 1024),
                                sdesc_sw128(sb + TC_SB + ks * 2048, 8192, 1024), ID_128, ks > 0);
                mma_commit(bar_ks);
            }
            bar_sync<BAR_TC_DD, TC_THREADS>();  // Delta and d o Delta are written
            if (lead) {  // K^T (d o Delta), then [T_b; M_Q] Delta
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16_ss(tmem + TM_U, sdesc_sw128(st + TS_KQ + ks * 2048, 2 * HALF, 1024),
                                sdesc_sw128(sb + TC_DD + ks * 2048, 8192, 1024), ID_KT, ks > 0);
                mma_commit(bar_u);
                if constexpr (OUTS) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ss(tmem + TM_O + 64 * par,
                                    sdesc_sw128(st + TS_REC + ks * 32, 16, 1024),
                                    sdesc_sw128(sb + TC_DU + ks * 2048, 8192, 1024), ID_R128, ks > 0);
                    mma_commit(bar_o);
                }
            }
        }
        // the compute warps' arrive after the last chunk
        if (nchunks > 0 && !stopped) bar_sync<BAR_TC_SB, TC_THREADS>();
        if (lead) {  // no product may still run when TMEM is freed (bounded wait)
            mma_commit(drain_bar);
            mbar_wait_drain(drain_bar, 0);
        }
    } else {
    // ---- the compute warps
    float g_prev = 0.f;  // gamma of my output row in the previous chunk
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % NSTAGE;
        const uint32_t st = sb + s * TS_STAGE;
        const uint8_t* stp = sm + s * TS_STAGE;
        const uint32_t par = c & 1;
        ok = mbar_wait(&bars[s], (c / NSTAGE) & 1, abort_flag);
        // (the issuing warp starts [K; Q] S); without outputs, the state entering
        // this chunk goes to its image while the warps wait for [K; Q] S (chunk
        // 0's went before the loop); this chunk's scalars come into registers;
        // the previous chunk's outputs
        if (!OUTS && c >= 1) save_image(c);
        const float* rv = reinterpret_cast<const float*>(stp + TS_REC + REC_VEC);
        const float g_row = rv[row & 63];         // gamma of my K row (quads 0-1) or Q row (2-3)
        const float g_C = rv[128];
        if (OUTS && c >= 1 && quad >= 2) ok = output(c - 1, g_prev) && ok;
        g_prev = g_row;
        ok = mbar_wait(bar_ks, par, abort_flag) && ok;
        tc_fence_after();
        // the previous chunk's stage gets the chunk NSTAGE after it (issued while the
        // tensor pipe waits for X, so that the copies land outside [K; Q] S)
        if (tid == TC_LOADER && c >= 1 && c - 1 + NSTAGE < nchunks) issue_chunk(issued++);
        if (quad < 2) {  // X = V - gamma o (K S), token row `row`
            float x[HN];
            tmem_cols<HN>(tl + TM_KQ + 64 * par, x);
            {
#pragma unroll
                for (int i = 0; i < HN / 8; ++i) {
                    const int j = c_lo / 8 + i;
                    const uint4 u = *reinterpret_cast<const uint4*>(stp + TS_V + row * 128 +
                                                                    ((j ^ (row & 7)) << 4));
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 v2 =
                            __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
                        x[8 * i + 2 * e] = v2.x - g_row * x[8 * i + 2 * e];
                        x[8 * i + 2 * e + 1] = v2.y - g_row * x[8 * i + 2 * e + 1];
                    }
                }
                put_cols<HN, F16>(sm, TC_X, row, c_lo, x, 1.f);  // read by ldmatrix only
            }
        }
        tc_fence_before();
        bar_sync<BAR_TC, TC_COMPUTE>();  // X is complete

        // Delta = T_b X on mma.sync: warp (quad, column half) takes rows 16 quad ..
        // + 15 of its half, so no commit, wake-up or TMEM read sits on the chain;
        // Delta and d o Delta go to shared memory as the next products' B operands
        {
            const int rlo = 16 * quad + (lane >> 2);
            const float dlo = rv[64 + rlo], dhi = rv[64 + rlo + 8];
            if (warp < 4)
                delta_half<NS / 8, 0, F16, TC_DU, TC_DD>(sm, st + TS_REC + REC_TB, sb + TC_X, quad,
                                                         lane, dlo, dhi);
            else
                delta_half<NS / 8, 1, F16, TC_DU, TC_DD>(sm, st + TS_REC + REC_TB, sb + TC_X, quad,
                                                         lane, dlo, dhi);
            fence_proxy_async_smem();
        }
        bar_arrive<BAR_TC_DD, TC_THREADS>();

        ok = mbar_wait(bar_u, par, abort_flag) && ok;
        tc_fence_after();
        {  // S <- gamma_C S + K^T (d o Delta), state row `row`; bf16 copy for K S and Q S
            float u[HN];
            tmem_cols<HN>(tl + TM_U, u);
#pragma unroll
            for (int j = 0; j < HN; ++j) Sr[j] = fmaf(g_C, Sr[j], u[j]);
            put_cols<HN>(sm, TC_SB, row, c_lo, Sr, 1.f);
            fence_proxy_async_smem();
            // with outputs, the next chunk's entering state goes to its image here
            // (at the chunk start it would delay the output rows: measured)
            if (OUTS) save_image(c + 1);
        }
        tc_fence_before();
        bar_arrive<BAR_TC_SB, TC_THREADS>();
        // (the compute warps leave the loop only here, after their last arrive)
        if (!bar_and<BAR_TC, TC_COMPUTE>(ok)) break;
    }
    if (OUTS && nchunks > 0 && !*abort_flag && quad >= 2) {  // the last chunk's outputs
        output(nchunks - 1, g_prev);
        tc_fence_before();
    }
    if (p.S_final && !*abort_flag) {
        float* sf = p.S_final + (((size_t)n * p.H_v + h) * D + row) * D + col0 + c_lo;
#pragma unroll
        for (int j = 0; j < HN / 4; ++j)
            if (c_lo + 4 * j < ncols)
                reinterpret_cast<float4*>(sf)[j] =
                    make_float4(Sr[4 * j], Sr[4 * j + 1], Sr[4 * j + 2], Sr[4 * j + 3]);
    }
    // the last copies land before the CTA exits (bounded waits)
    if (tid == TC_LOADER)
        for (int c = max(0, issued - NSTAGE); c < issued; ++c)
            mbar_wait_drain(&bars[c % NSTAGE], (c / NSTAGE) & 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

template <int NS, typename IO, bool F16, int MODE>
cudaError_t launch_state_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const PrefillParams& prm, cudaStream_t stream) {
    auto kern = state_tc_kernel<NS, IO, F16, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid((D + NS - 1) / NS, prm.H_v, prm.N);
    kern<<<grid, TC_THREADS, TC_SMEM, stream>>>(mq, mk, mv, prm);
    return cudaGetLastError();
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


// ---- segmented prefill (sequence parallelism within one GPU) -------------
// Each sequence is cut into P segments of whole chunks, run as P "virtual"
// sequences.  Phase A carries every segment's state from zero (R) and its
// propagator (P_s, the map of the segment on the entering state); a scan over
// the segments gives the true entering states, S <- P_s S + R_s; phase C reruns
// the segments from those states and writes the outputs.

// cu_v[n P + i] = start of segment i of sequence n (chunk-aligned), cu_v[N P] = T.
__global__ void segment_cu_kernel(const int32_t* __restrict__ cu, int N, int P,
                                  int32_t* __restrict__ cu_v) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx > N * P) return;
    if (idx == N * P) {
        cu_v[idx] = cu[N];
        return;
    }
    const int n = idx / P, i = idx - n * P;
    const int len = cu[n + 1] - cu[n];
    const int per = ((len + C - 1) / C + P - 1) / P;  // chunks per segment
    cu_v[idx] = cu[n] + min(i * per * C, len);
}

// x = hi + lo with both parts tf32: three tf32 products (hi hi, hi lo, lo hi)
// keep an fp32 product's accuracy.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_tf32_frag(float* d, const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Block (column block cb of 32, value head h, sequence n): S_entry[n P + s] is
// the state entering segment s, S_final[n] the state after the last one;
// S <- P_s S + R_s from S0[n] (or zero).  Each step stages P_s in shared
// memory (all its loads in flight at once) and multiplies on the tensor cores
// in split tf32 (three products per term: fp32 accuracy); warp w owns rows
// 16 w .. +15 of the 32 columns.  Row strides (132 and 40 floats) keep the
// fragment loads free of bank conflicts.
constexpr int SCAN_COLS = 32;
constexpr int SCAN_LD = D + 4;
constexpr int CUR_LD = SCAN_COLS + 8;
constexpr uint32_t SCAN_SMEM = (D * SCAN_LD + D * CUR_LD) * sizeof(float);  // 88,064 B
__global__ void __launch_bounds__(256)
    segment_scan_kernel(const float* __restrict__ S0, const float* __restrict__ R,
                        const float* __restrict__ Pm, float* __restrict__ S_entry,
                        float* S_final, int P, int H_v) {
    extern __shared__ float4 scan_sm4[];
    float* Ps = reinterpret_cast<float*>(scan_sm4);  // [D][SCAN_LD]
    float* cur = Ps + D * SCAN_LD;                   // [D][CUR_LD]
    const int cb = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g = lane >> 2, t4 = lane & 3;
    const size_t hs = (size_t)D * D;
    const size_t c0 = (size_t)cb * SCAN_COLS;
    for (int e = t; e < D * SCAN_COLS; e += blockDim.x) {
        const int r = e / SCAN_COLS, c = e % SCAN_COLS;
        cur[r * CUR_LD + c] = S0 ? S0[((size_t)n * H_v + h) * hs + (size_t)r * D + c0 + c] : 0.f;
    }
    const int r0 = 16 * warp;
    for (int sg = 0; sg < P; ++sg) {
        const size_t base = (((size_t)n * P + sg) * H_v + h) * hs;
        const float4* P4 = reinterpret_cast<const float4*>(Pm + base);
        for (int e = t; e < D * D / 4; e += blockDim.x) {
            const int r = e / (D / 4), c4 = e % (D / 4);
            *reinterpret_cast<float4*>(Ps + r * SCAN_LD + 4 * c4) = P4[e];
        }
        // accumulators start from R_s: rows r0 + g (+8), columns 8 nt + 2 t4 (+1)
        float d[4][4];
        const float* Rb = R + base + c0;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int col = 8 * nt + 2 * t4;
            const float2 lo = *reinterpret_cast<const float2*>(Rb + (size_t)(r0 + g) * D + col);
            const float2 hi = *reinterpret_cast<const float2*>(Rb + (size_t)(r0 + g + 8) * D + col);
            d[nt][0] = lo.x;
            d[nt][1] = lo.y;
            d[nt][2] = hi.x;
            d[nt][3] = hi.y;
        }
        __syncthreads();  // P_s staged; cur holds the entering state
        for (int e = t; e < D * SCAN_COLS; e += blockDim.x) {
            const int r = e / SCAN_COLS, c = e % SCAN_COLS;
            S_entry[base + (size_t)r * D + c0 + c] = cur[r * CUR_LD + c];
        }
#pragma unroll 4
        for (int ks = 0; ks < D / 8; ++ks) {
            uint32_t ah[4], al[4];
            const float* Ar = Ps + (r0 + g) * SCAN_LD + 8 * ks + t4;
            split_tf32(Ar[0], ah[0], al[0]);
            split_tf32(Ar[8 * SCAN_LD], ah[1], al[1]);
            split_tf32(Ar[4], ah[2], al[2]);
            split_tf32(Ar[8 * SCAN_LD + 4], ah[3], al[3]);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                uint32_t b0h, b0l, b1h, b1l;
                const float* Br = cur + (8 * ks + t4) * CUR_LD + 8 * nt + g;
                split_tf32(Br[0], b0h, b0l);
                split_tf32(Br[4 * CUR_LD], b1h, b1l);
                mma_tf32_frag(d[nt], ah, b0h, b1h);
                mma_tf32_frag(d[nt], ah, b0l, b1l);
                mma_tf32_frag(d[nt], al, b0h, b1h);
            }
        }
        __syncthreads();  // every warp has read the entering state and P_s
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int col = 8 * nt + 2 * t4;
            *reinterpret_cast<float2*>(cur + (r0 + g) * CUR_LD + col) = make_float2(d[nt][0], d[nt][1]);
            *reinterpret_cast<float2*>(cur + (r0 + g + 8) * CUR_LD + col) =
                make_float2(d[nt][2], d[nt][3]);
        }
        __syncthreads();
    }
    if (S_final)
        for (int e = t; e < D * SCAN_COLS; e += blockDim.x) {
            const int r = e / SCAN_COLS, c = e % SCAN_COLS;
            S_final[((size_t)n * H_v + h) * hs + (size_t)r * D + c0 + c] = cur[r * CUR_LD + c];
        }
}

template <int NS, typename IO, int MODE, bool F16 = false>
cudaError_t launch_pass2(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const PrefillParams& prm, int N, cudaStream_t stream) {
    auto kern = state_pass_kernel<NS, IO, MODE, F16>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, P2_SMEM);
    if (e != cudaSuccess) return e;
    dim3 grid((D + NS - 1) / NS * (MODE == P2_SEGMENT ? 2 : 1), prm.H_v, N);
    kern<<<grid, P2_THREADS, P2_SMEM, stream>>>(mq, mk, mv, prm);
    return cudaGetLastError();
}


size_t staging_bytes(int T, int H_qk, int H_v, bool bf16) {
    if (bf16) return 0;
    return up256((size_t)T * H_qk * D * 2) * 2 + up256((size_t)T * H_v * D * 2);
}

size_t record_bytes(int N, int T, int H_v) {
    const size_t slots = (size_t)N + ((size_t)T + C - 1) / C;
    return up256(slots * H_v * REC_BYTES);
}

}  // namespace

// ---- scratch for gdn_prefill_noalloc -------------------------------------
// A file-scope device array that stands in for the caller's workspace: the
// chunk-operator records (REC_BYTES per chunk slot and value head) and, for
// fp32 q, k, v, their bf16 copies; with a split of the sequences also the
// pieces' starts and states.  Every GPU that loads the library holds it until
// the process exits.  Its host-side name is not a device address: the address is
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

// per-segment states of the segmented prefill: R, P_s and the entering states
size_t segment_state_bytes(int N, int P, int H_v) {
    return up256((size_t)N * P * H_v * D * D * sizeof(float));
}
size_t segment_cu_bytes(int N, int P) { return up256(((size_t)N * P + 1) * sizeof(int32_t)); }

size_t prefill_workspace_bytes(int N, int T, int H_qk, int H_v, bool bf16, int P) {
    if (T == 0) return 0;
    if (P <= 1) return staging_bytes(T, H_qk, H_v, bf16) + record_bytes(N, T, H_v);
    return staging_bytes(T, H_qk, H_v, bf16) + record_bytes(N * P, T, H_v) +
           segment_cu_bytes(N, P) + 3 * segment_state_bytes(N, P, H_v);
}

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0) {
        cudaGetLastError();  // no device: clear the error, assume a B200
        return 148;
    }
    return sms;
}

// d_v slices per head for `units` (sequence, value head) chains: as many as fit
// in one wave of one block per SM (4 x 32, 3 x 48 or 2 x 64 columns)
static int pass2_slices(long long units, int sms) {
    return units * 4 <= sms ? 4 : (units * 3 <= sms ? 3 : 2);
}

int choose_segments(int N, int T, int H_v, int sms) {
    if (N <= 0 || T <= 0 || H_v <= 0) return 1;
    // Cost model in microseconds, from B200 measurements of one chunk step of a
    // state-pass block (one block per SM) by slice width -- with outputs (the
    // prefill proper, phase C) and without (phase A) -- and of one scan step.
    const double chunks = (double)T / N / C;
    auto waves = [&](long long blocks) { return (double)((blocks + sms - 1) / sms); };
    auto t_out = [](int slices) { return slices == 4 ? 1.50 : (slices == 3 ? 1.94 : 2.67); };
    auto t_seg = [](int slices) { return slices == 4 ? 1.11 : (slices == 3 ? 1.48 : 1.80); };
    const double t_scan = 3.0, t_fixed = 20.0;  // per segment; segment launches and scan setup
    const long long u1 = (long long)N * H_v;
    const int s1 = pass2_slices(u1, sms);
    double best = waves(u1 * s1) * t_out(s1) * chunks;
    int best_p = 1;
    for (int P = 2; P <= kMaxSegments; ++P) {
        const double per = std::ceil(chunks / P);
        if (per < 8) break;  // segments of at least 8 chunks
        const long long u = u1 * P;
        const int sa = pass2_slices(2 * u, sms), sc = pass2_slices(u, sms);
        const double cost = (waves(2 * u * sa) * t_seg(sa) + waves(u * sc) * t_out(sc)) * per +
                            t_scan * P + t_fixed;
        if (cost < 0.9 * best) {  // a split must win clearly
            best = cost;
            best_p = P;
        }
    }
    return best_p;
}

// The output state pass runs on tcgen05 when asked, or by default at 48- and
// 64-column slices, where it measured faster (the 16/48-head prefill: 1.10 vs
// 1.24 ms; eight packed sequences: 1.20 vs 1.41 ms); mma.sync at 32-column
// slices (a 2/6-head shard: 0.364 vs 0.369 ms).
static bool output_pass_is_tc(int state_pass, int slices) {
    return state_pass == STATE_PASS_TC || (state_pass == STATE_PASS_AUTO && slices != 4);
}

template <typename IO, bool F16, int MODE>
static cudaError_t launch_state_tc_slices(const CUtensorMap& mq, const CUtensorMap& mk,
                                          const CUtensorMap& mv, const PrefillParams& prm,
                                          int slices, cudaStream_t stream) {
    if (slices == 4) return launch_state_tc<32, IO, F16, MODE>(mq, mk, mv, prm, stream);
    if (slices == 3) return launch_state_tc<48, IO, F16, MODE>(mq, mk, mv, prm, stream);
    return launch_state_tc<64, IO, F16, MODE>(mq, mk, mv, prm, stream);
}

// f16_records: the records were written with fp16 tiles (read by the output
// passes, P2_OUT; the other modes take bf16 records).
template <typename IO, int MODE>
static cudaError_t run_pass2(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                             const PrefillParams& prm, int sms, cudaStream_t stream,
                             int state_pass = STATE_PASS_MMA, bool f16_records = false) {
    // one block per SM at most (each holds ~212 KB of shared memory): split every
    // value head into as many d_v slices as still fit in one wave
    const long long units = (long long)prm.N * prm.H_v * (MODE == P2_SEGMENT ? 2 : 1);
    const int slices = pass2_slices(units, sms);
    if constexpr (MODE == P2_OUT) {
        if (output_pass_is_tc(state_pass, slices))
            return f16_records
                       ? launch_state_tc_slices<IO, true, MODE>(mq, mk, mv, prm, slices, stream)
                       : launch_state_tc_slices<IO, false, MODE>(mq, mk, mv, prm, slices, stream);
    }
    if constexpr (MODE == P2_SAVE || MODE == P2_OUT_SAVE) {  // bf16 records
        if (output_pass_is_tc(state_pass, slices) && !f16_records)
            return launch_state_tc_slices<IO, false, MODE>(mq, mk, mv, prm, slices, stream);
    }
    if (f16_records) {
        if constexpr (MODE == P2_OUT) {
            if (slices == 4) return launch_pass2<32, IO, MODE, true>(mq, mk, mv, prm, prm.N, stream);
            if (slices == 3) return launch_pass2<48, IO, MODE, true>(mq, mk, mv, prm, prm.N, stream);
            return launch_pass2<64, IO, MODE, true>(mq, mk, mv, prm, prm.N, stream);
        }
        return cudaErrorInvalidValue;  // the other modes read bf16 records
    }
    if (slices == 4) return launch_pass2<32, IO, MODE>(mq, mk, mv, prm, prm.N, stream);
    if (slices == 3) return launch_pass2<48, IO, MODE>(mq, mk, mv, prm, prm.N, stream);
    return launch_pass2<64, IO, MODE>(mq, mk, mv, prm, prm.N, stream);
}

// f16_records: write the records' tiles as fp16 (for the output passes of the
// unsplit prefill; the segmented prefill and the gradients take bf16)
static cudaError_t run_pass1(const CUtensorMap& mq, const CUtensorMap& mk,
                             const PrefillParams& prm, cudaStream_t stream,
                             bool f16_records = false) {
    auto kern = f16_records ? chunk_ops_kernel<true> : chunk_ops_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, CO_SMEM);
    if (e != cudaSuccess) return e;
    // all of the unified L1 as shared memory, so that four CTAs fit on an SM
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int group = prm.H_v / prm.H_qk;
    const long long slots = (long long)prm.N + ((long long)prm.T + C - 1) / C;
    dim3 grid((unsigned)slots, prm.H_qk, (group + P1_MAX_GROUP - 1) / P1_MAX_GROUP);
    kern<<<grid, CO_THREADS, CO_SMEM, stream>>>(mq, mk, prm);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* S0, const int32_t* cu_seqlens, int N,
                           int T, int H_qk, int H_v, bool bf16, void* o, float* S_final,
                           void* workspace, int P, int state_pass, cudaStream_t stream) {
    if (T == 0) {  // every sequence is empty: S_final = S0 (or zeros)
        if (!S_final) return cudaSuccess;
        copy_state_kernel<<<592, 256, 0, stream>>>(S0, S_final, (size_t)N * H_v * D * D / 4);
        return cudaGetLastError();
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const void *qb = q, *kb = k, *vb = v;
    if (!bf16) {
        const size_t nqk = (size_t)T * H_qk * D, nv = (size_t)T * H_v * D;
        __nv_bfloat16* q16 = reinterpret_cast<__nv_bfloat16*>(ws);
        __nv_bfloat16* k16 = reinterpret_cast<__nv_bfloat16*>(ws + up256(nqk * 2));
        __nv_bfloat16* v16 = reinterpret_cast<__nv_bfloat16*>(ws + 2 * up256(nqk * 2));
        F32ToBf16Batch cv{};  // the three copies in one launch
        cv.src[0] = static_cast<const float*>(q), cv.dst[0] = q16, cv.n4[0] = nqk / 4;
        cv.src[1] = static_cast<const float*>(k), cv.dst[1] = k16, cv.n4[1] = nqk / 4;
        cv.src[2] = static_cast<const float*>(v), cv.dst[2] = v16, cv.n4[2] = nv / 4;
        f32_to_bf16_batch_kernel<<<592, 256, 0, stream>>>(cv);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        qb = q16;
        kb = k16;
        vb = v16;
    }
    uint8_t* records = ws + staging_bytes(T, H_qk, H_v, bf16);
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, qb, T, (uint64_t)H_qk * D) || !make_map(&mk, kb, T, (uint64_t)H_qk * D) ||
        !make_map(&mv, vb, T, (uint64_t)H_v * D))
        return cudaErrorInvalidValue;
    const int sms = device_sms();
    if (P <= 0) P = choose_segments(N, T, H_v, sms);
    cudaError_t e;
    if (P == 1) {
        // pass 1: every chunk's operators, all chunks at once; pass 2: the state
        // through the chunks
        const PrefillParams prm{log_alpha, beta, S0,      cu_seqlens, o, S_final,
                                records,   nullptr, H_qk, H_v,        N, T};
        // the records' tiles in fp16: both output passes then carry X and Delta in
        // fp16 (11 significant bits against bf16's 8)
        const bool f16 = true;
        if ((e = run_pass1(mq, mk, prm, stream, f16)) != cudaSuccess) return e;
        return bf16 ? run_pass2<__nv_bfloat16, P2_OUT>(mq, mk, mv, prm, sms, stream, state_pass, f16)
                    : run_pass2<float, P2_OUT>(mq, mk, mv, prm, sms, stream, state_pass, f16);
    }
    // segmented: N P virtual sequences
    const int Nv = N * P;
    uint8_t* w = records + record_bytes(Nv, T, H_v);
    int32_t* cu_v = reinterpret_cast<int32_t*>(w);
    w += segment_cu_bytes(N, P);
    float* R = reinterpret_cast<float*>(w);
    w += segment_state_bytes(N, P, H_v);
    float* Pm = reinterpret_cast<float*>(w);
    w += segment_state_bytes(N, P, H_v);
    float* S_entry = reinterpret_cast<float*>(w);
    segment_cu_kernel<<<(Nv + 1 + 255) / 256, 256, 0, stream>>>(cu_seqlens, N, P, cu_v);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // pass 1 over the segments (chunks never cross one, so the operators are those
    // of the unsegmented sequences)
    const PrefillParams pa{log_alpha, beta, nullptr, cu_v, nullptr, R, records, Pm, H_qk, H_v,
                           Nv,        T};
    if ((e = run_pass1(mq, mk, pa, stream)) != cudaSuccess) return e;
    // phase A: R (from zero) and P_s (from the identity, V = 0) of every segment
    e = bf16 ? run_pass2<__nv_bfloat16, P2_SEGMENT>(mq, mk, mv, pa, sms, stream)
             : run_pass2<float, P2_SEGMENT>(mq, mk, mv, pa, sms, stream);
    if (e != cudaSuccess) return e;
    // the entering state of every segment, and the final states
    if ((e = cudaFuncSetAttribute(segment_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  SCAN_SMEM)) != cudaSuccess)
        return e;
    segment_scan_kernel<<<dim3(D / SCAN_COLS, H_v, N), 256, SCAN_SMEM, stream>>>(
        S0, R, Pm, S_entry, S_final, P, H_v);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // phase C: every segment from its entering state, writing the outputs
    const PrefillParams pc{log_alpha, beta, S_entry, cu_v, o, nullptr, records, nullptr,
                           H_qk,      H_v,  Nv,      T};
    return bf16 ? run_pass2<__nv_bfloat16, P2_OUT>(mq, mk, mv, pc, sms, stream, state_pass)
                : run_pass2<float, P2_OUT>(mq, mk, mv, pc, sms, stream, state_pass);
}

// The forward pass the gradients start from (bf16 q, k, v): every chunk's
// operator record (records, N + ceil(T/64) slots x H_v) and entering state
// (S_saved, [slot, H_v, 128, 128] fp32).
cudaError_t launch_prefill_save(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta, const float* S0,
                                const int32_t* cu_seqlens, int N, int T, int H_qk, int H_v,
                                uint8_t* records, uint8_t* S_saved, void* o, float* S_final,
                                bool out_bf16, cudaStream_t stream) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, T, (uint64_t)H_qk * D) || !make_map(&mk, k, T, (uint64_t)H_qk * D) ||
        !make_map(&mv, v, T, (uint64_t)H_v * D))
        return cudaErrorInvalidValue;
    const PrefillParams prm{log_alpha, beta, S0,   cu_seqlens, o, S_final, records,
                            reinterpret_cast<float*>(S_saved), H_qk, H_v, N, T};
    cudaError_t e = run_pass1(mq, mk, prm, stream);
    if (e != cudaSuccess) return e;
    const int sms = device_sms();
    // the state pass on tcgen05 at 48-column slices, as for the prefill
    const int sp = STATE_PASS_AUTO;
    if (!o) return run_pass2<__nv_bfloat16, P2_SAVE>(mq, mk, mv, prm, sms, stream, sp);
    return out_bf16 ? run_pass2<__nv_bfloat16, P2_OUT_SAVE>(mq, mk, mv, prm, sms, stream, sp)
                    : run_pass2<float, P2_OUT_SAVE>(mq, mk, mv, prm, sms, stream, sp);
}

size_t prefill_record_bytes(int N, int T, int H_v) { return record_bytes(N, T, H_v); }

}  // namespace gdn
