// gdn_tiles.cuh -- chunk constants, the chunk-operator record layout, and the
// shared-memory tile helpers (128-byte-swizzled bf16 tiles, ldmatrix
// fragments, mma.sync m16n8k16 bf16 products, named barriers) used by the
// prefill and its gradients.
#pragma once

#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>

#include "gdn_common.cuh"

namespace gdn {
namespace {

constexpr int C = 64;            // chunk length
constexpr int D = 128;           // head dim (d_k = d_v)
constexpr uint32_t HALF = 8192;  // one 64 x 64 bf16 tile: 64 rows x 128 B
constexpr float LOG2E = 1.4426950408889634f;

// ---- chunk operator record (workspace), also its image in shared memory ----
constexpr uint32_t REC_TB = 0;                 // T diag(beta), 64 x 64 bf16, swizzled
constexpr uint32_t REC_MQ = HALF;              // M o Q K^T,    64 x 64 bf16, swizzled
constexpr uint32_t REC_VEC = 2 * HALF;         // gamma[64], d[64], gamma_C, pad -> 132 floats
constexpr uint32_t REC_VEC_FLOATS = 132;
constexpr uint32_t REC_BYTES = REC_VEC + REC_VEC_FLOATS * 4;  // 16,912
// A 128 x 128 state saved for the gradients: bf16, two 128-row halves of 64
// columns (16 KB apart), 128B-swizzled -- element (r, c) at
// taddr_e(0, r, c, 2 * HALF); the tile layout the gradient kernel multiplies.
constexpr uint32_t STATE_IMAGE_BYTES = D * D * 2;
static_assert(REC_BYTES % 16 == 0, "bulk copies move multiples of 16 bytes");

// Record slot of chunk c of sequence n (first token t0 = cu[n] + 64 c):
// j = n + floor(t0 / 64).  Distinct chunks get distinct slots, all below
// N + ceil(T / 64), without reading cu_seqlens on the host.
__host__ __device__ __forceinline__ long long record_slot(int n, int t0) {
    return (long long)n + t0 / C;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int ID, int N>
__device__ __forceinline__ void bar_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(N) : "memory");
}
// Arrive on a named barrier without waiting (producers of a producer/consumer
// hand-off; the consumers bar_sync on the same barrier and count).
template <int ID, int N>
__device__ __forceinline__ void bar_arrive() {
    asm volatile("bar.arrive %0, %1;" ::"n"(ID), "n"(N) : "memory");
}
// Named barrier that also returns the AND of every participant's `ok`.
template <int ID, int N>
__device__ __forceinline__ bool bar_and(bool ok) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok), "n"(ID), "n"(N)
        : "memory");
    return r != 0;
}

// Wait bounded in time only (used to drain in-flight copies after an abort).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const uint32_t addr = smem_u32(bar);
    const unsigned long long t0 = globaltimer();
    while (!mbar_try_wait(addr, parity)) {
        if (globaltimer() - t0 > kWaitLimitNs) {
            atomicOr(&g_status, GDN_DEV_TIMEOUT);
            return;
        }
    }
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

__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16x2(lo, hi); }

// fp32 -> bf16 copies of up to four row-major operands for fp32 I/O (the tensor
// maps read bf16), in one launch: n4[i] = elements / 4 of array i (0 for unused
// slots); the threads stride over the arrays end to end.  The pointers are
// picked by comparisons, not by indexing the parameter arrays at run time.
struct F32ToBf16Batch {
    const float* src[4];
    __nv_bfloat16* dst[4];
    size_t n4[4];
};
__global__ void f32_to_bf16_batch_kernel(const F32ToBf16Batch b) {
    const size_t e1 = b.n4[0], e2 = e1 + b.n4[1], e3 = e2 + b.n4[2], total = e3 + b.n4[3];
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
         i += (size_t)gridDim.x * blockDim.x) {
        const float* s;
        __nv_bfloat16* d;
        size_t j;
        if (i < e1) {
            s = b.src[0], d = b.dst[0], j = i;
        } else if (i < e2) {
            s = b.src[1], d = b.dst[1], j = i - e1;
        } else if (i < e3) {
            s = b.src[2], d = b.dst[2], j = i - e2;
        } else {
            s = b.src[3], d = b.dst[3], j = i - e3;
        }
        const float4 v = reinterpret_cast<const float4*>(s)[j];
        reinterpret_cast<uint2*>(d)[j] = make_uint2(pack2(v.x, v.y), pack2(v.z, v.w));
    }
}

inline size_t up256(size_t b) { return (b + 255) & ~size_t(255); }

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// D += A (16 x 8, fp32 rows of stride lda) * B (8 x 8, fp32 rows of stride ldb), both
// rounded to tf32, fp32 accumulate (m16n8k8).
__device__ __forceinline__ void mma_tf32(float* d, const float* A, int lda, const float* B,
                                         int ldb, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t a0 = to_tf32(A[g * lda + t]), a1 = to_tf32(A[(g + 8) * lda + t]);
    const uint32_t a2 = to_tf32(A[g * lda + t + 4]), a3 = to_tf32(A[(g + 8) * lda + t + 4]);
    const uint32_t b0 = to_tf32(B[t * ldb + g]), b1 = to_tf32(B[(t + 4) * ldb + g]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Store an accumulator tile (rows m0.., NT n-tiles from column 0) as bf16 into a
// swizzled tile, scaled per row by rs_lo (row g) and rs_hi (row g+8).
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

// Sequence n and chunk c of record slot j, or n = -1 if no chunk maps to j.
// The first slot of sequence n, n + floor(cu[n] / 64), increases strictly with
// n, so the owner of j is the last sequence whose first slot is <= j.
__device__ __forceinline__ void slot_owner(const int32_t* cu, int N, int j, int& n, int& c) {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (record_slot(mid, cu[mid]) <= j) lo = mid; else hi = mid - 1;
    }
    n = lo;
    c = j - (int)record_slot(lo, cu[lo]);
    const int nch = (cu[lo + 1] - cu[lo] + C - 1) / C;
    if (c < 0 || c >= nch) n = -1;
}

__device__ __forceinline__ void ldsm_x2_t(uint32_t a, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(a));
}
// B fragment of one n-tile (n0) x (k0..k0+15) from an MN-major tile (stored rows k, cols n).
__device__ __forceinline__ void ldb_mn1(uint32_t base, int n0, int k0, int lane, uint32_t* b) {
    ldsm_x2_t(taddr(base, k0 + (lane & 7) + (((lane >> 3) & 1) << 3), n0, 0), b);
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

}  // namespace
}  // namespace gdn
