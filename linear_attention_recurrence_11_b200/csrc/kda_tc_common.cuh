// Device helpers shared by the tensor-core prefill kernels (bf16, dk = dv = 128,
// chunks of 64 tokens): bf16 packing, tcgen05 MMA chains over 128-byte
// swizzled shared-memory operands, and the off-diagonal part of the
// unit-lower-triangular inverse T = (I + A)^{-1} with warp-level TF32 MMAs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "kda_sm100.cuh"

namespace kda {
namespace tc {

using namespace sm100;

constexpr int C = 64, D = 128;
constexpr int SUB = 16, NSUB = C / SUB;
// fp32 row strides (in floats) of the small matrices of the triangular inverse, chosen so that
// the warp-level MMA fragments below read shared memory without bank conflicts: rows of an A
// fragment are LDA apart (LDA = 4 mod 32), rows of a B fragment LDX apart (LDX = 8 mod 32).
constexpr int LDA = 68, LDT = 68, LDX = 40;
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at 2 GHz
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void st_bf2(uint8_t *p, float x, float y) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(x, y);
}
__device__ __forceinline__ uint32_t pack_bf2(float x, float y) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<uint32_t *>(&h);
}

// 16 fp32 values (times `scale`) -> 16 bf16 in two 16-byte words
__device__ __forceinline__ void pack16(const float *v, float scale, uint4 &w0, uint4 &w1) {
    w0.x = pack_bf2(scale * v[0], scale * v[1]);
    w0.y = pack_bf2(scale * v[2], scale * v[3]);
    w0.z = pack_bf2(scale * v[4], scale * v[5]);
    w0.w = pack_bf2(scale * v[6], scale * v[7]);
    w1.x = pack_bf2(scale * v[8], scale * v[9]);
    w1.y = pack_bf2(scale * v[10], scale * v[11]);
    w1.z = pack_bf2(scale * v[12], scale * v[13]);
    w1.w = pack_bf2(scale * v[14], scale * v[15]);
}

// ------------------------------------------------------------- thread groups
// A group of 256 threads that synchronise among themselves on named barrier `id` (0 is the
// CTA barrier, the same as __syncthreads for a 256-thread CTA); a 512-thread CTA can run two
// groups side by side on barriers 1 and 2.
__device__ __forceinline__ void group_sync(uint32_t id) { asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory"); }
__device__ __forceinline__ bool group_sync_or(uint32_t id, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, 256, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id)
        : "memory");
    return r != 0;
}
struct Group {
    int tid;           // 0..255 within the group
    uint32_t id;       // named barrier
    bool relinquish;   // the group is the whole CTA: give up the TMEM allocation permit after allocating
    __device__ __forceinline__ void sync() const { group_sync(id); }
    __device__ __forceinline__ bool sync_or(bool p) const { return group_sync_or(id, p); }
};

// ------------------------------------------------------------- MMA issue
// Operand tile in shared memory (128-byte swizzled rows): K-major tiles keep
// 64-wide K blocks `kblk` bytes apart; MN-major tiles keep 64-wide M/N blocks
// `lbo` bytes apart and advance 16 K-rows (2 KB) per MMA step.
struct Opnd {
    uint32_t base;
    bool mn;
    uint32_t kblk;
    uint32_t lbo;
};

template <int KSTEPS>
__device__ __forceinline__ void mma_chain(uint32_t d_tmem, const Opnd &A, const Opnd &B, uint32_t idesc,
                                          bool accumulate) {
    const uint64_t da = smem_desc_sw128(A.base, A.mn ? A.lbo : 16u, 1024u);
    const uint64_t db = smem_desc_sw128(B.base, B.mn ? B.lbo : 16u, 1024u);
#pragma unroll
    for (int k = 0; k < KSTEPS; ++k) {
        const uint32_t oa = A.mn ? (uint32_t)k * 2048u : (uint32_t)(k >> 2) * A.kblk + (uint32_t)(k & 3) * 32u;
        const uint32_t ob = B.mn ? (uint32_t)k * 2048u : (uint32_t)(k >> 2) * B.kblk + (uint32_t)(k & 3) * 32u;
        mma_bf16_ss(d_tmem, da + (oa >> 4), db + (ob >> 4), idesc, (accumulate || k > 0) ? 1u : 0u);
    }
}


// fp32 -> tf32 (round to nearest, ties away), for the warp-level MMAs below.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t y;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(y) : "f"(x));
    return y;
}

// One warp: C[16 x 8] = sum_k A[ar + 0..15][ac + k] * B[br + k][bc + 0..7], k < K,
// A and B fp32 in shared memory (row strides lda, ldb), with mma.sync m16n8k8 TF32
// (fp32 accumulation). Fragment (g = lane / 4, t = lane % 4): A rows g, g + 8 and
// columns t, t + 4; B rows t, t + 4 and column g; C rows g, g + 8, columns 2t, 2t + 1.
template <int K>
__device__ __forceinline__ void warp_mma_16x8(const float *A, int lda, int ar, int ac, const float *B, int ldb,
                                              int br, int bc, float (&c)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    c[0] = c[1] = c[2] = c[3] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t a0 = to_tf32(A[(ar + g) * lda + ac + k0 + t]);
        const uint32_t a1 = to_tf32(A[(ar + g + 8) * lda + ac + k0 + t]);
        const uint32_t a2 = to_tf32(A[(ar + g) * lda + ac + k0 + t + 4]);
        const uint32_t a3 = to_tf32(A[(ar + g + 8) * lda + ac + k0 + t + 4]);
        const uint32_t b0 = to_tf32(B[(br + k0 + t) * ldb + bc + g]);
        const uint32_t b1 = to_tf32(B[(br + k0 + t + 4) * ldb + bc + g]);
        asm volatile(
            "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}

// Store a C fragment of warp_mma_16x8 (times `scale`) at D[dr + .., dc + ..]; with tb, also
// the same values times beta[column] as bf16 at (row, column) of tb, a 128-byte swizzled tile.
__device__ __forceinline__ void warp_store_16x8(float *Dm, int ldd, int dr, int dc, const float (&c)[4],
                                                float scale, uint8_t *tb = nullptr, const float *beta = nullptr) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const float2 lo = make_float2(scale * c[0], scale * c[1]), hi = make_float2(scale * c[2], scale * c[3]);
    *reinterpret_cast<float2 *>(Dm + (dr + g) * ldd + dc + 2 * t) = lo;
    *reinterpret_cast<float2 *>(Dm + (dr + g + 8) * ldd + dc + 2 * t) = hi;
    if (tb) {
        const float b0 = beta[dc + 2 * t], b1 = beta[dc + 2 * t + 1];
        st_bf2(tb + sw128_offset(dr + g, dc + 2 * t), lo.x * b0, lo.y * b1);
        st_bf2(tb + sw128_offset(dr + g + 8, dc + 2 * t), hi.x * b0, hi.y * b1);
    }
}

// Off-diagonal part of T = (I + A)^{-1} (64 x 64 unit lower triangular) once the
// four 16 x 16 diagonal blocks T_ii are in place (zero above their diagonal, and
// zero in the 16 x 16 block to the right of T_00 and T_22):
//   level 1:  T_10 = -T_11 A_10 T_00,  T_32 = -T_33 A_32 T_22                 (16 x 16)
//   level 2:  T[32:64, 0:32] = -T[32:64, 32:64] A[32:64, 0:32] T[0:32, 0:32]  (32 x 32)
// i.e. the 2 x 2 block inverse applied twice; each product is a handful of
// warp-level TF32 MMAs. A: 64 x LDA fp32 (strictly lower), T: 64 x LDT fp32,
// XS: scratch of 32 x 36 fp32. With tb, every block of T computed here is also written
// times beta[column] as bf16 into tb (the A operand T Diag(beta), 128-byte swizzled rows).
__device__ __forceinline__ void tri_inverse_offdiag(const float *AF, float *TF, float *XS, int tid,
                                                    uint32_t bar_id = 0, uint8_t *tb = nullptr,
                                                    const float *beta = nullptr) {
    const int warp = tid >> 5;
    float c[4];
    // level 1: 2 blocks x 2 column tiles of 8 -> warps 0..3
    const int b = (warp >> 1) & 1, nt = warp & 1;
    const int i1 = 16 * (2 * b + 1), j1 = 16 * (2 * b);
    if (warp < 4) {
        warp_mma_16x8<16>(AF, LDA, i1, j1, TF, LDT, j1, j1 + 8 * nt, c);     // X = A_ij T_jj
        warp_store_16x8(XS, LDX, 16 * b, 8 * nt, c, 1.f);
        __syncwarp();  // the product below reads only the 16 x 8 tile of X this warp wrote
        warp_mma_16x8<16>(TF, LDT, i1, i1, XS, LDX, 16 * b, 8 * nt, c);       // T_ij = -T_ii X
        warp_store_16x8(TF, LDT, i1, j1 + 8 * nt, c, -1.f, tb, beta);
    }
    group_sync(bar_id);
    // level 2: 2 row tiles x 4 column tiles -> warps 0..7
    const int mt = warp >> 2, n2 = warp & 3;
    warp_mma_16x8<32>(AF, LDA, 32 + 16 * mt, 0, TF, LDT, 0, 8 * n2, c);        // X = A21 T_lo
    warp_store_16x8(XS, LDX, 16 * mt, 8 * n2, c, 1.f);
    group_sync(bar_id);
    warp_mma_16x8<32>(TF, LDT, 32 + 16 * mt, 32, XS, LDX, 0, 8 * n2, c);       // T21 = -T_hi X
    warp_store_16x8(TF, LDT, 32 + 16 * mt, 8 * n2, c, -1.f, tb, beta);
    group_sync(bar_id);
}

// ------------------------------------------------------------------ host side
// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
inline PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 3-D map over a token-major [tokens, H, 128] bf16 tensor; box = (inner, 1, 64 tokens).
inline bool make_map(CUtensorMap *m, const void *base, size_t tokens, int H, int inner, bool swizzle) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {(cuuint32_t)inner, 1, (cuuint32_t)C};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace kda
