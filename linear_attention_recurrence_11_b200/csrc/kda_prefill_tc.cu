// Chunked KDA prefill on the 5th-generation tensor cores (sm_100a):
// bf16 q/k/v/g/beta, fp32 state, dk = dv = 128, chunks of C = 64 tokens.
//
// One CTA (256 threads, ~220 KB shared memory, all 512 TMEM columns) owns one
// (sequence, head) unit and walks its chunks in order, carrying the state
// from chunk to chunk with the KCP composition ("Exercices", Q21-Q22): per
// chunk the incoming state S is mapped to Diag(Gamma_C) S + Kh^T (Ut - W S),
// i.e. the chunk's pair (Diag(Gamma_C) - Kh^T W, Kh^T Ut) applied to S.
//
// Per chunk (G = per-channel cumulative log-decay, Gamma = exp(G)):
//  1. TMA brings q, k, v (128-byte swizzled, straight into the operand tiles
//     they become) and g (plain) into shared memory.
//  2. CUDA cores: cumulative sums of g inside each 16-token subtile (the
//     pages' g_min = -5 bound: 16 x 5 = 80, e^80 fits bf16 and fp32, so every
//     exponent factor below is <= e^80) and the scaled bf16 operands of the
//     decayed Grams. Column block j (tokens 16j..16j+15) of
//        A_rs = beta_r sum_c k_rc k_sc e^{G_rc - G_sc},  P_rs = sum_c q_rc k_sc e^{G_rc - G_sc}
//     is the product of a left operand k_r e^{G_r - G_end(j)} (stacked with
//     q_r e^{G_r - G_end(j)}) and a right operand k_s e^{G_end(j) - G_s}; both
//     factors stay in [0, e^80].
//  3. tcgen05.mma (M=128, N=16, K=128) x 4 -> TMEM; readout to A (fp32) and P (bf16).
//  4. CUDA cores: T = (I + A)^{-1} by 16 x 16 blocks (forward substitution on
//     the diagonal blocks, then block rows by distance).
//  5. tcgen05.mma: [W | Ut] = T Diag(beta) [Gamma*K | V]           (M=128 padded, K=64)
//  6. tcgen05.mma: [U ; Qt S] = [Ut ; 0] + [-W ; Gamma*Q] S          (M=128, K=128)
//  7. tcgen05.mma: O = Qt S + P U (rows 64..127),  dS = Kh^T U       (K=64)
//     with Kh_s = e^{G_C - G_s} k_s; then S <- Diag(Gamma_C) S + dS in fp32
//     in TMEM (the state never leaves the SM between chunks; its bf16 copy
//     feeds step 6 of the next chunk).
// The next chunk's tiles are requested as soon as each staging tile has been
// consumed (g after step 2's cumulative sums, k after step 4, v after step 5,
// q after step 6), so their HBM latency overlaps the rest of the chunk.
// All matrices in shared memory use the 128-byte swizzled layout the TMA
// writes and the tcgen05 descriptors read. No cluster multicast is used.
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

#include <cudaTypedefs.h>

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64, D = 128, NT = 256;
constexpr int SUB = 16, NSUB = C / SUB;

// ---------------------------------------------------------- smem layout
constexpr uint32_t KB = 1024;
constexpr uint32_t OFF_WQ = 0;          // 32 KB  A operand [-W ; Qt], K-major, 128 rows x 128 (2 K-blocks); q lands in rows 64..127
constexpr uint32_t OFF_SB = 32 * KB;    // 32 KB  B operand S (bf16), MN-major [dk rows][dv] (2 N-blocks)
constexpr uint32_t OFF_KS = 64 * KB;    // 16 KB  k tile, [tok rows][dk] (2 blocks of 64 channels)
constexpr uint32_t OFF_V = 80 * KB;     // 16 KB  v: B operand MN-major [tok rows][dv] (2 N-blocks)
constexpr uint32_t OFF_G = 96 * KB;     // 16 KB  g, plain [64][128] bf16
constexpr uint32_t OFF_R = 112 * KB;    // 16 KB  Gram right operand, K-major [s rows][dk]; later U (MN-major B)
constexpr uint32_t OFF_PB = 128 * KB;   // 8 KB   rows 64..127 of the A operand [junk ; P], K-major, K = 64
constexpr uint32_t OFF_L = 136 * KB;    // 80 KB  Gram left operands L3, L2, L1, L0 (compact), then the aliases below
constexpr uint32_t OFF_MISC = 216 * KB;
// L region: compact left operands, L_j has 2 (64 - 16 j) rows (K part, then Q part).
__host__ __device__ constexpr uint32_t l_rows(int j) { return 2u * (64u - 16u * j); }
__host__ __device__ constexpr uint32_t l_off(int j) {
    return j == 3 ? 0u : j == 2 ? 8u * KB : j == 1 ? 24u * KB : 48u * KB;
}
// aliases inside the L region once the Gram MMAs are done
constexpr uint32_t OFF_TB = OFF_L + 0;             // 16 KB  A operand T Diag(beta), K-major, 128 rows x 64
constexpr uint32_t OFF_KT = OFF_L + 16 * KB;       // 16 KB  B operand Gamma*K, MN-major [tok][dk]
constexpr uint32_t OFF_AF = OFF_L + 32 * KB;       // 64 x 65 fp32  A (dead once T is known)
constexpr uint32_t OFF_KHAT = OFF_L + 32 * KB;     // 16 KB  A operand Kh, MN-major [tok][dk] (written after A is dead)
constexpr uint32_t OFF_TF = OFF_L + 49 * KB;       // 64 x 68 fp32  T
constexpr uint32_t OFF_XS = OFF_TF + 64 * 68 * 4;  // 3 x 16 x 20 fp32 scratch
static_assert(OFF_AF + 64 * 65 * 4 <= OFF_TF, "A overlaps T");
static_assert(OFF_XS + 3 * 16 * 20 * 4 <= OFF_MISC, "scratch overflows the L region");
// misc
constexpr uint32_t OFF_BAR = OFF_MISC;              // 2 mbarriers
constexpr uint32_t OFF_TMEMADDR = OFF_MISC + 16;
constexpr uint32_t OFF_BETA = OFF_MISC + 64;        // 64 fp32
constexpr uint32_t OFF_DSUM = OFF_BETA + 256;       // 4 x 128 fp32 subtile totals of g (log2 units)
constexpr uint32_t OFF_GAMC = OFF_DSUM + 2048;      // 128 fp32 Gamma_C
constexpr uint32_t SMEM_USED = OFF_GAMC + 512;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns (512 allocated): the Gram accumulators use the first 64 columns
// of the W region (read out before the W product is issued).
constexpr uint32_t TM_GRAM = 0, TM_W = 0, TM_U = 128, TM_KU = 256, TM_S = 384, TM_COLS = 512;
constexpr uint32_t TMA_BYTES = 6 * 8 * KB + 16 * KB;  // q, k, v: 2 boxes of 8 KB each; g: 1 box of 16 KB
constexpr long long kWaitCycles = 2000000000LL;        // ~1 s at 2 GHz
constexpr float kLog2e = 1.4426950408889634f;

struct TcParams {
    PrefillArgs a;
};

__device__ __forceinline__ float2 ld_bf2(const uint8_t *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ void st_bf2(uint8_t *p, float x, float y) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(x, y);
}
__device__ __forceinline__ uint32_t pack_bf2(float x, float y) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<uint32_t *>(&h);
}

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

__global__ void __launch_bounds__(NT, 1)
kda_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                      const TcParams prm) {
    const PrefillArgs &p = prm.a;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment of the shared-window address (the swizzle patterns key on it)
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + OFF_TMEMADDR);
    float *sBeta = reinterpret_cast<float *>(sm + OFF_BETA);
    float *sD = reinterpret_cast<float *>(sm + OFF_DSUM);
    float *sGamC = reinterpret_cast<float *>(sm + OFF_GAMC);
    float *AF = reinterpret_cast<float *>(sm + OFF_AF);
    float *TF = reinterpret_cast<float *>(sm + OFF_TF);
    float *XS = reinterpret_cast<float *>(sm + OFF_XS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
    const int h = blockIdx.x % p.H;
    const int n = blockIdx.x / p.H;
    const size_t H = (size_t)p.H;
    long long t_begin, len;
    if (p.cu_seqlens) {
        t_begin = p.cu_seqlens[n];
        len = (long long)p.cu_seqlens[n + 1] - t_begin;
    } else {
        t_begin = (long long)n * p.T;
        len = p.T;
    }
    const __nv_bfloat16 *beta = static_cast<const __nv_bfloat16 *>(p.beta);
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.o);
    const size_t state_base = ((size_t)n * H + h) * (size_t)(D * D);
    const long long nchunks = (len + C - 1) / C;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_g);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, TM_COLS);
        tmem_relinquish();
    }
    __syncthreads();

    auto issue_q = [&](long long tok) {
        tma_load_3d(sm + OFF_WQ + 8 * KB, &tm_q, bar_tma, 0, h, (int)tok);
        tma_load_3d(sm + OFF_WQ + 24 * KB, &tm_q, bar_tma, 64, h, (int)tok);
    };
    auto issue_k = [&](long long tok) {
        tma_load_3d(sm + OFF_KS, &tm_k, bar_tma, 0, h, (int)tok);
        tma_load_3d(sm + OFF_KS + 8 * KB, &tm_k, bar_tma, 64, h, (int)tok);
    };
    auto issue_v = [&](long long tok) {
        tma_load_3d(sm + OFF_V, &tm_v, bar_tma, 0, h, (int)tok);
        tma_load_3d(sm + OFF_V + 8 * KB, &tm_v, bar_tma, 64, h, (int)tok);
    };
    auto issue_g = [&](long long tok) { tma_load_3d(sm + OFF_G, &tm_g, bar_tma, 0, h, (int)tok); };
    if (nchunks > 0 && tid == 0) {
        mbar_arrive_expect_tx(bar_tma, TMA_BYTES);
        issue_g(t_begin);
        issue_k(t_begin);
        issue_v(t_begin);
        issue_q(t_begin);
    }
    float bnext = 0.f;  // beta of this thread's row in the next chunk (prefetched)
    if (tid < C && tid < len) bnext = __bfloat162float(beta[(size_t)(t_begin + tid) * H + h]);

    // Incoming state -> TMEM (fp32, lane = dk row, column = dv) and its bf16 copy
    // (B operand, MN-major: row = dk index, 64 dv per 128-byte row, N-block = half).
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    const int si = 32 * quarter + lane;
    {
        uint8_t *sb = sm + OFF_SB + half * 16 * KB;
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = 64 * half + 16 * gq + e;
                v[e] = p.S0 ? p.S0[state_base + (size_t)j * D + si] : 0.f;
            }
            tmem_st16(tmem + tlane + TM_S + 64u * half + 16u * gq, v);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint4 w;
                w.x = pack_bf2(v[8 * cc + 0], v[8 * cc + 1]);
                w.y = pack_bf2(v[8 * cc + 2], v[8 * cc + 3]);
                w.z = pack_bf2(v[8 * cc + 4], v[8 * cc + 5]);
                w.w = pack_bf2(v[8 * cc + 6], v[8 * cc + 7]);
                *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq + 8 * cc)) = w;
            }
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    uint32_t tma_phase = 0, mma_phase = 0;
    bool aborted = false, tma_pending = nchunks > 0;
    // wait for an MMA commit; every thread takes part
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar_mma, mma_phase, kWaitCycles);
        mma_phase ^= 1u;
        tc_fence_after();
        return __syncthreads_or(!ok) == 0;
    };

    // thread roles for the token-parallel passes: subtile ti, channel pair cp
    const int ti = tid >> 6;          // subtile 0..3
    const int cp = tid & 63;          // channel pair
    const int c0 = 2 * cp;            // first channel
    const int cblk = c0 >> 6;         // 64-wide block of the channel
    const int cin = c0 & 63;          // channel inside the block
    constexpr uint32_t idG = idesc_bf16_f32(128, 16, 0, 0);     // Gram: K-major x K-major, N = 16
    constexpr uint32_t idKM = idesc_bf16_f32(128, 128, 0, 1);   // K-major A, MN-major B, N = 128
    constexpr uint32_t idMM = idesc_bf16_f32(128, 128, 1, 1);   // MN-major A and B, N = 128

    for (long long ch = 0; ch < nchunks; ++ch) {
        const long long tok0 = t_begin + ch * C;
        const int Lc = (int)((len - ch * C) < C ? (len - ch * C) : C);
        const bool more = ch + 1 < nchunks;
        const long long tokn = tok0 + C;

        // ---- wait for this chunk's tiles
        {
            const bool ok = mbar_wait_bounded(bar_tma, tma_phase, kWaitCycles);
            tma_phase ^= 1u;
            tma_pending = false;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        if (tid < C) {
            sBeta[tid] = (tid < Lc) ? bnext : 0.f;
            if (more && tid < len - (ch + 1) * C) bnext = __bfloat162float(beta[(size_t)(tokn + tid) * H + h]);
        }
        if (Lc < C) {  // zero the rows past the end of the sequence
            for (int idx = tid; idx < (C - Lc) * 16; idx += NT) {
                const int r = Lc + idx / 16, q16 = idx % 16;  // 16-byte piece of a 256-byte row
                const uint4 z = make_uint4(0, 0, 0, 0);
                const int blk = q16 >> 3, pc = (q16 & 7) * 8;
                *reinterpret_cast<uint4 *>(sm + OFF_WQ + blk * 16 * KB + sw128_offset(64 + r, pc)) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_KS + blk * 8 * KB + sw128_offset(r, pc)) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_V + blk * 8 * KB + sw128_offset(r, pc)) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_G + r * 256 + q16 * 16) = z;
            }
        }
        __syncthreads();

        // ---- phase 1a: cumulative log2-decay inside subtile ti for channels c0, c0+1
        float gl[SUB][2];
        {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int rr = 0; rr < SUB; ++rr) {
                const float2 gv = ld_bf2(sm + OFF_G + (SUB * ti + rr) * 256 + c0 * 2);
                a0 = fmaf(gv.x, kLog2e, a0);
                a1 = fmaf(gv.y, kLog2e, a1);
                gl[rr][0] = a0;
                gl[rr][1] = a1;
            }
            sD[ti * D + c0] = a0;
            sD[ti * D + c0 + 1] = a1;
        }
        __syncthreads();
        if (more && tid == 0) {  // g tile consumed: start the next chunk's loads
            mbar_arrive_expect_tx(bar_tma, TMA_BYTES);
            issue_g(tokn);
        }

        // ---- phase 1b: Gram operands and Gamma * q; keep the exp factors for phase 3
        float F[SUB][2], Rf[SUB][2];
        float ed[NSUB][2], pg[2], post[2];
        {
            float Dm[NSUB][2];
#pragma unroll
            for (int m = 0; m < NSUB; ++m)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    Dm[m][e] = sD[m * D + c0 + e];
                    ed[m][e] = ex2(Dm[m][e]);
                }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float a = 1.f, b = 1.f;
#pragma unroll
                for (int m = 0; m < NSUB; ++m) {
                    if (m < ti) a *= ed[m][e];
                    if (m > ti) b *= ed[m][e];
                }
                pg[e] = a;     // Gamma at the start of subtile ti (relative to the chunk start)
                post[e] = b;   // decay from the end of subtile ti to the end of the chunk
            }
            if (ti == 0) {
#pragma unroll
                for (int e = 0; e < 2; ++e) sGamC[c0 + e] = ed[0][e] * ed[1][e] * ed[2][e] * ed[3][e];
            }
            float E[NSUB][2];  // E[j] = exp(G_start(ti) - G_end(j)) for j < ti, exp(-D_ti) for j = ti
#pragma unroll
            for (int j = 0; j < NSUB; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float acc = 1.f;
#pragma unroll
                    for (int m = 0; m < NSUB; ++m)
                        if (m > j && m < ti) acc *= ed[m][e];
                    E[j][e] = (j == ti) ? ex2(-Dm[ti][e]) : acc;
                }
            float dti[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) dti[e] = (ti == 0) ? Dm[0][e] : (ti == 1) ? Dm[1][e] : (ti == 2) ? Dm[2][e] : Dm[3][e];
#pragma unroll
            for (int rr = 0; rr < SUB; ++rr)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    F[rr][e] = ex2(gl[rr][e]);
                    Rf[rr][e] = ex2(dti[e] - gl[rr][e]);
                }
            uint8_t *const qrow = sm + OFF_WQ + cblk * 16 * KB;
            uint8_t *const krow = sm + OFF_KS + cblk * 8 * KB;
            uint8_t *const rrow = sm + OFF_R + cblk * 8 * KB;
#pragma unroll
            for (int rr = 0; rr < SUB; ++rr) {
                const int r = SUB * ti + rr;
                const uint32_t off_r = sw128_offset(r, cin);       // (r & 7) == (rr & 7)
                const uint32_t off_q = sw128_offset(64 + r, cin);
                const float2 kx = ld_bf2(krow + off_r);
                const float2 qx = ld_bf2(qrow + off_q);
                st_bf2(rrow + off_r, kx.x * Rf[rr][0], kx.y * Rf[rr][1]);
                const float kf0 = kx.x * F[rr][0], kf1 = kx.y * F[rr][1];
                const float qf0 = qx.x * F[rr][0], qf1 = qx.y * F[rr][1];
#pragma unroll
                for (int j = 0; j < NSUB; ++j) {
                    if (j > ti) continue;
                    const uint32_t rows = l_rows(j), hr = rows / 2;
                    uint8_t *Lb = sm + OFF_L + l_off(j) + cblk * rows * 128;
                    st_bf2(Lb + sw128_offset(r - 16 * j, cin), kf0 * E[j][0], kf1 * E[j][1]);
                    st_bf2(Lb + sw128_offset(hr + r - 16 * j, cin), qf0 * E[j][0], qf1 * E[j][1]);
                }
                st_bf2(qrow + off_q, qf0 * pg[0], qf1 * pg[1]);  // Gamma * q in place
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- Gram MMAs: column block j -> TMEM columns 16j..16j+15
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < NSUB; ++j) {
                Opnd A{sbase + OFF_L + l_off(j), false, l_rows(j) * 128u, 0};
                Opnd B{sbase + OFF_R + 16u * j * 128u, false, 8 * KB, 0};
                mma_chain<D / 16>(tmem + TM_GRAM + 16u * j, A, B, idG, false);
            }
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }

        // ---- phase 2: Gram readout -> A (fp32, strictly lower, times beta_r), P (bf16, lower)
        {
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * half + jj;
                float v[16];
                tmem_ld16(tmem + tlane + TM_GRAM + 16u * j, v);
                tmem_wait_ld();
                const int m = 32 * quarter + lane;
                const int kr = 64 - 16 * j;
                if (m < kr) {
                    const int r = 16 * j + m;
                    const float b = sBeta[r];
#pragma unroll
                    for (int s2 = 0; s2 < 16; ++s2) {
                        const int s = 16 * j + s2;
                        AF[r * 65 + s] = (s < r) ? b * v[s2] : 0.f;
                    }
                } else if (m < 2 * kr) {
                    const int r = 16 * j + (m - kr);
                    uint8_t *prow = sm + OFF_PB;
#pragma unroll
                    for (int s2 = 0; s2 < 16; s2 += 2) {
                        const int s = 16 * j + s2;
                        st_bf2(prow + sw128_offset(r, s), (s <= r) ? v[s2] : 0.f, (s + 1 <= r) ? v[s2 + 1] : 0.f);
                    }
                    if (r < 16 * (j + 1)) {  // diagonal block: zero the blocks to its right
                        for (int s = 16 * (j + 1); s < C; s += 8)
                            *reinterpret_cast<uint4 *>(prow + sw128_offset(r, s)) = make_uint4(0, 0, 0, 0);
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- phase 3: T = (I + A)^{-1} (unit lower triangular) by 16 x 16 blocks
        if (tid < 64) {  // diagonal blocks: forward substitution, one column per thread, in registers
            const int bi = tid >> 4, cc = tid & 15, o0 = 16 * bi;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                float acc = (rr == cc) ? 1.f : 0.f;
#pragma unroll
                for (int ss = 0; ss < rr; ++ss) acc = fmaf(-AF[(o0 + rr) * 65 + o0 + ss], x[ss], acc);
                x[rr] = acc;  // zero above the diagonal since x[ss < cc] = 0
                TF[(o0 + rr) * 68 + o0 + cc] = acc;
            }
        }
        __syncthreads();
        // off-diagonal blocks by distance: X = sum_{m=j}^{i-1} A_im T_mj, then T_ij = -T_ii X
#pragma unroll
        for (int dist = 1; dist < NSUB; ++dist) {
            const int nblk = NSUB - dist;
            const int b = tid >> 6, r = (tid & 63) >> 2, q0 = (tid & 3) * 4;
            const int bi = dist + b, bj = b;
            if (b < nblk) {
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int m = bj; m < bi; ++m) {
#pragma unroll
                    for (int kk = 0; kk < 16; ++kk) {
                        const float a = AF[(16 * bi + r) * 65 + 16 * m + kk];
                        const float4 t = *reinterpret_cast<const float4 *>(TF + (16 * m + kk) * 68 + 16 * bj + q0);
                        acc.x = fmaf(a, t.x, acc.x);
                        acc.y = fmaf(a, t.y, acc.y);
                        acc.z = fmaf(a, t.z, acc.z);
                        acc.w = fmaf(a, t.w, acc.w);
                    }
                }
                *reinterpret_cast<float4 *>(XS + b * 320 + r * 20 + q0) = acc;
            }
            __syncthreads();
            if (b < nblk) {
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    const float a = TF[(16 * bi + r) * 68 + 16 * bi + kk];
                    const float4 t = *reinterpret_cast<const float4 *>(XS + b * 320 + kk * 20 + q0);
                    acc.x = fmaf(a, t.x, acc.x);
                    acc.y = fmaf(a, t.y, acc.y);
                    acc.z = fmaf(a, t.z, acc.z);
                    acc.w = fmaf(a, t.w, acc.w);
                }
                *reinterpret_cast<float4 *>(TF + (16 * bi + r) * 68 + 16 * bj + q0) =
                    make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
            }
            __syncthreads();
        }
        // T Diag(beta) -> bf16 A operand (rows 0..63), zero rows 64..127
        for (int idx = tid; idx < 128 * 8; idx += NT) {
            const int r = idx >> 3, pc = (idx & 7) * 8;
            uint4 w = make_uint4(0, 0, 0, 0);
            if (r < C) {
                const float4 t0 = *reinterpret_cast<const float4 *>(TF + r * 68 + pc);
                const float4 t1 = *reinterpret_cast<const float4 *>(TF + r * 68 + pc + 4);
                const float t[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
                float u[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) u[e] = (pc + e <= r) ? t[e] * sBeta[pc + e] : 0.f;
                w.x = pack_bf2(u[0], u[1]);
                w.y = pack_bf2(u[2], u[3]);
                w.z = pack_bf2(u[4], u[5]);
                w.w = pack_bf2(u[6], u[7]);
            }
            *reinterpret_cast<uint4 *>(sm + OFF_TB + sw128_offset(r, pc)) = w;
        }
        // Gamma * k -> KT and Kh = exp(G_C - G_s) * k_s -> KHAT (A is dead now)
        {
            const uint8_t *krow = sm + OFF_KS + cblk * 8 * KB;
            uint8_t *ktrow = sm + OFF_KT + cblk * 8 * KB;
            uint8_t *khrow = sm + OFF_KHAT + cblk * 8 * KB;
#pragma unroll
            for (int rr = 0; rr < SUB; ++rr) {
                const uint32_t off_r = sw128_offset(SUB * ti + rr, cin);
                const float2 kx = ld_bf2(krow + off_r);
                st_bf2(ktrow + off_r, kx.x * F[rr][0] * pg[0], kx.y * F[rr][1] * pg[1]);
                st_bf2(khrow + off_r, kx.x * Rf[rr][0] * post[0], kx.y * Rf[rr][1] * post[1]);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- [W | Ut] = T Diag(beta) [Gamma*K | V]
        if (tid == 0) {
            if (more) issue_k(tokn);  // the k tile is consumed
            tc_fence_after();
            Opnd A{sbase + OFF_TB, false, 16 * KB, 0};
            Opnd BK{sbase + OFF_KT, true, 0, 8 * KB};
            Opnd BV{sbase + OFF_V, true, 0, 8 * KB};
            mma_chain<C / 16>(tmem + TM_W, A, BK, idKM, false);
            mma_chain<C / 16>(tmem + TM_U, A, BV, idKM, false);
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }
        if (more && tid == 0) issue_v(tokn);
        tma_pending = more;

        // ---- phase 4: -W (rows 0..63) into the [-W ; Qt] operand
        if (quarter < 2) {
            const int r = 32 * quarter + lane;
            uint8_t *base = sm + OFF_WQ + half * 16 * KB;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                float v[16];
                tmem_ld16(tmem + tlane + TM_W + 64u * half + 16u * gq, v);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint4 w;
                    w.x = pack_bf2(-v[8 * cc + 0], -v[8 * cc + 1]);
                    w.y = pack_bf2(-v[8 * cc + 2], -v[8 * cc + 3]);
                    w.z = pack_bf2(-v[8 * cc + 4], -v[8 * cc + 5]);
                    w.w = pack_bf2(-v[8 * cc + 6], -v[8 * cc + 7]);
                    *reinterpret_cast<uint4 *>(base + sw128_offset(r, 16 * gq + 8 * cc)) = w;
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- [U ; Qt S] = [Ut ; 0] + [-W ; Qt] S
        if (tid == 0) {
            tc_fence_after();
            Opnd A{sbase + OFF_WQ, false, 16 * KB, 0};
            Opnd B{sbase + OFF_SB, true, 0, 16 * KB};
            mma_chain<D / 16>(tmem + TM_U, A, B, idKM, true);
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }
        if (more && tid == 0) issue_q(tokn);  // rows 64..127 of the [-W ; Qt] operand are free

        // ---- phase 5: U (rows 0..63) -> bf16 B operand, MN-major [tok][dv]
        if (quarter < 2) {
            const int r = 32 * quarter + lane;
            uint8_t *base = sm + OFF_R + half * 8 * KB;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                float v[16];
                tmem_ld16(tmem + tlane + TM_U + 64u * half + 16u * gq, v);
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint4 w;
                    w.x = pack_bf2(v[8 * cc + 0], v[8 * cc + 1]);
                    w.y = pack_bf2(v[8 * cc + 2], v[8 * cc + 3]);
                    w.z = pack_bf2(v[8 * cc + 4], v[8 * cc + 5]);
                    w.w = pack_bf2(v[8 * cc + 6], v[8 * cc + 7]);
                    *reinterpret_cast<uint4 *>(base + sw128_offset(r, 16 * gq + 8 * cc)) = w;
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- O = Qt S + P U (rows 64..127 of the same accumulator), dS = Kh^T U
        if (tid == 0) {
            tc_fence_after();
            Opnd AP{sbase + OFF_PB - 8 * KB, false, 16 * KB, 0};
            Opnd BU{sbase + OFF_R, true, 0, 8 * KB};
            Opnd AK{sbase + OFF_KHAT, true, 0, 8 * KB};
            mma_chain<C / 16>(tmem + TM_KU, AK, BU, idMM, false);
            mma_chain<C / 16>(tmem + TM_U, AP, BU, idKM, true);
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }

        // ---- phase 6: outputs and the state update S <- Diag(Gamma_C) S + dS
        if (quarter >= 2) {
            const int r = 32 * quarter + lane - 64;
            uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)(tok0 + r) * H + h) * D + 64 * half);
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                float v[16];
                tmem_ld16(tmem + tlane + TM_U + 64u * half + 16u * gq, v);
                tmem_wait_ld();
                if (r < Lc) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        uint4 w;
                        w.x = pack_bf2(v[8 * cc + 0], v[8 * cc + 1]);
                        w.y = pack_bf2(v[8 * cc + 2], v[8 * cc + 3]);
                        w.z = pack_bf2(v[8 * cc + 4], v[8 * cc + 5]);
                        w.w = pack_bf2(v[8 * cc + 6], v[8 * cc + 7]);
                        dst[2 * gq + cc] = w;
                    }
                }
            }
        }
        {
            const float gam = sGamC[si];
            uint8_t *sb = sm + OFF_SB + half * 16 * KB;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                float sv[16], dv[16];
                const uint32_t col = 64u * half + 16u * gq;
                tmem_ld16(tmem + tlane + TM_S + col, sv);
                tmem_ld16(tmem + tlane + TM_KU + col, dv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) sv[e] = fmaf(gam, sv[e], dv[e]);
                tmem_st16(tmem + tlane + TM_S + col, sv);
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    uint4 w;
                    w.x = pack_bf2(sv[8 * cc + 0], sv[8 * cc + 1]);
                    w.y = pack_bf2(sv[8 * cc + 2], sv[8 * cc + 3]);
                    w.z = pack_bf2(sv[8 * cc + 4], sv[8 * cc + 5]);
                    w.w = pack_bf2(sv[8 * cc + 6], sv[8 * cc + 7]);
                    *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq + 8 * cc)) = w;
                }
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (aborted) {
        if (tid == 0 && p.dev_status) atomicExch(p.dev_status, (int)KDA_ERR_TIMEOUT);
        if (tma_pending && tid == 0) mbar_wait_bounded(bar_tma, tma_phase, kWaitCycles);
    } else if (p.ST) {
        tc_fence_after();
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
            float sv[16];
            tmem_ld16(tmem + tlane + TM_S + 64u * half + 16u * gq, sv);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = 64 * half + 16 * gq + e;
                p.ST[state_base + (size_t)j * D + si] = sv[e];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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
bool make_map(CUtensorMap *m, const void *base, size_t tokens, int H, int inner, bool swizzle) {
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

}  // namespace

bool prefill_tc_supported(int dk, int dv, int chunk, int dtype) {
    return dk == D && dv == D && chunk == C && dtype == KDA_DTYPE_BF16;
}

size_t prefill_tc_workspace(const PrefillArgs &) { return 0; }

int prefill_tc_launches(const PrefillArgs &a) { return (a.num_units > 0 && a.H > 0) ? 1 : 0; }

cudaError_t launch_prefill_tc(const PrefillArgs &a) {
    if (a.num_units == 0) return cudaSuccess;
    const size_t tokens = a.cu_seqlens ? (size_t)a.T : (size_t)a.B * (size_t)a.T;
    // A batch without tokens only copies S0 to S_T; the SIMT kernel does that.
    if (tokens == 0) return launch_prefill_simt(a);
    CUtensorMap mq, mk, mv, mg;
    if (!make_map(&mq, a.q, tokens, a.H, 64, true) || !make_map(&mk, a.k, tokens, a.H, 64, true) ||
        !make_map(&mv, a.v, tokens, a.H, 64, true) || !make_map(&mg, a.g, tokens, a.H, 128, false))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kda_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    TcParams prm{a};
    const unsigned grid = (unsigned)((size_t)a.num_units * a.H);
    kda_prefill_tc_kernel<<<grid, NT, SMEM_BYTES, a.stream>>>(mq, mk, mv, mg, prm);
    return cudaGetLastError();
}

}  // namespace kda
