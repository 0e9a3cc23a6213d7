// Chunked KDA prefill on the 5th-generation tensor cores (sm_100a):
// bf16 q/k/v/g/beta, fp32 state, dk = dv = 128, chunks of C = 64 tokens.
//
// One CTA (256 threads, ~220 KB shared memory, 448 TMEM columns) owns one
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
//     registers (the state never leaves the SM between chunks; its bf16 copy
//     feeds step 6 of the next chunk).
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
constexpr uint32_t OFF_WQ = 0;          // 32 KB  A operand [-W ; Qt], K-major, 128 rows x 128 (2 K-blocks)
constexpr uint32_t OFF_SB = 32 * KB;    // 32 KB  B operand S (bf16), MN-major [dk rows][dv] (2 N-blocks)
constexpr uint32_t OFF_KH = 64 * KB;    // 16 KB  k, then Kh: A operand MN-major [tok rows][dk] (2 M-blocks)
constexpr uint32_t OFF_V = 80 * KB;     // 16 KB  v: B operand MN-major [tok rows][dv] (2 N-blocks)
constexpr uint32_t OFF_G = 96 * KB;     // 16 KB  g, plain [64][128] bf16
constexpr uint32_t OFF_R = 112 * KB;    // 16 KB  Gram right operand, K-major [s rows][dk]; later U (MN-major B)
constexpr uint32_t OFF_PB = 128 * KB;   // 8 KB   rows 64..127 of the A operand [junk ; P], K-major, K = 64
constexpr uint32_t OFF_L = 136 * KB;    // 80 KB  Gram left operands L3, L2, L1, L0 (compact), then phase-4 scratch
constexpr uint32_t OFF_MISC = 216 * KB;
// L region: compact left operands, L_j has 2 (64 - 16 j) rows (K part, then Q part).
__host__ __device__ constexpr uint32_t l_rows(int j) { return 2u * (64u - 16u * j); }
__host__ __device__ constexpr uint32_t l_off(int j) {
    return j == 3 ? 0u : j == 2 ? 8u * KB : j == 1 ? 24u * KB : 48u * KB;
}
// phase-4 aliases inside the L region
constexpr uint32_t OFF_TB = OFF_L + 0;           // 16 KB  A operand T Diag(beta), K-major, 128 rows x 64
constexpr uint32_t OFF_KT = OFF_L + 16 * KB;     // 16 KB  B operand Gamma*K, MN-major [tok][dk]
constexpr uint32_t OFF_AF = OFF_L + 32 * KB;     // 64 x 65 fp32  A
constexpr uint32_t OFF_TF = OFF_AF + 64 * 65 * 4; // 64 x 65 fp32  T
constexpr uint32_t OFF_XS = OFF_TF + 64 * 65 * 4; // 3 x 16 x 17 fp32 scratch
static_assert(OFF_XS + 3 * 16 * 17 * 4 <= OFF_MISC, "phase-4 scratch overflows the L region");
// misc
constexpr uint32_t OFF_BAR = OFF_MISC;              // 2 mbarriers
constexpr uint32_t OFF_TMEMADDR = OFF_MISC + 16;
constexpr uint32_t OFF_BETA = OFF_MISC + 64;        // 64 fp32
constexpr uint32_t OFF_DSUM = OFF_BETA + 256;       // 4 x 128 fp32 subtile totals of g
constexpr uint32_t OFF_GAMC = OFF_DSUM + 2048;      // 128 fp32 Gamma_C
constexpr uint32_t SMEM_USED = OFF_GAMC + 512;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns
constexpr uint32_t TM_GRAM = 0, TM_W = 64, TM_U = 192, TM_KU = 320, TM_COLS = 512;
constexpr uint32_t TMA_BYTES = 6 * 8 * KB + 16 * KB;  // q, k, v: 2 boxes of 8 KB each; g: 1 box of 16 KB
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at 2 GHz

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
// A, B: K-major (kmaj) or MN-major operand tiles; see the layout notes above.
struct Opnd {
    uint32_t base;    // shared address
    bool mn;          // MN-major?
    uint32_t kblk;    // K-major: byte stride between 64-wide K blocks
    uint32_t lbo;     // MN-major: byte stride between 64-wide MN blocks
};

__device__ __forceinline__ uint64_t opnd_desc(const Opnd &o, int k) {
    // k = index of the 16-wide K step
    if (!o.mn) {
        const uint32_t a = o.base + (uint32_t)(k >> 2) * o.kblk + (uint32_t)(k & 3) * 32u;
        return smem_desc_sw128(a, 16u, 1024u);
    }
    const uint32_t a = o.base + (uint32_t)k * 2048u;  // 16 K-rows of 128 bytes
    return smem_desc_sw128(a, o.lbo, 1024u);
}

__device__ __forceinline__ void mma_chain(uint32_t d_tmem, const Opnd &A, const Opnd &B, int N, int ksteps,
                                          bool accumulate) {
    const uint32_t id = idesc_bf16_f32(128, N, A.mn ? 1 : 0, B.mn ? 1 : 0);
    for (int k = 0; k < ksteps; ++k)
        mma_bf16_ss(d_tmem, opnd_desc(A, k), opnd_desc(B, k), id, (accumulate || k > 0) ? 1u : 0u);
}

// 64 fp32 TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    float t[16];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        tmem_ld16(taddr + 16u * c, t);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[16 * c + i] = t[i];
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

    // Incoming state: thread owns dk row i = 32*quarter + lane, dv columns 64*half .. +63.
    const int si = 32 * quarter + lane;
    float S[64];
#pragma unroll
    for (int jj = 0; jj < 64; ++jj) {
        const int j = 64 * half + jj;
        S[jj] = p.S0 ? p.S0[state_base + (size_t)j * D + si] : 0.f;
    }
    // bf16 copy: B operand, MN-major: row = dk index, 64 dv per 128-byte row, N-block = half
    auto write_state_bf16 = [&]() {
        uint8_t *base = sm + OFF_SB + half * 16 * KB;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
            uint4 w;
            w.x = pack_bf2(S[8 * cc + 0], S[8 * cc + 1]);
            w.y = pack_bf2(S[8 * cc + 2], S[8 * cc + 3]);
            w.z = pack_bf2(S[8 * cc + 4], S[8 * cc + 5]);
            w.w = pack_bf2(S[8 * cc + 6], S[8 * cc + 7]);
            *reinterpret_cast<uint4 *>(base + sw128_offset(si, 8 * cc)) = w;
        }
    };
    write_state_bf16();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;

    const long long nchunks = (len + C - 1) / C;
    uint32_t tma_phase = 0, mma_phase = 0;
    bool aborted = false;

    auto issue_qk = [&](long long tok) {
        tma_load_3d(sm + OFF_WQ + 8 * KB, &tm_q, bar_tma, 0, h, (int)tok);
        tma_load_3d(sm + OFF_WQ + 24 * KB, &tm_q, bar_tma, 64, h, (int)tok);
        tma_load_3d(sm + OFF_KH, &tm_k, bar_tma, 0, h, (int)tok);
        tma_load_3d(sm + OFF_KH + 8 * KB, &tm_k, bar_tma, 64, h, (int)tok);
    };
    auto issue_vg = [&](long long tok) {
        tma_load_3d(sm + OFF_V, &tm_v, bar_tma, 0, h, (int)tok);
        tma_load_3d(sm + OFF_V + 8 * KB, &tm_v, bar_tma, 64, h, (int)tok);
        tma_load_3d(sm + OFF_G, &tm_g, bar_tma, 0, h, (int)tok);
    };
    // wait for an MMA commit; every thread takes part
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar_mma, mma_phase, kWaitCycles);
        mma_phase ^= 1u;
        tc_fence_after();
        return __syncthreads_or(!ok) == 0;
    };

    if (nchunks > 0 && tid == 0) {
        mbar_arrive_expect_tx(bar_tma, TMA_BYTES);
        issue_vg(t_begin);
        issue_qk(t_begin);
    }
    bool tma_pending = nchunks > 0;

    // thread roles for the token-parallel passes: subtile i, channel pair cp
    const int ti = tid >> 6;          // subtile 0..3
    const int cp = tid & 63;          // channel pair
    const int c0 = 2 * cp;            // first channel
    const int cblk = c0 >> 6;         // 64-wide block of the channel
    const int cin = c0 & 63;          // channel inside the block
    float gl[SUB][2];                 // in-subtile inclusive cumulative log-decay

    for (long long ch = 0; ch < nchunks; ++ch) {
        const long long tok0 = t_begin + ch * C;
        const int Lc = (int)((len - ch * C) < C ? (len - ch * C) : C);

        // ---- wait for this chunk's tiles
        {
            const bool ok = mbar_wait_bounded(bar_tma, tma_phase, kWaitCycles);
            tma_phase ^= 1u;
            tma_pending = false;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        if (tid < C) sBeta[tid] = (tid < Lc) ? __bfloat162float(beta[(size_t)(tok0 + tid) * H + h]) : 0.f;
        if (Lc < C) {  // zero the rows past the end of the sequence
            for (int idx = tid; idx < (C - Lc) * 16; idx += NT) {
                const int r = Lc + idx / 16, q16 = idx % 16;  // 16-byte piece of a 256-byte row
                const uint4 z = make_uint4(0, 0, 0, 0);
                const int blk = q16 >> 3, pc = (q16 & 7) * 8;
                *reinterpret_cast<uint4 *>(sm + OFF_WQ + blk * 16 * KB + sw128_offset(64 + r, pc)) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_KH + blk * 8 * KB + sw128_offset(r, pc)) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_V + blk * 8 * KB + sw128_offset(r, pc)) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_G + r * 256 + q16 * 16) = z;
            }
        }
        __syncthreads();

        // ---- phase 1a: cumulative log-decay inside subtile ti for channels c0, c0+1
        {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int rr = 0; rr < SUB; ++rr) {
                const float2 gv = ld_bf2(sm + OFF_G + (SUB * ti + rr) * 256 + c0 * 2);
                a0 += gv.x;
                a1 += gv.y;
                gl[rr][0] = a0;
                gl[rr][1] = a1;
            }
            sD[ti * D + c0] = a0;
            sD[ti * D + c0 + 1] = a1;
        }
        __syncthreads();

        // ---- phase 1b: Gram operands and Gamma * q
        float Dm[NSUB][2], ed[NSUB][2];
#pragma unroll
        for (int m = 0; m < NSUB; ++m)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                Dm[m][e] = sD[m * D + c0 + e];
                ed[m][e] = __expf(Dm[m][e]);
            }
        float pg[2];  // exp(G at the start of subtile ti) relative to the chunk start
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float acc = 1.f;
#pragma unroll
            for (int m = 0; m < NSUB; ++m)
                if (m < ti) acc *= ed[m][e];
            pg[e] = acc;
        }
        if (ti == 0) {
#pragma unroll
            for (int e = 0; e < 2; ++e) sGamC[c0 + e] = ed[0][e] * ed[1][e] * ed[2][e] * ed[3][e];
        }
        {
            float E[NSUB][2];  // E[j] = exp(G_start(ti) - G_end(j)) for j < ti, exp(-D_ti) for j = ti
#pragma unroll
            for (int j = 0; j < NSUB; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float acc = 1.f;
#pragma unroll
                    for (int m = 0; m < NSUB; ++m)
                        if (m > j && m < ti) acc *= ed[m][e];
                    E[j][e] = (j == ti) ? __expf(-Dm[ti][e]) : acc;
                }
#pragma unroll 4
            for (int rr = 0; rr < SUB; ++rr) {
                const int r = SUB * ti + rr;
                const uint32_t qoff = OFF_WQ + cblk * 16 * KB + sw128_offset(64 + r, cin);
                const uint32_t koff = OFF_KH + cblk * 8 * KB + sw128_offset(r, cin);
                const float2 kx = ld_bf2(sm + koff);
                const float2 qx = ld_bf2(sm + qoff);
                const float F0 = __expf(gl[rr][0]), F1 = __expf(gl[rr][1]);
                const float R0 = __expf(Dm[ti][0] - gl[rr][0]), R1 = __expf(Dm[ti][1] - gl[rr][1]);
                // right operand row r (column block ti)
                st_bf2(sm + OFF_R + cblk * 8 * KB + sw128_offset(r, cin), kx.x * R0, kx.y * R1);
                const float kf0 = kx.x * F0, kf1 = kx.y * F1, qf0 = qx.x * F0, qf1 = qx.y * F1;
#pragma unroll
                for (int j = 0; j < NSUB; ++j) {
                    if (j > ti) continue;
                    const uint32_t rows = l_rows(j), half_rows = rows / 2;
                    uint8_t *Lb = sm + OFF_L + l_off(j) + cblk * rows * 128;
                    st_bf2(Lb + sw128_offset(r - 16 * j, cin), kf0 * E[j][0], kf1 * E[j][1]);
                    st_bf2(Lb + sw128_offset(half_rows + r - 16 * j, cin), qf0 * E[j][0], qf1 * E[j][1]);
                }
                // Gamma * q in place (rows 64..127 of the [-W ; Qt] operand)
                st_bf2(sm + qoff, qf0 * pg[0], qf1 * pg[1]);
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
                mma_chain(tmem + TM_GRAM + 16u * j, A, B, 16, D / 16, false);
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
                        for (int s = 16 * (j + 1); s < C; s += 2) st_bf2(prow + sw128_offset(r, s), 0.f, 0.f);
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---- phase 3: T = (I + A)^{-1}, lower unit triangular, by 16 x 16 blocks
        if (tid < 64) {  // diagonal blocks: forward substitution, one column per thread
            const int bi = tid >> 4, cc = tid & 15, o0 = 16 * bi;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                float acc = (rr == cc) ? 1.f : 0.f;
                if (rr > cc) {
#pragma unroll
                    for (int ss = 0; ss < 16; ++ss)
                        if (ss >= cc && ss < rr) acc = fmaf(-AF[(o0 + rr) * 65 + o0 + ss], x[ss], acc);
                }
                x[rr] = acc;
                TF[(o0 + rr) * 65 + o0 + cc] = acc;
            }
        }
        __syncthreads();
        for (int dist = 1; dist < NSUB; ++dist) {
            const int nblk = NSUB - dist;
            // X = sum_{m=j}^{i-1} A_im T_mj  for blocks (i, j = i - dist)
            for (int idx = tid; idx < nblk * 256; idx += NT) {
                const int b = idx >> 8, rr = (idx >> 4) & 15, cc = idx & 15;
                const int bi = dist + b, bj = b;
                float acc = 0.f;
                for (int kk = 16 * bj + cc; kk < 16 * bi; ++kk)
                    acc = fmaf(AF[(16 * bi + rr) * 65 + kk], TF[kk * 65 + 16 * bj + cc], acc);
                XS[b * 272 + rr * 17 + cc] = acc;
            }
            __syncthreads();
            // T_ij = -T_ii X
            for (int idx = tid; idx < nblk * 256; idx += NT) {
                const int b = idx >> 8, rr = (idx >> 4) & 15, cc = idx & 15;
                const int bi = dist + b, bj = b;
                float acc = 0.f;
                for (int kk = 0; kk <= rr; ++kk)
                    acc = fmaf(TF[(16 * bi + rr) * 65 + 16 * bi + kk], XS[b * 272 + kk * 17 + cc], acc);
                TF[(16 * bi + rr) * 65 + 16 * bj + cc] = -acc;
            }
            __syncthreads();
        }
        // T Diag(beta) -> bf16 A operand (rows 0..63), zero rows 64..127
        for (int idx = tid; idx < 128 * 8; idx += NT) {
            const int r = idx >> 3, pc = (idx & 7) * 8;
            uint4 w = make_uint4(0, 0, 0, 0);
            if (r < C) {
                float t[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = pc + e;
                    t[e] = (s <= r) ? TF[r * 65 + s] * sBeta[s] : 0.f;
                }
                w.x = pack_bf2(t[0], t[1]);
                w.y = pack_bf2(t[2], t[3]);
                w.z = pack_bf2(t[4], t[5]);
                w.w = pack_bf2(t[6], t[7]);
            }
            *reinterpret_cast<uint4 *>(sm + OFF_TB + sw128_offset(r, pc)) = w;
        }
        // Gamma * k -> KT, and Kh = exp(G_C - G_s) * k_s in place of k
        {
            float sumD[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) sumD[e] = Dm[0][e] + Dm[1][e] + Dm[2][e] + Dm[3][e];
            float Gs[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < NSUB; ++m)
                    if (m < ti) acc += Dm[m][e];
                Gs[e] = acc;
            }
#pragma unroll 4
            for (int rr = 0; rr < SUB; ++rr) {
                const int r = SUB * ti + rr;
                const uint32_t koff = OFF_KH + cblk * 8 * KB + sw128_offset(r, cin);
                const float2 kx = ld_bf2(sm + koff);
                const float F0 = __expf(gl[rr][0]), F1 = __expf(gl[rr][1]);
                st_bf2(sm + OFF_KT + cblk * 8 * KB + sw128_offset(r, cin), kx.x * F0 * pg[0], kx.y * F1 * pg[1]);
                const float h0 = __expf(sumD[0] - Gs[0] - gl[rr][0]), h1 = __expf(sumD[1] - Gs[1] - gl[rr][1]);
                st_bf2(sm + koff, kx.x * h0, kx.y * h1);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- [W | Ut] = T Diag(beta) [Gamma*K | V]
        if (tid == 0) {
            tc_fence_after();
            Opnd A{sbase + OFF_TB, false, 16 * KB, 0};
            Opnd BK{sbase + OFF_KT, true, 0, 8 * KB};
            Opnd BV{sbase + OFF_V, true, 0, 8 * KB};
            mma_chain(tmem + TM_W, A, BK, 128, C / 16, false);
            mma_chain(tmem + TM_U, A, BV, 128, C / 16, false);
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }
        const bool more = ch + 1 < nchunks;
        if (more && tid == 0) {  // v, g tiles are free: start the next chunk's loads
            mbar_arrive_expect_tx(bar_tma, TMA_BYTES);
            issue_vg(tok0 + C);
        }
        tma_pending = more;

        // ---- phase 4: -W (rows 0..63) into the [-W ; Qt] operand
        if (quarter < 2) {
            float v[64];
            tmem_ld64(tmem + tlane + TM_W + 64u * half, v);
            tmem_wait_ld();
            const int r = 32 * quarter + lane;
            uint8_t *base = sm + OFF_WQ + half * 16 * KB;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint4 w;
                w.x = pack_bf2(-v[8 * cc + 0], -v[8 * cc + 1]);
                w.y = pack_bf2(-v[8 * cc + 2], -v[8 * cc + 3]);
                w.z = pack_bf2(-v[8 * cc + 4], -v[8 * cc + 5]);
                w.w = pack_bf2(-v[8 * cc + 6], -v[8 * cc + 7]);
                *reinterpret_cast<uint4 *>(base + sw128_offset(r, 8 * cc)) = w;
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
            mma_chain(tmem + TM_U, A, B, 128, D / 16, true);
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }

        // ---- phase 5: U (rows 0..63) -> bf16 B operand, MN-major [tok][dv]
        if (quarter < 2) {
            float v[64];
            tmem_ld64(tmem + tlane + TM_U + 64u * half, v);
            tmem_wait_ld();
            const int r = 32 * quarter + lane;
            uint8_t *base = sm + OFF_R + half * 8 * KB;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                uint4 w;
                w.x = pack_bf2(v[8 * cc + 0], v[8 * cc + 1]);
                w.y = pack_bf2(v[8 * cc + 2], v[8 * cc + 3]);
                w.z = pack_bf2(v[8 * cc + 4], v[8 * cc + 5]);
                w.w = pack_bf2(v[8 * cc + 6], v[8 * cc + 7]);
                *reinterpret_cast<uint4 *>(base + sw128_offset(r, 8 * cc)) = w;
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
            Opnd AK{sbase + OFF_KH, true, 0, 8 * KB};
            mma_chain(tmem + TM_U, AP, BU, 128, C / 16, true);
            mma_chain(tmem + TM_KU, AK, BU, 128, C / 16, false);
            mma_commit(bar_mma);
        }
        if (!wait_mma()) { aborted = true; break; }
        if (more && tid == 0) issue_qk(tok0 + C);

        // ---- phase 6: outputs and the state update
        if (quarter >= 2) {
            float v[64];
            tmem_ld64(tmem + tlane + TM_U + 64u * half, v);
            tmem_wait_ld();
            const int r = 32 * quarter + lane - 64;
            if (r < Lc) {
                uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)(tok0 + r) * H + h) * D + 64 * half);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    uint4 w;
                    w.x = pack_bf2(v[8 * cc + 0], v[8 * cc + 1]);
                    w.y = pack_bf2(v[8 * cc + 2], v[8 * cc + 3]);
                    w.z = pack_bf2(v[8 * cc + 4], v[8 * cc + 5]);
                    w.w = pack_bf2(v[8 * cc + 6], v[8 * cc + 7]);
                    dst[cc] = w;
                }
            }
        }
        {
            float v[64];
            tmem_ld64(tmem + tlane + TM_KU + 64u * half, v);
            tmem_wait_ld();
            const float gam = sGamC[si];
#pragma unroll
            for (int jj = 0; jj < 64; ++jj) S[jj] = fmaf(gam, S[jj], v[jj]);
            write_state_bf16();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    if (aborted) {
        if (tid == 0 && p.dev_status) atomicExch(p.dev_status, (int)KDA_ERR_TIMEOUT);
        if (tma_pending && tid == 0) mbar_wait_bounded(bar_tma, tma_phase, kWaitCycles);
    } else if (p.ST) {
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) {
            const int j = 64 * half + jj;
            p.ST[state_base + (size_t)j * D + si] = S[jj];
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
