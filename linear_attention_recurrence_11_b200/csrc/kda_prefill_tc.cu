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
//  2. CUDA cores: cumulative sums of g inside each 16-token subtile and the
//     scaled bf16 operands of the decayed Grams. Column block j (tokens
//     32j..32j+31) of
//        A_rs = beta_r sum_c k_rc k_sc e^{G_rc - G_sc},  P_rs = sum_c q_rc k_sc e^{G_rc - G_sc}
//     is the product of a left operand k_r e^{G_r - G_mid(j)} (stacked with
//     q_r e^{G_r - G_mid(j)}, rows r >= 32j) and a right operand
//     k_s e^{G_mid(j) - G_s}, referenced to the block's middle token
//     mid(j) = 32j + 16. The pages' g_min = -5 bound keeps every factor within
//     e^{+-80} (16 tokens x 5), which bf16 and fp32 hold; entries r < s of the
//     product may overflow, and the readout drops them by selection. A left
//     factor that underflows belongs to an entry below e^-12.
//  3. tcgen05.mma (M=128, N=32, K=128) x 2 -> TMEM; readout to A (fp32) and P (bf16).
//  4. CUDA cores: T = (I + A)^{-1} by 16 x 16 blocks (forward substitution on
//     the diagonal blocks, then block rows by distance).
//  5. tcgen05.mma: [W | Ut] = T Diag(beta) [Gamma*K | V]           (M=128 padded, K=64)
//  6. tcgen05.mma: [U ; Qt S] = [Ut ; 0] + [-W ; Gamma*Q] S          (M=128, K=128)
//  7. tcgen05.mma: O = Qt S + P U (rows 64..127),  S += Kh^T U      (K=64)
//     with Kh_s = e^{G_C - G_s} k_s, onto the fp32 state in TMEM that was
//     scaled by Diag(Gamma_C) while step 6 ran (the state never leaves the SM
//     between chunks; its bf16 copy feeds step 6 of the next chunk). The
//     outputs are staged in shared memory and written by TMA tensor stores.
// The next chunk's tiles are requested as soon as each staging tile has been
// consumed (g after step 2's cumulative sums, k after step 4, v after step 5,
// q after step 6), so their HBM latency overlaps the rest of the chunk.
// All matrices in shared memory use the 128-byte swizzled layout the TMA
// writes and the tcgen05 descriptors read. No cluster multicast is used.
#include "kda_internal.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_common.cuh"


namespace kda {
namespace {

using namespace sm100;
using namespace tc;

constexpr int NT = 256;

// ---------------------------------------------------------- smem layout
constexpr uint32_t KB = 1024;
constexpr uint32_t OFF_WQ = 0;          // 32 KB  [Gamma*K, then -W ; Gamma*Q], K-major, 128 rows x 128 (2 K-blocks); q lands in rows 64..127
constexpr uint32_t OFF_SB = 32 * KB;    // 32 KB  B operand S (bf16), MN-major [dk rows][dv] (2 N-blocks)
constexpr uint32_t OFF_KS = 64 * KB;    // 16 KB  k tile, [tok rows][dk] (2 blocks of 64 channels)
constexpr uint32_t OFF_V = 80 * KB;     // 16 KB  v: B operand MN-major [tok rows][dv] (2 N-blocks)
constexpr uint32_t OFF_G = 96 * KB;     // 16 KB  g, plain [64][128] bf16
constexpr uint32_t OFF_R = 112 * KB;    // 16 KB  Gram right operand, K-major [s rows][dk]; then scratch of the inverse
constexpr uint32_t OFF_PB = 128 * KB;   // 8 KB   rows 64..127 of the A operand [junk ; P], K-major, K = 64
constexpr uint32_t OFF_L = 136 * KB;    // 80 KB  Gram left operands L3, L2, L1 (compact), Kh, then the aliases below
constexpr uint32_t OFF_MISC = 216 * KB;
// L region: left operands of the two 32-token column blocks of the Gram, each referenced to
// the block's middle token: L0 = [k ; q] rows 0..63 (128 rows, K-blocks 16 KB apart), L1 =
// [k ; q] rows 32..63 (64 rows, K-blocks 8 KB apart). Read as 128-row operands, L1's second
// K-block ends 24 KB past L1 (the rows past its own land in accumulator lanes that are never
// read); Kh, written with the Gram operands and read by the last product of the chunk, starts
// there.
constexpr int kGramChains = 2;
constexpr uint32_t L0_OFF = 0, L1_OFF = 32 * KB;
// aliases inside the L region once the Gram MMAs are done
constexpr uint32_t OFF_TB = OFF_L + 0;             // 16 KB  A operand T Diag(beta), K-major, 128 rows x 64
// Gamma*K sits in rows 0..63 of the [-W ; Gamma*Q] tile until the W product is read out:
// the W product reads it as its B operand (MN-major).
constexpr uint32_t OFF_KT = OFF_WQ;
// (LDA, LDT, LDX: the row strides of the inverse's fp32 scratch, kda_tc_common.cuh)
constexpr uint32_t OFF_KHAT = OFF_L + 56 * KB;     // 16 KB  A operand Kh, MN-major [tok][dk]
constexpr uint32_t OFF_AF = OFF_L + 16 * KB;       // 64 x LDA fp32  A          (the Gram is done)
constexpr uint32_t OFF_UB = OFF_L + 0;             // 16 KB  B operand U, MN-major [tok][dv] (T Diag(beta) is done)
constexpr uint32_t OFF_TF = OFF_L + 33 * KB;       // 64 x LDT fp32  T
constexpr uint32_t OFF_XS = OFF_R;                 // 32 x LDX fp32 scratch (the Gram is done)
static_assert(OFF_L + L1_OFF + 8 * KB + 16 * KB <= OFF_KHAT, "Gram operand reads reach Kh");
static_assert(OFF_AF >= OFF_TB + 16 * KB && OFF_AF + 64 * LDA * 4 <= OFF_TF, "A overlaps T Diag(beta) or T");
static_assert(OFF_TF + 64 * LDT * 4 <= OFF_KHAT, "T overlaps Kh");
static_assert(OFF_KHAT + 16 * KB <= OFF_MISC, "Kh overflows the L region");
static_assert(32 * LDX * 4 <= 16 * KB, "scratch overflows the right-operand tile");
// misc
constexpr uint32_t OFF_BAR = OFF_MISC;              // 3 mbarriers
constexpr uint32_t OFF_TMEMADDR = OFF_MISC + 32;
constexpr uint32_t OFF_BETA = OFF_MISC + 64;        // 64 fp32
constexpr uint32_t OFF_DSUM = OFF_BETA + 256;       // 4 x 128 fp32 subtile totals of g (log2 units)
constexpr uint32_t OFF_GAMC = OFF_DSUM + 2048;      // 128 fp32 Gamma_C
constexpr uint32_t OFF_NORM = OFF_GAMC + 512;       // 2 x 64 x 2 fp32: per-row partial squared norms of k, q
constexpr uint32_t SMEM_USED = OFF_NORM + 1024;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns (512 allocated): the Gram accumulators use the first 64 columns
// of the W region (read out before the W product is issued).
constexpr uint32_t TM_GRAM = 0, TM_W = 0, TM_U = 128, TM_S = 384, TM_COLS = 512;
constexpr uint32_t TMA_BYTES = 6 * 8 * KB + 16 * KB;  // q, k, v: 2 boxes of 8 KB each; g: 1 box of 16 KB

struct TcParams {
    PrefillArgs a;
};

// kFused: the variant with the fused pre-operations (KDA_FUSE_* in p.fuse); the plain
// variant carries none of their code, so its schedule is not disturbed.
template <bool kFused>
__global__ void __launch_bounds__(NT, 1)
kda_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                      const __grid_constant__ CUtensorMap tm_o, const TcParams prm) {
    const PrefillArgs &p = prm.a;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment of the shared-window address (the swizzle patterns key on it)
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint64_t *bar_gram = bar_tma + 2;  // 2 arrivals: one commit per Gram column block
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + OFF_TMEMADDR);
    float *sBeta = reinterpret_cast<float *>(sm + OFF_BETA);
    float *sD = reinterpret_cast<float *>(sm + OFF_DSUM);
    float *sGamC = reinterpret_cast<float *>(sm + OFF_GAMC);
    float *sNorm = reinterpret_cast<float *>(sm + OFF_NORM);
    const bool fuse_gate = kFused && (p.fuse & KDA_FUSE_GATE_LOGITS) != 0;
    const bool fuse_norm = kFused && (p.fuse & KDA_FUSE_NORM_QK) != 0;
    float *AF = reinterpret_cast<float *>(sm + OFF_AF);
    float *TF = reinterpret_cast<float *>(sm + OFF_TF);
    float *XS = reinterpret_cast<float *>(sm + OFF_XS);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
    const int h = blockIdx.x % p.H;
    const int n = unit_seq(p, blockIdx.x / p.H);
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
        mbar_init(bar_gram, kGramChains);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_g);
        tma_prefetch_desc(&tm_o);
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
        if (!p.v) return;  // all-zero values: the V tile is zeroed once below
        tma_load_3d(sm + OFF_V, &tm_v, bar_tma, 0, h, (int)tok);
        tma_load_3d(sm + OFF_V + 8 * KB, &tm_v, bar_tma, 64, h, (int)tok);
    };
    const uint32_t tma_bytes = p.v ? TMA_BYTES : TMA_BYTES - 16 * KB;
    auto issue_g = [&](long long tok) { tma_load_3d(sm + OFF_G, &tm_g, bar_tma, 0, h, (int)tok); };
    if (nchunks > 0 && tid == 0) {
        mbar_arrive_expect_tx(bar_tma, tma_bytes);
        issue_g(t_begin);
        issue_k(t_begin);
        issue_v(t_begin);
        issue_q(t_begin);
    }
    // beta of this thread's row in the next chunk, prefetched as raw bf16 (converted when used)
    __nv_bfloat16 bnext = __float2bfloat16(0.f);
    if (tid < C && tid < len) bnext = beta[(size_t)(t_begin + tid) * H + h];

    if (!p.v) {  // all-zero values (the segment-pair pass): zero the V tile once
        for (int idx = tid; idx < 16 * KB / 16; idx += NT)
            *reinterpret_cast<uint4 *>(sm + OFF_V + 16 * idx) = make_uint4(0, 0, 0, 0);
    }
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

    uint32_t tma_phase = 0, mma_phase = 0, gram_phase = 0;
    // Unwinding state (meaningful in thread 0, which issues every copy and MMA):
    // tma_armed: the transaction count of phase tma_phase is armed and not yet consumed;
    // tma_issued: which of the next tiles (1 g, 2 k, 4 v, 8 q) have been requested for it;
    // mma_bar / mma_bar_phase: a commit that was waited for without success.
    bool aborted = false, tma_armed = nchunks > 0;
    uint32_t tma_issued = nchunks > 0 ? 15u : 0u;
    long long tma_tok = t_begin;
    uint64_t *mma_bar = nullptr;
    uint32_t mma_bar_phase = 0;
    // wait for an MMA commit in every thread; the barrier after the readout that follows both
    // publishes it and agrees on a wait that ran out
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar_mma, mma_phase, kWaitCycles);
        if (!ok) { mma_bar = bar_mma; mma_bar_phase = mma_phase; }
        mma_phase ^= 1u;
        tc_fence_after();
        return ok;
    };

    // thread roles for the token-parallel passes: subtile ti (a pair of warps), half hh of
    // the subtile (rows 8hh..8hh+7), and a quad of channels (4 consecutive channels, 8 bytes)
    // subtile of each warp pair; warps w and w + 4 share a scheduler, and subtiles 0, 1
    // write one Gram left-operand row pair per token, subtiles 2, 3 two, so each scheduler
    // gets one of each
    const int ti = warp >> 1;  // warps 0..7 -> 0,0,1,1,2,2,3,3
    const int hh = lane >> 4;                     // which 8 rows of the subtile
    const int cq = (warp & 1) * 16 + (lane & 15); // channel quad 0..31 (the two warps of a pair)
    const int c0 = 4 * cq;                        // first channel
    const int cblk = c0 >> 6;                     // 64-wide block of the channel
    const int cin = c0 & 63;                      // channel inside the block
    constexpr int HR = SUB / 2;                   // rows per thread
    constexpr uint32_t idG = idesc_bf16_f32(128, 32, 0, 0);     // Gram: K-major x K-major, N = 32
    constexpr uint32_t idKM = idesc_bf16_f32(128, 128, 0, 1);   // K-major A, MN-major B, N = 128
    constexpr uint32_t idMM = idesc_bf16_f32(128, 128, 1, 1);   // MN-major A and B, N = 128

    for (long long ch = 0; ch < nchunks; ++ch) {
        const long long tok0 = t_begin + ch * C;
        const int Lc = (int)((len - ch * C) < C ? (len - ch * C) : C);
        const bool more = ch + 1 < nchunks;
        const long long tokn = tok0 + C;

        // ---- wait for this chunk's tiles (every thread; the barrier after the decay pass agrees
        // on a wait that ran out, and on failure the phase stays the one to drain on the way out)
        const bool ok_tile = mbar_wait_bounded(bar_tma, tma_phase, kWaitCycles);
        if (ok_tile) {
            tma_phase ^= 1u;
            tma_armed = false;
        }
        if (tid < C) {
            sBeta[tid] = (tid < Lc) ? __bfloat162float(bnext) : 0.f;
            if (more && tid < len - (ch + 1) * C) bnext = beta[(size_t)(tokn + tid) * H + h];
        }
        if (Lc < C) {  // zero the q, k, v rows past the end of the sequence (read after the next barrier)
            for (int idx = tid; idx < (C - Lc) * 16; idx += NT) {
                const int r = Lc + idx / 16, q16 = idx % 16;  // 16-byte piece of a 256-byte row
                const uint4 z = make_uint4(0, 0, 0, 0);
                const int blk = q16 >> 3, pc = (q16 & 7) * 8;
                *reinterpret_cast<uint4 *>(sm + OFF_WQ + blk * 16 * KB + sw128_offset(64 + r, pc)) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_KS + blk * 8 * KB + sw128_offset(r, pc)) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_V + blk * 8 * KB + sw128_offset(r, pc)) = z;
            }
        }

        // ---- phase 1a: cumulative log2-decay inside subtile ti for channels c0..c0+3
        float gl[HR][4];
        {
            float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int rr = 0; rr < HR; ++rr) {
                const int row = SUB * ti + HR * hh + rr;  // rows past the end of the sequence decay by 1
                const uint2 raw = row < Lc ? *reinterpret_cast<const uint2 *>(sm + OFF_G + row * 256 + c0 * 2) : make_uint2(0, 0);
                float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
                float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
                if (fuse_gate && row < Lc) {  // g holds gate logits
                    g01 = make_float2(gate_from_logit(g01.x), gate_from_logit(g01.y));
                    g23 = make_float2(gate_from_logit(g23.x), gate_from_logit(g23.y));
                }
                a[0] = fmaf(g01.x, kLog2e, a[0]);
                a[1] = fmaf(g01.y, kLog2e, a[1]);
                a[2] = fmaf(g23.x, kLog2e, a[2]);
                a[3] = fmaf(g23.y, kLog2e, a[3]);
#pragma unroll
                for (int e = 0; e < 4; ++e) gl[rr][e] = a[e];
            }
            // the upper half adds the lower half's total (lane - 16 holds the same channels)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __shfl_sync(0xffffffffu, a[e], lane & 15);
                if (hh) {
#pragma unroll
                    for (int rr = 0; rr < HR; ++rr) gl[rr][e] += lo;
                }
            }
            if (hh) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sD[ti * D + c0 + e] = gl[HR - 1][e];
            }
        }
        if (fuse_norm) {
            // squared norms of this thread's k and q rows over its 4 channels, summed over the
            // 16 lanes of the half-warp (64 channels); the partner warp holds the other 64
            const uint8_t *krow = sm + OFF_KS + cblk * 8 * KB;
            const uint8_t *qrow = sm + OFF_WQ + cblk * 16 * KB;
#pragma unroll
            for (int rr = 0; rr < HR; ++rr) {
                const int r = SUB * ti + HR * hh + rr;
                const uint2 kr = *reinterpret_cast<const uint2 *>(krow + sw128_offset(r, cin));
                const uint2 qr = *reinterpret_cast<const uint2 *>(qrow + sw128_offset(64 + r, cin));
                const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kr.x));
                const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kr.y));
                const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qr.x));
                const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qr.y));
                // rows past the end are being zeroed in this same phase: count them as zero
                float sk = r < Lc ? k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y : 0.f;
                float sq = r < Lc ? q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y : 0.f;
#pragma unroll
                for (int off = 1; off < 16; off <<= 1) {
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                }
                if ((lane & 15) == rr) {
                    sNorm[(0 * C + r) * 2 + (warp & 1)] = sk;
                    sNorm[(1 * C + r) * 2 + (warp & 1)] = sq;
                }
            }
        }
        if (tid == 0) bulk_wait_read_all();  // the previous chunk's staged outputs have been read
        if (__syncthreads_or(!ok_tile)) { aborted = true; break; }
        if (more && tid == 0) {  // g tile consumed: start the next chunk's loads
            mbar_arrive_expect_tx(bar_tma, tma_bytes);
            issue_g(tokn);
            tma_armed = true;
            tma_tok = tokn;
            tma_issued = 1u;
        }

        // ---- phase 1b: Gram operands, Gamma * q and Gamma * k; keep the factors for Kh
        float F[HR][4], Fi[HR][4];
        float pg[4], post[4];
        {
            float Dm[NSUB][4], ed[NSUB][4];
#pragma unroll
            for (int m = 0; m < NSUB; ++m) {
                const float4 d4 = *reinterpret_cast<const float4 *>(sD + m * D + c0);
                Dm[m][0] = d4.x; Dm[m][1] = d4.y; Dm[m][2] = d4.z; Dm[m][3] = d4.w;
#pragma unroll
                for (int e = 0; e < 4; ++e) ed[m][e] = ex2(Dm[m][e]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float a = 1.f, b = 1.f;
#pragma unroll
                for (int m = 0; m < NSUB; ++m) {
                    if (m < ti) a *= ed[m][e];
                    if (m >= ti) b *= ed[m][e];
                }
                pg[e] = a;     // Gamma at the start of subtile ti (relative to the chunk start)
                post[e] = b;   // decay from the start of subtile ti to the end of the chunk
            }
            if (ti == 0 && hh == 0) {
                *reinterpret_cast<float4 *>(sGamC + c0) =
                    make_float4(ed[0][0] * ed[1][0] * ed[2][0] * ed[3][0], ed[0][1] * ed[1][1] * ed[2][1] * ed[3][1],
                                ed[0][2] * ed[1][2] * ed[2][2] * ed[3][2], ed[0][3] * ed[1][3] * ed[2][3] * ed[3][3]);
            }
            // column block b (tokens 32b..32b+31) is referenced to its middle token 32b + 16:
            // its left operand rows are x_r e^{G_r - G_mid(b)} (r >= 32b), its right operand
            // rows k_s e^{G_mid(b) - G_s}; every factor lies in [e^-80, e^80] within a block.
            // Here as multiples of this subtile's own factors (relative to its start):
            //   el0 = e^{G_start(ti) - G_16}, el1 = e^{G_start(ti) - G_48} (ti >= 2),
            //   er  = e^{G_mid(block of ti) - G_start(ti)}
            float el0[4], el1[4], er[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                el0[e] = ti == 0 ? ex2(-Dm[0][e]) : ti == 1 ? 1.f : ti == 2 ? ed[1][e] : ed[1][e] * ed[2][e];
                el1[e] = ti == 2 ? ex2(-Dm[2][e]) : 1.f;
                er[e] = ti == 0 ? ed[0][e] : ti == 2 ? ed[2][e] : 1.f;
            }
#pragma unroll
            for (int rr = 0; rr < HR; ++rr)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    F[rr][e] = ex2(gl[rr][e]);    // e^{G_r - G_start(ti)}, in [e^-80, 1]
                    Fi[rr][e] = ex2(-gl[rr][e]);  // e^{G_start(ti) - G_r}, in [1, e^80]
                }
            uint8_t *const qrow = sm + OFF_WQ + cblk * 16 * KB;
            uint8_t *const krow = sm + OFF_KS + cblk * 8 * KB;
            uint8_t *const rrow = sm + OFF_R + cblk * 8 * KB;
            uint8_t *const khrow = sm + OFF_KHAT + cblk * 8 * KB;
            auto st4 = [](uint8_t *p, float a, float b, float c, float d) {
                *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf2(a, b), pack_bf2(c, d));
            };
            auto ld4 = [](const uint8_t *p, float (&v)[4]) {
                const uint2 raw = *reinterpret_cast<const uint2 *>(p);
                const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
                const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
                v[0] = x.x; v[1] = x.y; v[2] = y.x; v[3] = y.y;
            };
#pragma unroll
            for (int rr = 0; rr < HR; ++rr) {
                const int r = SUB * ti + HR * hh + rr;
                const uint32_t off_r = sw128_offset(r, cin);       // (r & 7) == rr
                const uint32_t off_q = sw128_offset(64 + r, cin);
                float kx[4], qx[4], kf[4], qf[4];
                ld4(krow + off_r, kx);
                ld4(qrow + off_q, qx);
                if (fuse_norm) {  // k and q normalised per row (rows past the end stay zero)
                    const float nk = sNorm[(0 * C + r) * 2] + sNorm[(0 * C + r) * 2 + 1];
                    const float nq = sNorm[(1 * C + r) * 2] + sNorm[(1 * C + r) * 2 + 1];
                    const float ik = nk > 0.f ? rsqrtf(nk) : 0.f, iq = nq > 0.f ? rsqrtf(nq) : 0.f;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        kx[e] *= ik;
                        qx[e] *= iq;
                    }
                }
                // right operand row r: k_r e^{G_mid - G_r}; and Kh row r:
                // k_r e^{G_C - G_r} = (k_r e^{G_start(ti) - G_r}) e^{G_C - G_start(ti)}, both factors bounded
                float kr[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) kr[e] = kx[e] * Fi[rr][e];
                st4(rrow + off_r, kr[0] * er[0], kr[1] * er[1], kr[2] * er[2], kr[3] * er[3]);
                st4(khrow + off_r, kr[0] * post[0], kr[1] * post[1], kr[2] * post[2], kr[3] * post[3]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    kf[e] = kx[e] * F[rr][e];
                    qf[e] = qx[e] * F[rr][e];
                }
                {  // left operands: block 0 (every row), block 1 (rows >= 32)
                    uint8_t *L0 = sm + OFF_L + L0_OFF + cblk * 16 * KB;
                    st4(L0 + off_r, kf[0] * el0[0], kf[1] * el0[1], kf[2] * el0[2], kf[3] * el0[3]);
                    st4(L0 + off_q, qf[0] * el0[0], qf[1] * el0[1], qf[2] * el0[2], qf[3] * el0[3]);
                    if (ti >= 2) {
                        uint8_t *L1 = sm + OFF_L + L1_OFF + cblk * 8 * KB;
                        st4(L1 + sw128_offset(r - 32, cin), kf[0] * el1[0], kf[1] * el1[1], kf[2] * el1[2],
                            kf[3] * el1[3]);
                        st4(L1 + sw128_offset(r, cin), qf[0] * el1[0], qf[1] * el1[1], qf[2] * el1[2],
                            qf[3] * el1[3]);
                    }
                }
                st4(qrow + off_q, qf[0] * pg[0], qf[1] * pg[1], qf[2] * pg[2], qf[3] * pg[3]);  // Gamma * q
                st4(qrow + off_r, kf[0] * pg[0], kf[1] * pg[1], kf[2] * pg[2], kf[3] * pg[3]);  // Gamma * k, row r
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- Gram MMAs: column block j -> TMEM columns 32j..32j+31, issued by lane 0 of warp j
        if (lane == 0 && warp < kGramChains) {
            const int j = warp;
            tc_fence_after();
            Opnd A = (j == 0) ? Opnd{sbase + OFF_L + L0_OFF, false, 16 * KB, 0}
                              : Opnd{sbase + OFF_L + L1_OFF, false, 8 * KB, 0};
            Opnd B{sbase + OFF_R + 32u * j * 128u, false, 8 * KB, 0};
            mma_chain<D / 16>(tmem + TM_GRAM + 32u * j, A, B, idG, false);
            mma_commit(bar_gram);
        }
        if (more && tid == 0) {  // the k tile is consumed (Kh is written with the Gram operands)
            issue_k(tokn);
            tma_issued |= 2u;
        }
        const bool ok_gram = mbar_wait_bounded(bar_gram, gram_phase, kWaitCycles);
        if (!ok_gram) { mma_bar = bar_gram; mma_bar_phase = gram_phase; }
        gram_phase ^= 1u;
        tc_fence_after();

        // ---- phase 2: Gram readout -> A (fp32, strictly lower, times beta_r), P (bf16, lower).
        // Warps of column half j read block j's 32 columns; the masks select (never multiply)
        // so that the upper-triangle entries, which may overflow, are dropped.
        if (ok_gram) {
            float v2[2][16];
            tmem_ld16(tmem + tlane + TM_GRAM + 32u * half, v2[0]);
            tmem_ld16(tmem + tlane + TM_GRAM + 32u * half + 16u, v2[1]);
            tmem_wait_ld();
            const int j = half;
            const int m = 32 * quarter + lane;
            const int kr = 64 - 32 * j;  // k rows of block j's left operand (rows >= 32j)
            if (m < kr) {
                const int r = 32 * j + m;
                const float b = sBeta[r];
                float4 *arow = reinterpret_cast<float4 *>(AF + r * LDA + 32 * j);
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {
                    const float *v = v2[q4 >> 2] + 4 * (q4 & 3);
                    const int s = 32 * j + 4 * q4;
                    arow[q4] = make_float4((s < r) ? b * v[0] : 0.f, (s + 1 < r) ? b * v[1] : 0.f,
                                           (s + 2 < r) ? b * v[2] : 0.f, (s + 3 < r) ? b * v[3] : 0.f);
                }
            } else if (m < 2 * kr) {
                const int r = 32 * j + (m - kr);
                uint8_t *prow = sm + OFF_PB;
#pragma unroll
                for (int s2 = 0; s2 < 32; s2 += 2) {
                    const int s = 32 * j + s2;
                    const float *v = v2[s2 >> 4] + (s2 & 15);
                    st_bf2(prow + sw128_offset(r, s), (s <= r) ? v[0] : 0.f, (s + 1 <= r) ? v[1] : 0.f);
                }
                if (j == 0 && r < 32) {  // diagonal block of block 0: zero block 1's columns
                    for (int s = 32; s < C; s += 8)
                        *reinterpret_cast<uint4 *>(prow + sw128_offset(r, s)) = make_uint4(0, 0, 0, 0);
                }
            }
            // T Diag(beta) (bf16, 128 rows) starts as zeros: the inverse writes its lower blocks,
            // and rows 64..127 stay zero, the [Ut ; 0] the state product accumulates onto (the
            // Gram products that read this tile are done)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<uint4 *>(sm + OFF_TB + 16 * (tid + NT * i)) = make_uint4(0, 0, 0, 0);
        }
        tc_fence_before();
        if (__syncthreads_or(!ok_gram)) { aborted = true; break; }

        // ---- phase 3: T = (I + A)^{-1} (unit lower triangular) by 16 x 16 blocks
        if (warp < NSUB && lane < 16) {
            // diagonal block `warp`: forward substitution by rows (left-looking), one column of
            // T_ii per lane; each row of A_ii is one broadcast read shared by the 16 lanes
            const int o0 = 16 * warp, cc = lane;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                float a[16];
                const float4 *arow = reinterpret_cast<const float4 *>(AF + (o0 + rr) * LDA + o0);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    if (4 * q4 < rr) {
                        const float4 t = arow[q4];
                        a[4 * q4] = t.x; a[4 * q4 + 1] = t.y; a[4 * q4 + 2] = t.z; a[4 * q4 + 3] = t.w;
                    }
                }
                // x[rr] = [rr == cc] - sum_{ss < rr} A[rr][ss] x[ss], four partial sums
                float acc[4] = {(rr == cc) ? 1.f : 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ss = 0; ss < rr; ++ss) acc[ss & 3] = fmaf(-a[ss], x[ss], acc[ss & 3]);
                x[rr] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            }
            // T_ii, and its column times beta into T Diag(beta) (x is 0 above the diagonal)
            const float bcol = sBeta[o0 + cc];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                TF[(o0 + rr) * LDT + o0 + cc] = x[rr];
                *reinterpret_cast<__nv_bfloat16 *>(sm + OFF_TB + sw128_offset(o0 + rr, o0 + cc)) =
                    __float2bfloat16_rn(x[rr] * bcol);
            }
            if ((warp & 1) == 0) {  // the 16 x 16 block right of it, inside its 32 x 32 diagonal block
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) TF[(o0 + rr) * LDT + o0 + 16 + cc] = 0.f;
            }
        }
        __syncthreads();
        // the off-diagonal blocks of T, each also written times beta into T Diag(beta): the bf16
        // A operand of [W | Ut]
        tri_inverse_offdiag(AF, TF, XS, tid, 0, sm + OFF_TB, sBeta);
        fence_proxy_async_smem();
        __syncthreads();

        // ---- [W | Ut] = T Diag(beta) [Gamma*K | V]
        if (tid == 0) {
            tc_fence_after();
            Opnd A{sbase + OFF_TB, false, 16 * KB, 0};
            Opnd BK{sbase + OFF_KT, true, 0, 16 * KB};
            Opnd BV{sbase + OFF_V, true, 0, 8 * KB};
            mma_chain<C / 16>(tmem + TM_W, A, BK, idKM, false);
            mma_chain<C / 16>(tmem + TM_U, A, BV, idKM, false);
            mma_commit(bar_mma);
        }
        const bool ok_wu = wait_mma();
        if (ok_wu && more && tid == 0) {
            issue_v(tokn);
            tma_issued |= 4u;
        }

        // ---- phase 4: -W (rows 0..63) into the [-W ; Qt] operand
        if (ok_wu && quarter < 2) {
            const int r = 32 * quarter + lane;
            uint8_t *base = sm + OFF_WQ + half * 16 * KB;
            float v[4][16];
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + TM_W + 64u * half + 16u * gq, v[gq]);
            tmem_wait_ld();
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                uint4 w0, w1;
                pack16(v[gq], -1.f, w0, w1);
                *reinterpret_cast<uint4 *>(base + sw128_offset(r, 16 * gq)) = w0;
                *reinterpret_cast<uint4 *>(base + sw128_offset(r, 16 * gq + 8)) = w1;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok_wu)) { aborted = true; break; }

        // ---- [U ; Qt S] = [Ut ; 0] + [-W ; Qt] S
        if (tid == 0) {
            tc_fence_after();
            Opnd A{sbase + OFF_WQ, false, 16 * KB, 0};
            Opnd B{sbase + OFF_SB, true, 0, 16 * KB};
            mma_chain<D / 16>(tmem + TM_U, A, B, idKM, true);
            mma_commit(bar_mma);
        }
        // while it runs: S <- Diag(Gamma_C) S in TMEM, so that the dS product below can
        // accumulate onto the state directly
        {
            const float gam = sGamC[si];
            float sv[4][16];
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + TM_S + 64u * half + 16u * gq, sv[gq]);
            tmem_wait_ld();
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
#pragma unroll
                for (int e = 0; e < 16; ++e) sv[gq][e] *= gam;
                tmem_st16(tmem + tlane + TM_S + 64u * half + 16u * gq, sv[gq]);
            }
            tmem_wait_st();
            tc_fence_before();
        }
        const bool ok_u = wait_mma();
        if (ok_u && more && tid == 0) {  // rows 64..127 of the [-W ; Qt] operand are free
            issue_q(tokn);
            tma_issued |= 8u;
        }

        // ---- phase 5: U (rows 0..63) -> bf16 B operand, MN-major [tok][dv]
        if (ok_u && quarter < 2) {
            const int r = 32 * quarter + lane;
            uint8_t *base = sm + OFF_UB + half * 8 * KB;
            float v[4][16];
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + TM_U + 64u * half + 16u * gq, v[gq]);
            tmem_wait_ld();
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                uint4 w0, w1;
                pack16(v[gq], 1.f, w0, w1);
                *reinterpret_cast<uint4 *>(base + sw128_offset(r, 16 * gq)) = w0;
                *reinterpret_cast<uint4 *>(base + sw128_offset(r, 16 * gq + 8)) = w1;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok_u)) { aborted = true; break; }

        // ---- O = Qt S + P U (rows 64..127 of the same accumulator), S += dS = Kh^T U
        if (tid == 0) {
            tc_fence_after();
            Opnd AP{sbase + OFF_PB - 8 * KB, false, 16 * KB, 0};
            Opnd BU{sbase + OFF_UB, true, 0, 8 * KB};
            Opnd AK{sbase + OFF_KHAT, true, 0, 8 * KB};
            mma_chain<C / 16>(tmem + TM_S, AK, BU, idMM, true);
            mma_chain<C / 16>(tmem + TM_U, AP, BU, idKM, true);
            mma_commit(bar_mma);
        }
        const bool ok_o = wait_mma();

        // ---- phase 6: outputs, and the bf16 copy of the updated state. A full chunk of
        // outputs is staged in the U tile (free now, and already in the 128-byte swizzled
        // [token][dv] layout a tensor store reads) and written by two TMA stores; the
        // rows of a partial chunk are stored directly, so nothing lands past the sequence.
        if (ok_o && quarter >= 2 && p.o) {
            const int r = 32 * quarter + lane - 64;
            float v[4][16];
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + TM_U + 64u * half + 16u * gq, v[gq]);
            tmem_wait_ld();
            if (Lc == C) {
                uint8_t *base = sm + OFF_UB + half * 8 * KB;
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) {
                    uint4 w0, w1;
                    pack16(v[gq], 1.f, w0, w1);
                    *reinterpret_cast<uint4 *>(base + sw128_offset(r, 16 * gq)) = w0;
                    *reinterpret_cast<uint4 *>(base + sw128_offset(r, 16 * gq + 8)) = w1;
                }
            } else if (r < Lc) {
                uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)(tok0 + r) * H + h) * D + 64 * half);
#pragma unroll
                for (int gq = 0; gq < 4; ++gq) {
                    uint4 w0, w1;
                    pack16(v[gq], 1.f, w0, w1);
                    dst[2 * gq] = w0;
                    dst[2 * gq + 1] = w1;
                }
            }
        }
        if (ok_o) {
            uint8_t *sb = sm + OFF_SB + half * 16 * KB;
            float sv[4][16];
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + TM_S + 64u * half + 16u * gq, sv[gq]);
            tmem_wait_ld();
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                uint4 w0, w1;
                pack16(sv[gq], 1.f, w0, w1);
                *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq)) = w0;
                *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq + 8)) = w1;
            }
            // a snapshot of the state after this chunk (fp32, the S0 layout of one sequence)
            const long long done = (ch + 1) * C;
            if (p.snap_every && Lc == C && done % p.snap_every == 0) {
                const long long nsnap = p.T / p.snap_every;
                float *dst = p.S_snap + (((size_t)n * nsnap + (size_t)(done / p.snap_every - 1)) * H + h) * (size_t)(D * D);
#pragma unroll
                for (int gq = 0; gq < 4; ++gq)
#pragma unroll
                    for (int e = 0; e < 16; ++e) dst[(size_t)(64 * half + 16 * gq + e) * D + si] = sv[gq][e];
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok_o)) { aborted = true; break; }
        if (Lc == C && tid == 0 && p.o) {
            tma_store_3d(&tm_o, sm + OFF_UB, 0, h, (int)tok0);
            tma_store_3d(&tm_o, sm + OFF_UB + 8 * KB, 64, h, (int)tok0);
            bulk_commit();
        }
    }
    if (tid == 0) bulk_wait_all();  // the output stores are complete before the CTA exits

    if (aborted) {
        // Unwind without leaving work in flight: complete the armed transaction count by
        // requesting the tiles not yet requested and wait (bounded) for the copies, then
        // wait (bounded) for a commit that timed out, before TMEM is freed below.
        if (tid == 0) {
            if (p.dev_status) atomicExch(p.dev_status, (int)KDA_ERR_TIMEOUT);
            if (tma_armed) {
                if (!(tma_issued & 1u)) issue_g(tma_tok);
                if (!(tma_issued & 2u)) issue_k(tma_tok);
                if (!(tma_issued & 4u)) issue_v(tma_tok);
                if (!(tma_issued & 8u)) issue_q(tma_tok);
                mbar_wait_bounded(bar_tma, tma_phase, kWaitCycles);
            }
            if (mma_bar) mbar_wait_bounded(mma_bar, mma_bar_phase, kWaitCycles);
        }
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

}  // namespace

bool prefill_tc_supported(int dk, int dv, int chunk, int dtype) {
    return dk == D && dv == D && chunk == C && dtype == KDA_DTYPE_BF16;
}

size_t prefill_tc_workspace(const PrefillArgs &a) { return a.cu_seqlens ? seq_order_bytes(a.num_units) : 0; }

int prefill_tc_launches(const PrefillArgs &a) {
    if (a.num_units <= 0 || a.H <= 0) return 0;
    return 1 + ((a.cu_seqlens && seq_order_bytes(a.num_units) > 0) ? 1 : 0);
}

cudaError_t launch_prefill_tc(const PrefillArgs &a) {
    if (a.num_units == 0) return cudaSuccess;
    const size_t tokens = a.cu_seqlens ? (size_t)a.T : (size_t)a.B * (size_t)a.T;
    // A batch without tokens only copies S0 to S_T; the SIMT kernel does that.
    if (tokens == 0) return launch_prefill_simt(a);
    // v and o may be null inside the library (zero values, no outputs): their maps are then
    // copies of q's and are never used
    CUtensorMap mq, mk, mv, mg, mo;
    if (!make_map(&mq, a.q, tokens, a.H, 64, true) || !make_map(&mk, a.k, tokens, a.H, 64, true) ||
        !make_map(&mv, a.v ? a.v : a.q, tokens, a.H, 64, true) || !make_map(&mg, a.g, tokens, a.H, 128, false) ||
        !make_map(&mo, a.o ? a.o : a.q, tokens, a.H, 64, true))
        return cudaErrorInvalidValue;
    const auto kern = a.fuse ? kda_prefill_tc_kernel<true> : kda_prefill_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    TcParams prm{a};
    if (a.cu_seqlens && seq_order_bytes(a.num_units) > 0) {
        int32_t *order = static_cast<int32_t *>(a.workspace);
        e = launch_seq_order(a.cu_seqlens, a.num_units, order, a.stream);
        if (e != cudaSuccess) return e;
        prm.a.seq_order = order;
    }
    const unsigned grid = (unsigned)((size_t)a.num_units * a.H);
    kern<<<grid, NT, SMEM_BYTES, a.stream>>>(mq, mk, mv, mg, mo, prm);
    return cudaGetLastError();
}

}  // namespace kda
