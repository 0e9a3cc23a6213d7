// Split tensor-core prefill (sm_100a): bf16 q/k/v/g/beta, fp32 state,
// dk = dv = 128, chunks of C = 64 tokens, in two kernels.
//
// Only a small part of a chunk's work depends on the state S it receives: the
// KCP pair of the chunk ("Exercices", Q21-Q22) is (Diag(Gamma_C) - Kh^T W, Kh^T Ut),
// and everything in it (the decayed Grams, the triangular solve, W, Ut, Kh) is a
// function of the chunk's own q, k, v, g, beta. So:
//
//  1. kda_prep_kernel runs every (sequence, head, chunk) task independently,
//     persistent CTAs striding over the tasks (two CTAs per SM): the cumulative
//     log-decay inside 16-token subtiles ("Exercices", Q8), the Gram operands
//     referenced to the middle of each 32-token column block, the Gram products
//     A and P on tcgen05, T = (I + A)^{-1} (diagonal 16 x 16 blocks by forward
//     substitution, merges with warp-level TF32 MMAs), and [W | Ut] =
//     T Diag(beta) [Gamma k | v] on tcgen05. It writes one record per task to the
//     workspace: [-W ; Gamma q] (the A operand of the state product), Kh, Ut, P
//     and Gamma_C, each as the image of the shared-memory tile the second kernel
//     feeds to its tensor cores.
//  2. kda_chain_kernel walks each (sequence, head) unit's chunks in order with
//     the fp32 state resident in TMEM (the KCP left fold): per chunk one bulk
//     copy brings the record (double-buffered, a chunk ahead), then
//        [U ; Gamma Q S] = [-W ; Gamma Q] S        (the record's Ut added at readout)
//        O = Gamma Q S + P U,   S <- Diag(Gamma_C) S + Kh^T U
//     with the U / O accumulator alternating between two TMEM regions so that the
//     next chunk's state product runs while this chunk's outputs are read out.
//
// The state-independent work, most of a chunk's cycles, is thereby spread over
// all SMs instead of sitting on each unit's serial chain. No cluster multicast
// is used; every copy is a plain TMA tile load, a bulk copy or a tensor store.
#include "kda_internal.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_common.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace tc;

constexpr int NT = 256;
constexpr uint32_t KB = 1024;

// ------------------------------------------------ per-task record in the workspace
// Three contiguous pieces, each the image of the shared-memory tiles its consumer feeds to
// the tensor cores, in the order the state chain needs them: A = [-W ; Gamma q] and Gamma_C
// (the state product and the state's decay), B = Ut and P (the U readout and the output
// product), C = Kh (the state update).
constexpr uint32_t REC_WQ = 0;          // 32 KB [-W ; Gamma q], K-major, 128 rows x 128, K-blocks 16 KB apart
constexpr uint32_t REC_GC = 32 * KB;    // 512 B Gamma_C (fp32, one per channel)
constexpr uint32_t REC_UT = 33 * KB;    // 16 KB Ut (bf16), MN-major [tok][dv], N-blocks 8 KB apart
constexpr uint32_t REC_P = 49 * KB;     // 8 KB  P (bf16, s <= r), K-major [r][s]
constexpr uint32_t REC_KH = 57 * KB;    // 16 KB Kh = e^{G_C - G} k, MN-major [tok][dk], 64-channel blocks 8 KB apart
constexpr uint32_t REC_BYTES = 73 * KB;
// a publication flag in the padding after Gamma_C, for records produced beside their chain
constexpr uint32_t REC_FLAG = REC_GC + 512;
constexpr uint32_t REC_A_BYTES = 32 * KB + 512;  // piece A: [REC_WQ, REC_GC + 512)
constexpr uint32_t REC_B_BYTES = 24 * KB;        // piece B: [REC_UT, REC_KH)
constexpr uint32_t REC_C_BYTES = 16 * KB;        // piece C: [REC_KH, REC_BYTES)
static_assert(REC_UT + REC_B_BYTES == REC_KH && REC_KH + REC_C_BYTES == REC_BYTES, "record pieces");
static_assert(REC_UT % 1024 == 0 && REC_P % 1024 == 0 && REC_KH % 1024 == 0, "tiles stay 1 KB aligned");
static_assert(REC_FLAG + 4 <= REC_UT, "the flag lies outside every tile");

// ------------------------------------------------------------ prep smem layout
constexpr uint32_t P_L0 = 0;          // 32 KB k (rows 0..63) and q (rows 64..127) tiles, the Gram left operand L0 in place
constexpr uint32_t P_L1 = 32 * KB;    // 16 KB Gram left operand L1 ([k ; q] rows 32..63, K-blocks 8 KB apart)
constexpr uint32_t P_R = 48 * KB;     // 16 KB Gram right operand, K-major [s][dk]
constexpr uint32_t P_GK = 64 * KB;    // 16 KB Gamma k, B operand MN-major [tok][dk]
constexpr uint32_t P_GV = 80 * KB;    // 16 KB g (plain [64][128] bf16), then v (B operand MN-major [tok][dv])
constexpr uint32_t P_MISC = 96 * KB;
// aliases once the Gram products are done (L0, L1, R free)
constexpr uint32_t P_TB = 0;                          // 8 KB A operand T Diag(beta) rows 0..63 (the MMA reads 16 KB)
constexpr uint32_t P_AF = 8 * KB;                     // 64 x LDA fp32 A
constexpr uint32_t P_TF = P_AF + 64 * LDA * 4;        // 64 x LDT fp32 T
constexpr uint32_t P_XS = P_TF + 64 * LDT * 4;        // 32 x LDX fp32 scratch
constexpr uint32_t P_PST = 48 * KB;                   // 8 KB P staging (record image)
// once the W / Ut product is done (T Diag(beta), Gamma k, v free)
constexpr uint32_t P_WST = 32 * KB;                   // 16 KB -W staging: the record's two K-blocks, rows 0..63
constexpr uint32_t P_UST = 56 * KB;                   // 16 KB Ut staging (record image)
static_assert(P_XS + 32 * LDX * 4 <= P_PST, "inverse scratch reaches the P staging");
static_assert(P_WST + 16 * KB <= P_PST && P_PST + 8 * KB <= P_UST, "staging tiles overlap");
static_assert(P_L1 + 8 * KB + 16 * KB <= P_GK, "L1 read as a 128-row operand reaches Gamma k");
constexpr uint32_t P_BAR = P_MISC;                    // 4 mbarriers
constexpr uint32_t P_TMEMADDR = P_MISC + 64;
constexpr uint32_t P_BETA = P_MISC + 128;             // 64 fp32
constexpr uint32_t P_DSUM = P_BETA + 256;             // 4 x 128 fp32 subtile totals of g (log2 units)
constexpr uint32_t P_NORM = P_DSUM + 2048;            // fused variant: 2 x 64 x 2 fp32 partial squared norms of k, q
constexpr uint32_t P_SMEM_USED = P_NORM + 1024;
constexpr uint32_t P_SMEM_BYTES = P_SMEM_USED + 1024;  // slack for 1024-byte alignment
static_assert(2 * (P_SMEM_BYTES + 1024) <= 233472, "two prep CTAs per SM");
constexpr uint32_t P_TM_W = 0, P_TM_UT = 128, P_TM_COLS = 256;  // the Gram uses columns 0..63 first

// ----------------------------------------------------------- chain smem layout
constexpr uint32_t C_RECSTRIDE = REC_BYTES;           // 1 KB aligned
constexpr uint32_t C_SB = 2 * C_RECSTRIDE;            // 32 KB S (bf16), B operand MN-major [dk][dv], N-blocks 16 KB apart
constexpr uint32_t C_OST = C_SB + 32 * KB;            // 16 KB output staging ([tok][dv], N-blocks 8 KB apart)
constexpr uint32_t C_MISC = C_OST + 16 * KB;
constexpr uint32_t C_BAR = C_MISC;                    // 3 mbarriers
constexpr uint32_t C_TMEMADDR = C_MISC + 64;
constexpr uint32_t C_SMEM_BYTES = C_MISC + 128 + 1024;
static_assert(REC_BYTES <= C_RECSTRIDE && C_SMEM_BYTES <= 232448, "chain shared memory budget");
constexpr uint32_t C_TM_U0 = 0, C_TM_U1 = 128, C_TM_S = 256, C_TM_COLS = 512;

struct SplitParams {
    PrefillArgs a;
    uint8_t *rec;               // records, REC_BYTES each, task t at rec + t * REC_BYTES
    const int32_t *chunk_base;  // packed batches: [num_units + 1] first task chunk of each sequence
    int nch;                    // dense batches: chunks per sequence
    long long tasks;            // dense batches: number of tasks (units x chunks)
    long long flag_from = 0, flag_to = 0;  // prep kernel: clear the flags of records flag_from .. flag_to - 1
};

// Task t = (global chunk index) * H + head. The global chunk index runs over the
// chunks of sequence 0, then sequence 1, ...; heads vary fastest, so CTAs that
// run neighbouring tasks read neighbouring rows of the [tokens, H, d] inputs.
struct Task {
    long long t, tok0;
    int n, h, Lc;
    int chain;      // ring-buffer form: the chain that consumes the record, and its index there
    long long tau;
};

__device__ __forceinline__ Task task_at(const SplitParams &sp, long long t) {
    const PrefillArgs &p = sp.a;
    Task k;
    k.t = t;
    // 32-bit quotients: the number of tasks is below 2^31 (checked when the call is validated)
    const unsigned t32 = (unsigned)t;
    k.h = (int)(t32 % (unsigned)p.H);
    const unsigned gc = t32 / (unsigned)p.H;
    long long c, end;
    if (sp.chunk_base) {  // largest n with chunk_base[n] <= gc (empty sequences share a base)
        int lo = 0, hi = p.num_units;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (sp.chunk_base[mid] <= gc) lo = mid; else hi = mid;
        }
        k.n = lo;
        c = gc - sp.chunk_base[lo];
        k.tok0 = (long long)p.cu_seqlens[lo] + c * C;
        end = p.cu_seqlens[lo + 1];
    } else {
        k.n = (int)(gc / (unsigned)sp.nch);
        c = gc % (unsigned)sp.nch;
        k.tok0 = (long long)k.n * p.T + c * C;
        end = (long long)k.n * p.T + p.T;
    }
    k.Lc = (int)((end - k.tok0) < C ? (end - k.tok0) : C);
    return k;
}

// First task chunk of every packed sequence: base[n] = sum over m < n of ceil(len_m / C),
// base[num] = the total. One block, tiles of blockDim.x sequences with a running carry.
__global__ void chunk_base_kernel(const int32_t *cu, int num, int32_t *base) {
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry_s;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int start = 0; start < num; start += blockDim.x) {
        const int i = start + tid;
        int v = 0;
        if (i < num) {
            const int len = cu[i + 1] - cu[i];
            v = len > 0 ? (len + C - 1) / C : 0;
        }
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[wid] = x;
        __syncthreads();
        if (wid == 0) {
            int w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_sums[lane] = w;
        }
        __syncthreads();
        const int carry = carry_s;
        const int incl = carry + (wid ? warp_sums[wid - 1] : 0) + x;
        if (i < num) base[i] = incl - v;
        __syncthreads();
        if (tid == blockDim.x - 1) carry_s = incl;
        __syncthreads();
    }
    if (tid == 0) base[num] = carry_s;
}

// ======================================================================= prep
// Every task of the batch, strided over the grid; the record of task t is the t-th of the
// workspace (the two-kernel form: the chains run after this kernel has finished). The tasks
// are taken from the last to the first, so that the records still in L2 when the chains start
// are those of the first chunks, which the chains read first.
struct StaticTasks {
    static constexpr bool kPublish = false, kLatePublish = false;
    const SplitParams *sp;
    long long t, total;
    __device__ bool first(Task &k) {
        total = sp->chunk_base ? (long long)sp->chunk_base[sp->a.num_units] * sp->a.H : sp->tasks;
        t = blockIdx.x;
        if (t >= total) return false;
        k = task_at(*sp, total - 1 - t);
        return true;
    }
    __device__ bool next(Task &k) {
        t += gridDim.x;
        if (t >= total) return false;
        k = task_at(*sp, total - 1 - t);
        return true;
    }
    __device__ uint8_t *record(const Task &k) const { return sp->rec + (size_t)k.t * REC_BYTES; }
    __device__ bool acquire(const Task &) { return true; }
    __device__ void release(const Task &) {}
};

// Tasks first_task .. sp->tasks - 1 of a dense batch, strided over `stride` producers: the
// last chunks' records, produced beside the chains that consume them. A record is published by
// its flag once all of its stores have completed.
struct TailTasks {
    static constexpr bool kPublish = true, kLatePublish = true;
    const SplitParams *sp;
    long long first_task, rank, stride, t;
    __device__ bool first(Task &k) {
        t = first_task + rank;
        if (t >= sp->tasks) return false;
        k = task_at(*sp, t);
        return true;
    }
    __device__ bool next(Task &k) {
        t += stride;
        if (t >= sp->tasks) return false;
        k = task_at(*sp, t);
        return true;
    }
    __device__ uint8_t *record(const Task &k) const { return sp->rec + (size_t)k.t * REC_BYTES; }
    __device__ bool acquire(const Task &) { return true; }
    __device__ void release(const Task &k) {
        fence_proxy_async_global();
        __threadfence();
        st_release_gpu(reinterpret_cast<unsigned *>(record(k) + REC_FLAG), 1u);
    }
};

// The persistent loop of a record-producing CTA over the tasks its source hands out.
// Src::acquire (thread 0) returns once the task's record may be written, before its first
// store; Src::release (thread 0) publishes a record whose stores have completed (kPublish):
// at the next task's acquire, or (kLatePublish, for sources whose acquire never waits on a
// consumer) after that task's first bulk store, by which time the record's stores are done.
// kFused: the variant with the fused pre-operations (p.fuse: q, k normalised per row inside the
// operand pass, g computed from gate logits in the cumulative decay), a separate instantiation
// so that the plain variant carries none of it.
template <bool kFused, class Src>
__device__ __forceinline__ void prep_loop(const CUtensorMap &tm_q, const CUtensorMap &tm_k, const CUtensorMap &tm_v,
                                          const CUtensorMap &tm_g, const SplitParams &sp, Src &src, uint8_t *sm,
                                          const Group &grp) {
    const PrefillArgs &p = sp.a;
    const bool fuse_gate = kFused && (p.fuse & KDA_FUSE_GATE_LOGITS) != 0;
    const bool fuse_norm = kFused && (p.fuse & KDA_FUSE_NORM_QK) != 0;
    float *sNorm = reinterpret_cast<float *>(sm + P_NORM);
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + P_BAR);  // k, q, g of a task
    uint64_t *bar_v = bar_ld + 1;
    uint64_t *bar_gram = bar_ld + 2;                               // 2 arrivals
    uint64_t *bar_mma = bar_ld + 3;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + P_TMEMADDR);
    float *sBeta = reinterpret_cast<float *>(sm + P_BETA);
    float *sD = reinterpret_cast<float *>(sm + P_DSUM);
    float *AF = reinterpret_cast<float *>(sm + P_AF);
    float *TF = reinterpret_cast<float *>(sm + P_TF);
    float *XS = reinterpret_cast<float *>(sm + P_XS);

    const int tid = grp.tid, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const size_t H = (size_t)p.H;
    const __nv_bfloat16 *beta = static_cast<const __nv_bfloat16 *>(p.beta);

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_gram, 2);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_g);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, P_TM_COLS);
        if (grp.relinquish) tmem_relinquish();
    }
    grp.sync();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;

    auto issue_kqg = [&](const Task &k) {
        tma_load_3d(sm + P_L0, &tm_k, bar_ld, 0, k.h, (int)k.tok0);
        tma_load_3d(sm + P_L0 + 16 * KB, &tm_k, bar_ld, 64, k.h, (int)k.tok0);
        tma_load_3d(sm + P_L0 + 8 * KB, &tm_q, bar_ld, 0, k.h, (int)k.tok0);
        tma_load_3d(sm + P_L0 + 24 * KB, &tm_q, bar_ld, 64, k.h, (int)k.tok0);
        tma_load_3d(sm + P_GV, &tm_g, bar_ld, 0, k.h, (int)k.tok0);
    };
    auto issue_v = [&](const Task &k) {
        tma_load_3d(sm + P_GV, &tm_v, bar_v, 0, k.h, (int)k.tok0);
        tma_load_3d(sm + P_GV + 8 * KB, &tm_v, bar_v, 64, k.h, (int)k.tok0);
    };
    const bool has_v = p.v != nullptr;  // all-zero values (a segment's transition): no v, Ut = 0

    Task cur{};
    bool have = src.first(cur);
    Task pend{};  // a record whose stores were issued and that is not yet published
    bool has_pend = false;
    // unwinding state (thread 0): armed transaction counts and a commit whose wait ran out
    bool ld_armed = false, v_armed = false;
    uint64_t *mma_bar = nullptr;
    uint32_t mma_bar_phase = 0;
    uint32_t ld_phase = 0, v_phase = 0, gram_phase = 0, mma_phase = 0;
    bool aborted = false;
    if (have && tid == 0) {
        mbar_arrive_expect_tx(bar_ld, 48 * KB);
        issue_kqg(cur);
        ld_armed = true;
    }
    __nv_bfloat16 bcur = __float2bfloat16(0.f);
    if (have && tid < C && tid < cur.Lc) bcur = beta[(size_t)(cur.tok0 + tid) * H + cur.h];

    // thread roles of the token-parallel passes (as in the single-kernel prefill): subtile ti,
    // half hh of it (8 rows), a quad of channels c0..c0+3
    const int ti = warp >> 1;
    const int hh = lane >> 4;
    const int cq = (warp & 1) * 16 + (lane & 15);
    const int c0 = 4 * cq;
    const int cblk = c0 >> 6;
    const int cin = c0 & 63;
    constexpr int HR = SUB / 2;
    constexpr uint32_t idG = idesc_bf16_f32(128, 32, 0, 0);
    constexpr uint32_t idWU = idesc_bf16_f32(128, 256, 0, 1);
    static_assert(P_GV == P_GK + 16 * KB && P_TM_UT == P_TM_W + 128, "[Gamma k | v] and [W | Ut] are contiguous");

    while (have) {
        Task nxt{};
        const bool more = src.next(nxt);
        uint8_t *rec = src.record(cur);
        const int Lc = cur.Lc;
        if (more && tid == 0) {  // the next task's tiles into L2 now; its loads come late (below)
            tma_prefetch_l2_3d(&tm_k, 0, nxt.h, (int)nxt.tok0);
            tma_prefetch_l2_3d(&tm_k, 64, nxt.h, (int)nxt.tok0);
            tma_prefetch_l2_3d(&tm_q, 0, nxt.h, (int)nxt.tok0);
            tma_prefetch_l2_3d(&tm_q, 64, nxt.h, (int)nxt.tok0);
            tma_prefetch_l2_3d(&tm_g, 0, nxt.h, (int)nxt.tok0);
            if (has_v) {
                tma_prefetch_l2_3d(&tm_v, 0, nxt.h, (int)nxt.tok0);
                tma_prefetch_l2_3d(&tm_v, 64, nxt.h, (int)nxt.tok0);
            }
        }

        // ---- this task's k, q, g
        {
            const bool ok = mbar_wait_bounded(bar_ld, ld_phase, kWaitCycles);
            if (ok) { ld_phase ^= 1u; ld_armed = false; }
            if (grp.sync_or(!ok)) { aborted = true; break; }
        }
        __nv_bfloat16 bnext = __float2bfloat16(0.f);
        if (tid < C) {
            sBeta[tid] = (tid < Lc) ? __bfloat162float(bcur) : 0.f;
            if (more && tid < nxt.Lc) bnext = beta[(size_t)(nxt.tok0 + tid) * H + nxt.h];
        }
        if (Lc < C) {  // zero the k and q rows past the end of the sequence
            for (int idx = tid; idx < (C - Lc) * 16; idx += NT) {
                const int r = Lc + idx / 16, q16 = idx % 16;
                const int blk = q16 >> 3, pc = (q16 & 7) * 8;
                const uint4 z = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sm + P_L0 + blk * 16 * KB + sw128_offset(r, pc)) = z;
                *reinterpret_cast<uint4 *>(sm + P_L0 + blk * 16 * KB + sw128_offset(64 + r, pc)) = z;
            }
        }

        // ---- cumulative log2-decay inside subtile ti for channels c0..c0+3
        float gl[HR][4];
        {
            float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int rr = 0; rr < HR; ++rr) {
                const int row = SUB * ti + HR * hh + rr;  // rows past the end decay by 1
                const uint2 raw = row < Lc ? *reinterpret_cast<const uint2 *>(sm + P_GV + row * 256 + c0 * 2)
                                           : make_uint2(0, 0);
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
            // squared norms of this thread's 8 k and 8 q rows over its 4 channels, summed over the
            // 16 lanes of the half-warp (64 channels) by a reduce-scatter: lane l ends with the sum
            // of value l (k row l, or q row l - 8); the partner warp holds the other 64 channels
            const uint8_t *l0 = sm + P_L0 + cblk * 16 * KB;
            float nv[2 * HR];
#pragma unroll
            for (int rr = 0; rr < HR; ++rr) {
                const int r = SUB * ti + HR * hh + rr;
                const uint2 kr = *reinterpret_cast<const uint2 *>(l0 + sw128_offset(r, cin));
                const uint2 qr = *reinterpret_cast<const uint2 *>(l0 + sw128_offset(64 + r, cin));
                const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kr.x));
                const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&kr.y));
                const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qr.x));
                const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qr.y));
                nv[rr] = r < Lc ? k01.x * k01.x + k01.y * k01.y + k23.x * k23.x + k23.y * k23.y : 0.f;
                nv[HR + rr] = r < Lc ? q01.x * q01.x + q01.y * q01.y + q23.x * q23.x + q23.y * q23.y : 0.f;
            }
            const int l16 = lane & 15;
#pragma unroll
            for (int w = 8; w >= 1; w >>= 1) {  // keep half of the values, add the partner's copies
                const bool up = l16 & w;
#pragma unroll
                for (int i = 0; i < w; ++i)
                    nv[i] = (up ? nv[i + w] : nv[i]) + __shfl_xor_sync(0xffffffffu, up ? nv[i] : nv[i + w], w);
            }
            const int r = SUB * ti + HR * hh + (l16 & 7);
            sNorm[((l16 >> 3) * C + r) * 2 + (warp & 1)] = nv[0];
        }
        // the previous task's record stores have read their staging (and, where records are
        // published at this point, completed: then that record is published); this task's
        // record may be written
        bool slot_ok = true;
        if (tid == 0) {
            if (Src::kPublish && !Src::kLatePublish) {
                bulk_wait_all();
                if (has_pend) src.release(pend);
                has_pend = false;
            } else {
                bulk_wait_read_all();
            }
            slot_ok = src.acquire(cur);
        }
        if (grp.sync_or(!slot_ok)) { aborted = true; break; }
        if (tid == 0 && has_v) {  // g consumed: v lands in its tile
            mbar_arrive_expect_tx(bar_v, 16 * KB);
            issue_v(cur);
            v_armed = true;
        }

        // ---- Gram operands (L0 in place, L1, R), Gamma k; Gamma q, Kh and Gamma_C to the record
        {
            float Dm[NSUB][4], ed[NSUB][4];
#pragma unroll
            for (int m = 0; m < NSUB; ++m) {
                const float4 d4 = *reinterpret_cast<const float4 *>(sD + m * D + c0);
                Dm[m][0] = d4.x; Dm[m][1] = d4.y; Dm[m][2] = d4.z; Dm[m][3] = d4.w;
#pragma unroll
                for (int e = 0; e < 4; ++e) ed[m][e] = ex2(Dm[m][e]);
            }
            float pg[4], post[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float a = 1.f, b = 1.f;
#pragma unroll
                for (int m = 0; m < NSUB; ++m) {
                    if (m < ti) a *= ed[m][e];
                    if (m >= ti) b *= ed[m][e];
                }
                pg[e] = a;    // Gamma at the start of subtile ti
                post[e] = b;  // decay from the start of subtile ti to the end of the chunk
            }
            if (ti == 0 && hh == 0) {
                *reinterpret_cast<float4 *>(rec + REC_GC + 4 * c0) =
                    make_float4(ed[0][0] * ed[1][0] * ed[2][0] * ed[3][0], ed[0][1] * ed[1][1] * ed[2][1] * ed[3][1],
                                ed[0][2] * ed[1][2] * ed[2][2] * ed[3][2], ed[0][3] * ed[1][3] * ed[2][3] * ed[3][3]);
            }
            // column block b (tokens 32b..32b+31) referenced to its middle token 32b + 16:
            //   el0 = e^{G_start(ti) - G_16}, el1 = e^{G_start(ti) - G_48} (ti >= 2),
            //   er  = e^{G_mid(block of ti) - G_start(ti)}
            float el0[4], el1[4], er[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                el0[e] = ti == 0 ? ex2(-Dm[0][e]) : ti == 1 ? 1.f : ti == 2 ? ed[1][e] : ed[1][e] * ed[2][e];
                el1[e] = ti == 2 ? ex2(-Dm[2][e]) : 1.f;
                er[e] = ti == 0 ? ed[0][e] : ti == 2 ? ed[2][e] : 1.f;
            }
            const float2 er2[2] = {make_float2(er[0], er[1]), make_float2(er[2], er[3])};
            const float2 post2[2] = {make_float2(post[0], post[1]), make_float2(post[2], post[3])};
            const float2 el02[2] = {make_float2(el0[0], el0[1]), make_float2(el0[2], el0[3])};
            const float2 el12[2] = {make_float2(el1[0], el1[1]), make_float2(el1[2], el1[3])};
            const float2 pg2[2] = {make_float2(pg[0], pg[1]), make_float2(pg[2], pg[3])};
            uint8_t *const l0 = sm + P_L0 + cblk * 16 * KB;
            uint8_t *const l1 = sm + P_L1 + cblk * 8 * KB;
            uint8_t *const rrow = sm + P_R + cblk * 8 * KB;
            uint8_t *const gkrow = sm + P_GK + cblk * 8 * KB;
            uint8_t *const gq_rec = rec + REC_WQ + cblk * 16 * KB + 8 * KB;
            uint8_t *const kh_rec = rec + REC_KH + cblk * 8 * KB;
            auto ld4 = [](const uint8_t *ptr, float (&v)[4]) {
                const uint2 raw = *reinterpret_cast<const uint2 *>(ptr);
                const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
                const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
                v[0] = x.x; v[1] = x.y; v[2] = y.x; v[3] = y.y;
            };
#pragma unroll
            for (int rr = 0; rr < HR; ++rr) {
                const int r = SUB * ti + HR * hh + rr;
                const uint32_t off_r = sw128_offset(r, cin);
                const uint32_t off_q = sw128_offset(64 + r, cin);
                float kx[4], qx[4];
                ld4(l0 + off_r, kx);
                ld4(l0 + off_q, qx);
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
                // paired fp32 products (two channels per instruction, each the same IEEE product)
                float2 F[2], Fi[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    F[e] = make_float2(ex2(gl[rr][2 * e]), ex2(gl[rr][2 * e + 1]));      // e^{G_r - G_start(ti)}
                    Fi[e] = make_float2(ex2(-gl[rr][2 * e]), ex2(-gl[rr][2 * e + 1]));  // e^{G_start(ti) - G_r}
                }
                float2 kr[2], kf[2], qf[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float2 k2 = make_float2(kx[2 * e], kx[2 * e + 1]);
                    const float2 q2 = make_float2(qx[2 * e], qx[2 * e + 1]);
                    kr[e] = __fmul2_rn(k2, Fi[e]);
                    kf[e] = __fmul2_rn(k2, F[e]);
                    qf[e] = __fmul2_rn(q2, F[e]);
                }
                auto st2 = [](uint8_t *ptr, const float2 (&x)[2], const float2 (&f)[2]) {
                    const __nv_bfloat162 a = __float22bfloat162_rn(__fmul2_rn(x[0], f[0]));
                    const __nv_bfloat162 b = __float22bfloat162_rn(__fmul2_rn(x[1], f[1]));
                    *reinterpret_cast<uint2 *>(ptr) =
                        make_uint2(*reinterpret_cast<const uint32_t *>(&a), *reinterpret_cast<const uint32_t *>(&b));
                };
                st2(rrow + off_r, kr, er2);
                st2(kh_rec + off_r, kr, post2);
                st2(l0 + off_r, kf, el02);
                st2(l0 + off_q, qf, el02);
                if (ti >= 2) {
                    st2(l1 + sw128_offset(r - 32, cin), kf, el12);
                    st2(l1 + sw128_offset(r, cin), qf, el12);
                }
                st2(gq_rec + off_r, qf, pg2);
                st2(gkrow + off_r, kf, pg2);
            }
        }
        // this thread's record stores before the publication (late publication: fenced then)
        if (Src::kPublish && !Src::kLatePublish) __threadfence();
        fence_proxy_async_smem();
        grp.sync();

        // ---- Gram MMAs: column block j -> TMEM columns 32j..32j+31, issued by lane 0 of warp j
        if (lane == 0 && warp < 2) {
            const int j = warp;
            tc_fence_after();
            Opnd A = (j == 0) ? Opnd{sbase + P_L0, false, 16 * KB, 0} : Opnd{sbase + P_L1, false, 8 * KB, 0};
            Opnd B{sbase + P_R + 32u * j * 128u, false, 8 * KB, 0};
            mma_chain<D / 16>(tmem + P_TM_W + 32u * j, A, B, idG, false);
            mma_commit(bar_gram);
        }
        {
            const bool ok = mbar_wait_bounded(bar_gram, gram_phase, kWaitCycles);
            if (!ok) { mma_bar = bar_gram; mma_bar_phase = gram_phase; }
            gram_phase ^= 1u;
            tc_fence_after();
            if (grp.sync_or(!ok)) { aborted = true; break; }
        }

        // ---- Gram readout -> A (fp32, strictly lower, times beta_r), P (bf16, lower) staging.
        // The masks select (never multiply), so upper-triangle entries that overflow are dropped.
        {
            float v2[2][16];
            tmem_ld16(tmem + tlane + P_TM_W + 32u * half, v2[0]);
            tmem_ld16(tmem + tlane + P_TM_W + 32u * half + 16u, v2[1]);
            tmem_wait_ld();
            const int j = half;
            const int m = 32 * quarter + lane;
            const int kr = 64 - 32 * j;
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
                uint8_t *prow = sm + P_PST;
#pragma unroll
                for (int s2 = 0; s2 < 32; s2 += 2) {
                    const int s = 32 * j + s2;
                    const float *v = v2[s2 >> 4] + (s2 & 15);
                    st_bf2(prow + sw128_offset(r, s), (s <= r) ? v[0] : 0.f, (s + 1 <= r) ? v[1] : 0.f);
                }
                if (j == 0 && r < 32) {  // the diagonal block of block 0: zero block 1's columns
                    for (int s = 32; s < C; s += 8)
                        *reinterpret_cast<uint4 *>(prow + sw128_offset(r, s)) = make_uint4(0, 0, 0, 0);
                }
            }
            // T Diag(beta) (bf16, rows 0..63) starts as zeros: the inverse writes its lower blocks
            // (L0 is free: the Gram products are done)
            *reinterpret_cast<uint4 *>(sm + P_TB + 16 * tid) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sm + P_TB + 16 * NT + 16 * tid) = make_uint4(0, 0, 0, 0);
        }
        // (late publication) the previous record's direct stores, issued a task ago, before the
        // sync after which it is published
        if (Src::kLatePublish) __threadfence();
        fence_proxy_async_smem();
        tc_fence_before();
        grp.sync();
        if (tid == 0) {
            bulk_store(rec + REC_P, sm + P_PST, 8 * KB);
            bulk_commit();
            if (Src::kLatePublish && has_pend) {  // every group but this P store: the previous record
                bulk_wait_all_but_last();
                src.release(pend);
                has_pend = false;
            }
        }

        // ---- T = (I + A)^{-1} (unit lower triangular) by 16 x 16 blocks
        if (warp < NSUB && lane < 16) {
            const int o0 = 16 * warp, cc = lane;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                float a[16];
                const float4 *arow = reinterpret_cast<const float4 *>(AF + (o0 + rr) * LDA + o0);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    if (4 * q4 < rr) {
                        const float4 tt = arow[q4];
                        a[4 * q4] = tt.x; a[4 * q4 + 1] = tt.y; a[4 * q4 + 2] = tt.z; a[4 * q4 + 3] = tt.w;
                    }
                }
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
                *reinterpret_cast<__nv_bfloat16 *>(sm + P_TB + sw128_offset(o0 + rr, o0 + cc)) =
                    __float2bfloat16_rn(x[rr] * bcol);
            }
            if ((warp & 1) == 0) {
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) TF[(o0 + rr) * LDT + o0 + 16 + cc] = 0.f;
            }
        }
        grp.sync();
        // the off-diagonal blocks of T, each also written times beta into T Diag(beta): the bf16
        // A operand of [W | Ut], rows 0..63 (rows 64..127 of the product are never read)
        tri_inverse_offdiag(AF, TF, XS, tid, grp.id, sm + P_TB, sBeta);
        // ---- v of this task (zero rows past the end; all zero for a transition pass). Every
        // thread has seen the copy complete before it zeroes rows of it, and one barrier both
        // publishes the tile to the tensor cores and agrees on a wait that ran out.
        bool v_ok = true;
        if (has_v) {
            v_ok = mbar_wait_bounded(bar_v, v_phase, kWaitCycles);
            if (v_ok) { v_phase ^= 1u; v_armed = false; }
            if (v_ok && Lc < C) {
                for (int idx = tid; idx < (C - Lc) * 16; idx += NT) {
                    const int r = Lc + idx / 16, q16 = idx % 16;
                    *reinterpret_cast<uint4 *>(sm + P_GV + (q16 >> 3) * 8 * KB + sw128_offset(r, (q16 & 7) * 8)) =
                        make_uint4(0, 0, 0, 0);
                }
            }
        } else {
            for (int idx = tid; idx < 16 * KB / 16; idx += NT)
                *reinterpret_cast<uint4 *>(sm + P_GV + 16 * idx) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        if (grp.sync_or(!v_ok)) { aborted = true; break; }

        // ---- [W | Ut] = T Diag(beta) [Gamma K | V]: one N = 256 chain, Gamma k and v being four
        // consecutive 64-column blocks and W, Ut consecutive accumulators (an MMA instruction
        // costs about as much at N = 128 as at N = 256, so this halves the instructions)
        if (tid == 0) {
            tc_fence_after();
            Opnd A{sbase + P_TB, false, 16 * KB, 0};
            Opnd BKV{sbase + P_GK, true, 0, 8 * KB};
            mma_chain<C / 16>(tmem + P_TM_W, A, BKV, idWU, false);
            mma_commit(bar_mma);
        }
        {
            const bool ok = mbar_wait_bounded(bar_mma, mma_phase, kWaitCycles);
            if (!ok) { mma_bar = bar_mma; mma_bar_phase = mma_phase; }
            mma_phase ^= 1u;
            tc_fence_after();
            if (grp.sync_or(!ok)) { aborted = true; break; }
        }
        // the next task's k, q, g: L0 and the g / v tile are free
        if (more && tid == 0) {
            mbar_arrive_expect_tx(bar_ld, 48 * KB);
            issue_kqg(nxt);
            ld_armed = true;
        }

        // ---- -W and Ut (rows 0..63) -> staging -> record
        if (quarter < 2) {
            const int r = 32 * quarter + lane;
            float v[4][16];
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + P_TM_W + 64u * half + 16u * gq, v[gq]);
            tmem_wait_ld();
            uint8_t *wst = sm + P_WST + half * 8 * KB;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                uint4 w0, w1;
                pack16(v[gq], -1.f, w0, w1);
                *reinterpret_cast<uint4 *>(wst + sw128_offset(r, 16 * gq)) = w0;
                *reinterpret_cast<uint4 *>(wst + sw128_offset(r, 16 * gq + 8)) = w1;
            }
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + P_TM_UT + 64u * half + 16u * gq, v[gq]);
            tmem_wait_ld();
            uint8_t *ust = sm + P_UST + half * 8 * KB;
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                uint4 w0, w1;
                pack16(v[gq], 1.f, w0, w1);
                *reinterpret_cast<uint4 *>(ust + sw128_offset(r, 16 * gq)) = w0;
                *reinterpret_cast<uint4 *>(ust + sw128_offset(r, 16 * gq + 8)) = w1;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        grp.sync();
        if (tid == 0) {
            bulk_store(rec + REC_WQ, sm + P_WST, 8 * KB);
            bulk_store(rec + REC_WQ + 16 * KB, sm + P_WST + 8 * KB, 8 * KB);
            bulk_store(rec + REC_UT, sm + P_UST, 16 * KB);
            bulk_commit();
        }
        pend = cur;
        has_pend = true;
        cur = nxt;
        have = more;
        bcur = bnext;
    }
    if (tid == 0) {
        bulk_wait_all();  // record stores complete (the direct stores are ordinary writes)
        if (Src::kPublish && has_pend && !aborted) src.release(pend);
    }
    if (aborted && tid == 0) {
        // unwind with nothing in flight: armed copies complete (bounded), a timed-out commit is
        // waited for (bounded) before TMEM is freed
        if (p.dev_status) atomicExch(p.dev_status, (int)KDA_ERR_TIMEOUT);
        if (ld_armed) mbar_wait_bounded(bar_ld, ld_phase, kWaitCycles);
        if (v_armed) mbar_wait_bounded(bar_v, v_phase, kWaitCycles);
        if (mma_bar) mbar_wait_bounded(mma_bar, mma_bar_phase, kWaitCycles);
    }
    tc_fence_before();
    grp.sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, P_TM_COLS);
    }
}

template <bool kFused>
__global__ void __launch_bounds__(NT, 2)
kda_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                const SplitParams sp) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    // the flags of the records that a later launch produces beside its chains start cleared
    for (long long t = sp.flag_from + (long long)blockIdx.x * NT + threadIdx.x; t < sp.flag_to;
         t += (long long)gridDim.x * NT)
        *reinterpret_cast<unsigned *>(sp.rec + (size_t)t * REC_BYTES + REC_FLAG) = 0u;
    StaticTasks src{&sp, 0, 0};
    prep_loop<kFused>(tm_q, tm_k, tm_v, tm_g, sp, src, sm, Group{(int)threadIdx.x, 0u, true});
}

// ====================================================================== chain
// U = (-W S from TMEM) + Ut for one row r of a 64-column half, written as bf16 over the Ut tile
// (MN-major [tok][dv], 128-byte rows): all of the row's Ut is loaded before any of it is
// overwritten, in two passes of 32 columns.
__device__ __forceinline__ void u_readout(const uint8_t *ut, uint8_t *dst, int r, uint32_t taddr, bool add_ut = true) {
#pragma unroll
    for (int g2 = 0; g2 < 2; ++g2) {
        float v[2][16];
        tmem_ld16(taddr + 32u * g2, v[0]);
        tmem_ld16(taddr + 32u * g2 + 16u, v[1]);
        uint4 w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = *reinterpret_cast<const uint4 *>(ut + sw128_offset(r, 32 * g2 + 8 * i));
        tmem_wait_ld();
        uint4 o4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t ws[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
            float *x = v[i >> 1] + 8 * (i & 1);
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = add_ut ? __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ws[e]))
                                        : make_float2(0.f, 0.f);
                pk[e] = pack_bf2(x[2 * e] + f.x, x[2 * e + 1] + f.y);
            }
            o4[i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4 *>(dst + sw128_offset(r, 32 * g2 + 8 * i)) = o4[i];
    }
}

// When a chain's records are complete: all of them (an earlier kernel wrote the array), or
// (records produced beside the chains) those of tasks below `first`, the others once their
// flag is set. ready_now is a test, wait a bounded wait (thread 0).
struct AllReady {
    __device__ bool ready_now(long long) const { return true; }
    __device__ bool wait(long long) const { return true; }
};
struct FlagReady {
    const uint8_t *rec;
    long long first;
    __device__ const unsigned *flag(long long t) const {
        return reinterpret_cast<const unsigned *>(rec + (size_t)t * REC_BYTES + REC_FLAG);
    }
    __device__ bool ready_now(long long t) const {
        if (t < first) return true;
        if (ld_acquire_gpu(flag(t)) == 0u) return false;
        fence_proxy_async_global();  // the bulk copy out of the record follows its publication
        return true;
    }
    __device__ bool wait(long long t) const {
        if (t < first) return true;
        const bool ok = wait_counter(flag(t), 1u, kWaitCycles);
        fence_proxy_async_global();  // the bulk copy out of the record follows its publication
        return ok;
    }
};

// The state chain of unit (sequence n, head h) over the record array, one 256-thread group:
// fp32 state resident in TMEM (all 512 columns), records double-buffered a chunk ahead.
// kSnap: the instantiation that also stores the state every p.snap_every tokens.
template <bool kSnap, class Rdy>
__device__ __forceinline__ void chain_dbuf(const SplitParams &sp, const CUtensorMap &tm_o, uint8_t *sm, const Group &grp,
                                           int n, int h, const Rdy &rdy) {
    const PrefillArgs &p = sp.a;
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar_rec = reinterpret_cast<uint64_t *>(sm + C_BAR);  // [2]: the record of buffer b
    uint64_t *bar_mma = bar_rec + 2;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + C_TMEMADDR);

    const int tid = grp.tid, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const size_t H = (size_t)p.H;
    long long t_begin, len, cbase;
    if (p.cu_seqlens) {
        t_begin = p.cu_seqlens[n];
        len = (long long)p.cu_seqlens[n + 1] - t_begin;
        cbase = sp.chunk_base[n];
    } else {
        t_begin = (long long)n * p.T;
        len = p.T;
        cbase = (long long)n * sp.nch;
    }
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.o);
    const size_t state_base = ((size_t)n * H + h) * (size_t)(D * D);
    const long long nchunks = (len + C - 1) / C;
    auto task = [&](long long c) -> long long { return (cbase + c) * (long long)H + h; };
    auto record = [&](long long c) -> const uint8_t * { return sp.rec + (size_t)task(c) * REC_BYTES; };

    if (tid == 0) {
        mbar_init(&bar_rec[0], 1);
        mbar_init(&bar_rec[1], 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_o);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, C_TM_COLS);
        if (grp.relinquish) tmem_relinquish();
    }
    grp.sync();
    // bit b: buffer b has a record load armed and not yet waited for / the parity of its next phase
    uint32_t rec_armed = 0, rec_phase = 0;
    // (thread 0) per buffer, a record whose flag was not yet set when the buffer freed up: loaded
    // just before it is needed; flag_fail: a flag wait gave up
    long long rec_late[2] = {-1, -1};
    bool flag_fail = false;
    auto load_rec = [&](long long c) {
        const int b = (int)(c & 1);
        mbar_arrive_expect_tx(&bar_rec[b], REC_BYTES);
        bulk_load(sm + b * C_RECSTRIDE, record(c), REC_BYTES, &bar_rec[b]);
        rec_armed |= 1u << b;
    };
    if (tid == 0) {  // records 0 and 1; record c + 2 is requested once chunk c's products are done
        for (int b = 0; b < 2 && b < nchunks; ++b) {
            if (!rdy.wait(task(b))) { flag_fail = true; break; }
            load_rec(b);
        }
    }
    // incoming state -> TMEM (fp32, lane = dk row, column = dv) and its bf16 copy
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    const int si = 32 * quarter + lane;
    {
        uint8_t *sb = sm + C_SB + half * 16 * KB;
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = 64 * half + 16 * gq + e;
                v[e] = p.S0 ? p.S0[state_base + (size_t)j * D + si] : 0.f;
            }
            tmem_st16(tmem + tlane + C_TM_S + 64u * half + 16u * gq, v);
            uint4 w0, w1;
            pack16(v, 1.f, w0, w1);
            *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq)) = w0;
            *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq + 8)) = w1;
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    grp.sync();
    tc_fence_after();

    constexpr uint32_t idKM = idesc_bf16_f32(128, 128, 0, 1);
    constexpr uint32_t idMM = idesc_bf16_f32(128, 128, 1, 1);
    uint32_t mma_phase = 0;
    bool aborted = false, mma_pending = false;
    auto wait_rec = [&](int b) -> bool {  // every thread takes part
        const bool ok = !flag_fail && mbar_wait_bounded(&bar_rec[b], (rec_phase >> b) & 1u, kWaitCycles);
        if (ok) { rec_phase ^= 1u << b; rec_armed &= ~(1u << b); }
        return !grp.sync_or(!ok);
    };
    auto issue_u = [&](int b) {  // [U ; Gamma Q S] = [-W ; Gamma Q] S into the accumulator of buffer b
        tc_fence_after();
        Opnd A{sbase + b * C_RECSTRIDE + REC_WQ, false, 16 * KB, 0};
        Opnd B{sbase + C_SB, true, 0, 16 * KB};
        mma_chain<D / 16>(tmem + (b ? C_TM_U1 : C_TM_U0), A, B, idKM, false);
        mma_commit(bar_mma);
    };

    if (nchunks > 0) {
        if (!wait_rec(0)) aborted = true;
        else if (tid == 0) { issue_u(0); mma_pending = true; }
    }
    for (long long ch = 0; ch < nchunks && !aborted; ++ch) {
        const int b = (int)(ch & 1);
        uint8_t *buf = sm + b * C_RECSTRIDE;
        const uint32_t tmu = b ? C_TM_U1 : C_TM_U0;
        const long long tok0 = t_begin + ch * C;
        const int Lc = (int)((len - ch * C) < C ? (len - ch * C) : C);
        const bool more = ch + 1 < nchunks;

        // S <- Diag(Gamma_C) S in TMEM while the state product runs, so that Kh^T U
        // accumulates onto the state directly
        {
            const float gam = reinterpret_cast<const float *>(buf + REC_GC)[si];
            float sv[4][16];
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + C_TM_S + 64u * half + 16u * gq, sv[gq]);
            tmem_wait_ld();
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
#pragma unroll
                for (int e = 0; e < 16; ++e) sv[gq][e] *= gam;
                tmem_st16(tmem + tlane + C_TM_S + 64u * half + 16u * gq, sv[gq]);
            }
            tmem_wait_st();
            tc_fence_before();
        }
        // every thread sees the state product complete; one barrier then both publishes U and
        // agrees on a wait that ran out
        bool ok = mbar_wait_bounded(bar_mma, mma_phase, kWaitCycles);
        if (ok) { mma_phase ^= 1u; mma_pending = false; }
        tc_fence_after();

        // U = Ut - W S (rows 0..63) -> bf16 B operand, written over the record's Ut tile
        // (all-zero values, the transition pass of a segment: the record's Ut is left out)
        if (ok && quarter < 2)
            u_readout(buf + REC_UT + half * 8 * KB, buf + REC_UT + half * 8 * KB, 32 * quarter + lane,
                      tmem + tlane + tmu + 64u * half, p.v != nullptr);
        fence_proxy_async_smem();
        tc_fence_before();
        if (grp.sync_or(!ok)) { aborted = true; break; }

        // O = Gamma Q S + P U (rows 64..127 of the accumulator), S += Kh^T U
        if (tid == 0) {
            tc_fence_after();
            Opnd AK{sbase + b * C_RECSTRIDE + REC_KH, true, 0, 8 * KB};
            Opnd BU{sbase + b * C_RECSTRIDE + REC_UT, true, 0, 8 * KB};
            Opnd AP{sbase + b * C_RECSTRIDE + REC_P - 8 * KB, false, 16 * KB, 0};
            mma_chain<C / 16>(tmem + C_TM_S, AK, BU, idMM, true);
            mma_chain<C / 16>(tmem + tmu, AP, BU, idKM, true);
            mma_commit(bar_mma);
            mma_pending = true;
        }
        ok = mbar_wait_bounded(bar_mma, mma_phase, kWaitCycles);
        if (ok) { mma_phase ^= 1u; mma_pending = false; }
        tc_fence_after();
        // this buffer's record is consumed (its generic reads were before the barrier above, the
        // products that read it are complete): the record two chunks ahead
        if (ok && tid == 0 && ch + 2 < nchunks) {
            if (rdy.ready_now(task(ch + 2))) load_rec(ch + 2);
            else rec_late[b] = ch + 2;
        }

        // the bf16 copy of the updated state: the next chunk's state product waits on it
        if (ok) {
            uint8_t *sb = sm + C_SB + half * 16 * KB;
            float sv[4][16];
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + C_TM_S + 64u * half + 16u * gq, sv[gq]);
            tmem_wait_ld();
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                uint4 w0, w1;
                pack16(sv[gq], 1.f, w0, w1);
                *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq)) = w0;
                *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq + 8)) = w1;
            }
            // a snapshot of the state after this chunk (dense batches; fp32, the S0 layout of one
            // sequence), from the values just read for the bf16 copy
            const long long done = (ch + 1) * C;
            if (kSnap && p.snap_every && Lc == C && done % p.snap_every == 0) {
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
        if (tid == 0) {
            bulk_wait_read_all();  // the previous chunk's output stores have read their staging
            if (rec_late[b ^ 1] == ch + 1) {  // the next record, requested late: it is needed now
                if (rdy.wait(task(ch + 1))) load_rec(ch + 1);
                else flag_fail = true;
                rec_late[b ^ 1] = -1;
            }
        }
        // every thread sees the next record land; one barrier then publishes the state's copy,
        // and agrees on both waits
        bool rok = true;
        if (more) {
            const int nb = b ^ 1;
            rok = !flag_fail && mbar_wait_bounded(&bar_rec[nb], (rec_phase >> nb) & 1u, kWaitCycles);
            if (rok) { rec_phase ^= 1u << nb; rec_armed &= ~(1u << nb); }
        }
        if (grp.sync_or(!ok || !rok)) { aborted = true; break; }
        if (more && tid == 0) { issue_u(b ^ 1); mma_pending = true; }

        // outputs (rows 64..127 of this chunk's accumulator) while the next product runs. A
        // full chunk is staged in its own tile and leaves by two tensor stores; the rows of a
        // partial chunk are stored directly.
        if (quarter >= 2 && p.o) {
            const int r = 32 * quarter + lane - 64;
            float v[4][16];
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) tmem_ld16(tmem + tlane + tmu + 64u * half + 16u * gq, v[gq]);
            tmem_wait_ld();
            if (Lc == C) {
                uint8_t *base = sm + C_OST + half * 8 * KB;
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
        fence_proxy_async_smem();
        tc_fence_before();
        grp.sync();
        if (tid == 0) {
            if (Lc == C && p.o) {
                tma_store_3d(&tm_o, sm + C_OST, 0, h, (int)tok0);
                tma_store_3d(&tm_o, sm + C_OST + 8 * KB, 64, h, (int)tok0);
                bulk_commit();
            }

        }
    }
    if (tid == 0) bulk_wait_all();

    if (aborted) {
        if (tid == 0) {
            if (p.dev_status) atomicExch(p.dev_status, (int)KDA_ERR_TIMEOUT);
            // a record still unpublished when the chain gave up is never requested
            for (int b = 0; b < 2; ++b)
                if ((rec_armed >> b) & 1u) mbar_wait_bounded(&bar_rec[b], (rec_phase >> b) & 1u, kWaitCycles);
            if (mma_pending) mbar_wait_bounded(bar_mma, mma_phase, kWaitCycles);
        }
    } else if (p.ST) {
        tc_fence_after();
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
            float sv[16];
            tmem_ld16(tmem + tlane + C_TM_S + 64u * half + 16u * gq, sv);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = 64 * half + 16 * gq + e;
                p.ST[state_base + (size_t)j * D + si] = sv[e];
            }
        }
    }
    tc_fence_before();
    grp.sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C_TM_COLS);
    }
}

template <bool kSnap>
__global__ void __launch_bounds__(NT, 1)
kda_chain_kernel(const __grid_constant__ CUtensorMap tm_o, const SplitParams sp) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const PrefillArgs &p = sp.a;
    chain_dbuf<kSnap>(sp, tm_o, sm, Group{(int)threadIdx.x, 0u, true}, unit_seq(p, blockIdx.x / p.H),
                      (int)(blockIdx.x % p.H), AllReady{});
}

// ================================================= persistent pipeline (one launch)
// With no more (sequence, head) units than a GPU-wide fraction of its CTA slots, one
// cooperative launch runs both roles at once: CTA c < NC carries unit c's state chain, the
// other CTAs produce records into a ring of R slots per chain. A record's slot is free once
// its chain has copied all three pieces of the record R places before it into shared memory
// (consumed[c]); a record is ready once its stores have completed (ready[c][slot] = tau + 1).
// Both flags only grow, are written with release and read with acquire semantics at GPU
// scope, and every wait is bounded. The producers take tasks in order of (record index, chain),
// so the earliest unfinished task can always proceed (its slot's earlier record belongs to an
// older, finished task), and the chains consume in order: no cycle of waits can form. The
// ring (NC x R x 73 KB, 28 MB for 96 units) stays in L2, so records do not cost HBM traffic.
constexpr int kRingSlots = 4;

// pipeline chain-role smem layout (the record pieces at their record offsets, then S bf16)
constexpr uint32_t X_SB = REC_BYTES;                  // 32 KB S (bf16), B operand MN-major
constexpr uint32_t X_BAR = X_SB + 32 * KB;            // 4 mbarriers (pieces A, B, C; MMA)
constexpr uint32_t X_TMEMADDR = X_BAR + 64;
constexpr uint32_t X_SMEM_USED = X_BAR + 128;
constexpr uint32_t X_TM_U = 0, X_TM_S = 128, X_TM_COLS = 256;

struct PipeParams {
    SplitParams sp;
    uint8_t *ring;        // [NC][R] records
    unsigned *ready;      // [NC][R]: record tau of chain c is in slot tau % R once ready >= tau + 1
    unsigned *consumed;   // [NC]: records 0 .. consumed - 1 of chain c have been copied out
    int NC, nprep;        // chains (one per unit) and producing CTAs
    long long ntasks;     // NC x the most chunks a unit can have
};


// Task t of the ring form: record tau = t / NC of chain c = t % NC (unit c: sequence c / H,
// head c % H); tasks past the end of a unit's sequence are skipped.
struct RingTasks {
    static constexpr bool kPublish = true, kLatePublish = false;
    const PipeParams *pp;
    long long t;     // the next candidate task
    long long rank;  // this producer's index among the pp->nprep producers
    __device__ bool valid(long long tt, Task &k) const {
        const PrefillArgs &p = pp->sp.a;
        const int c = (int)(tt % pp->NC);
        const long long tau = tt / pp->NC;
        const int n = c / p.H;
        long long b, e;
        if (p.cu_seqlens) {
            b = p.cu_seqlens[n];
            e = p.cu_seqlens[n + 1];
        } else {
            b = (long long)n * p.T;
            e = b + p.T;
        }
        const long long tok0 = b + tau * C;
        if (tok0 >= e) return false;
        k.t = tt;
        k.n = n;
        k.h = c % p.H;
        k.tok0 = tok0;
        k.Lc = (int)((e - tok0) < C ? (e - tok0) : C);
        k.chain = c;
        k.tau = tau;
        return true;
    }
    __device__ bool advance(Task &k) {
        for (; t < pp->ntasks; t += pp->nprep)
            if (valid(t, k)) return true;
        return false;
    }
    __device__ bool first(Task &k) {
        t = rank;
        return advance(k);
    }
    __device__ bool next(Task &k) {
        t += pp->nprep;
        return advance(k);
    }
    __device__ uint8_t *record(const Task &k) const {
        return pp->ring + ((size_t)k.chain * kRingSlots + (size_t)(k.tau % kRingSlots)) * REC_BYTES;
    }
    __device__ bool acquire(const Task &k) {
        if (k.tau < kRingSlots) return true;
        const bool ok = wait_counter(pp->consumed + k.chain, (unsigned)(k.tau - kRingSlots + 1), kWaitCycles);
        fence_proxy_async_global();  // the slot's bulk stores come after the chain's copies out of it
        return ok;
    }
    __device__ void release(const Task &k) {
        fence_proxy_async_global();
        __threadfence();
        st_release_gpu(pp->ready + (size_t)k.chain * kRingSlots + (size_t)(k.tau % kRingSlots), (unsigned)(k.tau + 1));
    }
};

// Where the pipe form's chains find their records: record tau of chain c is in slot tau % R
// of the ring once the producers have published it, and its slot is handed back once all
// three pieces are in shared memory.
struct RingRecords {
    const PipeParams *pp;
    int c;
    __device__ const uint8_t *slot(long long tau) const {
        return pp->ring + ((size_t)c * kRingSlots + (size_t)(tau % kRingSlots)) * REC_BYTES;
    }
    __device__ bool wait_ready(long long tau) const {  // thread 0
        const bool ok = wait_counter(pp->ready + (size_t)c * kRingSlots + (size_t)(tau % kRingSlots),
                                     (unsigned)(tau + 1), kWaitCycles);
        fence_proxy_async_global();
        return ok;
    }
    __device__ void release(long long tau) const { st_release_gpu(pp->consumed + c, (unsigned)(tau + 1)); }
};

// The state chain of unit (sequence n, head h) with its records read piece by piece into one
// buffer as their shared-memory tiles free up: A (state product operand, decay) once the state
// product is done, B (Ut, P) once the output product is done, C (Kh) once the outputs staged
// over it have left. One 256-thread group, ~106 KB of shared memory, 256 TMEM columns.
template <class Rec>
__device__ __forceinline__ void chain_role(const PrefillArgs &p, const CUtensorMap &tm_o, uint8_t *sm, const Group &grp,
                                           int n, int h, const Rec &recs) {
    const uint32_t sbase = smem_u32(sm);
    uint64_t *bar_a = reinterpret_cast<uint64_t *>(sm + X_BAR);
    uint64_t *bar_b = bar_a + 1;  // B: Ut and P
    uint64_t *bar_c = bar_a + 2;
    uint64_t *bar_mma = bar_a + 3;
    uint8_t *const uo = sm + REC_UT;  // U goes over the record's Ut
    const uint32_t uo_addr = sbase + REC_UT;
    uint8_t *const ostage = sm + REC_KH;  // a full chunk's outputs are staged over Kh
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + X_TMEMADDR);

    const int tid = grp.tid, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const size_t H = (size_t)p.H;
    long long t_begin, len;
    if (p.cu_seqlens) {
        t_begin = p.cu_seqlens[n];
        len = (long long)p.cu_seqlens[n + 1] - t_begin;
    } else {
        t_begin = (long long)n * p.T;
        len = p.T;
    }
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.o);
    const size_t state_base = ((size_t)n * H + h) * (size_t)(D * D);
    const long long nchunks = (len + C - 1) / C;
    auto slot = [&](long long tau) -> const uint8_t * { return recs.slot(tau); };

    if (tid == 0) {
        mbar_init(bar_a, 1);
        mbar_init(bar_b, 1);
        mbar_init(bar_c, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_o);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, X_TM_COLS);
        if (grp.relinquish) tmem_relinquish();
    }
    grp.sync();
    // thread-0 state of the copies: armed bits (1 A, 2 B, 4 C) and the phase of each barrier
    uint32_t armed = 0, ph_a = 0, ph_b = 0, ph_c = 0, mma_phase = 0;
    bool flag_fail = false, aborted = false, mma_pending = false;
    auto load_a = [&](long long tau) {
        mbar_arrive_expect_tx(bar_a, REC_A_BYTES);
        bulk_load(sm + REC_WQ, slot(tau) + REC_WQ, REC_A_BYTES, bar_a);
        armed |= 1u;
    };
    auto load_b = [&](long long tau) {
        mbar_arrive_expect_tx(bar_b, REC_B_BYTES);
        bulk_load(sm + REC_UT, slot(tau) + REC_UT, REC_B_BYTES, bar_b);
        armed |= 2u;
    };
    auto load_c = [&](long long tau) {
        mbar_arrive_expect_tx(bar_c, REC_C_BYTES);
        bulk_load(sm + REC_KH, slot(tau) + REC_KH, REC_C_BYTES, bar_c);
        armed |= 4u;
    };
    if (tid == 0 && nchunks > 0) {
        if (!recs.wait_ready(0)) {
            flag_fail = true;
        } else {
            load_a(0);
            load_b(0);
            load_c(0);
        }
    }
    // incoming state -> TMEM (fp32, lane = dk row, column = dv) and its bf16 copy
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    const int si = 32 * quarter + lane;
    {
        uint8_t *sb = sm + X_SB + half * 16 * KB;
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = 64 * half + 16 * gq + e;
                v[e] = p.S0 ? p.S0[state_base + (size_t)j * D + si] : 0.f;
            }
            tmem_st16(tmem + tlane + X_TM_S + 64u * half + 16u * gq, v);
            uint4 w0, w1;
            pack16(v, 1.f, w0, w1);
            *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq)) = w0;
            *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 16 * gq + 8)) = w1;
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (grp.sync_or(flag_fail)) aborted = true;
    tc_fence_after();

    constexpr uint32_t idKM = idesc_bf16_f32(128, 128, 0, 1);
    constexpr uint32_t idMM = idesc_bf16_f32(128, 128, 1, 1);
    // bounded waits every thread takes part in; a failure anywhere (or a failed flag wait in
    // thread 0) aborts the chain on every thread
    auto wait_piece = [&](uint64_t *bar, uint32_t &ph, uint32_t bit) -> bool {
        const bool ok = mbar_wait_bounded(bar, ph, kWaitCycles);
        if (ok) { ph ^= 1u; armed &= ~bit; }
        return grp.sync_or(!ok || flag_fail) == 0;
    };
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait_bounded(bar_mma, mma_phase, kWaitCycles);
        if (ok) { mma_phase ^= 1u; mma_pending = false; }
        tc_fence_after();
        return grp.sync_or(!ok) == 0;
    };
    auto issue_u = [&]() {  // [U ; Gamma Q S] = [-W ; Gamma Q] S
        tc_fence_after();
        Opnd A{sbase + REC_WQ, false, 16 * KB, 0};
        Opnd B{sbase + X_SB, true, 0, 16 * KB};
        mma_chain<D / 16>(tmem + X_TM_U, A, B, idKM, false);
        mma_commit(bar_mma);
        mma_pending = true;
    };

    if (!aborted && nchunks > 0) {
        if (!wait_piece(bar_a, ph_a, 1u)) aborted = true;
        else if (tid == 0) issue_u();
    }
    for (long long tau = 0; tau < nchunks && !aborted; ++tau) {
        const long long tok0 = t_begin + tau * C;
        const int Lc = (int)((len - tau * C) < C ? (len - tau * C) : C);
        const bool more = tau + 1 < nchunks;

        // S <- Diag(Gamma_C) S while the state product runs
        {
            const float gam = reinterpret_cast<const float *>(sm + REC_GC)[si];
#pragma unroll
            for (int g2 = 0; g2 < 2; ++g2) {
                float sv[2][16];
#pragma unroll
                for (int gq = 0; gq < 2; ++gq)
                    tmem_ld16(tmem + tlane + X_TM_S + 64u * half + 32u * g2 + 16u * gq, sv[gq]);
                tmem_wait_ld();
#pragma unroll
                for (int gq = 0; gq < 2; ++gq) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) sv[gq][e] *= gam;
                    tmem_st16(tmem + tlane + X_TM_S + 64u * half + 32u * g2 + 16u * gq, sv[gq]);
                }
            }
            tmem_wait_st();
            tc_fence_before();
        }
        if (!wait_mma()) { aborted = true; break; }
        // piece A of the next record (the state product's operand and Gamma_C are consumed)
        if (tid == 0 && more) {
            if (!recs.wait_ready(tau + 1)) flag_fail = true;
            else load_a(tau + 1);
        }
        if (!wait_piece(bar_b, ph_b, 2u)) { aborted = true; break; }

        // U = Ut - W S (rows 0..63) -> bf16 B operand, over the record's Ut tile
        if (quarter < 2)
            u_readout(sm + REC_UT + half * 8 * KB, uo + half * 8 * KB, 32 * quarter + lane,
                      tmem + tlane + X_TM_U + 64u * half, p.v != nullptr);
        fence_proxy_async_smem();
        tc_fence_before();
        if (!wait_piece(bar_c, ph_c, 4u)) { aborted = true; break; }
        if (tid == 0) {
            // every piece of record tau is in shared memory: its slot may be refilled
            recs.release(tau);
            tc_fence_after();
            Opnd AK{sbase + REC_KH, true, 0, 8 * KB};
            Opnd BU{uo_addr, true, 0, 8 * KB};
            Opnd AP{sbase + REC_P - 8 * KB, false, 16 * KB, 0};
            mma_chain<C / 16>(tmem + X_TM_S, AK, BU, idMM, true);
            mma_chain<C / 16>(tmem + X_TM_U, AP, BU, idKM, true);
            mma_commit(bar_mma);
            mma_pending = true;
        }
        if (!wait_mma()) { aborted = true; break; }
        if (tid == 0 && more && !flag_fail) load_b(tau + 1);  // Ut, U and P are consumed

        // the bf16 copy of the updated state, and this chunk's outputs (rows 64..127 of the
        // accumulator) out of TMEM before the next state product overwrites it: a full chunk is
        // staged over the Kh tile (its product is done) for two tensor stores, the rows of a
        // partial chunk are stored directly
        {
            uint8_t *sb = sm + X_SB + half * 16 * KB;
#pragma unroll
            for (int g2 = 0; g2 < 2; ++g2) {
                float sv[2][16];
#pragma unroll
                for (int gq = 0; gq < 2; ++gq)
                    tmem_ld16(tmem + tlane + X_TM_S + 64u * half + 32u * g2 + 16u * gq, sv[gq]);
                tmem_wait_ld();
#pragma unroll
                for (int gq = 0; gq < 2; ++gq) {
                    uint4 w0, w1;
                    pack16(sv[gq], 1.f, w0, w1);
                    *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 32 * g2 + 16 * gq)) = w0;
                    *reinterpret_cast<uint4 *>(sb + sw128_offset(si, 32 * g2 + 16 * gq + 8)) = w1;
                }
            }
        }
        if (quarter >= 2 && p.o) {
            const int r = 32 * quarter + lane - 64;
#pragma unroll
            for (int g2 = 0; g2 < 2; ++g2) {
                float ov[2][16];
#pragma unroll
                for (int gq = 0; gq < 2; ++gq)
                    tmem_ld16(tmem + tlane + X_TM_U + 64u * half + 32u * g2 + 16u * gq, ov[gq]);
                tmem_wait_ld();
                if (Lc == C) {
                    uint8_t *base = ostage + half * 8 * KB;
#pragma unroll
                    for (int gq = 0; gq < 2; ++gq) {
                        uint4 w0, w1;
                        pack16(ov[gq], 1.f, w0, w1);
                        *reinterpret_cast<uint4 *>(base + sw128_offset(r, 32 * g2 + 16 * gq)) = w0;
                        *reinterpret_cast<uint4 *>(base + sw128_offset(r, 32 * g2 + 16 * gq + 8)) = w1;
                    }
                } else if (r < Lc) {
                    uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)(tok0 + r) * H + h) * D + 64 * half + 32 * g2);
#pragma unroll
                    for (int gq = 0; gq < 2; ++gq) {
                        uint4 w0, w1;
                        pack16(ov[gq], 1.f, w0, w1);
                        dst[2 * gq] = w0;
                        dst[2 * gq + 1] = w1;
                    }
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        grp.sync();
        if (more) {
            if (!wait_piece(bar_a, ph_a, 1u)) { aborted = true; break; }
            if (tid == 0) issue_u();
        }
        if (tid == 0) {
            if (Lc == C && p.o) {
                tma_store_3d(&tm_o, ostage, 0, h, (int)tok0);
                tma_store_3d(&tm_o, ostage + 8 * KB, 64, h, (int)tok0);
                bulk_commit();
            }
            if (more && !flag_fail) {  // Kh of the next record, once the outputs have left its tile
                bulk_wait_read_all();
                load_c(tau + 1);
            }
        }
    }
    if (tid == 0) bulk_wait_all();

    if (aborted) {
        if (tid == 0) {
            if (p.dev_status) atomicExch(p.dev_status, (int)KDA_ERR_TIMEOUT);
            if (armed & 1u) mbar_wait_bounded(bar_a, ph_a, kWaitCycles);
            if (armed & 2u) mbar_wait_bounded(bar_b, ph_b, kWaitCycles);
            if (armed & 4u) mbar_wait_bounded(bar_c, ph_c, kWaitCycles);
            if (mma_pending) mbar_wait_bounded(bar_mma, mma_phase, kWaitCycles);
        }
    } else if (p.ST) {
        tc_fence_after();
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
            float sv[16];
            tmem_ld16(tmem + tlane + X_TM_S + 64u * half + 16u * gq, sv);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int j = 64 * half + 16 * gq + e;
                p.ST[state_base + (size_t)j * D + si] = sv[e];
            }
        }
    }
    tc_fence_before();
    grp.sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, X_TM_COLS);
    }
}

// One CTA of two 256-thread groups per SM, each with half of the shared memory and its own 256
// TMEM columns (the occupancy calculator counts a CTA that allocates tensor memory once per
// SM, so a cooperative launch of two CTAs per SM is refused; two groups in one CTA are not).
// Group slot G = gi * gridDim.x + blockIdx.x: the first NC slots carry the chains (group 0 of
// the first NC CTAs, one chain per SM while there are SMs), the others produce records.
constexpr uint32_t PIPE_GROUP_BYTES = ((X_SMEM_USED > P_SMEM_USED ? X_SMEM_USED : P_SMEM_USED) + 1023) / 1024 * 1024;
constexpr uint32_t PIPE_SMEM = 2 * PIPE_GROUP_BYTES + 1024;
static_assert(PIPE_SMEM <= 232448, "two groups in one CTA");

__global__ void __launch_bounds__(2 * NT, 1)
kda_pipe_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                const __grid_constant__ CUtensorMap tm_o, const PipeParams pp) {
    extern __shared__ uint8_t smem_raw[];
    const int gi = (int)(threadIdx.x >> 8);
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u) + gi * PIPE_GROUP_BYTES;
    const Group grp{(int)(threadIdx.x & (NT - 1)), 1u + (uint32_t)gi, false};
    const int G = gi * (int)gridDim.x + (int)blockIdx.x;
    if (G < pp.NC) {
        const RingRecords recs{&pp, G};
        chain_role(pp.sp.a, tm_o, sm, grp, G / pp.sp.a.H, G % pp.sp.a.H, recs);
    } else {
        RingTasks src{&pp, 0, G - pp.NC};
        prep_loop<false>(tm_q, tm_k, tm_v, tm_g, pp.sp, src, sm, grp);
    }
}

// The tail form (dense batches of one sequence with SMs to spare beside its units): the prep
// kernel writes the records of the first chunks, then one cooperative launch runs every unit's
// chain on an SM of its own (CTA c < nchain, one 256-thread group) while the other CTAs, two
// producing groups each, write the last chunks' records; a chain waits for such a record by its
// flag. The chains use SMs the two-kernel form leaves idle while they run.
struct TailParams {
    SplitParams sp;   // the records; sp.tasks = every task of the batch
    long long first;  // the first task produced in this launch (its flag and all later ones cleared)
    int nchain;       // (sequence, head) units = chain CTAs
};
constexpr uint32_t TAIL_GROUP_BYTES = (P_SMEM_USED + 1023) / 1024 * 1024;
constexpr uint32_t TAIL_SMEM_USED = C_SMEM_BYTES - 1024 > 2 * TAIL_GROUP_BYTES ? C_SMEM_BYTES - 1024 : 2 * TAIL_GROUP_BYTES;
constexpr uint32_t TAIL_SMEM = TAIL_SMEM_USED + 1024;
static_assert(TAIL_SMEM <= 232448, "a chain, or two producing groups, in one CTA");

// kFused: the producers' fused pre-operations; kSnap: the chains' state snapshots
template <bool kFused, bool kSnap>
__global__ void __launch_bounds__(2 * NT, 1)
kda_tail_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                const __grid_constant__ CUtensorMap tm_o, const TailParams tp) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int gi = (int)(threadIdx.x >> 8);
    const PrefillArgs &p = tp.sp.a;
    if ((int)blockIdx.x < tp.nchain) {
        if (gi != 0) return;  // one group carries the chain, with all of the CTA's TMEM
        chain_dbuf<kSnap>(tp.sp, tm_o, base, Group{(int)threadIdx.x, 1u, true}, unit_seq(p, blockIdx.x / p.H),
                          (int)(blockIdx.x % p.H), FlagReady{tp.sp.rec, tp.first});
    } else {
        TailTasks src{&tp.sp, tp.first, 2LL * ((int)blockIdx.x - tp.nchain) + gi,
                      2LL * ((int)gridDim.x - tp.nchain), 0};
        prep_loop<kFused>(tm_q, tm_k, tm_v, tm_g, tp.sp, src, base + gi * TAIL_GROUP_BYTES,
                          Group{(int)(threadIdx.x & (NT - 1)), 1u + (uint32_t)gi, false});
    }
}

int num_sms() { return device_sm_count(); }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// One packed sequence (cu_seqlens = [0, T]) is the dense batch B = 1; the split form treats it
// so, which keeps its workspace the size kda_forward_workspace_size reports for num_seqs = 1.
bool packed(const PrefillArgs &a) { return a.cu_seqlens != nullptr && a.num_units > 1; }

// Upper bound of the number of tasks: dense batches exactly, packed ones by
// sum ceil(len / C) <= T / C + num_seqs.
long long split_tasks_bound(const PrefillArgs &a) {
    if (packed(a)) return ((long long)(a.T + C - 1) / C + a.num_units) * a.H;
    return (long long)a.B * ((a.T + C - 1) / C) * a.H;
}

// The one-launch form: one chain CTA per (sequence, head) unit, at most two thirds of the
// grid's CTA slots (two per SM), so that at least a third produce records.
long long pipe_units(const PrefillArgs &a) { return (long long)a.num_units * a.H; }
bool pipe_ok(const PrefillArgs &a) {
    const long long units = pipe_units(a);
    return units >= 1 && 3 * units <= 2 * (2LL * num_sms());
}
size_t pipe_ring_bytes(const PrefillArgs &a) { return align256((size_t)pipe_units(a) * kRingSlots * REC_BYTES); }
size_t pipe_flag_bytes(const PrefillArgs &a) {
    return align256((size_t)pipe_units(a) * (kRingSlots + 1) * sizeof(unsigned));
}

cudaError_t launch_pipe(const PrefillArgs &a, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                        const CUtensorMap &mg, const CUtensorMap &mo) {
    const int grid = num_sms();  // one CTA of two groups per SM, all resident (cooperative launch)
    int per_sm = 0;
    cudaError_t e = cudaFuncSetAttribute(kda_pipe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PIPE_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kda_pipe_kernel, 2 * NT, PIPE_SMEM);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    PipeParams pp{};
    pp.sp.a = a;
    if (!packed(a)) pp.sp.a.cu_seqlens = nullptr;
    pp.sp.nch = (a.T + C - 1) / C;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    pp.ring = ws;
    pp.ready = reinterpret_cast<unsigned *>(ws + pipe_ring_bytes(a));
    pp.NC = (int)pipe_units(a);
    pp.consumed = pp.ready + (size_t)pp.NC * kRingSlots;
    pp.nprep = 2 * grid - pp.NC;
    pp.ntasks = (long long)pp.NC * pp.sp.nch;  // a unit has at most ceil(T / C) chunks
    e = cudaMemsetAsync(pp.ready, 0, pipe_flag_bytes(a), a.stream);
    if (e != cudaSuccess) return e;
    void *args[] = {const_cast<CUtensorMap *>(&mq), const_cast<CUtensorMap *>(&mk), const_cast<CUtensorMap *>(&mv),
                    const_cast<CUtensorMap *>(&mg), const_cast<CUtensorMap *>(&mo), &pp};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kda_pipe_kernel), dim3(grid), dim3(2 * NT), args,
                                       PIPE_SMEM, a.stream);
}

}  // namespace

int device_sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
            n = v;
        else
            n = 148;
    }
    return n;
}

size_t prefill_split_workspace(const PrefillArgs &a) {
    size_t ws = align256((size_t)split_tasks_bound(a) * REC_BYTES);
    if (packed(a)) ws += align256((size_t)(a.num_units + 1) * sizeof(int32_t)) + align256(seq_order_bytes(a.num_units));
    return ws;
}

int prefill_split_launches(const PrefillArgs &a) {
    if (a.num_units <= 0 || a.H <= 0) return 0;
    const size_t tokens = a.cu_seqlens ? (size_t)a.T : (size_t)a.B * (size_t)a.T;
    if (tokens == 0) return prefill_simt_launches(a);
    return 2 + (packed(a) ? 1 + (seq_order_bytes(a.num_units) > 0 ? 1 : 0) : 0);
}

bool prefill_pipe_supported(const PrefillArgs &a) { return pipe_ok(a); }
size_t prefill_pipe_workspace(const PrefillArgs &a) { return pipe_ring_bytes(a) + pipe_flag_bytes(a); }
int prefill_pipe_launches(const PrefillArgs &a) {
    if (a.num_units <= 0 || a.H <= 0) return 0;
    const size_t tokens = a.cu_seqlens ? (size_t)a.T : (size_t)a.B * (size_t)a.T;
    return tokens == 0 ? prefill_simt_launches(a) : 1;
}

cudaError_t launch_prefill_pipe(const PrefillArgs &a) {
    if (a.num_units == 0) return cudaSuccess;
    const size_t tokens = a.cu_seqlens ? (size_t)a.T : (size_t)a.B * (size_t)a.T;
    if (tokens == 0) return launch_prefill_simt(a);
    if (!pipe_ok(a)) return cudaErrorInvalidConfiguration;
    CUtensorMap mq, mk, mv, mg, mo;
    if (!make_map(&mq, a.q, tokens, a.H, 64, true) || !make_map(&mk, a.k, tokens, a.H, 64, true) ||
        !make_map(&mv, a.v ? a.v : a.q, tokens, a.H, 64, true) || !make_map(&mg, a.g, tokens, a.H, 128, false) ||
        !make_map(&mo, a.o ? a.o : a.q, tokens, a.H, 64, true))
        return cudaErrorInvalidValue;
    return launch_pipe(a, mq, mk, mv, mg, mo);
}

cudaError_t launch_split_records(const PrefillArgs &a, SplitRecords *out) {
    *out = SplitRecords{};
    if (a.num_units == 0) return cudaSuccess;
    const size_t tokens = a.cu_seqlens ? (size_t)a.T : (size_t)a.B * (size_t)a.T;
    if (tokens == 0) return cudaSuccess;
    CUtensorMap mq, mk, mv, mg;
    if (!make_map(&mq, a.q, tokens, a.H, 64, true) || !make_map(&mk, a.k, tokens, a.H, 64, true) ||
        !make_map(&mv, a.v ? a.v : a.q, tokens, a.H, 64, true) || !make_map(&mg, a.g, tokens, a.H, 128, false))
        return cudaErrorInvalidValue;
    const auto prep = a.fuse ? kda_prep_kernel<true> : kda_prep_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(prep, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    SplitParams sp{};
    sp.a = a;
    if (!packed(a)) sp.a.cu_seqlens = nullptr;  // dense, or one packed sequence = B = 1 of T tokens
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    sp.rec = ws;
    const long long bound = split_tasks_bound(a);
    size_t off = align256((size_t)bound * REC_BYTES);
    if (packed(a)) {
        int32_t *base = reinterpret_cast<int32_t *>(ws + off);
        off += align256((size_t)(a.num_units + 1) * sizeof(int32_t));
        chunk_base_kernel<<<1, 1024, 0, a.stream>>>(a.cu_seqlens, a.num_units, base);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        sp.chunk_base = base;
        if (seq_order_bytes(a.num_units) > 0) {
            int32_t *order = reinterpret_cast<int32_t *>(ws + off);
            e = launch_seq_order(a.cu_seqlens, a.num_units, order, a.stream);
            if (e != cudaSuccess) return e;
            sp.a.seq_order = order;
        }
    } else {
        sp.nch = (a.T + C - 1) / C;
        sp.tasks = bound;
    }
    const long long grid_p = bound < 2LL * num_sms() ? bound : 2LL * num_sms();
    prep<<<(unsigned)grid_p, NT, P_SMEM_BYTES, a.stream>>>(mq, mk, mv, mg, sp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    out->rec = sp.rec;
    out->chunk_base = sp.chunk_base;
    out->seq_order = sp.a.seq_order;
    out->nch = sp.nch;
    out->tasks = sp.tasks;
    return cudaSuccess;
}

bool prefill_split_snapshots_ok(const PrefillArgs &a) {
    return !packed(a) && (long long)a.num_units * a.H <= num_sms();
}

cudaError_t launch_split_chain(const PrefillArgs &pass, const SplitRecords &r) {
    if (pass.num_units == 0) return cudaSuccess;
    if (pass.snap_every && !prefill_split_snapshots_ok(pass)) return cudaErrorInvalidValue;
    const size_t tokens = pass.cu_seqlens ? (size_t)pass.T : (size_t)pass.B * (size_t)pass.T;
    if (tokens == 0) return launch_prefill_simt(pass);
    CUtensorMap mo;
    if (!make_map(&mo, pass.o ? pass.o : pass.q, tokens, pass.H, 64, true)) return cudaErrorInvalidValue;
    // the double-buffered chains, one per SM, in as many waves as the units need (with more
    // units than SMs they beat one-buffer chains two per SM: 2 x 96 heads x 8192 tokens took
    // 1.22 ms per step against 1.39)
    cudaError_t e = cudaFuncSetAttribute(pass.snap_every ? kda_chain_kernel<true> : kda_chain_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    SplitParams sp{};
    sp.a = pass;
    if (!packed(pass)) sp.a.cu_seqlens = nullptr;
    sp.a.seq_order = r.seq_order;
    sp.rec = r.rec;
    sp.chunk_base = r.chunk_base;
    sp.nch = r.nch;
    sp.tasks = r.tasks;
    const unsigned grid_c = (unsigned)((size_t)pass.num_units * pass.H);
    if (pass.snap_every)
        kda_chain_kernel<true><<<grid_c, NT, C_SMEM_BYTES, pass.stream>>>(mo, sp);
    else
        kda_chain_kernel<false><<<grid_c, NT, C_SMEM_BYTES, pass.stream>>>(mo, sp);
    return cudaGetLastError();
}

// The tail form's split of the tasks: P producing groups keep pace with the chains over the
// last r x P x nch / units chunks, r the ratio of a chain's cycles per chunk to a producing
// group's cycles per task. Measured on B200 (96 heads, 8192 tokens): about 4.4K and 23K (two
// groups of one CTA per SM; the step is fastest at r = 0.19, 0.59 ms against 0.636 for the
// two-kernel form, with 26 of 128 chunks in the tail; the producers with fused pre-operations
// take about 1.4 times as long per task, and that step is fastest at r = 0.12, 16 chunks in the
// tail, 0.74 ms against 0.76 at 0.14); the prep kernel does the other chunks.
// With few units the chains dominate the step (8 heads x 65,536 tokens: 2.7 ms, the prep of all
// records 0.27 ms), and the tail form only adds its flag checks to them.
bool tail_ok(const PrefillArgs &a) {
    const long long units = (long long)a.num_units * a.H;
    return !packed(a) && a.num_units == 1 && !(a.fuse && a.snap_every) && units >= 32 &&
           units + 8 <= num_sms() && (a.T + C - 1) / C >= 4;
}
const void *tail_kernel_for(const PrefillArgs &a) {
    if (a.snap_every) return reinterpret_cast<const void *>(kda_tail_kernel<false, true>);
    return a.fuse ? reinterpret_cast<const void *>(kda_tail_kernel<true, false>)
                  : reinterpret_cast<const void *>(kda_tail_kernel<false, false>);
}
long long tail_first_task(const PrefillArgs &a) {
    const long long units = a.H, nch = (a.T + C - 1) / C;
    const long long producers = 2LL * (num_sms() - units);
    const double r = a.fuse ? 0.12 : 0.19;
    long long tail = (long long)((double)producers * (double)nch * r / (double)units);
    tail = tail < 1 ? 1 : (tail > nch - 1 ? nch - 1 : tail);
    return (nch - tail) * units;
}

// whether the tail kernel runs as one cooperative launch of a CTA per SM here
bool tail_launchable(const PrefillArgs &a) {
    const void *tail = tail_kernel_for(a);
    if (cudaFuncSetAttribute(tail, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TAIL_SMEM) != cudaSuccess)
        return false;
    int per_sm = 0, dev = 0, coop = 0;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tail, 2 * NT, TAIL_SMEM) == cudaSuccess && per_sm >= 1 &&
           cudaGetDevice(&dev) == cudaSuccess &&
           cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess && coop != 0;
}

cudaError_t launch_split_tail(const PrefillArgs &a) {
    const size_t tokens = (size_t)a.T;
    CUtensorMap mq, mk, mv, mg, mo;
    if (!make_map(&mq, a.q, tokens, a.H, 64, true) || !make_map(&mk, a.k, tokens, a.H, 64, true) ||
        !make_map(&mv, a.v ? a.v : a.q, tokens, a.H, 64, true) || !make_map(&mg, a.g, tokens, a.H, 128, false) ||
        !make_map(&mo, a.o ? a.o : a.q, tokens, a.H, 64, true))
        return cudaErrorInvalidValue;
    SplitParams sp{};
    sp.a = a;
    sp.a.cu_seqlens = nullptr;  // dense, or one packed sequence = B = 1 of T tokens
    sp.rec = static_cast<uint8_t *>(a.workspace);
    sp.nch = (a.T + C - 1) / C;
    const long long total = split_tasks_bound(a), first = tail_first_task(a);
    // the first chunks' records, clearing the flags of the others
    const auto prep = a.fuse ? kda_prep_kernel<true> : kda_prep_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(prep, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    SplitParams s1 = sp;
    s1.tasks = first;
    s1.flag_from = first;
    s1.flag_to = total;
    const long long grid_p = first < 2LL * num_sms() ? first : 2LL * num_sms();
    prep<<<(unsigned)grid_p, NT, P_SMEM_BYTES, a.stream>>>(mq, mk, mv, mg, s1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the chains, and the last chunks' records beside them
    const void *tail = tail_kernel_for(a);
    TailParams tp{};
    tp.sp = sp;
    tp.sp.tasks = total;
    tp.first = first;
    tp.nchain = a.H;
    void *args[] = {&mq, &mk, &mv, &mg, &mo, &tp};
    return cudaLaunchCooperativeKernel(tail, dim3(num_sms()), dim3(2 * NT), args, TAIL_SMEM, a.stream);
}

cudaError_t launch_prefill_split(const PrefillArgs &a) {
    if (a.num_units == 0) return cudaSuccess;
    const size_t tokens = a.cu_seqlens ? (size_t)a.T : (size_t)a.B * (size_t)a.T;
    if (tokens == 0) return launch_prefill_simt(a);
    if (tail_ok(a) && tail_launchable(a)) return launch_split_tail(a);
    SplitRecords r;
    cudaError_t e = launch_split_records(a, &r);
    if (e != cudaSuccess) return e;
    return launch_split_chain(a, r);
}

}  // namespace kda
