// Segment-parallel prefill: the KCP pair of every segment, a scan over the
// pairs, and a replay of every segment from its true incoming state
// ("Exercices", Q21-Q22: a segment maps an incoming state S to M S + S~, and
// pairs compose as (M2, S~2) o (M1, S~1) = (M2 M1, M2 S~1 + S~2); the pages'
// check script applies the same scan to a sequence split over 4 ranks).
//
// A long sequence with few heads has few (sequence, head) units, so the plain
// prefill leaves most SMs idle while each unit walks its chunks in order. Here
// each sequence is cut into segments of seg_len tokens that run as independent
// units in three passes over the tokens:
//   pass A  M_p  = the segment's transition: the prefill recurrence run from
//                  S = I with all values v = 0 (then S_out = M_p I + 0);
//   pass B  S~_p = the segment's local state: the recurrence run from S = 0;
//   scan    S_in,0 = S0, S_in,p+1 = M_p S_in,p + S~_p (fp32, one CTA per
//           (sequence, head), sequential over segments; the last one is S_T);
//   pass C  the recurrence run over every segment from S_in,p, writing o.
// On the tensor-core shapes (bf16, dk = dv = 128, chunks of 64) with at most three
// (segment, head) units per SM, the state-independent part of every chunk is computed
// once, as the split prefill's records, and passes A-C are three runs of its
// state-chain kernel over them (pass A leaves the records' Ut out); elsewhere passes
// A-C are the ordinary prefill kernels over the segments laid out as packed sequences.
// Packed batches (cu_seqlens) are planned on the device: every sequence is cut into
// max(1, ceil(len / seg_len)) segments and the scan walks each sequence's own count. M_p is a dk x dk matrix kept in the state layout
// ([column][dk], so pass A runs with dv = dk).
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

constexpr int kSegThreads = 256;

// cu_seg[u] for the B * P segments of a dense batch (segment p of sequence b is unit b * P + p;
// cu_seg null: none) and the identity as the starting "state" of pass A, [units, H, dk, dk] in
// the state layout.
__global__ void kda_segment_init_kernel(int32_t *cu_seg, float *Mbuf, int units, int B, int T, int P,
                                        int seg_len, int H, int dk) {
    const size_t gid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t u = gid; cu_seg && u <= (size_t)units; u += stride) {
        if (u == (size_t)units) {
            cu_seg[u] = B * T;
        } else {
            const int b = (int)(u / P), p = (int)(u % P);
            cu_seg[u] = b * T + p * seg_len;
        }
    }
    const size_t n = (size_t)units * H * dk * dk;
    for (size_t i = gid; i < n; i += stride) {
        const size_t e = i % ((size_t)dk * dk);
        Mbuf[i] = (e / dk == e % dk) ? 1.f : 0.f;
    }
}

// The segments of a packed batch (one block): sequence n of length len_n gets
// P_n = max(1, ceil(len_n / seg_len)) segments, seg_base[n] = sum of P_m over m < n, and
// segment p of it starts at cu[n] + p seg_len (the last ends at cu[n + 1]; an empty sequence is
// one empty segment). The units past the last segment, up to `units`, are empty segments at the
// end of the token axis. units >= seg_base[num] holds because P_n <= len_n / seg_len + 1.
__global__ void kda_segment_plan_kernel(const int32_t *cu, int num, int seg_len, int units, int32_t *seg_base,
                                        int32_t *cu_seg) {
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
            v = len > seg_len ? (len + seg_len - 1) / seg_len : 1;
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
        if (i < num) {  // clamped to the slots, should offsets past the token count ever arrive
            const int first = min(incl - v, units), last = min(incl, units);
            seg_base[i] = first;
            for (int u = first; u < last; ++u) cu_seg[u] = cu[i] + (u - first) * seg_len;
        }
        __syncthreads();
        if (tid == blockDim.x - 1) carry_s = incl;
        __syncthreads();
    }
    const int used = min(carry_s, units);
    if (tid == 0) seg_base[num] = used;
    for (int u = used + tid; u <= units; u += blockDim.x) cu_seg[u] = cu[num];
}

// Rows of the stored state (X[j][i] = S[i][j], [dv][dk]) evolve independently through
// S <- M S + S~ (M acts on the dk index): in the stored layout X <- X Ms + Zs with
// Ms[a][i] = M[i][a]. So one CTA per (sequence b, head h, block of kRowsPerCta rows)
// runs the whole scan for its rows: X <- S0 rows (or 0); for p = 0..P-1 { Sin[p] = X;
// X = X Ms_p + Zs_p }; S_T = X. fp32. Thread (r, ci) owns row r of the block and the
// columns ci + 32 c, so a warp's reads of Ms are consecutive and of X a broadcast.
// Blocks of 8 rows: 128 CTAs for 8 heads x 128 rows.
constexpr int kRowsPerCta = 8;
constexpr int kScanTpr = kSegThreads / kRowsPerCta;  // threads per row (32)

// The steps of a scan are sequential, so each step's transition Ms_p (DK x DK) and this
// CTA's rows of Zs_p are brought into shared memory two steps ahead by bulk copies (two
// buffers, one mbarrier each; no tensor map, no multicast): the copies of steps p + 1 and
// p + 2 are in flight while step p computes. The waits are bounded; a timeout sets
// KDA_ERR_TIMEOUT in the status word and the CTA stops (its copies in flight land first).
constexpr long long kScanWaitCycles = 2000000000LL;  // ~1 s at 2 GHz

template <int DK, int DV>
__global__ void __launch_bounds__(kSegThreads)
kda_kcp_scan_kernel(const float *S0, const float *Mbuf, const float *Zbuf, float *Sin, float *ST, int P, int H,
                    const int32_t *seg_base, int *dev_status) {
    using namespace sm100;
    constexpr int TI = DK / kScanTpr;                // columns per thread
    constexpr int RPI = kSegThreads / kScanTpr;      // rows covered per pass of the threads (8)
    constexpr int RP = kRowsPerCta / RPI;            // rows per thread (1)
    static_assert(TI >= 1 && RP == 1, "scan thread mapping");
    constexpr uint32_t kMBytes = DK * DK * sizeof(float), kZBytes = kRowsPerCta * DK * sizeof(float);
    extern __shared__ __align__(16) float smem[];
    float *Xs = smem;                                // [kRowsPerCta][DK]
    float *Ms = Xs + kRowsPerCta * DK;               // 2 x [DK][DK]
    float *Zs = Ms + 2 * DK * DK;                    // 2 x [kRowsPerCta][DK]
    uint64_t *bar = reinterpret_cast<uint64_t *>(Zs + 2 * kRowsPerCta * DK);
    const int b = blockIdx.x / H, h = blockIdx.x % H, j0 = blockIdx.y * kRowsPerCta, tid = threadIdx.x;
    const int r0 = tid / kScanTpr, ci = tid % kScanTpr;
    const size_t sbase = (((size_t)b * H + h) * DV + j0) * DK;
    // this sequence's segments: units u0 .. u0 + P - 1
    const size_t u0 = seg_base ? (size_t)seg_base[b] : (size_t)b * P;
    if (seg_base) P = seg_base[b + 1] - seg_base[b];
    auto fetch = [&](int p) {  // step p's Ms and Zs rows -> buffer p & 1 (one thread)
        const size_t u = u0 + p;
        const int buf = p & 1;
        mbar_arrive_expect_tx(&bar[buf], kMBytes + kZBytes);
        bulk_load(Ms + buf * DK * DK, Mbuf + (u * H + h) * DK * DK, kMBytes, &bar[buf]);
        bulk_load(Zs + buf * kRowsPerCta * DK, Zbuf + ((u * H + h) * DV + j0) * DK, kZBytes, &bar[buf]);
    };
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
        for (int p = 0; p < 2 && p < P; ++p) fetch(p);
    }
    for (int e = tid; e < kRowsPerCta * DK; e += kSegThreads) Xs[e] = S0 ? S0[sbase + e] : 0.f;
    __syncthreads();
    int p = 0;
    bool ok = true;
    for (; p < P; ++p) {
        const int buf = p & 1;
        const bool got = mbar_wait_bounded(&bar[buf], (uint32_t)(p >> 1) & 1u, kScanWaitCycles);
        if (__syncthreads_or(!got)) { ok = false; break; }
        const float *M = Ms + buf * DK * DK, *Z = Zs + buf * kRowsPerCta * DK;
        const size_t xbase = (((u0 + p) * H + h) * DV + j0) * DK;
        for (int e = tid; e < kRowsPerCta * DK; e += kSegThreads) Sin[xbase + e] = Xs[e];
        float acc[RP][TI];
#pragma unroll
        for (int rr = 0; rr < RP; ++rr)
#pragma unroll
            for (int c = 0; c < TI; ++c) acc[rr][c] = Z[(r0 + RPI * rr) * DK + ci + kScanTpr * c];
#pragma unroll 8
        for (int a = 0; a < DK; ++a) {
            float mv[TI];
#pragma unroll
            for (int c = 0; c < TI; ++c) mv[c] = M[a * DK + ci + kScanTpr * c];
#pragma unroll
            for (int rr = 0; rr < RP; ++rr) {
                const float xv = Xs[(r0 + RPI * rr) * DK + a];
#pragma unroll
                for (int c = 0; c < TI; ++c) acc[rr][c] = fmaf(xv, mv[c], acc[rr][c]);
            }
        }
        __syncthreads();  // every thread has read X and this step's buffer
        if (tid == 0 && p + 2 < P) {
            fence_proxy_async_smem();
            fetch(p + 2);
        }
#pragma unroll
        for (int rr = 0; rr < RP; ++rr)
#pragma unroll
            for (int c = 0; c < TI; ++c) Xs[(r0 + RPI * rr) * DK + ci + kScanTpr * c] = acc[rr][c];
        __syncthreads();
    }
    if (!ok) {
        if (tid == 0) {
            if (dev_status) atomicExch(dev_status, (int)KDA_ERR_TIMEOUT);
            const int issued = p + 2 < P ? p + 2 : P;  // steps p .. issued - 1 may be in flight
            for (int i = p; i < issued; ++i) mbar_wait_bounded(&bar[i & 1], (uint32_t)(i >> 1) & 1u, kScanWaitCycles);
        }
        return;
    }
    if (ST)
        for (int e = tid; e < kRowsPerCta * DK; e += kSegThreads) ST[sbase + e] = Xs[e];
}

template <int DK, int DV>
cudaError_t launch_scan_t(const SegmentedArgs &s, const float *Mbuf, const float *Zbuf, float *Sin,
                          const int32_t *seg_base) {
    const size_t smem = (size_t)(kRowsPerCta * DK + 2 * DK * DK + 2 * kRowsPerCta * DK) * sizeof(float) + 16;
    cudaError_t e = cudaFuncSetAttribute(kda_kcp_scan_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(s.B * s.H), DV / kRowsPerCta);
    kda_kcp_scan_kernel<DK, DV><<<grid, kSegThreads, smem, s.stream>>>(s.S0, Mbuf, Zbuf, Sin, s.ST, s.P, s.H,
                                                                      seg_base, s.dev_status);
    return cudaGetLastError();
}

template <int DK>
cudaError_t launch_scan_dv(const SegmentedArgs &s, const float *Mbuf, const float *Zbuf, float *Sin,
                           const int32_t *seg_base) {
    switch (s.dv) {
        case 32: return launch_scan_t<DK, 32>(s, Mbuf, Zbuf, Sin, seg_base);
        case 64: return launch_scan_t<DK, 64>(s, Mbuf, Zbuf, Sin, seg_base);
        case 128: return launch_scan_t<DK, 128>(s, Mbuf, Zbuf, Sin, seg_base);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_scan(const SegmentedArgs &s, const float *Mbuf, const float *Zbuf, float *Sin,
                        const int32_t *seg_base) {
    switch (s.dk) {
        case 32: return launch_scan_dv<32>(s, Mbuf, Zbuf, Sin, seg_base);
        case 64: return launch_scan_dv<64>(s, Mbuf, Zbuf, Sin, seg_base);
        case 128: return launch_scan_dv<128>(s, Mbuf, Zbuf, Sin, seg_base);
        default: return cudaErrorInvalidValue;
    }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Tokens on the flat axis: B dense sequences of T, or the T tokens of a packed batch.
long long seg_tokens(const SegmentedArgs &s) { return s.cu_seqlens ? (long long)s.T : (long long)s.B * s.T; }

// The segments of the B sequences as one packed batch (cu_seqlens filled on the device).
PrefillArgs segments_as_packed(const SegmentedArgs &s, const int32_t *cu_seg) {
    PrefillArgs a{};
    a.q = s.q; a.k = s.k; a.v = s.v; a.g = s.g; a.beta = s.beta;
    a.cu_seqlens = cu_seg;
    a.B = 1; a.T = (int)seg_tokens(s); a.H = s.H; a.dk = s.dk; a.dv = s.dv; a.chunk = s.chunk; a.dtype = s.dtype;
    a.num_units = s.units;
    a.dev_status = s.dev_status; a.stream = s.stream;
    return a;
}

// Whether passes A-C run on the split prefill's records: both tensor-core shapes, and no more
// (segment, head) units than three per SM (beyond that the single-kernel passes keep every SM
// busy on their own and the records would only add their traffic, as in kda_forward's choice).
bool records_path(const SegmentedArgs &s) {
    return prefill_tc_supported(s.dk, s.dk, s.chunk, s.dtype) && prefill_tc_supported(s.dk, s.dv, s.chunk, s.dtype) &&
           (long long)s.units * s.H <= 3LL * device_sm_count();
}

// Workspace carve-up (all pieces 256-byte aligned): segment offsets (and, for packed batches,
// each sequence's first segment), the longest-first schedule, M, S~ and S_in of every
// (segment, head), and the records where they are used.
struct SegLayout {
    size_t cu, base, order, M, Z, Sin, rec, total;
};
SegLayout seg_layout(const SegmentedArgs &s) {
    const size_t units = (size_t)s.units;
    SegLayout L;
    L.cu = 0;
    L.base = L.cu + align256((units + 1) * sizeof(int32_t));
    L.order = L.base + (s.cu_seqlens ? align256(((size_t)s.B + 1) * sizeof(int32_t)) : 0);
    L.M = L.order + seq_order_bytes((int)units);
    L.Z = L.M + align256(units * s.H * s.dk * s.dk * sizeof(float));
    L.Sin = L.Z + align256(units * s.H * s.dv * s.dk * sizeof(float));
    L.rec = L.Sin + align256(units * s.H * s.dv * s.dk * sizeof(float));
    L.total = L.rec;
    if (records_path(s)) {
        static const int32_t marker = 0;  // compared against null only
        L.total += align256(prefill_split_workspace(segments_as_packed(s, &marker)));
    }
    return L;
}

cudaError_t run_pass(const PrefillArgs &a, bool tc) { return tc ? launch_prefill_tc(a) : launch_prefill_simt(a); }

}  // namespace

size_t segmented_workspace(const SegmentedArgs &s) {
    return s.cu_seqlens == nullptr && s.P <= 1 ? 0 : seg_layout(s).total;
}

cudaError_t launch_kcp_scan(const SegmentedArgs &s, const float *Mbuf, const float *Zbuf, float *Sin,
                            const int32_t *seg_base) {
    return launch_scan(s, Mbuf, Zbuf, Sin, seg_base);
}

cudaError_t launch_segment_pair(const SegmentedArgs &s, float *M, float *Z, bool tc_pair, bool tc_state) {
    // identity start for the transition pass (no offsets needed: one segment per sequence)
    kda_segment_init_kernel<<<296, kSegThreads, 0, s.stream>>>(nullptr, M, s.B, s.B, s.T, 1, s.T, s.H, s.dk);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    PrefillArgs a{};
    a.q = s.q; a.k = s.k; a.g = s.g; a.beta = s.beta;
    a.B = s.B; a.T = s.T; a.H = s.H; a.dk = s.dk; a.chunk = s.chunk; a.dtype = s.dtype;
    a.num_units = s.B; a.dev_status = s.dev_status; a.stream = s.stream;
    PrefillArgs pa = a;
    pa.v = nullptr; pa.o = nullptr; pa.S0 = M; pa.ST = M; pa.dv = s.dk;
    if ((e = run_pass(pa, tc_pair)) != cudaSuccess) return e;
    PrefillArgs pb = a;
    pb.v = s.v; pb.o = nullptr; pb.S0 = nullptr; pb.ST = Z; pb.dv = s.dv;
    return run_pass(pb, tc_state);
}

int segmented_launches(const SegmentedArgs &s) {
    const int order = seq_order_bytes(s.units) > 0 ? 1 : 0;
    const int init = s.cu_seqlens ? 2 : 1;  // (segment plan +) identity start
    if (records_path(s))  // init, chunk offsets (+ schedule), records, three chain passes, scan
        return init + 1 + order + 1 + 3 + 1;
    return init + 3 * (1 + order) /* passes A, B, C */ + 1 /* scan */;
}

cudaError_t launch_segmented(const SegmentedArgs &s, bool tc_pair, bool tc_state) {
    const SegLayout L = seg_layout(s);
    uint8_t *ws = static_cast<uint8_t *>(s.workspace);
    int32_t *cu_seg = reinterpret_cast<int32_t *>(ws + L.cu);
    int32_t *seg_base = s.cu_seqlens ? reinterpret_cast<int32_t *>(ws + L.base) : nullptr;
    float *Mbuf = reinterpret_cast<float *>(ws + L.M);
    float *Zbuf = reinterpret_cast<float *>(ws + L.Z);
    float *Sin = reinterpret_cast<float *>(ws + L.Sin);
    const int units = s.units;

    if (s.cu_seqlens) {
        kda_segment_plan_kernel<<<1, 1024, 0, s.stream>>>(s.cu_seqlens, s.B, s.seg_len, units, seg_base, cu_seg);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    kda_segment_init_kernel<<<296, kSegThreads, 0, s.stream>>>(s.cu_seqlens ? nullptr : cu_seg, Mbuf, units, s.B,
                                                               s.T, s.P, s.seg_len, s.H, s.dk);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    if (records_path(s)) {
        PrefillArgs a = segments_as_packed(s, cu_seg);
        a.workspace = ws + L.rec;
        a.workspace_bytes = L.total - L.rec;
        SplitRecords r;
        if ((e = launch_split_records(a, &r)) != cudaSuccess) return e;
        // pass A: M_p from the identity with zero values; pass B: S~_p from zero
        PrefillArgs pa = a;
        pa.v = nullptr; pa.o = nullptr; pa.S0 = Mbuf; pa.ST = Mbuf; pa.dv = s.dk;
        if ((e = launch_split_chain(pa, r)) != cudaSuccess) return e;
        PrefillArgs pb = a;
        pb.o = nullptr; pb.S0 = nullptr; pb.ST = Zbuf;
        if ((e = launch_split_chain(pb, r)) != cudaSuccess) return e;
        if ((e = launch_scan(s, Mbuf, Zbuf, Sin, seg_base)) != cudaSuccess) return e;
        // pass C: outputs, every segment from its incoming state
        PrefillArgs pc = a;
        pc.o = s.o; pc.S0 = Sin; pc.ST = nullptr;
        return launch_split_chain(pc, r);
    }

    PrefillArgs a{};
    a.q = s.q; a.k = s.k; a.g = s.g; a.beta = s.beta;
    a.cu_seqlens = cu_seg;
    a.B = 1; a.T = (int)seg_tokens(s); a.H = s.H; a.dk = s.dk; a.chunk = s.chunk; a.dtype = s.dtype;
    a.num_units = units;
    a.workspace = ws + L.order; a.workspace_bytes = seq_order_bytes(units);
    a.dev_status = s.dev_status; a.stream = s.stream;

    // pass A: M_p, from the identity with zero values (dv = dk: M_p is dk x dk)
    PrefillArgs pa = a;
    pa.v = nullptr; pa.o = nullptr; pa.S0 = Mbuf; pa.ST = Mbuf; pa.dv = s.dk;
    if ((e = run_pass(pa, tc_pair)) != cudaSuccess) return e;
    // pass B: S~_p, from zero
    PrefillArgs pb = a;
    pb.v = s.v; pb.o = nullptr; pb.S0 = nullptr; pb.ST = Zbuf; pb.dv = s.dv;
    if ((e = run_pass(pb, tc_state)) != cudaSuccess) return e;
    // scan: incoming state of every segment, and S_T
    if ((e = launch_scan(s, Mbuf, Zbuf, Sin, seg_base)) != cudaSuccess) return e;
    // pass C: outputs, every segment from its incoming state
    PrefillArgs pc = a;
    pc.v = s.v; pc.o = s.o; pc.S0 = Sin; pc.ST = nullptr; pc.dv = s.dv;
    return run_pass(pc, tc_state);
}

}  // namespace kda
