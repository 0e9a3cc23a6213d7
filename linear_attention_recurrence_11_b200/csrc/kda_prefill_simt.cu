// Chunked KDA prefill on CUDA cores (fp32 arithmetic, fp32 or bf16 storage).
//
// One CTA owns one (sequence, head, 32-wide block of dv columns) unit and walks
// its chunks in order. The dv columns of S evolve independently (the
// recurrence acts on S from the left only), so splitting dv is exact; the
// dk-side work of a chunk (decayed Grams, triangular solve for W) is
// recomputed by each dv block.
//
// Per chunk of C tokens (zero-padded past the sequence end, which leaves the
// state and the stored outputs unchanged), with G the per-channel cumulative
// log-decay from the chunk start and Gamma = exp(G):
//   A_rs = beta_r sum_c k_rc k_sc exp(G_rc - G_sc)  (s < r)
//   P_rs = sum_c q_rc k_sc exp(G_rc - G_sc)         (s <= r)
//   (I + A) W  = Diag(beta) (Gamma * K)      (forward substitution)
//   (I + A) Ut = Diag(beta) V
//   U = Ut - W S,  O = (Gamma * Q) S + P U,  S <- Diag(Gamma_C) S + Kh^T U,
//   Kh_s = exp(G_C - G_s) * k_s.
// This is the chunked form of S_t = (I - b k k^T) Diag(e^g) S + b k v^T
// ("Exercices", Q7) with the chunk's KCP pair (Diag(Gamma_C) - Kh^T W, Kh^T Ut)
// applied to the incoming state ("Exercices", Q21-Q22). Every exponent here is
// a pairwise difference <= 0, so nothing overflows.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kDVB = 32;  // dv columns per CTA

template <int DK, int C>
struct SimtSmem {
    static constexpr int KP = DK + 1;   // padded row of a C x DK tile
    static constexpr int CP = C + 1;    // padded row of a C x C tile
    static constexpr int UP = kDVB + 1; // padded row of a C x DVB / DK x DVB tile
    static constexpr int floats = 4 * C * KP + 2 * C * CP + C * UP + DK * UP + C + DK;
    static constexpr size_t bytes = sizeof(float) * (size_t)floats;
};

template <typename Tin, int DK, int C>
__global__ void __launch_bounds__(kThreads, 1) kda_prefill_simt_kernel(const PrefillArgs p) {
    using L = SimtSmem<DK, C>;
    constexpr int KP = L::KP, CP = L::CP, UP = L::UP, DVB = kDVB;
    extern __shared__ float smem[];
    float *sQ = smem;            // C x KP: q, then Gamma * q
    float *sK = sQ + C * KP;     // C x KP: k, then Kh
    float *sG = sK + C * KP;     // C x KP: g, then cumulative G
    float *sW = sG + C * KP;     // C x KP: W
    float *sA = sW + C * KP;     // C x CP
    float *sP = sA + C * CP;     // C x CP
    float *sU = sP + C * CP;     // C x UP: v, then Ut, then U
    float *sS = sU + C * UP;     // DK x UP: state block S[i][j]
    float *sB = sS + DK * UP;    // C: beta
    float *sGam = sB + C;        // DK: Gamma_C

    const Tin *q = static_cast<const Tin *>(p.q), *k = static_cast<const Tin *>(p.k);
    const Tin *v = static_cast<const Tin *>(p.v), *g = static_cast<const Tin *>(p.g);
    const Tin *beta = static_cast<const Tin *>(p.beta);
    Tin *o = static_cast<Tin *>(p.o);
    const int tid = threadIdx.x;
    const int nblk = p.dv / DVB;
    const int dvb = blockIdx.x % nblk;
    const int h = (blockIdx.x / nblk) % p.H;
    const int n = unit_seq(p, blockIdx.x / (nblk * p.H));
    const size_t H = (size_t)p.H, dv = (size_t)p.dv;
    size_t t_begin, len;
    if (p.cu_seqlens) {
        t_begin = (size_t)p.cu_seqlens[n];
        len = (size_t)(p.cu_seqlens[n + 1] - p.cu_seqlens[n]);
    } else {
        t_begin = (size_t)n * p.T;
        len = (size_t)p.T;
    }
    const int j0 = dvb * DVB;
    const size_t sbase = (((size_t)n * H + h) * dv + j0) * DK;

    for (int idx = tid; idx < DK * DVB; idx += kThreads) {
        const int j = idx / DK, i = idx % DK;
        sS[i * UP + j] = p.S0 ? p.S0[sbase + (size_t)j * DK + i] : 0.f;
    }
    // (the loop below starts with a barrier-protected load phase)

    for (size_t c0 = 0; c0 < len; c0 += C) {
        const int Lc = (int)((len - c0) < (size_t)C ? (len - c0) : (size_t)C);
        __syncthreads();
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int r = idx / DK, i = idx % DK;
            float qv = 0.f, kv = 0.f, gv = 0.f;
            if (r < Lc) {
                const size_t off = ((t_begin + c0 + r) * H + h) * DK + i;
                qv = ld_elem(q, off);
                kv = ld_elem(k, off);
                gv = ld_elem(g, off);
            }
            sQ[r * KP + i] = qv;
            sK[r * KP + i] = kv;
            sG[r * KP + i] = gv;
        }
        for (int idx = tid; idx < C * DVB; idx += kThreads) {
            const int r = idx / DVB, j = idx % DVB;
            sU[r * UP + j] = (r < Lc && v) ? ld_elem(v, ((t_begin + c0 + r) * H + h) * dv + j0 + j) : 0.f;
        }
        for (int r = tid; r < C; r += kThreads)
            sB[r] = (r < Lc) ? ld_elem(beta, (t_begin + c0 + r) * H + h) : 0.f;
        __syncthreads();
        if (p.fuse) {  // fused pre-ops: g from gate logits, q and k normalised per row
            if (p.fuse & KDA_FUSE_GATE_LOGITS)
                for (int idx = tid; idx < Lc * DK; idx += kThreads) {
                    const int r = idx / DK, i = idx % DK;
                    sG[r * KP + i] = gate_from_logit(sG[r * KP + i]);
                }
            if (p.fuse & KDA_FUSE_NORM_QK) {
                const int lane = tid & 31, w = tid >> 5;
                for (int r = w; r < Lc; r += kThreads / 32) {
                    float sk = 0.f, sq = 0.f;
                    for (int i = lane; i < DK; i += 32) {
                        sk = fmaf(sK[r * KP + i], sK[r * KP + i], sk);
                        sq = fmaf(sQ[r * KP + i], sQ[r * KP + i], sq);
                    }
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) {
                        sk += __shfl_xor_sync(0xffffffffu, sk, off);
                        sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    }
                    const float ik = sk > 0.f ? rsqrtf(sk) : 0.f, iq = sq > 0.f ? rsqrtf(sq) : 0.f;
                    for (int i = lane; i < DK; i += 32) {
                        sK[r * KP + i] *= ik;
                        sQ[r * KP + i] *= iq;
                    }
                }
            }
            __syncthreads();
        }

        // cumulative log-decay over the chunk, per channel
        for (int i = tid; i < DK; i += kThreads) {
            float acc = 0.f;
            for (int r = 0; r < C; ++r) {
                acc += sG[r * KP + i];
                sG[r * KP + i] = acc;
            }
            sGam[i] = __expf(acc);
        }
        __syncthreads();

        // decayed Grams A (strictly lower, times beta_r) and P (lower)
        for (int idx = tid; idx < C * C; idx += kThreads) {
            const int r = idx / C, s = idx % C;
            float a = 0.f, pp = 0.f;
            if (s <= r) {
#pragma unroll 8
                for (int i = 0; i < DK; ++i) {
                    const float ks = sK[s * KP + i] * __expf(sG[r * KP + i] - sG[s * KP + i]);
                    a = fmaf(sK[r * KP + i], ks, a);
                    pp = fmaf(sQ[r * KP + i], ks, pp);
                }
            }
            sA[r * CP + s] = (s < r) ? sB[r] * a : 0.f;
            sP[r * CP + s] = pp;
        }
        __syncthreads();

        // right-hand side of W, and Gamma * q
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int r = idx / DK, i = idx % DK;
            const float gam = __expf(sG[r * KP + i]);
            sW[r * KP + i] = sB[r] * gam * sK[r * KP + i];
            sQ[r * KP + i] *= gam;
        }
        __syncthreads();

        // forward substitution with I + A, one column per thread (W and Ut)
        for (int col = tid; col < DK + DVB; col += kThreads) {
            float *X;
            int ldx;
            bool isU = col >= DK;
            if (!isU) { X = sW + col; ldx = KP; }
            else { X = sU + (col - DK); ldx = UP; }
            for (int r = 0; r < C; ++r) {
                float x = X[r * ldx];
                if (isU) x *= sB[r];
                for (int s = 0; s < r; ++s) x = fmaf(-sA[r * CP + s], X[s * ldx], x);
                X[r * ldx] = x;
            }
        }
        __syncthreads();

        // Kh = exp(G_C - G_s) * k_s, in place
        for (int idx = tid; idx < C * DK; idx += kThreads) {
            const int s = idx / DK, i = idx % DK;
            sK[s * KP + i] *= __expf(sG[(C - 1) * KP + i] - sG[s * KP + i]);
        }
        // U = Ut - W S (in place, each thread owns its elements)
        {
            const int j = tid % DVB, r0 = tid / DVB;
            constexpr int RS = kThreads / DVB;  // row stride
            for (int r = r0; r < C; r += RS) {
                float acc = 0.f;
#pragma unroll 8
                for (int i = 0; i < DK; ++i) acc = fmaf(sW[r * KP + i], sS[i * UP + j], acc);
                sU[r * UP + j] -= acc;
            }
        }
        __syncthreads();

        // O = (Gamma * Q) S + P U, rows < Lc stored (no outputs when o is null)
        if (o) {
            const int j = tid % DVB, r0 = tid / DVB;
            constexpr int RS = kThreads / DVB;
            for (int r = r0; r < Lc; r += RS) {
                float acc = 0.f;
#pragma unroll 8
                for (int i = 0; i < DK; ++i) acc = fmaf(sQ[r * KP + i], sS[i * UP + j], acc);
                for (int s = 0; s <= r; ++s) acc = fmaf(sP[r * CP + s], sU[s * UP + j], acc);
                st_elem(o, ((t_begin + c0 + r) * H + h) * dv + j0 + j, acc);
            }
        }
        __syncthreads();

        // S <- Diag(Gamma_C) S + Kh^T U
        {
            const int j = tid % DVB, i0 = tid / DVB;
            constexpr int IS = kThreads / DVB;
            for (int i = i0; i < DK; i += IS) {
                float acc = sGam[i] * sS[i * UP + j];
#pragma unroll 8
                for (int s = 0; s < C; ++s) acc = fmaf(sK[s * KP + i], sU[s * UP + j], acc);
                sS[i * UP + j] = acc;
            }
        }
        // a snapshot of the state after this chunk (fp32, the S0 layout of one sequence)
        if (p.snap_every && Lc == C && (c0 + C) % (size_t)p.snap_every == 0) {
            __syncthreads();
            const size_t nsnap = (size_t)p.T / p.snap_every, ps = (c0 + C) / p.snap_every - 1;
            float *dst = p.S_snap + (((size_t)n * nsnap + ps) * H + h) * dv * DK + (size_t)j0 * DK;
            for (int idx = tid; idx < DK * DVB; idx += kThreads) {
                const int j = idx / DK, i = idx % DK;
                dst[(size_t)j * DK + i] = sS[i * UP + j];
            }
        }
    }
    __syncthreads();
    if (p.ST)
        for (int idx = tid; idx < DK * DVB; idx += kThreads) {
            const int j = idx / DK, i = idx % DK;
            p.ST[sbase + (size_t)j * DK + i] = sS[i * UP + j];
        }
}

template <typename Tin, int DK, int C>
cudaError_t launch_typed(const PrefillArgs &a) {
    auto kern = kda_prefill_simt_kernel<Tin, DK, C>;
    const size_t smem = SimtSmem<DK, C>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)a.num_units * a.H * (a.dv / kDVB));
    kern<<<grid, kThreads, smem, a.stream>>>(a);
    return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t launch_dk(const PrefillArgs &a) {
    switch (a.chunk) {
        case 16: return launch_typed<Tin, DK, 16>(a);
        case 32: return launch_typed<Tin, DK, 32>(a);
        case 64: return launch_typed<Tin, DK, 64>(a);
        default: return cudaErrorInvalidValue;
    }
}

template <typename Tin>
cudaError_t launch_dtype(const PrefillArgs &a) {
    switch (a.dk) {
        case 32: return launch_dk<Tin, 32>(a);
        case 64: return launch_dk<Tin, 64>(a);
        case 128: return launch_dk<Tin, 128>(a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillArgs &a_in) {
    if (a_in.num_units == 0 || a_in.H == 0) return cudaSuccess;
    PrefillArgs a = a_in;
    if (a.cu_seqlens && seq_order_bytes(a.num_units) > 0) {
        int32_t *order = static_cast<int32_t *>(a.workspace);
        const cudaError_t e = launch_seq_order(a.cu_seqlens, a.num_units, order, a.stream);
        if (e != cudaSuccess) return e;
        a.seq_order = order;
    }
    return a.dtype == KDA_DTYPE_BF16 ? launch_dtype<__nv_bfloat16>(a) : launch_dtype<float>(a);
}

size_t prefill_simt_workspace(const PrefillArgs &a) { return a.cu_seqlens ? seq_order_bytes(a.num_units) : 0; }

int prefill_simt_launches(const PrefillArgs &a) {
    if (a.num_units <= 0 || a.H <= 0) return 0;
    return 1 + ((a.cu_seqlens && seq_order_bytes(a.num_units) > 0) ? 1 : 0);
}

}  // namespace kda
