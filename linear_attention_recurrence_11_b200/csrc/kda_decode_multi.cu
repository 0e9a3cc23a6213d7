// Multi-token decode with speculative acceptance ("Exercices", Q27: the state
// after any accepted prefix of draft tokens is determined by those tokens'
// inputs, which are far smaller than the state; so keep only the inputs,
// replay the recurrence on chip and write back the verified state).
//
// Per (request n, head h): T tokens t = 0..T-1 are applied in order to the
// state S (dk x dv, stored [dv][dk] fp32), each exactly as one decode step
//   S' = Diag(exp g_t) S,  s = S'^T k_t,  u = beta_t (v_t - s),
//   S <- S' + k_t u^T,     o_t = S'^T q_t + u (k_t^T q_t)
// and the state after the first n_acc tokens (n_acc = n_accept[n], or T) is
// written back in place; n_acc = 0 leaves S untouched. Outputs of all T
// tokens are written when o is given. A verification pass is n_accept = all
// zeros (outputs only, S read once and not written); the commit that follows
// is the same call with the accepted counts and o = NULL.
//
// Each state is read from HBM once and written at most once, whatever T is.
// Every column j of S (a contiguous dk-float row of the stored state) evolves
// independently of the others through all T tokens (the decay, both dot
// products and the rank-1 update act column by column). One CTA of 4 warps
// per (request, head) walks the state in passes of 32 columns, each pass one
// contiguous block (32 dk floats) that a bulk copy brings into shared memory:
// two buffers, so the copy of pass p + 1 (and p + 2) is in flight while pass p
// computes. In a pass, 8 lanes cover a column with 128-bit reads and each lane
// holds two columns; all T tokens are applied while the columns are in
// registers and a column goes back to HBM right after token n_acc. The
// tokens' q, k, exp(g), beta and v are staged in shared memory first; outputs
// are collected there and written as contiguous rows at the end. Without
// outputs (o = NULL) only the first n_acc tokens are applied, and a request
// with n_acc = 0 reads nothing.
//
// A verification (outputs of all T tokens, n_acc = 0, T <= kVerifyMaxT) does
// not need the intermediate states at all. With G_t the cumulative log-decay
// up to token t, the decayed state seen by token t is
//   S'_t = Diag(e^{G_t}) S + sum_{tau < t} Diag(e^{G_t - G_tau}) k_tau u_tau^T,
// so per column j of S, with a_t = (e^{G_t} k_t)^T S[:, j] and
// b_t = (e^{G_t} q_t)^T S[:, j],
//   u_t[j] = beta_t (v_t[j] - a_t - sum_{tau < t} A_{t tau} u_tau[j]),
//   o_t[j] = b_t + sum_{tau < t} P_{t tau} u_tau[j] + u_t[j] (k_t^T q_t),
// A_{t tau} = sum_i k_t[i] k_tau[i] e^{G_t[i] - G_tau[i]} and P likewise with
// q_t: the chunked form of the recurrence ("Exercices", Q21-Q22) applied to the
// T draft tokens. Each state element then takes 2T multiply-adds (two dot
// products per token, no dependency between tokens) instead of the four
// operations of a sequential step, and the T x T systems are solved per column
// after the state has streamed through.
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int kMtThreads = 128;
constexpr int kMtLanesPerRow = 8;
constexpr int kMtRowsPerPass = (kMtThreads / 32) * (32 / kMtLanesPerRow);  // 16
constexpr int kMtRowsInFlight = 2;
constexpr int kMtCols = kMtRowsPerPass * kMtRowsInFlight;                  // 32 columns per pass
constexpr long long kMtWaitCycles = 2000000000LL;                          // ~1 s at 2 GHz
constexpr int kVerifyMaxT = 16;  // verifications of up to this many tokens take the chunked form
constexpr int kVerifyGroup = 4;  // tokens per sweep over the columns held in registers
static_assert(kMtRowsInFlight * 2 * kVerifyGroup == 16 && kMtLanesPerRow == 8, "reduce_scatter8 layout");

// 16 bytes of elements -> floats (8 bf16 or 4 fp32)
__device__ __forceinline__ void unpack16(const uint4 &r, float (&x)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void unpack16(const uint4 &r, float (&x)[4]) {
    x[0] = __uint_as_float(r.x); x[1] = __uint_as_float(r.y);
    x[2] = __uint_as_float(r.z); x[3] = __uint_as_float(r.w);
}

// Sums of 16 values over the 8 lanes of a column group (xor 4, 2, 1), scattered: the lane whose
// index in the group has bits b2 b1 b0 ends with the complete sums of entries
// 8 b2 + 4 b1 + 2 b0 + {0, 1} in y[0], y[1] (14 shuffles instead of 48).
__device__ __forceinline__ void reduce_scatter8(const float (&v)[16], float (&y)[2], int sub) {
    const bool u4 = sub & 4, u2 = sub & 2, u1 = sub & 1;
    float w[8], x[4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        w[i] = (u4 ? v[i + 8] : v[i]) + __shfl_xor_sync(0xffffffffu, u4 ? v[i] : v[i + 8], 4);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        x[i] = (u2 ? w[i + 4] : w[i]) + __shfl_xor_sync(0xffffffffu, u2 ? w[i] : w[i + 4], 2);
#pragma unroll
    for (int i = 0; i < 2; ++i)
        y[i] = (u1 ? x[i + 2] : x[i]) + __shfl_xor_sync(0xffffffffu, u1 ? x[i] : x[i + 2], 1);
}

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kMtThreads) kda_decode_multi_kernel(const MultiDecodeArgs p) {
    constexpr int F4 = DK / (4 * kMtLanesPerRow);  // float4 per lane per column
    // per token: q, k, exp(g) [DK each], v [DV], beta, padded to 16 bytes; then the outputs [T][DV]
    constexpr int TOK = 3 * DK + DV + 4;
    constexpr int kPasses = DV / kMtCols;
    constexpr uint32_t kPassBytes = kMtCols * DK * sizeof(float);
    // shared: two pass buffers, two mbarriers (16 bytes), the tokens, the outputs
    extern __shared__ __align__(16) float smem_mt[];
    float *sBuf = smem_mt;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sBuf + 2 * kMtCols * DK);
    float *sIn = reinterpret_cast<float *>(bar + 2);
    const Tin *q = static_cast<const Tin *>(p.q), *k = static_cast<const Tin *>(p.k);
    const Tin *v = static_cast<const Tin *>(p.v), *g = static_cast<const Tin *>(p.g);
    const Tin *beta = static_cast<const Tin *>(p.beta);
    Tin *o = static_cast<Tin *>(p.o);
    const int T = p.T, H = p.H;
    const size_t unit = blockIdx.x;  // n * H + h
    const int n = (int)(unit / H), h = (int)(unit % H);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sub = lane & (kMtLanesPerRow - 1), rw = lane / kMtLanesPerRow;

    int n_acc = p.n_accept ? p.n_accept[n] : T;
    n_acc = n_acc < 0 ? 0 : (n_acc > T ? T : n_acc);
    const int t_end = o ? T : n_acc;  // tokens whose effect is needed
    const bool verify = o != nullptr && n_acc == 0 && T <= kVerifyMaxT;  // the chunked form
    float *Su = p.S + unit * (size_t)DV * DK;
    if (t_end > 0 && tid == 0) {  // the first two passes' columns -> shared memory
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
#pragma unroll
        for (int b = 0; b < 2 && b < kPasses; ++b) {
            mbar_arrive_expect_tx(&bar[b], kPassBytes);
            bulk_load(sBuf + b * kMtCols * DK, Su + (size_t)b * kMtCols * DK, kPassBytes, &bar[b]);
        }
    }
    if (t_end == 0) return;  // nothing to apply, nothing to write

    // the tokens' inputs -> shared memory (input layout [N, T, H, d]): 16-byte pieces of the
    // q, k, g and v rows, four per thread in flight before any is used
    {
        constexpr int VEC = 16 / (int)sizeof(Tin);      // elements per piece
        constexpr int NK = DK / VEC, NVV = DV / VEC;    // pieces per row
        constexpr int PER_TOK = 3 * NK + NVV;
        constexpr int UNR = 4;
        const int total = t_end * PER_TOK;
        for (int base = tid; base < total; base += UNR * kMtThreads) {
            uint4 raw[UNR];
            int dst[UNR];
            bool is_g[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int idx = base + u * kMtThreads;
                if (idx >= total) continue;
                const int t = idx / PER_TOK, c = idx % PER_TOK;
                const size_t tok = ((size_t)n * T + t) * H + h;
                const Tin *src;
                if (c < NK) { src = q + tok * DK + c * VEC; dst[u] = c * VEC; }
                else if (c < 2 * NK) { src = k + tok * DK + (c - NK) * VEC; dst[u] = DK + (c - NK) * VEC; }
                else if (c < 3 * NK) { src = g + tok * DK + (c - 2 * NK) * VEC; dst[u] = 2 * DK + (c - 2 * NK) * VEC; }
                else { src = v + tok * DV + (c - 3 * NK) * VEC; dst[u] = 3 * DK + (c - 3 * NK) * VEC; }
                is_g[u] = c >= 2 * NK && c < 3 * NK;
                dst[u] += t * TOK;
                raw[u] = __ldg(reinterpret_cast<const uint4 *>(src));
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                if (base + u * kMtThreads >= total) continue;
                float x[VEC];
                unpack16(raw[u], x);
                if (is_g[u] && !verify) {  // the chunked form keeps g and sums it
#pragma unroll
                    for (int e = 0; e < VEC; ++e) x[e] = __expf(x[e]);
                }
#pragma unroll
                for (int e = 0; e < VEC; e += 4)
                    *reinterpret_cast<float4 *>(sIn + dst[u] + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
            }
        }
        if (tid < t_end) sIn[tid * TOK + 3 * DK + DV] = ld_elem(beta, ((size_t)n * T + tid) * H + h);
    }
    float *sOut = sIn + T * TOK;  // outputs [T][DV]; the chunked form first keeps b_t there
    float *sA0 = sOut + T * DV;   // chunked form: a_t [T][DV], then A and P [T][T] each
    float *sAm = sA0 + T * DV, *sPm = sAm + T * T;
    __syncthreads();
    if (verify) {
        // G_t (cumulative log-decay, in place of g), then A and P (P_tt = k_t^T q_t), then the
        // decayed e^{G_t} q_t, e^{G_t} k_t in place of q_t, k_t
        for (int i = tid; i < DK; i += kMtThreads) {
            float acc = 0.f;
            for (int t = 0; t < T; ++t) {
                acc += sIn[t * TOK + 2 * DK + i];
                sIn[t * TOK + 2 * DK + i] = acc;
            }
        }
        __syncthreads();
        int pidx = 0;
        for (int t = 0; t < T; ++t) {
            const float *it = sIn + t * TOK;
            for (int tau = 0; tau <= t; ++tau, ++pidx) {
                if ((pidx & 3) != warp) continue;
                const float *iu = sIn + tau * TOK;
                float sa = 0.f, sp = 0.f;
#pragma unroll
                for (int i = lane; i < DK; i += 32) {
                    const float w = tau == t ? iu[DK + i] : iu[DK + i] * __expf(it[2 * DK + i] - iu[2 * DK + i]);
                    sa = fmaf(it[DK + i], w, sa);
                    sp = fmaf(it[i], w, sp);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sa += __shfl_xor_sync(0xffffffffu, sa, off);
                    sp += __shfl_xor_sync(0xffffffffu, sp, off);
                }
                if (lane == 0) {
                    sAm[t * T + tau] = sa;
                    sPm[t * T + tau] = sp;
                }
            }
        }
        __syncthreads();
        for (int idx = tid; idx < T * DK; idx += kMtThreads) {
            const int t = idx / DK, i = idx % DK;
            float *it = sIn + t * TOK;
            const float e = __expf(it[2 * DK + i]);
            it[i] *= e;
            it[DK + i] *= e;
        }
        __syncthreads();
    }

    int pass = 0;
    bool ok = true;
    for (; pass < kPasses; ++pass) {
        const int b = pass & 1;
        const float *buf = sBuf + b * kMtCols * DK;
        const bool got = mbar_wait_bounded(&bar[b], (uint32_t)(pass >> 1) & 1u, kMtWaitCycles);
        float4 s[kMtRowsInFlight][F4];
#pragma unroll
        for (int r = 0; r < kMtRowsInFlight; ++r) {
            const int jl = warp * (32 / kMtLanesPerRow) + rw + r * kMtRowsPerPass;  // column inside the pass
#pragma unroll
            for (int m = 0; m < F4; ++m)
                s[r][m] = *reinterpret_cast<const float4 *>(buf + jl * DK + 4 * (sub + kMtLanesPerRow * m));
        }
        // every thread holds its columns (or a wait gave up): the buffer can be refilled
        if (__syncthreads_or(!got)) { ok = false; break; }
        if (tid == 0 && pass + 2 < kPasses) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bar[b], kPassBytes);
            bulk_load(sBuf + b * kMtCols * DK, Su + (size_t)(pass + 2) * kMtCols * DK, kPassBytes, &bar[b]);
        }
        if (verify) {
            // a_t, b_t of this pass's columns, kVerifyGroup tokens per sweep over the registers
            for (int t0 = 0; t0 < T; t0 += kVerifyGroup) {
                float2 acc[kMtRowsInFlight][2][kVerifyGroup];
#pragma unroll
                for (int r = 0; r < kMtRowsInFlight; ++r)
#pragma unroll
                    for (int w = 0; w < 2; ++w)
#pragma unroll
                        for (int t4 = 0; t4 < kVerifyGroup; ++t4) acc[r][w][t4] = make_float2(0.f, 0.f);
#pragma unroll
                for (int t4 = 0; t4 < kVerifyGroup; ++t4) {
                    if (t0 + t4 >= T) break;
                    const float *in = sIn + (t0 + t4) * TOK;
#pragma unroll
                    for (int m = 0; m < F4; ++m) {
                        const int c = 4 * (sub + kMtLanesPerRow * m);
                        const float4 qd = *reinterpret_cast<const float4 *>(in + c);
                        const float4 kd = *reinterpret_cast<const float4 *>(in + DK + c);
#pragma unroll
                        for (int r = 0; r < kMtRowsInFlight; ++r) {
                            const float2 x0 = make_float2(s[r][m].x, s[r][m].y);
                            const float2 x1 = make_float2(s[r][m].z, s[r][m].w);
                            acc[r][0][t4] = __ffma2_rn(x0, make_float2(kd.x, kd.y), acc[r][0][t4]);
                            acc[r][0][t4] = __ffma2_rn(x1, make_float2(kd.z, kd.w), acc[r][0][t4]);
                            acc[r][1][t4] = __ffma2_rn(x0, make_float2(qd.x, qd.y), acc[r][1][t4]);
                            acc[r][1][t4] = __ffma2_rn(x1, make_float2(qd.z, qd.w), acc[r][1][t4]);
                        }
                    }
                }
                float v16[16];
#pragma unroll
                for (int r = 0; r < kMtRowsInFlight; ++r)
#pragma unroll
                    for (int w = 0; w < 2; ++w)
#pragma unroll
                        for (int t4 = 0; t4 < kVerifyGroup; ++t4)
                            v16[8 * r + 4 * w + t4] = acc[r][w][t4].x + acc[r][w][t4].y;
                float y[2];
                reduce_scatter8(v16, y, sub);
                const int r = (sub >> 2) & 1, w = (sub >> 1) & 1;
                const int j = pass * kMtCols + warp * (32 / kMtLanesPerRow) + rw + r * kMtRowsPerPass;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int t = t0 + 2 * (sub & 1) + i;
                    if (t < T) (w ? sOut : sA0)[t * DV + j] = y[i];
                }
            }
            continue;
        }
        for (int t = 0; t < t_end; ++t) {
            const float *in = sIn + t * TOK;
            // this lane's channels as pairs: the element-wise work runs on the paired fp32
            // pipe (__fmul2_rn / __ffma2_rn: per element the same IEEE operations, in the
            // same order, as scalar code)
            float2 kk[2 * F4], qq[2 * F4], a[2 * F4];
#pragma unroll
            for (int m = 0; m < F4; ++m) {
                const int c = 4 * (sub + kMtLanesPerRow * m);
                const float4 q4 = *reinterpret_cast<const float4 *>(in + c);
                const float4 k4 = *reinterpret_cast<const float4 *>(in + DK + c);
                const float4 a4 = *reinterpret_cast<const float4 *>(in + 2 * DK + c);
                qq[2 * m] = make_float2(q4.x, q4.y); qq[2 * m + 1] = make_float2(q4.z, q4.w);
                kk[2 * m] = make_float2(k4.x, k4.y); kk[2 * m + 1] = make_float2(k4.z, k4.w);
                a[2 * m] = make_float2(a4.x, a4.y); a[2 * m + 1] = make_float2(a4.z, a4.w);
            }
            float kq = 0.f;
#pragma unroll
            for (int e = 0; e < 2 * F4; ++e) {
                kq = fmaf(kk[e].x, qq[e].x, kq);
                kq = fmaf(kk[e].y, qq[e].y, kq);
            }
#pragma unroll
            for (int off = 1; off < kMtLanesPerRow; off <<= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
            const float bt = in[3 * DK + DV];
#pragma unroll
            for (int r = 0; r < kMtRowsInFlight; ++r) {
                const int j = pass * kMtCols + warp * (32 / kMtLanesPerRow) + rw + r * kMtRowsPerPass;
                // the tokens of a column are sequential, so the dot products keep four
                // partial sums each (short dependency chains between tokens)
                float2 pk[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                float2 pq[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                float2 x[2 * F4];
#pragma unroll
                for (int m = 0; m < F4; ++m) {
                    x[2 * m] = make_float2(s[r][m].x, s[r][m].y);
                    x[2 * m + 1] = make_float2(s[r][m].z, s[r][m].w);
                }
#pragma unroll
                for (int e = 0; e < 2 * F4; ++e) {
                    x[e] = __fmul2_rn(x[e], a[e]);
                    pk[e & 1] = __ffma2_rn(x[e], kk[e], pk[e & 1]);
                    pq[e & 1] = __ffma2_rn(x[e], qq[e], pq[e & 1]);
                }
                float sk = (pk[0].x + pk[0].y) + (pk[1].x + pk[1].y);
                float sq = (pq[0].x + pq[0].y) + (pq[1].x + pq[1].y);
#pragma unroll
                for (int off = 1; off < kMtLanesPerRow; off <<= 1) {
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                }
                const float u = bt * (in[3 * DK + j] - sk);
                const float2 uu = make_float2(u, u);
#pragma unroll
                for (int e = 0; e < 2 * F4; ++e) x[e] = __ffma2_rn(kk[e], uu, x[e]);
#pragma unroll
                for (int m = 0; m < F4; ++m) s[r][m] = make_float4(x[2 * m].x, x[2 * m].y, x[2 * m + 1].x, x[2 * m + 1].y);
                if (o && sub == 0) sOut[t * DV + j] = fmaf(u, kq, sq);
            }
            if (t + 1 == n_acc) {  // the column after the accepted prefix, in place
#pragma unroll
                for (int r = 0; r < kMtRowsInFlight; ++r) {
                    const int j = pass * kMtCols + warp * (32 / kMtLanesPerRow) + rw + r * kMtRowsPerPass;
#pragma unroll
                    for (int m = 0; m < F4; ++m)
                        __stcs(reinterpret_cast<float4 *>(Su + (size_t)j * DK + 4 * (sub + kMtLanesPerRow * m)), s[r][m]);
                }
            }
        }
    }
    if (!ok) {
        // a staging copy did not arrive in time: report it, and let the copies still in
        // flight (passes `pass` .. issued - 1) land before the CTA's shared memory is released
        if (tid == 0) {
            if (p.dev_status) atomicExch(p.dev_status, (int)KDA_ERR_TIMEOUT);
            const int issued = pass + 2 < kPasses ? pass + 2 : kPasses;
            for (int i = pass; i < issued; ++i)
                mbar_wait_bounded(&bar[i & 1], (uint32_t)(i >> 1) & 1u, kMtWaitCycles);
        }
        return;
    }
    if (verify) {  // the T x T systems, one column per thread
        __syncthreads();
        for (int j = tid; j < DV; j += kMtThreads) {
            float u[kVerifyMaxT];
#pragma unroll
            for (int t = 0; t < kVerifyMaxT; ++t) {
                if (t >= T) break;
                const float *in = sIn + t * TOK;
                float a = sA0[t * DV + j], b = sOut[t * DV + j];
#pragma unroll
                for (int tau = 0; tau < t; ++tau) {
                    a = fmaf(sAm[t * T + tau], u[tau], a);
                    b = fmaf(sPm[t * T + tau], u[tau], b);
                }
                u[t] = in[3 * DK + DV] * (in[3 * DK + j] - a);
                sOut[t * DV + j] = fmaf(u[t], sPm[t * T + t], b);
            }
        }
    }
    if (o) {  // outputs, one contiguous dv row per token
        __syncthreads();
        for (int idx = tid; idx < T * DV; idx += kMtThreads) {
            const int t = idx / DV, j = idx % DV;
            st_elem(o, (((size_t)n * T + t) * H + h) * DV + j, sOut[idx]);
        }
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_mt(const MultiDecodeArgs &a) {
    const size_t smem = 2 * (size_t)kMtCols * DK * sizeof(float) + 16 +
                        (size_t)a.T * (3 * DK + DV + 4 + DV) * sizeof(float) +
                        (a.T <= kVerifyMaxT ? (size_t)a.T * (DV + 2 * a.T) * sizeof(float) : 0);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kda_decode_multi_kernel<Tin, DK, DV>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kda_decode_multi_kernel<Tin, DK, DV><<<(unsigned)((size_t)a.N * a.H), kMtThreads, smem, a.stream>>>(a);
    return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t launch_mt_dv(const MultiDecodeArgs &a) {
    switch (a.dv) {
        case 32: return launch_mt<Tin, DK, 32>(a);
        case 64: return launch_mt<Tin, DK, 64>(a);
        case 128: return launch_mt<Tin, DK, 128>(a);
        default: return cudaErrorInvalidValue;
    }
}

template <typename Tin>
cudaError_t launch_mt_t(const MultiDecodeArgs &a) {
    switch (a.dk) {
        case 32: return launch_mt_dv<Tin, 32>(a);
        case 64: return launch_mt_dv<Tin, 64>(a);
        case 128: return launch_mt_dv<Tin, 128>(a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode_multi(const MultiDecodeArgs &a) {
    if ((size_t)a.N * a.H == 0 || a.T == 0) return cudaSuccess;
    return a.dtype == KDA_DTYPE_BF16 ? launch_mt_t<__nv_bfloat16>(a) : launch_mt_t<float>(a);
}

}  // namespace kda
