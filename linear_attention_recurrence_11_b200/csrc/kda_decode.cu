// One KDA decode step for a batch of requests, states updated in place.
//
// Per (request, head), with S in R^{dk x dv} stored as [dv][dk] fp32:
//   S' = Diag(exp g) S,  s = S'^T k,  u = beta (v - s),
//   S <- S' + k u^T,     o = S'^T q + u (k^T q)    (= S_new^T q)
// which is S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T with
// o_t = S_t^T q_t ("Exercices", Q7) for a single token.
//
// The step is bound by HBM bandwidth ("Exercices", Q4): every state is
// streamed once in and once out (2 x 64 KiB per head at dk = dv = 128) and the
// rest is a few hundred bytes. Layout of the work: one CTA of 4 warps per
// (request, head); 8 lanes cover one contiguous state row (a column j of S,
// dk floats) with 128-bit loads, so a warp touches 4 rows = 4 full 512-byte
// rows per load instruction; the two dot products over dk are finished with
// three xor-shuffles. Two rows per lane are in flight before any arithmetic.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDecThreads = 128;
constexpr int kLanesPerRow = 8;
constexpr int kRowsPerPass = (kDecThreads / 32) * (32 / kLanesPerRow);  // 16
constexpr int kRowsInFlight = 2;

__device__ __forceinline__ float4 ld_stream(const float *p) {
    return __ldcs(reinterpret_cast<const float4 *>(p));
}
__device__ __forceinline__ void st_stream(float *p, float4 x) {
    __stcs(reinterpret_cast<float4 *>(p), x);
}

template <typename Tin, int DK>
__global__ void __launch_bounds__(kDecThreads) kda_decode_kernel(const DecodeArgs p) {
    constexpr int F4 = DK / (4 * kLanesPerRow);  // float4 per lane per row
    constexpr int E = 4 * F4;                     // channels per lane
    const Tin *q = static_cast<const Tin *>(p.q), *k = static_cast<const Tin *>(p.k);
    const Tin *v = static_cast<const Tin *>(p.v), *g = static_cast<const Tin *>(p.g);
    const Tin *beta = static_cast<const Tin *>(p.beta);
    Tin *o = static_cast<Tin *>(p.o);

    const size_t unit = blockIdx.x;  // n * H + h
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane & (kLanesPerRow - 1), rw = lane / kLanesPerRow;

    float a[E], kk[E], qq[E];
    const size_t vb = unit * DK;
#pragma unroll
    for (int m = 0; m < F4; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = 4 * (sub + kLanesPerRow * m) + e;
            const float gi = ld_elem(g, vb + i);
            a[4 * m + e] = __expf((p.fuse & KDA_FUSE_GATE_LOGITS) ? gate_from_logit(gi) : gi);
            kk[4 * m + e] = ld_elem(k, vb + i);
            qq[4 * m + e] = ld_elem(q, vb + i);
        }
    if (p.fuse & KDA_FUSE_NORM_QK) {  // q and k normalised (the 8 lanes of a row hold all channels)
        float sk = 0.f, sq = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            sk = fmaf(kk[e], kk[e], sk);
            sq = fmaf(qq[e], qq[e], sq);
        }
#pragma unroll
        for (int off = 1; off < kLanesPerRow; off <<= 1) {
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
        }
        const float ik = sk > 0.f ? rsqrtf(sk) : 0.f, iq = sq > 0.f ? rsqrtf(sq) : 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            kk[e] *= ik;
            qq[e] *= iq;
        }
    }
    float kq = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) kq = fmaf(kk[e], qq[e], kq);
#pragma unroll
    for (int off = 1; off < kLanesPerRow; off <<= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    const float b = ld_elem(beta, unit);

    const int dv = p.dv;
    float *Su = p.S + unit * (size_t)dv * DK;
    for (int jb = warp * (32 / kLanesPerRow) + rw; jb < dv; jb += kRowsPerPass * kRowsInFlight) {
        float4 s[kRowsInFlight][F4];
        bool live[kRowsInFlight];
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            const int j = jb + r * kRowsPerPass;
            live[r] = j < dv;
#pragma unroll
            for (int m = 0; m < F4; ++m)
                s[r][m] = live[r] ? ld_stream(Su + (size_t)j * DK + 4 * (sub + kLanesPerRow * m))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            const int j = jb + r * kRowsPerPass;
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int m = 0; m < F4; ++m) {
                float *x = reinterpret_cast<float *>(&s[r][m]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[e] *= a[4 * m + e];
                    sk = fmaf(x[e], kk[4 * m + e], sk);
                    sq = fmaf(x[e], qq[4 * m + e], sq);
                }
            }
#pragma unroll
            for (int off = 1; off < kLanesPerRow; off <<= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
            }
            if (!live[r]) continue;
            const float u = b * (ld_elem(v, unit * dv + j) - sk);
#pragma unroll
            for (int m = 0; m < F4; ++m) {
                float *x = reinterpret_cast<float *>(&s[r][m]);
#pragma unroll
                for (int e = 0; e < 4; ++e) x[e] = fmaf(kk[4 * m + e], u, x[e]);
                st_stream(Su + (size_t)j * DK + 4 * (sub + kLanesPerRow * m), s[r][m]);
            }
            if (sub == 0) st_elem(o, unit * dv + j, fmaf(u, kq, sq));
        }
    }
}

template <typename Tin>
cudaError_t launch_decode_t(const DecodeArgs &a) {
    const unsigned grid = (unsigned)((size_t)a.N * a.H);
    switch (a.dk) {
        case 32: kda_decode_kernel<Tin, 32><<<grid, kDecThreads, 0, a.stream>>>(a); break;
        case 64: kda_decode_kernel<Tin, 64><<<grid, kDecThreads, 0, a.stream>>>(a); break;
        case 128: kda_decode_kernel<Tin, 128><<<grid, kDecThreads, 0, a.stream>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a) {
    if ((size_t)a.N * a.H == 0) return cudaSuccess;
    return a.dtype == KDA_DTYPE_BF16 ? launch_decode_t<__nv_bfloat16>(a) : launch_decode_t<float>(a);
}

}  // namespace kda
