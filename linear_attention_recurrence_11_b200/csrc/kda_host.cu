// Prefill from host memory: the inputs are uploaded, the prefill runs and the
// outputs come back in token pieces, so that the two copy directions and the
// kernels overlap (include/kda.h, kda_forward_host).
//
// The fixed-size state is all that a later part of a sequence needs of its past
// ("Exercices", Q6: the KDA state does not grow with the length; Q21: a
// segment acts on the state it receives), so a sequence can be cut at any
// chunk boundary and resumed from the fp32 state the first part ends in:
// piece p of every sequence (tokens [p L, (p+1) L)) is one prefill launch
// whose initial state is the state the launch of piece p-1 left in the same
// device buffer. With L a multiple of the chunk the chunks
// are the ones a single launch over all T tokens makes, and the result is the
// same bit for bit.
//
// Pipeline, two device slots for the pieces:
//   upload stream   : [wait: compute of piece p-2 done]  H2D of piece p   -> in[p % 2]
//   caller's stream : [wait: upload p, download p-2]      prefill piece p -> out[p % 2]
//   download stream : [wait: compute of piece p]          D2H of out[p % 2]
// and at the end the state's download, with the caller's stream made to wait
// for it, so that anything the caller enqueues after the call (an event, a
// synchronisation) sees the host outputs complete.
#include <mutex>

#include "kda_internal.cuh"

namespace {

constexpr int kMaxDevices = 64;

// Side streams and events of one device, made on first use and kept for the
// life of the process (calls on one device take the mutex while they enqueue).
struct HostPipe {
    std::once_flag once;
    cudaError_t init_error = cudaSuccess;
    std::mutex mu;
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t ev_start = nullptr, ev_done = nullptr;
    cudaEvent_t ev_up[2] = {nullptr, nullptr}, ev_comp[2] = {nullptr, nullptr}, ev_down[2] = {nullptr, nullptr};
};
HostPipe g_pipes[kMaxDevices];

cudaError_t pipe_init(HostPipe &hp) {
    cudaError_t e = cudaStreamCreateWithFlags(&hp.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.down, cudaStreamNonBlocking);
    cudaEvent_t *evs[] = {&hp.ev_start, &hp.ev_done, &hp.ev_up[0], &hp.ev_up[1],
                          &hp.ev_comp[0], &hp.ev_comp[1], &hp.ev_down[0], &hp.ev_down[1]};
    for (cudaEvent_t *ev : evs)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    return e;
}

size_t round_up(size_t x) { return (x + 255) & ~size_t(255); }

// Device workspace layout for pieces of up to Lp tokens.
struct HostLayout {
    size_t q, k, v, g, beta, o;  // bytes of one piece of each tensor
    size_t slot;                 // one slot: the six tensors, 256-byte aligned each
    size_t state;                // [B, H, dv, dk] fp32
    size_t scratch;              // the device prefill's workspace for one piece (pieces run in turn)
    size_t total;
};

HostLayout host_layout(int B, int Lp, int H, int dk, int dv, int chunk, int dtype) {
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    const size_t tok = (size_t)B * (size_t)Lp * (size_t)H;
    HostLayout L{};
    L.q = L.k = L.g = tok * dk * es;
    L.v = L.o = tok * dv * es;
    L.beta = tok * es;
    L.slot = round_up(L.q) + round_up(L.k) + round_up(L.v) + round_up(L.g) + round_up(L.beta) + round_up(L.o);
    L.state = round_up((size_t)B * H * dv * dk * sizeof(float));
    const size_t ws = Lp > 0 ? kda_forward_workspace_size(B, Lp, H, dk, dv, chunk, B, dtype) : 0;
    L.scratch = ws == (size_t)-1 ? 0 : round_up(ws);
    L.total = 2 * L.slot + L.state + L.scratch;
    return L;
}

// Copies tokens [t0, t0 + n) of every sequence of a [B, T, H, d] tensor between
// host and a contiguous [B, n, H, d] device piece: one strided copy of B rows.
cudaError_t copy_piece(void *dst, const void *src, int B, int T, long long t0, int n, size_t row_elems,
                       size_t es, bool to_device, cudaStream_t s) {
    const size_t width = (size_t)n * row_elems * es, full = (size_t)T * row_elems * es;
    const size_t off = (size_t)t0 * row_elems * es;
    if (to_device)
        return cudaMemcpy2DAsync(dst, width, static_cast<const char *>(src) + off, full, width, B,
                                 cudaMemcpyHostToDevice, s);
    return cudaMemcpy2DAsync(static_cast<char *>(dst) + off, full, src, width, width, B, cudaMemcpyDeviceToHost,
                             s);
}

int default_piece(int T, int chunk) {
    // about eight pieces, whole chunks, at least one chunk
    long long p = ((long long)T + 7) / 8;
    p = (p + chunk - 1) / chunk * chunk;
    return (int)(p < chunk ? chunk : p);
}

}  // namespace

extern "C" {

size_t kda_forward_host_workspace_size(int B, int T, int H, int dk, int dv, int chunk, int dtype, int piece_len) {
    if (kda::validate_prefill(B, T, H, dk, dv, chunk, dtype, KDA_PATH_AUTO) != KDA_OK) return (size_t)-1;
    if (piece_len < 0 || (piece_len > 0 && piece_len % chunk != 0)) return (size_t)-1;
    const int Lp0 = piece_len > 0 ? piece_len : default_piece(T, chunk);
    const int Lp = T < Lp0 ? T : Lp0;
    return host_layout(B, Lp, H, dk, dv, chunk, dtype).total;
}

int kda_forward_host(const void *q, const void *k, const void *v, const void *g, const void *beta,
                     const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv, int chunk,
                     int dtype, int piece_len, void *workspace, size_t workspace_bytes, int *dev_status,
                     void *stream, int path) {
    int st = kda::validate_prefill(B, T, H, dk, dv, chunk, dtype, path);
    if (st) return st;
    if (piece_len < 0 || (piece_len > 0 && piece_len % chunk != 0)) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    const int Lp0 = piece_len > 0 ? piece_len : default_piece(T, chunk);
    const int Lp = T < Lp0 ? T : Lp0;
    const HostLayout L = host_layout(B, Lp, H, dk, dv, chunk, dtype);
    if (!workspace || workspace_bytes < L.total) return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KDA_ERR_ALIGNMENT;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    HostPipe &hp = g_pipes[dev];
    std::call_once(hp.once, [&hp] { hp.init_error = pipe_init(hp); });
    if (hp.init_error != cudaSuccess) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(hp.mu);

    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    char *ws = static_cast<char *>(workspace);
    struct Slot { char *q, *k, *v, *g, *beta, *o; } slot[2];
    for (int s = 0; s < 2; ++s) {
        char *b = ws + s * L.slot;
        slot[s].q = b; b += round_up(L.q);
        slot[s].k = b; b += round_up(L.k);
        slot[s].v = b; b += round_up(L.v);
        slot[s].g = b; b += round_up(L.g);
        slot[s].beta = b; b += round_up(L.beta);
        slot[s].o = b;
    }
    float *state = reinterpret_cast<float *>(ws + 2 * L.slot);
    void *scratch = L.scratch ? ws + 2 * L.slot + L.state : nullptr;
    const size_t state_bytes = (size_t)B * H * dv * dk * sizeof(float);

#define KDA_TRY(x)                                   \
    do {                                             \
        if ((x) != cudaSuccess) return KDA_ERR_CUDA; \
    } while (0)
    // the side streams start after the work already on the caller's stream
    KDA_TRY(cudaEventRecord(hp.ev_start, cs));
    KDA_TRY(cudaStreamWaitEvent(hp.up, hp.ev_start, 0));
    KDA_TRY(cudaStreamWaitEvent(hp.down, hp.ev_start, 0));
    if (S0) KDA_TRY(cudaMemcpyAsync(state, S0, state_bytes, cudaMemcpyHostToDevice, hp.up));

    const long long npieces = T == 0 ? 1 : ((long long)T + Lp - 1) / Lp;
    for (long long p = 0; p < npieces; ++p) {
        const int s = (int)(p & 1);
        const long long t0 = p * Lp;
        const int n = (int)((T - t0) < Lp ? (T - t0) : Lp);
        // upload piece p once the launch of piece p - 2 has consumed the slot
        if (p >= 2) KDA_TRY(cudaStreamWaitEvent(hp.up, hp.ev_comp[s], 0));
        if (n > 0) {
            KDA_TRY(copy_piece(slot[s].q, q, B, T, t0, n, (size_t)H * dk, es, true, hp.up));
            KDA_TRY(copy_piece(slot[s].k, k, B, T, t0, n, (size_t)H * dk, es, true, hp.up));
            KDA_TRY(copy_piece(slot[s].v, v, B, T, t0, n, (size_t)H * dv, es, true, hp.up));
            KDA_TRY(copy_piece(slot[s].g, g, B, T, t0, n, (size_t)H * dk, es, true, hp.up));
            KDA_TRY(copy_piece(slot[s].beta, beta, B, T, t0, n, (size_t)H, es, true, hp.up));
        }
        KDA_TRY(cudaEventRecord(hp.ev_up[s], hp.up));
        // the prefill of piece p from the state piece p - 1 ended in (in place)
        KDA_TRY(cudaStreamWaitEvent(cs, hp.ev_up[s], 0));
        if (p >= 2) KDA_TRY(cudaStreamWaitEvent(cs, hp.ev_down[s], 0));
        st = kda_forward_ex(slot[s].q, slot[s].k, slot[s].v, slot[s].g, slot[s].beta,
                            (p == 0 && !S0) ? nullptr : state, slot[s].o, state, B, n, H, dk, dv, chunk, dtype,
                            nullptr, 0, scratch, L.scratch, dev_status, cs, path);
        if (st) return st;
        KDA_TRY(cudaEventRecord(hp.ev_comp[s], cs));
        // its outputs back to the host
        KDA_TRY(cudaStreamWaitEvent(hp.down, hp.ev_comp[s], 0));
        if (n > 0) KDA_TRY(copy_piece(o, slot[s].o, B, T, t0, n, (size_t)H * dv, es, false, hp.down));
        KDA_TRY(cudaEventRecord(hp.ev_down[s], hp.down));
    }
    if (S_T) KDA_TRY(cudaMemcpyAsync(S_T, state, state_bytes, cudaMemcpyDeviceToHost, hp.down));
    KDA_TRY(cudaEventRecord(hp.ev_done, hp.down));
    KDA_TRY(cudaStreamWaitEvent(cs, hp.ev_done, 0));
#undef KDA_TRY
    return KDA_OK;
}

}  // extern "C"
