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
#include <vector>

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

// Packed batches: the flat token axis [0, T) is cut into pieces of about Lp tokens, each
// boundary moved down onto the chunk grid of the sequence it falls in (that sequence's chunks
// start at cu[n]), so that every part of a sequence inside a piece starts at one of its own
// chunk boundaries. Piece i covers tokens [cut[i], cut[i + 1]) and sequences first[i] ..
// last[i] (the ones with a token in it); local[i] are its offsets relative to cut[i].
struct PackedPlan {
    std::vector<long long> cut;
    std::vector<int> first, last;
    std::vector<int32_t> local;    // all pieces' local offsets, piece i's at local_at[i]
    std::vector<size_t> local_at;
    int max_tokens = 0, max_seqs = 0;
};

// the sequence holding token t (cu[n] <= t < cu[n + 1]; empty sequences hold none)
int seq_of(const int32_t *cu, int num, long long t) {
    int lo = 0, hi = num;  // cu[lo] <= t < cu[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) / 2;
        if (cu[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}

bool plan_packed(const int32_t *cu, int num, long long T, int Lp, int chunk, PackedPlan &P) {
    P = PackedPlan{};
    P.cut.push_back(0);
    while (P.cut.back() < T) {
        const long long t0 = P.cut.back();
        long long b = t0 + Lp;
        if (b < T) {
            const int n = seq_of(cu, num, b);
            const long long aligned = cu[n] + (b - cu[n]) / chunk * chunk;
            b = aligned > t0 ? aligned : (long long)(cu[n] + ((t0 - cu[n]) / chunk + 1) * chunk);
            if (b > cu[n + 1]) b = cu[n + 1];
            if (b <= t0 || b > T) return false;
        } else {
            b = T;
        }
        P.cut.push_back(b);
    }
    const size_t pieces = P.cut.size() - 1;
    for (size_t i = 0; i < pieces; ++i) {
        const long long t0 = P.cut[i], t1 = P.cut[i + 1];
        const int f = seq_of(cu, num, t0), l = seq_of(cu, num, t1 - 1);
        P.first.push_back(f);
        P.last.push_back(l);
        P.local_at.push_back(P.local.size());
        for (int n = f; n <= l + 1; ++n) {
            long long x = n == f ? t0 : (n == l + 1 ? t1 : (long long)cu[n]);
            P.local.push_back((int32_t)(x - t0));
        }
        while (P.local.size() % 4) P.local.push_back(0);  // each piece's offsets 16-byte aligned
        if (t1 - t0 > P.max_tokens) P.max_tokens = (int)(t1 - t0);
        if (l - f + 1 > P.max_seqs) P.max_seqs = l - f + 1;
    }
    return true;
}

// Device workspace of the packed form: two slots of max_tokens, every sequence's state, the
// pieces' local offsets, and the device prefill's workspace for the largest piece.
struct PackedLayout {
    HostLayout slots;  // slot sizes for B = 1 and max_tokens (its state / scratch fields unused)
    size_t state, local, scratch, total;
};

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

namespace {
PackedLayout packed_layout(const PackedPlan &P, int num, int H, int dk, int dv, int chunk, int dtype) {
    PackedLayout L{};
    L.slots = host_layout(1, P.max_tokens, H, dk, dv, chunk, dtype);
    L.state = round_up((size_t)num * H * dv * dk * sizeof(float));
    L.local = round_up(P.local.size() * sizeof(int32_t));
    const size_t ws = P.max_tokens > 0 ? kda_forward_workspace_size(1, P.max_tokens, H, dk, dv, chunk,
                                                                     P.max_seqs > 1 ? P.max_seqs : 1, dtype)
                                       : 0;
    L.scratch = ws == (size_t)-1 ? 0 : round_up(ws);
    L.total = 2 * L.slots.slot + L.state + L.local + L.scratch;
    return L;
}

int check_host_varlen(int T, int H, int dk, int dv, int chunk, int dtype, const int32_t *cu, int num,
                      int piece_len, int path) {
    int st = kda::validate_prefill(1, T, H, dk, dv, chunk, dtype, path);
    if (st) return st;
    if (!cu || num <= 0) return KDA_ERR_INVALID_ARG;
    if (cu[0] != 0 || cu[num] != T) return KDA_ERR_INVALID_ARG;
    for (int n = 0; n < num; ++n)
        if (cu[n + 1] < cu[n]) return KDA_ERR_INVALID_ARG;
    if (piece_len < 0 || (piece_len > 0 && piece_len % chunk != 0)) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}
}  // namespace

size_t kda_forward_host_varlen_workspace_size(int T, int H, int dk, int dv, int chunk, int dtype,
                                              const int32_t *cu_seqlens, int num_seqs, int piece_len) {
    if (check_host_varlen(T, H, dk, dv, chunk, dtype, cu_seqlens, num_seqs, piece_len, KDA_PATH_AUTO) != KDA_OK)
        return (size_t)-1;
    PackedPlan P;
    if (!plan_packed(cu_seqlens, num_seqs, T, piece_len > 0 ? piece_len : default_piece(T, chunk), chunk, P))
        return (size_t)-1;
    return packed_layout(P, num_seqs, H, dk, dv, chunk, dtype).total;
}

int kda_forward_host_varlen(const void *q, const void *k, const void *v, const void *g, const void *beta,
                            const float *S0, void *o, float *S_T, int T, int H, int dk, int dv, int chunk,
                            int dtype, const int32_t *cu_seqlens, int num_seqs, int piece_len, void *workspace,
                            size_t workspace_bytes, int *dev_status, void *stream, int path) {
    int st = check_host_varlen(T, H, dk, dv, chunk, dtype, cu_seqlens, num_seqs, piece_len, path);
    if (st) return st;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    PackedPlan P;
    if (!plan_packed(cu_seqlens, num_seqs, T, piece_len > 0 ? piece_len : default_piece(T, chunk), chunk, P))
        return KDA_ERR_INVALID_ARG;
    const PackedLayout L = packed_layout(P, num_seqs, H, dk, dv, chunk, dtype);
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
    const HostLayout &S = L.slots;
    for (int i = 0; i < 2; ++i) {
        char *b = ws + i * S.slot;
        slot[i].q = b; b += round_up(S.q);
        slot[i].k = b; b += round_up(S.k);
        slot[i].v = b; b += round_up(S.v);
        slot[i].g = b; b += round_up(S.g);
        slot[i].beta = b; b += round_up(S.beta);
        slot[i].o = b;
    }
    float *state = reinterpret_cast<float *>(ws + 2 * S.slot);
    int32_t *local = reinterpret_cast<int32_t *>(ws + 2 * S.slot + L.state);
    void *scratch = L.scratch ? ws + 2 * S.slot + L.state + L.local : nullptr;
    const size_t unit_state = (size_t)H * dv * dk;
    const size_t state_bytes = (size_t)num_seqs * unit_state * sizeof(float);

#define KDA_TRY(x)                                   \
    do {                                             \
        if ((x) != cudaSuccess) return KDA_ERR_CUDA; \
    } while (0)
    KDA_TRY(cudaEventRecord(hp.ev_start, cs));
    KDA_TRY(cudaStreamWaitEvent(hp.up, hp.ev_start, 0));
    KDA_TRY(cudaStreamWaitEvent(hp.down, hp.ev_start, 0));
    // every sequence's state (S0 or zeros) and the pieces' local offsets, once
    if (S0) KDA_TRY(cudaMemcpyAsync(state, S0, state_bytes, cudaMemcpyHostToDevice, hp.up));
    else KDA_TRY(cudaMemsetAsync(state, 0, state_bytes, hp.up));
    KDA_TRY(cudaMemcpyAsync(local, P.local.data(), P.local.size() * sizeof(int32_t), cudaMemcpyHostToDevice, hp.up));

    const size_t rowq = (size_t)H * dk * es, rowv = (size_t)H * dv * es, rowb = (size_t)H * es;
    const char *hq = static_cast<const char *>(q), *hk = static_cast<const char *>(k);
    const char *hv = static_cast<const char *>(v), *hg = static_cast<const char *>(g);
    const char *hb = static_cast<const char *>(beta);
    char *ho = static_cast<char *>(o);
    const size_t pieces = P.cut.size() - 1;
    for (size_t p = 0; p < pieces; ++p) {
        const int s = (int)(p & 1);
        const long long t0 = P.cut[p];
        const int n = (int)(P.cut[p + 1] - t0);
        // upload piece p once the launch of piece p - 2 has consumed the slot: contiguous rows
        if (p >= 2) KDA_TRY(cudaStreamWaitEvent(hp.up, hp.ev_comp[s], 0));
        KDA_TRY(cudaMemcpyAsync(slot[s].q, hq + t0 * rowq, n * rowq, cudaMemcpyHostToDevice, hp.up));
        KDA_TRY(cudaMemcpyAsync(slot[s].k, hk + t0 * rowq, n * rowq, cudaMemcpyHostToDevice, hp.up));
        KDA_TRY(cudaMemcpyAsync(slot[s].v, hv + t0 * rowv, n * rowv, cudaMemcpyHostToDevice, hp.up));
        KDA_TRY(cudaMemcpyAsync(slot[s].g, hg + t0 * rowq, n * rowq, cudaMemcpyHostToDevice, hp.up));
        KDA_TRY(cudaMemcpyAsync(slot[s].beta, hb + t0 * rowb, n * rowb, cudaMemcpyHostToDevice, hp.up));
        KDA_TRY(cudaEventRecord(hp.ev_up[s], hp.up));
        // the packed prefill of piece p: its sequences' states in place
        KDA_TRY(cudaStreamWaitEvent(cs, hp.ev_up[s], 0));
        if (p >= 2) KDA_TRY(cudaStreamWaitEvent(cs, hp.ev_down[s], 0));
        float *st_p = state + (size_t)P.first[p] * unit_state;
        const int ns = P.last[p] - P.first[p] + 1;
        st = kda_forward_ex(slot[s].q, slot[s].k, slot[s].v, slot[s].g, slot[s].beta, st_p, slot[s].o, st_p, 1, n,
                            H, dk, dv, chunk, dtype, local + P.local_at[p], ns, scratch, L.scratch, dev_status, cs,
                            path);
        if (st) return st;
        KDA_TRY(cudaEventRecord(hp.ev_comp[s], cs));
        KDA_TRY(cudaStreamWaitEvent(hp.down, hp.ev_comp[s], 0));
        KDA_TRY(cudaMemcpyAsync(ho + t0 * rowv, slot[s].o, n * rowv, cudaMemcpyDeviceToHost, hp.down));
        KDA_TRY(cudaEventRecord(hp.ev_down[s], hp.down));
    }
    // the state copies above were on the upload stream: the download waits for them
    KDA_TRY(cudaEventRecord(hp.ev_up[0], hp.up));
    KDA_TRY(cudaStreamWaitEvent(hp.down, hp.ev_up[0], 0));
    if (S_T) KDA_TRY(cudaMemcpyAsync(S_T, state, state_bytes, cudaMemcpyDeviceToHost, hp.down));
    KDA_TRY(cudaEventRecord(hp.ev_done, hp.down));
    KDA_TRY(cudaStreamWaitEvent(cs, hp.ev_done, 0));
#undef KDA_TRY
    return KDA_OK;
}

}  // extern "C"
