// C ABI of libkda.so: argument validation and kernel dispatch (include/kda.h).
#include <stdint.h>

#include "kda_internal.cuh"

namespace {

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }
bool chunk_ok(int c) { return c == 16 || c == 32 || c == 64; }
bool dtype_ok(int t) { return t == KDA_DTYPE_F32 || t == KDA_DTYPE_BF16; }

// Validates the shape arguments shared by kda_forward_* and fills the sizes.
int check_prefill_sizes(int B, int T, int H, int dk, int dv, int chunk, int dtype,
                        bool has_cu, int num_seqs, int path, kda::PrefillArgs *a) {
    if (B <= 0 || T < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (!dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv) || !chunk_ok(chunk)) return KDA_ERR_UNSUPPORTED;
    if (has_cu && (B != 1 || num_seqs <= 0)) return KDA_ERR_INVALID_ARG;
    if (path < KDA_PATH_AUTO || path > KDA_PATH_TC_PIPE) return KDA_ERR_INVALID_ARG;
    if (path >= KDA_PATH_TC && !kda::prefill_tc_supported(dk, dv, chunk, dtype)) return KDA_ERR_UNSUPPORTED;
    // the kernels index tokens with size_t and units with 32-bit grid indices
    const size_t units = (size_t)(has_cu ? num_seqs : B) * (size_t)H;
    if (units * (size_t)(dv / 32) > 0x7fffffffu) return KDA_ERR_UNSUPPORTED;
    a->B = B; a->T = T; a->H = H; a->dk = dk; a->dv = dv; a->chunk = chunk; a->dtype = dtype;
    a->num_units = has_cu ? num_seqs : B;
    if (path == KDA_PATH_TC_PIPE && !kda::prefill_pipe_supported(*a)) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

// Marks "packed sequences are used" in size-only queries, where the real device
// pointer is not at hand; it is compared against null and never dereferenced.
const int32_t kPackedMarker = 0;

bool use_tc(const kda::PrefillArgs &a, int path) {
    if (path == KDA_PATH_SIMT) return false;
    return kda::prefill_tc_supported(a.dk, a.dv, a.chunk, a.dtype);
}

// The prefill form a call runs (kda_path): the SIMT kernel or one of the three tensor-core
// forms. AUTO and TC take the single kernel for batches of more (sequence, head) units than
// the split form's records pay for (the single kernel keeps every SM busy then and adds no
// record traffic): eight per SM for dense batches, three for packed ones, whose chains can be
// as uneven as their lengths. Measured on B200 (96 heads, 8192 tokens per sequence): the split
// form took 2.21, 3.25 and 4.48 ms for 4, 6 and 8 sequences against 2.52, 3.40 and 4.98 for
// the single kernel; 8 packed sequences of 4K to 98K tokens (768 units) 24.4 ms against 23.6.
// Otherwise the two-kernel split form when the workspace holds its records, then the
// one-launch form when its ring fits, then the single kernel.
enum class Form { Simt, Single, Split, Pipe };
bool many_units(const kda::PrefillArgs &a) {
    const bool packed = a.cu_seqlens != nullptr && a.num_units > 1;
    return (long long)a.num_units * a.H > (packed ? 3LL : 8LL) * kda::device_sm_count();
}
Form choose_form(const kda::PrefillArgs &a, int path, size_t workspace_bytes, bool workspace_known) {
    if (!use_tc(a, path)) return Form::Simt;
    if (path == KDA_PATH_TC_SINGLE) return Form::Single;
    if (path == KDA_PATH_TC_SPLIT) return Form::Split;
    if (path == KDA_PATH_TC_PIPE) return Form::Pipe;
    if (many_units(a)) return Form::Single;
    if (!workspace_known) return Form::Split;  // size queries assume the reported workspace
    if (workspace_bytes >= kda::prefill_split_workspace(a)) return Form::Split;
    if (kda::prefill_pipe_supported(a) && workspace_bytes >= kda::prefill_pipe_workspace(a)) return Form::Pipe;
    return Form::Single;
}

size_t form_workspace(const kda::PrefillArgs &a, Form f) {
    switch (f) {
        case Form::Simt: return kda::prefill_simt_workspace(a);
        case Form::Single: return kda::prefill_tc_workspace(a);
        case Form::Pipe: return kda::prefill_pipe_workspace(a);
        default: return kda::prefill_split_workspace(a);
    }
}

cudaError_t form_launch(const kda::PrefillArgs &a, Form f) {
    switch (f) {
        case Form::Simt: return kda::launch_prefill_simt(a);
        case Form::Single: return kda::launch_prefill_tc(a);
        case Form::Pipe: return kda::launch_prefill_pipe(a);
        default: return kda::launch_prefill_split(a);
    }
}

}  // namespace

namespace kda {
namespace {
thread_local cudaError_t g_last_cuda_error = cudaSuccess;
}
int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return KDA_OK;
    g_last_cuda_error = e;
    return KDA_ERR_CUDA;
}
int validate_prefill(int B, int T, int H, int dk, int dv, int chunk, int dtype, int path) {
    PrefillArgs a{};
    return check_prefill_sizes(B, T, H, dk, dv, chunk, dtype, false, 0, path, &a);
}
}  // namespace kda

extern "C" {

const char *kda_status_string(int status) {
    switch (status) {
        case KDA_OK: return "ok";
        case KDA_ERR_INVALID_ARG: return "invalid argument";
        case KDA_ERR_UNSUPPORTED: return "unsupported size, dtype or path";
        case KDA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case KDA_ERR_WORKSPACE: return "workspace missing or too small";
        case KDA_ERR_CUDA: return "CUDA error";
        case KDA_ERR_TIMEOUT: return "bounded wait timed out";
        case KDA_ERR_SCRATCH_LIMIT: return "more packed sequences than the no-alloc entry point's fixed scratch holds";
        default: return "unknown status";
    }
}

int kda_abi_version(void) { return 2; }

const char *kda_last_cuda_error(void) {
    const cudaError_t e = kda::g_last_cuda_error;
    return e == cudaSuccess ? "none" : cudaGetErrorName(e);
}

size_t kda_forward_workspace_size_ex(int B, int T, int H, int dk, int dv, int chunk, int num_seqs, int dtype,
                                     int path) {
    kda::PrefillArgs a{};
    // packed sequences (cu_seqlens) are recognised by B == 1 and num_seqs > 1
    const bool has_cu = B == 1 && num_seqs > 1;
    if (check_prefill_sizes(B, T, H, dk, dv, chunk, dtype, has_cu, num_seqs, path, &a)) return (size_t)-1;
    a.cu_seqlens = has_cu ? &kPackedMarker : nullptr;
    const Form f = choose_form(a, path, 0, false);
    size_t ws = form_workspace(a, f);
    if (f == Form::Simt) return ws;
    // the SIMT kernel is the fallback of every tensor-core form (empty batches)
    const size_t s = kda::prefill_simt_workspace(a);
    return s > ws ? s : ws;
}

size_t kda_forward_workspace_size(int B, int T, int H, int dk, int dv, int chunk, int num_seqs, int dtype) {
    return kda_forward_workspace_size_ex(B, T, H, dk, dv, chunk, num_seqs, dtype, KDA_PATH_AUTO);
}

int kda_forward_launches(int B, int T, int H, int dk, int dv, int chunk, int dtype,
                         int has_cu_seqlens, int num_seqs, int path) {
    kda::PrefillArgs a{};
    if (check_prefill_sizes(B, T, H, dk, dv, chunk, dtype, has_cu_seqlens != 0, num_seqs, path, &a))
        return -1;
    a.cu_seqlens = has_cu_seqlens ? &kPackedMarker : nullptr;
    switch (choose_form(a, path, 0, false)) {
        case Form::Simt: return kda::prefill_simt_launches(a);
        case Form::Single: return kda::prefill_tc_launches(a);
        case Form::Pipe: return kda::prefill_pipe_launches(a);
        default: return kda::prefill_split_launches(a);
    }
}

int kda_forward_ex(const void *q, const void *k, const void *v, const void *g, const void *beta,
                   const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv,
                   int chunk, int dtype, const int32_t *cu_seqlens, int num_seqs, void *workspace,
                   size_t workspace_bytes, int *dev_status, void *stream, int path) {
    kda::PrefillArgs a{};
    int st = check_prefill_sizes(B, T, H, dk, dv, chunk, dtype, cu_seqlens != nullptr, num_seqs,
                                 path, &a);
    if (st) return st;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, g, beta, (const void *)S0, (const void *)o, (const void *)S_T,
                          (const void *)cu_seqlens, (const void *)workspace, (const void *)dev_status})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
    a.S0 = S0; a.o = o; a.ST = S_T; a.cu_seqlens = cu_seqlens;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes; a.dev_status = dev_status;
    a.stream = static_cast<cudaStream_t>(stream);
    const Form f = choose_form(a, path, workspace == nullptr ? 0 : workspace_bytes, true);
    const size_t need = form_workspace(a, f);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return KDA_ERR_WORKSPACE;
    const cudaError_t e = form_launch(a, f);
    return kda::cuda_status(e);
}

int kda_forward_snapshots(const void *q, const void *k, const void *v, const void *g, const void *beta,
                          const float *S0, void *o, float *S_T, float *S_snap, int snap_every, int B, int T,
                          int H, int dk, int dv, int chunk, int dtype, void *workspace, size_t workspace_bytes,
                          int *dev_status, void *stream, int path) {
    kda::PrefillArgs a{};
    int st = check_prefill_sizes(B, T, H, dk, dv, chunk, dtype, false, 0, path, &a);
    if (st) return st;
    if (snap_every <= 0 || snap_every % chunk != 0) return KDA_ERR_INVALID_ARG;
    if (T / snap_every > 0 && !S_snap) return KDA_ERR_INVALID_ARG;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, g, beta, (const void *)S0, (const void *)o, (const void *)S_T,
                          (const void *)S_snap, (const void *)workspace, (const void *)dev_status})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
    a.S0 = S0; a.o = o; a.ST = S_T;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes; a.dev_status = dev_status;
    a.stream = static_cast<cudaStream_t>(stream);
    a.S_snap = S_snap; a.snap_every = T / snap_every > 0 ? snap_every : 0;
    // the split form (when it is the form kda_forward_ex would run and its chains can store the
    // snapshots) or the single form; the pipe form does not write snapshots
    if (path == KDA_PATH_TC_PIPE) return KDA_ERR_UNSUPPORTED;
    const bool split_ok = use_tc(a, path) && kda::prefill_split_snapshots_ok(a);
    if (path == KDA_PATH_TC_SPLIT && !split_ok) return KDA_ERR_UNSUPPORTED;
    const Form f = choose_form(a, path, workspace_bytes, true);
    if (f == Form::Split && split_ok) {
        if (workspace == nullptr || workspace_bytes < kda::prefill_split_workspace(a)) return KDA_ERR_WORKSPACE;
        return kda::cuda_status(kda::launch_prefill_split(a));
    }
    const bool tc = use_tc(a, path);
    const cudaError_t e = tc ? kda::launch_prefill_tc(a) : kda::launch_prefill_simt(a);
    return kda::cuda_status(e);
}

int kda_forward_fused(const void *q, const void *k, const void *v, const void *g, const void *beta,
                      const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv, int chunk,
                      int dtype, const int32_t *cu_seqlens, int num_seqs, void *workspace,
                      size_t workspace_bytes, int *dev_status, void *stream, int path, int flags) {
    if (flags & ~(KDA_FUSE_NORM_QK | KDA_FUSE_GATE_LOGITS)) return KDA_ERR_INVALID_ARG;
    kda::PrefillArgs a{};
    int st = check_prefill_sizes(B, T, H, dk, dv, chunk, dtype, cu_seqlens != nullptr, num_seqs, path, &a);
    if (st) return st;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, g, beta, (const void *)S0, (const void *)o, (const void *)S_T,
                          (const void *)cu_seqlens, (const void *)workspace, (const void *)dev_status})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta;
    a.S0 = S0; a.o = o; a.ST = S_T; a.cu_seqlens = cu_seqlens;
    a.workspace = workspace; a.workspace_bytes = workspace_bytes; a.dev_status = dev_status;
    a.stream = static_cast<cudaStream_t>(stream);
    a.fuse = flags;
    if (!flags)
        return kda_forward_ex(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, chunk, dtype, cu_seqlens, num_seqs,
                              workspace, workspace_bytes, dev_status, stream, path);
    if (path == KDA_PATH_TC_PIPE) return KDA_ERR_UNSUPPORTED;  // the pipe form has no fused variant
    // the form kda_forward_ex would run (the pipe form's place taken by the single form)
    const Form f = choose_form(a, path, workspace_bytes, true);
    if (f == Form::Split) {
        if (workspace == nullptr || workspace_bytes < kda::prefill_split_workspace(a)) return KDA_ERR_WORKSPACE;
        return kda::cuda_status(kda::launch_prefill_split(a));
    }
    const bool tc = f != Form::Simt;
    const size_t need = tc ? kda::prefill_tc_workspace(a) : kda::prefill_simt_workspace(a);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return KDA_ERR_WORKSPACE;
    const cudaError_t e = tc ? kda::launch_prefill_tc(a) : kda::launch_prefill_simt(a);
    return kda::cuda_status(e);
}

int kda_forward(const void *q, const void *k, const void *v, const void *g, const void *beta,
                const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv,
                int chunk, int dtype, const int32_t *cu_seqlens, int num_seqs, void *workspace,
                size_t workspace_bytes, int *dev_status, void *stream) {
    return kda_forward_ex(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, chunk, dtype, cu_seqlens,
                          num_seqs, workspace, workspace_bytes, dev_status, stream, KDA_PATH_AUTO);
}

namespace {
// Shared validation of kda_forward_segmented and its queries; fills s (not the pointers).
int check_segmented(int B, int T, int H, int dk, int dv, int chunk, int dtype, int seg_len, int path,
                    kda::SegmentedArgs *s, bool *tc_pair, bool *tc_state) {
    kda::PrefillArgs a{};
    int st = check_prefill_sizes(B, T, H, dk, dv, chunk, dtype, false, 0, path, &a);
    if (st) return st;
    if (seg_len <= 0 || seg_len % chunk != 0) return KDA_ERR_INVALID_ARG;
    const long long P = T == 0 ? 0 : ((long long)T + seg_len - 1) / seg_len;
    if (P > 1) {  // the segments run as packed sequences of one flat token axis
        if ((long long)B * T > 0x7fffffffLL || (long long)B * P > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
        if ((size_t)(B * P) * (size_t)H * (size_t)(dv > dk ? dv : dk) / 32 > 0x7fffffffu) return KDA_ERR_UNSUPPORTED;
        if (path >= KDA_PATH_TC && !kda::prefill_tc_supported(dk, dk, chunk, dtype)) return KDA_ERR_UNSUPPORTED;
    }
    *s = kda::SegmentedArgs{};
    s->B = B; s->T = T; s->H = H; s->dk = dk; s->dv = dv; s->chunk = chunk; s->dtype = dtype;
    s->seg_len = seg_len; s->P = (int)P; s->units = B * (int)P;
    *tc_pair = path != KDA_PATH_SIMT && kda::prefill_tc_supported(dk, dk, chunk, dtype);
    *tc_state = path != KDA_PATH_SIMT && kda::prefill_tc_supported(dk, dv, chunk, dtype);
    return KDA_OK;
}

// The same for packed batches: num_seqs sequences over T tokens in all. *cut is false when no
// sequence can be longer than seg_len (T <= seg_len): the call is then kda_forward_ex.
int check_segmented_varlen(int T, int H, int dk, int dv, int chunk, int dtype, int num_seqs, int seg_len,
                           int path, kda::SegmentedArgs *s, bool *tc_pair, bool *tc_state, bool *cut) {
    kda::PrefillArgs a{};
    int st = check_prefill_sizes(1, T, H, dk, dv, chunk, dtype, true, num_seqs, path, &a);
    if (st) return st;
    if (seg_len <= 0 || seg_len % chunk != 0) return KDA_ERR_INVALID_ARG;
    *cut = T > seg_len;
    const long long units = (long long)T / seg_len + num_seqs;  // bound on the number of segments
    if (*cut) {
        if (units >= 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
        if ((size_t)units * (size_t)H * (size_t)(dv > dk ? dv : dk) / 32 > 0x7fffffffu) return KDA_ERR_UNSUPPORTED;
        if (path >= KDA_PATH_TC && !kda::prefill_tc_supported(dk, dk, chunk, dtype)) return KDA_ERR_UNSUPPORTED;
    }
    *s = kda::SegmentedArgs{};
    s->B = num_seqs; s->T = T; s->H = H; s->dk = dk; s->dv = dv; s->chunk = chunk; s->dtype = dtype;
    s->seg_len = seg_len; s->P = 0; s->units = (int)units;
    s->cu_seqlens = &kPackedMarker;  // replaced by the caller's offsets in the call itself
    *tc_pair = path != KDA_PATH_SIMT && kda::prefill_tc_supported(dk, dk, chunk, dtype);
    *tc_state = path != KDA_PATH_SIMT && kda::prefill_tc_supported(dk, dv, chunk, dtype);
    return KDA_OK;
}
}  // namespace

size_t kda_forward_segmented_workspace_size(int B, int T, int H, int dk, int dv, int chunk, int dtype,
                                            int seg_len) {
    kda::SegmentedArgs s;
    bool tp, ts;
    if (check_segmented(B, T, H, dk, dv, chunk, dtype, seg_len, KDA_PATH_AUTO, &s, &tp, &ts)) return (size_t)-1;
    if (s.P <= 1) return kda_forward_workspace_size(B, T, H, dk, dv, chunk, B, dtype);
    return kda::segmented_workspace(s);
}

int kda_forward_segmented_launches(int B, int T, int H, int dk, int dv, int chunk, int dtype, int seg_len,
                                   int path) {
    kda::SegmentedArgs s;
    bool tp, ts;
    if (check_segmented(B, T, H, dk, dv, chunk, dtype, seg_len, path, &s, &tp, &ts)) return -1;
    if (s.P <= 1) return kda_forward_launches(B, T, H, dk, dv, chunk, dtype, 0, B, path);
    return kda::segmented_launches(s);
}

int kda_forward_segmented(const void *q, const void *k, const void *v, const void *g, const void *beta,
                          const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv, int chunk,
                          int dtype, int seg_len, void *workspace, size_t workspace_bytes, int *dev_status,
                          void *stream, int path) {
    kda::SegmentedArgs s;
    bool tc_pair, tc_state;
    int st = check_segmented(B, T, H, dk, dv, chunk, dtype, seg_len, path, &s, &tc_pair, &tc_state);
    if (st) return st;
    if (s.P <= 1)  // one segment: the plain prefill
        return kda_forward_ex(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, chunk, dtype, nullptr, 0, workspace,
                              workspace_bytes, dev_status, stream, path);
    if (!q || !k || !v || !g || !beta || !o) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, g, beta, (const void *)S0, (const void *)o, (const void *)S_T,
                          (const void *)workspace, (const void *)dev_status})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    s.q = q; s.k = k; s.v = v; s.g = g; s.beta = beta; s.S0 = S0; s.o = o; s.ST = S_T;
    s.workspace = workspace; s.workspace_bytes = workspace_bytes; s.dev_status = dev_status;
    s.stream = static_cast<cudaStream_t>(stream);
    if (workspace == nullptr || workspace_bytes < kda::segmented_workspace(s)) return KDA_ERR_WORKSPACE;
    return kda::cuda_status(kda::launch_segmented(s, tc_pair, tc_state));
}

size_t kda_forward_segmented_varlen_workspace_size(int T, int H, int dk, int dv, int chunk, int dtype, int num_seqs,
                                                   int seg_len) {
    kda::SegmentedArgs s;
    bool tp, ts, cut;
    if (check_segmented_varlen(T, H, dk, dv, chunk, dtype, num_seqs, seg_len, KDA_PATH_AUTO, &s, &tp, &ts, &cut))
        return (size_t)-1;
    if (!cut) return kda_forward_workspace_size(1, T, H, dk, dv, chunk, num_seqs, dtype);
    return kda::segmented_workspace(s);
}

int kda_forward_segmented_varlen_launches(int T, int H, int dk, int dv, int chunk, int dtype, int num_seqs,
                                          int seg_len, int path) {
    kda::SegmentedArgs s;
    bool tp, ts, cut;
    if (check_segmented_varlen(T, H, dk, dv, chunk, dtype, num_seqs, seg_len, path, &s, &tp, &ts, &cut)) return -1;
    if (!cut) return kda_forward_launches(1, T, H, dk, dv, chunk, dtype, 1, num_seqs, path);
    return kda::segmented_launches(s);
}

int kda_forward_segmented_varlen(const void *q, const void *k, const void *v, const void *g, const void *beta,
                                 const float *S0, void *o, float *S_T, int T, int H, int dk, int dv, int chunk,
                                 int dtype, const int32_t *cu_seqlens, int num_seqs, int seg_len, void *workspace,
                                 size_t workspace_bytes, int *dev_status, void *stream, int path) {
    kda::SegmentedArgs s;
    bool tc_pair, tc_state, cut;
    int st = check_segmented_varlen(T, H, dk, dv, chunk, dtype, num_seqs, seg_len, path, &s, &tc_pair, &tc_state,
                                    &cut);
    if (st) return st;
    if (!cu_seqlens) return KDA_ERR_INVALID_ARG;
    if (!cut)  // no sequence is longer than a segment: the plain prefill
        return kda_forward_ex(q, k, v, g, beta, S0, o, S_T, 1, T, H, dk, dv, chunk, dtype, cu_seqlens, num_seqs,
                              workspace, workspace_bytes, dev_status, stream, path);
    if (!q || !k || !v || !g || !beta || !o) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, g, beta, (const void *)S0, (const void *)o, (const void *)S_T,
                          (const void *)workspace, (const void *)dev_status})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    s.q = q; s.k = k; s.v = v; s.g = g; s.beta = beta; s.S0 = S0; s.o = o; s.ST = S_T;
    s.cu_seqlens = cu_seqlens;
    s.workspace = workspace; s.workspace_bytes = workspace_bytes; s.dev_status = dev_status;
    s.stream = static_cast<cudaStream_t>(stream);
    if (workspace == nullptr || workspace_bytes < kda::segmented_workspace(s)) return KDA_ERR_WORKSPACE;
    return kda::cuda_status(kda::launch_segmented(s, tc_pair, tc_state));
}

int kda_decode_step_fused(const void *q, const void *k, const void *v, const void *g, const void *beta,
                          float *S, void *o, int N, int H, int dk, int dv, int dtype, void *stream, int flags) {
    if (flags & ~(KDA_FUSE_NORM_QK | KDA_FUSE_GATE_LOGITS)) return KDA_ERR_INVALID_ARG;
    if (N <= 0 || H <= 0 || !dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if ((size_t)N * (size_t)H > 0x7fffffffu) return KDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !g || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, g, beta, (const void *)S, (const void *)o})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    kda::DecodeArgs a{q, k, v, g, beta, S, o, N, H, dk, dv, dtype, static_cast<cudaStream_t>(stream)};
    a.fuse = flags;
    return kda::cuda_status(kda::launch_decode(a));
}

int kda_decode_step(const void *q, const void *k, const void *v, const void *g, const void *beta,
                    float *S, void *o, int N, int H, int dk, int dv, int dtype, void *stream) {
    if (N <= 0 || H <= 0 || !dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if ((size_t)N * (size_t)H > 0x7fffffffu) return KDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !g || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, g, beta, (const void *)S, (const void *)o})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    kda::DecodeArgs a{q, k, v, g, beta, S, o, N, H, dk, dv, dtype, static_cast<cudaStream_t>(stream)};
    return kda::cuda_status(kda::launch_decode(a));
}

int kda_segment_pair(const void *q, const void *k, const void *v, const void *g, const void *beta, float *M,
                     float *Z, int B, int T, int H, int dk, int dv, int chunk, int dtype, int *dev_status,
                     void *stream, int path) {
    kda::PrefillArgs a{};
    int st = check_prefill_sizes(B, T, H, dk, dv, chunk, dtype, false, 0, path, &a);
    if (st) return st;
    if (path >= KDA_PATH_TC && !kda::prefill_tc_supported(dk, dk, chunk, dtype)) return KDA_ERR_UNSUPPORTED;
    if (!M || !Z || (T > 0 && (!q || !k || !v || !g || !beta))) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, g, beta, (const void *)M, (const void *)Z, (const void *)dev_status})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    kda::SegmentedArgs s{};
    s.q = q; s.k = k; s.v = v; s.g = g; s.beta = beta;
    s.B = B; s.T = T; s.H = H; s.dk = dk; s.dv = dv; s.chunk = chunk; s.dtype = dtype; s.P = 1; s.seg_len = T;
    s.dev_status = dev_status; s.stream = static_cast<cudaStream_t>(stream);
    const bool tc_pair = path != KDA_PATH_SIMT && kda::prefill_tc_supported(dk, dk, chunk, dtype);
    const bool tc_state = path != KDA_PATH_SIMT && kda::prefill_tc_supported(dk, dv, chunk, dtype);
    return kda::cuda_status(kda::launch_segment_pair(s, M, Z, tc_pair, tc_state));
}

int kda_kcp_scan(const float *S0, const float *M, const float *Z, float *S_in, float *S_T, int B, int P, int H,
                 int dk, int dv, void *stream) {
    if (B <= 0 || P <= 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if ((size_t)B * P * H > 0x7fffffffu) return KDA_ERR_UNSUPPORTED;
    if (!M || !Z || !S_in) return KDA_ERR_INVALID_ARG;
    for (const void *p : {(const void *)S0, (const void *)M, (const void *)Z, (const void *)S_in, (const void *)S_T})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    kda::SegmentedArgs s{};
    s.S0 = S0; s.ST = S_T; s.B = B; s.P = P; s.H = H; s.dk = dk; s.dv = dv;
    s.stream = static_cast<cudaStream_t>(stream);
    return kda::cuda_status(kda::launch_kcp_scan(s, M, Z, S_in));
}

int kda_decode_multi(const void *q, const void *k, const void *v, const void *g, const void *beta, float *S,
                     void *o, const int32_t *n_accept, int N, int T, int H, int dk, int dv, int dtype,
                     int *dev_status, void *stream) {
    if (N <= 0 || T <= 0 || H <= 0 || !dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if (T > kda::kMaxMultiTokens) return KDA_ERR_UNSUPPORTED;
    if (!head_dim_ok(dk) || !head_dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if ((size_t)N * (size_t)H > 0x7fffffffu || (size_t)N * T * H > 0x7fffffffu) return KDA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !g || !beta || !S) return KDA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, g, beta, (const void *)S, (const void *)o, (const void *)n_accept,
                          (const void *)dev_status})
        if (!aligned16(p)) return KDA_ERR_ALIGNMENT;
    kda::MultiDecodeArgs a{q, k, v, g, beta, S, o, n_accept, dev_status, N, T, H, dk, dv, dtype,
                           static_cast<cudaStream_t>(stream)};
    return kda::cuda_status(kda::launch_decode_multi(a));
}

}  // extern "C"
