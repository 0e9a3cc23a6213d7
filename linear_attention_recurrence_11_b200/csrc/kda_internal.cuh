// Internal declarations shared by the libkda.so translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// Arguments of one prefill call, as validated by the C ABI layer.
// Prefill arguments. Inside the library (the segment-pair pass of kda_forward_segmented)
// v may be null, meaning all-zero values, and o may be null, meaning no outputs.
struct PrefillArgs {
    const void *q, *k, *v, *g, *beta;
    const float *S0;
    void *o;
    float *ST;
    const int32_t *cu_seqlens;  // device offsets or nullptr
    const int32_t *seq_order;   // device: block b runs sequence seq_order[b / H] (nullptr: b / H)
    int B, T, H, dk, dv, chunk, dtype;
    int num_units;              // N: sequences (B, or num_seqs with cu_seqlens)
    void *workspace;
    size_t workspace_bytes;
    int *dev_status;
    cudaStream_t stream;
    // kda_forward_snapshots (dense batches): every snap_every tokens (a multiple of chunk) the
    // state after that prefix goes to S_snap [B, T / snap_every, H, dv, dk]; 0 = none
    float *S_snap = nullptr;
    int snap_every = 0;
    int fuse = 0;  // KDA_FUSE_* bits: q, k normalised and / or g from gate logits inside the kernel
};

// kda_forward_segmented: B dense sequences of T tokens, each cut into P = ceil(T / seg_len)
// segments that run as independent units (kda_segmented.cu).
struct SegmentedArgs {
    const void *q, *k, *v, *g, *beta;
    const float *S0;
    void *o;
    float *ST;
    int B, T, H, dk, dv, chunk, dtype, seg_len, P;
    void *workspace;
    size_t workspace_bytes;
    int *dev_status;
    cudaStream_t stream;
    // kda_forward_segmented_varlen: B = num_seqs packed sequences (device offsets) over T tokens
    // in all, every one cut into max(1, ceil(len / seg_len)) segments; P is unused
    const int32_t *cu_seqlens = nullptr;
    int units = 0;  // segment slots: B * P for dense batches, T / seg_len + B for packed ones
};

struct DecodeArgs {
    const void *q, *k, *v, *g, *beta;
    float *S;
    void *o;
    int N, H, dk, dv, dtype;
    cudaStream_t stream;
    int fuse = 0;  // KDA_FUSE_* bits
};

// g from a gate logit x: g_min sigmoid(x) = -5 / (1 + e^{-x}), in [g_min, 0]
__device__ __forceinline__ float gate_from_logit(float x) { return -5.f / (1.f + __expf(-x)); }

// kda_decode_multi: T tokens per request, the state after n_accept[n] of them written back.
struct MultiDecodeArgs {
    const void *q, *k, *v, *g, *beta;
    float *S;
    void *o;                   // may be null: no outputs
    const int32_t *n_accept;   // device [N] or null (all T)
    int *dev_status;           // device status word or null
    int N, T, H, dk, dv, dtype;
    cudaStream_t stream;
};
constexpr int kMaxMultiTokens = 64;

// Element loads/stores in the storage dtype, computed in fp32.
__device__ __forceinline__ float ld_elem(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld_elem(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_elem(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_elem(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// Longest-first ordering of packed sequences (workspace-backed, up to this many).
constexpr int kMaxOrderedSeqs = 2048;
size_t seq_order_bytes(int num_seqs);  // 0 when no ordering is done
cudaError_t launch_seq_order(const int32_t *cu_seqlens, int num_seqs, int32_t *order, cudaStream_t stream);

// Sequence index run by prefill block `b` (one block per (sequence, head) unit).
__device__ __forceinline__ int unit_seq(const PrefillArgs &p, int b_over_h) {
    return p.seq_order ? p.seq_order[b_over_h] : b_over_h;
}

// Launchers (return cudaSuccess or the launch error).
cudaError_t launch_prefill_simt(const PrefillArgs &a);
size_t prefill_simt_workspace(const PrefillArgs &a);
int prefill_simt_launches(const PrefillArgs &a);

bool prefill_tc_supported(int dk, int dv, int chunk, int dtype);
size_t segmented_workspace(const SegmentedArgs &s);
int segmented_launches(const SegmentedArgs &s);
// tc_pair / tc_state: run the M_p pass (dv = dk) / the other passes on the tensor-core kernel
cudaError_t launch_segmented(const SegmentedArgs &s, bool tc_pair, bool tc_state);
// one segment per sequence: M [B, H, dk, dk] (from the identity, zero values), Z [B, H, dv, dk] (from 0)
cudaError_t launch_segment_pair(const SegmentedArgs &s, float *M, float *Z, bool tc_pair, bool tc_state);
// s.S0 / s.ST / s.B / s.P / s.H / s.dk / s.dv / s.stream: incoming states of P segments per sequence
// (seg_base non-null: sequence b has the segments seg_base[b] .. seg_base[b + 1] - 1)
cudaError_t launch_kcp_scan(const SegmentedArgs &s, const float *Mbuf, const float *Zbuf, float *Sin,
                            const int32_t *seg_base = nullptr);
cudaError_t launch_prefill_tc(const PrefillArgs &a);
size_t prefill_tc_workspace(const PrefillArgs &a);
int prefill_tc_launches(const PrefillArgs &a);
// the split tensor-core form: chunk-parallel records in the workspace, then the state chains
cudaError_t launch_prefill_split(const PrefillArgs &a);
// its two stages: the records of every chunk of `a` (in a.workspace), and one pass of the
// state chains over them with pass's S0 / S_T / o (the q, k, g, beta, sizes and layout of
// `a`; pass.v == nullptr leaves every record's Ut out: all-zero values)
struct SplitRecords {
    uint8_t *rec;
    const int32_t *chunk_base, *seq_order;
    int nch;
    long long tasks;
};
cudaError_t launch_split_records(const PrefillArgs &a, SplitRecords *out);
cudaError_t launch_split_chain(const PrefillArgs &pass, const SplitRecords &r);
size_t prefill_split_workspace(const PrefillArgs &a);
int prefill_split_launches(const PrefillArgs &a);
// the split form writes S_snap (dense batches of up to one unit per SM: the double-buffered chains)
bool prefill_split_snapshots_ok(const PrefillArgs &a);
// the one-launch form: chains and record producers in one cooperative launch, records in a ring
bool prefill_pipe_supported(const PrefillArgs &a);
cudaError_t launch_prefill_pipe(const PrefillArgs &a);
size_t prefill_pipe_workspace(const PrefillArgs &a);
int prefill_pipe_launches(const PrefillArgs &a);

cudaError_t launch_decode(const DecodeArgs &a);
cudaError_t launch_decode_multi(const MultiDecodeArgs &a);
// SMs of the current device (148 when no device answers, e.g. size queries on a host
// without a GPU); cached after the first call
int device_sm_count();
// KDA_OK for cudaSuccess; otherwise KDA_ERR_CUDA, the error kept for kda_last_cuda_error
int cuda_status(cudaError_t e);
// KDA_OK, or the status kda_forward_ex returns for these sizes (dense batches)
int validate_prefill(int B, int T, int H, int dk, int dv, int chunk, int dtype, int path);

}  // namespace kda
