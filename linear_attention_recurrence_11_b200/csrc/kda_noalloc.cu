// kda_forward_noalloc: chunked prefill for callers that cannot allocate device
// memory (see include/kda.h for who they are).
//
// The only scratch kda_forward ever needs is the longest-first schedule of a
// packed batch (one int32 per sequence, up to kda::kMaxOrderedSeqs sequences).
// Here that scratch is a fixed array in this library's own device memory, so
// the caller passes inputs and outputs and nothing else. Everything else is
// the regular kda_forward path, called with this array as its workspace.
#include <mutex>

#include "kda_internal.cuh"

namespace {

// Fixed scratch: the schedule of at most kda::kMaxOrderedSeqs packed sequences
// (8 KiB). Every GPU that loads the library holds one copy until the process
// exits. Every call writes the entries it reads (order[0..num_seqs-1]) before
// reading them, so nothing has to start at zero; it keeps the last call's
// contents. Calls that overlap on the GPU (different streams, or host threads
// racing on one device) share it and race.
static __device__ __align__(256) int32_t kda_noalloc_scratch[kda::kMaxOrderedSeqs];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device. In host code the
// array's name only stands in for the symbol; the address is looked up with the
// device current. It is looked up again on every call made outside a stream
// capture, so a context torn down and rebuilt (after cudaDeviceReset) never
// leaves a stale address behind; inside a capture the address from the last
// uncaptured call on that device is used (the lookup is not made during capture).
int scratch_address(cudaStream_t stream, void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (cap == cudaStreamCaptureStatusNone || g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, kda_noalloc_scratch) != cudaSuccess || p == nullptr) return KDA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return KDA_OK;
}

}  // namespace

extern "C" int kda_forward_noalloc(const void *q, const void *k, const void *v, const void *g,
                                   const void *beta, const float *S0, void *o, float *S_T, int B, int T,
                                   int H, int dk, int dv, int chunk, int dtype, const int32_t *cu_seqlens,
                                   int num_seqs, int *dev_status, void *stream) {
    if (cu_seqlens != nullptr && num_seqs > kda::kMaxOrderedSeqs) return KDA_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    const int st = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
    if (st != KDA_OK) return st;
    return kda_forward(q, k, v, g, beta, S0, o, S_T, B, T, H, dk, dv, chunk, dtype, cu_seqlens, num_seqs,
                       scratch, sizeof(kda_noalloc_scratch), dev_status, stream);
}
