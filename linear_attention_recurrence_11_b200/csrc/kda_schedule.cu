// Longest-first order of packed variable-length sequences.
//
// The prefill kernels give each (sequence, head) unit one CTA, and a unit's
// chunks run one after the other, so a batch of very different lengths
// finishes fastest when the longest sequences start first (longest processing
// time first). One block ranks the sequences by length (descending, ties by
// index, so the order is deterministic) and writes order[rank] = sequence; the
// prefill kernels then map block b to sequence order[b / H].
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kSchedThreads = 1024;

__global__ void __launch_bounds__(kSchedThreads) kda_longest_first_kernel(const int32_t *__restrict__ cu, int n,
                                                                         int32_t *__restrict__ order) {
    __shared__ int32_t len[kMaxOrderedSeqs];
    for (int i = threadIdx.x; i < n; i += kSchedThreads) len[i] = cu[i + 1] - cu[i];
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kSchedThreads) {
        const int32_t li = len[i];
        int rank = 0;
        for (int j = 0; j < n; ++j) {
            const int32_t lj = len[j];
            rank += (lj > li) || (lj == li && j < i);
        }
        order[rank] = i;
    }
}

}  // namespace

size_t seq_order_bytes(int num_seqs) {
    if (num_seqs <= 1 || num_seqs > kMaxOrderedSeqs) return 0;
    return ((size_t)num_seqs * sizeof(int32_t) + 255) & ~(size_t)255;
}

cudaError_t launch_seq_order(const int32_t *cu_seqlens, int num_seqs, int32_t *order, cudaStream_t stream) {
    kda_longest_first_kernel<<<1, kSchedThreads, 0, stream>>>(cu_seqlens, num_seqs, order);
    return cudaGetLastError();
}

}  // namespace kda
