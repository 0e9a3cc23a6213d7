// Self-test of the bounded waits of the tensor-core prefill: a kernel waits, with
// the same helpers and the same reporting, on an mbarrier that nothing ever
// arrives on (every wait on a copy or an MMA), then on a flag in global memory
// that nothing ever sets (a chain waiting for a record produced by another CTA
// of its launch). Each wait gives up after max_cycles SM clocks and the kernel
// records KDA_ERR_TIMEOUT, for the mbarrier in dev_status[0] and for the flag in
// dev_status[2] (dev_status[1] is the flag, zero on entry); nothing faults, traps
// or hangs, and the context stays usable. Used by the failure-detection tests.
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

__global__ void kda_wait_selftest_kernel(int *dev_status, long long max_cycles) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    // phase 0 never completes: no thread arrives and no copy is in flight
    const bool ok = sm100::mbar_wait_bounded(&bar, 0, max_cycles);
    if (__syncthreads_or(!ok) && threadIdx.x == 0) atomicExch(dev_status, (int)KDA_ERR_TIMEOUT);
    // the flag stays zero: nothing in this launch sets it
    if (threadIdx.x == 0 &&
        !sm100::wait_counter(reinterpret_cast<const unsigned *>(dev_status + 1), 1u, max_cycles))
        atomicExch(dev_status + 2, (int)KDA_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_selftest(int *dev_status, long long max_cycles, cudaStream_t stream) {
    kda_wait_selftest_kernel<<<1, 64, 0, stream>>>(dev_status, max_cycles);
    return cudaGetLastError();
}

}  // namespace kda

extern "C" int kda_selftest_wait_timeout(int *dev_status, long long max_cycles, void *stream) {
    if (!dev_status || max_cycles <= 0 || max_cycles > 4000000000LL) return KDA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(dev_status) & 15u) != 0) return KDA_ERR_ALIGNMENT;
    return kda::launch_wait_selftest(dev_status, max_cycles, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? KDA_OK
               : KDA_ERR_CUDA;
}
