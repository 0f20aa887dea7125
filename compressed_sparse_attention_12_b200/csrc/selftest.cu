// selftest.cu -- a check of the library's bounded waits (the ones the
// tensor-core indexer's producer, MMA and epilogue warps use): one CTA waits on
// an mbarrier phase that nothing completes; the wait gives up after the
// library's limit (1 s of GPU time) and the kernel records CSA_ERR_TIMEOUT in
// the caller's status word, leaving the context usable.
#include "common.cuh"
#include "tc.cuh"

namespace csa {

__global__ void wait_timeout_kernel(int32_t *status, int32_t *waited_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(tc::saddr(&bar), 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = tc::globaltimer();
        // phase 0 of a fresh barrier with one expected arrival and none made
        const bool done = tc::mbar_wait(tc::saddr(&bar), 0u, nullptr);
        const uint64_t t1 = tc::globaltimer();
        if (!done) report(status, CSA_ERR_TIMEOUT);
        const uint64_t dt = t1 - t0;
        if (waited_ns) *waited_ns = (int32_t)(dt < 2147483647ull ? dt : 2147483647ull);
    }
}

}  // namespace csa

extern "C" csa_status_t csa_selftest_wait_timeout(int32_t *status, int32_t *waited_ns,
                                                  void *stream) {
    if (!status) return CSA_ERR_INVALID;
    csa::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status,
                                                                                   waited_ns);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}
