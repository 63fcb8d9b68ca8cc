// selftest.cu -- exercises the bounded mbarrier wait used by every kernel:
// one CTA waits on a barrier that nobody arrives at and must give up after the
// given limit, recording LKA_ERR_TIMEOUT in the workspace status word.
#include "common.cuh"
#include "host_util.h"

namespace lka {

__global__ void wait_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
    __shared__ alignas(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, status, limit_ns);  // nobody arrives: runs out
    __syncthreads();
}

}  // namespace lka

extern "C" lka_status_t lka_selftest_wait_timeout(void* ws, size_t ws_bytes, int limit_us, void* stream) {
    if (!ws || ws_bytes < lka::kWsHeaderBytes) return LKA_ERR_WORKSPACE;
    if (limit_us < 1 || limit_us > 1000000) return LKA_ERR_INVALID_ARG;
    lka::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<uint32_t*>(ws),
                                                                  (uint64_t)limit_us * 1000ull);
    return cudaPeekAtLastError() == cudaSuccess ? LKA_OK : LKA_ERR_CUDA;
}
