// Bounded-wait self-test: checks, on the device, the path every pipeline wait
// of the library takes when its barrier phase never completes.
//
// One thread initialises an mbarrier that expects one arrival and waits for its
// first phase, which nothing ever completes (no copy, no MMA, no other thread
// signals it). The wait gives up after the given limit, records
// PISA_ERR_TIMEOUT with its site in the workspace status word, and the kernel
// returns; pisa_check_status then reports it and the context stays usable. No
// asynchronous operation is in flight when the kernel exits.
#include <cuda_runtime.h>

#include "pisa.h"
#include "pisa_device.cuh"

namespace pisa {

__global__ void __launch_bounds__(32) selftest_wait_kernel(uint32_t* status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait(&bar, 0, status, (kKernSelftest << 8) | 0x01u, limit_ns);
}

}  // namespace pisa

using namespace pisa;

extern "C" pisa_status pisa_selftest_wait_timeout(void* ws, uint32_t limit_us, pisa_stream_t stream) {
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 15u) != 0) return PISA_ERR_INVALID_ARG;
    if (limit_us == 0 || limit_us > 1000000u) return PISA_ERR_INVALID_ARG;
    if (injected_launch_failure()) return PISA_ERR_CUDA;
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(ws),
                                                                               uint64_t(limit_us) * 1000u);
    return cudaGetLastError() == cudaSuccess ? PISA_OK : PISA_ERR_CUDA;
}
