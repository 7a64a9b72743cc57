// selftest.cu -- kda_selftest_device_timeout: exercises the bounded-wait failure path.
//
// Every mbarrier wait in the library's kernels gives up after a time limit, records
// KDA_ERR_DEVICE_TIMEOUT in the per-device status word and lets the kernel return, so a
// broken pipeline ends with an error the host can read instead of a hung GPU.  This entry
// point makes that path observable without breaking anything: one thread initialises an
// mbarrier that expects one arrival which never comes, and waits on it with a short limit.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

__global__ void timeout_kernel(unsigned long long limit_ns, unsigned int *status)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0)
        return;
    mbar_init(&bar, 1);
    fence_mbar_init_cluster();
    mbar_wait_bounded(&bar, 0, status, limit_ns);  // nothing arrives: runs out after limit_ns
}

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" kda_status kda_selftest_device_timeout(uint32_t limit_us, kda_stream_t stream)
{
    if (limit_us < 1 || limit_us > 2000000u)
        return KDA_ERR_INVALID_ARG;
    unsigned int *status = device_status_ptr();
    if (!status)
        return KDA_ERR_CUDA;
    timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned long long)limit_us * 1000ull, status);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
