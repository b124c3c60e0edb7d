// Failure-detection self-test: one thread waits, with the same bounded mbarrier wait every
// tensor-core kernel uses, on a phase that nothing completes.  When the wait gives up it
// records a timeout in the device status word, as a kernel that lost a transfer would, and
// the block returns; nothing faults and the context stays usable.
#include "gdn2_internal.cuh"
#include "tc_util.cuh"

namespace gdn2 {
namespace {

__global__ void selftest_timeout_kernel(int *status, unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    tc::mbar_init(&bar, 1);  // one arrival expected; none ever comes
    tc::fence_mbar_init();
    if (!tc::mbar_wait(&bar, 0, limit_ns)) atomicExch(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_selftest_timeout(int limit_us, int *status, cudaStream_t s)
{
    selftest_timeout_kernel<<<1, 32, 0, s>>>(status, (unsigned long long)limit_us * 1000ull);
    return cudaGetLastError();
}

}  // namespace gdn2
