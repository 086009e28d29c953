// kvattn_selftest_bounded_wait: the bounded mbarrier wait of the decode
// kernels, exercised on the device.  One wait must see a completed phase; the
// other waits on a barrier nothing arrives on and must give up after its cap,
// set the timeout bit and return, leaving the context usable.
#include "kvattn_internal.cuh"
#include "sm100.cuh"

namespace kvattn {
namespace {

__global__ void __launch_bounds__(32) bounded_wait_kernel(int *result, uint32_t tries)
{
    __shared__ __align__(8) uint64_t bars[2];
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);      // completed below
        mbar_init(&bars[1], 1);      // never arrived on
        fence_mbar_init();
        mbar_arrive(&bars[0]);
        if (!mbar_wait(&bars[0], 0, tries))
            atomicOr(result, KVATTN_SELFTEST_MISSED_PHASE);
        if (!mbar_wait(&bars[1], 0, tries))
            raise_error(result, KVATTN_DEVERR_WAIT_TIMEOUT);
    }
    __syncwarp();
}

}  // namespace
}  // namespace kvattn

extern "C" int kvattn_selftest_bounded_wait(int32_t *result, int32_t tries, void *stream)
{
    if (!result || tries < 1 || tries > 65536)
        return KVATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(result) % 4)
        return KVATTN_ERR_MISALIGNED;
    kvattn::bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(result, (uint32_t)tries);
    return cudaGetLastError() == cudaSuccess ? KVATTN_OK : KVATTN_ERR_CUDA;
}
