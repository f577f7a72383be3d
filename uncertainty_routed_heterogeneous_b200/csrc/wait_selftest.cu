// wait_selftest.cu -- exercises the bounded-wait path every kernel relies on.
//
// The attention kernel's threads wait on mbarriers (TMA arrivals, MMA
// commits, other warps); each wait gives up after a wall-time limit or as
// soon as another thread of the CTA has raised the abort flag, and the kernel
// then reports HETA_ERR_TIMEOUT and returns.  This kernel makes that happen
// on purpose, with no fault and nothing left in flight: warp 0 waits on a
// barrier nothing arrives on until its (short) limit, then raises the flag
// and the status; warp 1 waits on another dead barrier with a limit far
// longer than the test (5 s) and must be released by the flag.  The paper has no
// counterpart; it is a test hook of this library.
#include "heta_internal.cuh"
#include "ptx_sm100.cuh"

namespace heta {
namespace {

using namespace ptx;

__global__ void __launch_bounds__(64, 1)
wait_selftest_kernel(uint64_t limit_ns, int32_t *status, unsigned long long *elapsed_ns)
{
    __shared__ uint64_t dead[2];
    __shared__ int abort;
    const int tid = threadIdx.x;
    if (tid == 0) {
        mbar_init(smem_addr(&dead[0]), 1);
        mbar_init(smem_addr(&dead[1]), 1);
        abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const uint64_t t0 = globaltimer_ns();
    if (tid == 0) {
        if (!mbar_wait(smem_addr(&dead[0]), 0, &abort, limit_ns)) {
            atomicExch(&abort, 1);
            raise_status(status, HETA_ERR_TIMEOUT);
        }
    } else if (tid == 32) {
        // released by the abort flag, not by its own 5 s limit
        mbar_wait(smem_addr(&dead[1]), 0, &abort, 5ull * 1000000000ull);
    }
    __syncthreads();
    if (tid == 0 && elapsed_ns) *elapsed_ns = globaltimer_ns() - t0;
}

}  // namespace
}  // namespace heta

extern "C" {

HETA_API heta_status heta_selftest_wait_timeout(uint64_t limit_ns, int32_t *status_dev,
                                                unsigned long long *elapsed_ns_dev,
                                                void *stream)
{
    if (limit_ns == 0 || limit_ns > 10ull * 1000000000ull || !status_dev)
        return HETA_ERR_INVALID_ARG;
    heta::wait_selftest_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(
        limit_ns, status_dev, elapsed_ns_dev);
    return cudaGetLastError() == cudaSuccess ? HETA_OK : HETA_ERR_CUDA;
}

}  // extern "C"
