// lf_selftest_bounded_wait: a check of the failure path that every bounded
// device wait of this library takes when it gives up.
//
// One CTA initialises an mbarrier and waits, with the same bounded-wait
// routine the attention and GEMM kernels use, for a phase that nothing ever
// completes.  The wait gives up after the caller's limit, the CTA records
// LF_ERR_DEVICE_TIMEOUT in the device status word and returns.  Nothing else
// is in flight in that CTA (no copy, no tensor-core work, no aligned
// collective instruction), so giving up leaves nothing behind.
#include "lf_internal.h"
#include "sm100.cuh"

namespace lf {
namespace {

// Accepted wait limits: 1 us to 100 ms.
constexpr unsigned long long kSelftestMinWaitNs = 1000ull;
constexpr unsigned long long kSelftestMaxWaitNs = 100000000ull;

__global__ void bounded_wait_kernel(unsigned long long limit_ns, int* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
    // Phase 0 never completes: no thread arrives on the barrier.
    const bool done = sm100::mbar_wait(&bar, 0, &abort_flag, limit_ns);
    if (!done) record_status(status, 0, LF_ERR_DEVICE_TIMEOUT);
}

}  // namespace
}  // namespace lf

using namespace lf;

extern "C" lf_status lf_selftest_bounded_wait(unsigned long long limit_ns, lf_stream_t stream) {
    if (limit_ns < kSelftestMinWaitNs || limit_ns > kSelftestMaxWaitNs) return LF_ERR_BAD_DIM;
    lf_status st;
    DeviceCtx* d = current_device(&st);
    if (!d) return st;
    bounded_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns, d->status);
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}
