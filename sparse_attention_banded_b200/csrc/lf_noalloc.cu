// lf_attention_forward_noalloc: the tensor-core attention path for callers
// that must not allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code running inside another
// framework's memory pool that forbids outside allocations, allocation-free
// real-time or embedded paths, or callers that must not add allocations of
// their own to an externally budgeted device.  The regular lf_attention_forward
// grows a library-owned scratch buffer with cudaMalloc; this variant instead
// takes its scratch from a fixed array that is part of the library's device
// image.
#include <mutex>

#include "lf_internal.h"

namespace lf {
namespace {

// Scratch of the no-allocation path: 32 MiB on every device that runs it
// (it covers, for example, 32 heads at L = 4096 and w = 256).
constexpr size_t kNoAllocScratchBytes = 32ull << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
// Device status word of this path (same encoding as the library's word).
static __device__ __align__(256) int g_noalloc_status = LF_STATUS_CLEAR;

struct NoAllocDevice {
    bool ready = false;
    void* scratch = nullptr;  // device address of g_noalloc_scratch
    int* status = nullptr;    // device address of g_noalloc_status
    int sm_count = 0;
};
NoAllocDevice g_noalloc[64];
std::mutex g_noalloc_mutex;

// Once per device, with that device current: resolve the arrays' device
// addresses.  In host code the array names are host-side stand-ins, never
// device addresses, so the kernel only ever gets what cudaGetSymbolAddress
// returns.
lf_status noalloc_device(NoAllocDevice** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LF_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoAllocDevice* d = &g_noalloc[dev];
    if (!d->ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return LF_ERR_CUDA;
        if (major != 10 || minor != 0) return LF_ERR_UNSUPPORTED_DEVICE;
        void* scratch = nullptr;
        void* status = nullptr;
        if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess) return LF_ERR_CUDA;
        if (cudaGetSymbolAddress(&status, g_noalloc_status) != cudaSuccess) return LF_ERR_CUDA;
        d->scratch = scratch;
        d->status = static_cast<int*>(status);
        d->sm_count = sms;
        d->ready = true;
    }
    *out = d;
    return LF_OK;
}

}  // namespace
}  // namespace lf

using namespace lf;

extern "C" lf_status lf_attention_forward_noalloc(const void* q, const void* k, const void* v, const void* qg,
                                                  const void* kg, const void* vg, const float* local_mask,
                                                  const float* global_mask, int B, int H, int L, int w,
                                                  lf_dtype dtype, lf_stream_t stream, void* out) {
    if (!q || !k || !v || !qg || !kg || !vg || !local_mask || !global_mask || !out) return LF_ERR_NULL;
    lf_status st = check_shape(B, H, L, w);
    if (st != LF_OK) return st;
    if (dtype != LF_F16 && dtype != LF_BF16) return LF_ERR_DTYPE;
    const void* ptrs[] = {q, k, v, qg, kg, vg, local_mask, global_mask, out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return LF_ERR_MISALIGNED;
    if (attention_tc_scratch_bytes(B, H, L, w) > kNoAllocScratchBytes) return LF_ERR_SCRATCH_LIMIT;
    NoAllocDevice* d = nullptr;
    st = noalloc_device(&d);
    if (st != LF_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // The array keeps the previous call's contents: the scheduler and split
    // counters must start at zero, so clear them (a memset, no allocation).
    if (cudaMemsetAsync(d->scratch, 0, attention_tc_scratch_zero_bytes(B, H, L, w), s) != cudaSuccess)
        return LF_ERR_CUDA;
    return launch_attention_tc(q, k, v, qg, kg, vg, local_mask, global_mask, B, H, L, w, 0.125f, dtype, out,
                               d->scratch, d->status, d->sm_count, s);
}

extern "C" lf_status lf_noalloc_device_status(lf_stream_t stream, int reset) {
    NoAllocDevice* d = nullptr;
    lf_status st = noalloc_device(&d);
    if (st != LF_OK) return st;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return LF_ERR_CUDA;
    int word = LF_STATUS_CLEAR;
    if (cudaMemcpy(&word, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LF_ERR_CUDA;
    if (reset) {
        const int clear = LF_STATUS_CLEAR;
        if (cudaMemcpy(d->status, &clear, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return LF_ERR_CUDA;
    }
    return word == LF_STATUS_CLEAR ? LF_OK : (lf_status)(word & 0xff);
}
