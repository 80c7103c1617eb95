// C ABI entry points of liblf.so: argument validation, per-device context,
// scratch management and dispatch to the kernels.
#include <mutex>

#include "lf_internal.h"

namespace lf {

namespace {
constexpr int kMaxDevices = 64;
DeviceCtx g_devices[kMaxDevices];
std::mutex g_mutex;
}  // namespace

DeviceCtx* current_device(lf_status* st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *st = LF_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceCtx* d = &g_devices[dev];
    if (!d->init) {
        if (cudaDeviceGetAttribute(&d->sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d->cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d->cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            *st = LF_ERR_CUDA;
            return nullptr;
        }
        if (d->cc_major != 10 || d->cc_minor != 0) {
            *st = LF_ERR_UNSUPPORTED_DEVICE;
            return nullptr;
        }
        int* word = nullptr;
        if (cudaMalloc(&word, 256) != cudaSuccess) {
            *st = LF_ERR_CUDA;
            return nullptr;
        }
        int clear = LF_STATUS_CLEAR;
        if (cudaMemcpy(word, &clear, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) {
            cudaFree(word);
            *st = LF_ERR_CUDA;
            return nullptr;
        }
        d->status = word;
        d->ordinal = dev;
        d->init = true;
    }
    *st = LF_OK;
    return d;
}

lf_status ensure_scratch(DeviceCtx* d, size_t bytes) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (bytes <= d->scratch_bytes) return LF_OK;
    if (d->scratch) {
        cudaDeviceSynchronize();  // the old buffer may still be in use
        cudaFree(d->scratch);
        d->scratch = nullptr;
        d->scratch_bytes = 0;
        d->scratch_clean = 0;
    }
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) return LF_ERR_CUDA;
    if (cudaMemset(p, 0, bytes) != cudaSuccess) {
        cudaFree(p);
        return LF_ERR_CUDA;
    }
    d->scratch = p;
    d->scratch_bytes = bytes;
    d->scratch_clean = bytes;
    return LF_OK;
}

lf_status prepare_scratch_counters(DeviceCtx* d, size_t zero_bytes, cudaStream_t stream) {
    // Under stream capture the clear is always recorded: the graph may be
    // replayed after calls of other shapes have written the scratch.
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
        cudaGetLastError();  // not a launch error of this call
        cs = cudaStreamCaptureStatusNone;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (zero_bytes > d->scratch_clean || cs == cudaStreamCaptureStatusActive) {
        // A call of another shape (whose partials reached into this range)
        // or another use of the scratch left other bytes here.
        if (cudaMemsetAsync(d->scratch, 0, zero_bytes, stream) != cudaSuccess) {
            d->scratch_clean = 0;
            return LF_ERR_CUDA;
        }
    }
    d->scratch_clean = zero_bytes;
    return LF_OK;
}

void scratch_dirty(DeviceCtx* d) {
    std::lock_guard<std::mutex> lock(g_mutex);
    d->scratch_clean = 0;
}

lf_status check_shape(int B, int H, int L, int w) {
    if (B <= 0 || H <= 0 || L <= 0 || w <= 0) return LF_ERR_BAD_DIM;
    if (L % w != 0) return LF_ERR_L_NOT_MULTIPLE_OF_W;
    if (L < 2 * w) return LF_ERR_L_LT_2W;
    // Index arithmetic inside the kernels is 32-bit over (sample, head, row).
    if ((long long)B * H * L >= (1LL << 31) || B >= (1 << 23)) return LF_ERR_TOO_LARGE;
    return LF_OK;
}

}  // namespace lf

namespace lf {
namespace {

// lf_attention_forward, and with gidx / gnum also the partition of
// lf_init_global_idx (for fp16 / bf16 inside the attention kernel's launch).
lf_status attention_entry(const void* q, const void* k, const void* v, const void* qg, const void* kg,
                          const void* vg, const float* local_mask, const float* global_mask, int B, int H, int L,
                          int w, lf_dtype dtype, lf_stream_t stream, void* out, int32_t* gidx, int32_t* gnum) {
    if (!q || !k || !v || !qg || !kg || !vg || !local_mask || !global_mask || !out) return LF_ERR_NULL;
    lf_status st = check_shape(B, H, L, w);
    if (st != LF_OK) return st;
    if (dtype != LF_F32 && dtype != LF_F16 && dtype != LF_BF16) return LF_ERR_DTYPE;
    const void* ptrs[] = {q, k, v, qg, kg, vg, local_mask, global_mask, out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return LF_ERR_MISALIGNED;
    if (gidx && (!aligned16(gidx) || !aligned16(gnum))) return LF_ERR_MISALIGNED;
    DeviceCtx* d = current_device(&st);
    if (!d) return st;
    const float scale = 0.125f;  // 1/sqrt(64)
    cudaStream_t s = (cudaStream_t)stream;
    if (dtype == LF_F32)
        return launch_attention_simt_f32((const float*)q, (const float*)k, (const float*)v,
                                         (const float*)qg, (const float*)kg, (const float*)vg,
                                         local_mask, global_mask, B, H, L, w, scale, (float*)out,
                                         d->status, s, nullptr, gidx, gnum);
    st = ensure_scratch(d, attention_tc_scratch_bytes(B, H, L, w));
    if (st != LF_OK) return st;
    st = prepare_scratch_counters(d, attention_tc_scratch_zero_bytes(B, H, L, w), s);
    if (st != LF_OK) return st;
    st = launch_attention_tc(q, k, v, qg, kg, vg, local_mask, global_mask, B, H, L, w, scale, dtype, out,
                             d->scratch, d->status, d->sm_count, s, nullptr, gidx, gnum);
    if (st != LF_OK) scratch_dirty(d);
    return st;
}

}  // namespace
}  // namespace lf

using namespace lf;

extern "C" {

const char* lf_status_string(int s) {
    switch (s) {
        case LF_OK: return "LF_OK";
        case LF_ERR_NULL: return "LF_ERR_NULL: a required pointer is NULL";
        case LF_ERR_BAD_DIM: return "LF_ERR_BAD_DIM: B, H, L and w must be positive";
        case LF_ERR_L_NOT_MULTIPLE_OF_W: return "LF_ERR_L_NOT_MULTIPLE_OF_W: L % w != 0";
        case LF_ERR_L_LT_2W: return "LF_ERR_L_LT_2W: L < 2w";
        case LF_ERR_G_GT_W: return "LF_ERR_G_GT_W: more global tokens than w";
        case LF_ERR_GLOBAL_NOT_PREFIX: return "LF_ERR_GLOBAL_NOT_PREFIX: global tokens are not positions 0..g-1";
        case LF_ERR_DTYPE: return "LF_ERR_DTYPE: unsupported dtype";
        case LF_ERR_MISALIGNED: return "LF_ERR_MISALIGNED: device pointers must be 16-byte aligned";
        case LF_ERR_CUDA: return "LF_ERR_CUDA: CUDA runtime error";
        case LF_ERR_DEVICE_TIMEOUT: return "LF_ERR_DEVICE_TIMEOUT: a bounded device wait expired";
        case LF_ERR_UNSUPPORTED_DEVICE: return "LF_ERR_UNSUPPORTED_DEVICE: needs compute capability 10.0 (B200)";
        case LF_ERR_WORKSPACE: return "LF_ERR_WORKSPACE: workspace missing or too small";
        case LF_ERR_TOO_LARGE: return "LF_ERR_TOO_LARGE: size beyond the supported maximum";
        case LF_ERR_SCRATCH_LIMIT: return "LF_ERR_SCRATCH_LIMIT: shape needs more than the 32 MiB scratch of the no-allocation entry point";
        default: return "unknown lf_status";
    }
}

int lf_version(void) { return 104; }  // 1.4: lf_attention_forward_idx

lf_status lf_device_status(lf_stream_t stream, int reset) {
    lf_status st;
    DeviceCtx* d = current_device(&st);
    if (!d) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return LF_ERR_CUDA;
    int word = LF_STATUS_CLEAR;
    if (cudaMemcpy(&word, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LF_ERR_CUDA;
    if (reset) {
        int clear = LF_STATUS_CLEAR;
        if (cudaMemcpy(d->status, &clear, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return LF_ERR_CUDA;
    }
    return word == LF_STATUS_CLEAR ? LF_OK : (lf_status)(word & 0xff);
}

lf_status lf_init_global_idx(const float* global_mask, int B, int L, int w, int32_t* global_idx,
                             int32_t* global_token_nums, int* max_global_out, lf_stream_t stream) {
    if (!global_mask || !global_idx || !global_token_nums) return LF_ERR_NULL;
    if (B <= 0 || L <= 0 || w <= 0) return LF_ERR_BAD_DIM;
    if (L % w != 0) return LF_ERR_L_NOT_MULTIPLE_OF_W;
    if (L < 2 * w) return LF_ERR_L_LT_2W;
    if ((long long)B * L >= (1LL << 31) || B >= (1 << 23)) return LF_ERR_TOO_LARGE;
    if (!aligned16(global_mask) || !aligned16(global_idx) || !aligned16(global_token_nums))
        return LF_ERR_MISALIGNED;
    lf_status st;
    DeviceCtx* d = current_device(&st);
    if (!d) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (max_global_out) {
        int clear = LF_STATUS_CLEAR;
        if (cudaMemcpyAsync(d->status, &clear, sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess)
            return LF_ERR_CUDA;
    }
    st = launch_global_idx(global_mask, B, L, w, global_idx, global_token_nums, d->status, s);
    if (st != LF_OK || !max_global_out) return st;
    int* nums = new int[B];
    int word = LF_STATUS_CLEAR;
    bool ok = cudaMemcpyAsync(nums, global_token_nums, sizeof(int) * (size_t)B, cudaMemcpyDeviceToHost, s) == cudaSuccess &&
              cudaMemcpyAsync(&word, d->status, sizeof(int), cudaMemcpyDeviceToHost, s) == cudaSuccess &&
              cudaStreamSynchronize(s) == cudaSuccess;
    int mx = 0;
    for (int b = 0; ok && b < B; ++b) mx = nums[b] > mx ? nums[b] : mx;
    delete[] nums;
    if (!ok) return LF_ERR_CUDA;
    *max_global_out = mx;
    return word == LF_STATUS_CLEAR ? LF_OK : (lf_status)(word & 0xff);
}

size_t lf_attention_scratch_bytes(int B, int H, int L, int w, lf_dtype dtype) {
    if (check_shape(B, H, L, w) != LF_OK) return 0;
    if (dtype == LF_F16 || dtype == LF_BF16) return attention_tc_scratch_bytes(B, H, L, w);
    return 0;
}

lf_status lf_attention_forward(const void* q, const void* k, const void* v, const void* qg,
                               const void* kg, const void* vg, const float* local_mask,
                               const float* global_mask, int B, int H, int L, int w, lf_dtype dtype,
                               lf_stream_t stream, void* out) {
    return attention_entry(q, k, v, qg, kg, vg, local_mask, global_mask, B, H, L, w, dtype, stream, out, nullptr,
                           nullptr);
}

lf_status lf_attention_forward_idx(const void* q, const void* k, const void* v, const void* qg,
                                   const void* kg, const void* vg, const float* local_mask,
                                   const float* global_mask, int B, int H, int L, int w, lf_dtype dtype,
                                   lf_stream_t stream, void* out, int32_t* global_idx,
                                   int32_t* global_token_nums) {
    if (!global_idx || !global_token_nums) return LF_ERR_NULL;
    return attention_entry(q, k, v, qg, kg, vg, local_mask, global_mask, B, H, L, w, dtype, stream, out,
                           global_idx, global_token_nums);
}

size_t lf_attention_any_globals_scratch_bytes(int B, int H, int L, int w, lf_dtype dtype) {
    if (check_shape(B, H, L, w) != LF_OK) return 0;
    const bool tc = dtype == LF_F16 || dtype == LF_BF16;
    return (tc ? attention_tc_scratch_bytes(B, H, L, w) : 0) + any_globals_bytes(B, H, L, w, tc);
}

lf_status lf_attention_forward_any_globals(const void* q, const void* k, const void* v, const void* qg,
                                           const void* kg, const void* vg, const float* local_mask,
                                           const float* global_mask, int B, int H, int L, int w,
                                           lf_dtype dtype, lf_stream_t stream, void* out) {
    if (!q || !k || !v || !qg || !kg || !vg || !local_mask || !global_mask || !out) return LF_ERR_NULL;
    lf_status st = check_shape(B, H, L, w);
    if (st != LF_OK) return st;
    if (dtype != LF_F32 && dtype != LF_F16 && dtype != LF_BF16) return LF_ERR_DTYPE;
    const void* ptrs[] = {q, k, v, qg, kg, vg, local_mask, global_mask, out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return LF_ERR_MISALIGNED;
    DeviceCtx* d = current_device(&st);
    if (!d) return st;
    const float scale = 0.125f;  // 1/sqrt(64)
    cudaStream_t s = (cudaStream_t)stream;
    const bool tc = dtype != LF_F32;
    // scratch: [attention scratch (16-bit)][partition outputs + slot buffers]
    const size_t att = tc ? attention_tc_scratch_bytes(B, H, L, w) : 0;
    st = ensure_scratch(d, att + any_globals_bytes(B, H, L, w, tc));
    if (st != LF_OK) return st;
    const AnyGlobals a = any_globals_layout(static_cast<uint8_t*>(d->scratch) + att, B, H, L, w, tc);
    if (tc) {
        st = prepare_scratch_counters(d, attention_tc_scratch_zero_bytes(B, H, L, w), s);
        if (st != LF_OK) return st;
    } else {
        scratch_dirty(d);  // the partition's outputs start at the scratch's first byte
    }
    if (!tc) {
        st = launch_global_idx(global_mask, B, L, w, const_cast<int32_t*>(a.global_idx),
                               const_cast<int32_t*>(a.global_token_nums), d->status, s,
                               const_cast<int32_t*>(a.rank), false);
        if (st != LF_OK) return st;
        return launch_attention_simt_f32((const float*)q, (const float*)k, (const float*)v,
                                         (const float*)qg, (const float*)kg, (const float*)vg,
                                         local_mask, global_mask, B, H, L, w, scale, (float*)out,
                                         d->status, s, &a);
    }
    // partition + gather of the global tokens' rows in one launch
    st = launch_partition_gather(global_mask, local_mask, qg, k, v, a, B, H, L, w, d->status, s);
    if (st == LF_OK)
        st = launch_attention_tc(q, k, v, qg, kg, vg, local_mask, global_mask, B, H, L, w, scale, dtype, out,
                                 d->scratch, d->status, d->sm_count, s, &a);
    if (st != LF_OK) scratch_dirty(d);
    return st;
}

lf_status lf_release_scratch(void) {
    lf_status st;
    DeviceCtx* d = current_device(&st);
    if (!d) return st;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (d->scratch) {
        if (cudaDeviceSynchronize() != cudaSuccess) return LF_ERR_CUDA;
        cudaFree(d->scratch);
        d->scratch = nullptr;
        d->scratch_bytes = 0;
        d->scratch_clean = 0;
    }
    return LF_OK;
}

}  // extern "C"
