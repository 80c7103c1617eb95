// LayerNorm of the AddBiasResidualLayerNorm steps (FasterTransformer
// Longformer page, §Longformer Encoder 计算流程 / 每个 Transformer 层 steps 5
// and 6): the GEMM epilogue has already added bias and residual into an fp32
// row; this kernel normalises each row with the population variance,
// y = gamma * (z - mean) / sqrt(var + eps) + beta, and rounds to the dtype.
// One warp per row, the row held in registers; HBM-bound (4 bytes read and
// 2 written per element).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "lf_internal.h"

namespace lf {
namespace {

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <typename T, int VPL>
__global__ void __launch_bounds__(256) layernorm_kernel(const float* __restrict__ z, const float* __restrict__ gamma,
                                                        const float* __restrict__ beta, int rows, int N, float eps,
                                                        T* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const float* zr = z + (size_t)row * N;
    float v[VPL];
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        v[k] = zr[k * 32 + lane];
        s += v[k];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / (float)N;
    float q = 0.0f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const float d = v[k] - mean;
        q = fmaf(d, d, q);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float inv = rsqrtf(q / (float)N + eps);
    T* orow = out + (size_t)row * N;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int c = k * 32 + lane;
        orow[c] = from_f<T>(fmaf((v[k] - mean) * inv, gamma[c], beta[c]));
    }
}

template <typename T>
lf_status launch_t(const float* z, const float* gamma, const float* beta, int rows, int N, float eps, void* out,
                   cudaStream_t stream) {
    const int blocks = (rows + 7) / 8;
    T* o = reinterpret_cast<T*>(out);
    switch (N / 32) {
        case 4: layernorm_kernel<T, 4><<<blocks, 256, 0, stream>>>(z, gamma, beta, rows, N, eps, o); break;
        case 8: layernorm_kernel<T, 8><<<blocks, 256, 0, stream>>>(z, gamma, beta, rows, N, eps, o); break;
        case 12: layernorm_kernel<T, 12><<<blocks, 256, 0, stream>>>(z, gamma, beta, rows, N, eps, o); break;
        case 16: layernorm_kernel<T, 16><<<blocks, 256, 0, stream>>>(z, gamma, beta, rows, N, eps, o); break;
        case 20: layernorm_kernel<T, 20><<<blocks, 256, 0, stream>>>(z, gamma, beta, rows, N, eps, o); break;
        case 24: layernorm_kernel<T, 24><<<blocks, 256, 0, stream>>>(z, gamma, beta, rows, N, eps, o); break;
        case 28: layernorm_kernel<T, 28><<<blocks, 256, 0, stream>>>(z, gamma, beta, rows, N, eps, o); break;
        case 32: layernorm_kernel<T, 32><<<blocks, 256, 0, stream>>>(z, gamma, beta, rows, N, eps, o); break;
        default: return LF_ERR_BAD_DIM;
    }
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

}  // namespace

lf_status launch_layernorm(const float* z, const float* gamma, const float* beta, int rows, int N, float eps,
                           lf_dtype dtype, void* out, cudaStream_t stream) {
    if (dtype == LF_F16) return launch_t<__half>(z, gamma, beta, rows, N, eps, out, stream);
    if (dtype == LF_BF16) return launch_t<__nv_bfloat16>(z, gamma, beta, rows, N, eps, out, stream);
    return LF_ERR_DTYPE;
}

}  // namespace lf
