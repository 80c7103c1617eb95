// LayerNorm of the AddBiasResidualLayerNorm steps (FasterTransformer
// Longformer page, §Longformer Encoder 计算流程 / 每个 Transformer 层 steps 5
// and 6): the GEMM epilogue has already added bias and residual into an fp32
// row; this kernel normalises each row with the population variance,
// y = gamma * (z - mean) / sqrt(var + eps) + beta, and rounds to the dtype.
// One warp per row, the row held in registers (16-byte loads, 8-byte
// stores); memory-bound (4 bytes read and 2 written per element).
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

template <typename T>
__device__ __forceinline__ uint32_t pack2(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// VPL = N / 128: lane l holds columns 4 (k 32 + l) .. +3 for k < VPL, read
// and written with 16- and 8-byte accesses.
template <typename T, int VPL>
__global__ void __launch_bounds__(256) layernorm_kernel(const float* __restrict__ z, const float* __restrict__ gamma,
                                                        const float* __restrict__ beta, int rows, int N, float eps,
                                                        T* __restrict__ out) {
    // Let the next kernel in the stream be scheduled; wait for the one before
    // (launched as a programmatic dependent) before touching memory.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const float4* zr = reinterpret_cast<const float4*>(z + (size_t)row * N);
    float4 v[VPL];
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        v[k] = zr[k * 32 + lane];
        s += (v[k].x + v[k].y) + (v[k].z + v[k].w);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / (float)N;
    float q = 0.0f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const float a = v[k].x - mean, b = v[k].y - mean, c = v[k].z - mean, d = v[k].w - mean;
        q = fmaf(a, a, fmaf(b, b, fmaf(c, c, fmaf(d, d, q))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float inv = rsqrtf(q / (float)N + eps);
    uint2* orow = reinterpret_cast<uint2*>(out + (size_t)row * N);
    const float4* g4 = reinterpret_cast<const float4*>(gamma);
    const float4* b4 = reinterpret_cast<const float4*>(beta);
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int c = k * 32 + lane;
        const float4 g = g4[c], bb = b4[c];
        uint2 u;
        u.x = pack2<T>(fmaf((v[k].x - mean) * inv, g.x, bb.x), fmaf((v[k].y - mean) * inv, g.y, bb.y));
        u.y = pack2<T>(fmaf((v[k].z - mean) * inv, g.z, bb.z), fmaf((v[k].w - mean) * inv, g.w, bb.w));
        orow[c] = u;
    }
}

template <typename T>
lf_status launch_t(const float* z, const float* gamma, const float* beta, int rows, int N, float eps, void* out,
                   cudaStream_t stream) {
    const int blocks = (rows + 7) / 8;
    T* o = reinterpret_cast<T*>(out);
    void (*kern)(const float*, const float*, const float*, int, int, float, T*);
    switch (N / 128) {
        case 1: kern = layernorm_kernel<T, 1>; break;
        case 2: kern = layernorm_kernel<T, 2>; break;
        case 3: kern = layernorm_kernel<T, 3>; break;
        case 4: kern = layernorm_kernel<T, 4>; break;
        case 5: kern = layernorm_kernel<T, 5>; break;
        case 6: kern = layernorm_kernel<T, 6>; break;
        case 7: kern = layernorm_kernel<T, 7>; break;
        case 8: kern = layernorm_kernel<T, 8>; break;
        default: return LF_ERR_BAD_DIM;
    }
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, z, gamma, beta, rows, N, eps, o) != cudaSuccess) return LF_ERR_CUDA;
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
