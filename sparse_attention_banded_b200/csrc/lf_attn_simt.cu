// fp32 Longformer attention on the CUDA cores (exact FP32 FMA, expf).
//
// FasterTransformer Longformer page, §Longformer Encoder 计算流程 / 每个
// Transformer 层 steps 3-5.  fp32 inputs have no tensor-core path that keeps
// the 1e-4 error bound, so this kernel computes the same function as the
// tensor-core kernel with plain FMAs:
//   one warp per output row (b, h, i); the row's key set is walked in chunks
//   of 32 keys (lane = key) with an online softmax; lane c then owns output
//   channels c and c + 32.
// Key set (local row i >= g_b): [0, g_b) then [max(i - w, g_b), min(i + w,
// L - 1)], each key once; global row i < g_b: [0, L) with qg/kg/vg.  Score
// = scale * <q_i, k_j> + lb[j], lb[j] = fmaf(local_mask[j], 1e4, -1e4).
#include "lf_internal.h"

namespace lf {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Number of leading 0.0 entries of global_mask[b, :], capped at w + 1.
__device__ int leading_globals(const float* gm_row, int L, int w, int lane) {
    const int cap = min(w + 1, L);
    for (int c0 = 0; c0 < cap; c0 += 32) {
        const int j = c0 + lane;
        const bool nonzero = j < cap && gm_row[j] != 0.0f;
        const unsigned m = __ballot_sync(0xffffffffu, nonzero);
        if (m) return c0 + __ffs(m) - 1;
    }
    return cap;
}

struct RowState {
    float m, l, o0, o1;
};

// Process keys [j_begin, j_end] (inclusive) of one row.
__device__ __forceinline__ void process_range(RowState& st, const float* sq, const float* K, const float* V,
                                              const float* lm_row, int j_begin, int j_end, float scale,
                                              int lane) {
    for (int base = j_begin; base <= j_end; base += 32) {
        const int j = base + lane;
        const bool valid = j <= j_end;
        float s = -INFINITY;
        if (valid) {
            const float4* kr = reinterpret_cast<const float4*>(K + (size_t)j * 64);
            float acc = 0.0f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float4 kv = kr[c];
                acc = fmaf(sq[4 * c + 0], kv.x, acc);
                acc = fmaf(sq[4 * c + 1], kv.y, acc);
                acc = fmaf(sq[4 * c + 2], kv.z, acc);
                acc = fmaf(sq[4 * c + 3], kv.w, acc);
            }
            s = fmaf(acc, scale, fmaf(lm_row[j], 10000.0f, -10000.0f));
        }
        const float m_new = fmaxf(st.m, warp_max(s));
        const float alpha = (st.m == -INFINITY) ? 0.0f : expf(st.m - m_new);
        const float p = valid ? expf(s - m_new) : 0.0f;
        st.l = st.l * alpha + warp_sum(p);
        st.o0 *= alpha;
        st.o1 *= alpha;
        const int n = min(32, j_end - base + 1);
        for (int t = 0; t < n; ++t) {
            const float pt = __shfl_sync(0xffffffffu, p, t);
            const float* vr = V + (size_t)(base + t) * 64;
            st.o0 = fmaf(pt, vr[lane], st.o0);
            st.o1 = fmaf(pt, vr[lane + 32], st.o1);
        }
        st.m = m_new;
    }
}

__global__ void __launch_bounds__(kWarps * 32)
attention_simt_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                      const float* __restrict__ qg, const float* __restrict__ kg,
                      const float* __restrict__ vg, const float* __restrict__ local_mask,
                      const float* __restrict__ global_mask, int B, int H, int L, int w, float scale,
                      float* __restrict__ out, int* status) {
    __shared__ __align__(16) float sq_all[kWarps][64];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    float* sq = sq_all[wid];
    const long long total = (long long)B * H * L;
    const long long nwarps = (long long)gridDim.x * kWarps;
    for (long long r = (long long)blockIdx.x * kWarps + wid; r < total; r += nwarps) {
        const int i = (int)(r % L);
        const int h = (int)((r / L) % H);
        const int b = (int)(r / ((long long)L * H));
        const float* lm_row = local_mask + (size_t)b * L;
        const float* gm_row = global_mask + (size_t)b * L;
        float* o = out + (((size_t)b * L + i) * H + h) * 64;

        const int g = leading_globals(gm_row, L, w, lane);
        const bool bad_sample = g > w;
        if (bad_sample && lane == 0 && h == 0 && i == 0) record_status(status, b, LF_ERR_G_GT_W);
        if (!bad_sample && i >= g && gm_row[i] == 0.0f && lane == 0 && h == 0)
            record_status(status, b, LF_ERR_GLOBAL_NOT_PREFIX);
        if (bad_sample || fmaf(lm_row[i], 10000.0f, -10000.0f) != 0.0f) {
            o[lane] = 0.0f;
            o[lane + 32] = 0.0f;
            continue;
        }
        const bool global_row = i < g;
        const size_t head = ((size_t)b * H + h) * (size_t)L * 64;
        const float* Q = (global_row ? qg : q) + head;
        const float* K = (global_row ? kg : k) + head;
        const float* V = (global_row ? vg : v) + head;
        sq[lane] = Q[(size_t)i * 64 + lane];
        sq[lane + 32] = Q[(size_t)i * 64 + lane + 32];
        __syncwarp();

        RowState st{-INFINITY, 0.0f, 0.0f, 0.0f};
        if (global_row) {
            process_range(st, sq, K, V, lm_row, 0, L - 1, scale, lane);
        } else {
            const int lo = max(i - w, g), hi = min(i + w, L - 1);
            if (g > 0) process_range(st, sq, K, V, lm_row, 0, g - 1, scale, lane);
            process_range(st, sq, K, V, lm_row, lo, hi, scale, lane);
        }
        const float inv = 1.0f / st.l;
        o[lane] = st.o0 * inv;
        o[lane + 32] = st.o1 * inv;
        __syncwarp();
    }
}

}  // namespace

lf_status launch_attention_simt_f32(const float* q, const float* k, const float* v, const float* qg,
                                    const float* kg, const float* vg, const float* local_mask,
                                    const float* global_mask, int B, int H, int L, int w, float scale,
                                    float* out, int* status, cudaStream_t stream) {
    const long long rows = (long long)B * H * L;
    long long blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 148 * 16) blocks = 148 * 16;
    attention_simt_kernel<<<(int)blocks, kWarps * 32, 0, stream>>>(q, k, v, qg, kg, vg, local_mask, global_mask,
                                                                  B, H, L, w, scale, out, status);
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

}  // namespace lf
