// fp32 Longformer attention on the CUDA cores (exact FP32 FMA, expf).
//
// FasterTransformer Longformer page, §Longformer Encoder 计算流程 / 每个
// Transformer 层 steps 3-5.  fp32 inputs have no tensor-core path that keeps
// the 1e-4 error bound, so this kernel computes the same function as the
// tensor-core kernel with plain FMAs:
//   one CTA per output row (b, h, i); its warps walk interleaved chunks of
//   32 keys of the row's key set (lane = key) with an online softmax each,
//   lane c owning output channels c and c + 32, and the partial results are
//   merged (log-sum-exp) in shared memory.
// Key set (local row i >= g_b): [0, g_b) then [max(i - w, g_b), min(i + w,
// L - 1)], each key once; global row i < g_b: [0, L) with qg/kg/vg.  Score
// = scale * <q_i, k_j> + lb[j], lb[j] = fmaf(local_mask[j], 1e4, -1e4).
// Global tokens at any position (the HuggingFace arrangement that the page's
// §使用前提 item 4 sets apart): a row is global iff global_mask[i] == 0.0; a
// local row's list is the sample's global positions global_idx[b, 0..g_b)
// then its window [max(i - w, 0), min(i + w, L - 1)], where window keys that
// are global are skipped (each key once).
#include "lf_internal.h"
#include "lf_partition.cuh"

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

// Keys at list positions [pos0, pos0 + 32) of one row (lane = key): the
// row's key list is [0, g_seg) followed by [lo, hi], each key once.  With
// kAny (global tokens at any position) the first g_seg entries are
// gl[0..g_seg), and for a local row (skip_g) window keys with gm_row[j] == 0
// (global, already listed) are skipped; a global row keeps all of [0, L).
template <bool kAny>
__device__ __forceinline__ void process_chunk(RowState& st, const float* sq, const float* K, const float* V,
                                              const float* lm_row, int pos0, int g_seg, int lo, int n_keys,
                                              float scale, int lane, const int32_t* gl, const float* gm_row,
                                              bool skip_g) {
    const int pos = pos0 + lane;
    bool valid = pos < n_keys;
    int j = valid ? (pos < g_seg ? (kAny ? gl[pos] : pos) : lo + (pos - g_seg)) : 0;
    if (kAny && skip_g && valid && pos >= g_seg && gm_row[j] == 0.0f) {
        valid = false;
        j = 0;
    }
    float s = -INFINITY;
    if (valid) {
        const float4* kr = reinterpret_cast<const float4*>(K + (size_t)j * 64);
        // four partial sums over interleaved columns, added at the end
        float a4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const float4 kv = kr[c];
            a4[c & 3] = fmaf(sq[4 * c + 0], kv.x, a4[c & 3]);
            a4[c & 3] = fmaf(sq[4 * c + 1], kv.y, a4[c & 3]);
            a4[c & 3] = fmaf(sq[4 * c + 2], kv.z, a4[c & 3]);
            a4[c & 3] = fmaf(sq[4 * c + 3], kv.w, a4[c & 3]);
        }
        const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
        s = fmaf(acc, scale, fmaf(lm_row[j], 10000.0f, -10000.0f));
    }
    const float m_new = fmaxf(st.m, warp_max(s));
    const float alpha = (st.m == -INFINITY) ? 0.0f : expf(st.m - m_new);
    const float p = valid ? expf(s - m_new) : 0.0f;
    st.l = st.l * alpha + warp_sum(p);
    st.o0 *= alpha;
    st.o1 *= alpha;
    // fixed trip count so that the V-row loads are issued together; keys
    // past the end have p = 0 and read key 0
#pragma unroll 8
    for (int t = 0; t < 32; ++t) {
        const float pt = __shfl_sync(0xffffffffu, p, t);
        const int jt = __shfl_sync(0xffffffffu, j, t);
        const float* vr = V + (size_t)jt * 64;
        st.o0 = fmaf(pt, vr[lane], st.o0);
        st.o1 = fmaf(pt, vr[lane + 32], st.o1);
    }
    st.m = m_new;
}

// One CTA per output row (b, h, i): the kWarps warps take interleaved
// 32-key chunks of the row's key list (warp w: chunks w, w + kWarps, ...),
// each with its own online softmax, and warp 0 merges the partial (m, l, o)
// through shared memory.  Many short chains per SM instead of one long one
// keep the L2 latency of the K/V rows hidden, global rows included.
template <bool kAny>
__global__ void __launch_bounds__(kWarps * 32, 4)
attention_simt_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                      const float* __restrict__ qg, const float* __restrict__ kg,
                      const float* __restrict__ vg, const float* __restrict__ local_mask,
                      const float* __restrict__ global_mask, int B, int H, int L, int w, float scale,
                      float* __restrict__ out, int* status, const int32_t* __restrict__ gidx,
                      const int32_t* __restrict__ gnum, int32_t* __restrict__ gidx_out,
                      int32_t* __restrict__ gnum_out) {
    __shared__ __align__(16) float sq[64];
    __shared__ float part_ml[kWarps][2];
    __shared__ float part_o[kWarps][64];
    __shared__ int part_sm[5];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    // Prefix instance, optional: the global-index partition in the same
    // launch, sample b by the first four warps of CTA b (the other warps
    // wait for them at the first row's barrier).
    if (!kAny && gidx_out && wid < 4)
        for (int b = blockIdx.x; b < B; b += gridDim.x)
            partition_sample(global_mask + (size_t)b * L, L, w, gidx_out + (size_t)b * L, gnum_out + b, b, status,
                             threadIdx.x, wid, lane, part_sm);
    const long long total = (long long)B * H * L;
    for (long long r = blockIdx.x; r < total; r += gridDim.x) {
        const int i = (int)(r % L);
        const int h = (int)((r / L) % H);
        const int b = (int)(r / ((long long)L * H));
        const float* lm_row = local_mask + (size_t)b * L;
        const float* gm_row = global_mask + (size_t)b * L;
        float* o = out + (((size_t)b * L + i) * H + h) * 64;

        // gidx: global tokens at any position, g from the partition
        const int g = kAny ? gnum[b] : leading_globals(gm_row, L, w, lane);  // same in every warp
        const bool bad_sample = g > w;
        const int32_t* gl = kAny ? gidx + (size_t)b * L : nullptr;
        if (wid == 0) {
            if (bad_sample && lane == 0 && h == 0 && i == 0) record_status(status, b, LF_ERR_G_GT_W);
            if (!kAny && !bad_sample && i >= g && gm_row[i] == 0.0f && lane == 0 && h == 0)
                record_status(status, b, LF_ERR_GLOBAL_NOT_PREFIX);
        }
        if (bad_sample || fmaf(lm_row[i], 10000.0f, -10000.0f) != 0.0f) {
            if (wid == 0) {
                o[lane] = 0.0f;
                o[lane + 32] = 0.0f;
            }
            continue;  // uniform over the CTA
        }
        const bool global_row = kAny ? gm_row[i] == 0.0f : i < g;
        const size_t head = ((size_t)b * H + h) * (size_t)L * 64;
        const float* Q = (global_row ? qg : q) + head;
        const float* K = (global_row ? kg : k) + head;
        const float* V = (global_row ? vg : v) + head;
        if (wid == 0) {
            sq[lane] = Q[(size_t)i * 64 + lane];
            sq[lane + 32] = Q[(size_t)i * 64 + lane + 32];
        }
        __syncthreads();

        // key list: global row [0, L); local row [0, g) then [max(i - w, g), min(i + w, L - 1)]
        // (any position: global_idx[b, 0..g) then [max(i - w, 0), min(i + w, L - 1)])
        int g_seg, lo, n_keys;
        if (global_row) {
            g_seg = 0;
            lo = 0;
            n_keys = L;
        } else {
            lo = max(i - w, kAny ? 0 : g);
            g_seg = g;
            n_keys = g + (min(i + w, L - 1) - lo + 1);
        }
        RowState st{-INFINITY, 0.0f, 0.0f, 0.0f};
        for (int pos0 = wid * 32; pos0 < n_keys; pos0 += kWarps * 32)
            process_chunk<kAny>(st, sq, K, V, lm_row, pos0, g_seg, lo, n_keys, scale, lane, gl, gm_row,
                                !global_row);
        if (lane == 0) {
            part_ml[wid][0] = st.m;
            part_ml[wid][1] = st.l;
        }
        part_o[wid][lane] = st.o0;
        part_o[wid][lane + 32] = st.o1;
        __syncthreads();
        if (wid == 0) {
            float M = -INFINITY;
#pragma unroll
            for (int u = 0; u < kWarps; ++u) M = fmaxf(M, part_ml[u][0]);
            float lsum = 0.0f, o0 = 0.0f, o1 = 0.0f;
#pragma unroll
            for (int u = 0; u < kWarps; ++u) {
                const float mu = part_ml[u][0];
                const float f = mu == -INFINITY ? 0.0f : expf(mu - M);
                lsum = fmaf(part_ml[u][1], f, lsum);
                o0 = fmaf(part_o[u][lane], f, o0);
                o1 = fmaf(part_o[u][lane + 32], f, o1);
            }
            const float inv = 1.0f / lsum;
            o[lane] = o0 * inv;
            o[lane + 32] = o1 * inv;
        }
        __syncthreads();  // shared buffers are reused by the next row
    }
}

}  // namespace

lf_status launch_attention_simt_f32(const float* q, const float* k, const float* v, const float* qg,
                                    const float* kg, const float* vg, const float* local_mask,
                                    const float* global_mask, int B, int H, int L, int w, float scale,
                                    float* out, int* status, cudaStream_t stream, const AnyGlobals* any,
                                    int32_t* gidx_out, int32_t* gnum_out) {
    const long long rows = (long long)B * H * L;
    long long blocks = rows;
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (any)
        attention_simt_kernel<true><<<(int)blocks, kWarps * 32, 0, stream>>>(
            q, k, v, qg, kg, vg, local_mask, global_mask, B, H, L, w, scale, out, status, any->global_idx,
            any->global_token_nums, nullptr, nullptr);
    else
        attention_simt_kernel<false><<<(int)blocks, kWarps * 32, 0, stream>>>(
            q, k, v, qg, kg, vg, local_mask, global_mask, B, H, L, w, scale, out, status, nullptr, nullptr,
            gidx_out, gnum_out);
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

}  // namespace lf
