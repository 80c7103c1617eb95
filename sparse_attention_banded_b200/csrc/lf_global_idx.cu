// Global-token index partition (invokeInitLongformerIdx of the
// FasterTransformer Longformer page, §Longformer Encoder 计算流程 / 预处理).
//
// One CTA (1024 threads) per sample walks the row in chunks of 4096 positions.  Each
// thread flags its 4 positions (global_mask == 0.0f), a block-wide exclusive
// scan of the per-thread counts gives every flagged position its slot at the
// front (ascending) and every unflagged one its slot at the back
// (descending), which is the output order of a stable flagged partition that
// writes rejected items from the end.  The CTA also checks the page's
// constraints 3 and 4 (§使用前提): the flagged positions must be exactly
// 0..g-1 and g <= w.
//
// The work is one pass over the mask: L * 4 bytes read, L * 4 bytes written
// per sample -- HBM-bound and tiny next to the attention kernel.
#include "lf_internal.h"

namespace lf {
namespace {

constexpr int kThreads = 1024;
constexpr int kItems = 4;

__global__ void __launch_bounds__(kThreads)
global_idx_kernel(const float* __restrict__ global_mask, int L, int w, int32_t* __restrict__ global_idx,
                  int32_t* __restrict__ global_token_nums, int* status) {
    const int b = blockIdx.x;
    const float* row = global_mask + (size_t)b * L;
    int32_t* idx = global_idx + (size_t)b * L;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    __shared__ int warp_tot[kThreads / 32 + 1];
    __shared__ int first_unflagged;
    if (tid == 0) first_unflagged = L;
    __syncthreads();

    int base = 0;  // flagged positions before this chunk (uniform)
    for (int c0 = 0; c0 < L; c0 += kThreads * kItems) {
        const int j0 = c0 + tid * kItems;
        bool f[kItems];
        int cnt = 0;
        if (j0 + kItems <= L && (L & 3) == 0) {
            float4 m4 = *reinterpret_cast<const float4*>(row + j0);
            f[0] = m4.x == 0.0f; f[1] = m4.y == 0.0f; f[2] = m4.z == 0.0f; f[3] = m4.w == 0.0f;
        } else {
#pragma unroll
            for (int t = 0; t < kItems; ++t) f[t] = (j0 + t < L) && row[j0 + t] == 0.0f;
        }
        int my_first = L;
#pragma unroll
        for (int t = 0; t < kItems; ++t) {
            cnt += f[t];
            if (!f[t] && j0 + t < L && my_first == L) my_first = j0 + t;
        }
        if (my_first < L) atomicMin(&first_unflagged, my_first);

        // block-wide exclusive scan of cnt
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {  // exclusive scan of the 32 warp totals; slot 32 = chunk total
            const int t = warp_tot[lane];
            int x = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            warp_tot[lane] = x - t;
            if (lane == 31) warp_tot[32] = x;
        }
        __syncthreads();
        const int warp_base = warp_tot[warp], chunk_tot = warp_tot[32];
        int sel = base + warp_base + incl - cnt;  // flagged before position j0
#pragma unroll
        for (int t = 0; t < kItems; ++t) {
            const int j = j0 + t;
            if (j < L) {
                if (f[t]) {
                    idx[sel] = j;
                    ++sel;
                } else {
                    idx[L - 1 - (j - sel)] = j;  // j - sel = unflagged positions before j
                }
            }
        }
        base += chunk_tot;
        __syncthreads();  // warp_tot is rewritten by the next chunk
    }
    if (tid == 0) {
        global_token_nums[b] = base;
        if (first_unflagged < base) record_status(status, b, LF_ERR_GLOBAL_NOT_PREFIX);
        else if (base > w) record_status(status, b, LF_ERR_G_GT_W);
    }
}

}  // namespace

lf_status launch_global_idx(const float* global_mask, int B, int L, int w, int32_t* global_idx,
                            int32_t* global_token_nums, int* status, cudaStream_t stream) {
    global_idx_kernel<<<B, kThreads, 0, stream>>>(global_mask, L, w, global_idx, global_token_nums, status);
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

}  // namespace lf
