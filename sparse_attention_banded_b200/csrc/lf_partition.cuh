// The global-index partition of one sample on 128 threads (four warps) of a
// CTA, for the kernels that compute it in the same launch as the attention
// (FasterTransformer Longformer page, §Longformer Encoder 计算流程 / 预处理,
// invokeInitLongformerIdx): the positions with global_mask == 0.0 in
// ascending order, then the other positions in descending order (the order
// of a stable flagged partition that writes rejected items from the back),
// their count, and the content check of the prefix rule, as the partition
// kernel writes them.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "lf_internal.h"

namespace lf {

// row: global_mask[b, 0..L); idx: global_idx[b, 0..L) and *gnum: the count,
// written.  te = 0..127 (this thread among the 128), ew = te / 32, lane =
// te % 32; sm: 5 ints of shared memory; named barrier 1 with 128 threads.
__device__ __forceinline__ void partition_sample(const float* row, int L, int w, int32_t* idx, int32_t* gnum, int b,
                                                 int* status, int te, int ew, int lane, int* sm) {
    constexpr int kN = 128, kIt = 4;
    if (te == 0) sm[4] = L;  // first position that is not global
    asm volatile("bar.sync 1, %0;" ::"r"(kN) : "memory");
    int base = 0;  // global positions before this chunk
    for (int c0 = 0; c0 < L; c0 += kN * kIt) {
        const int j0 = c0 + te * kIt;
        bool f[kIt];
        if (j0 + kIt <= L && (L & 3) == 0) {
            const float4 m4 = *reinterpret_cast<const float4*>(row + j0);
            f[0] = m4.x == 0.0f;
            f[1] = m4.y == 0.0f;
            f[2] = m4.z == 0.0f;
            f[3] = m4.w == 0.0f;
        } else {
#pragma unroll
            for (int t = 0; t < kIt; ++t) f[t] = (j0 + t < L) && row[j0 + t] == 0.0f;
        }
        int cnt = 0, my_first = L;
#pragma unroll
        for (int t = 0; t < kIt; ++t) {
            cnt += f[t];
            if (!f[t] && j0 + t < L && my_first == L) my_first = j0 + t;
        }
        if (my_first < L) atomicMin(&sm[4], my_first);
        int incl = cnt;  // inclusive scan of the counts within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) sm[ew] = incl;
        asm volatile("bar.sync 1, %0;" ::"r"(kN) : "memory");
        int wbase = 0;
        for (int u = 0; u < ew; ++u) wbase += sm[u];
        const int tot = sm[0] + sm[1] + sm[2] + sm[3];
        int sel = base + wbase + incl - cnt;  // global positions before j0
#pragma unroll
        for (int t = 0; t < kIt; ++t) {
            const int j = j0 + t;
            if (j < L) {
                if (f[t]) {
                    idx[sel] = j;
                    ++sel;
                } else {
                    idx[L - 1 - (j - sel)] = j;  // j - sel: other positions before j
                }
            }
        }
        base += tot;
        asm volatile("bar.sync 1, %0;" ::"r"(kN) : "memory");  // sm[0..3] are rewritten by the next chunk
    }
    if (te == 0) {
        *gnum = base;
        if (sm[4] < base) record_status(status, b, LF_ERR_GLOBAL_NOT_PREFIX);
        else if (base > w) record_status(status, b, LF_ERR_G_GT_W);
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kN) : "memory");  // sm[4] is reset for the next sample only after it was read
}

}  // namespace lf
