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
// 0..g-1 (unless global tokens may lie anywhere) and g <= w.
//
// For global tokens at any position the same scan also gives the rank table
// rank[b, j] = flagged positions before j (j = 0..L, rank[b, L] = g), from
// which a row's window [i - w, i + w] maps to the range [rank[i - w],
// rank[i + w + 1]) of global-token slots it covers.
//
// The work is one pass over the mask: L * 4 bytes read, L * 4 bytes written
// per sample -- HBM-bound and tiny next to the attention kernel.
#include <atomic>

#include "lf_internal.h"

namespace lf {
namespace {

constexpr int kThreads = 1024;
constexpr int kItems = 4;

__global__ void __launch_bounds__(kThreads)
global_idx_kernel(const float* __restrict__ global_mask, int L, int w, int32_t* __restrict__ global_idx,
                  int32_t* __restrict__ global_token_nums, int32_t* __restrict__ rank, int require_prefix,
                  int* status) {
    // Launched as a programmatic dependent: the next kernel may be scheduled
    // at once, and nothing is read before the kernel before has completed.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int b = blockIdx.x;
    const float* row = global_mask + (size_t)b * L;
    int32_t* idx = global_idx + (size_t)b * L;
    int32_t* rk = rank ? rank + (size_t)b * (L + 1) : nullptr;
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
                if (rk) rk[j] = sel;
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
        if (rk) rk[L] = base;
        if (require_prefix && first_unflagged < base) record_status(status, b, LF_ERR_GLOBAL_NOT_PREFIX);
        else if (base > w) record_status(status, b, LF_ERR_G_GT_W);
    }
}

}  // namespace

lf_status launch_global_idx(const float* global_mask, int B, int L, int w, int32_t* global_idx,
                            int32_t* global_token_nums, int* status, cudaStream_t stream, int32_t* rank,
                            bool require_prefix) {
    return launch_pdl(global_idx_kernel, dim3(B), dim3(kThreads), 0, stream, global_mask, L, w, global_idx,
                      global_token_nums, rank, require_prefix ? 1 : 0, status);
}

}  // namespace lf

// ---------------------------------------------------------------- global tokens at any position
//
// The tensor-core attention kernel reads the global tokens' rows through
// compact per-head buffers: slot c of sample b holds the row of position
// global_idx[b, c] (the c-th global token), so that the global rows form
// whole 128-row query tiles and the global keys whole 128-key blocks, each
// one TMA box, wherever the tokens lie in the sequence.

namespace lf {
namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// One CTA of 256 threads per 32 slots of one (b, h): thread t copies the
// 16-byte column part t % 8 of slot c0 + t / 8 for qg (unless qg is NULL:
// the encoder layer projects the slots' qg rows itself), k and v; slots past
// g up to the end of their 128-slot block are zero (finite rows for the
// masked tail of a block).  The h == 0 CTAs also write the slots' local_mask
// values.
__global__ void __launch_bounds__(256)
gather_globals_kernel(const uint4* __restrict__ qg, const uint4* __restrict__ k, const uint4* __restrict__ v,
                      const float* __restrict__ local_mask, const int32_t* __restrict__ gidx,
                      const int32_t* __restrict__ gnum, int H, int L, int gcap, uint4* __restrict__ qg_c,
                      uint4* __restrict__ k_c, uint4* __restrict__ v_c, float* __restrict__ lm_c) {
    // Launched as a programmatic dependent: the next kernel may be scheduled
    // at once, and nothing is read before the kernel before has completed.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int per = gcap / 32;  // CTAs per (b, h)
    const int bh = blockIdx.x / per, b = bh / H, h = bh % H;
    const int c0 = (blockIdx.x % per) * 32;
    const int c = c0 + (threadIdx.x >> 3), part = threadIdx.x & 7;
    // a sample with g > w is rejected by the attention kernel; min() keeps
    // the slots in range (c < g <= L also keeps the index read in range)
    const int g = min(gnum[b], gcap);
    if (h == 0 && threadIdx.x < 32) {
        const int cc = c0 + threadIdx.x;
        lm_c[(size_t)b * gcap + cc] = cc < g ? local_mask[(size_t)b * L + gidx[(size_t)b * L + cc]] : 0.0f;
    }
    // the attention kernel reads the slot blocks that hold slots < g
    if (c >= (g + 127) / 128 * 128) return;
    const size_t dst = ((size_t)bh * gcap + c) * 8 + part;
    if (c < g) {
        const int j = gidx[(size_t)b * L + c];
        const size_t src = ((size_t)bh * L + j) * 8 + part;
        const uint4 kk = k[src], vv = v[src];
        if (qg) qg_c[dst] = qg[src];
        k_c[dst] = kk;
        v_c[dst] = vv;
    } else {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        if (qg) qg_c[dst] = z;
        k_c[dst] = z;
        v_c[dst] = z;
    }
}

// The partition and the gather in one launch, for the attention call: one
// CTA of 1024 threads per (b, h).  Every CTA scans sample b's mask as the
// partition kernel does and keeps the positions of its first gcap global
// tokens in shared memory; the h == 0 CTA also writes global_idx,
// global_token_nums, the rank table and the slots' local_mask values.  Then
// each CTA copies its head's qg, k and v rows into the slots (zero from g to
// the end of the last slot block read).
__global__ void __launch_bounds__(kThreads)
partition_gather_kernel(const float* __restrict__ global_mask, const float* __restrict__ local_mask, int H, int L,
                        int w, int gcap, const uint4* __restrict__ qg, const uint4* __restrict__ k,
                        const uint4* __restrict__ v, int32_t* __restrict__ global_idx,
                        int32_t* __restrict__ global_token_nums, int32_t* __restrict__ rank, uint4* __restrict__ qg_c,
                        uint4* __restrict__ k_c, uint4* __restrict__ v_c, float* __restrict__ lm_c, int* status) {
    // Launched as a programmatic dependent: the next kernel may be scheduled
    // at once, and nothing is read before the kernel before has completed.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    extern __shared__ int slot_pos[];  // [gcap]
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const bool lead = h == 0;  // writes the partition's outputs
    const float* row = global_mask + (size_t)b * L;
    int32_t* idx = global_idx + (size_t)b * L;
    int32_t* rk = rank + (size_t)b * (L + 1);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int warp_tot[kThreads / 32 + 1];

    int base = 0;
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
#pragma unroll
        for (int t = 0; t < kItems; ++t) cnt += f[t];
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
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
        int sel = base + warp_tot[warp] + incl - cnt;
        const int chunk_tot = warp_tot[32];
#pragma unroll
        for (int t = 0; t < kItems; ++t) {
            const int j = j0 + t;
            if (j < L) {
                if (lead) rk[j] = sel;
                if (f[t]) {
                    if (lead) idx[sel] = j;
                    if (sel < gcap) slot_pos[sel] = j;
                    ++sel;
                } else if (lead) {
                    idx[L - 1 - (j - sel)] = j;
                }
            }
        }
        base += chunk_tot;
        __syncthreads();
    }
    const int g = min(base, gcap);
    if (lead) {
        if (tid == 0) {
            global_token_nums[b] = base;
            rk[L] = base;
            if (base > w) record_status(status, b, LF_ERR_G_GT_W);
        }
        for (int c = tid; c < gcap; c += kThreads)
            lm_c[(size_t)b * gcap + c] = c < g ? local_mask[(size_t)b * L + slot_pos[c]] : 0.0f;
    }
    // this head's rows: 8 threads of 16 bytes per row, 128 rows per pass
    const int end = (g + 127) / 128 * 128;
    const int part = tid & 7;
    for (int c = tid >> 3; c < end; c += kThreads / 8) {
        const size_t dst = ((size_t)bh * gcap + c) * 8 + part;
        if (c < g) {
            const size_t src = ((size_t)bh * L + slot_pos[c]) * 8 + part;
            const uint4 a = qg[src], kk = k[src], vv = v[src];
            qg_c[dst] = a;
            k_c[dst] = kk;
            v_c[dst] = vv;
        } else {
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            qg_c[dst] = z;
            k_c[dst] = z;
            v_c[dst] = z;
        }
    }
}

// Rows of a [B][L][D] 16-bit matrix at the global tokens' positions into
// [B][gcap][D] (slot c = position global_idx[b, c]; slots past g zero).  One
// CTA of 128 threads per slot, 16 bytes per thread and step.
__global__ void __launch_bounds__(128)
gather_rows_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ gidx,
                   const int32_t* __restrict__ gnum, int L, int gcap, int parts, uint4* __restrict__ dst) {
    // Launched as a programmatic dependent: the next kernel may be scheduled
    // at once, and nothing is read before the kernel before has completed.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int b = blockIdx.x / gcap, c = blockIdx.x % gcap;
    const int g = min(gnum[b], gcap);
    uint4* d = dst + ((size_t)b * gcap + c) * parts;
    if (c < g) {
        const uint4* s = src + ((size_t)b * L + gidx[(size_t)b * L + c]) * parts;
        for (int t = threadIdx.x; t < parts; t += 128) d[t] = s[t];
    } else {
        for (int t = threadIdx.x; t < parts; t += 128) d[t] = make_uint4(0u, 0u, 0u, 0u);
    }
}

}  // namespace

lf_status launch_gather_rows(const void* src, const AnyGlobals& a, int B, int L, int D, void* dst,
                             cudaStream_t stream) {
    const long long blocks = (long long)B * a.gcap;
    if (blocks >= (1LL << 31)) return LF_ERR_TOO_LARGE;
    return launch_pdl(gather_rows_kernel, dim3((unsigned)blocks), dim3(128), 0, stream,
                      reinterpret_cast<const uint4*>(src), a.global_idx, a.global_token_nums, L, a.gcap, D * 2 / 16,
                      reinterpret_cast<uint4*>(dst));
}

lf_status launch_partition_gather(const float* global_mask, const float* local_mask, const void* qg, const void* k,
                                  const void* v, const AnyGlobals& a, int B, int H, int L, int w, int* status,
                                  cudaStream_t stream) {
    const size_t smem = (size_t)a.gcap * sizeof(int);
    if (smem > 200 * 1024) return LF_ERR_TOO_LARGE;
    if (smem > 48 * 1024) {
        // the shared-memory opt-in is a per-device function attribute
        static std::atomic<bool> attr[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LF_ERR_CUDA;
        if (!attr[dev].load()) {
            if (cudaFuncSetAttribute(partition_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     200 * 1024) != cudaSuccess)
                return LF_ERR_CUDA;
            attr[dev].store(true);
        }
    }
    return launch_pdl(partition_gather_kernel, dim3(B * H), dim3(kThreads), smem, stream, global_mask, local_mask, H,
                      L, w, a.gcap, reinterpret_cast<const uint4*>(qg), reinterpret_cast<const uint4*>(k),
                      reinterpret_cast<const uint4*>(v), const_cast<int32_t*>(a.global_idx),
                      const_cast<int32_t*>(a.global_token_nums), const_cast<int32_t*>(a.rank),
                      reinterpret_cast<uint4*>(a.qg_c), reinterpret_cast<uint4*>(a.k_c),
                      reinterpret_cast<uint4*>(a.v_c), a.lm_c, status);
}

size_t any_globals_bytes(int B, int H, int L, int w, bool compact) {
    size_t n = align256((size_t)B * L * 4) + align256((size_t)B * 4) + align256((size_t)B * (L + 1) * 4);
    if (compact) {
        const size_t gcap = (size_t)any_globals_gcap(w);
        n += 3 * align256((size_t)B * H * gcap * 64 * 2) + align256((size_t)B * gcap * 4);
    }
    return n;
}

AnyGlobals any_globals_layout(void* base, int B, int H, int L, int w, bool compact) {
    AnyGlobals a{};
    uint8_t* s = reinterpret_cast<uint8_t*>(base);
    a.global_idx = reinterpret_cast<int32_t*>(s);
    s += align256((size_t)B * L * 4);
    a.global_token_nums = reinterpret_cast<int32_t*>(s);
    s += align256((size_t)B * 4);
    a.rank = reinterpret_cast<int32_t*>(s);
    s += align256((size_t)B * (L + 1) * 4);
    a.gcap = any_globals_gcap(w);
    if (compact) {
        const size_t tb = align256((size_t)B * H * a.gcap * 64 * 2);
        a.qg_c = s;
        a.k_c = s + tb;
        a.v_c = s + 2 * tb;
        a.lm_c = reinterpret_cast<float*>(s + 3 * tb);
    }
    return a;
}

lf_status launch_gather_globals(const void* qg, const void* k, const void* v, const float* local_mask,
                                const AnyGlobals& a, int B, int H, int L, int w, cudaStream_t stream) {
    (void)w;
    const long long blocks = (long long)B * H * (a.gcap / 32);
    if (blocks >= (1LL << 31)) return LF_ERR_TOO_LARGE;
    // (qg may be NULL: qg_c is then left to the caller)
    return launch_pdl(gather_globals_kernel, dim3((unsigned)blocks), dim3(256), 0, stream,
                      reinterpret_cast<const uint4*>(qg), reinterpret_cast<const uint4*>(k),
                      reinterpret_cast<const uint4*>(v), local_mask, a.global_idx, a.global_token_nums, H, L,
                      a.gcap, reinterpret_cast<uint4*>(a.qg_c), reinterpret_cast<uint4*>(a.k_c),
                      reinterpret_cast<uint4*>(a.v_c), a.lm_c);
}

}  // namespace lf
