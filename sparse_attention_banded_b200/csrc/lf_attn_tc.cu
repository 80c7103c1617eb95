// Longformer banded + global self-attention on the sm_100a tensor cores.
//
// The FasterTransformer Longformer page ("FasterTransformer Longformer 推理加速
// 实践"), §Longformer Encoder 计算流程 / 每个 Transformer 层 steps 3-5, runs
// this layer as window GEMMs over head/middle/tail segments, a separate
// masked-softmax kernel and a transpose kernel.  Here it is ONE persistent
// kernel per call:
//
//   work item "band"   (b, h, 128-query tile t): the tile's key blocks are the
//       128-key blocks overlapping rows' windows |i - j| <= w, plus the blocks
//       holding global keys 0..g_b-1 that some row of the tile sees outside its
//       window.  Every key block is visited once, with the mask
//       allowed(i, j) = j < g_b || |i - j| <= w, so a global key inside the
//       window is counted once.
//   work item "global" (b, h, row tile rt, key split s): rows i < g_b attend
//       to all keys through qg/kg/vg; the keys are split into chunks of
//       kChunkBlocks blocks, each item leaves (m, l, O) partials in scratch and
//       the last item of a (b, h, rt) to finish merges them (log-sum-exp) and
//       writes the rows.
//
// Per CTA: warp 0 issues TMA loads (Q tile double-buffered, K/V blocks in a
// kStages ring), warp 1 issues tcgen05.mma (S = Q K^T into TMEM, double
// buffered; O_blk = P V into TMEM, double buffered), warps 2-5 (one thread per
// query row) read S from TMEM, apply scale, padding bias and mask, run the
// online softmax, write P (fp16/bf16) to shared memory in the 128B-swizzled
// K-major layout the MMA reads, and accumulate O in registers.  All waits are
// bounded; on expiry the CTA records LF_ERR_DEVICE_TIMEOUT and winds down.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "lf_internal.h"
#include "sm100.cuh"

namespace lf {
namespace {

using namespace sm100;

constexpr int kBM = 128;           // query rows per tile
constexpr int kBN = 128;           // keys per block
constexpr int kHD = 64;            // head dim
constexpr int kStages = 3;         // K/V ring depth
constexpr int kChunkBlocks = 4;    // key blocks per global-row split
constexpr int kThreads = 192;      // 6 warps
constexpr int kSoftmaxWarp0 = 2;
constexpr uint32_t kTileBytes = kBM * kHD * 2;  // 16 KB
constexpr uint32_t kPBytes = kBM * kBN * 2;     // 32 KB
constexpr float kLog2e = 1.4426950408889634f;

// Shared memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t kOffQ = 0;                                // 2 x 16 KB
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;           // kStages x 16 KB
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;     // kStages x 16 KB
constexpr uint32_t kOffP = kOffV + kStages * kTileBytes;     // 2 x 32 KB
constexpr uint32_t kOffBias = kOffP + 2 * kPBytes;           // 4 warps x 2 x 128 floats
constexpr uint32_t kOffBar = kOffBias + 4 * 2 * kBN * 4;
constexpr uint32_t kNumBars = 2 + 2 + 2 * kStages + 2 + 2 + 2 + 2 + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack

// TMEM columns: S[0..1] at 0 / 128, PV[0..1] at 256 / 320.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemPV = 256;

struct Params {
    int B, H, L, w;
    int NKB;       // key blocks per head
    int NT;        // query tiles per head
    int RT;        // global row tiles per head (ceil(w / 128))
    int NS;        // key splits per global row tile
    int n_glob;    // number of global items (they come first)
    int n_items;
    float scale_log2;
    const float* local_mask;
    const float* global_mask;
    void* out;
    float* part_o;    // [B*H*RT*NS][128][64]
    float* part_ml;   // [B*H*RT*NS][128][2]
    int* counters;    // [B*H*RT][4]: one per 32-row group of a global row tile
    int* status;
};

struct Maps {
    CUtensorMap q, k, v, qg, kg, vg;
};

struct Item {
    int global;   // 1 = global-row item
    int b, h, bh;
    int tile;     // t (band) or rt (global)
    int split;
    int r0;       // first query row
};

__device__ __forceinline__ Item decode_item(const Params& p, int id) {
    Item it;
    if (id < p.n_glob) {
        it.global = 1;
        it.split = id % p.NS;
        const int r = id / p.NS;
        it.tile = r % p.RT;
        it.bh = r / p.RT;
    } else {
        const int id2 = id - p.n_glob;
        it.global = 0;
        it.split = 0;
        it.tile = id2 % p.NT;
        it.bh = id2 / p.NT;
    }
    it.b = it.bh / p.H;
    it.h = it.bh % p.H;
    it.r0 = it.tile * kBM;
    return it;
}

// Leading 0.0 entries of global_mask[b, :] capped at w + 1 (whole warp).
__device__ int leading_globals(const Params& p, int b) {
    const int lane = threadIdx.x & 31;
    const float* row = p.global_mask + (size_t)b * p.L;
    const int cap = min(p.w + 1, p.L);
    for (int c0 = 0; c0 < cap; c0 += 32) {
        const int j = c0 + lane;
        const unsigned m = __ballot_sync(0xffffffffu, j < cap && row[j] != 0.0f);
        if (m) return c0 + __ffs(m) - 1;
    }
    return cap;
}

struct Blocks {
    int n;        // number of key blocks
    int glob_hi;  // blocks [0, glob_hi) are global-key blocks
    int band_lo;  // then blocks band_lo, band_lo + 1, ...
};

__device__ __forceinline__ Blocks block_list(const Params& p, const Item& it, int g) {
    Blocks bl{0, 0, 0};
    if (g > p.w) return bl;  // invalid sample: no compute
    if (it.global) {
        if (it.r0 >= g) return bl;
        bl.band_lo = it.split * kChunkBlocks;
        const int hi = min(p.NKB, bl.band_lo + kChunkBlocks) - 1;
        bl.n = hi - bl.band_lo + 1;
        return bl;
    }
    const int lo = it.r0 - p.w;
    bl.band_lo = lo <= 0 ? 0 : lo / kBN;
    const int hi = min(p.NKB - 1, (it.r0 + kBM - 1 + p.w) / kBN);
    bl.glob_hi = min((g + kBN - 1) / kBN, bl.band_lo);
    bl.n = bl.glob_hi + hi - bl.band_lo + 1;
    return bl;
}

__device__ __forceinline__ int block_at(const Blocks& bl, int n) {
    return n < bl.glob_hi ? n : bl.band_lo + (n - bl.glob_hi);
}

template <typename T>
struct Pack;
template <>
struct Pack<__half> {
    static constexpr uint32_t fmt = 0;
    __device__ static uint32_t two(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};
template <>
struct Pack<__nv_bfloat16> {
    static constexpr uint32_t fmt = 1;
    __device__ static uint32_t two(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

template <typename T>
__device__ __forceinline__ void store_row(void* out_base, size_t elem_off, const float* o, float scale) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<T*>(out_base) + elem_off);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u;
        u.x = Pack<T>::two(o[8 * c + 0] * scale, o[8 * c + 1] * scale);
        u.y = Pack<T>::two(o[8 * c + 2] * scale, o[8 * c + 3] * scale);
        u.z = Pack<T>::two(o[8 * c + 4] * scale, o[8 * c + 5] * scale);
        u.w = Pack<T>::two(o[8 * c + 6] * scale, o[8 * c + 7] * scale);
        dst[c] = u;
    }
}

__device__ __forceinline__ void store_zero_row(void* out_base, size_t elem_off, int elem_bytes) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<char*>(out_base) + elem_off * elem_bytes);
#pragma unroll
    for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
attention_tc_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 2;
    uint64_t* kv_full = bars + 4;
    uint64_t* kv_empty = bars + 4 + kStages;
    uint64_t* s_full = bars + 4 + 2 * kStages;
    uint64_t* p_full = s_full + 2;
    uint64_t* pv_full = p_full + 2;
    uint64_t* pv_free = pv_full + 2;
    uint64_t* drain = pv_free + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&pv_full[i], 1);
            mbar_init(&pv_free[i], 4);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&maps.q);
        prefetch_tensormap(&maps.k);
        prefetch_tensormap(&maps.v);
        prefetch_tensormap(&maps.qg);
        prefetch_tensormap(&maps.kg);
        prefetch_tensormap(&maps.vg);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        uint32_t kv_cnt = 0, item_cnt = 0;
        int cached_b = -1, g = 0;
        bool ok = true;
        for (int id = blockIdx.x; id < p.n_items && ok; id += gridDim.x) {
            const Item it = decode_item(p, id);
            if (it.b != cached_b) {
                g = leading_globals(p, it.b);
                cached_b = it.b;
            }
            const Blocks bl = block_list(p, it, g);
            if (bl.n == 0) continue;
            if (lane == 0) {
                const uint32_t qb = item_cnt & 1;
                ok = mbar_wait(&q_empty[qb], ((item_cnt >> 1) & 1) ^ 1, abort_flag);
                if (ok) {
                    mbar_arrive_expect_tx(&q_full[qb], kTileBytes);
                    tma_load_3d(smem + kOffQ + qb * kTileBytes, it.global ? &maps.qg : &maps.q, &q_full[qb], 0,
                                it.r0, it.bh);
                }
                for (int n = 0; n < bl.n && ok; ++n) {
                    const uint32_t st = kv_cnt % kStages;
                    ok = mbar_wait(&kv_empty[st], ((kv_cnt / kStages) & 1) ^ 1, abort_flag);
                    if (!ok) break;
                    const int kb = block_at(bl, n);
                    mbar_arrive_expect_tx(&kv_full[st], 2 * kTileBytes);
                    tma_load_3d(smem + kOffK + st * kTileBytes, it.global ? &maps.kg : &maps.k, &kv_full[st], 0,
                                kb * kBN, it.bh);
                    tma_load_3d(smem + kOffV + st * kTileBytes, it.global ? &maps.vg : &maps.v, &kv_full[st], 0,
                                kb * kBN, it.bh);
                    ++kv_cnt;
                }
            }
            ++item_cnt;
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        // Wind-down: let issued copies land before the CTA can exit.
        if (lane == 0 && !ok) {
            for (uint32_t c = (kv_cnt > kStages ? kv_cnt - kStages : 0); c < kv_cnt; ++c) {
                volatile int never = 0;
                mbar_wait(&kv_full[c % kStages], (c / kStages) & 1, &never, 200000000ull);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_qk = idesc_f16(Pack<T>::fmt, kBM, kBN, 0, 0);
        constexpr uint32_t idesc_pv = idesc_f16(Pack<T>::fmt, kBM, kHD, 0, 1);
        uint32_t kv_cnt = 0, blk = 0, item_cnt = 0;
        int cached_b = -1, g = 0;
        bool ok = true;
        for (int id = blockIdx.x; id < p.n_items && ok; id += gridDim.x) {
            const Item it = decode_item(p, id);
            if (it.b != cached_b) {
                g = leading_globals(p, it.b);
                cached_b = it.b;
            }
            const Blocks bl = block_list(p, it, g);
            if (bl.n == 0) continue;
            if (lane == 0) {
                const uint32_t qb = item_cnt & 1;
                ok = mbar_wait(&q_full[qb], (item_cnt >> 1) & 1, abort_flag);
                tc_fence_after();
                const uint32_t q_addr = smem_u32(smem + kOffQ + qb * kTileBytes);
                uint32_t prev_st = 0;
                for (int n = 0; n <= bl.n && ok; ++n) {
                    uint32_t st = 0;
                    if (n < bl.n) {
                        st = kv_cnt % kStages;
                        ok = mbar_wait(&kv_full[st], (kv_cnt / kStages) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t sb = (blk + n) & 1;
                        const uint32_t k_addr = smem_u32(smem + kOffK + st * kTileBytes);
#pragma unroll
                        for (int kk = 0; kk < kHD / 16; ++kk)
                            mma_f16_ss(tmem + kTmemS + sb * kBN, desc_sw128(q_addr + kk * 32),
                                       desc_sw128(k_addr + kk * 32), idesc_qk, kk > 0);
                        tc_commit(&s_full[sb]);
                        if (n == bl.n - 1) tc_commit(&q_empty[qb]);
                    }
                    if (n >= 1) {
                        const uint32_t j = blk + n - 1;
                        const uint32_t pb = j & 1;
                        ok = mbar_wait(&p_full[pb], (j >> 1) & 1, abort_flag);
                        if (ok) ok = mbar_wait(&pv_free[pb], ((j >> 1) & 1) ^ 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t p_addr = smem_u32(smem + kOffP + pb * kPBytes);
                        const uint32_t v_addr = smem_u32(smem + kOffV + prev_st * kTileBytes);
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; ++kk)
                            mma_f16_ss(tmem + kTmemPV + pb * kHD,
                                       desc_sw128(p_addr + (kk >> 2) * (kBM * 128) + (kk & 3) * 32),
                                       desc_sw128(v_addr + kk * 2048, 0), idesc_pv, kk > 0);
                        tc_commit(&pv_full[pb]);
                        tc_commit(&kv_empty[prev_st]);
                    }
                    if (n < bl.n) {
                        prev_st = st;
                        ++kv_cnt;
                    }
                }
            }
            blk += bl.n;
            ++item_cnt;
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        // Wind-down after an abort: wait for the MMAs already issued.
        if (lane == 0 && !ok) {
            tc_commit(drain);
            volatile int never = 0;
            mbar_wait(drain, 0, &never, 200000000ull);
        }
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        const int sp = warp & 3;            // TMEM sub-partition of this warp
        const int r = sp * 32 + lane;       // query row within the tile
        const uint32_t lane_off = (uint32_t)(sp * 32) << 16;
        float* bias_w = reinterpret_cast<float*>(smem + kOffBias) + sp * 2 * kBN;  // this warp's copy
        uint32_t blk = 0;
        int cached_b = -1, g = 0;
        bool ok = true;
        for (int id = blockIdx.x; id < p.n_items && ok; id += gridDim.x) {
            const Item it = decode_item(p, id);
            if (it.b != cached_b) {
                g = leading_globals(p, it.b);
                cached_b = it.b;
            }
            const float* lm = p.local_mask + (size_t)it.b * p.L;
            const int i = it.r0 + r;
            if (g > p.w) {  // invalid sample: zero output, record once
                if (!it.global) {
                    if (i < p.L) store_zero_row(p.out, ((size_t)(it.b * p.L + i) * p.H + it.h) * kHD, sizeof(T));
                    if (r == 0 && it.tile == 0 && it.h == 0) record_status(p.status, it.b, LF_ERR_G_GT_W);
                }
                continue;
            }
            const Blocks bl = block_list(p, it, g);
            if (bl.n == 0) continue;
            if (!it.global && i < p.L && i >= g && p.global_mask[(size_t)it.b * p.L + i] == 0.0f)
                record_status(p.status, it.b, LF_ERR_GLOBAL_NOT_PREFIX);

            float o[kHD];
#pragma unroll
            for (int c = 0; c < kHD; ++c) o[c] = 0.0f;
            float m_run = -INFINITY, l_run = 0.0f, a_prev = 0.0f;

            for (int n = 0; n <= bl.n && ok; ++n) {
                float a_cur = 0.0f;
                if (n < bl.n) {
                    const uint32_t j = blk + n;
                    const uint32_t sb = j & 1;
                    const int kb = block_at(bl, n);
                    const int c0 = kb * kBN;
#pragma unroll
                    for (int t = 0; t < kBN / 32; ++t) {
                        const int key = c0 + t * 32 + lane;
                        bias_w[sb * kBN + t * 32 + lane] =
                            key < p.L ? fmaf(lm[key], 10000.0f, -10000.0f) * kLog2e : -INFINITY;
                    }
                    __syncwarp();
                    ok = mbar_wait(&s_full[sb], (j >> 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();

                    // Mask geometry for this row and block.
                    const int d0 = it.r0 + r - c0;           // i - c0
                    const bool full = it.global ||
                                      (max(it.r0 + kBM - 1 - c0, c0 + kBN - 1 - it.r0) <= p.w);
                    const int lo_c = d0 - p.w, hi_c = d0 + p.w, gl_c = g - c0;

                    float x[kBN];
                    const float* bias = bias_w + sb * kBN;
#pragma unroll
                    for (int ch = 0; ch < kBN / 32; ++ch) {
                        uint32_t raw[32];
                        tmem_ld32(tmem + lane_off + kTmemS + sb * kBN + ch * 32, raw);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int cc = ch * 32 + c;
                            float v = fmaf(__uint_as_float(raw[c]), p.scale_log2, bias[cc]);
                            if (!full) {
                                const bool allowed = (cc < gl_c) || (cc >= lo_c && cc <= hi_c);
                                v = allowed ? v : -INFINITY;
                            }
                            x[cc] = v;
                        }
                    }
                    float mb = -INFINITY;
#pragma unroll
                    for (int c = 0; c < kBN; ++c) mb = fmaxf(mb, x[c]);
                    const float m_new = fmaxf(m_run, mb);
                    const float m_use = m_new == -INFINITY ? 0.0f : m_new;
                    a_cur = ex2(m_run - m_use);
                    float sum = 0.0f;
                    uint8_t* pbuf = smem + kOffP + sb * kPBytes;
#pragma unroll
                    for (int chunk = 0; chunk < kBN / 8; ++chunk) {
                        float e[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            e[t] = ex2(x[chunk * 8 + t] - m_use);
                            sum += e[t];
                        }
                        uint4 u;
                        u.x = Pack<T>::two(e[0], e[1]);
                        u.y = Pack<T>::two(e[2], e[3]);
                        u.z = Pack<T>::two(e[4], e[5]);
                        u.w = Pack<T>::two(e[6], e[7]);
                        const int atom = chunk >> 3, cidx = chunk & 7;
                        *reinterpret_cast<uint4*>(pbuf + atom * (kBM * 128) + r * 128 + ((cidx ^ (r & 7)) << 4)) = u;
                    }
                    l_run = l_run * a_cur + sum;
                    m_run = m_new;
                    fence_proxy_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&p_full[sb]);
                }
                if (n >= 1) {
                    const uint32_t j = blk + n - 1;
                    const uint32_t pb = j & 1;
                    ok = mbar_wait(&pv_full[pb], (j >> 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    uint32_t pv0[32], pv1[32];
                    tmem_ld32(tmem + lane_off + kTmemPV + pb * kHD, pv0);
                    tmem_ld32(tmem + lane_off + kTmemPV + pb * kHD + 32, pv1);
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pv_free[pb]);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        o[c] = fmaf(o[c], a_prev, __uint_as_float(pv0[c]));
                        o[c + 32] = fmaf(o[c + 32], a_prev, __uint_as_float(pv1[c]));
                    }
                }
                a_prev = a_cur;
            }
            if (!ok) break;
            blk += bl.n;

            // ---------------------------------------------------- epilogue
            if (!it.global) {
                if (i < p.L && i >= g) {
                    const size_t off = ((size_t)(it.b * p.L + i) * p.H + it.h) * kHD;
                    if (fmaf(lm[i], 10000.0f, -10000.0f) != 0.0f) store_zero_row(p.out, off, sizeof(T));
                    else store_row<T>(p.out, off, o, 1.0f / l_run);
                }
            } else if (it.r0 + sp * 32 < g) {
                // Split-KV partials of this warp's 32 rows; the warp that
                // completes the last split of its row group merges them.
                const int slot = (it.bh * p.RT + it.tile) * p.NS + it.split;
                if (i < g) {
                    float4* po = reinterpret_cast<float4*>(p.part_o + ((size_t)slot * kBM + r) * kHD);
#pragma unroll
                    for (int c = 0; c < kHD / 4; ++c)
                        __stcg(po + c, make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]));
                    __stcg(reinterpret_cast<float2*>(p.part_ml + ((size_t)slot * kBM + r) * 2),
                           make_float2(m_run, l_run));
                }
                __threadfence();
                __syncwarp();
                int* counter = p.counters + (it.bh * p.RT + it.tile) * 4 + sp;
                int last = 0;
                if (lane == 0) last = (atomicAdd(counter, 1) == p.NS - 1) ? 1 : 0;
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __threadfence();
                    if (i < g) {
                        const size_t off = ((size_t)(it.b * p.L + i) * p.H + it.h) * kHD;
                        if (fmaf(lm[i], 10000.0f, -10000.0f) != 0.0f) {
                            store_zero_row(p.out, off, sizeof(T));
                        } else {
                            const int slot0 = (it.bh * p.RT + it.tile) * p.NS;
                            float M = -INFINITY;
                            for (int s = 0; s < p.NS; ++s)
                                M = fmaxf(M, __ldcg(p.part_ml + ((size_t)(slot0 + s) * kBM + r) * 2));
                            float acc[kHD];
#pragma unroll
                            for (int c = 0; c < kHD; ++c) acc[c] = 0.0f;
                            float lsum = 0.0f;
                            for (int s = 0; s < p.NS; ++s) {
                                const float2 ml = __ldcg(
                                    reinterpret_cast<const float2*>(p.part_ml + ((size_t)(slot0 + s) * kBM + r) * 2));
                                const float wgt = ml.x == -INFINITY ? 0.0f : ex2(ml.x - M);
                                lsum = fmaf(ml.y, wgt, lsum);
                                const float4* po =
                                    reinterpret_cast<const float4*>(p.part_o + ((size_t)(slot0 + s) * kBM + r) * kHD);
#pragma unroll
                                for (int c = 0; c < kHD / 4; ++c) {
                                    const float4 t4 = __ldcg(po + c);
                                    acc[4 * c] = fmaf(t4.x, wgt, acc[4 * c]);
                                    acc[4 * c + 1] = fmaf(t4.y, wgt, acc[4 * c + 1]);
                                    acc[4 * c + 2] = fmaf(t4.z, wgt, acc[4 * c + 2]);
                                    acc[4 * c + 3] = fmaf(t4.w, wgt, acc[4 * c + 3]);
                                }
                            }
                            store_row<T>(p.out, off, acc, 1.0f / lsum);
                        }
                    }
                    if (lane == 0) *counter = 0;
                }
            }
        }
    }

    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) record_status(p.status, 0, LF_ERR_DEVICE_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// [B*H][L][64] 16-bit tensor, box 64 x 128 rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int BH, int L) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kHD, (cuuint64_t)L, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)kHD * 2, (cuuint64_t)L * kHD * 2};
    cuuint32_t box[3] = {(cuuint32_t)kHD, (cuuint32_t)kBM, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Geometry {
    int NKB, NT, RT, NS;
    size_t counters_bytes, part_o_bytes, part_ml_bytes;
};

Geometry geometry(int B, int H, int L, int w) {
    Geometry g;
    g.NKB = (L + kBN - 1) / kBN;
    g.NT = (L + kBM - 1) / kBM;
    g.RT = (w + kBM - 1) / kBM;
    g.NS = (g.NKB + kChunkBlocks - 1) / kChunkBlocks;
    const size_t slots = (size_t)B * H * g.RT * g.NS;
    g.counters_bytes = (((size_t)B * H * g.RT * 4 * sizeof(int)) + 255) & ~size_t(255);
    g.part_o_bytes = slots * kBM * kHD * sizeof(float);
    g.part_ml_bytes = slots * kBM * 2 * sizeof(float);
    return g;
}

}  // namespace

size_t attention_tc_scratch_bytes(int B, int H, int L, int w) {
    const Geometry g = geometry(B, H, L, w);
    return g.counters_bytes + g.part_o_bytes + g.part_ml_bytes;
}

lf_status launch_attention_tc(const void* q, const void* k, const void* v, const void* qg, const void* kg,
                              const void* vg, const float* local_mask, const float* global_mask, int B, int H,
                              int L, int w, float scale, lf_dtype dtype, void* out, void* scratch, int* status,
                              int sm_count, cudaStream_t stream) {
    const Geometry geo = geometry(B, H, L, w);
    Maps maps;
    const int BH = B * H;
    if (!make_map(&maps.q, q, BH, L) || !make_map(&maps.k, k, BH, L) || !make_map(&maps.v, v, BH, L) ||
        !make_map(&maps.qg, qg, BH, L) || !make_map(&maps.kg, kg, BH, L) || !make_map(&maps.vg, vg, BH, L))
        return LF_ERR_CUDA;
    Params p;
    p.B = B;
    p.H = H;
    p.L = L;
    p.w = w;
    p.NKB = geo.NKB;
    p.NT = geo.NT;
    p.RT = geo.RT;
    p.NS = geo.NS;
    p.n_glob = BH * geo.RT * geo.NS;
    p.n_items = p.n_glob + BH * geo.NT;
    p.scale_log2 = scale * kLog2e;
    p.local_mask = local_mask;
    p.global_mask = global_mask;
    p.out = out;
    uint8_t* s = reinterpret_cast<uint8_t*>(scratch);
    p.counters = reinterpret_cast<int*>(s);
    p.part_o = reinterpret_cast<float*>(s + geo.counters_bytes);
    p.part_ml = reinterpret_cast<float*>(s + geo.counters_bytes + geo.part_o_bytes);
    p.status = status;

    const int grid = p.n_items < sm_count ? p.n_items : sm_count;
    cudaError_t err;
    if (dtype == LF_F16) {
        static bool attr = false;
        if (!attr) {
            cudaFuncSetAttribute(attention_tc_kernel<__half>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
            attr = true;
        }
        attention_tc_kernel<__half><<<grid, kThreads, kSmemBytes, stream>>>(maps, p);
    } else {
        static bool attr = false;
        if (!attr) {
            cudaFuncSetAttribute(attention_tc_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
            attr = true;
        }
        attention_tc_kernel<__nv_bfloat16><<<grid, kThreads, kSmemBytes, stream>>>(maps, p);
    }
    err = cudaGetLastError();
    return err == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

}  // namespace lf
