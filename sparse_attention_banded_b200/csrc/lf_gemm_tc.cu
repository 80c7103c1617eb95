// Dense GEMM with fused epilogues on the sm_100a tensor cores, for the
// projections, the output projection and the FFN of one encoder layer
// (FasterTransformer Longformer page, §Longformer Encoder 计算流程 / 每个
// Transformer 层 steps 1, 2, 5 and 6).
//
//   C[b, m, n] = sum_k A[b, m, k] * W[n, k]      (W in nn.Linear layout [out, in])
//
// A is [batches][rows][K] (rows of one batch contiguous, the batch stride may
// exceed rows so that only the first rows of each sample are multiplied),
// both operands K-major fp16/bf16, fp32 accumulation in TMEM.  Tiles are
// 128 x 256 (one M=128, N=256 tcgen05.mma per 16-wide K step: per byte
// brought in from L2 this does a third more math than 128 x 128 tiles, which
// the L2 bandwidth of the projections' and FFN's operands needs) with 64-wide
// K steps through a kStages-deep TMA ring; N only needs to be a multiple of
// 128 (the last tile's second half is zero-filled by TMA and not stored).  One
// persistent CTA per SM: warp 0 issues TMA loads, warp 1 issues tcgen05.mma
// into one of two TMEM accumulators, warps 4-11 run the epilogue of the
// previous tile while the next tile accumulates (one thread per row, two
// warps per TMEM lane quarter, each taking half of the tile's columns, so
// that the GELU epilogue keeps up with the MMAs).
//
// Epilogues:
//   kEpiHeads  : + bias, round, scatter column n to head layout
//                out[n / D][b][h][m][d] with h = (n % D) / 64, d = n % 64
//                (AddBiasTransposeToMultiHead, step 2)
//   kEpiGelu   : + bias, GELU (erf form), round, row-major out[b*rows + m][n]
//   kEpiResid  : + bias + residual (same dtype, row-major [.., N]), fp32
//                row-major out (the LayerNorm kernel reads it)
//   kEpiResidLN: + bias + residual, then LayerNorm over the row (step 5's
//                AddBiasResidualLayerNorm and step 6's), rounded, row-major
//                out: the N / 256 CTAs of a row tile form a cluster; each
//                sends its columns' sum and centred second moment of every
//                row to the others through distributed shared memory (one
//                exchange), and all combine them in the same order
// Roofline: tensor-bound (2*M*N*K flops over (M*K + N*K)*2 + out bytes).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <mutex>

#include "lf_gelu.cuh"
#include "lf_internal.h"
#include "sm100_cluster.cuh"

namespace lf {
namespace {

using namespace sm100;

constexpr int kTM = 128, kTN = 256, kTK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 384;  // 12 warps: 0 TMA, 1 MMA, 2-3 idle, 4-11 epilogue
constexpr int kEpiWarps = 8;
constexpr uint32_t kABytes = kTM * kTK * 2;  // 16 KB
constexpr uint32_t kBBytes = kTN * kTK * 2;  // 32 KB
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kABytes;
constexpr uint32_t kOffBias = kOffB + kStages * kBBytes;        // epilogue warps x kTN / 2 floats
// kEpiResidLN: the LayerNorm's gamma and beta of each warp's columns
constexpr uint32_t kOffGamma = kOffBias + kEpiWarps * (kTN / 2) * 4;
constexpr uint32_t kOffBeta = kOffGamma + kEpiWarps * (kTN / 2) * 4;
// kEpiResidLN: [2 moments][2 halves][kTM] partial row sums of the two warps of a row
constexpr uint32_t kOffRed = kOffBeta + kEpiWarps * (kTN / 2) * 4;
constexpr int kMaxLnCtas = 4;  // N <= 1024
// kEpiResidLN: [2 buffers][kMaxLnCtas][2 moments][kTM], every CTA's row moments
constexpr uint32_t kOffXch = kOffRed + 4 * kTM * 4;
constexpr uint32_t kOffBar = kOffXch + 2 * kMaxLnCtas * 2 * kTM * 4;
constexpr uint32_t kNumBars = 2 * kStages + 4 + 1 + 2;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
constexpr uint32_t kTmemCols = 512;  // two 256-column fp32 accumulators

// One GEMM problem of a launch: per batch, rows x N outputs.
struct GemmProb {
    int rows, N;
    int mtiles, ntiles, tiles;
    const void* bias;    // [N] of T
    void* out;
    int heads_L;         // kEpiHeads: rows of the head-layout tensors
};

// A launch runs one problem, or two sharing batches, K and the epilogue
// mode (the second one's tiles follow the first's).
struct GemmParams {
    int batches, K, ktiles, tiles;
    // The last n_split of the t_full + n_split full-width tiles are run as
    // two 128-column halves each (tiles t_full .. t_full + 2 n_split - 1),
    // so that the launch's last round fills the SMs.
    int t_full, n_split;
    GemmProb pr[2];
    int mode;
    const void* resid;   // kEpiResid: [batches*rows][N] of T
    int heads_D;         // kEpiHeads: columns per output tensor (H*64)
    int heads_H;
    int* status;
    // The weights are not written by the kernel before this one: the TMA
    // warp loads the first stages' W tiles before waiting for that kernel.
    int w_early;
    // kEpiResidLN: LayerNorm parameters; ln_ctas = CTAs per cluster (one
    // per 256-column tile of the row tile)
    const float* ln_gamma;
    const float* ln_beta;
    float ln_eps;
    int ln_ctas;
};

struct TileAt {
    int pi, nt, mt, b;
    int col0, width;  // output columns [col0, col0 + width) of problem pi
};
__device__ __forceinline__ TileAt tile_at(const GemmParams& p, int t) {
    TileAt a;
    int part = -1;  // half tiles: which half
    if (t >= p.t_full) {
        const int h = t - p.t_full;
        part = h & 1;
        t = p.t_full + (h >> 1);
    }
    a.pi = t >= p.pr[0].tiles ? 1 : 0;
    if (a.pi) t -= p.pr[0].tiles;
    const GemmProb& q = p.pr[a.pi];
    a.nt = t % q.ntiles;
    const int bm = t / q.ntiles;
    a.mt = bm % q.mtiles;
    a.b = bm / q.mtiles;
    a.col0 = a.nt * kTN + (part > 0 ? kTN / 2 : 0);
    a.width = part < 0 ? kTN : kTN / 2;
    return a;
}

template <typename T>
struct Cvt;
template <>
struct Cvt<__half> {
    static constexpr uint32_t fmt = 0;
    __device__ static float to_f(__half x) { return __half2float(x); }
    __device__ static uint32_t two(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};
template <>
struct Cvt<__nv_bfloat16> {
    static constexpr uint32_t fmt = 1;
    __device__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ static uint32_t two(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
};

__device__ __forceinline__ void tmem_ld32v(uint32_t taddr, float (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]), "=f"(r[7]),
          "=f"(r[8]), "=f"(r[9]), "=f"(r[10]), "=f"(r[11]), "=f"(r[12]), "=f"(r[13]), "=f"(r[14]), "=f"(r[15]),
          "=f"(r[16]), "=f"(r[17]), "=f"(r[18]), "=f"(r[19]), "=f"(r[20]), "=f"(r[21]), "=f"(r[22]), "=f"(r[23]),
          "=f"(r[24]), "=f"(r[25]), "=f"(r[26]), "=f"(r[27]), "=f"(r[28]), "=f"(r[29]), "=f"(r[30]), "=f"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32v(uint32_t taddr, const float (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "f"(r[0]), "f"(r[1]), "f"(r[2]), "f"(r[3]), "f"(r[4]), "f"(r[5]), "f"(r[6]), "f"(r[7]), "f"(r[8]),
        "f"(r[9]), "f"(r[10]), "f"(r[11]), "f"(r[12]), "f"(r[13]), "f"(r[14]), "f"(r[15]), "f"(r[16]), "f"(r[17]),
        "f"(r[18]), "f"(r[19]), "f"(r[20]), "f"(r[21]), "f"(r[22]), "f"(r[23]), "f"(r[24]), "f"(r[25]), "f"(r[26]),
        "f"(r[27]), "f"(r[28]), "f"(r[29]), "f"(r[30]), "f"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float gelu_erf(float x) { return gelu_erf_as(x); }

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_w,
               const __grid_constant__ CUtensorMap map_a2, const __grid_constant__ CUtensorMap map_w2,
               const __grid_constant__ CUtensorMap map_wh, const __grid_constant__ CUtensorMap map_w2h,
               const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* acc_full = bars + 2 * kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* xbar = drain + 1;  // [2] kEpiResidLN: every CTA of the cluster has delivered its row moments (one per buffer)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // The next kernel in the stream may be scheduled now: its CTAs take the
    // SMs this grid leaves idle in its last wave and set themselves up there.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_init(&xbar[0], p.ln_ctas);
        mbar_init(&xbar[1], p.ln_ctas);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&map_a);
        prefetch_tensormap(&map_w);
        if (p.pr[1].tiles > 0) {
            prefetch_tensormap(&map_a2);
            prefetch_tensormap(&map_w2);
        }
        if (p.n_split > 0) {
            prefetch_tensormap(&map_wh);
            if (p.pr[1].tiles > 0) prefetch_tensormap(&map_w2h);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // every CTA's barriers are initialised before a peer arrives on them
    if (p.mode == kEpiResidLN) cluster_sync();
    const uint32_t tmem = *tmem_slot;
    // Launched as a programmatic dependent, this grid may have started while
    // the kernel before it still runs: no global memory is read or written
    // before that kernel has completed (the TMA warp waits after its early
    // weight loads, see below).
    if (warp != 0) asm volatile("griddepcontrol.wait;" ::: "memory");

    // The TMA and MMA warps run their loops with all 32 lanes (lane 0 issues
    // the copies, tensor-core instructions and commits): a lone lane running
    // the loop while the other 31 wait at a warp barrier is several times
    // slower at every hand-off.
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    if (warp == 0) {
        uint32_t kc = 0;
        bool ok = true;
        // W tiles of the first stages, issued before the wait when the
        // weights do not come from the kernel before this one
        uint32_t pre = 0;
        if (p.w_early && (int)blockIdx.x < p.tiles) {
            const TileAt at = tile_at(p, blockIdx.x);
            const CUtensorMap* mw = at.width == kTN ? (at.pi ? &map_w2 : &map_w) : (at.pi ? &map_w2h : &map_wh);
            const uint32_t bytes = kABytes + (at.width == kTN ? kBBytes : kBBytes / 2);
            pre = p.ktiles < kStages ? (uint32_t)p.ktiles : (uint32_t)kStages;
            if (lane == 0)
                for (uint32_t st = 0; st < pre; ++st) {
                    mbar_arrive_expect_tx(&full[st], bytes);
                    tma_load_2d(smem + kOffB + st * kBBytes, mw, &full[st], (int)st * kTK, at.col0);
                }
            __syncwarp();
        }
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
            const TileAt at = tile_at(p, t);
            const CUtensorMap* ma = at.pi ? &map_a2 : &map_a;
            const CUtensorMap* mw = at.width == kTN ? (at.pi ? &map_w2 : &map_w) : (at.pi ? &map_w2h : &map_wh);
            const uint32_t bytes = kABytes + (at.width == kTN ? kBBytes : kBBytes / 2);
            for (int kt = 0; kt < p.ktiles && ok; ++kt, ++kc) {
                const uint32_t st = kc % kStages;
                if (kc < pre) {  // fresh stage, its W tile already on the way
                    if (lane == 0)
                        tma_load_3d(smem + kOffA + st * kABytes, ma, &full[st], kt * kTK, at.mt * kTM, at.b);
                    __syncwarp();
                    continue;
                }
                ok = wait_all(&empty[st], ((kc / kStages) & 1) ^ 1);
                if (!ok) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[st], bytes);
                    tma_load_3d(smem + kOffA + st * kABytes, ma, &full[st], kt * kTK, at.mt * kTM, at.b);
                    tma_load_2d(smem + kOffB + st * kBBytes, mw, &full[st], kt * kTK, at.col0);
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {  // wind-down: let issued copies land
            for (uint32_t c = (kc > kStages ? kc - kStages : 0); c < kc; ++c) {
                volatile int never = 0;
                mbar_wait(&full[c % kStages], (c / kStages) & 1, &never, 200000000ull);
            }
        }
    } else if (warp == 1) {
        constexpr uint32_t idesc_full = idesc_f16(Cvt<T>::fmt, kTM, kTN, 0, 0);
        constexpr uint32_t idesc_half = idesc_f16(Cvt<T>::fmt, kTM, kTN / 2, 0, 0);
        uint32_t kc = 0, tc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++tc) {
            const uint32_t idesc = t < p.t_full ? idesc_full : idesc_half;
            const uint32_t ab = tc & 1;
            ok = wait_all(&acc_empty[ab], ((tc >> 1) & 1) ^ 1);
            if (!ok) break;
            tc_fence_after();
            for (int kt = 0; kt < p.ktiles && ok; ++kt, ++kc) {
                const uint32_t st = kc % kStages;
                ok = wait_all(&full[st], (kc / kStages) & 1);
                if (!ok) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a_addr = smem_u32(smem + kOffA + st * kABytes);
                    const uint32_t b_addr = smem_u32(smem + kOffB + st * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < kTK / 16; ++kk)
                        mma_f16_ss(tmem + ab * kTN, desc_sw128(a_addr + kk * 32), desc_sw128(b_addr + kk * 32), idesc,
                                   (kt > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&empty[st]);
                }
                __syncwarp();
            }
            if (ok && lane == 0) tc_commit(&acc_full[ab]);
            __syncwarp();
        }
        if (!ok && lane == 0) {
            tc_commit(drain);
            volatile int never = 0;
            mbar_wait(drain, 0, &never, 200000000ull);
        }
    } else if (warp >= 4) {
        const int sp = warp & 3;               // TMEM lane quarter
        const int half = (warp - 4) >> 2;      // which half of the tile's columns
        const int r = sp * 32 + lane;
        const uint32_t lane_off = (uint32_t)(sp * 32) << 16;
        float* bias_w = reinterpret_cast<float*>(smem + kOffBias) + (warp - 4) * (kTN / 2);
        // kEpiResidLN.  Each CTA holds a row's kTN columns (column tile =
        // cluster rank); a row's two warps each hold half of them.  red: the
        // two halves' partial sums; xch: every CTA's (column sum, centred
        // second moment) of each row, in two buffers used by alternate tiles.
        float* red = reinterpret_cast<float*>(smem + kOffRed);
        float* xch = reinterpret_cast<float*>(smem + kOffXch);
        float* gam_w = reinterpret_cast<float*>(smem + kOffGamma) + (warp - 4) * (kTN / 2);
        float* bet_w = reinterpret_cast<float*>(smem + kOffBeta) + (warp - 4) * (kTN / 2);
        const uint32_t rank = p.mode == kEpiResidLN ? cluster_ctarank() : 0;
        uint32_t ln_cnt = 0;
        // kEpiResidLN, one tile: z = acc + bias + resid kept in TMEM; this
        // CTA's column sum S_c and, about its own mean S_c / n_c, the centred
        // second moment M2_c; one exchange of (S_c, M2_c) over the cluster;
        // then mean = sum S_q / N and M2 = sum (M2_q + n_q (S_q / n_q - mean)^2)
        // (the pairwise update of Chan, Golub and LeVeque), added in CTA
        // order so that every CTA normalises with the same bits; finally
        // (z - mean) * rsqrt(M2 / N + eps) * gamma + beta, rounded and stored.
        // False on a failure (all epilogue warps alike).
        auto ln_tile = [&](const TileAt& at, const GemmProb& q, uint32_t ab, uint32_t tcn, int n0, int ncols,
                           int wcols) -> bool {
            bool fail = !__all_sync(0xffffffffu, mbar_wait(&acc_full[ab], (tcn >> 1) & 1, abort_flag));
            const int m = at.mt * kTM + r;
            const bool row_ok = m < q.rows;
            const size_t grow = (size_t)at.b * q.rows + m;
            const uint32_t tz = tmem + lane_off + ab * kTN + half * wcols;
            float s1 = 0.0f;
            if (!fail) {
                tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < ncols; c0 += 32) {
                    float z[32];
                    __syncwarp();
                    tmem_ld32v(tz + c0, z);
                    tmem_ld_wait();
                    regs_ready<32>(z);
                    const float4* b4 = reinterpret_cast<const float4*>(bias_w + c0);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 v = b4[c];
                        z[4 * c] += v.x;
                        z[4 * c + 1] += v.y;
                        z[4 * c + 2] += v.z;
                        z[4 * c + 3] += v.w;
                    }
                    if (row_ok) {
                        const uint4* rs =
                            reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.resid) + grow * q.N + n0 + c0);
#pragma unroll
                        for (int u4 = 0; u4 < 4; ++u4) {
                            uint4 u = rs[u4];
                            const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
                            for (int j = 0; j < 8; ++j) z[u4 * 8 + j] += Cvt<T>::to_f(e[j]);
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 32; ++c) s1 += z[c];
                    tmem_st32v(tz + c0, z);
                }
                tmem_st_wait();
            }
            // this CTA's columns of the row: n_c of them, sum S_c, mean m_c
            red[half * kTM + r] = s1;
            if (named_bar_any(1, kEpiWarps * 32, fail)) return false;
            const int n_c = min(kTN, q.N - at.col0);
            const float sum_c = red[r] + red[kTM + r];
            const float mean_c = sum_c / (float)n_c;
            float s2 = 0.0f;
#pragma unroll 1
            for (int c0 = 0; c0 < ncols; c0 += 32) {
                float z[32];
                __syncwarp();
                tmem_ld32v(tz + c0, z);
                tmem_ld_wait();
                regs_ready<32>(z);
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float d = z[c] - mean_c;
                    s2 = fmaf(d, d, s2);
                }
            }
            red[(2 + half) * kTM + r] = s2;
            named_bar_sync(1, kEpiWarps * 32);
            // (S_c, M2_c) into every CTA's slot for this CTA, then one
            // arrival on each CTA's barrier of this buffer
            const uint32_t e = ln_cnt & 1, parity = (ln_cnt >> 1) & 1;
            ++ln_cnt;
            if (half == 0) {
                const float m2_c = red[2 * kTM + r] + red[3 * kTM + r];
                const uint32_t slot = smem_u32(xch + ((e * kMaxLnCtas + rank) * 2) * kTM + r);
                for (int qq = 0; qq < p.ln_ctas; ++qq) {
                    st_cluster_f32(mapa_shared(slot, (uint32_t)qq), sum_c);
                    st_cluster_f32(mapa_shared(slot + kTM * 4, (uint32_t)qq), m2_c);
                }
                fence_acq_rel_cluster();
            }
            named_bar_sync(1, kEpiWarps * 32);
            if (warp == 4 && lane == 0)
                for (int qq = 0; qq < p.ln_ctas; ++qq)
                    mbar_arrive_cluster(mapa_shared(smem_u32(&xbar[e]), (uint32_t)qq));
            const bool got = __all_sync(0xffffffffu, mbar_wait_cluster(&xbar[e], parity, abort_flag));
            if (named_bar_any(1, kEpiWarps * 32, !got)) return false;
            const float* xe = xch + (size_t)e * kMaxLnCtas * 2 * kTM + r;
            float tot = 0.0f;
            for (int qq = 0; qq < p.ln_ctas; ++qq) tot += xe[qq * 2 * kTM];
            const float mean = tot / (float)q.N;
            float m2 = 0.0f;
            for (int qq = 0; qq < p.ln_ctas; ++qq) {
                const float n_q = (float)min(kTN, q.N - qq * kTN);
                const float d = xe[qq * 2 * kTM] / n_q - mean;
                m2 += fmaf(n_q * d, d, xe[(qq * 2 + 1) * kTM]);
            }
            const float inv = rsqrtf(m2 / (float)q.N + p.ln_eps);
#pragma unroll 1
            for (int c0 = 0; c0 < ncols; c0 += 32) {
                float z[32];
                __syncwarp();
                tmem_ld32v(tz + c0, z);
                tmem_ld_wait();
                regs_ready<32>(z);
                if (row_ok) {
                    const int n = n0 + c0;
                    uint4* d4 = reinterpret_cast<uint4*>(reinterpret_cast<T*>(q.out) + grow * q.N + n);
                    const float4* g4 = reinterpret_cast<const float4*>(gam_w + c0);
                    const float4* be4 = reinterpret_cast<const float4*>(bet_w + c0);
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4) {
                        const float4 ga = g4[2 * u4], gb = g4[2 * u4 + 1];
                        const float4 ba = be4[2 * u4], bb = be4[2 * u4 + 1];
                        const float gm[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
                        const float bt[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
                        float y[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) y[j] = fmaf((z[u4 * 8 + j] - mean) * inv, gm[j], bt[j]);
                        uint4 u;
                        u.x = Cvt<T>::two(y[0], y[1]);
                        u.y = Cvt<T>::two(y[2], y[3]);
                        u.z = Cvt<T>::two(y[4], y[5]);
                        u.w = Cvt<T>::two(y[6], y[7]);
                        d4[u4] = u;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
            return true;
        };
        uint32_t tc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++tc) {
            const TileAt at = tile_at(p, t);
            const GemmProb& q = p.pr[at.pi];
            const int mt = at.mt, b = at.b;
            const T* bias = reinterpret_cast<const T*>(q.bias);
            const int wcols = at.width / 2;                // columns of each of the two warps
            const int n0 = at.col0 + half * wcols;         // this warp's columns
            int ncols = q.N - n0 < wcols ? q.N - n0 : wcols;  // a multiple of 32, maybe <= 0
            if (ncols < 0) ncols = 0;
            // this warp's copy of its columns' bias
#pragma unroll
            for (int c = 0; c < kTN / 64; ++c)
                if (c * 32 < ncols) bias_w[c * 32 + lane] = Cvt<T>::to_f(bias[n0 + c * 32 + lane]);
            if (p.mode == kEpiResidLN) {  // and of its columns' gamma and beta
#pragma unroll
                for (int c = 0; c < kTN / 64; ++c)
                    if (c * 32 < ncols) {
                        gam_w[c * 32 + lane] = p.ln_gamma[n0 + c * 32 + lane];
                        bet_w[c * 32 + lane] = p.ln_beta[n0 + c * 32 + lane];
                    }
            }
            __syncwarp();
            const uint32_t ab = tc & 1;
            if (p.mode == kEpiResidLN) {
                if (!ln_tile(at, q, ab, tc, n0, ncols, wcols)) {
                    ok = false;
                    break;
                }
                continue;
            }
            ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[ab], (tc >> 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const int m = mt * kTM + r;  // row within the batch
            const bool row_ok = m < q.rows;
            const size_t grow = (size_t)b * q.rows + m;  // global row (row-major outputs)
#pragma unroll 1
            for (int c0 = 0; c0 < ncols; c0 += 32) {
                float acc[32];
                __syncwarp();  // tcgen05.ld is .sync.aligned: whole warp, converged
                tmem_ld32v(tmem + lane_off + ab * kTN + half * wcols + c0, acc);
                tmem_ld_wait();
                regs_ready<32>(acc);
#pragma unroll
                for (int c = 0; c < 32; ++c) acc[c] += bias_w[c0 + c];
                const int n = n0 + c0;
                if (p.mode == kEpiGelu) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) acc[c] = gelu_erf(acc[c]);
                }
                if (!row_ok) {
                } else if (p.mode == kEpiResid) {
                    const uint4* rs = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.resid) + grow * q.N + n);
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4) {
                        uint4 u = rs[u4];
                        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[u4 * 8 + j] += Cvt<T>::to_f(e[j]);
                    }
                    float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(q.out) + grow * q.N + n);
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        dst[v] = make_float4(acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3]);
                } else {
                    T* dst;
                    if (p.mode == kEpiHeads) {
                        const int which = n / p.heads_D;
                        const int h = (n % p.heads_D) / 64, d = n % 64;
                        dst = reinterpret_cast<T*>(q.out) +
                              ((((size_t)which * p.batches + b) * p.heads_H + h) * q.heads_L + m) * 64 + d;
                    } else {
                        dst = reinterpret_cast<T*>(q.out) + grow * q.N + n;
                    }
                    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 u;
                        u.x = Cvt<T>::two(acc[8 * q + 0], acc[8 * q + 1]);
                        u.y = Cvt<T>::two(acc[8 * q + 2], acc[8 * q + 3]);
                        u.z = Cvt<T>::two(acc[8 * q + 4], acc[8 * q + 5]);
                        u.w = Cvt<T>::two(acc[8 * q + 6], acc[8 * q + 7]);
                        d4[q] = u;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
    }

    __syncthreads();
    // no CTA leaves while a peer may still write into its exchange slots
    if (p.mode == kEpiResidLN) cluster_sync();
    if (threadIdx.x == 0 && *abort_flag) record_status(p.status, 0, LF_ERR_DEVICE_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

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

// A [batches][batch_stride rows][K] (tiles over the first `rows` of each
// batch) and W [N][K], both K-major.
bool encode_w(EncodeTiledFn enc, CUtensorMap* mw, const void* W, int N, int K, int box_rows) {
    cuuint64_t wdims[2] = {(cuuint64_t)K, (cuuint64_t)N};
    cuuint64_t wstr[1] = {(cuuint64_t)K * 2};
    cuuint32_t wbox[2] = {(cuuint32_t)kTK, (cuuint32_t)box_rows};
    cuuint32_t e2[2] = {1, 1};
    return enc(mw, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(W), wdims, wstr, wbox, e2,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_ab(EncodeTiledFn enc, CUtensorMap* ma, CUtensorMap* mw, const void* A, int batches, int rows,
               int batch_stride, int K, const void* W, int N) {
    cuuint64_t adims[3] = {(cuuint64_t)K, (cuuint64_t)rows, (cuuint64_t)batches};
    cuuint64_t astr[2] = {(cuuint64_t)K * 2, (cuuint64_t)batch_stride * K * 2};
    cuuint32_t abox[3] = {(cuuint32_t)kTK, (cuuint32_t)kTM, 1};
    cuuint32_t e3[3] = {1, 1, 1};
    if (enc(ma, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(A), adims, astr, abox, e3,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    return encode_w(enc, mw, W, N, K, kTN);
}

GemmProb make_prob(int batches, int rows, int N, const void* bias, void* out, int heads_L) {
    GemmProb q;
    q.rows = rows;
    q.N = N;
    q.mtiles = (rows + kTM - 1) / kTM;
    q.ntiles = (N + kTN - 1) / kTN;
    q.tiles = batches * q.mtiles * q.ntiles;
    q.bias = bias;
    q.out = out;
    q.heads_L = heads_L;
    return q;
}

template <typename T>
lf_status launch_t(const GemmArgs& g, int sm_count, cudaStream_t stream) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return LF_ERR_CUDA;
    CUtensorMap ma, mw, ma2, mw2, mwh, mw2h;
    if (!encode_ab(enc, &ma, &mw, g.A, g.batches, g.rows, g.batch_stride, g.K, g.W, g.N) ||
        !encode_w(enc, &mwh, g.W, g.N, g.K, kTN / 2))
        return LF_ERR_CUDA;
    GemmParams p;
    p.batches = g.batches;
    p.K = g.K;
    p.ktiles = g.K / kTK;
    p.pr[0] = make_prob(g.batches, g.rows, g.N, g.bias, g.out, g.heads_L);
    p.pr[1] = make_prob(g.batches, 0, 128, nullptr, nullptr, 0);
    p.pr[1].tiles = 0;
    if (g.rows2 > 0) {
        if (!encode_ab(enc, &ma2, &mw2, g.A2, g.batches, g.rows2, g.batch_stride2, g.K, g.W2, g.N2) ||
            !encode_w(enc, &mw2h, g.W2, g.N2, g.K, kTN / 2))
            return LF_ERR_CUDA;
        p.pr[1] = make_prob(g.batches, g.rows2, g.N2, g.bias2, g.out2, g.heads_L2);
    } else {
        ma2 = ma;
        mw2 = mw;
        mw2h = mwh;
    }
    // Whole rounds of full tiles, then the remaining R tiles as 2R halves
    // when they fit in one round (R <= grid / 2): that round then takes half
    // a tile's time on up to every SM instead of a whole one on R of them.
    const int nt = p.pr[0].tiles + p.pr[1].tiles;
    int G = nt < sm_count ? nt : sm_count;
    const int R = nt % G;
    p.n_split = (nt > G && R > 0 && 2 * R <= G) ? R : 0;
    // kEpiResidLN: the row tile's column tiles form a cluster, whole tiles only
    const bool ln = g.mode == kEpiResidLN;
    const int C = ln ? p.pr[0].ntiles : 1;
    if (ln) {
        if (C > kMaxLnCtas || g.rows2 > 0 || !g.ln_gamma || !g.ln_beta) return LF_ERR_BAD_DIM;
        p.n_split = 0;
        G = G / C * C;
    }
    p.t_full = nt - p.n_split;
    p.tiles = nt + p.n_split;
    p.ln_gamma = g.ln_gamma;
    p.ln_beta = g.ln_beta;
    p.ln_eps = g.ln_eps;
    p.ln_ctas = C;
    p.mode = g.mode;
    p.w_early = g.w_early ? 1 : 0;
    p.resid = g.resid;
    p.heads_D = g.heads_D;
    p.heads_H = g.heads_H;
    p.status = g.status;
    // the shared-memory opt-in is a per-device function attribute
    static std::atomic<bool> attr[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LF_ERR_CUDA;
    if (!attr[dev].load()) {
        if (cudaFuncSetAttribute(gemm_tc_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
            cudaSuccess)
            return LF_ERR_CUDA;
        attr[dev].store(true);
    }
    const int grid = G;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = C;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = ln ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, gemm_tc_kernel<T>, ma, mw, ma2, mw2, mwh, mw2h, p) != cudaSuccess) return LF_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

}  // namespace

lf_status launch_gemm_tc(const GemmArgs& g, lf_dtype dtype, int sm_count, cudaStream_t stream) {
    if (g.N % 128 != 0 || g.K % kTK != 0 || g.rows <= 0 || g.batches <= 0) return LF_ERR_BAD_DIM;
    if (g.rows2 > 0 && (g.N2 % 128 != 0 || g.N2 <= 0 || g.mode != kEpiHeads)) return LF_ERR_BAD_DIM;
    if (dtype == LF_F16) return launch_t<__half>(g, sm_count, stream);
    if (dtype == LF_BF16) return launch_t<__nv_bfloat16>(g, sm_count, stream);
    return LF_ERR_DTYPE;
}

}  // namespace lf
