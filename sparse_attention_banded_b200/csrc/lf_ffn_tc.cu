// Fused GELU feed-forward network on the sm_100a tensor cores: the fused
// linear -> GELU -> linear of the PaddleNLP FastFFN page (§FastFFN融合计算),
// applied to step 6 of the FasterTransformer Longformer page's layer
// (§Longformer Encoder 计算流程 / 每个 Transformer 层, GeluFfnLayer):
//
//   z[r, :] = h[r, :] + b_2 + GELU(h[r, :] W_1^T + b_1) W_2^T     (fp32 out)
//
// with the F-wide intermediate kept on chip, in 128-wide chunks, and rounded
// to T as the two-GEMM path stores it.
//
// A cluster of CS CTAs (CS = 1, 2 or 4) owns a 128-row tile of h.  CTA r of
// the cluster holds the output columns [r*NQ, (r+1)*NQ), NQ = D/CS <= 256,
// as an fp32 accumulator in TMEM, and produces every CS-th chunk of the
// intermediate: chunk c = t*CS + r in round t.
//   warp 0      TMA loads through a ring of 32 KB stages, in the MMA order
//   warp 1      tcgen05.mma: round t's own chunk (h tile x 128 rows of W_1,
//               M=128 N=128 K=D) into one of two 128-column TMEM buffers,
//               then the CS chunks of round t-1 (chunk x its NQ x 128 block
//               of W_2, M=128 N=NQ K=128) into the output accumulator, in
//               chunk order
//   warp 2      hands "chunk consumed" on to the chunk's producer (an
//               mbarrier arrive in that CTA) when this CTA's MMAs on it are
//               done
//   warps 4-11  the chunk epilogue (TMEM -> + b_1 -> GELU -> T, written into
//               shared memory in the 128-byte-swizzled K-major operand
//               layout), then one thread copies the chunk into the same slot
//               of every other CTA of the cluster (bulk shared-to-distributed
//               -shared copies, each to one CTA and completing on its
//               mbarrier); after the last round the output epilogue
//               (+ b_2 + h, fp32 stores)
// Every CTA's sums over the intermediate run over k in the order of the
// two-GEMM path (chunk by chunk, 16 at a time), as do the sums over D.
//
// TMEM (512 columns): output accumulator [0, NQ), chunk buffers at 256 and
// 384.  Shared memory: CS chunk slots of 32 KB (two 64-wide swizzle atoms of
// 128 rows) and the ring, about 224 KB, so one CTA per SM.
// Roofline: tensor-bound, 4*M*D*F flops; the operands stream from L2.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>

#include "lf_gelu.cuh"
#include "lf_internal.h"
#include "sm100_cluster.cuh"

namespace lf {
namespace {

using namespace sm100;

constexpr int kTM = 128;        // rows per tile
constexpr int kChunk = 128;     // intermediate columns per chunk
constexpr int kTK = 64;         // K per ring stage (one swizzle atom)
constexpr int kThreads = 384;   // 12 warps: 0 TMA, 1 MMA, 2 forwarder, 3 idle, 4-11 epilogue
constexpr int kEpiWarps = 8;
constexpr uint32_t kStageBytes = 32768;
constexpr uint32_t kSlotBytes = kTM * kChunk * 2;  // 32 KB
constexpr uint32_t kAtomBytes = kTM * kTK * 2;     // 16 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemChunk = 256;  // first chunk buffer's column

template <int CS>
struct Cfg {
    static constexpr int kSlots = CS;
    static constexpr int kStages = CS == 4 ? 3 : CS == 2 ? 5 : 6;
    static constexpr uint32_t kOffRing = 0;
    static constexpr uint32_t kOffSlot = kOffRing + kStages * kStageBytes;
    static constexpr uint32_t kOffBar = kOffSlot + kSlots * kSlotBytes;
    // full, empty (ring); chunk_full, chunk_empty (TMEM buffers); slot_full,
    // consumed (per slot); slot_free; out_full; drain
    static constexpr uint32_t kNumBars = 2 * kStages + 4 + 2 * kSlots + 3;
    static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
    static constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory");
};

struct FfnParams {
    int M, D, F;
    int NQ;       // output columns per CTA
    int rounds;   // F / (kChunk * CS)
    const void* b1;     // [F]
    const void* b2;     // [D]
    const void* resid;  // [M][D]
    float* out;         // [M][D]
    int* status;
};

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

__device__ __forceinline__ void tmem_ld32f(uint32_t taddr, float (&r)[32]) {
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

// The erf form of GELU, as the two-GEMM path's epilogue computes it.
__device__ __forceinline__ float gelu_erf(float x) { return gelu_erf_as(x); }

template <typename T, int CS>
__global__ void __launch_bounds__(kThreads, 1)
ffn_fused_kernel(const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_w1,
                 const __grid_constant__ CUtensorMap map_w2, const __grid_constant__ FfnParams p) {
    using C = Cfg<CS>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* full = bars;
    uint64_t* empty = full + S;
    uint64_t* chunk_full = empty + S;    // [2] MMA -> epilogue: a chunk's pre-activation is in TMEM
    uint64_t* chunk_empty = chunk_full + 2;  // [2] epilogue -> MMA: that TMEM buffer is read
    uint64_t* slot_full = chunk_empty + 2;   // [CS] the chunk of producer p is in slot p (this CTA)
    uint64_t* consumed = slot_full + CS;     // [CS] this CTA's MMAs on slot p are done
    uint64_t* slot_free = consumed + CS;     // every CTA's MMAs on this CTA's chunk are done (CS arrivals)
    uint64_t* out_full = slot_free + 1;      // the output accumulator is final
    uint64_t* drain = out_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    // [CS] phases of slot_full[q] the MMA warp has taken (for the wind-down)
    volatile uint32_t* slot_used = reinterpret_cast<volatile uint32_t*>(smem + C::kOffMisc + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = CS > 1 ? cluster_ctarank() : 0;
    const int m0 = (int)(CS > 1 ? cluster_id_x() : blockIdx.x) * kTM;
    const int NQ = p.NQ;
    const int R = p.rounds;
    // The next kernel in the stream may be scheduled now (it waits for this
    // one before touching memory).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&chunk_full[i], 1);
            mbar_init(&chunk_empty[i], kEpiWarps);
        }
        for (int i = 0; i < CS; ++i) {
            mbar_init(&slot_full[i], 1);
            mbar_init(&consumed[i], 1);
            slot_used[i] = 0;
        }
        mbar_init(slot_free, CS);
        mbar_init(out_full, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&map_h);
        prefetch_tensormap(&map_w1);
        prefetch_tensormap(&map_w2);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // every CTA's barriers are initialised before any peer arrives on them
    if (CS > 1) cluster_sync();
    const uint32_t tmem = *tmem_slot;
    // Launched as a programmatic dependent: no global memory is read or
    // written before the kernel before this one has completed.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    auto wait_all_cluster = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait_cluster(bar, parity, abort_flag));
    };
    const int ksteps = p.D / kTK;  // ring stages of one round's own chunk
    const uint32_t w2_bytes = (uint32_t)NQ * kTK * 2;

    if (warp == 0) {
        // ---- TMA: round t's own chunk (h, W_1), then round t-1's W_2 blocks
        uint32_t kc = 0;
        bool ok = true;
        for (int t = 0; t <= R && ok; ++t) {
            if (t < R) {
                const int c = t * CS + (int)rank;
                for (int kt = 0; kt < ksteps && ok; ++kt, ++kc) {
                    const uint32_t st = kc % S;
                    ok = wait_all(&empty[st], ((kc / S) & 1) ^ 1);
                    if (!ok) break;
                    if (lane == 0) {
                        uint8_t* stage = smem + C::kOffRing + st * kStageBytes;
                        mbar_arrive_expect_tx(&full[st], 2 * kAtomBytes);
                        tma_load_2d(stage, &map_h, &full[st], kt * kTK, m0);
                        tma_load_2d(stage + kAtomBytes, &map_w1, &full[st], kt * kTK, c * kChunk);
                    }
                    __syncwarp();
                }
            }
            if (t >= 1) {
                for (int q = 0; q < CS && ok; ++q) {
                    const int c = (t - 1) * CS + q;
                    for (int a = 0; a < 2 && ok; ++a, ++kc) {
                        const uint32_t st = kc % S;
                        ok = wait_all(&empty[st], ((kc / S) & 1) ^ 1);
                        if (!ok) break;
                        if (lane == 0) {
                            uint8_t* stage = smem + C::kOffRing + st * kStageBytes;
                            mbar_arrive_expect_tx(&full[st], w2_bytes);
                            tma_load_2d(stage, &map_w2, &full[st], c * kChunk + a * kTK, (int)rank * NQ);
                        }
                        __syncwarp();
                    }
                }
            }
        }
        if (!ok && lane == 0) {  // wind-down: let issued copies land
            for (uint32_t c = (kc > (uint32_t)S ? kc - S : 0); c < kc; ++c) {
                volatile int never = 0;
                mbar_wait(&full[c % S], (c / S) & 1, &never, 200000000ull);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue
        constexpr uint32_t idesc1 = idesc_f16(Cvt<T>::fmt, kTM, kChunk, 0, 0);
        const uint32_t idesc2 = idesc_f16(Cvt<T>::fmt, kTM, (uint32_t)NQ, 0, 0);
        uint32_t kc = 0;
        bool ok = true;
        for (int t = 0; t <= R && ok; ++t) {
            if (t < R) {
                const uint32_t hb = t & 1;
                ok = wait_all(&chunk_empty[hb], ((t >> 1) & 1) ^ 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d = tmem + kTmemChunk + hb * kChunk;
                for (int kt = 0; kt < ksteps && ok; ++kt, ++kc) {
                    const uint32_t st = kc % S;
                    ok = wait_all(&full[st], (kc / S) & 1);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t a_addr = smem_u32(smem + C::kOffRing + st * kStageBytes);
                        const uint32_t b_addr = a_addr + kAtomBytes;
#pragma unroll
                        for (int kk = 0; kk < kTK / 16; ++kk)
                            mma_f16_ss(d, desc_sw128(a_addr + kk * 32), desc_sw128(b_addr + kk * 32), idesc1,
                                       (kt > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(&empty[st]);
                    }
                    __syncwarp();
                }
                if (ok && lane == 0) tc_commit(&chunk_full[hb]);
                __syncwarp();
            }
            if (t >= 1) {
                for (int q = 0; q < CS && ok; ++q) {
                    const int c = (t - 1) * CS + q;
                    ok = wait_all_cluster(&slot_full[q], (t - 1) & 1);
                    if (!ok) break;
                    if (lane == 0) slot_used[q] = (uint32_t)t;
                    const uint32_t slot = smem_u32(smem + C::kOffSlot + q * kSlotBytes);
                    for (int a = 0; a < 2 && ok; ++a, ++kc) {
                        const uint32_t st = kc % S;
                        ok = wait_all(&full[st], (kc / S) & 1);
                        if (!ok) break;
                        tc_fence_after();
                        if (lane == 0) {
                            const uint32_t b_addr = smem_u32(smem + C::kOffRing + st * kStageBytes);
#pragma unroll
                            for (int kk = 0; kk < kTK / 16; ++kk)
                                mma_f16_ss(tmem, desc_sw128(slot + a * kAtomBytes + kk * 32),
                                           desc_sw128(b_addr + kk * 32), idesc2, (c > 0 || a > 0 || kk > 0) ? 1u : 0u);
                            tc_commit(&empty[st]);
                        }
                        __syncwarp();
                    }
                    if (ok && lane == 0) tc_commit(&consumed[q]);
                    __syncwarp();
                }
            }
        }
        if (ok && lane == 0) tc_commit(out_full);
        __syncwarp();
        if (!ok && lane == 0) {
            tc_commit(drain);
            volatile int never = 0;
            mbar_wait(drain, 0, &never, 200000000ull);
        }
    } else if (warp == 2) {
        // ---- "consumed" forwarder: chunk c's slot may be refilled by its
        // producer once every CTA's MMAs on it are done
        const uint32_t free_local = smem_u32(slot_free);
        bool ok = true;
        for (int c = 0; c < R * CS && ok; ++c) {
            const int q = c % CS, t = c / CS;
            ok = wait_all(&consumed[q], t & 1);
            if (ok && lane == 0) mbar_arrive_cluster(CS > 1 ? mapa_shared(free_local, (uint32_t)q) : free_local);
            __syncwarp();
        }
    } else if (warp >= 4) {
        // ---- epilogue: one thread per row, two warps per TMEM lane quarter
        // (each takes 64 of a chunk's columns, i.e. one swizzle atom)
        const int sp = warp & 3;
        const int half = (warp - 4) >> 2;
        const int r = sp * 32 + lane;
        const uint32_t lane_off = (uint32_t)(sp * 32) << 16;
        const T* b1 = reinterpret_cast<const T*>(p.b1);
        uint8_t* slot_own = smem + C::kOffSlot + rank * kSlotBytes;
        bool ok = true;
        for (int t = 0; t < R; ++t) {
            const int c = t * CS + (int)rank;
            const uint32_t hb = t & 1;
            // this chunk's 64 biases, fetched before the wait (off the critical path)
            uint4 bq[8];
            const uint4* bb = reinterpret_cast<const uint4*>(b1 + c * kChunk + half * 64);
#pragma unroll
            for (int q = 0; q < 8; ++q) bq[q] = bb[q];
            bool fail = !__all_sync(0xffffffffu, mbar_wait(&chunk_full[hb], (t >> 1) & 1, abort_flag));
            float v[2][32];
            if (!fail) {
                tc_fence_after();
                tmem_ld32f(tmem + lane_off + kTmemChunk + hb * kChunk + half * 64, v[0]);
                tmem_ld32f(tmem + lane_off + kTmemChunk + hb * kChunk + half * 64 + 32, v[1]);
                tmem_ld_wait();
                regs_ready<32>(v[0]);
                regs_ready<32>(v[1]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&chunk_empty[hb]);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint4 u = bq[q];
                    const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float& x = v[q >> 2][(q & 3) * 8 + j];
                        x += Cvt<T>::to_f(e[j]);
                        x = gelu_erf(x);
                    }
                }
                // this CTA's slot is refilled once every CTA's MMAs on its
                // previous chunk are done
                if (t > 0) fail = !__all_sync(0xffffffffu, mbar_wait_cluster(slot_free, (t - 1) & 1, abort_flag));
            }
            if (!fail) {
                uint8_t* row = slot_own + half * kAtomBytes + r * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float* x = &v[j >> 2][(j & 3) * 8];
                    uint4 u;
                    u.x = Cvt<T>::two(x[0], x[1]);
                    u.y = Cvt<T>::two(x[2], x[3]);
                    u.z = Cvt<T>::two(x[4], x[5]);
                    u.w = Cvt<T>::two(x[6], x[7]);
                    *reinterpret_cast<uint4*>(row + ((j ^ (r & 7)) << 4)) = u;
                }
                fence_proxy_async_smem();
            }
            // every epilogue warp takes the same branch: the barrier reduces
            // the failures of all of them
            if (named_bar_any(1, kEpiWarps * 32, fail)) {
                ok = false;
                break;
            }
            if (warp == 4 && lane == 0) {
                mbar_arrive(&slot_full[rank]);
                const uint32_t bar_local = smem_u32(&slot_full[rank]);
                const uint32_t dst_local = smem_u32(slot_own);
                for (int q = 1; q < CS; ++q) {
                    const uint32_t peer = (rank + (uint32_t)q) % CS;
                    const uint32_t bar_peer = mapa_shared(bar_local, peer);
                    mbar_arrive_expect_tx_cluster(bar_peer, kSlotBytes);
                    bulk_copy_to_peer(mapa_shared(dst_local, peer), slot_own, kSlotBytes, bar_peer);
                }
            }
            __syncwarp();
        }
        if (ok && __all_sync(0xffffffffu, mbar_wait(out_full, 0, abort_flag))) {
            // output: + b_2 + h, fp32 row-major
            tc_fence_after();
            // the two warps of a lane quarter split the NQ / 32 column groups
            const int groups = NQ / 32, g0 = (groups + 1) / 2;
            const int col0 = half == 0 ? 0 : g0 * 32;
            const int ncols = (half == 0 ? g0 : groups - g0) * 32;
            const int n0 = (int)rank * NQ + col0;
            const int row = m0 + r;
            const bool row_ok = row < p.M;
            const T* b2 = reinterpret_cast<const T*>(p.b2);
            const T* res = reinterpret_cast<const T*>(p.resid) + (size_t)row * p.D + n0;
            float* dst = p.out + (size_t)row * p.D + n0;
#pragma unroll 1
            for (int c0 = 0; c0 < ncols; c0 += 32) {
                float acc[32];
                __syncwarp();
                tmem_ld32f(tmem + lane_off + col0 + c0, acc);
                tmem_ld_wait();
                regs_ready<32>(acc);
                const uint4* bb = reinterpret_cast<const uint4*>(b2 + n0 + c0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 u = bb[q];
                    const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[q * 8 + j] += Cvt<T>::to_f(e[j]);
                }
                if (row_ok) {
                    const uint4* rs = reinterpret_cast<const uint4*>(res + c0);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 u = rs[q];
                        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[q * 8 + j] += Cvt<T>::to_f(e[j]);
                    }
                    float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        d4[q] = make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]);
                }
            }
            tc_fence_before();
        }
    }

    __syncthreads();
    // no CTA leaves while a peer may still arrive on or copy into it
    if (CS > 1) {
        cluster_sync();
        // Every copy into this CTA has been issued by now.  A CTA that gave
        // up may not have taken the last phase of a peer's slot: wait, with
        // a short limit, for that phase (a copy in flight lands within
        // microseconds; a peer that sent nothing leaves it to time out),
        // then leave together, so that no copy's source or destination goes
        // away while it is in flight.
        if (warp == 1 && *abort_flag) {
            for (int q = 0; q < CS; ++q) {
                if (q == (int)rank) continue;
                volatile int never = 0;
                mbar_wait_cluster(&slot_full[q], slot_used[q] & 1u, &never, 2000000ull);
            }
        }
        __syncwarp();
        cluster_sync();
    }
    if (threadIdx.x == 0 && *abort_flag) record_status(p.status, 0, LF_ERR_DEVICE_TIMEOUT);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}
}  // namespace
}  // namespace lf

namespace lf {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn ffn_encode_fn() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load();
    if (!f) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            f = reinterpret_cast<EncodeTiledFn>(ptr);
            fn.store(f);
        }
    }
    return f;
}

// 2-D K-major fp16/bf16 matrix [rows][cols] with a box of 64 columns x box_rows.
bool encode_2d(EncodeTiledFn enc, CUtensorMap* m, const void* base, int cols, int rows, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t str[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)kTK, (cuuint32_t)box_rows};
    cuuint32_t e[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, str, box, e,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int CS>
lf_status launch_fused_t(const FfnArgs& a, cudaStream_t stream) {
    using C = Cfg<CS>;
    EncodeTiledFn enc = ffn_encode_fn();
    if (!enc) return LF_ERR_CUDA;
    const int NQ = a.D / CS;
    CUtensorMap mh, m1, m2;
    if (!encode_2d(enc, &mh, a.h, a.D, a.M, kTM) || !encode_2d(enc, &m1, a.W1, a.D, a.F, kChunk) ||
        !encode_2d(enc, &m2, a.W2, a.F, a.D, NQ))
        return LF_ERR_CUDA;
    FfnParams p;
    p.M = a.M;
    p.D = a.D;
    p.F = a.F;
    p.NQ = NQ;
    p.rounds = a.F / (kChunk * CS);
    p.b1 = a.b1;
    p.b2 = a.b2;
    p.resid = a.h;
    p.out = a.out;
    p.status = a.status;
    // the shared-memory opt-in is a per-device function attribute
    static std::atomic<bool> attr[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LF_ERR_CUDA;
    if (!attr[dev].load()) {
        if (cudaFuncSetAttribute(ffn_fused_kernel<T, CS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes) != cudaSuccess)
            return LF_ERR_CUDA;
        attr[dev].store(true);
    }
    const int mtiles = (a.M + kTM - 1) / kTM;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = CS;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(mtiles * CS));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = CS > 1 ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, ffn_fused_kernel<T, CS>, mh, m1, m2, p) != cudaSuccess) return LF_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

template <typename T>
lf_status launch_fused_cs(const FfnArgs& a, cudaStream_t stream) {
    switch (ffn_fused_cluster(a.D)) {
        case 1: return launch_fused_t<T, 1>(a, stream);
        case 2: return launch_fused_t<T, 2>(a, stream);
        case 4: return launch_fused_t<T, 4>(a, stream);
        default: return LF_ERR_BAD_DIM;
    }
}

}  // namespace

int ffn_fused_cluster(int D) {
    if (D <= 0 || D % 128 != 0 || D > 1024) return 0;
    return D <= 256 ? 1 : D <= 512 ? 2 : 4;
}

bool ffn_fused_supported(int M, int D, int F) {
    const int cs = ffn_fused_cluster(D);
    return cs > 0 && M > 0 && F > 0 && F % (kChunk * cs) == 0;
}

lf_status launch_ffn_fused(const FfnArgs& a, lf_dtype dtype, cudaStream_t stream) {
    if (!ffn_fused_supported(a.M, a.D, a.F)) return LF_ERR_BAD_DIM;
    if (dtype == LF_F16) return launch_fused_cs<__half>(a, stream);
    if (dtype == LF_BF16) return launch_fused_cs<__nv_bfloat16>(a, stream);
    return LF_ERR_DTYPE;
}

}  // namespace lf
