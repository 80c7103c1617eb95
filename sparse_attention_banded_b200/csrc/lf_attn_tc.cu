// Longformer banded + global self-attention on the sm_100a tensor cores.
//
// The FasterTransformer Longformer page ("FasterTransformer Longformer 推理加速
// 实践"), §Longformer Encoder 计算流程 / 每个 Transformer 层 steps 3-5, runs
// this layer as window GEMMs over head/middle/tail segments, a separate
// masked-softmax kernel and a transpose kernel.  Here it is ONE persistent
// kernel per call.
//
// Work items: CTA c takes item c first, later ones come from a global atomic
// counter.  Global pairs come first (the longest items; their split merges
// then overlap the band work that follows), then the band pairs away from
// the sequence ends, then the band pairs at the sequence ends:
//   global pair (b, h, row tile rt, splits 2s and 2s+1): rows i < g_b attend
//       to every key through qg/kg/vg.  Keys are cut into chunks of `chunk`
//       128-key blocks (picked per shape on the host so that the items pack
//       evenly onto the SMs); each split leaves (m, l, O) partials in
//       scratch and the epilogue warp that finishes the last split of its 32
//       rows merges them (log-sum-exp) and writes the rows.
//   band pair (b, h, tiles 2p and 2p+1 of 128 query rows): each tile visits
//       the 128-key blocks that meet its rows' windows |i - j| <= w and the
//       blocks of global keys 0..g_b-1 seen outside the window, with the mask
//       allowed(i, j) = j < g_b || |i - j| <= w, so a global key inside a
//       window counts once.  The two tiles share every K/V block they both
//       need (loaded once).
//
// Roles (512 threads = 4 warpgroups): warp 0 issues TMA loads (Q of both
// tiles, K/V blocks into a kStages ring); warp 2 fetches items and publishes
// their plans through a ring; warps 1 and 3 issue the tcgen05.mma work of
// tile A and tile B; warpgroups 1 and 2 are the softmax warps of tiles A and
// B (one thread per query row); warpgroup 3 is the epilogue of both tiles.
// Registers are rebalanced with setmaxnreg from 128 per thread to 88, 152
// and 120.  Each tile owns 256 TMEM columns: S (fp32), P (fp16/bf16 pairs)
// and O (fp32).  Per tile X and key block j:
//   S_X = Q_X K_j^T            (issued once the softmax has read S of j - 1)
//   softmax warps: read S_X, scale, padding bias, mask, row max; rescale the
//   TMEM accumulator O_X only when the running max grows by more than 8 (in
//   log2 units, so P <= 2^8); write P = exp2(x - m) as fp16/bf16 pairs
//   O_X += P_X V_j             (tcgen05.mma with A from TMEM)
// so a tile's next S runs while its softmax works on the current block, and
// the two tiles never wait on each other.  All waits are bounded; on expiry
// the CTA records LF_ERR_DEVICE_TIMEOUT and winds down.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <stdlib.h>

#include <algorithm>
#include <atomic>
#include <functional>
#include <mutex>
#include <vector>

#include "lf_internal.h"
#include "lf_pair_math.cuh"
#include "lf_partition.cuh"
#include "sm100.cuh"

namespace lf {
namespace {

using namespace sm100;

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // keys per block
constexpr int kHD = 64;           // head dim
constexpr int kStages = 5;        // K/V ring depth
constexpr int kMinChunk = 4;      // key blocks per global-row split: chosen per
constexpr int kMaxChunk = 16;     // shape in [kMinChunk, kMaxChunk] on the host
constexpr int kRing = 4;          // item-id ring depth
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kSoftmaxWarp0 = 4;  // warps 4-7: tile A, 8-11: tile B
constexpr int kEpiWarp0 = 12;     // warps 12-15: epilogue of both tiles
constexpr uint32_t kRegsProducer = 88;
constexpr uint32_t kRegsSoftmax = 152;
constexpr uint32_t kRegsEpi = 120;
static_assert(4 * 32 * kRegsProducer + 8 * 32 * kRegsSoftmax + 4 * 32 * kRegsEpi <= 65536, "register split");
constexpr int kItemConsumers = 1 + 2 + 8 + 4;  // TMA + 2 MMA + softmax + epilogue warps
constexpr uint32_t kTileBytes = kBM * kHD * 2;  // 16 KB
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;

// Shared memory map (offsets from a 1024-byte aligned base).
// Q of the current item's two tiles: the next item's Q is loaded once the
// current item's last S products are done, which frees the shared memory
// of a fifth K/V stage (the next item's first blocks load a block earlier).
constexpr uint32_t kOffQ = 0;                                 // [2 tile] x 16 KB
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;            // kStages x 16 KB
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;      // kStages x 16 KB
constexpr uint32_t kOffBias = kOffV + kStages * kTileBytes;   // 8 warps x 128 floats
constexpr uint32_t kOffStats = kOffBias + 8 * kBN * 4;        // [2 tiles][128 rows] (m, l)
constexpr uint32_t kOffPlans = kOffStats + 2 * kBM * 8;       // kRing plans
constexpr uint32_t kOffBar = kOffPlans + kRing * 128;
constexpr uint32_t kNumBars = 1 + 1 + 2 * kStages + 2 * 7 + 2 * kRing + 2 + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack

// TMEM columns per tile x (base x * 256): S [0,128) fp32, P [128,192)
// fp16/bf16 pairs, O [192,256) fp32.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemTile = 256;
constexpr uint32_t kTmemP = 128;
constexpr uint32_t kTmemO = 192;
static_assert(2 * kTmemTile <= kTmemCols && kTmemO + kHD <= kTmemTile, "TMEM budget");

struct Params {
    int B, H, L, w;
    int NKB;     // key blocks per head
    int NT;      // query tiles per head
    int RT;      // global row tiles per head (ceil(w / 128))
    int NS;      // key splits per global row tile
    int NSP;     // split pairs per global row tile
    int NTP;     // tile pairs per head
    int chunk;   // key blocks per global-row split
    int n_inner; // band pairs away from the sequence ends (after the global pairs)
    int n_glob;  // global pair items (first in the order)
    int n_items;
    float scale_log2;  // scale * log2(e)
    float inv_scale;   // 1 / scale: the padding bias in raw score units
    const float* local_mask;
    const float* global_mask;
    void* out;
    float* part_o;   // [B*H*RT*NS][128][64]
    float* part_ml;  // [B*H*RT*NS][128][2]
    int* counters;   // [B*H*RT][4]: per 32-row group of a global row tile
    int* sched;      // [0] next item, [1] finished CTAs
    int* status;
    int* trace;      // diagnostic builds only: [CTA][16 roles][4] wait sites, then [CTA][16 roles][16] cycle counts
    // Global tokens at any position (kernel instance kAny): the partition's
    // outputs and the slot buffers gathered from them.  Global row tiles
    // then hold slots (the c-th global token of the sample) instead of
    // positions, and a band tile's global key blocks are slot blocks read
    // from the compact k / v maps.
    const int* gnum;    // [B] global tokens per sample
    const int* gidx;    // [B][L] slot -> position (first gnum[b] entries)
    const int* grank;   // [B][L + 1] global tokens before each position
    const float* lm_c;  // [B][gcap] local_mask of each slot (0 past gnum[b])
    int gcap;           // slots per (b, h) in the compact buffers
    // Prefix instance, optional: the global-index partition of global_mask
    // (as lf_init_global_idx writes it), computed by the epilogue warps of
    // CTA b while the first items' scores are being computed.
    int32_t* gidx_out;  // [B][L] or NULL
    int32_t* gnum_out;  // [B]
    // The masks are not written by the kernel before this one (inside a
    // layer call): the planner builds its first plan and the softmax warps
    // read their masks before waiting for that kernel.
    int masks_early;
};

// Diagnostic builds (-DLF_TRACE=1) record per CTA and role the cycles spent
// in each wait and phase (written at the end of the role); with
// -DLF_TRACE_STATES=1 they also record the wait site each role is at, into
// host-mapped memory readable while the kernel runs (for locating a hang).
#ifndef LF_TRACE
#define LF_TRACE 0
#endif
// Wait-site states (each write is a system-scope fence: for locating a hang,
// not for timing).
#ifndef LF_TRACE_STATES
#define LF_TRACE_STATES 0
#endif
#if LF_TRACE && LF_TRACE_STATES
#define TRACE(role, state, item, a, b)                                                 \
    do {                                                                               \
        if (p.trace) {                                                                 \
            volatile int* t_ = p.trace + ((blockIdx.x * 16 + (role)) * 4);             \
            t_[1] = (int)(item);                                                       \
            t_[2] = (int)(a);                                                          \
            t_[3] = (int)(b);                                                          \
            __threadfence_system();                                                    \
            t_[0] = (state);                                                           \
        }                                                                              \
    } while (0)
#else
#define TRACE(role, state, item, a, b) \
    do {                               \
    } while (0)
#endif
#if LF_TRACE
// Cycle accounting per role: TIMED(k, stmt) adds the clock64() cycles of
// stmt to slot k; TDUMP(role) writes the 16 slots after the state words.
#define TDECL                  \
    long long tacc[16] = {0}; \
    const long long tstart_ = clock64()
#define TIMED(k, stmt)                   \
    do {                                 \
        const long long t0_ = clock64(); \
        stmt;                            \
        tacc[k] += clock64() - t0_;      \
    } while (0)
#define TCOUNT(k) (tacc[k] += 1)
#define TDUMP(role)                                                                             \
    do {                                                                                        \
        if (p.trace) {                                                                          \
            tacc[15] = clock64() - tstart_;                                                     \
            volatile int* d_ = p.trace + gridDim.x * 16 * 4 + (blockIdx.x * 16 + (role)) * 16;  \
            for (int k_ = 0; k_ < 16; ++k_) d_[k_] = (int)tacc[k_];                             \
        }                                                                                       \
    } while (0)
#else
#define TDECL \
    do {      \
    } while (0)
#define TIMED(k, stmt) \
    do {               \
        stmt;          \
    } while (0)
#define TCOUNT(k) \
    do {          \
    } while (0)
#define TDUMP(role) \
    do {            \
    } while (0)
#endif

struct Maps {
    CUtensorMap q, k, v, qg, kg, vg;
    CUtensorMap kc, vc;  // kAny: k / v rows of the global tokens by slot (qg then also by slot)
};

struct Tile {
    int present;         // has key blocks
    int r0;              // first query row
    int split;           // global: key split
    int glob_hi, lo, hi; // band: blocks [0, glob_hi) U [lo, hi]; global: [lo, hi]
};

struct Plan {
    int id;       // item id, -1 = no more items
    int global;
    int b, h, bh, rt;
    int g;        // leading global count (valid sample iff g <= w)
    Tile t[2];
    int nloads;
    int e1, lo_min;  // band pair: loads are [0, e1) then lo_min, lo_min + 1, ...
    int zero_only[2]; // band tile with no work but rows to zero (padded rows)
};

// Leading 0.0 entries of global_mask[b, :] capped at w + 1 (whole warp).
// 256 entries per round, all loads of a round in flight together.
__device__ int leading_globals(const Params& p, int b) {
    const int lane = threadIdx.x & 31;
    const float* row = p.global_mask + (size_t)b * p.L;
    const int cap = min(p.w + 1, p.L);
    for (int c0 = 0; c0 < cap; c0 += 256) {
        float v[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int j = c0 + 32 * t + lane;
            v[t] = j < cap ? row[j] : 0.0f;
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const unsigned m = __ballot_sync(0xffffffffu, v[t] != 0.0f);
            if (m) return c0 + 32 * t + __ffs(m) - 1;
        }
    }
    return cap;
}

// Global tokens of sample b: the leading 0.0 entries of global_mask
// (capped at w + 1), or with kAny the partition's count.
template <bool kAny>
__device__ __forceinline__ int sample_globals(const Params& p, int b) {
    if constexpr (kAny) return p.gnum[b];
    else return leading_globals(p, b);
}

// Whole warp: for each of the two band tiles starting at r0[x], does it have
// a row g <= i < L that is not padded (work), and padded rows in [g, L)?
// (kAny: any row i < L; rows of global tokens are left out of the output
// later.)  The local_mask loads of both tiles are issued before the global
// count is needed, so the first plan of a sample costs one round of loads.
template <bool kAny>
__device__ void band_rows2(const Params& p, int b, const int (&r0)[2], int& cached_b, int& g, int (&work)[2],
                           int (&padded)[2]) {
    const int lane = threadIdx.x & 31;
    const float* lm = p.local_mask + (size_t)b * p.L;
    float v[2][4];
#pragma unroll
    for (int x = 0; x < 2; ++x)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int i = r0[x] + lane + 32 * k;
            v[x][k] = i < p.L ? lm[i] : 1.0f;
        }
    if (b != cached_b) {
        g = sample_globals<kAny>(p, b);
        cached_b = b;
    }
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        bool w_ = false, pd = false;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int i = r0[x] + lane + 32 * k;
            if (i < p.L && (kAny || i >= g)) {
                const bool tok = v[x][k] == 1.0f;
                w_ |= tok;
                pd |= !tok;
            }
        }
        work[x] = __any_sync(0xffffffffu, w_);
        padded[x] = __any_sync(0xffffffffu, pd);
    }
}

// Whole warp: the item's plan (identical in every role).
template <bool kAny>
__device__ Plan make_plan(const Params& p, int id, int& cached_b, int& g) {
    Plan pl;
    pl.id = id;
    // Item order: the global pairs first (the longest items; the epilogue
    // warps merge their splits while the softmax warps already run band
    // work, so no merge is left at the end of the launch), then the interior
    // band pairs, then the band pairs at both ends of each sequence, which
    // are short and end the launch.
    const int inner_per = p.NTP > 2 ? p.NTP - 2 : 0;
    const int edge_per = p.NTP < 2 ? p.NTP : 2;
    if (id < p.n_glob) {
        const int id2 = id;
        pl.global = 1;
        const int sp = id2 % p.NSP;
        const int r = id2 / p.NSP;
        pl.rt = r % p.RT;
        pl.bh = r / p.RT;
        pl.t[0].split = 2 * sp;
        pl.t[1].split = 2 * sp + 1;
        pl.t[0].r0 = pl.t[1].r0 = pl.rt * kBM;  // set before any early return: every role reads it
    } else {
        int tp;
        if (id < p.n_glob + p.n_inner) {
            tp = 1 + (id - p.n_glob) % inner_per;
            pl.bh = (id - p.n_glob) / inner_per;
        } else {
            const int e = id - p.n_inner - p.n_glob;
            tp = (e % edge_per == 0) ? 0 : p.NTP - 1;
            pl.bh = e / edge_per;
        }
        pl.global = 0;
        pl.rt = 0;
        pl.t[0].r0 = 2 * tp * kBM;
        pl.t[1].r0 = (2 * tp + 1) * kBM;
        pl.t[0].split = pl.t[1].split = 0;
    }
    pl.b = pl.bh / p.H;
    pl.h = pl.bh % p.H;
    int work[2] = {0, 0}, padded[2] = {0, 0};
    if (pl.global) {
        if (pl.b != cached_b) {
            g = sample_globals<kAny>(p, pl.b);
            cached_b = pl.b;
        }
    } else {
        const int r0[2] = {pl.t[0].r0, pl.t[1].r0};
        band_rows2<kAny>(p, pl.b, r0, cached_b, g, work, padded);
    }
    pl.g = g;
    pl.nloads = 0;
    pl.e1 = 0;
    pl.lo_min = 0;
    pl.zero_only[0] = pl.zero_only[1] = 0;
    for (int x = 0; x < 2; ++x) {
        pl.t[x].present = 0;
        pl.t[x].glob_hi = pl.t[x].lo = 0;
        pl.t[x].hi = -1;
    }
    if (g > p.w) return pl;  // invalid sample: zero output only
    if (pl.global) {
        const int r0 = pl.rt * kBM;
        for (int x = 0; x < 2; ++x) {
            Tile& t = pl.t[x];
            t.r0 = r0;
            if (r0 < g && t.split < p.NS) {
                t.present = 1;
                t.lo = t.split * p.chunk;
                t.hi = min(p.NKB, t.lo + p.chunk) - 1;
            }
        }
        const int nA = pl.t[0].present ? pl.t[0].hi - pl.t[0].lo + 1 : 0;
        const int nB = pl.t[1].present ? pl.t[1].hi - pl.t[1].lo + 1 : 0;
        pl.nloads = nA + nB;
        return pl;
    }
    int G = 0, lo_min = 1 << 30, hi_max = -1;
    for (int x = 0; x < 2; ++x) {
        Tile& t = pl.t[x];
        t.split = 0;
        if (t.r0 >= p.L) continue;
        if (!work[x]) {
            pl.zero_only[x] = padded[x];
            continue;
        }
        t.present = 1;
        const int lo = t.r0 - p.w;
        t.lo = lo <= 0 ? 0 : lo / kBN;
        t.hi = min(p.NKB - 1, (t.r0 + kBM - 1 + p.w) / kBN);
        // Global key blocks: the blocks of positions [0, g) that the band
        // does not load anyway; kAny: the slot blocks of [0, g), all of them
        // (global tokens inside a row's window are masked in the slot block).
        t.glob_hi = kAny ? (g + kBN - 1) / kBN : min((g + kBN - 1) / kBN, t.lo);
        G = max(G, t.glob_hi);
        lo_min = min(lo_min, t.lo);
        hi_max = max(hi_max, t.hi);
    }
    if (hi_max < 0) return pl;
    pl.e1 = kAny ? G : min(G, lo_min);
    pl.lo_min = lo_min;
    pl.nloads = pl.e1 + (hi_max - lo_min + 1);
    return pl;
}

// Load q of an item: key block kb (a slot block of the compact maps when
// cmp is set) and which tiles use it.
template <bool kAny>
__device__ __forceinline__ void load_at(const Plan& pl, int q, int& kb, int& needA, int& needB, int& cmp) {
    cmp = 0;
    if (pl.global) {
        const int nA = pl.t[0].present ? pl.t[0].hi - pl.t[0].lo + 1 : 0;
        const int nB = pl.t[1].present ? pl.t[1].hi - pl.t[1].lo + 1 : 0;
        const int m = min(nA, nB);
        int x, idx;
        if (q < 2 * m) {
            x = q & 1;
            idx = q >> 1;
        } else {
            x = nA > nB ? 0 : 1;
            idx = m + (q - 2 * m);
        }
        kb = pl.t[x].lo + idx;
        needA = x == 0;
        needB = x == 1;
        return;
    }
    kb = q < pl.e1 ? q : pl.lo_min + (q - pl.e1);
    const Tile& A = pl.t[0];
    const Tile& Bt = pl.t[1];
    if (kAny && q < pl.e1) {  // slot block q
        cmp = 1;
        needA = A.present && q < A.glob_hi;
        needB = Bt.present && q < Bt.glob_hi;
        return;
    }
    needA = A.present && ((!kAny && kb < A.glob_hi) || (kb >= A.lo && kb <= A.hi));
    needB = Bt.present && ((!kAny && kb < Bt.glob_hi) || (kb >= Bt.lo && kb <= Bt.hi));
}

// Key blocks of one tile of an item.
__device__ __forceinline__ int tile_blocks(const Tile& t) { return t.present ? t.glob_hi + (t.hi - t.lo + 1) : 0; }
template <typename T>
struct Pack;
template <>
struct Pack<__half> {
    static constexpr uint32_t fmt = 0;
    __device__ static uint32_t two(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ static float2 unpack(uint32_t u) { return __half22float2(*reinterpret_cast<__half2*>(&u)); }
};
template <>
struct Pack<__nv_bfloat16> {
    static constexpr uint32_t fmt = 1;
    __device__ static uint32_t two(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ static float2 unpack(uint32_t u) { return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u)); }
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// Same as tmem_ld32 into float registers (bit patterns are kept).
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
__device__ __forceinline__ float fast_rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

enum : int { kSkip = 0, kFull = 1, kPart = 2 };

// Bits 0..n-1 set (n clamped to [0, 32]).
__device__ __forceinline__ uint32_t low_bits(int n) {
    n = min(max(n, 0), 32);
    return (uint32_t)((1ull << n) - 1ull);
}
// Bits lo..hi set (inclusive, clamped to [0, 31]; empty when lo > hi).
__device__ __forceinline__ uint32_t range_bits(int lo, int hi) {
    return low_bits(hi + 1) & ~low_bits(lo);
}

// kAny: global tokens at any position (slot-indexed global rows and global
// key blocks, see Params); otherwise the global tokens are positions 0..g-1.
template <typename T, bool kAny>
__global__ void __launch_bounds__(kThreads, 1)
attention_tc_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bars + 0;   // Q of the current item loaded (one phase per item)
    uint64_t* q_empty = bars + 1;  // ... and read by both tiles' last S products
    uint64_t* kv_full = bars + 2;
    uint64_t* kv_empty = kv_full + kStages;
    uint64_t* s_full = kv_empty + kStages;  // [tile]: S of the tile's next block computed
    uint64_t* s_free = s_full + 2;          // [tile]: its 4 softmax warps have read S
    uint64_t* p_full = s_free + 2;          // [tile]: ... and written P
    uint64_t* pv_done = p_full + 2;         // [tile]: one phase per P V product of the tile
    uint64_t* o_free = pv_done + 2;         // [tile]: the epilogue has read O
    uint64_t* st_full = o_free + 2;         // [tile]: row (m, l) of an item written
    uint64_t* st_free = st_full + 2;        // [tile]: ... and read by the epilogue
    uint64_t* item_full = st_free + 2;      // [kRing]
    uint64_t* item_empty = item_full + kRing;
    uint64_t* drain = item_empty + kRing;   // [tile]: wind-down of an MMA warp
    uint64_t* tma_done = drain + 2;         // the TMA warp finished issuing an item's loads
    static_assert(1 + 1 + 2 * kStages + 2 * 7 + 2 * kRing + 2 + 1 == kNumBars, "barriers");
    Plan* plans = reinterpret_cast<Plan*>(smem + kOffPlans);
    static_assert(sizeof(Plan) <= 128, "plan slot");
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // The next kernel in the stream may be scheduled now: its CTAs take the
    // SMs this grid's tail leaves idle and set themselves up there (a kernel
    // of this library launched after it waits for it before touching memory).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#if LF_TRACE
    if (threadIdx.x == 0 && p.trace) {  // kernel entry time
        volatile int* d_ = p.trace + gridDim.x * 16 * 4 + (blockIdx.x * 16 + 15) * 16;
        const unsigned long long t = globaltimer();
        d_[0] = (int)(t & 0xffffffffu);
        d_[1] = (int)(t >> 32);
    }
#endif

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 2);  // one commit per MMA warp
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_free[i], 4);
            mbar_init(&p_full[i], 4);
            mbar_init(&pv_done[i], 1);
            mbar_init(&o_free[i], 4);
            mbar_init(&st_full[i], 4);
            mbar_init(&st_free[i], 4);
            mbar_init(&drain[i], 1);
        }
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 2);  // one arrival per MMA warp
        }
        for (int s = 0; s < kRing; ++s) {
            mbar_init(&item_full[s], 1);
            mbar_init(&item_empty[s], kItemConsumers);
        }
        mbar_init(tma_done, 1);
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
        if (kAny) {
            prefetch_tensormap(&maps.kc);
            prefetch_tensormap(&maps.vc);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Launched as a programmatic dependent, this grid may have started while
    // the kernel before it still runs (and may still be writing this
    // kernel's inputs): no global memory is touched before it has completed,
    // except the masks when masks_early says the kernel before does not
    // write them (the planner then waits before its first atomic; the MMA
    // warps touch no global memory).
    {
        const bool early = p.masks_early != 0 && !kAny;
        const bool reads_masks_only = warp == 2 || (warp >= kSoftmaxWarp0 && warp < kEpiWarp0);
        const bool no_global = warp == 1 || warp == 3;
        if (!(early && (reads_masks_only || no_global))) asm volatile("griddepcontrol.wait;" ::: "memory");
    }
#if LF_TRACE
    if (threadIdx.x == 0 && p.trace) {
        volatile int* d_ = p.trace + gridDim.x * 16 * 4 + (blockIdx.x * 16 + 14) * 16;
        const unsigned long long t = globaltimer();
        d_[0] = (int)(t & 0xffffffffu);
        d_[1] = (int)(t >> 32);
    }
#endif

    // Every role but the planner reads the item plans in order, in place in
    // the shared-memory ring: the slot of item k - 1 is handed back when the
    // role asks for item k (so no role keeps a copy of a plan).
    auto next_plan = [&](uint32_t k) -> const Plan* {
        if (k > 0) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&item_empty[(k - 1) % kRing]);
        }
        const uint32_t slot = k % kRing;
        // every lane waits (and so acquires the planner's writes of the plan)
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&item_full[slot], (k / kRing) & 1, abort_flag));
        if (!ok) return nullptr;
        return &plans[slot];
    };

    if (warp < kSoftmaxWarp0) {
    regs_dec<kRegsProducer>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp runs the control flow; lane 0 issues the copies.
        TDECL;
        uint32_t kv_cnt = 0, item_cnt = 0;
        bool ok = true;
        auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
        };
        for (uint32_t k = 0; ok; ++k) {
            const Plan* plp = nullptr;
            TIMED(0, plp = next_plan(k));
            ok = plp != nullptr;
            if (!ok) break;
            const Plan& pl = *plp;
            if (pl.id < 0) break;
            if (pl.nloads == 0) {
                if (lane == 0) mbar_arrive(tma_done);
                continue;
            }
            if (lane == 0) TRACE(0, 12, pl.id, item_cnt, 0);
            // the previous item's last S products have read Q
            TIMED(1, ok = wait_all(q_empty, (item_cnt & 1) ^ 1));
            if (ok && lane == 0) {
                const int nq = pl.t[0].present + pl.t[1].present;
                mbar_arrive_expect_tx(q_full, nq * kTileBytes);
                for (int x = 0; x < 2; ++x)
                    if (pl.t[x].present)
                        tma_load_3d(smem + kOffQ + x * kTileBytes, pl.global ? &maps.qg : &maps.q, q_full, 0,
                                    pl.t[x].r0, pl.bh);
            }
            // Every load of the plan is issued (the MMA warp maps a tile's
            // blocks to ring stages by load index).
            for (int q = 0; q < pl.nloads && ok; ++q) {
                int kb, nA, nB, cmp;
                load_at<kAny>(pl, q, kb, nA, nB, cmp);
                const uint32_t st = kv_cnt % kStages;
                if (lane == 0) TRACE(0, 13, pl.id, q, kv_cnt);
                TIMED(2, ok = wait_all(&kv_empty[st], ((kv_cnt / kStages) & 1) ^ 1));
                if (!ok) break;
                if (lane == 0) {
                    const CUtensorMap* mk = pl.global ? &maps.kg : (cmp ? &maps.kc : &maps.k);
                    const CUtensorMap* mv = pl.global ? &maps.vg : (cmp ? &maps.vc : &maps.v);
                    mbar_arrive_expect_tx(&kv_full[st], 2 * kTileBytes);
                    tma_load_3d(smem + kOffK + st * kTileBytes, mk, &kv_full[st], 0, kb * kBN, pl.bh);
                    tma_load_3d(smem + kOffV + st * kTileBytes, mv, &kv_full[st], 0, kb * kBN, pl.bh);
                }
                ++kv_cnt;
            }
            if (ok && lane == 0) mbar_arrive(tma_done);
            __syncwarp();
            ++item_cnt;
        }
        if (lane == 0) TRACE(0, 19, ok ? 1 : 0, item_cnt, kv_cnt);
        if (lane == 0) TDUMP(0);
        if (lane == 0 && !ok) {  // wind-down: let issued copies land
            for (uint32_t c = (kv_cnt > kStages ? kv_cnt - kStages : 0); c < kv_cnt; ++c) {
                volatile int never = 0;
                mbar_wait(&kv_full[c % kStages], (c / kStages) & 1, &never, 200000000ull);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ planner
        // Takes items from the global counter, works out each item's plan
        // (reads of the masks included) once and publishes it through the
        // ring, running up to kRing items ahead of the other roles.
        int cached_b = -1, g = 0;
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            const uint32_t slot = k % kRing;
            int id = -1;
            // Take item k only once the TMA warp has issued every load of
            // item k-1: a CTA holds at most one item in reserve, taken a few
            // K/V stages before it is needed, so items are not hoarded by
            // early CTAs while others idle.  (The whole warp waits.)
            if (k > 0) ok = __all_sync(0xffffffffu, mbar_wait(tma_done, (k - 1) & 1, abort_flag));
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&item_empty[slot], ((k / kRing) & 1) ^ 1, abort_flag));
            if (!ok) break;
            if (lane == 0) {
                // The first item of CTA c is item c (no atomic on the critical
                // path of the start); later ones come from the counter, which
                // counts past the first gridDim.x items.
                if (k == 1 && p.masks_early && !kAny) asm volatile("griddepcontrol.wait;" ::: "memory");
                id = k == 0 ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(p.sched, 1);
                if (id >= p.n_items) id = -1;
            }
            id = __shfl_sync(0xffffffffu, id, 0);
            Plan pl;
            if (id >= 0) pl = make_plan<kAny>(p, id, cached_b, g);
            else pl.id = -1;
            if (lane == 0) {
                plans[slot] = pl;
                mbar_arrive(&item_full[slot]);
            }
            if (id < 0) break;
        }
    } else {
        // ------------------------------------------------------------ MMA issuers
        // Warp 1 issues the tensor-core work of tile A, warp 3 that of tile B.
        // Per block j of its tile: S_j = Q K_j^T into the tile's S columns as
        // soon as the softmax warps have read S_(j-1), then O += P_(j-1) V_(j-1)
        // once they have written P_(j-1).  So a tile's next S is computed while
        // its softmax still works on the current block, and neither tile
        // waits on the other.  Every K/V stage is released by both warps: by a
        // commit after its P V where the tile used it, else at once.
        const int x = warp == 1 ? 0 : 1;
        constexpr uint32_t idesc_qk = idesc_f16(Pack<T>::fmt, kBM, kBN, 0, 0);
        constexpr uint32_t idesc_pv = idesc_f16(Pack<T>::fmt, kBM, kHD, 0, 1);
        // Descriptors of the first Q / K / V tile; the others are reached by
        // adding (byte offset >> 4) to the start-address field.
        const uint64_t dq0 = desc_sw128(smem_u32(smem + kOffQ));
        const uint64_t dk0 = desc_sw128(smem_u32(smem + kOffK));
        const uint64_t dv0 = desc_sw128(smem_u32(smem + kOffV), 0);
        constexpr uint32_t kTileStep = kTileBytes >> 4;
        const uint32_t t_s = tmem + x * kTmemTile, t_p = t_s + kTmemP, t_o = t_s + kTmemO;
        TDECL;
        uint32_t kv_cnt = 0, item_cnt = 0;
        uint32_t s_use = 0;  // S products issued (s_free phases)
        uint32_t p_use = 0;  // P blocks consumed (p_full phases)
        uint32_t o_use = 0;  // items with blocks (o_free phases)
        // The whole warp runs the control flow together (a single lane running
        // it while the other 31 wait at a warp barrier made every step of it
        // take microseconds); only the tensor-core instructions, commits and
        // arrivals are issued by lane 0.
        auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
        };
        // O (+)= P V for the tile's block j read from stage st; the stage is
        // released when the product is done.
        auto issue_pv = [&](int j, uint32_t st) -> bool {
            bool w_ok;
            TIMED(3, w_ok = wait_all(&p_full[x], p_use & 1u));
            if (!w_ok) return false;
            ++p_use;
            TCOUNT(5);
            if (j == 0) {
                TIMED(4, w_ok = wait_all(&o_free[x], (o_use & 1u) ^ 1u));
                if (!w_ok) return false;
                ++o_use;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint64_t dv = dv0 + st * kTileStep;
#if LF_TRACE
                const long long tp0_ = clock64();
#endif
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk)
                    mma_f16_ts(t_o, t_p + kk * 8, dv + kk * (2048 >> 4), idesc_pv, (j == 0 && kk == 0) ? 0u : 1u);
                tc_commit(&pv_done[x]);
                tc_commit(&kv_empty[st]);
#if LF_TRACE
                tacc[8] += clock64() - tp0_;
#endif
            }
            __syncwarp();
            return true;
        };
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            const Plan* plp = nullptr;
            TIMED(0, plp = next_plan(k));
            ok = plp != nullptr;
            if (!ok) break;
            const Plan& pl = *plp;
            if (pl.id < 0) break;
            if (pl.nloads == 0) continue;

            const int nA = tile_blocks(pl.t[0]), nB = tile_blocks(pl.t[1]);
            const int nx = x ? nB : nA;
            const int glob = pl.global, e1 = pl.e1, lo_min = pl.lo_min;
            const int gh = pl.t[x].glob_hi, lo = pl.t[x].lo, hi = pl.t[x].hi;
            const int m = min(nA, nB);
            // load index of this tile's block j
            auto load_idx = [&](int j) -> int {
                if (glob) return j < m ? 2 * j + x : m + j;
                if (kAny) return j < gh ? j : e1 + (lo + (j - gh) - lo_min);  // slot blocks first
                const int kb = j < gh ? j : lo + (j - gh);
                return kb < e1 ? kb : e1 + (kb - lo_min);
            };
            // is load q one of this tile's blocks?
            auto mine = [&](int q) -> bool {
                if (nx == 0) return false;
                if (glob) return q < 2 * m ? (q & 1) == x : nx > m;
                if (kAny && q < e1) return q < gh;
                const int kb = q < e1 ? q : lo_min + (q - e1);
                return (!kAny && kb < gh) || (kb >= lo && kb <= hi);
            };
            int q_ready = -1;
            // wait for loads up to q; loads this tile does not use are released at once
            auto take_loads = [&](int q) -> bool {
                while (q_ready < q) {
                    ++q_ready;
                    const uint32_t c = kv_cnt + q_ready, st = c % kStages;
                    bool w_ok;
                    TIMED(2, w_ok = wait_all(&kv_full[st], (c / kStages) & 1));
                    if (!w_ok) return false;
                    if (!mine(q_ready) && lane == 0) mbar_arrive(&kv_empty[st]);
                }
                return true;
            };
            if (nx > 0) TIMED(1, ok = wait_all(q_full, item_cnt & 1));
            const uint64_t dqx = dq0 + x * kTileStep;
            uint32_t st_prev = 0;
            for (int j = 0; j < nx && ok; ++j) {
                const int q = load_idx(j);
                ok = take_loads(q);
                if (!ok) break;
                // the softmax warps have read the previous S
                TIMED(6, ok = wait_all(&s_free[x], (s_use & 1u) ^ 1u));
                if (!ok) break;
                ++s_use;
                tc_fence_after();
                const uint32_t st = (kv_cnt + q) % kStages;
                if (lane == 0) {
                    const uint64_t dk = dk0 + st * kTileStep;
#if LF_TRACE
                    const long long tq0_ = clock64();
#endif
#pragma unroll
                    for (int kk = 0; kk < kHD / 16; ++kk)
                        mma_f16_ss(t_s, dqx + kk * 2, dk + kk * 2, idesc_qk, kk > 0);
                    tc_commit(&s_full[x]);
                    if (j == nx - 1) tc_commit(q_empty);  // the item's last S: Q is free once it is done
#if LF_TRACE
                    tacc[7] += clock64() - tq0_;
#endif
                }
                __syncwarp();
                if (j > 0) ok = issue_pv(j - 1, st_prev);
                st_prev = st;
            }
            if (ok && nx > 0) ok = issue_pv(nx - 1, st_prev);
            if (ok) ok = take_loads(pl.nloads - 1);
            if (ok && lane == 0 && nx == 0) mbar_arrive(q_empty);
            __syncwarp();
            ++item_cnt;
            kv_cnt += pl.nloads;
        }
        if (lane == 0) TDUMP(1 + 2 * x);
        if (lane == 0 && !ok) {  // wind-down: wait for the MMAs already issued
            tc_commit(&drain[x]);
            volatile int never = 0;
            mbar_wait(&drain[x], 0, &never, 200000000ull);
        }
    }
    } else if (warp < kEpiWarp0) {
        regs_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax warps
        const int x = (warp - kSoftmaxWarp0) >> 2;  // tile handled by this warpgroup
        const int sp = warp & 3;           // TMEM sub-partition (rows sp*32 .. +31)
        const int r = sp * 32 + lane;      // query row within the tile
        const uint32_t lane_off = (uint32_t)(sp * 32) << 16;
        const uint32_t tS = tmem + lane_off + x * kTmemTile, tP = tS + kTmemP, tO = tS + kTmemO;
        float* bias_w = reinterpret_cast<float*>(smem + kOffBias) + (warp - kSoftmaxWarp0) * kBN;
        float2* stats = reinterpret_cast<float2*>(smem + kOffStats) + x * kBM;
        uint32_t npv = 0;     // this tile's blocks in earlier items (its P V products)
        uint32_t st_cnt = 0;  // items in which this tile had blocks
        TDECL;
        bool ok = true;
        for (uint32_t k = 0; ok; ++k) {
            const Plan* plp = nullptr;
            TIMED(0, plp = next_plan(k));
            ok = plp != nullptr;
            if (!ok) break;
            const Plan& pl = *plp;
            if (pl.id < 0) break;
            if (pl.nloads == 0) continue;
            const int nA = tile_blocks(pl.t[0]), nB = tile_blocks(pl.t[1]);
            const int nblk = x == 0 ? nA : nB;
            if (nblk == 0) continue;
            const int g = pl.g;
            const Tile& me = pl.t[x];
            const float* lm = p.local_mask + (size_t)pl.b * p.L;
            // kAny: local_mask of the slots (global rows, slot key blocks)
            const float* lmc = kAny ? p.lm_c + (size_t)pl.b * p.gcap : nullptr;
            const int i = me.r0 + r;
            // Only these few scalars stay live through the block loop.
            const int is_global = pl.global;
            const int blk_gh = me.glob_hi, blk_lo = me.lo;

            // Does this warp have rows whose output is kept?
            const int wr0 = me.r0 + sp * 32;
            bool row_kept;
            // kAny band rows: the slots [clo, chi) of the global tokens inside
            // the row's window, which the band blocks already hold
            int clo = 0, chi = 0;
            if (is_global) {
                row_kept = i < g && (kAny ? lmc[i] : lm[i]) == 1.0f;
            } else if (kAny) {
                row_kept = false;
                if (i < p.L) {
                    const int* rk = p.grank + (size_t)pl.b * (p.L + 1);
                    const float lmi = lm[i], gmi = p.global_mask[(size_t)pl.b * p.L + i];
                    clo = rk[max(0, i - p.w)];
                    chi = rk[min(p.L, i + p.w + 1)];
                    row_kept = lmi == 1.0f && gmi != 0.0f;
                }
            } else {
                row_kept = i < p.L && i >= g && lm[i] == 1.0f;
            }
            const bool warp_active = __any_sync(0xffffffffu, row_kept);

            float m_used = -INFINITY, l_run = 0.0f;
            // Which of the tile's key blocks hold padded keys (bit j for block
            // j < 32; later blocks are always treated as padded): worked out
            // once per item, eight blocks' loads in flight at a time, while
            // the first S of the item is still being computed.
            uint32_t padbits = 0;
            if (warp_active) {
                for (int j0 = 0; j0 < nblk && j0 < 32; j0 += 8) {
                    float v[8][4];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = j0 + u;
                        const int c2 = (j < blk_gh ? j : blk_lo + (j - blk_gh)) * kBN;
                        const bool cmp = kAny && !is_global && j < blk_gh;  // slot block
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const int key = c2 + t * 32 + lane;
                            if (kAny && cmp) v[u][t] = (j < nblk && key < g) ? lmc[key] : 1.0f;
                            else v[u][t] = (j < nblk && key < p.L) ? lm[key] : 1.0f;
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const bool pad = v[u][0] != 1.0f || v[u][1] != 1.0f || v[u][2] != 1.0f || v[u][3] != 1.0f;
                        if (__any_sync(0xffffffffu, pad)) padbits |= 1u << (j0 + u);
                    }
                }
            }
            for (int n = 0; n < nblk && ok; ++n) {
#if LF_TRACE
                const long long tpro_ = clock64();
#endif
                const bool first = n == 0;
                const int kb = n < blk_gh ? n : blk_lo + (n - blk_gh);
                const int c0 = kb * kBN;  // first key (kAny slot block: first slot)
                const bool cmp = kAny && !is_global && n < blk_gh;
                // Padding bias of the block's keys (keys >= L are masked instead).
                const bool has_pad = warp_active && (n >= 32 || ((padbits >> n) & 1u));
                if (has_pad) {
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int key = c0 + t * 32 + lane;
                        float mv;
                        if (kAny && cmp) mv = key < g ? lmc[key] : 1.0f;
                        else mv = key < p.L ? lm[key] : 1.0f;
                        bias_w[t * 32 + lane] = fmaf(mv, 10000.0f, -10000.0f) * p.inv_scale;
                    }
                    __syncwarp();
                }
                // Chunk states (warp-uniform): skip / full / masked, two bits
                // per chunk so that a rolled loop can index them.  They depend
                // only on where the block lies, so they are worked out before
                // the wait for its S, not after.
                uint32_t states = 0;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const int cj0 = c0 + ch * 32;
                    int s;
                    if (kAny && cmp) {
                        s = cj0 >= g ? kSkip : kPart;  // slots past g; window overlap per row
                    } else if (cj0 >= p.L) {
                        s = kSkip;
                    } else if (is_global) {
                        s = (cj0 + 31 < p.L) ? kFull : kPart;
                    } else {
                        const bool any_g = !kAny && cj0 < g;
                        const bool all_g = !kAny && cj0 + 31 < g;
                        const bool overlap = cj0 <= wr0 + 31 + p.w && cj0 + 31 >= wr0 - p.w;
                        const bool inside = (wr0 + 31 - cj0 <= p.w) && (cj0 + 31 - wr0 <= p.w);
                        if (!any_g && !overlap) s = kSkip;
                        else if ((all_g || inside) && cj0 + 31 < p.L) s = kFull;
                        else s = kPart;
                    }
                    states |= (uint32_t)s << (2 * ch);
                }
                if (lane == 0) TRACE(2 + warp - kSoftmaxWarp0, 32, pl.id, n, 0);
                // every lane waits; the result is made warp-uniform so that an
                // abort never splits the warp before a .sync.aligned instruction
#if LF_TRACE
                const long long tsw_ = clock64();
                tacc[10] += tsw_ - tpro_;
#endif
                TIMED(1, ok = __all_sync(0xffffffffu, mbar_wait(&s_full[x], (npv + n) & 1u, abort_flag)));
#if LF_TRACE
                const long long tb0_ = clock64();
                if (first) tacc[9] += tb0_ - tsw_;
#endif
                if (!ok) break;
                tc_fence_after();
                // P of the previous block is read by its P V product until
                // that completes: waited once, before this block's first P
                // write or O access.  (It also keeps every later wait on
                // pv_done within one phase of the barrier.)
                bool pv_ok = npv + n == 0;
                auto ensure_pv = [&]() {
                    if (!pv_ok) {
                        bool w_ok;
                        TIMED(3, w_ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[x], (npv + n - 1) & 1u, abort_flag)));
                        if (!w_ok) ok = false;
                        tc_fence_after();
                        pv_ok = true;
                    }
                };
                // S is handed back to the MMA warp once its last chunk this warp
                // reads has landed in registers (or at once when it reads none).
                int last_ld = -1;
                if (warp_active) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch)
                        if (((states >> (2 * ch)) & 3u) != kSkip) last_ld = ch;
                }
                auto release_s = [&]() {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s_free[x]);
                };
                if (last_ld < 0) release_s();
                if (warp_active) {
                    auto state_of = [&](int ch) -> int { return (int)((states >> (2 * ch)) & 3u); };
                    const int d0 = i - c0;
                    const int lo_c = d0 - p.w, hi_c = d0 + p.w, gl_c = g - c0, lim_c = p.L - c0;
                    auto chunk_bits = [&](int ch) -> uint32_t {
                        const int b0 = ch * 32;
                        if (kAny && cmp)  // slots < g outside the row's window
                            return low_bits(gl_c - b0) & ~range_bits(clo - c0 - b0, chi - 1 - c0 - b0);
                        uint32_t bits = low_bits(lim_c - b0);
                        if (!is_global) {
                            if (kAny) bits &= range_bits(lo_c - b0, hi_c - b0);
                            else bits &= low_bits(gl_c - b0) | range_bits(lo_c - b0, hi_c - b0);
                        }
                        return bits;
                    };
                    // bias and mask of chunk ch, applied to raw scores in r
                    auto fix_chunk = [&](int ch, float (&r)[32]) {
                        if (has_pad) {
                            const float4* b4p = reinterpret_cast<const float4*>(bias_w + ch * 32);
#pragma unroll
                            for (int c = 0; c < 32; c += 4) {
                                const float4 b4 = b4p[c / 4];
                                r[c] += b4.x;
                                r[c + 1] += b4.y;
                                r[c + 2] += b4.z;
                                r[c + 3] += b4.w;
                            }
                        }
                        if (state_of(ch) == kPart) {
                            const uint32_t bits = chunk_bits(ch);
#pragma unroll
                            for (int c = 0; c < 32; ++c) r[c] = ((bits >> c) & 1u) ? r[c] : -INFINITY;
                        }
                    };
                    // One pass over S in 32-column chunks (rolled loop, 32 live
                    // scores): each chunk is read once, biased and masked, and
                    // exponentiated against the running row max m.  m only
                    // moves when a row's max grows by more than 8 (log2 units,
                    // so P <= 2^8); the whole warp then rescales (tcgen05.ld/st
                    // are .sync.aligned): the sums so far, this block's P
                    // chunks already in TMEM and, past the item's first block,
                    // the O accumulator, once the previous block's P V is done.
                    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
                    float2 sm2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
                    // exponentials of one chunk, packed to 16 words of P
                    auto exp_chunk = [&](float (&r)[32], uint32_t (&pk)[16], float2 nm2) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const float2 a = ffma2(make_float2(r[2 * c], r[2 * c + 1]), sc2, nm2);
                            // about a third of the pairs on the FMA pipe, the rest on MUFU
                            const float2 e = (c % 3 == 2) ? exp2_poly2(a) : make_float2(ex2(a.x), ex2(a.y));
                            sm2[c & 1] = fadd2(sm2[c & 1], e);
                            pk[c] = Pack<T>::two(e.x, e.y);
                        }
                    };
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t pk[16];
                        if (state_of(ch) == kSkip) {
#pragma unroll
                            for (int c = 0; c < 16; ++c) pk[c] = 0u;
                        } else {
                            float r[32];
                            tmem_ld32f(tS + ch * 32, r);
                            tmem_ld_wait();
                            regs_ready<32>(r);
                            if (ch == last_ld) release_s();
                            fix_chunk(ch, r);
                            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                            for (int c = 0; c < 32; c += 8) {
                                mx[0] = max3(mx[0], r[c], r[c + 1]);
                                mx[1] = max3(mx[1], r[c + 2], r[c + 3]);
                                mx[2] = max3(mx[2], r[c + 4], r[c + 5]);
                                mx[3] = max3(mx[3], r[c + 6], r[c + 7]);
                            }
                            const float cm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
                            const bool need = cm > m_used + kRescaleThreshold;
                            if (__any_sync(0xffffffffu, need)) {
                                // rows with a finite previous max rescale what they
                                // have so far; rows at -inf have nothing yet (zeros)
                                const bool real = need && m_used != -INFINITY;
                                if (__any_sync(0xffffffffu, real)) {
                                    const float factor = real ? ex2(m_used - cm) : 1.0f;
                                    l_run *= factor;
                                    sm2[0] = make_float2(sm2[0].x * factor, sm2[0].y * factor);
                                    sm2[1] = make_float2(sm2[1].x * factor, sm2[1].y * factor);
                                    for (int pc = 0; pc < ch; ++pc) {  // this block's earlier P
                                        uint32_t pb16[16];
                                        tmem_ld16(tP + pc * 16, pb16);
                                        tmem_ld_wait();
                                        regs_ready<16>(pb16);
#pragma unroll
                                        for (int c = 0; c < 16; ++c) {
                                            const float2 v = Pack<T>::unpack(pb16[c]);
                                            pb16[c] = Pack<T>::two(v.x * factor, v.y * factor);
                                        }
                                        tmem_st16(tP + pc * 16, pb16);
                                    }
                                    if (!first) {
                                        // O holds the tile's blocks so far once the
                                        // previous block's P V has completed
                                        ensure_pv();
                                        TCOUNT(8);
#pragma unroll
                                        for (int c0o = 0; c0o < kHD && ok; c0o += 16) {
                                            uint32_t ob[16];
                                            tmem_ld16(tO + c0o, ob);
                                            tmem_ld_wait();
                                            regs_ready<16>(ob);
#pragma unroll
                                            for (int c = 0; c < 16; ++c)
                                                ob[c] = __float_as_uint(__uint_as_float(ob[c]) * factor);
                                            tmem_st16(tO + c0o, ob);
                                        }
                                    }
                                }
                                if (need) m_used = cm;
                            }
                            const float m_use = m_used == -INFINITY ? 0.0f : m_used;
                            exp_chunk(r, pk, make_float2(-m_use, -m_use));
                        }
                        ensure_pv();
                        tmem_st16(tP + ch * 16, pk);
                    }
                    l_run += (sm2[0].x + sm2[0].y) + (sm2[1].x + sm2[1].y);
                    tmem_st_wait();
                }
#if LF_TRACE
                tacc[2] += clock64() - tb0_;
                TCOUNT(5);
#endif
                ensure_pv();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[x]);
            }
            if (!ok) break;
            // Row (m, l) to the epilogue warps.
            TIMED(4, ok = __all_sync(0xffffffffu, mbar_wait(&st_free[x], (st_cnt & 1) ^ 1, abort_flag)));
            TCOUNT(6);
            if (!ok) break;
            stats[r] = make_float2(m_used, l_run);
            __syncwarp();
            if (lane == 0) mbar_arrive(&st_full[x]);
            ++st_cnt;
            npv += nblk;
        }
        if (lane == 0) TDUMP(2 + warp - kSoftmaxWarp0);
    } else {
        regs_dec<kRegsEpi>();
        // ------------------------------------------------------------ epilogue warps
        // Per item and tile: wait for the tile's last P V, read O and the row
        // (m, l), hand O back, then write the rows (band tiles), or the
        // split-KV partials and, for the last split of a row group, the
        // merged rows (global tiles).  Also zeroes padded rows of tiles
        // without key blocks and rows of samples that break the constraints.
        const int sp = warp & 3;
        const int r = sp * 32 + lane;
        const uint32_t lane_off = (uint32_t)(sp * 32) << 16;
        const float2* stats = reinterpret_cast<const float2*>(smem + kOffStats);
        uint32_t npv[2] = {0, 0}, st_cnt[2] = {0, 0};
        TDECL;
        bool ok = true;
        if constexpr (!kAny) {
            // the partition, while this CTA's first scores are computed
            if (p.gidx_out) {
                int* sm_i = reinterpret_cast<int*>(smem + kOffMisc + 16);
                for (int b = blockIdx.x; b < p.B; b += gridDim.x)
                    partition_sample(p.global_mask + (size_t)b * p.L, p.L, p.w, p.gidx_out + (size_t)b * p.L,
                                     p.gnum_out + b, b, p.status, r, sp, lane, sm_i);
            }
        }
#if LF_TRACE
        const unsigned long long tent_ = globaltimer();
#endif
        for (uint32_t k = 0; ok; ++k) {
            const Plan* plp = nullptr;
            TIMED(0, plp = next_plan(k));
            ok = plp != nullptr;
            if (!ok) break;
            const Plan& pl = *plp;
            if (pl.id < 0) break;
#if LF_TRACE
            if (k < 3) tacc[11 + k] = (long long)(globaltimer() - tent_);
#endif
            const int g = pl.g;
            const float* lm = p.local_mask + (size_t)pl.b * p.L;
            for (int x = 0; x < 2 && ok; ++x) {
                const Tile& me = pl.t[x];
                const int i = me.r0 + r;
#if LF_TRACE
                const long long te0_ = clock64();
#endif
                // This row's mask values, loaded before any wait so that
                // their latency is hidden; a global_mask 0.0 past the prefix
                // is recorded at the end of the tile.
                const bool in_row = me.r0 < p.L && i < p.L;
                // kAny global tiles hold slots: their local_mask values and
                // the positions their rows are written to
                float lmi;
                int pos = i;
                if (kAny && pl.global) {
                    lmi = i < p.gcap ? p.lm_c[(size_t)pl.b * p.gcap + i] : 0.0f;
                    if (i < g && g <= p.w) pos = p.gidx[(size_t)pl.b * p.L + i];
                } else {
                    lmi = in_row ? lm[i] : 1.0f;
                }
                const float gmi = (in_row && !pl.global) ? p.global_mask[(size_t)pl.b * p.L + i] : 1.0f;
                // band rows whose output this tile writes (not global tokens)
                const bool local_row = kAny ? gmi != 0.0f : i >= g;
                const bool not_prefix = !kAny && !pl.global && g <= p.w && in_row && i >= g;
                if (!pl.global) {
                    if (g > p.w) {  // invalid sample: zero output, record once
                        if (in_row) store_zero_row(p.out, ((size_t)(pl.b * p.L + i) * p.H + pl.h) * kHD, sizeof(T));
                        if (x == 0 && r == 0 && me.r0 == 0 && pl.h == 0) record_status(p.status, pl.b, LF_ERR_G_GT_W);
                        continue;
                    }
                    if (pl.zero_only[x]) {
                        if (in_row && local_row && lmi != 1.0f)
                            store_zero_row(p.out, ((size_t)(pl.b * p.L + i) * p.H + pl.h) * kHD, sizeof(T));
                        if (not_prefix && gmi == 0.0f) record_status(p.status, pl.b, LF_ERR_GLOBAL_NOT_PREFIX);
                        continue;
                    }
                }
                const int nblk = tile_blocks(me);
#if LF_TRACE
                tacc[7] += clock64() - te0_;
#endif
                if (nblk == 0) {
                    if (not_prefix && gmi == 0.0f) record_status(p.status, pl.b, LF_ERR_GLOBAL_NOT_PREFIX);
                    continue;
                }
                // (m, l) first: they are written after the tile's last block,
                // whose P V is then at most one phase ahead of this wait.
                if (lane == 0) TRACE(10 + sp, 40 + x, pl.id, st_cnt[x], npv[x]);
                TIMED(1, ok = __all_sync(0xffffffffu, mbar_wait(&st_full[x], st_cnt[x] & 1, abort_flag)));
                if (!ok) break;
                const float2 ml = stats[x * kBM + r];
                TIMED(2, ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[x], (npv[x] + nblk - 1) & 1u, abort_flag)));
                if (!ok) break;
                tc_fence_after();
                // O of this tile's rows, read once; P V is complete.
#if LF_TRACE
                const long long te1_ = clock64();
#endif
                float o[kHD];
                {
                    const uint32_t tO = tmem + lane_off + x * kTmemTile + kTmemO;
                    tmem_ld32f(tO, *reinterpret_cast<float(*)[32]>(&o[0]));
                    tmem_ld32f(tO + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
                    tmem_ld_wait();
                    regs_ready<kHD>(o);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&o_free[x]);
                    mbar_arrive(&st_free[x]);
                }
                ++st_cnt[x];
                npv[x] += nblk;
#if LF_TRACE
                const long long te2_ = clock64();
                tacc[3] += te2_ - te1_;
#endif

                if (!pl.global) {
                    if (in_row && local_row) {
                        const size_t off = ((size_t)(pl.b * p.L + i) * p.H + pl.h) * kHD;
                        if (lmi != 1.0f) store_zero_row(p.out, off, sizeof(T));
                        else store_row<T>(p.out, off, o, fast_rcp(ml.y));
                    }
                    if (not_prefix && gmi == 0.0f) record_status(p.status, pl.b, LF_ERR_GLOBAL_NOT_PREFIX);
#if LF_TRACE
                    tacc[4] += clock64() - te2_;
                    TCOUNT(8);
#endif
                } else if (me.r0 + sp * 32 < g) {
                    // Split-KV partials of this warp's 32 rows; the warp that
                    // completes the last split of its row group merges them.
                    const int slot0 = (pl.bh * p.RT + pl.rt) * p.NS;
                    const int sl = slot0 + me.split;
                    if (i < g) {
                        float4* po = reinterpret_cast<float4*>(p.part_o + ((size_t)sl * kBM + r) * kHD);
#pragma unroll
                        for (int c = 0; c < kHD / 4; ++c)
                            __stcg(po + c, make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]));
                        __stcg(reinterpret_cast<float2*>(p.part_ml + ((size_t)sl * kBM + r) * 2), ml);
                    }
                    __threadfence();
                    __syncwarp();
                    int* counter = p.counters + (pl.bh * p.RT + pl.rt) * 4 + sp;
                    int last = 0;
                    if (lane == 0) last = (atomicAdd(counter, 1) == p.NS - 1) ? 1 : 0;
                    last = __shfl_sync(0xffffffffu, last, 0);
#if LF_TRACE
                    const long long te3_ = clock64();
                    tacc[5] += te3_ - te2_;
                    TCOUNT(9);
#endif
                    if (last) {
                        __threadfence();
                        if (i < g) {
                            const size_t off = ((size_t)(pl.b * p.L + pos) * p.H + pl.h) * kHD;
                            if (lmi != 1.0f) {
                                store_zero_row(p.out, off, sizeof(T));
                            } else {
                                // Merge by log-sum-exp, with the loads of a
                                // round in flight together: the (m, l) of up
                                // to 16 splits, then per column half each
                                // split's 32 values with its (m, l).
                                const float2* pml = reinterpret_cast<const float2*>(p.part_ml) + (size_t)slot0 * kBM + r;
                                float M = -INFINITY;
                                for (int s0 = 0; s0 < p.NS; s0 += 16) {
                                    float mx[16];
#pragma unroll
                                    for (int u = 0; u < 16; ++u)
                                        mx[u] = s0 + u < p.NS ? __ldcg(pml + (size_t)(s0 + u) * kBM).x : -INFINITY;
#pragma unroll
                                    for (int u = 0; u < 16; ++u) M = fmaxf(M, mx[u]);
                                }
                                float lsum = 0.0f;
                                for (int h = 0; h < 2; ++h) {
                                    float acc[32];
#pragma unroll
                                    for (int c = 0; c < 32; ++c) acc[c] = 0.0f;
                                    for (int s1 = 0; s1 < p.NS; ++s1) {
                                        const float4* po = reinterpret_cast<const float4*>(
                                            p.part_o + ((size_t)(slot0 + s1) * kBM + r) * kHD + 32 * h);
                                        float4 t4[8];
#pragma unroll
                                        for (int c = 0; c < 8; ++c) t4[c] = __ldcg(po + c);
                                        const float2 m2 = __ldcg(pml + (size_t)s1 * kBM);
                                        const float wgt = m2.x == -INFINITY ? 0.0f : ex2(m2.x - M);
                                        if (h == 0) lsum = fmaf(m2.y, wgt, lsum);
#pragma unroll
                                        for (int c = 0; c < 8; ++c) {
                                            acc[4 * c] = fmaf(t4[c].x, wgt, acc[4 * c]);
                                            acc[4 * c + 1] = fmaf(t4[c].y, wgt, acc[4 * c + 1]);
                                            acc[4 * c + 2] = fmaf(t4[c].z, wgt, acc[4 * c + 2]);
                                            acc[4 * c + 3] = fmaf(t4[c].w, wgt, acc[4 * c + 3]);
                                        }
                                    }
                                    // lsum is complete after the first half
                                    const float inv = fast_rcp(lsum);
                                    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.out) + off + 32 * h);
#pragma unroll
                                    for (int c = 0; c < 4; ++c) {
                                        uint4 u4;
                                        u4.x = Pack<T>::two(acc[8 * c + 0] * inv, acc[8 * c + 1] * inv);
                                        u4.y = Pack<T>::two(acc[8 * c + 2] * inv, acc[8 * c + 3] * inv);
                                        u4.z = Pack<T>::two(acc[8 * c + 4] * inv, acc[8 * c + 5] * inv);
                                        u4.w = Pack<T>::two(acc[8 * c + 6] * inv, acc[8 * c + 7] * inv);
                                        dst[c] = u4;
                                    }
                                }
                            }
                        }
                        if (lane == 0) *counter = 0;
#if LF_TRACE
                        tacc[6] += clock64() - te3_;
                        TCOUNT(10);
#endif
                    }
                }
            }
        }
#if LF_TRACE
        tacc[14] = (long long)(globaltimer() - tent_);
#endif
        if (lane == 0) TDUMP(10 + sp);
    }

#if LF_TRACE
    if (threadIdx.x == 0 && p.trace) {  // CTA start/end time
        volatile int* d_ = p.trace + gridDim.x * 16 * 4 + (blockIdx.x * 16 + 14) * 16;
        const unsigned long long t = globaltimer();
        d_[2] = (int)(t & 0xffffffffu);
        d_[3] = (int)(t >> 32);
    }
#endif
    __syncthreads();
    volatile int* last_cta = abort_flag + 1;
    if (threadIdx.x == 0) {
        if (*abort_flag) record_status(p.status, 0, LF_ERR_DEVICE_TIMEOUT);
        __threadfence();
        *last_cta = atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (*last_cta) {
        // The last CTA to finish resets the scheduler and the split counters
        // for the next launch (the counters are already zero unless a
        // launch was aborted part-way).
        __threadfence();
        const int n_counters = p.B * p.H * p.RT * 4;
        for (int c = threadIdx.x; c < n_counters; c += kThreads) p.counters[c] = 0;
        if (threadIdx.x == 0) {
            p.sched[0] = 0;
            p.sched[1] = 0;
        }
        __threadfence();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
#if LF_TRACE
    if (threadIdx.x == 32 && p.trace) {  // exit time (after the TMEM release)
        volatile int* d_ = p.trace + gridDim.x * 16 * 4 + (blockIdx.x * 16 + 15) * 16;
        const unsigned long long t = globaltimer();
        d_[2] = (int)(t & 0xffffffffu);
        d_[3] = (int)(t >> 32);
    }
#endif
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

// Global-row split size.  Items are taken from a counter by the CTAs as they
// free up, so the kernel ends when the last CTA finishes its last item; with
// only a few items per CTA the split size decides how evenly the work packs.
// The host replays that list schedule (global pairs, inner band pairs, edge
// pairs) for each candidate size with a cost model of the kernel and keeps
// the size with the earliest finish.  Relative costs, fitted to split-size
// sweeps of the kernel on B200 (workloads of 4096 and 16384 tokens): a key
// block 60 (band or global: a global block has no skipped chunks, but only
// the warps holding rows i < g work on it), an item 25 (its first S and the
// epilogue), a split merge 15.  Leading globals are taken as g <= 128 (one
// global row tile with work, one block of global keys per band tile); the
// choice only affects speed.
int choose_chunk(int B, int H, int L, int w, int sm_count) {
    const int NKB = (L + kBN - 1) / kBN;
    const int NT = (L + kBM - 1) / kBM;
    const int NTP = (NT + 1) / 2;
    const int RT = (w + kBM - 1) / kBM;
    const int BH = B * H;
    const int lo_c = kMinChunk < NKB ? kMinChunk : NKB;
    const int hi_c = kMaxChunk < NKB ? kMaxChunk : NKB;
    const long long n_band = (long long)BH * NTP;
    if (sm_count <= 0 || n_band * (hi_c - lo_c + 1) > 4000000LL) return lo_c;
    struct Key {
        int B, H, L, w, sm, chunk;
    };
    static std::mutex mu;
    static Key cache[16];
    static int n_cache = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < n_cache; ++i)
            if (cache[i].B == B && cache[i].H == H && cache[i].L == L && cache[i].w == w && cache[i].sm == sm_count)
                return cache[i].chunk;
    }
    constexpr long long kBlock = 60, kGlobBlock = 60, kItem = 25, kMerge = 15, kEmpty = 2;
    auto band_blocks = [&](int r0) -> int {
        if (r0 >= L) return 0;
        const int lo = (r0 - w <= 0 ? 0 : r0 - w) / kBN;
        const int hi = (r0 + kBM - 1 + w) / kBN < NKB - 1 ? (r0 + kBM - 1 + w) / kBN : NKB - 1;
        return (lo > 0 ? 1 : 0) + hi - lo + 1;
    };
    auto pair_cost = [&](int tp) -> long long {
        const int a = band_blocks(2 * tp * kBM), b = band_blocks((2 * tp + 1) * kBM);
        return (a > b ? a : b) * kBlock + kItem;
    };
    std::vector<long long> costs;
    std::vector<long long> heap;
    long long best = -1;
    int best_c = lo_c;
    for (int c = lo_c; c <= hi_c; ++c) {
        const int NS = (NKB + c - 1) / c, NSP = (NS + 1) / 2;
        costs.clear();
        for (int bh = 0; bh < BH; ++bh)
            for (int rt = 0; rt < RT; ++rt)
                for (int sp = 0; sp < NSP; ++sp) {
                    if (rt > 0) {
                        costs.push_back(kEmpty);
                        continue;
                    }
                    int m = 0;
                    for (int s = 2 * sp; s < 2 * sp + 2 && s < NS; ++s) {
                        const int n = (NKB < s * c + c ? NKB : s * c + c) - s * c;
                        m = n > m ? n : m;
                    }
                    costs.push_back(m * kGlobBlock + kItem + kMerge);
                }
        for (int bh = 0; bh < BH; ++bh)
            for (int tp = 1; tp + 1 < NTP; ++tp) costs.push_back(pair_cost(tp));
        for (int bh = 0; bh < BH; ++bh) {
            costs.push_back(pair_cost(0));
            if (NTP > 1) costs.push_back(pair_cost(NTP - 1));
        }
        heap.assign(sm_count, 0);  // min-heap of CTA finish times
        for (long long cst : costs) {
            std::pop_heap(heap.begin(), heap.end(), std::greater<long long>());
            heap.back() += cst;
            std::push_heap(heap.begin(), heap.end(), std::greater<long long>());
        }
        const long long span = *std::max_element(heap.begin(), heap.end());
        if (best < 0 || span < best) {
            best = span;
            best_c = c;
        }
    }
    {
        std::lock_guard<std::mutex> lock(mu);
        if (n_cache < 16) cache[n_cache++] = Key{B, H, L, w, sm_count, best_c};
    }
    return best_c;
}

int current_sm_count() {
    static int sms[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        sms[dev] = n;
    }
    return sms[dev];
}

template <typename T, bool kAny>
lf_status launch_instance(int grid, const Maps& maps, const Params& p, cudaStream_t stream) {
    // The shared-memory opt-in is a per-device function attribute: set once
    // per device and instance, with the device current.
    static std::atomic<bool> attr[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LF_ERR_CUDA;
    if (!attr[dev].load()) {
        if (cudaFuncSetAttribute(attention_tc_kernel<T, kAny>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes) != cudaSuccess)
            return LF_ERR_CUDA;
        attr[dev].store(true);
    }
    // The prefix instance reads nothing that the kernel before it may still
    // be writing when that kernel is this library's partition kernel (the
    // only kernel here that lets a dependent start early), so it is launched
    // with programmatic stream serialization and overlaps it.  Any other
    // preceding work completes first, as usual.
    cudaLaunchAttribute attr_pdl[1];
    attr_pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr_pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr_pdl;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, attention_tc_kernel<T, kAny>, maps, p) != cudaSuccess) return LF_ERR_CUDA;
    return LF_OK;
}

struct Geometry {
    int NKB, NT, RT, NS, NSP, NTP, chunk;
    size_t sched_bytes, counters_bytes, part_o_bytes, part_ml_bytes;
};

Geometry geometry(int B, int H, int L, int w, int sm_count) {
    Geometry g;
    g.NKB = (L + kBN - 1) / kBN;
    g.NT = (L + kBM - 1) / kBM;
    g.RT = (w + kBM - 1) / kBM;
    g.chunk = choose_chunk(B, H, L, w, sm_count);
    g.NS = (g.NKB + g.chunk - 1) / g.chunk;
    g.NSP = (g.NS + 1) / 2;
    g.NTP = (g.NT + 1) / 2;
    const size_t slots = (size_t)B * H * g.RT * g.NS;
    g.sched_bytes = 256;
    g.counters_bytes = (((size_t)B * H * g.RT * 4 * sizeof(int)) + 255) & ~size_t(255);
    g.part_o_bytes = slots * kBM * kHD * sizeof(float);
    g.part_ml_bytes = slots * kBM * 2 * sizeof(float);
    return g;
}

}  // namespace

size_t attention_tc_scratch_bytes(int B, int H, int L, int w) {
    const Geometry g = geometry(B, H, L, w, current_sm_count());
    return g.sched_bytes + g.counters_bytes + g.part_o_bytes + g.part_ml_bytes;
}

size_t attention_tc_scratch_zero_bytes(int B, int H, int L, int w) {
    const Geometry g = geometry(B, H, L, w, current_sm_count());
    return g.sched_bytes + g.counters_bytes;
}

lf_status launch_attention_tc(const void* q, const void* k, const void* v, const void* qg, const void* kg,
                              const void* vg, const float* local_mask, const float* global_mask, int B, int H,
                              int L, int w, float scale, lf_dtype dtype, void* out, void* scratch, int* status,
                              int sm_count, cudaStream_t stream, const AnyGlobals* any, int32_t* gidx_out,
                              int32_t* gnum_out, bool masks_early) {
    const Geometry geo = geometry(B, H, L, w, sm_count);
    Maps maps;
    const int BH = B * H;
    if (!make_map(&maps.q, q, BH, L) || !make_map(&maps.k, k, BH, L) || !make_map(&maps.v, v, BH, L) ||
        !make_map(&maps.kg, kg, BH, L) || !make_map(&maps.vg, vg, BH, L))
        return LF_ERR_CUDA;
    if (any) {  // global rows and global key blocks by slot
        if (!make_map(&maps.qg, any->qg_c, BH, any->gcap) || !make_map(&maps.kc, any->k_c, BH, any->gcap) ||
            !make_map(&maps.vc, any->v_c, BH, any->gcap))
            return LF_ERR_CUDA;
    } else {
        if (!make_map(&maps.qg, qg, BH, L)) return LF_ERR_CUDA;
        maps.kc = maps.k;
        maps.vc = maps.v;
    }
    Params p;
    p.B = B;
    p.H = H;
    p.L = L;
    p.w = w;
    p.NKB = geo.NKB;
    p.NT = geo.NT;
    p.RT = geo.RT;
    p.NS = geo.NS;
    p.NSP = geo.NSP;
    p.NTP = geo.NTP;
    p.chunk = geo.chunk;
    p.n_inner = BH * (geo.NTP > 2 ? geo.NTP - 2 : 0);
    p.n_glob = BH * geo.RT * geo.NSP;
    p.n_items = p.n_glob + BH * geo.NTP;
    p.scale_log2 = scale * kLog2e;
    p.inv_scale = 1.0f / scale;
    p.local_mask = local_mask;
    p.global_mask = global_mask;
    p.out = out;
    uint8_t* s = reinterpret_cast<uint8_t*>(scratch);
    p.sched = reinterpret_cast<int*>(s);
    p.counters = reinterpret_cast<int*>(s + geo.sched_bytes);
    p.part_o = reinterpret_cast<float*>(s + geo.sched_bytes + geo.counters_bytes);
    p.part_ml = reinterpret_cast<float*>(s + geo.sched_bytes + geo.counters_bytes + geo.part_o_bytes);
    p.status = status;
    p.trace = nullptr;
    p.gnum = any ? any->global_token_nums : nullptr;
    p.gidx = any ? any->global_idx : nullptr;
    p.grank = any ? any->rank : nullptr;
    p.lm_c = any ? any->lm_c : nullptr;
    p.gcap = any ? any->gcap : 0;
    p.gidx_out = any ? nullptr : gidx_out;
    p.gnum_out = any ? nullptr : gnum_out;
    p.masks_early = masks_early ? 1 : 0;
#if LF_TRACE
    if (const char* a = getenv("LF_TRACE_ADDR")) p.trace = reinterpret_cast<int*>(strtoull(a, nullptr, 10));
#endif

    const int grid = p.n_items < sm_count ? p.n_items : sm_count;
    lf_status st;
    if (dtype == LF_F16) st = any ? launch_instance<__half, true>(grid, maps, p, stream)
                                  : launch_instance<__half, false>(grid, maps, p, stream);
    else st = any ? launch_instance<__nv_bfloat16, true>(grid, maps, p, stream)
                  : launch_instance<__nv_bfloat16, false>(grid, maps, p, stream);
    if (st != LF_OK) return st;
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

}  // namespace lf
