// Internal declarations shared by the liblf.so translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "lf.h"

namespace lf {

// Device status word: holds LF_STATUS_CLEAR or (sample << 8) | code, and is
// only ever lowered with atomicMin, so the word keeps the error of the
// lowest-numbered failing sample (lowest code within a sample).
constexpr int LF_STATUS_CLEAR = 0x7fffffff;

__device__ __forceinline__ void record_status(int* word, int sample, int code) {
    atomicMin(word, (sample << 8) | code);
}

struct DeviceCtx {
    bool init = false;
    int ordinal = -1;
    int sm_count = 0;
    int cc_major = 0, cc_minor = 0;
    int* status = nullptr;  // device word, see LF_STATUS_CLEAR
    void* scratch = nullptr;
    size_t scratch_bytes = 0;
    // Leading bytes of the scratch known to be zero when the next call
    // starts (the attention kernel's scheduler and split counters must be).
    size_t scratch_clean = 0;
};

// Current device's context (initialised on first use; NULL + status on error).
DeviceCtx* current_device(lf_status* st);
// Make sure the current device's library scratch holds `bytes` (grows by
// cudaMalloc; the new region is zeroed).
lf_status ensure_scratch(DeviceCtx* dev, size_t bytes);
// Before an attention launch on the library scratch: clears its first
// `zero_bytes` on `stream` unless they are known to be zero already, and
// records that after the launch only they are (the kernel re-zeroes its
// counters; what follows them is written).
lf_status prepare_scratch_counters(DeviceCtx* dev, size_t zero_bytes, cudaStream_t stream);
// Records that a call wrote the scratch from its start (nothing is known
// to be zero any more).
void scratch_dirty(DeviceCtx* dev);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch as a programmatic dependent of the work before it on the stream:
// the kernel must wait (griddepcontrol.wait) before touching memory.
template <typename... KArgs, typename... Args>
lf_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     Args... args) {
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) return LF_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

lf_status check_shape(int B, int H, int L, int w);

// ---- launchers (return LF_OK or LF_ERR_CUDA) ----
// rank (may be NULL): [B][L + 1] global tokens before each position.
// require_prefix: record LF_ERR_GLOBAL_NOT_PREFIX for global tokens that are
// not positions 0..g-1.
lf_status launch_global_idx(const float* global_mask, int B, int L, int w, int32_t* global_idx,
                            int32_t* global_token_nums, int* status, cudaStream_t stream,
                            int32_t* rank = nullptr, bool require_prefix = true);

// Global tokens at any position: the partition's outputs and the rows of
// the global tokens gathered from them into compact per-head buffers (slot
// c = the c-th global token of the sample, slots g..gcap-1 zero).
struct AnyGlobals {
    const int32_t* global_idx;         // [B][L]
    const int32_t* global_token_nums;  // [B]
    const int32_t* rank;               // [B][L + 1]
    void* qg_c;                        // [B*H][gcap][64] dtype
    void* k_c;                         // [B*H][gcap][64] dtype
    void* v_c;                         // [B*H][gcap][64] dtype
    float* lm_c;                       // [B][gcap]: local_mask of each slot (0 past g)
    int gcap;                          // w rounded up to a multiple of 128
};
inline int any_globals_gcap(int w) { return (w + 127) / 128 * 128; }
// Bytes of the partition outputs and compact buffers (each part 256-aligned).
size_t any_globals_bytes(int B, int H, int L, int w, bool compact);
// Carves an AnyGlobals out of `base` (any_globals_bytes(..) bytes).
AnyGlobals any_globals_layout(void* base, int B, int H, int L, int w, bool compact);
// 16-bit dtypes: fills qg_c, k_c, v_c and lm_c from the partition's outputs
// (qg NULL: qg_c is not written).
lf_status launch_gather_globals(const void* qg, const void* k, const void* v, const float* local_mask,
                                const AnyGlobals& a, int B, int H, int L, int w, cudaStream_t stream);
// The partition (with the rank table, no prefix check) and the gather of
// qg, k, v and local_mask in one launch of B*H CTAs (16-bit dtypes).
lf_status launch_partition_gather(const float* global_mask, const float* local_mask, const void* qg, const void* k,
                                  const void* v, const AnyGlobals& a, int B, int H, int L, int w, int* status,
                                  cudaStream_t stream);
// Rows of a [B][L][D] 16-bit matrix at the global tokens' positions into
// [B][gcap][D] (slots past g zero).  D % 8 == 0.
lf_status launch_gather_rows(const void* src, const AnyGlobals& a, int B, int L, int D, void* dst,
                             cudaStream_t stream);

// any (may be NULL): global tokens at any position (global_idx and
// global_token_nums are used).
lf_status launch_attention_simt_f32(const float* q, const float* k, const float* v, const float* qg,
                                    const float* kg, const float* vg, const float* local_mask,
                                    const float* global_mask, int B, int H, int L, int w,
                                    float scale, float* out, int* status, cudaStream_t stream,
                                    const AnyGlobals* any = nullptr, int32_t* gidx_out = nullptr,
                                    int32_t* gnum_out = nullptr);

// Tensor-core path (fp16 / bf16).  `scratch` must hold
// attention_tc_scratch_bytes(B, H, L, w) bytes whose counter region is zero
// on entry (the kernel leaves it zero).
size_t attention_tc_scratch_bytes(int B, int H, int L, int w);
// Leading part of that scratch (scheduler and split counters) that must be
// zero when a launch starts.
size_t attention_tc_scratch_zero_bytes(int B, int H, int L, int w);
// any (may be NULL): global tokens at any position, with the compact
// buffers filled by launch_gather_globals.  gidx_out / gnum_out (prefix
// path, may be NULL): the kernel also writes the global-index partition
// (as launch_global_idx with the prefix check) into them.  masks_early: the
// work queued right before does not write the masks (inside a layer call).
lf_status launch_attention_tc(const void* q, const void* k, const void* v, const void* qg,
                              const void* kg, const void* vg, const float* local_mask,
                              const float* global_mask, int B, int H, int L, int w, float scale,
                              lf_dtype dtype, void* out, void* scratch, int* status,
                              int sm_count, cudaStream_t stream, const AnyGlobals* any = nullptr,
                              int32_t* gidx_out = nullptr, int32_t* gnum_out = nullptr, bool masks_early = false);

// ---- dense GEMM with fused epilogues (encoder layer) ----
enum { kEpiHeads = 0, kEpiGelu = 1, kEpiResid = 2, kEpiResidLN = 3 };
struct GemmArgs {
    const void* A;     // [batches][batch_stride][K], K-major
    int batches, rows, batch_stride, K;
    const void* W;     // [N][K] (nn.Linear layout)
    int N;
    const void* bias;  // [N]
    int mode;          // kEpi*
    const void* resid; // kEpiResid: [batches*rows][N]
    void* out;
    int heads_D, heads_H, heads_L;  // kEpiHeads
    int* status;
    // Optional second problem of the same launch (kEpiHeads only; rows2 > 0
    // enables it): same batches, K, heads_D and heads_H; its tiles run after
    // the first problem's, on the SMs its last wave leaves free.
    const void* A2;    // [batches][batch_stride2][K]
    int rows2, batch_stride2;
    const void* W2;    // [N2][K]
    int N2;
    const void* bias2; // [N2]
    void* out2;
    int heads_L2;
    // The weights are not written by the work queued right before this
    // launch (a kernel that may let it start early): their first tiles are
    // loaded before the wait for that work.
    bool w_early;
    // kEpiResidLN: out = LayerNorm(A W^T + bias + resid) in dtype, over
    // rows of N <= 1024 columns (population variance; gamma, beta fp32).
    const float* ln_gamma;
    const float* ln_beta;
    float ln_eps;
};
// N % 128 == 0, K % 64 == 0; fp16 / bf16.
lf_status launch_gemm_tc(const GemmArgs& g, lf_dtype dtype, int sm_count, cudaStream_t stream);

// ---- fused GELU FFN: out = h + b2 + GELU(h W1^T + b1) W2^T (fp32) ----
struct FfnArgs {
    const void* h;    // [M][D] (also the residual)
    const void* W1;   // [F][D]
    const void* b1;   // [F]
    const void* W2;   // [D][F]
    const void* b2;   // [D]
    int M, D, F;
    float* out;       // [M][D]
    int* status;
};
// CTAs per cluster of the fused kernel for model width D (0: unsupported).
int ffn_fused_cluster(int D);
bool ffn_fused_supported(int M, int D, int F);
lf_status launch_ffn_fused(const FfnArgs& a, lf_dtype dtype, cudaStream_t stream);

// LayerNorm over rows of an fp32 [rows][N] matrix into dtype (N % 32 == 0, N <= 1024).
lf_status launch_layernorm(const float* z, const float* gamma, const float* beta, int rows, int N, float eps,
                           lf_dtype dtype, void* out, cudaStream_t stream);

}  // namespace lf
