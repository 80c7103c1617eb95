/*
 * lf.h -- C ABI of liblf.so: Longformer banded + global self-attention on
 * NVIDIA B200 (sm_100a).
 *
 * "FTL" below is the page "FasterTransformer Longformer 推理加速实践：
 * PyTorch 集成、输入约束与端到端性能解析"; each entry point cites the
 * section of that page defining the operation it performs.
 *
 * Conventions for every entry point:
 *   - Tensor arguments are DEVICE pointers to caller-owned, dense, row-major
 *     memory on the current CUDA device, unless marked "host".  The library
 *     never frees or retains them after the call's work has finished.
 *   - Device pointers must be 16-byte aligned (LF_ERR_MISALIGNED otherwise).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous unless the description says otherwise.
 *   - Host-side validation happens before anything is launched; a non-zero
 *     return means nothing was enqueued (except LF_ERR_CUDA, which reports a
 *     failed launch).
 *   - Errors that depend on mask CONTENTS are found on the device.  Kernels
 *     record the first such error in a per-device status word, read (and
 *     optionally cleared) by lf_device_status().
 *   - Outputs must not alias inputs.
 *   - head_dim is fixed at 64 (FTL §使用前提：四条硬性约束, item 2): there is no
 *     head-dim argument.
 */
#ifndef LF_H_
#define LF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* lf_stream_t;

typedef enum {
    LF_OK = 0,
    LF_ERR_NULL = 1,                 /* a required pointer is NULL */
    LF_ERR_BAD_DIM = 2,              /* B, H, L or w <= 0 */
    LF_ERR_L_NOT_MULTIPLE_OF_W = 3,  /* FTL §使用前提 item 1: L % w != 0 */
    LF_ERR_L_LT_2W = 4,              /* FTL §使用前提 item 1: L < 2w */
    LF_ERR_G_GT_W = 5,               /* FTL §使用前提 item 3: global tokens > w */
    LF_ERR_GLOBAL_NOT_PREFIX = 6,    /* FTL §使用前提 item 4: globals not at 0..g-1 */
    LF_ERR_DTYPE = 7,                /* unsupported dtype value */
    LF_ERR_MISALIGNED = 8,           /* a device pointer is not 16-byte aligned */
    LF_ERR_CUDA = 9,                 /* a CUDA runtime call or launch failed */
    LF_ERR_DEVICE_TIMEOUT = 10,      /* a bounded device-side wait expired */
    LF_ERR_UNSUPPORTED_DEVICE = 11,  /* current device is not compute capability 10.0 */
    LF_ERR_WORKSPACE = 12,           /* workspace pointer/size too small */
    LF_ERR_TOO_LARGE = 13,           /* a size exceeds the documented maximum */
    LF_ERR_SCRATCH_LIMIT = 14        /* shape needs more scratch than lf_attention_forward_noalloc holds */
} lf_status;

typedef enum { LF_F32 = 0, LF_F16 = 1, LF_BF16 = 2 } lf_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* lf_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int lf_version(void);

/*
 * lf_device_status -- synchronise `stream`, then return the first
 * content-dependent error recorded by this library's kernels on the current
 * device since the last reset (LF_OK if none).  reset != 0 clears the word.
 * Errors recorded: LF_ERR_G_GT_W, LF_ERR_GLOBAL_NOT_PREFIX,
 * LF_ERR_DEVICE_TIMEOUT.
 */
lf_status lf_device_status(lf_stream_t stream, int reset);

/*
 * lf_init_global_idx -- global-token index partition.
 * FTL §Longformer Encoder 计算流程 / 预处理 (invokeInitLongformerIdx): for each
 * sample b, positions j with global_mask[b,j] == 0.0f are "global".
 *
 *   global_mask       [B, L] float32, device.  0.0 = global token, any other
 *                     value (the page uses -10000.0) = not global.
 *   global_idx        [B, L] int32, device, written: the global positions in
 *                     ascending order, followed by the other positions in
 *                     descending order (the order of a stable flagged
 *                     partition that writes rejected items from the back).
 *   global_token_nums [B] int32, device, written: g_b = number of globals.
 *   max_global_out    HOST int*, may be NULL.  If non-NULL the call
 *                     synchronises `stream`, writes max_b g_b there and
 *                     returns the content check below directly; the device
 *                     status word is cleared before the launch in that mode.
 *
 * Content check (FTL §使用前提 items 3 and 4): every g_b <= w and the globals
 * of each sample are exactly positions 0..g_b-1; otherwise
 * LF_ERR_G_GT_W / LF_ERR_GLOBAL_NOT_PREFIX (device status word, or the
 * return value in synchronous mode).  Outputs are written in full either way.
 * Shape checks: B, L, w > 0, L % w == 0, L >= 2w (FTL §使用前提 item 1).
 */
lf_status lf_init_global_idx(const float* global_mask, int B, int L, int w,
                             int32_t* global_idx, int32_t* global_token_nums,
                             int* max_global_out, lf_stream_t stream);

/*
 * lf_attention_forward -- Longformer self-attention of one layer.
 * FTL §Longformer Encoder 计算流程 / 每个 Transformer 层, steps 3-5
 * (LongformerAttentionLayer::forward, longformerMHASoftmax and
 * TransposeMultiHeadToSingle), fused into one kernel.
 *
 *   q, k, v, qg, kg, vg  [B, H, L, 64] of `dtype`, device (the layout after
 *                        AddBiasTransposeToMultiHead, step 2).  qg is read
 *                        only at rows i < g_b.
 *   local_mask           [B, L] float32: 1.0 = token, 0.0 = padding.
 *   global_mask          [B, L] float32: 0.0 = global, -10000.0 = not.
 *   out                  [B, L, H*64] of `dtype`, device, written in full.
 *
 * With lb[j] = fmaf(local_mask[b,j], 10000, -10000), s = 1/8 and
 * g_b = number of leading 0.0 entries of global_mask[b]:
 *   row i with lb[i] != 0                -> out row = 0;
 *   row i <  g_b (global row)            -> softmax_j(s*qg_i.kg_j + lb[j]) over
 *                                           all j, values vg;
 *   row i >= g_b (local row)             -> softmax over the set
 *                                           {|i-j| <= w} U {0..g_b-1} (each key
 *                                           once) of s*q_i.k_j + lb[j], values v.
 * dtype: LF_F32 (CUDA-core FMA path), LF_F16 or LF_BF16 (tensor-core path,
 * fp32 accumulation and softmax, output rounded to nearest even).
 * Shape checks as lf_init_global_idx.  Content: a sample with g_b > w records
 * LF_ERR_G_GT_W and gets an all-zero output; a 0.0 entry of global_mask after
 * position g_b records LF_ERR_GLOBAL_NOT_PREFIX (output computed with g_b).
 * Scratch: the call uses a library-owned per-device scratch buffer, allocated
 * (cudaMalloc) on the first call on a device and regrown when a call needs
 * more.  Make the largest call before any stream capture: regrowing frees
 * the old buffer, which graphs captured earlier still reference.  The
 * scratch's counters must be zero when the kernel starts: a call clears
 * them (a cudaMemsetAsync on `stream`) when a call of another shape or dtype
 * may have left other data there, and always while `stream` is capturing,
 * so that a captured call stays correct whatever runs between replays.
 * Calls that overlap on the GPU (different streams) share the scratch and
 * must not overlap.
 */
lf_status lf_attention_forward(const void* q, const void* k, const void* v,
                               const void* qg, const void* kg, const void* vg,
                               const float* local_mask, const float* global_mask,
                               int B, int H, int L, int w, lf_dtype dtype,
                               lf_stream_t stream, void* out);

/* Bytes of scratch lf_attention_forward needs for this shape (0 if none). */
size_t lf_attention_scratch_bytes(int B, int H, int L, int w, lf_dtype dtype);

/*
 * lf_attention_forward_idx -- lf_init_global_idx (asynchronous mode) and
 * lf_attention_forward in one call: FTL §Longformer Encoder 计算流程 /
 * 预处理 followed by steps 3-5, in ONE kernel launch: CTA b of the attention
 * kernel also computes the partition of sample b (for fp16 / bf16 its
 * epilogue warps, while the first scores are computed).  Arguments as
 * lf_attention_forward, plus global_idx [B, L] and global_token_nums [B]
 * (int32, device, written exactly as lf_init_global_idx writes them, with
 * its content check recorded in the device status word).  Errors: as
 * lf_attention_forward; LF_ERR_NULL / LF_ERR_MISALIGNED also for the two
 * partition outputs.  Asynchronous on `stream`.
 */
lf_status lf_attention_forward_idx(const void* q, const void* k, const void* v,
                                   const void* qg, const void* kg, const void* vg,
                                   const float* local_mask, const float* global_mask,
                                   int B, int H, int L, int w, lf_dtype dtype,
                                   lf_stream_t stream, void* out,
                                   int32_t* global_idx, int32_t* global_token_nums);

/*
 * lf_attention_forward_any_globals -- lf_attention_forward with the global
 * tokens at any positions of the sequence: the HuggingFace arrangement that
 * FTL §使用前提 item 4 names as unsupported by FT, gathered through the
 * global_idx of the partition (invokeInitLongformerIdx, FTL §计算流程 /
 * 预处理) instead of being read as a prefix.
 *
 * Arguments, layouts, dtypes, shape checks and the scratch rules are those of
 * lf_attention_forward.  With G_b = { j : global_mask[b,j] == 0.0 } and
 * g_b = |G_b|:
 *   row i with lb[i] != 0                -> out row = 0 (global rows too);
 *   row i in G_b (global row)            -> softmax_j(s*qg_i.kg_j + lb[j]) over
 *                                           all j, values vg;
 *   any other row (local row)            -> softmax over the set
 *                                           {|i-j| <= w} U G_b (each key once)
 *                                           of s*q_i.k_j + lb[j], values v.
 * qg is read only at the rows of G_b.  A sample with g_b > w records
 * LF_ERR_G_GT_W and gets an all-zero output.  With G_b = {0..g_b-1} the
 * result is that of lf_attention_forward.  The call runs the partition into
 * its scratch (global_idx, global_token_nums and a per-position count of the
 * global tokens before it), then for LF_F16 / LF_BF16 a gather of the global
 * tokens' qg, k and v rows into per-head slot buffers, then the attention
 * kernel; all three are asynchronous on `stream`.
 */
lf_status lf_attention_forward_any_globals(const void* q, const void* k, const void* v,
                                           const void* qg, const void* kg, const void* vg,
                                           const float* local_mask, const float* global_mask,
                                           int B, int H, int L, int w, lf_dtype dtype,
                                           lf_stream_t stream, void* out);

/* Bytes of scratch lf_attention_forward_any_globals needs for this shape. */
size_t lf_attention_any_globals_scratch_bytes(int B, int H, int L, int w, lf_dtype dtype);

/* Free the library-owned scratch of the current device (synchronises it). */
lf_status lf_release_scratch(void);

/*
 * One Longformer encoder layer: FTL §Longformer Encoder 计算流程 / 每个
 * Transformer 层, steps 1-6 (LongformerEncoder::forwardLayer):
 *   [q k v kg vg] = x W^T + b      (step 1; the five weights contiguous, as
 *                                    §PyTorch OP requires)   -> [B,H,L,64] (step 2)
 *   qg            = x W_qg^T + b_qg over the rows that can be global (i <
 *                   ceil(w/128)*128), as the page's separate Qg GEMM
 *   a             = attention(q, k, v, qg, kg, vg)   (steps 3-5, scale attn_scale)
 *   h             = LN1(a W_o^T + b_o + x)           (step 5, AddBiasResidualLayerNorm)
 *   y             = LN2(GELU(h W_1^T + b_1) W_2^T + b_2 + h)   (step 6, GeluFfnLayer)
 * GELU is the erf form; LN uses the population variance and ln_eps.
 * All weights use the nn.Linear layout [out_features][in_features] in the
 * layer's dtype; LayerNorm parameters are fp32.  D = H*64.
 */
typedef struct {
    int ffn_dim;                 /* F: FFN inner size (multiple of 128) */
    const void* W_qkv_kgvg;      /* [5][D][D]: q, k, v, kg, vg weights, contiguous */
    const void* b_qkv_kgvg;      /* [5][D] */
    const void* W_qg;            /* [D][D] */
    const void* b_qg;            /* [D] */
    const void* W_o;             /* [D][D] */
    const void* b_o;             /* [D] */
    const float* ln1_gamma;      /* [D] */
    const float* ln1_beta;       /* [D] */
    const void* W_1;             /* [F][D] */
    const void* b_1;             /* [F] */
    const void* W_2;             /* [D][F] */
    const void* b_2;             /* [D] */
    const float* ln2_gamma;      /* [D] */
    const float* ln2_beta;       /* [D] */
} lf_layer_weights;

/* Bytes of device workspace lf_encoder_layer_forward needs (0 on bad sizes). */
size_t lf_encoder_layer_workspace_bytes(int B, int H, int L, int w, int ffn_dim, lf_dtype dtype);

/*
 * lf_encoder_layer_forward -- the layer above.  x and out are [B, L, D] of
 * `dtype` (LF_F16 or LF_BF16), masks as lf_attention_forward.  `workspace`
 * is caller-owned device memory of at least
 * lf_encoder_layer_workspace_bytes(...) bytes, 256-byte aligned; its
 * contents need not be initialised and are overwritten.  Shape rules: those
 * of lf_attention_forward, plus D = H*64 a multiple of 128 (H even),
 * D <= 1024 (LayerNorm keeps a row in registers) and F a multiple of 128.
 * Errors: LF_ERR_WORKSPACE if the workspace is missing, misaligned or too
 * small; otherwise as lf_attention_forward.  Asynchronous on `stream`.
 */
lf_status lf_encoder_layer_forward(const void* x, const float* local_mask, const float* global_mask,
                                   const lf_layer_weights* weights, int B, int H, int L, int w,
                                   float attn_scale, float ln_eps, lf_dtype dtype,
                                   void* workspace, size_t workspace_bytes,
                                   lf_stream_t stream, void* out);

/*
 * lf_encoder_forward -- the encoder: n_layers layers of lf_encoder_layer_forward
 * applied in turn (FasterTransformer Longformer page, §Longformer Encoder
 * 计算流程: preprocessing once, then the layer loop; the attention of every
 * layer derives g_b from the global_mask prefix itself, so no separate
 * preprocessing pass is needed).  layers is a HOST array of n_layers weight
 * sets (each as for lf_encoder_layer_forward, all with the same ffn_dim).
 * x and out are [B, L, D] of `dtype`; they must not alias.  `workspace` is
 * caller-owned device memory of at least lf_encoder_workspace_bytes(...)
 * bytes, 256-byte aligned: one layer's workspace plus, for n_layers > 1, two
 * [B, L, D] activation buffers the layers alternate between.
 * Errors: LF_ERR_BAD_DIM for n_layers <= 0 or differing ffn_dim; every
 * layer's weights are checked (LF_ERR_NULL, LF_ERR_MISALIGNED) before the
 * first layer is launched; otherwise as lf_encoder_layer_forward.
 * Asynchronous on `stream`.
 */
size_t lf_encoder_workspace_bytes(int n_layers, int B, int H, int L, int w, int ffn_dim, lf_dtype dtype);
lf_status lf_encoder_forward(const void* x, const float* local_mask, const float* global_mask,
                             const lf_layer_weights* layers, int n_layers, int B, int H, int L, int w,
                             float attn_scale, float ln_eps, lf_dtype dtype,
                             void* workspace, size_t workspace_bytes,
                             lf_stream_t stream, void* out);

/*
 * lf_encoder_layer_forward_any_globals, lf_encoder_forward_any_globals -- the
 * layer and the encoder with the global tokens at any positions (the
 * attention as in lf_attention_forward_any_globals: global rows are the
 * positions with global_mask == 0.0, a local row attends its window and
 * every global token).  Arguments, layouts, validation and errors as for
 * lf_encoder_layer_forward / lf_encoder_forward, with the workspace sizes
 * below.  The partition of global_mask (with a count of the global tokens
 * before each position) runs once per call, before the first layer; each
 * layer projects qg only for the global tokens' rows of its input, gathered
 * through global_idx, and gathers their k / v rows after its projections.
 * A sample with more than w global tokens records LF_ERR_G_GT_W and gets a
 * zero attention output in every layer.  Asynchronous on `stream`.
 */
size_t lf_encoder_layer_any_globals_workspace_bytes(int B, int H, int L, int w, int ffn_dim, lf_dtype dtype);
lf_status lf_encoder_layer_forward_any_globals(const void* x, const float* local_mask, const float* global_mask,
                                               const lf_layer_weights* wts, int B, int H, int L, int w,
                                               float attn_scale, float ln_eps, lf_dtype dtype,
                                               void* workspace, size_t workspace_bytes,
                                               lf_stream_t stream, void* out);
size_t lf_encoder_any_globals_workspace_bytes(int n_layers, int B, int H, int L, int w, int ffn_dim,
                                              lf_dtype dtype);
lf_status lf_encoder_forward_any_globals(const void* x, const float* local_mask, const float* global_mask,
                                         const lf_layer_weights* layers, int n_layers, int B, int H, int L,
                                         int w, float attn_scale, float ln_eps, lf_dtype dtype,
                                         void* workspace, size_t workspace_bytes,
                                         lf_stream_t stream, void* out);

/*
 * The GELU feed-forward network of the layer (FTL §Longformer Encoder
 * 计算流程 / 每个 Transformer 层 step 6, GeluFfnLayer) before its LayerNorm:
 *   z[r, :] = h[r, :] + b_2 + GELU(h[r, :] W_1^T + b_1) W_2^T
 * GELU in the erf form; the F-wide intermediate is rounded to `dtype`
 * (where the page's layer stores it).  Two paths compute it:
 *   LF_FFN_UNFUSED  two GEMMs with fused epilogues; the intermediate
 *                   [rows, F] goes through `workspace`
 *   LF_FFN_FUSED    one kernel (the fused linear -> GELU -> linear of the
 *                   PaddleNLP FastFFN page, §FastFFN融合计算): clusters of
 *                   CTAs keep the intermediate on chip in 128-wide chunks
 *                   (needs F a multiple of 128 * c, c = 1, 2, 4 for D <= 256,
 *                   <= 512, <= 1024); no workspace
 *   LF_FFN_AUTO     the path measured faster on B200: fused for d_model
 *                   <= 256 (one CTA holds a row tile's whole output), the
 *                   two GEMMs above that
 * Both sum over D and over F in the same order and give the same result bit
 * for bit.
 */
typedef enum { LF_FFN_AUTO = 0, LF_FFN_UNFUSED = 1, LF_FFN_FUSED = 2 } lf_ffn_path;

/* Bytes of workspace lf_gelu_ffn_forward needs for `path` (0 when it needs
 * none or the sizes are invalid). */
size_t lf_gelu_ffn_workspace_bytes(int rows, int d_model, int ffn_dim, lf_dtype dtype, int path);

/*
 * lf_gelu_ffn_forward -- the FFN above.
 *   h     [rows, d_model] of dtype (LF_F16 or LF_BF16); also the residual
 *   W_1   [ffn_dim, d_model], b_1 [ffn_dim]; W_2 [d_model, ffn_dim],
 *         b_2 [d_model] (nn.Linear layout, dtype)
 *   z     [rows, d_model] float32, written
 *   workspace: device memory of lf_gelu_ffn_workspace_bytes(...) bytes,
 *         256-byte aligned (may be NULL when that is 0)
 * Shape rules: rows > 0; d_model a multiple of 128, <= 1024; ffn_dim a
 * multiple of 128.  Errors: LF_ERR_NULL, LF_ERR_MISALIGNED, LF_ERR_DTYPE,
 * LF_ERR_BAD_DIM (shape rules, unknown path, or LF_FFN_FUSED for a shape it
 * does not take), LF_ERR_WORKSPACE, LF_ERR_CUDA; a device-side wait that
 * expires records LF_ERR_DEVICE_TIMEOUT (lf_device_status).  Asynchronous.
 */
lf_status lf_gelu_ffn_forward(const void* h, const void* W_1, const void* b_1, const void* W_2, const void* b_2,
                              int rows, int d_model, int ffn_dim, lf_dtype dtype, int path,
                              void* workspace, size_t workspace_bytes, lf_stream_t stream, float* z);

/*
 * lf_set_ffn_path -- the FFN path (lf_ffn_path) the encoder-layer and
 * encoder entry points use from now on, in this process (default
 * LF_FFN_AUTO; a shape the fused path does not take always runs unfused).
 * The layer workspace sizes do not depend on it.  Returns LF_ERR_BAD_DIM for
 * an unknown value.  lf_get_ffn_path returns the current setting.
 */
lf_status lf_set_ffn_path(int path);
int lf_get_ffn_path(void);

/*
 * lf_attention_forward_noalloc -- lf_attention_forward for callers that
 * cannot allocate device memory.  The pages describe no such entry point: it
 * exists for code that may not call cudaMalloc (for example code running
 * inside another framework's device-memory pool, or allocation-free real-time
 * paths) and so cannot let the library grow its scratch buffer.
 *
 * Same arguments, layouts and results as lf_attention_forward, for LF_F16 and
 * LF_BF16 only (LF_F32 needs no scratch: use lf_attention_forward).  The
 * caller still provides every input and the output.  This call allocates
 * nothing: its scratch is a fixed 32 MiB array in the library's device image,
 * reserved on every device where the library's module is loaded (any device
 * that has made any lf call) until the process exits.  A shape whose scratch
 * (lf_attention_scratch_bytes) exceeds 32 MiB returns LF_ERR_SCRATCH_LIMIT
 * before anything is launched.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress); make that first call before
 * any stream capture.  Each call clears the array's counter region on
 * `stream` (cudaMemsetAsync) before its kernel.  All calls share the one
 * array: calls that overlap on the GPU (different streams) race and must not
 * overlap.  Content errors (g_b > w, globals not a prefix) and expired
 * device waits are recorded in a status word of this entry point, separate
 * from the library's, read by lf_noalloc_device_status.
 */
lf_status lf_attention_forward_noalloc(const void* q, const void* k, const void* v,
                                       const void* qg, const void* kg, const void* vg,
                                       const float* local_mask, const float* global_mask,
                                       int B, int H, int L, int w, lf_dtype dtype,
                                       lf_stream_t stream, void* out);

/*
 * lf_noalloc_device_status -- as lf_device_status, for the status word of
 * lf_attention_forward_noalloc (no counterpart on the pages): synchronise
 * `stream`, return the first error recorded by that entry point's kernel on
 * the current device since the last reset (LF_OK if none; LF_ERR_G_GT_W,
 * LF_ERR_GLOBAL_NOT_PREFIX or LF_ERR_DEVICE_TIMEOUT otherwise); reset != 0
 * clears the word.  Allocates nothing.
 */
lf_status lf_noalloc_device_status(lf_stream_t stream, int reset);

/*
 * lf_selftest_bounded_wait -- a check of the library's failure detection
 * (no counterpart on the pages).  Every device-side wait of the kernels is
 * bounded; when one gives up, the kernel records LF_ERR_DEVICE_TIMEOUT in the
 * device status word and returns instead of hanging.  This call launches one
 * CTA that waits, with that same bounded routine, on an mbarrier phase that
 * nothing completes, giving up after limit_ns nanoseconds; it then records
 * LF_ERR_DEVICE_TIMEOUT (read by lf_device_status) and returns.  limit_ns
 * must lie in [1000, 100000000] (LF_ERR_BAD_DIM otherwise).  Asynchronous on
 * `stream`; nothing else is in flight in that CTA when the wait gives up.
 */
lf_status lf_selftest_bounded_wait(unsigned long long limit_ns, lf_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LF_H_ */
