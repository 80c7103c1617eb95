// One Longformer encoder layer on the tensor cores: the composition of the
// FasterTransformer Longformer page, §Longformer Encoder 计算流程 / 每个
// Transformer 层 steps 1-6, as a sequence of this library's kernels on one
// stream (no host synchronisation):
//   GEMM(x, W_qkv_kgvg) + bias -> q, k, v, kg, vg in head layout, and in the
//     same launch GEMM(x rows < ceil(w/128)*128, W_qg) + bias -> qg in head
//     layout, whose few tiles run on the SMs the large one's last wave
//     leaves free
//   banded + global attention -> a [B, L, D]
//   GEMM(a, W_o) + b_o + x, LayerNorm in its epilogue -> h
//   GEMM(h, W_1) + b_1, GELU -> f;  GEMM(f, W_2) + b_2 + h, LayerNorm in its
//     epilogue -> out  (or the fused FFN kernel, which keeps f on chip,
//     -> z (fp32), then the LayerNorm kernel -> out)
// With the global tokens at any position (the _any_globals entry points) the
// partition (with its rank table) runs once per forward, the qg projection
// multiplies only the global tokens' rows of x, gathered through global_idx,
// and writes them straight into the slot buffer of the attention kernel, and
// the k / v rows of the global tokens are gathered after the projections.
#include <atomic>

#include "lf_internal.h"

namespace lf {
namespace {

struct Workspace {
    size_t qkv, qg, att, z, h, f, scratch, any, xg, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// any: global tokens at any position (partition outputs and slot buffers,
// and the gathered rows of x; no position-indexed qg buffer).
Workspace layout(int B, int H, int L, int w, int F, int elem, bool any) {
    const size_t D = (size_t)H * 64, rows = (size_t)B * L;
    Workspace s;
    size_t o = 0;
    s.qkv = o; o += align256(5 * rows * D * elem);
    s.qg = o; if (!any) o += align256(rows * D * elem);
    s.att = o; o += align256(rows * D * elem);
    s.z = o; o += align256(rows * D * 4);
    s.h = o; o += align256(rows * D * elem);
    s.f = o; o += align256(rows * (size_t)F * elem);
    s.scratch = o; o += align256(attention_tc_scratch_bytes(B, H, L, w));
    s.any = s.xg = o;
    if (any) {
        o += align256(any_globals_bytes(B, H, L, w, true));
        s.xg = o; o += align256((size_t)B * any_globals_gcap(w) * D * elem);
    }
    s.total = o;
    return s;
}

lf_status check_weights(const lf_layer_weights* wt) {
    const void* wptrs[] = {wt->W_qkv_kgvg, wt->b_qkv_kgvg, wt->W_qg, wt->b_qg, wt->W_o, wt->b_o,
                           wt->ln1_gamma, wt->ln1_beta, wt->W_1, wt->b_1, wt->W_2, wt->b_2,
                           wt->ln2_gamma, wt->ln2_beta};
    for (const void* p : wptrs) {
        if (!p) return LF_ERR_NULL;
        if (!aligned16(p)) return LF_ERR_MISALIGNED;
    }
    return LF_OK;
}

lf_status check_layer(int B, int H, int L, int w, int F, lf_dtype dtype) {
    lf_status st = check_shape(B, H, L, w);
    if (st != LF_OK) return st;
    if (dtype != LF_F16 && dtype != LF_BF16) return LF_ERR_DTYPE;
    const int D = H * 64;
    if (D % 128 != 0 || D > 1024 || F <= 0 || F % 128 != 0) return LF_ERR_BAD_DIM;
    return LF_OK;
}

}  // namespace
}  // namespace lf

using namespace lf;

namespace lf {
namespace {

std::atomic<int> g_ffn_path{LF_FFN_AUTO};

// The path a call with FFN path setting `path` takes for this shape.  AUTO
// takes the fused kernel where it measured faster on B200: when one CTA
// holds a row tile's whole output (D <= 256).  With clusters of 2 or 4 CTAs
// both paths stream the same operand bytes per flop from L2, and the fused
// kernel has less shared memory for its TMA ring and fills 128 of the 148
// SMs at 4096 rows; there the two GEMMs are faster.
int ffn_path_for(int M, int D, int F, int path) {
    if (path == LF_FFN_UNFUSED || !ffn_fused_supported(M, D, F)) return LF_FFN_UNFUSED;
    if (path == LF_FFN_AUTO && ffn_fused_cluster(D) != 1) return LF_FFN_UNFUSED;
    return LF_FFN_FUSED;
}

// Step 6 before its LayerNorm: z = h + b_2 + GELU(h W_1^T + b_1) W_2^T,
// fused or as two GEMMs through f ([M][F] of dtype).  w_early: the work
// queued before does not write the weights (inside a layer call).
lf_status gelu_ffn(const void* h, const void* W1, const void* b1, const void* W2, const void* b2, int M, int D, int F,
                   lf_dtype dtype, int path, void* f, float* z, DeviceCtx* d, cudaStream_t s, bool w_early = false) {
    if (path == LF_FFN_FUSED) {
        FfnArgs a{};
        a.h = h; a.W1 = W1; a.b1 = b1; a.W2 = W2; a.b2 = b2;
        a.M = M; a.D = D; a.F = F; a.out = z; a.status = d->status;
        return launch_ffn_fused(a, dtype, s);
    }
    lf_status st;
    GemmArgs f1{};
    f1.A = h; f1.batches = 1; f1.rows = M; f1.batch_stride = M; f1.K = D;
    f1.W = W1; f1.N = F; f1.bias = b1; f1.mode = kEpiGelu; f1.out = f; f1.status = d->status;
    f1.w_early = w_early;
    if ((st = launch_gemm_tc(f1, dtype, d->sm_count, s)) != LF_OK) return st;
    GemmArgs f2{};
    f2.A = f; f2.batches = 1; f2.rows = M; f2.batch_stride = M; f2.K = F;
    f2.W = W2; f2.N = D; f2.bias = b2; f2.mode = kEpiResid; f2.resid = h; f2.out = z; f2.status = d->status;
    f2.w_early = true;  // W_2 is not written by the FFN1 GEMM before it
    return launch_gemm_tc(f2, dtype, d->sm_count, s);
}

// One layer on the workspace `base` (layout ws).  any: global tokens at any
// position; first: the first layer of the call, which runs the partition
// (any) and clears the attention kernel's scheduler and split counters in
// the workspace (every attention launch leaves them zero for the next
// layer).  Arguments are validated by the callers.
lf_status layer_forward(const void* x, const float* local_mask, const float* global_mask, const lf_layer_weights* wt,
                        int B, int H, int L, int w, float attn_scale, float ln_eps, lf_dtype dtype, uint8_t* base,
                        const Workspace& ws, bool any, bool first, DeviceCtx* d, cudaStream_t s, void* out) {
    lf_status st;
    const int D = H * 64, F = wt->ffn_dim;
    if (first &&
        cudaMemsetAsync(base + ws.scratch, 0, attention_tc_scratch_zero_bytes(B, H, L, w), s) != cudaSuccess)
        return LF_ERR_CUDA;
    const size_t head_elems = (size_t)B * H * L * 64;
    uint8_t* qkv = base + ws.qkv;  // [5][B][H][L][64]
    auto slot = [&](int i) { return qkv + (size_t)i * head_elems * 2; };
    AnyGlobals a{};
    if (any) {
        a = any_globals_layout(base + ws.any, B, H, L, w, true);
        if (first &&
            (st = launch_global_idx(global_mask, B, L, w, const_cast<int32_t*>(a.global_idx),
                                    const_cast<int32_t*>(a.global_token_nums), d->status, s,
                                    const_cast<int32_t*>(a.rank), false)) != LF_OK)
            return st;
    }

    // steps 1-2: the five projections with bias, scattered to head layout,
    // and the Qg projection as a second problem of the same launch (its
    // tiles run on the SMs the five projections' last wave leaves free)
    GemmArgs g{};
    g.A = x; g.batches = B; g.rows = L; g.batch_stride = L; g.K = D;
    g.W = wt->W_qkv_kgvg; g.N = 5 * D; g.bias = wt->b_qkv_kgvg; g.mode = kEpiHeads;
    g.out = qkv; g.heads_D = D; g.heads_H = H; g.heads_L = L; g.status = d->status;
    g.W2 = wt->W_qg; g.N2 = D; g.bias2 = wt->b_qg;
    g.w_early = true;  // inside a layer call no kernel writes the weights
    if (any) {
        // Qg of the global tokens only: their rows of x, gathered, into the
        // slot buffer (slot layout [B][H][gcap][64])
        if ((st = launch_gather_rows(x, a, B, L, D, base + ws.xg, s)) != LF_OK) return st;
        g.A2 = base + ws.xg; g.rows2 = a.gcap; g.batch_stride2 = a.gcap; g.heads_L2 = a.gcap; g.out2 = a.qg_c;
    } else {
        // Qg over the rows that can be global tokens (g_b <= w)
        const int qrows = ((w + 127) / 128) * 128 < L ? ((w + 127) / 128) * 128 : L;
        g.A2 = x; g.rows2 = qrows; g.batch_stride2 = L; g.heads_L2 = L; g.out2 = base + ws.qg;
    }
    if ((st = launch_gemm_tc(g, dtype, d->sm_count, s)) != LF_OK) return st;
    // the global tokens' k / v rows and local_mask values into their slots
    if (any && (st = launch_gather_globals(nullptr, slot(1), slot(2), local_mask, a, B, H, L, w, s)) != LF_OK)
        return st;
    // steps 3-5: attention (launched right after the projections, it waits
    // for them on the device; its counters are zero, see above)
    if ((st = launch_attention_tc(slot(0), slot(1), slot(2), any ? a.qg_c : base + ws.qg, slot(3), slot(4),
                                  local_mask, global_mask, B, H, L, w, attn_scale, dtype, base + ws.att,
                                  base + ws.scratch, d->status, d->sm_count, s, any ? &a : nullptr, nullptr,
                                  nullptr, true)) != LF_OK)
        return st;
    // step 5: output projection + bias + residual with its LayerNorm in the
    // GEMM's epilogue (the D-wide row tile's CTAs form a cluster)
    GemmArgs o{};
    o.A = base + ws.att; o.batches = B; o.rows = L; o.batch_stride = L; o.K = D;
    o.W = wt->W_o; o.N = D; o.bias = wt->b_o; o.mode = kEpiResidLN; o.resid = x; o.out = base + ws.h;
    o.ln_gamma = wt->ln1_gamma; o.ln_beta = wt->ln1_beta; o.ln_eps = ln_eps;
    o.status = d->status; o.w_early = true;
    if ((st = launch_gemm_tc(o, dtype, d->sm_count, s)) != LF_OK) return st;
    // step 6: GELU FFN + bias + residual, LayerNorm
    const int path = ffn_path_for(B * L, D, F, g_ffn_path.load());
    if (path == LF_FFN_UNFUSED) {
        // two GEMMs, the LayerNorm in the second one's epilogue
        GemmArgs f1{};
        f1.A = base + ws.h; f1.batches = 1; f1.rows = B * L; f1.batch_stride = B * L; f1.K = D;
        f1.W = wt->W_1; f1.N = F; f1.bias = wt->b_1; f1.mode = kEpiGelu; f1.out = base + ws.f;
        f1.status = d->status; f1.w_early = true;
        if ((st = launch_gemm_tc(f1, dtype, d->sm_count, s)) != LF_OK) return st;
        GemmArgs f2{};
        f2.A = base + ws.f; f2.batches = 1; f2.rows = B * L; f2.batch_stride = B * L; f2.K = F;
        f2.W = wt->W_2; f2.N = D; f2.bias = wt->b_2; f2.mode = kEpiResidLN; f2.resid = base + ws.h; f2.out = out;
        f2.ln_gamma = wt->ln2_gamma; f2.ln_beta = wt->ln2_beta; f2.ln_eps = ln_eps;
        f2.status = d->status; f2.w_early = true;
        return launch_gemm_tc(f2, dtype, d->sm_count, s);
    }
    if ((st = gelu_ffn(base + ws.h, wt->W_1, wt->b_1, wt->W_2, wt->b_2, B * L, D, F, dtype, path, base + ws.f,
                       reinterpret_cast<float*>(base + ws.z), d, s, true)) != LF_OK)
        return st;
    return launch_layernorm(reinterpret_cast<float*>(base + ws.z), wt->ln2_gamma, wt->ln2_beta, B * L, D, ln_eps,
                            dtype, out, s);
}

size_t layer_workspace_bytes(int B, int H, int L, int w, int ffn_dim, lf_dtype dtype, bool any) {
    if (check_layer(B, H, L, w, ffn_dim, dtype) != LF_OK) return 0;
    return layout(B, H, L, w, ffn_dim, 2, any).total;
}

lf_status layer_entry(const void* x, const float* local_mask, const float* global_mask, const lf_layer_weights* wt,
                      int B, int H, int L, int w, float attn_scale, float ln_eps, lf_dtype dtype, void* workspace,
                      size_t workspace_bytes, lf_stream_t stream, void* out, bool any) {
    if (!x || !local_mask || !global_mask || !wt || !out) return LF_ERR_NULL;
    const int F = wt->ffn_dim;
    lf_status st = check_layer(B, H, L, w, F, dtype);
    if (st != LF_OK) return st;
    if ((st = check_weights(wt)) != LF_OK) return st;
    const void* ptrs[] = {x, local_mask, global_mask, out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return LF_ERR_MISALIGNED;
    const Workspace ws = layout(B, H, L, w, F, 2, any);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < ws.total)
        return LF_ERR_WORKSPACE;
    DeviceCtx* d = current_device(&st);
    if (!d) return st;
    return layer_forward(x, local_mask, global_mask, wt, B, H, L, w, attn_scale, ln_eps, dtype,
                         reinterpret_cast<uint8_t*>(workspace), ws, any, true, d, (cudaStream_t)stream, out);
}

}  // namespace
}  // namespace lf

extern "C" size_t lf_encoder_layer_workspace_bytes(int B, int H, int L, int w, int ffn_dim, lf_dtype dtype) {
    return layer_workspace_bytes(B, H, L, w, ffn_dim, dtype, false);
}

extern "C" lf_status lf_encoder_layer_forward(const void* x, const float* local_mask, const float* global_mask,
                                              const lf_layer_weights* wt, int B, int H, int L, int w,
                                              float attn_scale, float ln_eps, lf_dtype dtype, void* workspace,
                                              size_t workspace_bytes, lf_stream_t stream, void* out) {
    return layer_entry(x, local_mask, global_mask, wt, B, H, L, w, attn_scale, ln_eps, dtype, workspace,
                       workspace_bytes, stream, out, false);
}

extern "C" size_t lf_encoder_layer_any_globals_workspace_bytes(int B, int H, int L, int w, int ffn_dim,
                                                               lf_dtype dtype) {
    return layer_workspace_bytes(B, H, L, w, ffn_dim, dtype, true);
}

extern "C" lf_status lf_encoder_layer_forward_any_globals(const void* x, const float* local_mask,
                                                          const float* global_mask, const lf_layer_weights* wt,
                                                          int B, int H, int L, int w, float attn_scale, float ln_eps,
                                                          lf_dtype dtype, void* workspace, size_t workspace_bytes,
                                                          lf_stream_t stream, void* out) {
    return layer_entry(x, local_mask, global_mask, wt, B, H, L, w, attn_scale, ln_eps, dtype, workspace,
                       workspace_bytes, stream, out, true);
}

// ---------------------------------------------------------------- the FFN alone

extern "C" size_t lf_gelu_ffn_workspace_bytes(int rows, int d_model, int ffn_dim, lf_dtype dtype, int path) {
    if (rows <= 0 || d_model <= 0 || d_model % 128 != 0 || d_model > 1024 || ffn_dim <= 0 || ffn_dim % 128 != 0)
        return 0;
    if (dtype != LF_F16 && dtype != LF_BF16) return 0;
    if (path < LF_FFN_AUTO || path > LF_FFN_FUSED) return 0;
    if (path == LF_FFN_FUSED && !ffn_fused_supported(rows, d_model, ffn_dim)) return 0;  // rejected by the call
    if (ffn_path_for(rows, d_model, ffn_dim, path) == LF_FFN_FUSED) return 0;
    return (size_t)rows * ffn_dim * 2;
}

extern "C" lf_status lf_gelu_ffn_forward(const void* h, const void* W_1, const void* b_1, const void* W_2,
                                         const void* b_2, int rows, int d_model, int ffn_dim, lf_dtype dtype,
                                         int path, void* workspace, size_t workspace_bytes, lf_stream_t stream,
                                         float* z) {
    const void* ptrs[] = {h, W_1, b_1, W_2, b_2, z};
    for (const void* p : ptrs)
        if (!p) return LF_ERR_NULL;
    for (const void* p : ptrs)
        if (!aligned16(p)) return LF_ERR_MISALIGNED;
    if (dtype != LF_F16 && dtype != LF_BF16) return LF_ERR_DTYPE;
    if (rows <= 0 || d_model <= 0 || d_model % 128 != 0 || d_model > 1024 || ffn_dim <= 0 || ffn_dim % 128 != 0)
        return LF_ERR_BAD_DIM;
    if (path < LF_FFN_AUTO || path > LF_FFN_FUSED) return LF_ERR_BAD_DIM;
    if (path == LF_FFN_FUSED && !ffn_fused_supported(rows, d_model, ffn_dim)) return LF_ERR_BAD_DIM;
    const int use = ffn_path_for(rows, d_model, ffn_dim, path);
    if (use == LF_FFN_UNFUSED &&
        (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
         workspace_bytes < (size_t)rows * ffn_dim * 2))
        return LF_ERR_WORKSPACE;
    lf_status st;
    DeviceCtx* d = current_device(&st);
    if (!d) return st;
    return gelu_ffn(h, W_1, b_1, W_2, b_2, rows, d_model, ffn_dim, dtype, use, workspace, z, d, (cudaStream_t)stream);
}

extern "C" lf_status lf_set_ffn_path(int path) {
    if (path < LF_FFN_AUTO || path > LF_FFN_FUSED) return LF_ERR_BAD_DIM;
    g_ffn_path.store(path);
    return LF_OK;
}

extern "C" int lf_get_ffn_path(void) { return g_ffn_path.load(); }

// ---------------------------------------------------------------- the stack

namespace lf {
namespace {

size_t encoder_workspace_bytes(int n_layers, int B, int H, int L, int w, int ffn_dim, lf_dtype dtype, bool any) {
    if (n_layers <= 0) return 0;
    const size_t layer = layer_workspace_bytes(B, H, L, w, ffn_dim, dtype, any);
    if (layer == 0) return 0;
    const size_t act = align256((size_t)B * L * H * 64 * 2);
    return layer + (n_layers > 1 ? 2 * act : 0);
}

// The page's encoder (§Longformer Encoder 计算流程) runs its preprocessing
// once per forward and then the layer loop.  With prefix global tokens every
// layer's attention reads g_b from the mask prefix itself, so the loop is
// the whole forward; with global tokens at any position the partition runs
// once, before the first layer, and every layer reuses its outputs.
lf_status encoder_entry(const void* x, const float* local_mask, const float* global_mask,
                        const lf_layer_weights* layers, int n_layers, int B, int H, int L, int w, float attn_scale,
                        float ln_eps, lf_dtype dtype, void* workspace, size_t workspace_bytes, lf_stream_t stream,
                        void* out, bool any) {
    if (!x || !local_mask || !global_mask || !layers || !out) return LF_ERR_NULL;
    if (n_layers <= 0) return LF_ERR_BAD_DIM;
    const int F = layers[0].ffn_dim;
    lf_status st = check_layer(B, H, L, w, F, dtype);
    if (st != LF_OK) return st;
    // every layer is checked before the first one is launched
    for (int i = 0; i < n_layers; ++i) {
        if (layers[i].ffn_dim != F) return LF_ERR_BAD_DIM;
        if ((st = check_weights(&layers[i])) != LF_OK) return st;
    }
    const void* ptrs[] = {x, local_mask, global_mask, out};
    for (const void* p : ptrs)
        if (!aligned16(p)) return LF_ERR_MISALIGNED;
    const size_t need = encoder_workspace_bytes(n_layers, B, H, L, w, F, dtype, any);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
        return LF_ERR_WORKSPACE;
    DeviceCtx* d = current_device(&st);
    if (!d) return st;
    const Workspace ws = layout(B, H, L, w, F, 2, any);
    uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
    uint8_t* act[2] = {base + ws.total, nullptr};
    act[1] = act[0] + align256((size_t)B * L * H * 64 * 2);
    for (int i = 0; i < n_layers; ++i) {
        const void* in = i == 0 ? x : act[(i - 1) & 1];
        void* o = i == n_layers - 1 ? out : act[i & 1];
        st = layer_forward(in, local_mask, global_mask, &layers[i], B, H, L, w, attn_scale, ln_eps, dtype, base, ws,
                           any, i == 0, d, (cudaStream_t)stream, o);
        if (st != LF_OK) return st;
    }
    return LF_OK;
}

}  // namespace
}  // namespace lf

extern "C" size_t lf_encoder_workspace_bytes(int n_layers, int B, int H, int L, int w, int ffn_dim, lf_dtype dtype) {
    return encoder_workspace_bytes(n_layers, B, H, L, w, ffn_dim, dtype, false);
}

extern "C" lf_status lf_encoder_forward(const void* x, const float* local_mask, const float* global_mask,
                                        const lf_layer_weights* layers, int n_layers, int B, int H, int L, int w,
                                        float attn_scale, float ln_eps, lf_dtype dtype, void* workspace,
                                        size_t workspace_bytes, lf_stream_t stream, void* out) {
    return encoder_entry(x, local_mask, global_mask, layers, n_layers, B, H, L, w, attn_scale, ln_eps, dtype,
                         workspace, workspace_bytes, stream, out, false);
}

extern "C" size_t lf_encoder_any_globals_workspace_bytes(int n_layers, int B, int H, int L, int w, int ffn_dim,
                                                         lf_dtype dtype) {
    return encoder_workspace_bytes(n_layers, B, H, L, w, ffn_dim, dtype, true);
}

extern "C" lf_status lf_encoder_forward_any_globals(const void* x, const float* local_mask, const float* global_mask,
                                                    const lf_layer_weights* layers, int n_layers, int B, int H, int L,
                                                    int w, float attn_scale, float ln_eps, lf_dtype dtype,
                                                    void* workspace, size_t workspace_bytes, lf_stream_t stream,
                                                    void* out) {
    return encoder_entry(x, local_mask, global_mask, layers, n_layers, B, H, L, w, attn_scale, ln_eps, dtype,
                         workspace, workspace_bytes, stream, out, true);
}
