/*
 * Longformer banded + global self-attention: float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header or constant
 * table with the CUDA library.
 *
 * Source of every rule below ("FTL" = the page "FasterTransformer Longformer
 * 推理加速实践：PyTorch 集成、输入约束与端到端性能解析"):
 *   - FTL §使用前提：四条硬性约束 (input constraints 1-4): L % w == 0,
 *     L >= 2w, head size 64, number of global tokens <= w, global tokens
 *     contiguous at the start of the sequence.
 *   - FTL §Longformer Encoder 计算流程 (input list): local_attn_mask 1.0 =
 *     attend / 0.0 = padding; global_attn_mask 0.0 = global token, -10000.0
 *     = non-global.
 *   - FTL §计算流程 / 预处理, invokeInitLongformerIdx: the per-sample global
 *     index partition (flagged partition of positions by global_attn_mask).
 *   - FTL §计算流程 / 预处理, invokeLocalAttnMaskShift: additive key bias
 *     fma(local_mask, 10000, -10000).
 *   - FTL §计算流程 / 每个 Transformer 层, step 4 (longformerMHASoftmax):
 *     a local row normalises over its window and the global tokens; a global
 *     row normalises over the whole sequence; a row whose shifted mask is
 *     non-zero is zeroed.
 *   - FTL §计算流程 / 每个 Transformer 层, steps 1-3: global rows use their
 *     own qg/kg/vg projections.
 *
 * Readings where the page is silent (each listed in the design notes):
 *   - w is one-sided: row i's window is |i - j| <= w (2w+1 keys).
 *   - A local row's key set is the SET union of its window and the global
 *     tokens: a global token inside the window is counted once.
 *   - Local rows use the regular k/v for global columns; only global rows
 *     use qg/kg/vg.
 *   - global_attn_mask[j] is added to the score on global columns of local
 *     rows only (it is 0.0 there); band columns and global rows get the
 *     padding bias alone.
 *   - scale = 1/sqrt(64) = 0.125.
 *   - The partition's output order is that of a stable flagged partition:
 *     selected indices ascending at the front, rejected ones in reverse
 *     order at the back.
 *   - Global tokens at any position (the "_any" entry points): FTL
 *     §使用前提 item 4 names placing global tokens anywhere as the
 *     HuggingFace behaviour that FT does not support.  There the global set
 *     is G_b = { j : global_mask[b, j] == 0.0 } wherever its members lie; a
 *     row i in G_b is a global row (qg/kg/vg over the whole sequence), any
 *     other row attends its window united with all of G_b, each key once.
 *     Constraint 3 (g_b <= w) is kept.  With G_b a prefix this is exactly
 *     the prefix definition above.
 *
 * Arithmetic: IEEE double throughout, no fast-math; exp() from libm.  The
 * bias is formed in float with fmaf exactly as the page writes it, then
 * widened (it is exactly 0 or -10000 for 0/1 masks).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define LFO_D 64

/* Status codes: numerically the same values the library documents, written
 * out here independently. */
enum {
    LFO_OK = 0,
    LFO_ERR_BAD_DIM = 2,
    LFO_ERR_L_NOT_MULTIPLE_OF_W = 3,
    LFO_ERR_L_LT_2W = 4,
    LFO_ERR_G_GT_W = 5,
    LFO_ERR_GLOBAL_NOT_PREFIX = 6
};

int lfo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Shape constraints, FTL §使用前提 items 1-2 (head size is fixed at 64). */
int lfo_check_shape(int B, int H, int L, int w)
{
    if (B <= 0 || H <= 0 || L <= 0 || w <= 0) return LFO_ERR_BAD_DIM;
    if (L % w != 0) return LFO_ERR_L_NOT_MULTIPLE_OF_W;
    if (L < 2 * w) return LFO_ERR_L_LT_2W;
    return LFO_OK;
}

/* The set G_b of global positions of sample b is { j : global_mask == 0.0 }
 * (FTL input list).  Constraint 4 requires G_b == {0..g_b-1} (checked
 * unless any_pos), constraint 3 g_b <= w.  Returns the status and writes
 * g_b. */
static int global_count(const float* gm_row, int L, int w, int any_pos, int* g_out)
{
    int g = 0;
    for (int j = 0; j < L; ++j)
        if (gm_row[j] == 0.0f) ++g;
    if (!any_pos)
        for (int j = 0; j < g; ++j)
            if (gm_row[j] != 0.0f) return LFO_ERR_GLOBAL_NOT_PREFIX;
    *g_out = g;
    if (g > w) return LFO_ERR_G_GT_W;
    return LFO_OK;
}

/* invokeInitLongformerIdx (FTL §计算流程 / 预处理): flagged partition of the
 * positions 0..L-1 of each sample by the flag global_mask == 0.0.
 * global_idx[b, 0..g_b-1] = flagged positions in ascending order;
 * global_idx[b, g_b..L-1] = unflagged positions in descending order;
 * global_token_nums[b] = g_b.  The outputs are written even when the
 * constraints fail; the first failing sample's status is returned. */
static int global_partition(const float* global_mask, int B, int L, int w, int any_pos,
                            int32_t* global_idx, int32_t* global_token_nums)
{
    int status = LFO_OK;
    for (int b = 0; b < B; ++b) {
        const float* row = global_mask + (size_t)b * L;
        int32_t* idx = global_idx + (size_t)b * L;
        int front = 0, back = L - 1;
        for (int j = 0; j < L; ++j) {
            if (row[j] == 0.0f) idx[front++] = j;
            else idx[back--] = j;
        }
        global_token_nums[b] = front;
        int g;
        int st = global_count(row, L, w, any_pos, &g);
        if (st != LFO_OK && status == LFO_OK) status = st;
    }
    return status;
}

int lfo_global_partition(const float* global_mask, int B, int L, int w,
                         int32_t* global_idx, int32_t* global_token_nums)
{
    return global_partition(global_mask, B, L, w, 0, global_idx, global_token_nums);
}

/* The same partition with the global tokens at any position (only g_b <= w
 * is checked). */
int lfo_global_partition_any(const float* global_mask, int B, int L, int w,
                             int32_t* global_idx, int32_t* global_token_nums)
{
    return global_partition(global_mask, B, L, w, 1, global_idx, global_token_nums);
}

/* Shifted local mask, invokeLocalAttnMaskShift (FTL §计算流程 / 预处理). */
static double local_bias(float m)
{
    return (double)fmaf(m, 10000.0f, -10000.0f);
}

static double dot64(const double* a, const double* b)
{
    double s = 0.0;
    for (int c = 0; c < LFO_D; ++c) s += a[c] * b[c];
    return s;
}

typedef struct {
    const double *q, *k, *v, *qg, *kg, *vg; /* [B,H,L,64] */
    const float *local_mask, *global_mask;  /* [B,L] */
    const int* g;                            /* per-sample global count */
    const int* gpos;                         /* [B][L]: sample b's global positions, ascending */
    int B, H, L, w;
    double scale;
    int any_pos;                             /* global tokens may lie anywhere */
} lfo_ctx;

/* One output row out[b, i, h, :] of the attention layer.
 *   e_j = scale * <q_i, k_j> + lb[j] (+ global_mask[j] on global columns)
 *   p_j = exp(e_j - max e) / sum exp(e - max e)   over the row's key set
 *   out = sum_j p_j * v_j
 * Key set: local row i (not in G_b) -> window [max(0,i-w), min(L-1,i+w)]
 * united with the global positions G_b; global row i in G_b -> all of
 * [0, L) with qg/kg/vg.  (G_b = [0, g_b) unless any_pos.)  A row with
 * lb[i] != 0 is zero. */
static void attention_row(const lfo_ctx* c, int b, int h, int i, double* o,
                          double* e /* scratch [L] */, int* keys /* scratch [L] */)
{
    const int L = c->L, w = c->w, g = c->g[b];
    const float* lm = c->local_mask + (size_t)b * L;
    const float* gm = c->global_mask + (size_t)b * L;
    const size_t head = ((size_t)b * c->H + h) * (size_t)L * LFO_D;

    for (int d = 0; d < LFO_D; ++d) o[d] = 0.0;
    if (local_bias(lm[i]) != 0.0) return; /* padded query row: zero */

    const int* G = c->gpos + (size_t)b * L; /* G[0..g) */
    const int global_row = gm[i] == 0.0f;
    const double* qi = (global_row ? c->qg : c->q) + head + (size_t)i * LFO_D;
    const double* K = (global_row ? c->kg : c->k) + head;
    const double* V = (global_row ? c->vg : c->v) + head;

    /* Build the key set, each key once. */
    int n = 0;
    if (global_row) {
        for (int j = 0; j < L; ++j) keys[n++] = j;
    } else {
        int lo = i - w < 0 ? 0 : i - w;
        int hi = i + w > L - 1 ? L - 1 : i + w;
        for (int t = 0; t < g; ++t) keys[n++] = G[t];          /* global tokens */
        for (int j = lo; j <= hi; ++j)                         /* window minus globals */
            if (gm[j] != 0.0f) keys[n++] = j;
    }

    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
        int j = keys[t];
        double s = c->scale * dot64(qi, K + (size_t)j * LFO_D) + local_bias(lm[j]);
        if (!global_row && t < g) s += (double)gm[j];          /* global column */
        e[t] = s;
        if (s > m) m = s;
    }
    double sum = 0.0;
    for (int t = 0; t < n; ++t) {
        e[t] = exp(e[t] - m);
        sum += e[t];
    }
    for (int t = 0; t < n; ++t) {
        const double* vj = V + (size_t)keys[t] * LFO_D;
        double p = e[t] / sum;
        for (int d = 0; d < LFO_D; ++d) o[d] += p * vj[d];
    }
}

/* Per-sample global counts and position lists (gpos: [B][L]). */
static int prepare(lfo_ctx* c, int* g, int* gpos)
{
    int st = lfo_check_shape(c->B, c->H, c->L, c->w);
    if (st != LFO_OK) return st;
    for (int b = 0; b < c->B; ++b) {
        const float* row = c->global_mask + (size_t)b * c->L;
        st = global_count(row, c->L, c->w, c->any_pos, &g[b]);
        if (st != LFO_OK) return st;
        int n = 0;
        for (int j = 0; j < c->L; ++j)
            if (row[j] == 0.0f) gpos[(size_t)b * c->L + n++] = j;
    }
    c->g = g;
    c->gpos = gpos;
    return LFO_OK;
}

/* Full attention layer: out[B, L, H, 64] (the multi-head-to-single layout of
 * FTL step 5).  Returns a status; out is untouched on error. */
static int attention_all(const double* q, const double* k, const double* v,
                         const double* qg, const double* kg, const double* vg,
                         const float* local_mask, const float* global_mask,
                         int B, int H, int L, int w, double scale, int any_pos, double* out)
{
    lfo_ctx c = {q, k, v, qg, kg, vg, local_mask, global_mask, NULL, NULL, B, H, L, w, scale, any_pos};
    int* g = (int*)malloc(sizeof(int) * (size_t)(B > 0 ? B : 1));
    int* gpos = (int*)malloc(sizeof(int) * (size_t)(B > 0 ? B : 1) * (size_t)(L > 0 ? L : 1));
    int st = prepare(&c, g, gpos);
    if (st == LFO_OK) {
        long long total = (long long)B * H * L;
#pragma omp parallel
        {
            double* e = (double*)malloc(sizeof(double) * (size_t)L);
            int* keys = (int*)malloc(sizeof(int) * (size_t)L);
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < total; ++r) {
                int i = (int)(r % L);
                int h = (int)((r / L) % H);
                int b = (int)(r / ((long long)L * H));
                attention_row(&c, b, h, i, out + (((size_t)b * L + i) * H + h) * LFO_D, e, keys);
            }
            free(e);
            free(keys);
        }
    }
    free(g);
    free(gpos);
    return st;
}

int lfo_attention(const double* q, const double* k, const double* v,
                  const double* qg, const double* kg, const double* vg,
                  const float* local_mask, const float* global_mask,
                  int B, int H, int L, int w, double scale, double* out)
{
    return attention_all(q, k, v, qg, kg, vg, local_mask, global_mask, B, H, L, w, scale, 0, out);
}

/* Global tokens at any position. */
int lfo_attention_any(const double* q, const double* k, const double* v,
                      const double* qg, const double* kg, const double* vg,
                      const float* local_mask, const float* global_mask,
                      int B, int H, int L, int w, double scale, double* out)
{
    return attention_all(q, k, v, qg, kg, vg, local_mask, global_mask, B, H, L, w, scale, 1, out);
}

/* Selected rows only: rows[3*r .. 3*r+2] = (b, h, i); out_rows[r, 64]. */
int lfo_attention_rows(const double* q, const double* k, const double* v,
                       const double* qg, const double* kg, const double* vg,
                       const float* local_mask, const float* global_mask,
                       int B, int H, int L, int w, double scale, int any_pos,
                       const int32_t* rows, long long n_rows, double* out_rows)
{
    lfo_ctx c = {q, k, v, qg, kg, vg, local_mask, global_mask, NULL, NULL, B, H, L, w, scale, any_pos};
    int* g = (int*)malloc(sizeof(int) * (size_t)(B > 0 ? B : 1));
    int* gpos = (int*)malloc(sizeof(int) * (size_t)(B > 0 ? B : 1) * (size_t)(L > 0 ? L : 1));
    int st = prepare(&c, g, gpos);
    if (st == LFO_OK) {
#pragma omp parallel
        {
            double* e = (double*)malloc(sizeof(double) * (size_t)L);
            int* keys = (int*)malloc(sizeof(int) * (size_t)L);
#pragma omp for schedule(dynamic, 4)
            for (long long r = 0; r < n_rows; ++r)
                attention_row(&c, rows[3 * r], rows[3 * r + 1], rows[3 * r + 2],
                              out_rows + (size_t)r * LFO_D, e, keys);
            free(e);
            free(keys);
        }
    }
    free(g);
    free(gpos);
    return st;
}
