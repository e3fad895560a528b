/*
 * oracle.c - plain CPU oracle of the llama2.c single-token decode step.
 *
 * TEST INFRASTRUCTURE ONLY: the reference that the GPU library is checked
 * against.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg load it.  It shares no code with the GPU library.
 *
 * Sources (web pages about karpathy's llama2.c; cited by title and section):
 *   [hub]   "Llama 2 in Pure C: 一个周末Hack的AI奇迹" (pomoai.com llama2.c hub),
 *           sections 架构实现 (architecture list), 数据格式 (file format),
 *           量化支持 (Q8_0).
 *   [news]  "技术深度解析" (ainews.cool llama2.c article): plain nested-loop
 *           matmul, no allocation during inference.
 *   [port]  "超精简LLM部署：llama2.c嵌入式移植全攻略" (blog.gitcode.com),
 *           §1 INT8量化压缩 (the quantize() listing), §2 内存优化策略 (KV cache
 *           allocation), 智能家居控制案例 (forward + sample_argmax usage).
 *   [qa]    "Karpathy 技術學習庫 - Q&A 問答集", 技術細節: KV Cache 在 C 中如何
 *           管理, 為什麼 QKV 的維度不同 (GQA), RoPE 在 C 中的實作, 跳過
 *           freq_cis, shared_weights 參數的作用; 效能相關: 13B+ overflow.
 *   [essay] "LLM底层原理与工程实践：从参数文件到C语言推理" (m.mht18.com),
 *           §3.2 (sampling with a temperature after the logits).
 *
 * Readings where the pages are silent (each repeated where it is used):
 *   RMSNorm eps = 1e-5 inside the square root; RoPE base 10000 on adjacent
 *   pairs within each head, freq = 1/10000^(j/hs) for even j; attention scale
 *   1/sqrt(hs) over positions 0..pos inclusive; query head i uses KV head
 *   i / (n_heads/n_kv_heads); SwiGLU = silu(W1 x) * (W3 x); Q8_0 covers every
 *   matvec weight and the embedding table, and every matvec input is
 *   quantized at the same group size; an all-zero group has scale 0, codes 0;
 *   Q4_0 is the same rule with codes in [-7, 7] (scale = max|x| / 7) on the
 *   same tensors, its matvec inputs still Q8_0.
 *
 * Arithmetic: fp32 storage; sums in double, rounded to fp32 once per step
 * (orc_set_fp32_accum(1) gives the pages' fp32 loops instead).  Every offset
 * is 64-bit: the Q&A page traces llama2.c's 13B failure to int overflow in
 * pointer arithmetic.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

static int g_fp32 = 0;
void orc_set_fp32_accum(int on) { g_fp32 = on ? 1 : 0; }

#define RMS_EPS 1e-5

/* RMSNorm [hub §架构实现 names it; the formula is the Llama-2 one]:
 * o = w * x / sqrt(mean(x^2) + eps). */
void orc_rmsnorm(float* o, const float* x, const float* w, int n) {
    if (g_fp32) {
        float ss = 0.0f;
        for (int j = 0; j < n; j++) ss += x[j] * x[j];
        ss /= (float)n;
        ss += 1e-5f;
        ss = 1.0f / sqrtf(ss);
        for (int j = 0; j < n; j++) o[j] = w[j] * (ss * x[j]);
        return;
    }
    double ss = 0.0;
    for (int j = 0; j < n; j++) ss += (double)x[j] * (double)x[j];
    double inv = 1.0 / sqrt(ss / (double)n + RMS_EPS);
    for (int j = 0; j < n; j++) o[j] = (float)((double)w[j] * (inv * (double)x[j]));
}

/* matvec [news §技术深度解析: hand-written nested loops, no BLAS]:
 * o[i] = sum_j W[i][j] * x[j], W row-major [d][n].  Rows run in parallel
 * (the pages' runomp build); each row's sum is sequential. */
void orc_matvec(float* o, const float* x, const float* W, int n, int d) {
    #pragma omp parallel for schedule(static)
    for (int i = 0; i < d; i++) {
        const float* row = W + (size_t)i * (size_t)n;
        if (g_fp32) {
            float v = 0.0f;
            for (int j = 0; j < n; j++) v += row[j] * x[j];
            o[i] = v;
        } else {
            double v = 0.0;
            for (int j = 0; j < n; j++) v += (double)row[j] * (double)x[j];
            o[i] = (float)v;
        }
    }
}

/* RoPE frequency of the pair starting at even in-head index j:
 * 1 / 10000^(j / hs), evaluated in fp32 as llama2.c does. */
float orc_rope_freq(int j, int head_size) {
    return 1.0f / powf(10000.0f, (float)j / (float)head_size);
}

/* RoPE on the fly [qa §RoPE 在 C 中的實作: the C code evaluates
 * cosf(pos*freq) and sinf(pos*freq) during forward instead of a table]:
 * every adjacent pair (v[i], v[i+1]), i even, is rotated by
 * theta = (float)pos * freq(i mod hs).  The angle is the pages' fp32
 * product; its cosine and sine are taken in double (nearer the exact
 * rotation than cosf/sinf, which the fp32 mode uses). */
void orc_rope(float* v, int n, int head_size, int pos) {
    for (int i = 0; i < n; i += 2) {
        float freq = orc_rope_freq(i % head_size, head_size);
        float theta = (float)pos * freq;
        double c, s;
        if (g_fp32) { c = (double)cosf(theta); s = (double)sinf(theta); }
        else { c = cos((double)theta); s = sin((double)theta); }
        double a = (double)v[i], b = (double)v[i + 1];
        v[i] = (float)(a * c - b * s);
        v[i + 1] = (float)(a * s + b * c);
    }
}

/* softmax over x[0..n) in place: subtract the max, exponentiate, normalise. */
void orc_softmax(double* x, int n) {
    double mx = x[0];
    for (int i = 1; i < n; i++) if (x[i] > mx) mx = x[i];
    double sum = 0.0;
    for (int i = 0; i < n; i++) { x[i] = exp(x[i] - mx); sum += x[i]; }
    for (int i = 0; i < n; i++) x[i] /= sum;
}

static void orc_softmax_f32(float* x, int n) {
    float mx = x[0];
    for (int i = 1; i < n; i++) if (x[i] > mx) mx = x[i];
    float sum = 0.0f;
    for (int i = 0; i < n; i++) { x[i] = expf(x[i] - mx); sum += x[i]; }
    for (int i = 0; i < n; i++) x[i] /= sum;
}

/* Grouped-query attention for one layer [qa §GQA: q has n_heads*hs values,
 * k and v have n_kv_heads*hs; several query heads share one KV head;
 * qa §KV Cache: positions 0..pos of the cache are attended].
 * kc, vc: this layer's caches, [positions][kv_dim].  out: [n_heads*hs]. */
void orc_attention(float* out, const float* q, const float* kc, const float* vc, int pos,
                   int n_heads, int n_kv_heads, int head_size) {
    int kv_dim = n_kv_heads * head_size;
    int rep = n_heads / n_kv_heads;
    int T = pos + 1;
    #pragma omp parallel for schedule(static)
    for (int h = 0; h < n_heads; h++) {
        int g = h / rep;
        const float* qh = q + (size_t)h * head_size;
        float* oh = out + (size_t)h * head_size;
        if (g_fp32) {
            float* att = (float*)malloc(sizeof(float) * (size_t)T);
            for (int t = 0; t < T; t++) {
                const float* kt = kc + (size_t)t * kv_dim + (size_t)g * head_size;
                float s = 0.0f;
                for (int i = 0; i < head_size; i++) s += qh[i] * kt[i];
                att[t] = s / sqrtf((float)head_size);
            }
            orc_softmax_f32(att, T);
            for (int i = 0; i < head_size; i++) oh[i] = 0.0f;
            for (int t = 0; t < T; t++) {
                const float* vt = vc + (size_t)t * kv_dim + (size_t)g * head_size;
                for (int i = 0; i < head_size; i++) oh[i] += att[t] * vt[i];
            }
            free(att);
            continue;
        }
        double* att = (double*)malloc(sizeof(double) * (size_t)T);
        double scale = 1.0 / sqrt((double)head_size);
        for (int t = 0; t < T; t++) {
            const float* kt = kc + (size_t)t * kv_dim + (size_t)g * head_size;
            double s = 0.0;
            for (int i = 0; i < head_size; i++) s += (double)qh[i] * (double)kt[i];
            att[t] = s * scale;
        }
        orc_softmax(att, T);
        for (int i = 0; i < head_size; i++) {
            double acc = 0.0;
            for (int t = 0; t < T; t++)
                acc += att[t] * (double)vc[(size_t)t * kv_dim + (size_t)g * head_size + i];
            oh[i] = (float)acc;
        }
        free(att);
    }
}

/* SwiGLU [hub §架构实现 names it]: silu(z) = z / (1 + e^-z). */
double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* hb[i] = silu(hb[i]) * hb2[i], where hb = W1 x and hb2 = W3 x. */
void orc_swiglu(float* hb, const float* hb2, int n) {
    for (int i = 0; i < n; i++) {
        if (g_fp32) {
            float z = hb[i];
            hb[i] = z * (1.0f / (1.0f + expf(-z))) * hb2[i];
        } else {
            hb[i] = (float)(orc_silu((double)hb[i]) * (double)hb2[i]);
        }
    }
}

/* Quantize [port §1 INT8量化压缩, the quantize() listing] with the largest
 * code qmax as a parameter: for each group of gs consecutive values,
 * wmax = max|x|, scale = wmax / qmax (fp32), q = (int8) round(x / scale) with
 * the quotient in fp32 and C round() (half away from zero).  Reading where
 * the listing divides 0 by 0: a group whose wmax is 0 gets scale 0 and all
 * codes 0.  Returns -1 if n % gs != 0. */
static int orc_quantize_qmax(const float* x, int64_t n, int gs, float qmax, int8_t* q, float* s) {
    if (gs <= 0 || n % gs != 0) return -1;
    int64_t ng = n / gs;
    #pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < ng; g++) {
        const float* xg = x + g * gs;
        float wmax = 0.0f;
        for (int i = 0; i < gs; i++) {
            float val = fabsf(xg[i]);
            if (val > wmax) wmax = val;
        }
        float scale = wmax / qmax;
        s[g] = scale;
        for (int i = 0; i < gs; i++) {
            if (scale == 0.0f) { q[g * gs + i] = 0; continue; }
            float quot = xg[i] / scale;
            q[g * gs + i] = (int8_t)round((double)quot);
        }
    }
    return 0;
}

/* Q8_0 [port §1, the quantize() listing]: qmax = 127. */
int orc_quantize(const float* x, int64_t n, int gs, int8_t* q, float* s) {
    return orc_quantize_qmax(x, n, gs, 127.0f, q, s);
}

/* Q4_0 [news 技术深度解析, the 整数量化路径 item: runq.c with 4-bit integer
 * groups, "like llama.cpp's"; the page gives no rule].  Reading: the Q8_0
 * rule above with 4-bit codes, qmax = 7: scale = wmax / 7 in fp32, codes
 * round(x / scale) in [-7, 7], one fp32 scale per group of gs. */
int orc_quantize4(const float* x, int64_t n, int gs, int8_t* q, float* s) {
    return orc_quantize_qmax(x, n, gs, 7.0f, q, s);
}

/* x ~= q * scale of its group, one fp32 multiply per element. */
void orc_dequantize(const int8_t* q, const float* s, int64_t n, int gs, float* out) {
    for (int64_t i = 0; i < n; i++) out[i] = (float)q[i] * s[i / gs];
}

/* A KV row of n values in place: quantize() in groups of gs, then code * scale. */
void orc_kv8_row(float* row, int n, int gs) {
    int8_t* q = (int8_t*)malloc((size_t)n);
    float* sc = (float*)malloc(sizeof(float) * (size_t)(n / gs + 1));
    if (q && sc && orc_quantize(row, n, gs, q, sc) == 0) orc_dequantize(q, sc, n, gs, row);
    free(q);
    free(sc);
}

/* Exact int32 dot products of every (row, group):
 * out[i][g] = sum_{k<gs} qw[i][g*gs+k] * qx[g*gs+k].  qw is [d][n]. */
void orc_q80_group_dots(int32_t* out, const int8_t* qx, const int8_t* qw, int n, int d, int gs) {
    int ng = n / gs;
    for (int i = 0; i < d; i++) {
        const int8_t* row = qw + (size_t)i * (size_t)n;
        for (int g = 0; g < ng; g++) {
            int32_t acc = 0;
            for (int k = 0; k < gs; k++) acc += (int32_t)row[g * gs + k] * (int32_t)qx[g * gs + k];
            out[(size_t)i * ng + g] = acc;
        }
    }
}

/* Q8_0 matvec: o[i] = sum_g ival(i,g) * sw[i][g] * sx[g] with ival the exact
 * int32 group dot; the sum over groups is double here (fp32 under
 * orc_set_fp32_accum(1), as runq.c does it). */
void orc_matvec_q80(float* o, const int8_t* qx, const float* sx, const int8_t* qw, const float* sw,
                    int n, int d, int gs) {
    int ng = n / gs;
    #pragma omp parallel for schedule(static)
    for (int i = 0; i < d; i++) {
        const int8_t* row = qw + (size_t)i * (size_t)n;
        const float* srow = sw + (size_t)i * (size_t)ng;
        double vd = 0.0;
        float vf = 0.0f;
        for (int g = 0; g < ng; g++) {
            int32_t ival = 0;
            for (int k = 0; k < gs; k++) ival += (int32_t)row[g * gs + k] * (int32_t)qx[g * gs + k];
            if (g_fp32) vf += ((float)ival) * srow[g] * sx[g];
            else vd += (double)ival * (double)srow[g] * (double)sx[g];
        }
        o[i] = g_fp32 ? vf : (float)vd;
    }
}

/* sample_argmax [port 智能家居控制案例]: the index of the largest value,
 * the lowest index among equal maxima. */
int orc_argmax(const float* x, int n) {
    int best = 0;
    for (int i = 1; i < n; i++) if (x[i] > x[best]) best = i;
    return best;
}

static int cmp_desc(const void* a, const void* b) {
    const double x = *(const double*)a, y = *(const double*)b;
    return x < y ? 1 : (x > y ? -1 : 0);
}

/* Sampling after the logits [essay §3.2: a temperature divides the logits
 * before the softmax; port 智能家居控制案例: the greedy sample_argmax].  The
 * pages give no more, so the reading taken is:
 *   temperature == 0: the greedy argmax.
 *   otherwise weights q_i = exp((z_i - max z) / T) in double (the softmax
 *   up to its normalisation Z = sum q_i);
 *   topp < 1 restricts the draw to the smallest set of most probable tokens
 *   whose weight reaches topp * Z (every token tied with the last one taken
 *   is in the set): tau = the weight at which the running sum, over the
 *   weights sorted in decreasing order, first reaches topp * Z, and the set
 *   is {i : q_i >= tau};
 *   the draw uses the caller's coin u in [0, 1): the first index i, in index
 *   order, of the set at which the running sum of the set's weights exceeds
 *   u * Z_set (the last index of the set if rounding leaves none). */
int orc_sample(const float* z, int n, float temperature, float topp, double coin) {
    if (n <= 0) return -1;
    if (temperature == 0.0f) return orc_argmax(z, n);
    float mx = z[0];
    for (int i = 1; i < n; i++) if (z[i] > mx) mx = z[i];
    double* q = (double*)malloc(sizeof(double) * (size_t)n);
    double Z = 0.0;
    for (int i = 0; i < n; i++) {
        q[i] = exp(((double)z[i] - (double)mx) / (double)temperature);
        Z += q[i];
    }
    double tau = 0.0;
    if (topp < 1.0f) {
        double* sorted = (double*)malloc(sizeof(double) * (size_t)n);
        memcpy(sorted, q, sizeof(double) * (size_t)n);
        qsort(sorted, (size_t)n, sizeof(double), cmp_desc);
        const double target = (double)topp * Z;
        double cum = 0.0;
        tau = sorted[n - 1];
        for (int k = 0; k < n; k++) {
            cum += sorted[k];
            if (cum >= target) {
                tau = sorted[k];
                break;
            }
        }
        free(sorted);
    }
    double zset = 0.0;
    for (int i = 0; i < n; i++) if (q[i] >= tau) zset += q[i];
    const double target = coin * zset;
    double cum = 0.0;
    int last = -1, pick = -1;
    for (int i = 0; i < n && pick < 0; i++) {
        if (q[i] < tau) continue;
        cum += q[i];
        last = i;
        if (cum > target) pick = i;
    }
    free(q);
    return pick >= 0 ? pick : last;
}

/* ---------------------------------------------------------------- model -- */

typedef struct { int8_t* q; float* s; } orc_qt;

/* One quantized copy of the weights: every matvec weight and the embedding
 * table in groups of gs (gs = 0: not made). */
typedef struct {
    int gs;
    orc_qt E, wq, wk, wv, wo, w1, w2, w3, wcls;
} orc_qset;

struct orc_model {
    orc_config c;
    int shared, n_seq;
    int kv8; /* 1: the KV cache holds Q8_0 rows (see orc_enable_kv8) */
    const float *E, *w_att, *wq, *wk, *wv, *wo, *w_ffn, *w1, *w2, *w3, *w_final, *wcls;
    orc_qset q8, q4; /* Q8_0 (orc_enable_q80) and Q4_0 (orc_enable_q40) */
    float *kcache, *vcache; /* [n_seq][L][S][kv_dim] */
    float *x, *xb, *xb2, *hb, *hb2, *q;
    int8_t* aq; /* activation codes, max(dim, hidden) */
    float* as;  /* activation scales */
};

/* Blob size: the tensors in llama2.c's checkpoint order [hub §数据格式: a
 * config header then contiguous fp32 arrays; qa §跳過 freq_cis: two legacy
 * RoPE tables of seq_len*hs/2 floats each sit before the classifier; qa
 * §shared_weights: a separate classifier follows only when untied]. */
size_t orc_blob_floats(const orc_config* c, int shared_weights) {
    size_t d = (size_t)c->dim, h = (size_t)c->hidden_dim, L = (size_t)c->n_layers;
    size_t hs = d / (size_t)c->n_heads, kvd = (size_t)c->n_kv_heads * hs;
    size_t V = (size_t)c->vocab_size, S = (size_t)c->seq_len;
    size_t n = V * d + L * d + 2 * L * d * d + 2 * L * kvd * d + L * d + 3 * L * h * d + d + S * hs;
    return shared_weights ? n : n + V * d;
}

static int orc_config_ok(const orc_config* c) {
    if (c->dim <= 0 || c->hidden_dim <= 0 || c->n_layers <= 0 || c->n_heads <= 0 ||
        c->n_kv_heads <= 0 || c->vocab_size <= 0 || c->seq_len <= 0) return 0;
    if (c->dim % c->n_heads != 0 || c->n_heads % c->n_kv_heads != 0) return 0;
    if ((c->dim / c->n_heads) % 2 != 0) return 0;
    return 1;
}

orc_model* orc_create(const orc_config* c, const float* blob, size_t blob_floats, int shared_weights,
                      int n_seq) {
    if (!c || !blob || !orc_config_ok(c) || n_seq <= 0) return NULL;
    if (blob_floats != orc_blob_floats(c, shared_weights)) return NULL;
    orc_model* m = (orc_model*)calloc(1, sizeof(orc_model));
    if (!m) return NULL;
    m->c = *c;
    m->shared = shared_weights ? 1 : 0;
    m->n_seq = n_seq;
    size_t d = (size_t)c->dim, h = (size_t)c->hidden_dim, L = (size_t)c->n_layers;
    size_t hs = d / (size_t)c->n_heads, kvd = (size_t)c->n_kv_heads * hs;
    size_t V = (size_t)c->vocab_size, S = (size_t)c->seq_len;
    const float* p = blob;
    m->E = p; p += V * d;
    m->w_att = p; p += L * d;
    m->wq = p; p += L * d * d;
    m->wk = p; p += L * kvd * d;
    m->wv = p; p += L * kvd * d;
    m->wo = p; p += L * d * d;
    m->w_ffn = p; p += L * d;
    m->w1 = p; p += L * h * d;
    m->w2 = p; p += L * d * h;
    m->w3 = p; p += L * h * d;
    m->w_final = p; p += d;
    p += S * hs / 2; /* legacy freq_cis_real */
    p += S * hs / 2; /* legacy freq_cis_imag */
    m->wcls = m->shared ? m->E : p;
    size_t cache = (size_t)n_seq * L * S * kvd;
    m->kcache = (float*)calloc(cache, sizeof(float));
    m->vcache = (float*)calloc(cache, sizeof(float));
    size_t mx = d > h ? d : h;
    m->x = (float*)calloc(d, sizeof(float));
    m->xb = (float*)calloc(d, sizeof(float));
    m->xb2 = (float*)calloc(d, sizeof(float));
    m->hb = (float*)calloc(h, sizeof(float));
    m->hb2 = (float*)calloc(h, sizeof(float));
    m->q = (float*)calloc(d, sizeof(float));
    m->aq = (int8_t*)calloc(mx, 1);
    m->as = (float*)calloc(mx, sizeof(float));
    if (!m->kcache || !m->vcache || !m->x || !m->xb || !m->xb2 || !m->hb || !m->hb2 || !m->q ||
        !m->aq || !m->as) {
        orc_destroy(m);
        return NULL;
    }
    return m;
}

static int orc_qt_make(orc_qt* t, const float* w, size_t n, int gs, int four) {
    t->q = (int8_t*)malloc(n);
    t->s = (float*)malloc(sizeof(float) * (n / (size_t)gs));
    if (!t->q || !t->s) return -1;
    return four ? orc_quantize4(w, (int64_t)n, gs, t->q, t->s) : orc_quantize(w, (int64_t)n, gs, t->q, t->s);
}

static void orc_qt_free(orc_qt* t) { free(t->q); free(t->s); t->q = NULL; t->s = NULL; }

static void orc_qset_free(orc_qset* z, int shared) {
    orc_qt_free(&z->E);
    orc_qt_free(&z->wq); orc_qt_free(&z->wk); orc_qt_free(&z->wv); orc_qt_free(&z->wo);
    orc_qt_free(&z->w1); orc_qt_free(&z->w2); orc_qt_free(&z->w3);
    if (!shared) orc_qt_free(&z->wcls);
    z->gs = 0;
}

/* Quantizes every matvec weight and the embedding table with group size gs
 * (groups run along the flattened tensor, which is along rows since every
 * input width is a multiple of gs), Q8_0 codes or (four = 1) Q4_0 codes.  A
 * tied classifier shares E's codes. */
static int orc_qset_make(orc_model* m, orc_qset* z, int gs, int four) {
    const orc_config* c = &m->c;
    size_t d = (size_t)c->dim, h = (size_t)c->hidden_dim, L = (size_t)c->n_layers;
    size_t hs = d / (size_t)c->n_heads, kvd = (size_t)c->n_kv_heads * hs, V = (size_t)c->vocab_size;
    if (gs <= 0 || d % (size_t)gs || h % (size_t)gs) return -1;
    if (z->gs) return z->gs == gs ? 0 : -1;
    int rc = 0;
    rc |= orc_qt_make(&z->E, m->E, V * d, gs, four);
    rc |= orc_qt_make(&z->wq, m->wq, L * d * d, gs, four);
    rc |= orc_qt_make(&z->wk, m->wk, L * kvd * d, gs, four);
    rc |= orc_qt_make(&z->wv, m->wv, L * kvd * d, gs, four);
    rc |= orc_qt_make(&z->wo, m->wo, L * d * d, gs, four);
    rc |= orc_qt_make(&z->w1, m->w1, L * h * d, gs, four);
    rc |= orc_qt_make(&z->w2, m->w2, L * d * h, gs, four);
    rc |= orc_qt_make(&z->w3, m->w3, L * h * d, gs, four);
    if (m->shared) z->wcls = z->E;
    else rc |= orc_qt_make(&z->wcls, m->wcls, V * d, gs, four);
    if (rc) {
        z->gs = 1; /* any nonzero: free what was made */
        orc_qset_free(z, m->shared);
        return -1;
    }
    z->gs = gs;
    return 0;
}

/* Q8_0 weights [port §1; hub §量化支持]. */
int orc_enable_q80(orc_model* m, int gs) { return orc_qset_make(m, &m->q8, gs, 0); }

/* Q4_0 weights [news 技术深度解析, 整数量化路径] (the reading of orc_quantize4);
 * the inputs of their matvecs are Q8_0 at the same group size, as in the
 * Q8_0 step. */
int orc_enable_q40(orc_model* m, int gs) { return orc_qset_make(m, &m->q4, gs, 1); }

/* matvec through a quantized set: quantize the input to Q8_0 at the set's
 * group size, then the exact-int32 group matvec on layer l of a stacked
 * [L][d][n] tensor. */
static void orc_qmatvec(orc_model* m, const orc_qset* z, float* o, const float* x, const orc_qt* t, size_t l, int n,
                        int d) {
    int gs = z->gs;
    orc_quantize(x, n, gs, m->aq, m->as);
    size_t off = l * (size_t)d * (size_t)n;
    orc_matvec_q80(o, m->aq, m->as, t->q + off, t->s + off / (size_t)gs, n, d, gs);
}

/* One decode step for sequence `seq`: token at position pos -> logits[V].
 * Step order [qa §KV Cache, §GQA, §RoPE; hub §架构实现]: embedding row;
 * per layer RMSNorm, q/k/v matvecs with k and v written straight into the
 * cache slot [layer][pos], RoPE on q and k, attention over 0..pos, wo matvec
 * plus residual, RMSNorm, SwiGLU FFN plus residual; final RMSNorm and the
 * classifier matvec (the embedding table when tied, qa §shared_weights).
 * q80 picks the weights: 0 fp32, 1 the Q8_0 set, 2 the Q4_0 set. */
int orc_forward(orc_model* m, int seq, int token, int pos, int q80, float* logits) {
    const orc_config* c = &m->c;
    if (seq < 0 || seq >= m->n_seq || token < 0 || token >= c->vocab_size || pos < 0 ||
        pos >= c->seq_len || !logits) return -1;
    if (q80 < 0 || q80 > 2) return -1;
    const orc_qset* z = q80 == 2 ? &m->q4 : (q80 ? &m->q8 : NULL);
    if (z && !z->gs) return -1;
    int d = c->dim, h = c->hidden_dim, H = c->n_heads, Hkv = c->n_kv_heads;
    int hs = d / H, kvd = Hkv * hs;
    size_t L = (size_t)c->n_layers, S = (size_t)c->seq_len;
    float* x = m->x;
    if (z) orc_dequantize(z->E.q + (size_t)token * d, z->E.s + (size_t)token * d / z->gs, d, z->gs, x);
    else memcpy(x, m->E + (size_t)token * d, sizeof(float) * (size_t)d);
    for (size_t l = 0; l < L; l++) {
        size_t loff = ((size_t)seq * L + l) * S * (size_t)kvd;
        float* kc = m->kcache + loff;
        float* vc = m->vcache + loff;
        float* k = kc + (size_t)pos * kvd;
        float* v = vc + (size_t)pos * kvd;
        orc_rmsnorm(m->xb, x, m->w_att + l * d, d);
        if (z) {
            orc_qmatvec(m, z, m->q, m->xb, &z->wq, l, d, d);
            orc_qmatvec(m, z, k, m->xb, &z->wk, l, d, kvd);
            orc_qmatvec(m, z, v, m->xb, &z->wv, l, d, kvd);
        } else {
            orc_matvec(m->q, m->xb, m->wq + l * (size_t)d * d, d, d);
            orc_matvec(k, m->xb, m->wk + l * (size_t)kvd * d, d, kvd);
            orc_matvec(v, m->xb, m->wv + l * (size_t)kvd * d, d, kvd);
        }
        orc_rope(m->q, d, hs, pos);
        orc_rope(k, kvd, hs, pos);
        if (m->kv8) {
            orc_kv8_row(k, kvd, hs);
            orc_kv8_row(v, kvd, hs);
        }
        orc_attention(m->xb, m->q, kc, vc, pos, H, Hkv, hs);
        if (z) orc_qmatvec(m, z, m->xb2, m->xb, &z->wo, l, d, d);
        else orc_matvec(m->xb2, m->xb, m->wo + l * (size_t)d * d, d, d);
        for (int i = 0; i < d; i++) x[i] += m->xb2[i];
        orc_rmsnorm(m->xb, x, m->w_ffn + l * d, d);
        if (z) {
            orc_qmatvec(m, z, m->hb, m->xb, &z->w1, l, d, h);
            orc_qmatvec(m, z, m->hb2, m->xb, &z->w3, l, d, h);
        } else {
            orc_matvec(m->hb, m->xb, m->w1 + l * (size_t)h * d, d, h);
            orc_matvec(m->hb2, m->xb, m->w3 + l * (size_t)h * d, d, h);
        }
        orc_swiglu(m->hb, m->hb2, h);
        if (z) orc_qmatvec(m, z, m->xb, m->hb, &z->w2, l, h, d);
        else orc_matvec(m->xb, m->hb, m->w2 + l * (size_t)d * h, h, d);
        for (int i = 0; i < d; i++) x[i] += m->xb[i];
    }
    orc_rmsnorm(x, x, m->w_final, d);
    if (z) orc_qmatvec(m, z, logits, x, &z->wcls, 0, d, c->vocab_size);
    else orc_matvec(logits, x, m->wcls, d, c->vocab_size);
    return 0;
}

int orc_kv_load(orc_model* m, int seq, int n_pos, const float* k, const float* v) {
    const orc_config* c = &m->c;
    if (seq < 0 || seq >= m->n_seq || n_pos < 0 || n_pos > c->seq_len) return -1;
    int hs = c->dim / c->n_heads;
    size_t kvd = (size_t)c->n_kv_heads * (size_t)hs;
    size_t L = (size_t)c->n_layers, S = (size_t)c->seq_len;
    for (size_t l = 0; l < L; l++) {
        size_t dst = (((size_t)seq * L + l) * S) * kvd;
        size_t src = l * (size_t)n_pos * kvd;
        if (k) memcpy(m->kcache + dst, k + src, sizeof(float) * (size_t)n_pos * kvd);
        if (v) memcpy(m->vcache + dst, v + src, sizeof(float) * (size_t)n_pos * kvd);
        if (m->kv8)
            for (int t = 0; t < n_pos; t++) {
                if (k) orc_kv8_row(m->kcache + dst + (size_t)t * kvd, (int)kvd, hs);
                if (v) orc_kv8_row(m->vcache + dst + (size_t)t * kvd, (int)kvd, hs);
            }
    }
    return 0;
}

/* int8 KV cache (reading of the int8 KV cache variant; the pages give none):
 * every K and V row, when it is stored, becomes Q8_0 groups of head_size
 * values (one group per KV head), quantized with the quantize() rule of
 * [port §1], and attention reads code * scale (one fp32 multiply).  The
 * cache keeps those dequantized values in fp32, which is the same arithmetic
 * as keeping the codes and scales.  Enabling it quantizes the rows already in
 * the cache. */
int orc_enable_kv8(orc_model* m) {
    const orc_config* c = &m->c;
    int hs = c->dim / c->n_heads;
    size_t kvd = (size_t)c->n_kv_heads * (size_t)hs;
    size_t rows = (size_t)m->n_seq * (size_t)c->n_layers * (size_t)c->seq_len;
    if (!m->kv8)
        for (size_t r = 0; r < rows; r++) {
            orc_kv8_row(m->kcache + r * kvd, (int)kvd, hs);
            orc_kv8_row(m->vcache + r * kvd, (int)kvd, hs);
        }
    m->kv8 = 1;
    return 0;
}

int orc_kv_read(orc_model* m, int seq, int n_pos, float* k, float* v) {
    const orc_config* c = &m->c;
    if (seq < 0 || seq >= m->n_seq || n_pos < 0 || n_pos > c->seq_len) return -1;
    size_t kvd = (size_t)c->n_kv_heads * (size_t)(c->dim / c->n_heads);
    size_t L = (size_t)c->n_layers, S = (size_t)c->seq_len;
    for (size_t l = 0; l < L; l++) {
        size_t src = (((size_t)seq * L + l) * S) * kvd;
        size_t dst = l * (size_t)n_pos * kvd;
        if (k) memcpy(k + dst, m->kcache + src, sizeof(float) * (size_t)n_pos * kvd);
        if (v) memcpy(v + dst, m->vcache + src, sizeof(float) * (size_t)n_pos * kvd);
    }
    return 0;
}

int orc_kv_reset(orc_model* m, int seq) {
    const orc_config* c = &m->c;
    if (seq < 0 || seq >= m->n_seq) return -1;
    size_t kvd = (size_t)c->n_kv_heads * (size_t)(c->dim / c->n_heads);
    size_t n = (size_t)c->n_layers * (size_t)c->seq_len * kvd;
    memset(m->kcache + (size_t)seq * n, 0, sizeof(float) * n);
    memset(m->vcache + (size_t)seq * n, 0, sizeof(float) * n);
    return 0;
}

int orc_generate(orc_model* m, int seq, int token0, int pos0, int steps, int q80, int32_t* tokens_out,
                 float* logits_out) {
    int V = m->c.vocab_size;
    float* lg = (float*)malloc(sizeof(float) * (size_t)V);
    if (!lg) return -1;
    int tok = token0;
    for (int t = 0; t < steps; t++) {
        if (orc_forward(m, seq, tok, pos0 + t, q80, lg)) { free(lg); return -1; }
        if (logits_out) memcpy(logits_out + (size_t)t * V, lg, sizeof(float) * (size_t)V);
        tok = orc_argmax(lg, V);
        tokens_out[t] = tok;
    }
    free(lg);
    return 0;
}

void orc_destroy(orc_model* m) {
    if (!m) return;
    if (m->q8.gs) orc_qset_free(&m->q8, m->shared);
    if (m->q4.gs) orc_qset_free(&m->q4, m->shared);
    free(m->kcache); free(m->vcache);
    free(m->x); free(m->xb); free(m->xb2); free(m->hb); free(m->hb2); free(m->q);
    free(m->aq); free(m->as);
    free(m);
}
