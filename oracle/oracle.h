/*
 * oracle.h - plain CPU oracle of the llama2.c single-token decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the slow, obviously correct restatement
 * that the GPU library is checked against.  Only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it; the GPU library
 * never does, and the two share no code.
 *
 * Arithmetic: storage is fp32 like llama2.c; every dot product and reduction
 * (matvec rows, sum of squares, attention scores, softmax, weighted V sums) is
 * accumulated in double and rounded to fp32 once at the end of its step.
 * orc_set_fp32_accum(1) switches these sums to the pages' plain fp32
 * left-to-right loops, to show how far the pages' own rounding sits from the
 * double result.  Q8_0 / Q4_0 codes and int32 group dot products are exact.
 */
#ifndef L2C_ORACLE_H
#define L2C_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int32_t dim, hidden_dim, n_layers, n_heads, n_kv_heads, vocab_size, seq_len;
} orc_config;

typedef struct orc_model orc_model;

/* 0 = double accumulation (default), 1 = fp32 sequential accumulation. */
void orc_set_fp32_accum(int on);

/* ---- primitives ---- */
void orc_rmsnorm(float* o, const float* x, const float* w, int n);
void orc_matvec(float* o, const float* x, const float* W, int n, int d);
float orc_rope_freq(int j, int head_size);
void orc_rope(float* v, int n, int head_size, int pos);
void orc_softmax(double* x, int n);
void orc_attention(float* out, const float* q, const float* kc, const float* vc, int pos,
                   int n_heads, int n_kv_heads, int head_size);
double orc_silu(double z);
void orc_swiglu(float* hb, const float* hb2, int n);
int orc_quantize(const float* x, int64_t n, int gs, int8_t* q, float* s);
/* Q4_0: the same rule with scale = max|x| / 7, codes in [-7, 7] (one int8 each). */
int orc_quantize4(const float* x, int64_t n, int gs, int8_t* q, float* s);
void orc_dequantize(const int8_t* q, const float* s, int64_t n, int gs, float* out);
void orc_q80_group_dots(int32_t* out, const int8_t* qx, const int8_t* qw, int n, int d, int gs);
void orc_matvec_q80(float* o, const int8_t* qx, const float* sx, const int8_t* qw, const float* sw,
                    int n, int d, int gs);
int orc_argmax(const float* x, int n);
int orc_sample(const float* z, int n, float temperature, float topp, double coin);

/* ---- whole model ---- */
size_t orc_blob_floats(const orc_config* c, int shared_weights);
/* The model keeps a pointer to `blob` (no copy): the caller keeps it alive. */
orc_model* orc_create(const orc_config* c, const float* blob, size_t blob_floats, int shared_weights,
                      int n_seq);
int orc_enable_q80(orc_model* m, int gs);
/* Q4_0 weights (matvec inputs stay Q8_0 at the same group size). */
int orc_enable_q40(orc_model* m, int gs);
/* int8 KV cache: K and V rows stored as Q8_0 groups of head_size values. */
int orc_enable_kv8(orc_model* m);
void orc_kv8_row(float* row, int n, int gs);
/* q80: 0 fp32 weights, 1 the Q8_0 set, 2 the Q4_0 set. */
int orc_forward(orc_model* m, int seq, int token, int pos, int q80, float* logits);
int orc_kv_load(orc_model* m, int seq, int n_pos, const float* k, const float* v);
int orc_kv_reset(orc_model* m, int seq);
/* Reads back the cache slots of positions [0, n_pos) as [L][n_pos][kv_dim]. */
int orc_kv_read(orc_model* m, int seq, int n_pos, float* k, float* v);
/* Greedy: tok_0 = token0; logits_t = forward(tok_t, pos0 + t); tok_{t+1} = argmax.
 * tokens_out[t] = tok_{t+1}; logits_out (optional) gets all [steps][V]. */
int orc_generate(orc_model* m, int seq, int token0, int pos0, int steps, int q80, int32_t* tokens_out,
                 float* logits_out);
void orc_destroy(orc_model* m);

#ifdef __cplusplus
}
#endif
#endif
