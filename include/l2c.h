/*
 * l2c.h - C ABI of the B200 decode-step library for Llama-2 decoders.
 *
 * One call runs one autoregressive decode step of llama2.c's transformer:
 * the single-token forward() of run.c (fp32 weights) or of runq.c (Q8_0
 * weights and activations), on one GPU, as a CUDA graph of hand-written
 * sm_100a kernels.  Sources: web pages about karpathy's llama2.c, cited by
 * title and section:
 *   [hub]  "Llama 2 in Pure C: 一个周末Hack的AI奇迹" (pomoai.com), sections
 *          架构实现 (RMSNorm, SwiGLU, RoPE, GQA, KV cache), 数据格式 (the .bin
 *          weight file), 量化支持 (Q8_0 with per-group scales).
 *   [port] "超精简LLM部署：llama2.c嵌入式移植全攻略" (blog.gitcode.com),
 *          §1 INT8量化压缩 (quantize()), §2 内存优化策略 (KV cache),
 *          智能家居控制案例 (build_transformer / forward / sample_argmax).
 *   [qa]   "Karpathy 技術學習庫 - Q&A 問答集", 技術細節 (KV cache indexing,
 *          GQA, RoPE on the fly, skipped freq_cis, shared_weights) and
 *          效能相關 (13B pointer overflow).
 *
 * Conventions for every entry point:
 *   - Return value: L2C_OK (0) or a negative L2C_E_* code; l2c_last_error()
 *     gives a one-line reason.  Nothing aborts the process.
 *   - Pointers named *_dev are device pointers on the handle's GPU; *_host
 *     are host pointers.  "host or device" arguments are detected with
 *     cudaPointerGetAttributes.
 *   - The library never keeps a caller pointer past the call: inputs are
 *     copied, outputs written.  Buffers the library returns stay owned by
 *     the handle and stay valid until the next call on the same handle.
 *   - One handle, one CUDA stream.  Calls on one handle are not thread-safe.
 *     Work is enqueued on the handle's stream; l2c_sync() waits for it and
 *     reports device-side errors (bad token or position, a bounded wait that
 *     gave up, a NaN logit) recorded by the kernels.
 *   - Sizes and offsets are 64-bit internally ([qa] 效能相關: llama2.c's 13B
 *     failure was int overflow in pointer arithmetic).
 */
#ifndef L2C_H
#define L2C_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define L2C_API __attribute__((visibility("default")))
#else
#define L2C_API
#endif

#define L2C_OK 0
#define L2C_E_ARG (-1)    /* invalid argument or unsupported shape */
#define L2C_E_OOM (-2)    /* device allocation failed */
#define L2C_E_CUDA (-3)   /* a CUDA runtime call failed */
#define L2C_E_DEVICE (-4) /* a kernel recorded an error (see l2c_last_error) */
#define L2C_E_STATE (-5)  /* call not valid in the handle's state (e.g. Q8_0 not enabled) */
#define L2C_E_SCRATCH (-6) /* the problem needs more than l2c_attention_noalloc's fixed scratch */

/* The model shape: the seven integers of llama2.c's checkpoint header
 * ([hub] 数据格式: "layers, dimensions, heads ..."; [qa] GQA: kv heads).
 * head_size = dim / n_heads, kv_dim = n_kv_heads * head_size. */
typedef struct {
    int32_t dim, hidden_dim, n_layers, n_heads, n_kv_heads, vocab_size, seq_len;
} l2c_config;

typedef struct l2c_ctx l2c_ctx;

/* Number of fp32 values in a weight blob of this shape (see l2c_create). */
L2C_API size_t l2c_blob_floats(const l2c_config* cfg, int shared_weights);

/*
 * l2c_create - build_transformer() of [port] 智能家居控制案例.
 *
 * blob: the fp32 weights in llama2.c's checkpoint order, without the header
 *   ([hub] 数据格式: contiguous fp32 arrays after the config; [qa] 跳過
 *   freq_cis): E[V][d], rms_att[L][d], Wq[L][d][d], Wk[L][kvd][d],
 *   Wv[L][kvd][d], Wo[L][d][d], rms_ffn[L][d], W1[L][h][d], W2[L][d][h],
 *   W3[L][h][d], rms_final[d], two legacy RoPE tables of seq_len*hs/2 floats
 *   each (skipped), then Wcls[V][d] only when shared_weights == 0.
 *   Host or device memory; blob_floats must equal l2c_blob_floats().  The
 *   blob is copied (and re-tiled) into device memory; the caller keeps it.
 * shared_weights: 1 = the classifier is the embedding table ([qa]
 *   shared_weights: a positive vocab_size in the header), 0 = a separate
 *   classifier follows the legacy tables.
 * max_batch: sequences the handle serves (each gets its own KV cache of
 *   n_layers*seq_len*kv_dim fp32 for K and for V, [port] §2); >= 1.
 * cuda_stream: the cudaStream_t to enqueue on (NULL = the legacy stream).
 * Errors: L2C_E_ARG for a bad shape (dim % n_heads, n_heads % n_kv_heads,
 *   odd head_size, a row width not a multiple of 4, an unsupported
 *   head_size/GQA ratio) or blob size; L2C_E_OOM; L2C_E_CUDA.
 */
L2C_API int l2c_create(const l2c_config* cfg, const float* blob, size_t blob_floats, int shared_weights,
               int max_batch, void* cuda_stream, l2c_ctx** out);

/*
 * l2c_enable_q80 - makes the Q8_0 weight set of runq.c ([hub] 量化支持).
 * Every matvec weight (Wq, Wk, Wv, Wo, W1, W2, W3, the classifier) and the
 * embedding table are quantized on the device with the rule of quantize()
 * ([port] §1 INT8量化压缩): per group of gs consecutive values along a row,
 * scale = max|x| / 127 (fp32) and code = round(x / scale).  The fp32 set is
 * kept, so both paths stay usable.  gs must divide dim and hidden_dim and be
 * a multiple of 16 (16..256).  Calling it again with the same gs is a no-op;
 * another gs gives L2C_E_STATE.
 */
L2C_API int l2c_enable_q80(l2c_ctx* h, int gs);

/*
 * l2c_enable_q40 - makes a Q4_0 weight set, beside the fp32 and Q8_0 ones.
 * "技术深度解析" (ainews.cool llama2.c article), 整数量化路径: runq.c with 4-bit
 * integer groups; the page gives no rule, so the reading is quantize() of
 * [port] §1 with 4-bit codes: per group of gs values along a row, scale =
 * max|x| / 7 (fp32) and code = round(x / scale), in [-7, 7].  The same
 * tensors as l2c_enable_q80 (every matvec weight and the embedding table);
 * the GEMVs stream two codes per byte plus one fp32 scale per group.  gs must
 * be 32, 64 or 128 and divide dim and hidden_dim, dim + 2 * kv_dim must be a
 * multiple of 4 and vocab_size even (the 4-bit GEMV takes rows in groups of 4
 * and 2); otherwise L2C_E_ARG.  Calling
 * it again with the same gs is a no-op; another gs gives L2C_E_STATE.
 * L2C_E_OOM if the device memory runs out.  Blocks.
 */
L2C_API int l2c_enable_q40(l2c_ctx* h, int gs);

/*
 * l2c_forward - forward(transformer, token, pos) of run.c ([port]
 * 智能家居控制案例): one decode step of sequence 0 in fp32.  Embedding row,
 * then per layer RMSNorm, q/k/v matvecs, RoPE as cos/sin(pos*freq) computed
 * in the kernel ([qa] RoPE), the K/V write at cache[layer][pos] ([qa] KV
 * Cache), grouped-query attention over positions 0..pos ([qa] GQA), wo plus
 * residual, RMSNorm, SwiGLU FFN plus residual; final RMSNorm and classifier.
 * Returns the handle-owned DEVICE logits [vocab_size] (valid until the next
 * call on the handle; the step may still be running: use the handle's stream
 * or l2c_sync()), or NULL if token is not in [0, vocab_size) or pos not in
 * [0, seq_len) (l2c_last_error says which).
 */
L2C_API const float* l2c_forward(l2c_ctx* h, int token, int pos);

/* l2c_forward_q80 - the same step through the Q8_0 weights (runq.c): every
 * matvec input is quantized at the same group size and each output is the
 * sum over groups of the exact int32 group dot times both scales.  NULL also
 * when l2c_enable_q80 has not been called. */
L2C_API const float* l2c_forward_q80(l2c_ctx* h, int token, int pos);

/* l2c_forward_q40 - the same step through the Q4_0 weights: every matvec input
 * is quantized to Q8_0 at the Q4_0 group size, and each output is the sum
 * over groups of the exact int32 dot of the 4-bit and 8-bit codes times both
 * scales.  NULL also when l2c_enable_q40 has not been called. */
L2C_API const float* l2c_forward_q40(l2c_ctx* h, int token, int pos);

/*
 * l2c_argmax - sample_argmax() of [port] 智能家居控制案例: the index of the
 * largest of n device floats, the lowest index among equal maxima.  Blocks
 * until the result is on the host.  A NaN in the input gives L2C_E_DEVICE.
 */
L2C_API int l2c_argmax(l2c_ctx* h, const float* logits_dev, int n, int* out_idx_host);

/*
 * l2c_sample - the token draw after the logits: a temperature divides the
 * logits before the softmax ("LLM底层原理与工程实践" §3.2), temperature 0 is the
 * greedy sample_argmax of [port] 智能家居控制案例 (l2c_argmax).  Otherwise
 * (reading taken where the pages stop): weights q_i = exp((z_i - max z) / T)
 * in double; top-p keeps the smallest set of most probable tokens whose
 * weight reaches topp * sum q, every token tied with the last one included
 * (topp >= 1: all tokens); the coin u picks the first index, in index order,
 * of the set at which the running weight exceeds u * the set's weight.
 * logits_dev [n] device fp32 (e.g. the logits of l2c_forward, on the same
 * stream); temperature >= 0, topp > 0, coin in [0, 1) (the caller draws it:
 * the library keeps no random state).  Blocks until the index is on the host.
 * A NaN logit gives L2C_E_DEVICE.  The first call with a larger n allocates
 * a scratch row of n doubles in the handle.
 */
L2C_API int l2c_sample(l2c_ctx* h, const float* logits_dev, int n, float temperature, float topp, double coin,
                       int* out_idx_host);

/*
 * l2c_generate - greedy decoding with the token fed back on the device:
 * tok_0 = token0; for t = 0..steps-1: logits = forward(tok_t, pos0 + t),
 * tok_{t+1} = argmax(logits).  tokens_out_host[t] = tok_{t+1}.
 * q80 picks the weights: 0 fp32, 1 Q8_0, 2 Q4_0 (other values: L2C_E_ARG;
 * weights not made: L2C_E_STATE).  pos0 + steps must not exceed seq_len.
 * Blocks until the tokens are on the host.
 */
L2C_API int l2c_generate(l2c_ctx* h, int token0, int pos0, int steps, int q80, int32_t* tokens_out_host);

/*
 * l2c_forward_batch - B independent sequences, one token each: sequence b
 * runs the step with tokens[b] at position pos[b] against its own KV cache.
 * Each matvec of the step runs as one GEMM over the B sequences (Q8_0: int8
 * tensor cores, exact int32 group dots, double group sums; fp32: fp32 FMAs).
 * tokens, pos: host or device int32 [B]; B <= max_batch and B <= 32.
 * logits_out_dev: device [B][vocab_size].  q80 = 1 selects the Q8_0 path
 * (0 fp32; other values, Q4_0 included, give L2C_E_ARG).
 */
L2C_API int l2c_forward_batch(l2c_ctx* h, int B, const int32_t* tokens, const int32_t* pos, int q80,
                      float* logits_out_dev);

/*
 * l2c_prefill - a prompt at once: tokens[0..n-1] at positions pos0..pos0+n-1
 * of sequence seq.  The pages feed a prompt through forward one token at a
 * time ([port] 智能家居控制案例: encode, then forward(tokens[0], 0), ...);
 * this computes the same K/V cache rows and logits as those n steps, in
 * chunks of up to 32 tokens that run as GEMMs (each weight row read once per
 * chunk), with causal attention: token i of a chunk attends to positions
 * 0..pos0+i of the sequence's cache, which holds the rows of earlier chunks
 * and calls.  Same arithmetic per element as the batched step: Q8_0 on the
 * int8 tensor cores with double group sums; fp32 with fp32 FMAs.
 * tokens: host int32 [n]; 0 <= seq < max_batch; n >= 1; pos0 + n <= seq_len.
 * logits_last_dev: device [vocab_size] receives the logits of the last token
 * (NULL: not written).  q80 = 1 needs l2c_enable_q80 with gs a multiple of 32
 * that the batched GEMM tiles (else L2C_E_ARG); q80 is 0 or 1 (Q4_0 serves
 * the single-sequence step only: L2C_E_ARG).  The first call allocates the
 * chunk activations in the handle.  Blocks until the cache is written.
 */
L2C_API int l2c_prefill(l2c_ctx* h, int seq, int n, const int32_t* tokens, int pos0, int q80, float* logits_last_dev);

/*
 * l2c_enable_kv8 - the int8 KV cache (on = 1) or the fp32 one (on = 0).  The
 * pages give no int8 KV cache; the reading: every K and V row, when it is
 * stored, becomes Q8_0 groups of head_size values (one per KV head) with the
 * quantize() rule of [port] §1, and attention reads code * scale (one fp32
 * multiply).  It serves the quantized steps (l2c_forward_q80, l2c_forward_q40,
 * l2c_generate with q80 = 1 or 2), whose attention then streams the codes and scales (a quarter of
 * the bytes); the fp32 cache rows are overwritten with the same code * scale
 * values (l2c_kv_read returns those).  Enabling it quantizes every row
 * already in the cache (all sequences); l2c_kv_load quantizes the rows it
 * loads.  The first call allocates the codes (2 * max_batch * n_layers *
 * seq_len * kv_dim bytes) and scales.  While it is on, the fp32 step
 * (l2c_forward, l2c_generate with q80 = 0), l2c_forward_batch and
 * l2c_prefill return L2C_E_STATE.
 * Errors: L2C_E_ARG for a head size / GQA ratio without an attention kernel
 * (head_size a multiple of 4, at most 128); L2C_E_OOM.  Blocks.
 */
L2C_API int l2c_enable_kv8(l2c_ctx* h, int on);

/*
 * l2c_quantize_q80 - quantize() of [port] §1 INT8量化压缩 on n device
 * floats: for each group of gs values, s[g] = max|x| / 127 (fp32) and
 * q[i] = round(x[i] / s[g]) (fp32 quotient, half away from zero); a group of
 * zeros gets s = 0 and codes 0.  x_dev [n], q_dev [n], s_dev [n / gs];
 * n % gs == 0, 1 <= gs <= 1024.  Asynchronous on the handle's stream.
 */
L2C_API int l2c_quantize_q80(l2c_ctx* h, const float* x_dev, int64_t n, int gs, int8_t* q_dev, float* s_dev);

/*
 * l2c_q80_group_dots - the exact int32 dot product of every (row, group) of
 * Q8_0 codes: out[r][g] = sum_k qw[r][g*gs+k] * qx[g*gs+k].  For gs = 32, 64
 * or 128 with K % 64 == 0 (K <= 32768, 16-byte aligned qw_dev and qx_dev) it
 * runs the Q8_0 matvec's own 64-byte chunk routine (the one every Q8_0 step
 * uses at those group sizes); otherwise the generic matvec's 16-byte chunk
 * loop.  qw_dev [rows][K] int8, qx_dev [K] int8, out_dev [rows][K/gs] int32;
 * K % gs == 0, gs a multiple of 16 (16..512).  Asynchronous on the handle's
 * stream.
 */
L2C_API int l2c_q80_group_dots(l2c_ctx* h, const int8_t* qw_dev, const int8_t* qx_dev, int rows, int K, int gs,
                       int32_t* out_dev);

/*
 * l2c_kv_load - fills the KV cache of sequence seq at positions [0, n_pos)
 * from k and v laid out [n_layers][n_pos][kv_dim] (host or device); slots
 * from n_pos on are left as they are.  Used to start a step from a given
 * context without decoding it.
 */
L2C_API int l2c_kv_load(l2c_ctx* h, int seq, int n_pos, const float* k, const float* v);

/* l2c_kv_read - copies the cache slots [0, n_pos) of sequence seq into host
 * buffers k_host, v_host laid out [n_layers][n_pos][kv_dim].  Blocks. */
L2C_API int l2c_kv_read(l2c_ctx* h, int seq, int n_pos, float* k_host, float* v_host);

/* l2c_kv_reset - zeroes the KV cache of sequence seq (-1: all sequences). */
L2C_API int l2c_kv_reset(l2c_ctx* h, int seq);

/*
 * l2c_attention - the grouped-query attention of one layer ([qa] GQA and KV
 * Cache) run alone with the handle's head layout: for query head i, with KV
 * head g = i / (n_heads / n_kv_heads), scores q_i . k_t / sqrt(head_size)
 * over t = 0..pos, softmax, and out_i = sum_t a_t v_t.  q_dev [n_heads *
 * head_size] (already rotated), k_dev and v_dev [>= pos+1][kv_dim] (one
 * layer's caches), out_dev [n_heads * head_size]; all device fp32, 16-byte
 * aligned (L2C_E_ARG otherwise).  precision: 0 accumulates in fp32 (as the
 * fp32 step does), 1 in double (as the Q8_0 step does).  pos must be in
 * [0, seq_len).  Uses the handle's scratch and position split (the same as
 * the decode step's); asynchronous on the handle's stream.
 */
L2C_API int l2c_attention(l2c_ctx* h, const float* q_dev, const float* k_dev, const float* v_dev, int pos,
                          int precision, float* out_dev);

/*
 * l2c_attention_noalloc - l2c_attention for callers that cannot allocate
 * device memory, with no handle.  (The pages have no counterpart: this is an
 * interface of this library, not a step of llama2.c.)
 *
 * Who needs it: a process whose device memory belongs to another allocator
 * (a framework's pool or a serving engine that reserves HBM up front, where a
 * stray cudaMalloc fails or breaks the owner's accounting), or code on a
 * latency-critical path where cudaMalloc/cudaFree may synchronize the device.
 * Such callers cannot create an l2c handle either (it owns weights, caches and
 * scratch), so this entry point takes every shape argument explicitly and
 * calls no cudaMalloc, cudaFree or allocating library routine.
 *
 * Computes what l2c_attention computes, with the same kernel but its own
 * position split (chunks of 64 positions, where a handle picks the split from
 * the SM count), so results agree with l2c_attention within rounding: for
 * query head i and KV head g = i / (n_heads / n_kv_heads), scores
 * q_i . k_t / sqrt(head_size) over t = 0..pos, softmax, out_i = sum a_t v_t.
 * q_dev [n_heads * head_size], k_dev and v_dev [>= pos+1][n_kv_heads *
 * head_size], out_dev [n_heads * head_size]: device fp32, 16-byte aligned,
 * owned by the caller.  precision: 0 = fp32 accumulation, 1 = double.
 * Supported head sizes and GQA ratios are those of l2c_create.  Enqueued on
 * cuda_stream (NULL = the legacy stream); returns before the kernels finish.
 * The kernels wait on nothing (no barrier across CTAs; the last CTA of a KV
 * head to finish merges its chunks), so there is no device-side error to
 * report.
 *
 * Scratch: a fixed 4 MiB device array in the library (every GPU that loads
 * the library holds it until the process exits).  A call needs
 * 256 + 4*n_kv_heads (rounded up to 256) + n_kv_heads * (pos/64 + 1) *
 * (n_heads/n_kv_heads) * (head_size + 2) * (4 or 8 for precision 0 or 1)
 * bytes; a larger problem is rejected with L2C_E_SCRATCH before anything is
 * enqueued.  (For 32 heads of 128 that is about 8000 positions in double.)
 * All calls share the array, so calls that overlap on the GPU (different
 * streams, or different host threads, without ordering between them) race
 * and may corrupt each other's results; order them on one stream.  Each call
 * clears the counters it uses before its kernel runs.
 *
 * Set-up: the first call on a device, with that device current, looks up the
 * array's device address (cudaGetSymbolAddress) and sets the attention
 * kernels' shared-memory limit (cudaFuncSetAttribute); it does so again in a
 * new CUDA context (after a device reset, the library's module and its array
 * are loaded anew).  Make
 * that first call before capturing work on the device's streams.  Devices
 * with an ordinal of 64 or more are not supported (L2C_E_CUDA).
 * Errors: L2C_E_ARG (null or unaligned pointer, bad shape, unsupported head
 * size or ratio), L2C_E_SCRATCH, L2C_E_CUDA.
 */
L2C_API int l2c_attention_noalloc(const float* q_dev, const float* k_dev, const float* v_dev, int n_heads,
                                  int n_kv_heads, int head_size, int pos, int precision, float* out_dev,
                                  void* cuda_stream);

/*
 * l2c_time_kernel - measurement hook: runs kernel `kind` of the fp32 (q80 = 0),
 * Q8_0 (1) or Q4_0 (2) step alone, iters times back to back on the handle's stream, and
 * stores the average time per launch in ms (two CUDA events around the
 * loop).  Launch i uses layer i % n_layers, so consecutive launches stream
 * different weights.  kind: 0 = RMSNorm+QKV+RoPE, 1 = attention, 2 = wo,
 * 3 = RMSNorm+W1/W3+SwiGLU, 4 = W2, 5 = final RMSNorm+classifier.  The kernels use the handle's current
 * token/position and update its state (KV slot, activations) as in a step.
 * Blocks.
 */
L2C_API int l2c_time_kernel(l2c_ctx* h, int kind, int q80, int iters, float* avg_ms);

/* l2c_sync - waits for the handle's stream, then reads and clears the
 * device error word: L2C_E_DEVICE if a kernel recorded an error since the
 * last check. */
L2C_API int l2c_sync(l2c_ctx* h);

/* l2c_stream - the cudaStream_t the handle enqueues on. */
L2C_API void* l2c_stream(l2c_ctx* h);

/* l2c_last_status - the L2C_E_* code of the last failed call on the handle
 * (L2C_OK if none failed); use it after l2c_forward / l2c_forward_q80 return
 * NULL. */
L2C_API int l2c_last_status(l2c_ctx* h);

/* l2c_last_error - copies the last error message (NUL-terminated, at most
 * len bytes) and returns its full length. */
L2C_API int l2c_last_error(l2c_ctx* h, char* buf, int len);

/* l2c_destroy - frees all device memory and graphs of the handle. */
L2C_API void l2c_destroy(l2c_ctx* h);

#ifdef __cplusplus
}
#endif
#endif
