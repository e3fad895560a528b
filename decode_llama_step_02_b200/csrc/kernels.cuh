// kernels.cuh - the decode step's hand-written sm_100a kernels.
//
// One decode step of a Llama-2 decoder (llama2.c's forward(): token
// embedding; per layer RMSNorm, q/k/v matvecs, RoPE evaluated on the fly as
// cos/sin(pos*freq), the KV-cache write at [layer][pos][kv_dim], grouped-query
// attention over positions 0..pos, the wo matvec plus residual, RMSNorm, the
// SwiGLU FFN plus residual; then the final RMSNorm and the classifier) runs
// as five kernels per layer plus one:
//
//   gemv<QKV>   RMSNorm prologue, [Wq;Wk;Wv] rows, RoPE + cache-write epilogue
//   attention   flash-decode over position chunks, last CTA merges the chunks
//   gemv<RESID> wo rows, residual epilogue (x += Wo att)
//   gemv<W13>   RMSNorm prologue, interleaved (W1 row i, W3 row i), SwiGLU epilogue
//   gemv<RESID> W2 rows, residual epilogue (x += W2 hb)
//   gemv<CLS>   final RMSNorm prologue, classifier rows, argmax epilogue
//
// fp32 weights stream through registers with 128-bit non-allocating loads.
// Q8_0 weights are row records [K int8 codes | K/GS fp32 scales | pad to 16 B]
// staged through a shared-memory ring by 1-D bulk copies (TMA) and reduced
// with dp4a into exact int32 group sums.  Every kernel is launched with
// programmatic dependent launch: it prefetches its weights (L2 bulk prefetch,
// and for Q8_0 the first ring stages) before waiting on the previous kernel.
//
// Precision.  Activations are stored in fp32.  RMSNorm, RoPE, SwiGLU, the
// Q8_0 group sums and (on the Q8_0 path) attention are evaluated in double
// and rounded once to fp32, so every value that decides a Q8_0 code is the
// same fp32 number a double-accumulating reference produces.  The fp32 path
// accumulates its matvec rows and its attention in fp32.
#pragma once
#include "attention.cuh"
#include "common.cuh"

namespace l2c {

enum GemvMode : int { M_QKV = 0, M_RESID = 1, M_W13 = 2, M_CLS = 3 };

struct GemvArgs {
    const void* W;           // fp32 [rows][ldw] or Q8_0 row records [rows][rb]
    int rows;                // output rows of this matrix
    int K;                   // input width
    size_t ld;               // fp32: row stride in floats; Q8_0: record size in bytes
    const float* in;         // input vector (x, attention output or hb)
    const float* norm_w;     // RMSNorm gain; nullptr = the input is used as is
    const void* emb;         // layer 0: embedding table (fp32 rows or Q8_0 records)
    float* x_resid;          // layer 0: receives the embedding row (residual stream)
    float* out;              // q / x (residual) / hb / logits
    float* kslot;            // this layer's key cache   [S][kvd]
    float* vslot;            // this layer's value cache [S][kvd]
    const float* freq;       // RoPE frequencies [hs/2]
    int d, kvd, hs, vocab, seq_len;
    int gs;                  // Q8_0 group size
    const int* tp;           // {token, pos}
    unsigned long long* amax;  // argmax key (classifier); reset by layer 0
    int* err;
    size_t prefetch_bytes;   // L2 prefetch of the CTA's first weights, issued before the dependency wait
    int late_trigger;        // fp32: 1 = let the next kernel launch only after this CTA's last weight loads
    int early;               // Q8_0: 1 = let the next kernel launch as soon as this one starts (else at its end)
    unsigned long long wait_ns;  // limit of every barrier wait
    int* stall;              // test switch (Q8_0): CTA 0 withholds one ring copy once if *stall != 0
};


// ----------------------------------------------------------------- epilogues --

__device__ __forceinline__ double silu_d(double z) { return z / (1.0 + exp(-z)); }

// Rotates the pair (a, b) at in-head index j (even) by theta = pos*freq[j/2]
// (fp32 product); cos/sin of that angle in double.
__device__ __forceinline__ void rope_pair(float a, float b, int j, int pos, const float* freq, float& o0,
                                          float& o1) {
    float theta = (float)pos * freq[j >> 1];
    double s, c;
    sincos((double)theta, &s, &c);
    o0 = (float)((double)a * c - (double)b * s);
    o1 = (float)((double)a * s + (double)b * c);
}

// The same rotation from a table cs[j/2] = (cos, sin) of the pair's angle.
__device__ __forceinline__ void rope_pair_tab(float a, float b, int j, const double2* cs, float& o0, float& o1) {
    const double2 t = cs[j >> 1];
    o0 = (float)((double)a * t.x - (double)b * t.y);
    o1 = (float)((double)a * t.y + (double)b * t.x);
}

// Fills cs[i] = (cos, sin)(pos * freq[i]) for the hs/2 pair frequencies: one
// sincos per pair index per CTA instead of one per output pair.
__device__ __forceinline__ void rope_table(const GemvArgs& a, int pos, double2* cs) {
    for (int i = threadIdx.x; i < a.hs / 2; i += blockDim.x) {
        const float theta = (float)pos * a.freq[i];
        double sn, c;
        sincos((double)theta, &sn, &c);
        cs[i] = make_double2(c, sn);
    }
}

// Unit u of the QKV matrix is the row pair (2u, 2u+1); v0/v1 its two outputs.
__device__ __forceinline__ void epi_qkv(const GemvArgs& a, int u, float v0, float v1, int pos, const double2* cs) {
    int r = 2 * u;
    if (r < a.d) {
        float o0, o1;
        rope_pair_tab(v0, v1, r % a.hs, cs, o0, o1);
        a.out[r] = o0;
        a.out[r + 1] = o1;
    } else if (r < a.d + a.kvd) {
        int i = r - a.d;
        float o0, o1;
        rope_pair_tab(v0, v1, i % a.hs, cs, o0, o1);
        float* k = a.kslot + (size_t)pos * a.kvd;
        k[i] = o0;
        k[i + 1] = o1;
    } else {
        int i = r - a.d - a.kvd;
        float* v = a.vslot + (size_t)pos * a.kvd;
        v[i] = v0;
        v[i + 1] = v1;
    }
}

__device__ __forceinline__ void epi_w13(const GemvArgs& a, int u, float g, float up) {
    a.out[u] = (float)(silu_d((double)g) * (double)up);
}

// ------------------------------------------------------------ input prologue --

// Reads the step's token/pos, checks them, and returns the input row pointer
// (the embedding row on layer 0).  Out-of-range values set the error word and
// are clamped so that no access leaves its buffer.
__device__ __forceinline__ void read_tp(const GemvArgs& a, int& token, int& pos) {
    token = a.tp[0];
    pos = a.tp[1];
    if (token < 0 || token >= a.vocab) {
        if (threadIdx.x == 0 && blockIdx.x == 0) set_error(a.err, DERR_TOKEN);
        token = 0;
    }
    if (pos < 0 || pos >= a.seq_len) {
        if (threadIdx.x == 0 && blockIdx.x == 0) set_error(a.err, DERR_POS);
        pos = 0;
    }
}

// fp32 GEMV input, in two halves around the dependency wait.  Thread t owns
// the float4 elements t + j*blockDim (j < F32_PER).  pre: the RMSNorm gain and,
// on layer 0, the embedding row E[token] (neither is written by the step's
// kernels).  post: the input vector written by the previous kernel, then
// RMSNorm in double into shared memory; CTA 0 also stores the embedding row as
// the residual x.  Requires K % 4 == 0 and K/4 <= F32_PER * blockDim.
constexpr int F32_PER = 4;

struct F32Pre {
    float4 v[F32_PER];
    float4 w[F32_PER];
};

__device__ __forceinline__ bool f32_pre_fits(const GemvArgs& a) { return (a.K >> 2) <= F32_PER * (int)blockDim.x; }

__device__ __forceinline__ void f32_pre_load(const GemvArgs& a, int token, F32Pre& r) {
    const int K4 = a.K >> 2, nt = blockDim.x;
    const float4* nw = reinterpret_cast<const float4*>(a.norm_w);
    const float4* emb = a.emb ? reinterpret_cast<const float4*>(static_cast<const float*>(a.emb) + (size_t)token * a.K)
                              : nullptr;
#pragma unroll
    for (int j = 0; j < F32_PER; j++) {
        const int i = threadIdx.x + j * nt;
        r.w[j] = (nw && i < K4) ? nw[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        r.v[j] = (emb && i < K4) ? emb[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

__device__ __forceinline__ void f32_post_load(const GemvArgs& a, F32Pre& r, float* xs, double* red) {
    const int K4 = a.K >> 2, nt = blockDim.x;
    float4* xs4 = reinterpret_cast<float4*>(xs);
    if (!a.emb) {
        const float4* in = reinterpret_cast<const float4*>(a.in);
#pragma unroll
        for (int j = 0; j < F32_PER; j++) {
            const int i = threadIdx.x + j * nt;
            r.v[j] = i < K4 ? in[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    } else if (blockIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < F32_PER; j++) {
            const int i = threadIdx.x + j * nt;
            if (i < K4) reinterpret_cast<float4*>(a.x_resid)[i] = r.v[j];
        }
    }
    if (a.norm_w) {
        double ss = 0.0;
#pragma unroll
        for (int j = 0; j < F32_PER; j++)
            ss += (double)r.v[j].x * r.v[j].x + (double)r.v[j].y * r.v[j].y + (double)r.v[j].z * r.v[j].z +
                  (double)r.v[j].w * r.v[j].w;
        ss = block_sum(ss, red);
        const double inv = 1.0 / sqrt(ss / (double)a.K + 1e-5);
#pragma unroll
        for (int j = 0; j < F32_PER; j++) {
            const float4 g = r.w[j];
            r.v[j].x = (float)((double)g.x * (inv * (double)r.v[j].x));
            r.v[j].y = (float)((double)g.y * (inv * (double)r.v[j].y));
            r.v[j].z = (float)((double)g.z * (inv * (double)r.v[j].z));
            r.v[j].w = (float)((double)g.w * (inv * (double)r.v[j].w));
        }
    }
#pragma unroll
    for (int j = 0; j < F32_PER; j++) {
        const int i = threadIdx.x + j * nt;
        if (i < K4) xs4[i] = r.v[j];
    }
}

// Wide inputs (K/4 > F32_PER * blockDim): a plain strided loop after the wait.
static __device__ void load_input_f32_wide(const GemvArgs& a, int token, float* xs, double* red) {
    const int K4 = a.K >> 2, nt = blockDim.x;
    const float4* in = reinterpret_cast<const float4*>(
        a.emb ? static_cast<const float*>(a.emb) + (size_t)token * a.K : a.in);
    float4* xs4 = reinterpret_cast<float4*>(xs);
    for (int i = threadIdx.x; i < K4; i += nt) {
        xs4[i] = in[i];
        if (a.emb && blockIdx.x == 0) reinterpret_cast<float4*>(a.x_resid)[i] = in[i];
    }
    if (a.norm_w) {
        __syncthreads();
        double ss = 0.0;
        for (int i = threadIdx.x; i < a.K; i += nt) ss += (double)xs[i] * (double)xs[i];
        ss = block_sum(ss, red);
        const double inv = 1.0 / sqrt(ss / (double)a.K + 1e-5);
        for (int i = threadIdx.x; i < a.K; i += nt) xs[i] = (float)((double)a.norm_w[i] * (inv * (double)xs[i]));
    }
}

// ------------------------------------------------------------ fp32 GEMV ------

template <int R, int U>
__device__ __forceinline__ void dot_rows_f32(const float* __restrict__ w, size_t ldw, int K4,
                                             const float4* __restrict__ xs, uint64_t pol, float (&out)[R]) {
    const int lane = threadIdx.x & 31;
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; r++) acc[r] = 0.f;
    int j = lane;
    for (; j + 32 * (U - 1) < K4; j += 32 * U) {
        float4 wv[R][U];
#pragma unroll
        for (int u = 0; u < U; u++)
#pragma unroll
            for (int r = 0; r < R; r++)
                wv[r][u] = ld_stream_f4(reinterpret_cast<const float4*>(w + r * ldw) + j + 32 * u, pol);
#pragma unroll
        for (int u = 0; u < U; u++) {
            float4 xv = xs[j + 32 * u];
#pragma unroll
            for (int r = 0; r < R; r++) {
                acc[r] = fmaf(wv[r][u].x, xv.x, acc[r]);
                acc[r] = fmaf(wv[r][u].y, xv.y, acc[r]);
                acc[r] = fmaf(wv[r][u].z, xv.z, acc[r]);
                acc[r] = fmaf(wv[r][u].w, xv.w, acc[r]);
            }
        }
    }
    if (j < K4) {  // tail: one predicated batch, all loads in flight together
        float4 wv[R][U];
#pragma unroll
        for (int u = 0; u < U; u++)
#pragma unroll
            for (int r = 0; r < R; r++)
                wv[r][u] = j + 32 * u < K4
                               ? ld_stream_f4(reinterpret_cast<const float4*>(w + r * ldw) + j + 32 * u, pol)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < U; u++) {
            const float4 xv = j + 32 * u < K4 ? xs[j + 32 * u] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < R; r++) {
                acc[r] = fmaf(wv[r][u].x, xv.x, acc[r]);
                acc[r] = fmaf(wv[r][u].y, xv.y, acc[r]);
                acc[r] = fmaf(wv[r][u].z, xv.z, acc[r]);
                acc[r] = fmaf(wv[r][u].w, xv.w, acc[r]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; r++) out[r] = warp_sum(acc[r]);
}

constexpr int F32_THREADS = 512;

// Requires K % (4*ks) == 0 (rows are 16-byte aligned).  Dynamic shared
// memory: K floats of input, then the partial sums [rows of the CTA][ks].
// Each CTA owns a contiguous range of rows (an even start for the row-pair
// epilogues); a warp's unit is one K/ks slice of one row, taken round-robin,
// so the CTA's ks*rows slices spread evenly over its 16 warps.  After a
// barrier the CTA sums the slices of each row in a fixed order and runs the
// epilogue (RoPE and the cache write, SwiGLU, the residual, or argmax).
template <int MODE>
__global__ void __launch_bounds__(F32_THREADS, 2) k_gemv_f32(const GemvArgs a, const int ks) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    float* part = xs + a.K;
    __shared__ double red[32];
    __shared__ unsigned long long best_s[32];
    __shared__ double2 rope_cs[MODE == M_QKV ? 128 : 1];
    constexpr int PAIR = (MODE == M_QKV || MODE == M_W13) ? 2 : 1;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int npair = a.rows / PAIR;
    const int r0 = PAIR * (int)((long long)npair * blockIdx.x / gridDim.x);
    const int r1 = PAIR * (int)((long long)npair * (blockIdx.x + 1) / gridDim.x);
    const float* W = static_cast<const float*>(a.W);
    const uint64_t pol = policy_evict_first();
    // before the wait: token/position (written before the step), RMSNorm gain,
    // embedding row, RoPE table; then the L2 prefetch of this CTA's weights
    int token = 0, pos = 0;
    if (MODE == M_QKV) read_tp(a, token, pos);
    F32Pre pre;
    const bool fits = f32_pre_fits(a);
    if (fits) f32_pre_load(a, token, pre);
    if (MODE == M_QKV) rope_table(a, pos, rope_cs);
    if (threadIdx.x == 0 && r1 > r0 && a.prefetch_bytes) {
        size_t bytes = (size_t)(r1 - r0) * a.ld * sizeof(float);
        if (bytes > a.prefetch_bytes) bytes = a.prefetch_bytes;
        prefetch_l2_range(W + (size_t)r0 * a.ld, bytes, policy_evict_last());
    }
    grid_dep_wait();
    if (!a.late_trigger) grid_dep_launch();
    if (MODE == M_QKV && a.amax && blockIdx.x == 0 && threadIdx.x == 0) *a.amax = 0ull;
    // residual: thread j fetches x of row r0 + j now, for the epilogue
    float xres = 0.f;
    if (MODE == M_RESID && (int)threadIdx.x < r1 - r0) xres = __ldcg(a.out + r0 + threadIdx.x);
    if (fits) f32_post_load(a, pre, xs, red);
    else load_input_f32_wide(a, token, xs, red);
    __syncthreads();
    const int kp4 = (a.K >> 2) / ks;  // float4 per slice
    const int nunits = (r1 - r0) * ks;
    for (int u = warp; u < nunits; u += nwarps) {
        const int rr = u / ks, p = u - rr * ks;
        float acc[1];
        dot_rows_f32<1, 8>(W + (size_t)(r0 + rr) * a.ld + (size_t)p * kp4 * 4, a.ld, kp4,
                           reinterpret_cast<const float4*>(xs) + (size_t)p * kp4, pol, acc);
        if (lane == 0) part[u] = acc[0];
    }
    if (a.late_trigger) grid_dep_launch();
    __syncthreads();
    unsigned long long best = 0ull;
    for (int j = threadIdx.x; j < (r1 - r0) / PAIR; j += blockDim.x) {
        float v[PAIR];
#pragma unroll
        for (int q = 0; q < PAIR; q++) {
            float t = 0.f;
            for (int p = 0; p < ks; p++) t += part[(PAIR * j + q) * ks + p];
            v[q] = t;
        }
        const int r = r0 + PAIR * j;
        if (MODE == M_QKV) {
            epi_qkv(a, r / 2, v[0], v[PAIR - 1], pos, rope_cs);
        } else if (MODE == M_W13) {
            epi_w13(a, r / 2, v[0], v[PAIR - 1]);
        } else if (MODE == M_RESID) {
            a.out[r] = (j == (int)threadIdx.x ? xres : __ldcg(a.out + r)) + v[0];
        } else {
            a.out[r] = v[0];
            if (v[0] != v[0]) set_error(a.err, DERR_NAN);
            unsigned long long k = argmax_key(v[0], r);
            best = k > best ? k : best;
        }
    }
    if (MODE == M_CLS) {
        for (int o = 16; o > 0; o >>= 1) {
            unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other > best ? other : best;
        }
        if (lane == 0) best_s[warp] = best;
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned long long b = 0ull;
            for (int i = 0; i < nwarps; i++) b = best_s[i] > b ? best_s[i] : b;
            if (b) atomicMax(a.amax, b);
        }
    }
}

// ------------------------------------------------------------ Q8_0 GEMV ------

// Quantizes the input vector x[0..K) (already in shared memory as fp32) into
// codes and scales in shared memory, one warp per group, with the rule of the
// quantize() listing: scale = max|x| / 127 in fp32, code = round(x / scale)
// (fp32 quotient, half away from zero); a zero group gets scale 0, codes 0.
__device__ __forceinline__ float quantize_group_warp(const float* x, int gs, int8_t* q, float* s) {
    const int lane = threadIdx.x & 31;
    float m = 0.f;
    for (int i = lane; i < gs; i += 32) m = fmaxf(m, fabsf(x[i]));
    m = warp_max(m);
    float scale = m / 127.0f;
    for (int i = lane; i < gs; i += 32) {
        float v = scale == 0.f ? 0.f : roundf(x[i] / scale);
        q[i] = (int8_t)(int)v;
    }
    if (lane == 0 && s) *s = scale;
    return scale;
}

// The value of input element i of a Q8_0 GEMV: the embedding row on layer 0
// (code * scale in fp32), else the input vector; RMSNorm'd (double, rounded
// once to fp32) when norm_w is set.
__device__ __forceinline__ float q8_input_value(const GemvArgs& a, const int8_t* eq, const float* es, double inv,
                                                int i) {
    float v = eq ? (float)eq[i] * es[i / a.gs] : __ldcg(a.in + i);
    if (a.norm_w) v = (float)((double)a.norm_w[i] * (inv * (double)v));
    return v;
}

// Quantizes the GEMV input (embedding row or input vector, RMSNorm'd when
// norm_w is set) into shared codes and scales, for any group size: one group
// at a time straight from global memory.  Every thread of `sy` calls it.
template <typename SY>
__device__ __noinline__ void q8_quantize_input_loop(const GemvArgs& a, const int8_t* eq, const float* es, int8_t* xq,
                                                    float* xsc, double* red, const SY sy) {
    const int nt = sy.nthreads(), lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = nt >> 5;
    const int K = a.K, gs = a.gs;
    double inv = 1.0;
    if (a.norm_w) {
        double ss = 0.0;
        for (int i = threadIdx.x; i < K; i += nt) {
            const float v = eq ? (float)eq[i] * es[i / gs] : __ldcg(a.in + i);
            ss += (double)v * (double)v;
        }
        ss = warp_sum(ss);
        if (lane == 0) red[warp] = ss;
        sy.sync();
        double tot = 0.0;
        for (int i = 0; i < nw; i++) tot += red[i];
        inv = 1.0 / sqrt(tot / (double)K + 1e-5);
    }
    if (a.emb && blockIdx.x == 0)
        for (int i = threadIdx.x; i < K; i += nt) a.x_resid[i] = (float)eq[i] * es[i / gs];
    for (int g = warp; g < K / gs; g += nw) {
        float m = 0.f;
        for (int i = lane; i < gs; i += 32) m = fmaxf(m, fabsf(q8_input_value(a, eq, es, inv, g * gs + i)));
        m = warp_max(m);
        const float scale = m / 127.0f;
        for (int i = lane; i < gs; i += 32) {
            const float v = q8_input_value(a, eq, es, inv, g * gs + i);
            xq[g * gs + i] = (int8_t)(int)(scale == 0.f ? 0.f : roundf(v / scale));
        }
        if (lane == 0) xsc[g] = scale;
    }
}

// Fast path for gs = 32 * EPL.  Pass 1 (RMSNorm only): the sum of squares
// from 16-byte loads, four in flight per thread.  Pass 2: warp w quantizes its
// groups w, w + nw, ... in batches of QB, issuing the loads of a whole batch
// before using them.  A few round trips to L2 in all, with little code.
template <int EPL, bool NORM, typename SY>
__device__ __forceinline__ void q8_quantize_input_batched(const GemvArgs& a, const int8_t* eq, const float* es,
                                                          int8_t* xq, float* xsc, double* red, const SY& sy) {
    constexpr int QB = 8;
    const int nt = sy.nthreads(), lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = nt >> 5;
    const int K = a.K, gs = 32 * EPL;
    const int ng = K / gs;
    if (NORM) {
        // the whole vector and gain in registers (one round trip): the sum of
        // squares and the codes both come from the same loaded values
        constexpr int GM = 16 / EPL;
        if ((ng + nw - 1) / nw <= GM) {
            float v[GM][EPL], w[GM][EPL];
#pragma unroll
            for (int j = 0; j < GM; j++) {
                const int g = warp + j * nw;
#pragma unroll
                for (int e = 0; e < EPL; e++) {
                    const int i = g * gs + lane + 32 * e;
                    v[j][e] = g < ng ? (eq ? (float)eq[i] * es[g] : __ldcg(a.in + i)) : 0.f;
                    w[j][e] = g < ng ? a.norm_w[i] : 0.f;
                }
            }
            double ss = 0.0;
#pragma unroll
            for (int j = 0; j < GM; j++)
#pragma unroll
                for (int e = 0; e < EPL; e++) ss += (double)v[j][e] * (double)v[j][e];
            ss = warp_sum(ss);
            if (lane == 0) red[warp] = ss;
            sy.sync();
            double tot = 0.0;
            for (int i = 0; i < nw; i++) tot += red[i];
            const double inv = 1.0 / sqrt(tot / (double)K + 1e-5);
#pragma unroll
            for (int j = 0; j < GM; j++) {
                const int g = warp + j * nw;
                if (g < ng) {  // warp-uniform
                    if (a.emb && blockIdx.x == 0) {
#pragma unroll
                        for (int e = 0; e < EPL; e++) a.x_resid[g * gs + lane + 32 * e] = v[j][e];
                    }
                    float m = 0.f;
#pragma unroll
                    for (int e = 0; e < EPL; e++) {
                        v[j][e] = (float)((double)w[j][e] * (inv * (double)v[j][e]));
                        m = fmaxf(m, fabsf(v[j][e]));
                    }
                    m = warp_max(m);
                    const float scale = m / 127.0f;
#pragma unroll
                    for (int e = 0; e < EPL; e++) {
                        const float q = scale == 0.f ? 0.f : roundf(v[j][e] / scale);
                        xq[g * gs + lane + 32 * e] = (int8_t)(int)q;
                    }
                    if (lane == 0) xsc[g] = scale;
                }
            }
            return;
        }
    }
    double inv = 1.0;
    if (NORM) {
        double ss = 0.0;
        const int K4 = K >> 2;
#pragma unroll 4
        for (int i4 = threadIdx.x; i4 < K4; i4 += nt) {
            float4 v;
            if (eq) {
                const char4 c4 = reinterpret_cast<const char4*>(eq)[i4];
                const float sc = es[(4 * i4) / gs];
                v = make_float4((float)c4.x * sc, (float)c4.y * sc, (float)c4.z * sc, (float)c4.w * sc);
            } else {
                v = __ldcg(reinterpret_cast<const float4*>(a.in) + i4);
            }
            ss += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
        }
        ss = warp_sum(ss);
        if (lane == 0) red[warp] = ss;
        sy.sync();
        double tot = 0.0;
        for (int i = 0; i < nw; i++) tot += red[i];
        inv = 1.0 / sqrt(tot / (double)K + 1e-5);
    }
    for (int g0 = warp; g0 < ng; g0 += QB * nw) {
        float v[QB][EPL];
        float w[NORM ? QB : 1][EPL];
#pragma unroll
        for (int j = 0; j < QB; j++) {
            const int g = g0 + j * nw;
#pragma unroll
            for (int e = 0; e < EPL; e++) {
                const int i = g * gs + lane + 32 * e;
                v[j][e] = g < ng ? (eq ? (float)eq[i] * es[g] : __ldcg(a.in + i)) : 0.f;
                if (NORM) w[NORM ? j : 0][e] = g < ng ? a.norm_w[i] : 0.f;
            }
        }
#pragma unroll
        for (int j = 0; j < QB; j++) {
            const int g = g0 + j * nw;
            if (g < ng) {  // warp-uniform
                if (a.emb && blockIdx.x == 0) {
#pragma unroll
                    for (int e = 0; e < EPL; e++) a.x_resid[g * gs + lane + 32 * e] = v[j][e];
                }
                float m = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; e++) {
                    if (NORM) v[j][e] = (float)((double)w[NORM ? j : 0][e] * (inv * (double)v[j][e]));
                    m = fmaxf(m, fabsf(v[j][e]));
                }
                m = warp_max(m);
                const float scale = m / 127.0f;
#pragma unroll
                for (int e = 0; e < EPL; e++) {
                    const float q = scale == 0.f ? 0.f : roundf(v[j][e] / scale);
                    xq[g * gs + lane + 32 * e] = (int8_t)(int)q;
                }
                if (lane == 0) xsc[g] = scale;
            }
        }
    }
}

// Quantizes the GEMV input (embedding row or input vector, RMSNorm'd when
// norm_w is set) into shared codes and scales; every thread of the CTA calls
// it.
template <bool NORM, typename SY = SyncCTA>
__device__ __forceinline__ void q8_quantize_input(const GemvArgs& a, const int8_t* eq, const float* es, int8_t* xq,
                                                  float* xsc, double* red, const SY sy = SY()) {
    if (a.gs == 32) q8_quantize_input_batched<1, NORM>(a, eq, es, xq, xsc, red, sy);
    else if (a.gs == 64) q8_quantize_input_batched<2, NORM>(a, eq, es, xq, xsc, red, sy);
    else if (a.gs == 128) q8_quantize_input_batched<4, NORM>(a, eq, es, xq, xsc, red, sy);
    else q8_quantize_input_loop(a, eq, es, xq, xsc, red, sy);
}

// The exact int32 group dots of one 64-byte chunk of a row.  Lane chunk t
// covers bytes [64t, 64t+64) of the row and of the input codes: one group at
// GS = 64 (g[0]), two at GS = 32 (g[0], g[1]), half of one at GS = 128 (the
// lane pair 2m, 2m+1 adds its halves with one shuffle, so every lane of the
// warp must call it; both lanes of a pair hold the group's dot in g[0]).  The
// four 16-byte reads are rotated by rot = (lane >> 1) & 3 so that a
// quarter-warp touches eight distinct 16-byte bank groups; xv holds the input
// chunks in that rotated order.  Out-of-range lanes (in = false) read nothing.
template <int GS>
__device__ __forceinline__ void q8_chunk_dots(const uint8_t* row, const int4 (&xv)[4], int t, bool in, int rot,
                                              int (&g)[GS == 32 ? 2 : 1]) {
    int c[4];
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const int f = (j + rot) & 3;
        const int4 wv = in ? *reinterpret_cast<const int4*>(row + 64 * t + 16 * f) : make_int4(0, 0, 0, 0);
        int dd = __dp4a(wv.x, xv[j].x, 0);
        dd = __dp4a(wv.y, xv[j].y, dd);
        dd = __dp4a(wv.z, xv[j].z, dd);
        c[j] = __dp4a(wv.w, xv[j].w, dd);
    }
    if (GS == 32) {
        // chunk f: the lane's first group is made of chunks f < 2
        int lo = 0, hi = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int f = (j + rot) & 3;
            lo += f < 2 ? c[j] : 0;
            hi += f < 2 ? 0 : c[j];
        }
        g[0] = lo;
        g[GS == 32 ? 1 : 0] = hi;
    } else {
        int d = (c[0] + c[1]) + (c[2] + c[3]);
        if (GS == 128) d += __shfl_xor_sync(0xffffffffu, d, 1);
        g[0] = d;
    }
}

// The input codes of lane chunk t, in the rotated order of q8_chunk_dots.
__device__ __forceinline__ void q8_chunk_x(const int8_t* xq, int t, bool in, int rot, int4 (&xv)[4]) {
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const int f = (j + rot) & 3;
        xv[j] = in ? *reinterpret_cast<const int4*>(xq + 64 * t + 16 * f) : make_int4(0, 0, 0, 0);
    }
}

// x * 2^-896 as a double, exactly, for every finite float x: the float's bits
// with the exponent left unbiased (integer operations only; the conversion
// instruction issues on a narrow unit).
__device__ __forceinline__ double widen_f32_scaled(float x) {
    const uint32_t b = __float_as_uint(x);
    const uint32_t hi = ((b & 0x7fffffffu) >> 3) | (b & 0x80000000u);
    return __hiloint2double((int)hi, (int)(b << 29));
}

// UR rows (records at rec, stride rb) against the input codes xq: the exact
// group dots of q8_chunk_dots, each times the row's group scale and the
// input's group scale, summed per lane in double.  The input scales (fp32,
// xs) are converted once per chunk and times 2^896, the row scales widened
// as sw * 2^-896, so each term is the double product (ival * sw) * sx.
// Requires K % 64 == 0.
template <int GS, int UR>
__device__ __forceinline__ void q8_rows_dot64(const uint8_t* rec, size_t rb, const int8_t* xq, const float* xs,
                                              int K, double (&acc)[UR]) {
    const int lane = threadIdx.x & 31;
    const int n64 = K >> 6;
    const int rot = (lane >> 1) & 3;
#pragma unroll
    for (int r = 0; r < UR; r++) acc[r] = 0.0;
#pragma unroll 2
    for (int t0 = 0; t0 < n64; t0 += 32) {
        const int t = t0 + lane;
        const bool in = t < n64;
        int4 xv[4];
        q8_chunk_x(xq, t, in, rot, xv);
        double sx0 = 0.0, sx1 = 0.0;
        if (in) {
            if (GS == 64) sx0 = (double)xs[t] * 0x1p896;
            else if (GS == 32) { sx0 = (double)xs[2 * t] * 0x1p896; sx1 = (double)xs[2 * t + 1] * 0x1p896; }
            else sx0 = (double)xs[t >> 1] * 0x1p896;
        }
#pragma unroll
        for (int r = 0; r < UR; r++) {
            const uint8_t* row = rec + r * rb;
            int gd[GS == 32 ? 2 : 1];
            q8_chunk_dots<GS>(row, xv, t, in, rot, gd);
            const float* sw = reinterpret_cast<const float*>(row + K);
            if (!in) continue;
            if (GS == 64) {
                acc[r] = fma(i2d_exact(gd[0]) * widen_f32_scaled(sw[t]), sx0, acc[r]);
            } else if (GS == 32) {
                acc[r] = fma(i2d_exact(gd[0]) * widen_f32_scaled(sw[2 * t]), sx0, acc[r]);
                acc[r] = fma(i2d_exact(gd[GS == 32 ? 1 : 0]) * widen_f32_scaled(sw[2 * t + 1]), sx1, acc[r]);
            } else if ((t & 1) == 0) {  // GS == 128: the even lane of the pair
                acc[r] = fma(i2d_exact(gd[0]) * widen_f32_scaled(sw[t >> 1]), sx0, acc[r]);
            }
        }
    }
}

// Q4_0 row records: [K/2 bytes of 4-bit codes | K/GS fp32 scales | pad to
// 16 B], each code stored as code + 8 (1..15 for codes in [-7, 7]).  Two
// layouts of the code bytes: with K % 64 == 0 the values 64t..64t+63 (chunk
// t) sit in the 32 bytes at 32t, byte b holding value 64t+b in its low
// nibble and 64t+32+b in its high one (q4_rows_dot64); otherwise (K an odd
// multiple of 32, GS = 32) the values 32t..32t+31 sit in the 16 bytes at 16t,
// byte b holding 32t+b low and 32t+16+b high (q4_rows_dot32).
__host__ __device__ inline size_t q4_record_bytes(int K, int gs) {
    return (size_t)K / 2 + (((size_t)(K / gs) * 4 + 15) & ~size_t(15));
}

// UR Q4_0 rows (records at rec, stride rb) against the Q8_0 input codes xq:
// per lane chunk t one 16-byte load of a row and two of the input (its
// halves read in the order h = j ^ r, r = bit 2 of the lane, so that the
// eight lanes of a quarter-warp touch distinct 16-byte bank groups).  The
// low nibbles of a row chunk pair with input half 0, the high ones with half
// 1; the chunk's exact dot is sum((code + 8) * x) - corr[t], corr[t] = 8 *
// (sum of the chunk's input codes), and the CPG = GS/32 chunks of a group
// (consecutive lanes) add up with shuffles.  Each group's exact int32 dot
// times the row's group scale and the input's, summed per lane in double as
// in q8_rows_dot64.  Requires K % 32 == 0, GS in {32, 64, 128}, K % GS == 0.
template <int GS, int UR>
__device__ __forceinline__ void q4_rows_dot32(const uint8_t* rec, size_t rb, const int8_t* xq, const float* xs,
                                              const int* corr, int K, double (&acc)[UR]) {
    constexpr int CPG = GS / 32;
    const int lane = threadIdx.x & 31;
    const int n32 = K >> 5;
    const int r = (lane >> 2) & 1;
#pragma unroll
    for (int u = 0; u < UR; u++) acc[u] = 0.0;
#pragma unroll 2
    for (int t0 = 0; t0 < n32; t0 += 32) {
        const int t = t0 + lane;
        const bool in = t < n32;
        int4 xv[2];
#pragma unroll
        for (int j = 0; j < 2; j++)
            xv[j] = in ? *reinterpret_cast<const int4*>(xq + 32 * t + 16 * (j ^ r)) : make_int4(0, 0, 0, 0);
        const int cr = in ? corr[t] : 0;
        const bool head = in && (t & (CPG - 1)) == 0;  // the lane that holds its group's dot
        const double sx = head ? (double)xs[t / CPG] * 0x1p896 : 0.0;
#pragma unroll
        for (int u = 0; u < UR; u++) {
            const uint8_t* row = rec + u * rb;
            const int4 wv = in ? *reinterpret_cast<const int4*>(row + 16 * t) : make_int4(0, 0, 0, 0);
            int dd = -cr;
#pragma unroll
            for (int j = 0; j < 2; j++) {
                const int sh = 4 * (j ^ r);
                dd = __dp4a((int)(((uint32_t)wv.x >> sh) & 0x0f0f0f0fu), xv[j].x, dd);
                dd = __dp4a((int)(((uint32_t)wv.y >> sh) & 0x0f0f0f0fu), xv[j].y, dd);
                dd = __dp4a((int)(((uint32_t)wv.z >> sh) & 0x0f0f0f0fu), xv[j].z, dd);
                dd = __dp4a((int)(((uint32_t)wv.w >> sh) & 0x0f0f0f0fu), xv[j].w, dd);
            }
#pragma unroll
            for (int o = 1; o < CPG; o <<= 1) dd += __shfl_xor_sync(0xffffffffu, dd, o);
            if (head) {
                const float* sw = reinterpret_cast<const float*>(row + K / 2);
                acc[u] = fma(i2d_exact(dd) * widen_f32_scaled(sw[t / CPG]), sx, acc[u]);
            }
        }
    }
}

// d + sum of the four byte products of a (unsigned bytes) and b (signed bytes).
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int d) {
    int r;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(d));
    return r;
}

// UR Q4_0 rows in the 64-value chunk layout against the Q8_0 input codes xq.
// Lane chunk t: two 16-byte loads of a row (halves h) and four of the input
// (quarters f).  Quarter f pairs with the low (f < 2) or high nibbles of half
// f & 1.  The loads are rotated so that the eight lanes of a quarter-warp
// touch distinct 16-byte bank groups: with rot = bit 2 of the lane | (bit 1 of
// the lane) << 1, input slot j holds quarter j ^ rot and row register jj half
// jj ^ (rot & 1), so slot j pairs with register j & 1 and a nibble picked by
// a per-lane mask.  The high nibbles are taken in place (byte = 16 * code),
// so one AND per word: sum over slots 0-1 and 2-3 with unsigned-by-signed
// dp4a, then lo + (hi >> 4) - corr per group (corr = 8 * the input codes'
// sum over 32 values).  Group scaling as in q8_rows_dot64.  Requires K % 64
// == 0, GS in {32, 64, 128}.
template <int GS, int UR>
__device__ __forceinline__ void q4_rows_dot64(const uint8_t* rec, size_t rb, const int8_t* xq, const float* xs,
                                              const int* corr, int K, double (&acc)[UR]) {
    const int lane = threadIdx.x & 31;
    const int n64 = K >> 6;
    const int rot = ((lane >> 2) & 1) | (lane & 2);
    const uint32_t mA = (rot >> 1) ? 0xf0f0f0f0u : 0x0f0f0f0fu;  // nibble of slots 0, 1
    const uint32_t mB = ~mA;                                      // nibble of slots 2, 3
#pragma unroll
    for (int u = 0; u < UR; u++) acc[u] = 0.0;
#pragma unroll 2
    for (int t0 = 0; t0 < n64; t0 += 32) {
        const int t = t0 + lane;
        const bool in = t < n64;
        int4 xv[4];
#pragma unroll
        for (int j = 0; j < 4; j++)
            xv[j] = in ? *reinterpret_cast<const int4*>(xq + 64 * t + 16 * (j ^ rot)) : make_int4(0, 0, 0, 0);
        const int2 cr = in ? *reinterpret_cast<const int2*>(corr + 2 * t) : make_int2(0, 0);
        double sx0 = 0.0, sx1 = 0.0;
        if (in) {
            if (GS == 64) sx0 = (double)xs[t] * 0x1p896;
            else if (GS == 32) { sx0 = (double)xs[2 * t] * 0x1p896; sx1 = (double)xs[2 * t + 1] * 0x1p896; }
            else sx0 = (double)xs[t >> 1] * 0x1p896;
        }
#pragma unroll
        for (int u = 0; u < UR; u++) {
            const uint8_t* row = rec + u * rb;
            int4 wv[2];
#pragma unroll
            for (int jj = 0; jj < 2; jj++)
                wv[jj] = in ? *reinterpret_cast<const int4*>(row + 32 * t + 16 * (jj ^ (rot & 1)))
                            : make_int4(0, 0, 0, 0);
            int sA = 0, sB = 0;
#pragma unroll
            for (int j = 0; j < 2; j++) {
                const int4 w = wv[j];
                sA = dp4a_us((uint32_t)w.x & mA, xv[j].x, sA);
                sA = dp4a_us((uint32_t)w.y & mA, xv[j].y, sA);
                sA = dp4a_us((uint32_t)w.z & mA, xv[j].z, sA);
                sA = dp4a_us((uint32_t)w.w & mA, xv[j].w, sA);
                sB = dp4a_us((uint32_t)w.x & mB, xv[j + 2].x, sB);
                sB = dp4a_us((uint32_t)w.y & mB, xv[j + 2].y, sB);
                sB = dp4a_us((uint32_t)w.z & mB, xv[j + 2].z, sB);
                sB = dp4a_us((uint32_t)w.w & mB, xv[j + 2].w, sB);
            }
            const int lo = (rot >> 1) ? sB : sA;         // quarters 0, 1: values 64t..64t+31
            const int hi = ((rot >> 1) ? sA : sB) >> 4;  // quarters 2, 3 (16 * code, exact shift)
            const float* sw = reinterpret_cast<const float*>(row + K / 2);
            if (GS == 32) {
                if (in) {
                    acc[u] = fma(i2d_exact(lo - cr.x) * widen_f32_scaled(sw[2 * t]), sx0, acc[u]);
                    acc[u] = fma(i2d_exact(hi - cr.y) * widen_f32_scaled(sw[2 * t + 1]), sx1, acc[u]);
                }
            } else {
                int dd = lo + hi - (cr.x + cr.y);
                if (GS == 128) dd += __shfl_xor_sync(0xffffffffu, dd, 1);
                if (in && (GS == 64 || (t & 1) == 0))
                    acc[u] = fma(i2d_exact(dd) * widen_f32_scaled(sw[GS == 64 ? t : (t >> 1)]), sx0, acc[u]);
            }
        }
    }
}

// Input quantization of the 64-byte-per-lane Q8_0 path (K % 64 == 0, GS 32,
// 64 or 128), split around the dependency wait.  The input is taken in chunks
// of 64 values, two per warp step: half-warp h of warp w takes chunk
// 2*(w + NW*it) + h, its lane i the values 4i..4i+3 (one 16-byte load).  A
// group is 8, 16 or 32 lanes, so its max is 3, 4 or 5 shuffles, and a lane
// packs its four codes into one 32-bit store.  With an RMSNorm the values
// stay in registers (at most MAXIT steps) between the sum of squares and the
// codes; the gain, and on layer 0 the embedding row, are loaded before the
// wait (no kernel of the step writes them).  Arithmetic as the listing's rule
// and RMSNorm elsewhere: sums of squares in double, w * (inv * x) in double
// rounded once to fp32, scale = max|x| / 127 in fp32, code = round(x / scale).
template <int GS, bool NORM, int NW, int MAXIT>
struct Q8Prologue {
    static constexpr int IT = NORM ? MAXIT : 1;
    float4 v[IT], w[IT];
    int steps;

    // whether the input fits this path
    static __device__ __forceinline__ bool fits(const GemvArgs& a) {
        if (a.K % 64 || a.gs != GS) return false;
        const int npair = (a.K / 64 + 1) / 2;
        return !NORM || (npair + NW - 1) / NW <= MAXIT;
    }
    __device__ __forceinline__ int chunk(int it) const {
        return 2 * ((threadIdx.x >> 5) + NW * it) + ((threadIdx.x >> 4) & 1);
    }
    __device__ __forceinline__ float4 load_value(const GemvArgs& a, const int8_t* eq, const float* es, int it) const {
        const int c = chunk(it), i = threadIdx.x & 15;
        if (c >= a.K / 64) return make_float4(0.f, 0.f, 0.f, 0.f);
        const int idx = c * 64 + 4 * i;
        if (eq) {
            const char4 q = *reinterpret_cast<const char4*>(eq + idx);
            const float sc = es[idx / a.gs];
            return make_float4((float)q.x * sc, (float)q.y * sc, (float)q.z * sc, (float)q.w * sc);
        }
        return __ldcg(reinterpret_cast<const float4*>(a.in + idx));
    }
    // before the wait: the gain and the embedding row
    __device__ __forceinline__ void pre(const GemvArgs& a, const int8_t* eq, const float* es) {
        const int npair = (a.K / 64 + 1) / 2;
        steps = (npair - (int)(threadIdx.x >> 5) + NW - 1) / NW;
        if (NORM) {
#pragma unroll
            for (int it = 0; it < IT; it++) {
                const int c = chunk(it);
                const bool on = it < steps && c < a.K / 64;
                w[it] = on ? *reinterpret_cast<const float4*>(a.norm_w + c * 64 + 4 * (threadIdx.x & 15))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
                if (eq) v[it] = on ? load_value(a, eq, es, it) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    }
    // the group max, scale and codes of the four values of step `it`
    __device__ __forceinline__ void quantize(const GemvArgs& a, float4 x, int it, int8_t* xq, float* xsc) const {
        const int c = chunk(it), i = threadIdx.x & 15;
        float m = fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w)));
        constexpr int LANES = GS / 4;  // lanes of one group
#pragma unroll
        for (int o = 1; o < LANES; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (c >= a.K / 64) return;
        const float scale = m / 127.0f;
        int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
        if (scale != 0.f) {
            q0 = (int)roundf(x.x / scale); q1 = (int)roundf(x.y / scale);
            q2 = (int)roundf(x.z / scale); q3 = (int)roundf(x.w / scale);
        }
        *reinterpret_cast<uint32_t*>(xq + c * 64 + 4 * i) =
            (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) | ((uint32_t)(q2 & 0xff) << 16) |
            ((uint32_t)(q3 & 0xff) << 24);
        if ((threadIdx.x & (LANES - 1)) == 0) xsc[(c * 64 + 4 * i) / GS] = scale;
    }
    // after the wait: the input, the RMSNorm, the codes
    __device__ __forceinline__ void post(const GemvArgs& a, const int8_t* eq, const float* es, int8_t* xq, float* xsc,
                                         double* red) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const bool resid = a.emb && blockIdx.x == 0;  // layer 0: CTA 0 stores the embedding row as x
        if (!NORM) {
            // the loads of a block of steps first, all in flight, then the codes
            constexpr int RB = 12;
            for (int i0 = 0; i0 < steps; i0 += RB) {
                float4 xs[RB];
#pragma unroll
                for (int k = 0; k < RB; k++)
                    xs[k] = i0 + k < steps ? load_value(a, eq, es, i0 + k) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int k = 0; k < RB; k++) {
                    if (i0 + k >= steps) break;  // warp-uniform
                    const int it = i0 + k;
                    if (resid && chunk(it) < a.K / 64)
                        reinterpret_cast<float4*>(a.x_resid)[(chunk(it) * 64 + 4 * (threadIdx.x & 15)) / 4] = xs[k];
                    quantize(a, xs[k], it, xq, xsc);
                }
            }
            return;
        }
        if (!eq) {
#pragma unroll
            for (int it = 0; it < IT; it++)
                v[it] = it < steps ? load_value(a, eq, es, it) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        double ss = 0.0;
#pragma unroll
        for (int it = 0; it < IT; it++) {
            ss += (double)v[it].x * (double)v[it].x + (double)v[it].y * (double)v[it].y;
            ss += (double)v[it].z * (double)v[it].z + (double)v[it].w * (double)v[it].w;
            if (resid && it < steps && chunk(it) < a.K / 64)
                reinterpret_cast<float4*>(a.x_resid)[(chunk(it) * 64 + 4 * (threadIdx.x & 15)) / 4] = v[it];
        }
        ss = warp_sum(ss);
        if (lane == 0) red[warp] = ss;
        __syncthreads();
        double tot = 0.0;
#pragma unroll
        for (int k = 0; k < NW; k++) tot += red[k];
        const double inv = 1.0 / sqrt(tot / (double)a.K + 1e-5);
#pragma unroll
        for (int it = 0; it < IT; it++) {
            if (it >= steps) break;  // warp-uniform
            float4 x = v[it];
            x.x = (float)((double)w[it].x * (inv * (double)x.x));
            x.y = (float)((double)w[it].y * (inv * (double)x.y));
            x.z = (float)((double)w[it].z * (inv * (double)x.z));
            x.w = (float)((double)w[it].w * (inv * (double)x.w));
            quantize(a, x, it, xq, xsc);
        }
    }
};

constexpr int Q8_WARPS = 8;                  // warps of a Q8_0 GEMV CTA
constexpr int Q8_THREADS = 32 * Q8_WARPS;

// A Q8_0 GEMV CTA's rings: `ns` slots per warp of one unit (UNIT row
// records) each.
struct Q8Ring {
    int ns;
    uint32_t unit_bytes;  // UNIT * record bytes
};

// Q8_0 / Q4_0 GEMV.  A unit is UM row records, or UM row pairs for QKV and
// W1/W3 (UNIT rows); the CTA owns a contiguous range of units and warp w takes its
// units w, w + 8, ..., streaming them with 1-D bulk copies through its own
// ring of `ns` shared-memory slots: its parity waits follow its own copies in
// order, and it refills a slot as soon as it has read it.  Before the
// dependency wait the kernel loads what no earlier kernel of the step writes
// (the RMSNorm gain, the embedding row on layer 0, the RoPE table) and
// prefetches the first a.prefetch_bytes of the CTA's weights into L2; right
// after it, the rings are filled and the input is quantized (the listing's
// rule, bit-exact) into shared codes.  Then per unit: exact int32 group dots
// by dp4a, (ival * sw) * sx summed per lane in double, one reduce-scatter for
// the unit's row sums, the epilogue.  GS is the group size of the
// 64-byte-per-lane dot (32, 64 or 128, K % 64 == 0), or 0 for the generic
// 16-byte-per-lane loop.  W4 = 0: Q8_0 row records; 1, 2: Q4_0 records in the
// 32- or 64-value chunk layout (q4_rows_dot32 / q4_rows_dot64), whose input
// code sums are computed once per CTA after the quantization.  Every wait is bounded (a.wait_ns); a warp that gives
// up records DERR_TIMEOUT, makes the others stop (a shared abort flag) and
// lets its copies in flight land before the CTA leaves.  Dynamic shared
// memory: the rings [Q8_WARPS][ns][unit], the input codes and scales, the
// barriers.
struct Q8Smem {
    size_t xq, xsc, sxd, bars, total;
};

// sxd holds the input's double scales (generic Q8_0 path) or the Q4_0
// chunk corrections (K/32 ints).
__host__ __device__ inline Q8Smem q8_smem(int ns, uint32_t unit_bytes, int K, int gs) {
    Q8Smem m;
    const size_t ng = (size_t)(K / gs);
    const size_t aux = ng * 8 > (size_t)(K / 32) * 4 ? ng * 8 : (size_t)(K / 32) * 4;
    m.xq = (size_t)Q8_WARPS * ns * unit_bytes;
    m.xsc = m.xq + (((size_t)K + 15) & ~size_t(15));
    m.sxd = m.xsc + ((ng * 4 + 15) & ~size_t(15));
    m.bars = m.sxd + ((aux + 7) & ~size_t(7));
    m.total = m.bars + 8 * (size_t)Q8_WARPS * ns;
    return m;
}

template <int MODE, int GS, int W4 = 0, int UM = 1>
__global__ void __launch_bounds__(Q8_THREADS, 1) k_gemv_q8(const GemvArgs a, const Q8Ring R) {
    extern __shared__ __align__(128) uint8_t smem[];
    // rows per unit: pairs for QKV and W1/W3 (RoPE / SwiGLU pairs), single rows
    // otherwise, times UM (1, 2 or 4): more rows per unit give a warp more independent
    // dot chains for the same ring bytes (the 4-bit rows are half the bytes)
    constexpr int UNIT = ((MODE == M_QKV || MODE == M_W13) ? 2 : 1) * UM;
    static_assert(UNIT <= 8, "warp_sum_scatter takes at most 8 rows");
    __shared__ double red[Q8_WARPS];
    __shared__ unsigned long long best_s[Q8_WARPS];
    __shared__ double2 rope_cs[MODE == M_QKV ? 128 : 1];
    __shared__ int abort_s;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int K = a.K, gs = a.gs, ns = R.ns;
    const uint32_t ub = R.unit_bytes;  // UNIT * record bytes
    const size_t rb = a.ld;
    const Q8Smem lay = q8_smem(ns, ub, K, gs);
    uint8_t* slots = smem + (size_t)warp * ns * ub;
    int8_t* xq = reinterpret_cast<int8_t*>(smem + lay.xq);
    float* xsc = reinterpret_cast<float*>(smem + lay.xsc);
    double* sxd = reinterpret_cast<double*>(smem + lay.sxd);  // generic path only
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars) + warp * ns;
    const int units = a.rows / UNIT;
    const int u0 = (int)((long long)units * blockIdx.x / gridDim.x);
    const int u1 = (int)((long long)units * (blockIdx.x + 1) / gridDim.x);
    const int nmine = (u1 - u0 - warp + Q8_WARPS - 1) / Q8_WARPS;  // units of this warp
    const uint8_t* Wb = static_cast<const uint8_t*>(a.W);
    const uint64_t pol = policy_evict_first();
    auto unit_src = [&](int k) { return Wb + (size_t)(u0 + warp + k * Q8_WARPS) * ub; };
    if (lane == 0) {
        for (int s = 0; s < ns; s++) mbar_init(&full[s], 1);
        mbar_fence_init();
    }
    if (threadIdx.x == 0) abort_s = 0;
    if (a.early) grid_dep_launch();
    // before the dependency wait: what earlier kernels of the step do not write
    constexpr bool NORM = MODE != M_RESID;
    Q8Prologue<GS == 0 ? 64 : GS, NORM, Q8_WARPS, 8> pro;
    const bool fast = GS != 0 && (NORM == (a.norm_w != nullptr)) && pro.fits(a);
    int token = 0, pos = 0;
    if (MODE == M_QKV) read_tp(a, token, pos);
    const int8_t* eq = nullptr;
    const float* es = nullptr;
    if (a.emb) {
        // the embedding rows are Q8_0-layout records (holding 4-bit codes beside Q4_0 weights)
        const size_t erb = W4 ? (size_t)K + (((size_t)(K / gs) * 4 + 15) & ~size_t(15)) : rb;
        const uint8_t* rec = static_cast<const uint8_t*>(a.emb) + (size_t)token * erb;
        eq = reinterpret_cast<const int8_t*>(rec);
        es = reinterpret_cast<const float*>(rec + K);
    }
    if (fast) pro.pre(a, eq, es);
    if (MODE == M_QKV) rope_table(a, pos, rope_cs);
    if (threadIdx.x == 0 && a.prefetch_bytes && u1 > u0) {
        size_t bytes = (size_t)(u1 - u0) * ub;
        if (bytes > a.prefetch_bytes) bytes = a.prefetch_bytes;
        prefetch_l2_range(Wb + (size_t)u0 * ub, bytes, policy_evict_last());
    }
    __syncthreads();  // barrier inits visible
    grid_dep_wait();
    // test switch: CTA 0's warp 0 withholds its first copy once (a wait then runs out)
    bool skip0 = false;
    if (threadIdx.x == 0) skip0 = a.stall && blockIdx.x == 0 && nmine > 0 && atomicExch(a.stall, 0);
    if (lane == 0) {
        for (int k = 0; k < ns && k < nmine; k++) {
            if (k == 0 && skip0) continue;
            mbar_arrive_expect_tx(&full[k], ub);
            bulk_g2s(slots + (size_t)k * ub, unit_src(k), ub, &full[k], pol);
        }
    }
    if (MODE == M_QKV && a.amax && blockIdx.x == 0 && threadIdx.x == 0) *a.amax = 0ull;
    // residual: lane j fetches the x of this warp's j-th unit (its UNIT rows), for the epilogue
    constexpr int XR = MODE == M_RESID ? UNIT : 1;
    float xres[XR];
#pragma unroll
    for (int r = 0; r < XR; r++) xres[r] = 0.f;
    if (MODE == M_RESID && lane < nmine) {
        const size_t r0 = (size_t)(u0 + warp + lane * Q8_WARPS) * UNIT;
#pragma unroll
        for (int r = 0; r < XR; r++) xres[r] = __ldcg(a.out + r0 + r);
    }
    if (fast) pro.post(a, eq, es, xq, xsc, red);
    else q8_quantize_input<NORM>(a, eq, es, xq, xsc, red);
    __syncthreads();
    if (GS == 0) {
        for (int g = threadIdx.x; g < K / gs; g += Q8_THREADS) sxd[g] = (double)xsc[g];
        __syncthreads();
    }
    int* corr = reinterpret_cast<int*>(smem + lay.sxd);  // Q4_0: 8 * (sum of the input codes) per 32-chunk
    if (W4) {
        for (int t = threadIdx.x; t < K / 32; t += Q8_THREADS) {
            const int4 c0 = *reinterpret_cast<const int4*>(xq + 32 * t);
            const int4 c1 = *reinterpret_cast<const int4*>(xq + 32 * t + 16);
            int sum = __dp4a(c0.x, 0x01010101, 0);
            sum = __dp4a(c0.y, 0x01010101, sum);
            sum = __dp4a(c0.z, 0x01010101, sum);
            sum = __dp4a(c0.w, 0x01010101, sum);
            sum = __dp4a(c1.x, 0x01010101, sum);
            sum = __dp4a(c1.y, 0x01010101, sum);
            sum = __dp4a(c1.z, 0x01010101, sum);
            sum = __dp4a(c1.w, 0x01010101, sum);
            corr[t] = 8 * sum;
        }
        __syncthreads();
    }

    const int nchunk = K >> 4, cpg = gs >> 4, iters = (nchunk + 31) >> 5;
    unsigned long long best = 0ull;
    int k = 0;
    for (; k < nmine; k++) {
        const int s = k % ns;
        if (!mbar_wait_bounded(&full[s], (k / ns) & 1, a.err, a.wait_ns, &abort_s)) {
            abort_s = 1;
            break;
        }
        const uint8_t* base = slots + (size_t)s * ub;
        double acc[UNIT];
        if (W4 == 2) {
            q4_rows_dot64<GS == 0 ? 64 : GS, UNIT>(base, rb, xq, xsc, corr, K, acc);
        } else if (W4 == 1) {
            q4_rows_dot32<GS == 0 ? 32 : GS, UNIT>(base, rb, xq, xsc, corr, K, acc);
        } else if (GS != 0) {
            q8_rows_dot64<GS == 0 ? 64 : GS, UNIT>(base, rb, xq, xsc, K, acc);
        } else {
#pragma unroll
            for (int r = 0; r < UNIT; r++) acc[r] = 0.0;
            for (int it = 0; it < iters; it++) {
                const int c = lane + 32 * it;
                const bool in = c < nchunk;
                int4 xv = in ? *reinterpret_cast<const int4*>(xq + 16 * c) : make_int4(0, 0, 0, 0);
#pragma unroll
                for (int r = 0; r < UNIT; r++) {
                    int dsum = 0;
                    if (in) {
                        const int4 wv = *reinterpret_cast<const int4*>(base + r * rb + 16 * c);
                        dsum = __dp4a(wv.x, xv.x, dsum);
                        dsum = __dp4a(wv.y, xv.y, dsum);
                        dsum = __dp4a(wv.z, xv.z, dsum);
                        dsum = __dp4a(wv.w, xv.w, dsum);
                    }
                    for (int o = 1; o < cpg; o <<= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
                    if (in && (c & (cpg - 1)) == 0) {
                        const int g = c / cpg;
                        const float* sw = reinterpret_cast<const float*>(base + r * rb + K);
                        acc[r] += (double)dsum * (double)sw[g] * sxd[g];
                    }
                }
            }
        }
        // refill the slot with the unit ns ahead once every lane is done with it
        __syncwarp();
        if (lane == 0 && k + ns < nmine) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive_expect_tx(&full[s], ub);
            bulk_g2s(slots + (size_t)s * ub, unit_src(k + ns), ub, &full[s], pol);
        }
        // lanes [32r/UNIT, 32(r+1)/UNIT) hold the sum of the unit's row r
        const double tot = warp_sum_scatter<UNIT>(acc);
        const int u = u0 + warp + k * Q8_WARPS;
        constexpr int LPR = 32 / UNIT;  // lanes per row after the scatter
        if (MODE == M_QKV || MODE == M_W13) {
            // pairs (rows 2i, 2i+1): lane 0 (and lane 16 when UNIT = 4) takes one pair
            const double odd = __shfl_down_sync(0xffffffffu, tot, LPR);
            if ((lane & (2 * LPR - 1)) == 0) {
                const int pr = u * (UNIT / 2) + lane / (2 * LPR);
                if (MODE == M_QKV) epi_qkv(a, pr, (float)tot, (float)odd, pos, rope_cs);
                else epi_w13(a, pr, (float)tot, (float)odd);
            }
        } else {
            // the x of this lane's row (row lane / LPR of the unit)
            float x0 = 0.f;
            if (MODE == M_RESID) {
#pragma unroll
                for (int r = 0; r < XR; r++) {
                    const float xr = __shfl_sync(0xffffffffu, xres[r], k & 31);
                    if (lane / LPR == r) x0 = xr;
                }
            }
            if ((lane & (LPR - 1)) == 0) {
                const int row = u * UNIT + lane / LPR;
                if (MODE == M_RESID) {
                    a.out[row] = (k < 32 ? x0 : __ldcg(a.out + row)) + (float)tot;
                } else {
                    const float v = (float)tot;
                    a.out[row] = v;
                    if (v != v) set_error(a.err, DERR_NAN);
                    const unsigned long long key = argmax_key(v, row);
                    best = key > best ? key : best;
                }
            }
        }
    }
    if (!a.early) grid_dep_launch();
    // a warp that gave up lets its copies in flight land before the CTA leaves
    if (k < nmine && lane == 0)
        for (int j = k; j < nmine && j < k + ns; j++)
            if (!(j == 0 && skip0)) mbar_wait_bounded(&full[j % ns], (j / ns) & 1, a.err, a.wait_ns);
    if (MODE == M_CLS) {
        // lanes 0, 32/UNIT, ... hold keys
#pragma unroll
        for (int o = 16; o >= 32 / UNIT; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other > best ? other : best;
        }
        if (lane == 0) best_s[warp] = best;
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned long long b = 0ull;
            for (int i = 0; i < Q8_WARPS; i++) b = best_s[i] > b ? best_s[i] : b;
            if (b) atomicMax(a.amax, b);
        }
    }
}

// ------------------------------------------------------------- small kernels --

static __global__ void k_set_tp(int* tp, int token, int pos) {
    tp[0] = token;
    tp[1] = pos;
}

// Greedy feedback between steps: token <- argmax of the step, pos += 1, and
// the token is appended to the output ring.
static __global__ void k_advance(int* tp, const unsigned long long* amax, int* out_tokens, int* counter) {
    int tok = argmax_key_index(*amax);
    tp[0] = tok;
    tp[1] += 1;
    int i = *counter;
    out_tokens[i] = tok;
    *counter = i + 1;
}

static __global__ void k_argmax_index(const unsigned long long* amax, int* out) { *out = argmax_key_index(*amax); }

// Block-reduced argmax over n values: per-thread best key, then one 64-bit
// atomicMax per block (first index among equal maxima).
static __global__ void k_argmax(const float* x, int n, unsigned long long* key, int* err) {
    unsigned long long best = 0ull;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        float v = x[i];
        if (v != v) set_error(err, DERR_NAN);
        unsigned long long k = argmax_key(v, i);
        best = k > best ? k : best;
    }
    for (int o = 16; o > 0; o >>= 1) {
        unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
        best = other > best ? other : best;
    }
    __shared__ unsigned long long s[32];
    if ((threadIdx.x & 31) == 0) s[threadIdx.x >> 5] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 0; i < (int)(blockDim.x >> 5); i++) best = s[i] > best ? s[i] : best;
        if (best) atomicMax(key, best);
    }
}

// Standalone Q8_0 quantization: one warp per group (bit-exact with the rule
// of the quantize() listing).
static __global__ void k_quantize(const float* x, long long ngroups, int gs, int8_t* q, float* s) {
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long g = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); g < ngroups; g += warps)
        quantize_group_warp(x + g * gs, gs, q + g * gs, s + g);
}

// Re-lays an fp32 matrix [rows][K] as Q8_0 row records [codes | scales | pad].
static __global__ void k_quantize_rows(const float* W, long long rows, int K, int gs, uint8_t* out, size_t rb) {
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    const int ng = K / gs;
    const long long total = rows * ng;
    for (long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < total; t += warps) {
        const long long r = t / ng;
        const int g = (int)(t % ng);
        uint8_t* rec = out + (size_t)r * rb;
        quantize_group_warp(W + (size_t)r * K + (size_t)g * gs, gs, reinterpret_cast<int8_t*>(rec) + g * gs,
                            reinterpret_cast<float*>(rec + K) + g);
    }
}

// Re-lays an fp32 matrix [rows][K] as Q4_0 with the 4-bit rule (scale =
// max|x| / 7 in fp32, code = round(x / scale), half away from zero, in
// [-7, 7]; a zero group gets scale 0, codes 0).  mode 0: packed records in the
// 32-value chunk layout (gs a multiple of 32); mode 2: packed records in the
// 64-value chunk layout (K % 64 == 0); mode 1: the Q8_0 record layout [K int8
// codes | scales | pad] holding the 4-bit codes (the embedding table, read one
// row at a time by the Q8_0 input path).  One warp per task of `span` values
// of a row (whole groups and whole chunks): lane l takes the values
// i0 + l and i0 + half + l of each step i0 (half = 16 or 32 for the chunk
// layouts), which share one byte of a packed record.
static __global__ void k_quantize_rows_q4(const float* W, long long rows, int K, int gs, uint8_t* out, size_t rb,
                                          int mode) {
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    const int lane = threadIdx.x & 31;
    const int span = mode == 2 && gs < 64 ? 64 : gs;  // 64: two groups of 32 share each byte
    const int tasks = K / span;
    const long long total = rows * tasks;
    for (long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < total; t += warps) {
        const long long r = t / tasks;
        const int base = (int)(t % tasks) * span;
        const float* x = W + (size_t)r * K + base;
        uint8_t* rec = out + (size_t)r * rb;
        float* sc = reinterpret_cast<float*>(rec + (mode == 1 ? (size_t)K : (size_t)K / 2));
        // the scales of the task's groups (one, or two of 32 values)
        float m0 = 0.f, m1 = 0.f;
        for (int i = lane; i < span; i += 32) {
            if (span > gs && i >= gs) m1 = fmaxf(m1, fabsf(x[i]));
            else m0 = fmaxf(m0, fabsf(x[i]));
        }
        m0 = warp_max(m0);
        m1 = warp_max(m1);
        const float s0 = m0 / 7.0f, s1 = m1 / 7.0f;
        auto code = [&](int i) {
            const float sc_i = (span > gs && i >= gs) ? s1 : s0;
            return sc_i == 0.f ? 0 : (int)roundf(x[i] / sc_i);
        };
        if (mode == 1) {
            for (int i = lane; i < span; i += 32) reinterpret_cast<int8_t*>(rec)[base + i] = (int8_t)code(i);
        } else {
            const int half = mode == 2 ? 32 : 16;
            for (int i0 = 0; i0 < span; i0 += 2 * half) {
                // lane l < half writes byte (base + i0) / 2 + l: value i0 + l low, i0 + half + l high
                const int lo = code(i0 + lane);
                const int hi = mode == 2 ? code(i0 + 32 + lane) : __shfl_down_sync(0xffffffffu, lo, 16);
                if (lane < half) rec[(size_t)(base + i0) / 2 + lane] = (uint8_t)((lo + 8) | ((hi + 8) << 4));
            }
        }
        if (lane == 0) {
            sc[base / gs] = s0;
            if (span > gs) sc[base / gs + 1] = s1;
        }
    }
}

// Exact int32 group dot products, out[r][g] = sum_k qw[r][g*gs+k] *
// qx[g*gs+k], through the Q8_0 GEMV's own chunk routine (q8_chunk_dots) for
// GS = 32, 64, 128 with K % 64 == 0: one warp per row, the input codes staged
// in shared memory as in the GEMV.  Dynamic shared memory: K bytes.
template <int GS>
__global__ void k_group_dots64(const int8_t* qw, const int8_t* qx, int rows, int K, int* out) {
    extern __shared__ __align__(16) int8_t gx[];
    for (int i = threadIdx.x; i < K / 16; i += blockDim.x)
        reinterpret_cast<int4*>(gx)[i] = reinterpret_cast<const int4*>(qx)[i];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;  // warp-uniform
    const int n64 = K >> 6, rot = (lane >> 1) & 3;
    const uint8_t* row = reinterpret_cast<const uint8_t*>(qw) + (size_t)r * K;
    int* o = out + (size_t)r * (K / GS);
    for (int t0 = 0; t0 < n64; t0 += 32) {
        const int t = t0 + lane;
        const bool in = t < n64;
        int4 xv[4];
        q8_chunk_x(gx, t, in, rot, xv);
        int gd[GS == 32 ? 2 : 1];
        q8_chunk_dots<GS>(row, xv, t, in, rot, gd);
        if (!in) continue;
        if (GS == 64) {
            o[t] = gd[0];
        } else if (GS == 32) {
            o[2 * t] = gd[0];
            o[2 * t + 1] = gd[GS == 32 ? 1 : 0];
        } else if ((t & 1) == 0) {
            o[t >> 1] = gd[0];
        }
    }
}

// Exact int32 group dot products for the other group sizes and widths, with
// the generic GEMV's 16-byte chunk loop: one warp per row.
static __global__ void k_group_dots(const int8_t* qw, const int8_t* qx, int rows, int K, int gs, int* out) {
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int nchunk = K >> 4, cpg = gs >> 4, iters = (nchunk + 31) >> 5;
    const int8_t* rec = qw + (size_t)r * K;
    for (int it = 0; it < iters; it++) {
        const int c = lane + 32 * it;
        int dsum = 0;
        if (c < nchunk) {
            int4 wv = *reinterpret_cast<const int4*>(rec + 16 * c);
            int4 xv = *reinterpret_cast<const int4*>(qx + 16 * c);
            dsum = __dp4a(wv.x, xv.x, dsum);
            dsum = __dp4a(wv.y, xv.y, dsum);
            dsum = __dp4a(wv.z, xv.z, dsum);
            dsum = __dp4a(wv.w, xv.w, dsum);
        }
        for (int o = 1; o < cpg; o <<= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
        if (c < nchunk && (c & (cpg - 1)) == 0) out[(size_t)r * (K / gs) + c / cpg] = dsum;
    }
}

}  // namespace l2c
