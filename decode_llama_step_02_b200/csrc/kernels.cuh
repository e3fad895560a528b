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
    size_t prefetch_bytes;   // L2 prefetch issued before the dependency wait
    int late_trigger;        // 1: let the next kernel launch only after this CTA's last weight loads
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
// norm_w is set) into shared codes and scales; all threads of the CTA call it.
// Warp w owns groups w, w + Q8_WARPS, ...; a lane holds elements
// g*gs + lane + 32e of each of them in registers, so the loads of the whole
// vector are in flight at once (one round trip to L2) instead of a chain of
// dependent loads.  Falls back to a plain loop when a lane would need more
// than Q8_VPL values.
// Slow path: one group at a time straight from global memory.
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
            if (warp == 0) L2C_STAMP(5);
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

// Exact-int32 group dots of UNIT rows (records at rec, stride rb) with the
// input codes xq, scaled and summed per lane in double.  Lane t covers the 64
// contiguous bytes [64t, 64t+64) of a row: one group at GS = 64, two at
// GS = 32, half of one at GS = 128 (a lane pair).  The four 16-byte reads of a
// lane are rotated by (lane >> 1) & 3 so that a quarter-warp touches eight
// distinct 16-byte bank groups.  Requires K % 64 == 0.
template <int GS, int UNIT>
__device__ __forceinline__ void q8_rows_dot64(const uint8_t* rec, size_t rb, const int8_t* xq, const double* sxd,
                                              int K, double (&acc)[UNIT]) {
    const int lane = threadIdx.x & 31;
    const int n64 = K >> 6;
    const int rot = (lane >> 1) & 3;
#pragma unroll
    for (int r = 0; r < UNIT; r++) acc[r] = 0.0;
#pragma unroll 2
    for (int t0 = 0; t0 < n64; t0 += 32) {
        const int t = t0 + lane;
        const bool in = t < n64;
        int4 xv[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int f = (j + rot) & 3;
            xv[j] = in ? *reinterpret_cast<const int4*>(xq + 64 * t + 16 * f) : make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < UNIT; r++) {
            const uint8_t* row = rec + r * rb;
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
            const float* sw = reinterpret_cast<const float*>(row + K);
            if (GS == 64) {
                const int d = (c[0] + c[1]) + (c[2] + c[3]);
                if (in) acc[r] += i2d_exact(d) * (double)sw[t] * sxd[t];
            } else if (GS == 32) {
                // chunk f of step j: the group of the lane's first 32 bytes is f < 2
                int lo = 0, hi = 0;
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const int f = (j + rot) & 3;
                    lo += f < 2 ? c[j] : 0;
                    hi += f < 2 ? 0 : c[j];
                }
                if (in) {
                    acc[r] += i2d_exact(lo) * (double)sw[2 * t] * sxd[2 * t];
                    acc[r] += i2d_exact(hi) * (double)sw[2 * t + 1] * sxd[2 * t + 1];
                }
            } else {  // GS == 128: lanes 2m and 2m+1 hold the two halves of group t/2
                int d = (c[0] + c[1]) + (c[2] + c[3]);
                d += __shfl_xor_sync(0xffffffffu, d, 1);
                if (in && (t & 1) == 0) acc[r] += i2d_exact(d) * (double)sw[t >> 1] * sxd[t >> 1];
            }
        }
    }
}

// Registers of the split prologue (gs = 32 * EPL): warp w holds groups
// w + j*nw (j < GM), a lane elements lane + 32e of each; w holds the RMSNorm
// gain when NORM.
template <int EPL, int GM, bool NORM>
struct Q8Pre {
    float v[GM][EPL];
    float w[NORM ? GM : 1][EPL];
};

// Group slots per warp of the register prologue: 16 values per lane with an
// RMSNorm gain, 48 without.
template <int EPL, bool NORM>
struct Q8PreGM {
    static constexpr int value = (NORM ? 16 : 48) / EPL;
};

template <int EPL, int GM>
__device__ __forceinline__ bool q8_pre_fits(const GemvArgs& a, int nw) {
    const int ng = a.K / (32 * EPL);
    return a.gs == 32 * EPL && (ng + nw - 1) / nw <= GM;
}

// Loads the gain (gain = true) or the values (from src, or the embedding
// codes eq * scale es) of the warp's groups.
template <int EPL, int GM, bool NORM>
__device__ __forceinline__ void q8_pre_load(const GemvArgs& a, const float* src, const int8_t* eq, const float* es,
                                            bool gain, Q8Pre<EPL, GM, NORM>& r, int nw) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gs = 32 * EPL, ng = a.K / gs;
#pragma unroll
    for (int j = 0; j < GM; j++) {
        const int g = warp + j * nw;
#pragma unroll
        for (int e = 0; e < EPL; e++) {
            const int i = g * gs + lane + 32 * e;
            if (gain) {
                if (NORM) r.w[NORM ? j : 0][e] = g < ng ? a.norm_w[i] : 0.f;
            } else {
                r.v[j][e] = g < ng ? (eq ? (float)eq[i] * es[g] : __ldcg(src + i)) : 0.f;
            }
        }
    }
}

// RMSNorm (double, when NORM) and Q8_0 codes of the values in r.  The
// reductions of all groups run interleaved so their latencies overlap.
template <int EPL, int GM, bool NORM, typename AfterLoads, typename SY = SyncCTA>
__device__ __forceinline__ void q8_pre_finish(const GemvArgs& a, Q8Pre<EPL, GM, NORM>& r, int8_t* xq, float* xsc,
                                              double* red, AfterLoads after_loads, const SY sy = SY()) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = sy.nthreads() >> 5;
    const int gs = 32 * EPL, ng = a.K / gs;
    if (a.emb && blockIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < GM; j++) {
            const int g = warp + j * nw;
            if (g < ng) {
#pragma unroll
                for (int e = 0; e < EPL; e++) a.x_resid[g * gs + lane + 32 * e] = r.v[j][e];
            }
        }
    }
    if (NORM) {
        double part[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int j = 0; j < GM; j++)
#pragma unroll
            for (int e = 0; e < EPL; e++) part[(j * EPL + e) & 3] += (double)r.v[j][e] * (double)r.v[j][e];
        double ss = (part[0] + part[1]) + (part[2] + part[3]);
        after_loads();  // every value has arrived by now
        ss = warp_sum(ss);
        if (lane == 0) red[warp] = ss;
        sy.sync();
        double tot = 0.0;
        for (int i = 0; i < nw; i++) tot += red[i];
        const double inv = 1.0 / sqrt(tot / (double)a.K + 1e-5);
#pragma unroll
        for (int j = 0; j < GM; j++)
#pragma unroll
            for (int e = 0; e < EPL; e++)
                r.v[j][e] = (float)((double)r.w[NORM ? j : 0][e] * (inv * (double)r.v[j][e]));
    }
    float m[GM];
#pragma unroll
    for (int j = 0; j < GM; j++) {
        m[j] = fabsf(r.v[j][0]);
#pragma unroll
        for (int e = 1; e < EPL; e++) m[j] = fmaxf(m[j], fabsf(r.v[j][e]));
    }
    if (!NORM) {
        float all = 0.f;
#pragma unroll
        for (int j = 0; j < GM; j++) all = fmaxf(all, m[j]);
        asm volatile("" ::"f"(all));  // every value has arrived by now
        after_loads();
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int j = 0; j < GM; j++) m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], o));
#pragma unroll
    for (int j = 0; j < GM; j++) {
        const int g = warp + j * nw;
        const float scale = m[j] / 127.0f;
        if (g < ng) {
#pragma unroll
            for (int e = 0; e < EPL; e++) {
                const float q = scale == 0.f ? 0.f : roundf(r.v[j][e] / scale);
                xq[g * gs + lane + 32 * e] = (int8_t)(int)q;
            }
            if (lane == 0) xsc[g] = scale;
        }
    }
}

struct Q8Layout {
    int nslot;          // ring slots per warp, one unit (UNIT row records) each
    size_t unit_bytes;  // UNIT * record bytes
};

constexpr int Q8_WARPS = 8;

// Every warp streams its own units (round-robin over the CTA's contiguous
// range) through its own ring of `nslot` shared-memory slots filled by 1-D bulk
// copies; lane 0 issues a copy as soon as the warp has finished with a slot,
// so nslot-1 units per warp stay in flight.  GS is the group size of the
// 64-byte-per-lane dot (32, 64 or 128, K % 64 == 0), or 0 for the generic
// 16-byte-per-lane loop.  Dynamic shared memory:
//   slots [Q8_WARPS][nslot][unit_bytes] | x codes [K, padded to 16] |
//   x scales [K/gs] fp32 | x scales [K/gs] double | barriers [Q8_WARPS][nslot]
template <int MODE, int GS>
__global__ void __launch_bounds__(32 * Q8_WARPS, 1) k_gemv_q8(const GemvArgs a, const Q8Layout L) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int UNIT = (MODE == M_QKV || MODE == M_W13) ? 2 : 1;
    __shared__ double red[Q8_WARPS];
    __shared__ unsigned long long best_s[Q8_WARPS];
    __shared__ double2 rope_cs[MODE == M_QKV ? 128 : 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int K = a.K, gs = a.gs;
    const size_t rb = a.ld;
    const int ns = L.nslot;
    uint8_t* slots = smem + (size_t)warp * ns * L.unit_bytes;
    int8_t* xq = reinterpret_cast<int8_t*>(smem + (size_t)Q8_WARPS * ns * L.unit_bytes);
    float* xsc = reinterpret_cast<float*>(xq + ((K + 15) & ~15));
    double* sxd = reinterpret_cast<double*>((reinterpret_cast<uintptr_t>(xsc + K / gs) + 15) & ~uintptr_t(15));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sxd + ((K / gs + 1) & ~1));
    uint64_t* full = bars + warp * ns;

    const int units = a.rows / UNIT;
    const int u0 = (int)((long long)units * blockIdx.x / gridDim.x);
    const int u1 = (int)((long long)units * (blockIdx.x + 1) / gridDim.x);
    const int nmine = (u1 - u0 - warp + Q8_WARPS - 1) / Q8_WARPS;  // units of this warp
    const uint8_t* Wb = static_cast<const uint8_t*>(a.W);
    const uint64_t pol = policy_evict_first();
    auto unit_src = [&](int k) { return Wb + (size_t)(u0 + warp + k * Q8_WARPS) * UNIT * rb; };

    if (warp == 0) L2C_STAMP(0);
    // ---- before the dependency wait: everything that earlier kernels of the
    // step do not write.  The small loads (token/position, RMSNorm gain,
    // embedding row, RoPE frequencies) go first, then the L2 prefetch of this
    // CTA's weights, so that those loads do not queue behind it in HBM.
    if (lane == 0) {
        for (int s = 0; s < ns; s++) mbar_init(&full[s], 1);
        mbar_fence_init();
    }
    constexpr int EPL = GS > 0 ? GS / 32 : 1;
    constexpr bool NORM = MODE != M_RESID;
    constexpr int GM = Q8PreGM<EPL, NORM>::value;
    Q8Pre<EPL, GM, NORM> pre;
    const bool split = GS > 0 && (NORM == (a.norm_w != nullptr)) && q8_pre_fits<EPL, GM>(a, Q8_WARPS);  // CTA-uniform
    int token = 0, pos = 0;
    if (MODE == M_QKV) read_tp(a, token, pos);  // written before the step's first kernel
    const int8_t* eq = nullptr;
    const float* es = nullptr;
    if (a.emb) {
        const uint8_t* rec = static_cast<const uint8_t*>(a.emb) + (size_t)token * a.ld;
        eq = reinterpret_cast<const int8_t*>(rec);
        es = reinterpret_cast<const float*>(rec + K);
    }
    if (split) {
        if (NORM) q8_pre_load<EPL, GM, NORM>(a, nullptr, nullptr, nullptr, true, pre, Q8_WARPS);
        if (eq) q8_pre_load<EPL, GM, NORM>(a, nullptr, eq, es, false, pre, Q8_WARPS);
    }
    if (MODE == M_QKV) rope_table(a, pos, rope_cs);
    if (warp == 0 && lane == 0 && a.prefetch_bytes) {
        const size_t first = (size_t)u0 * UNIT * rb;
        const size_t last = (size_t)u1 * UNIT * rb;
        if (last > first) {
            size_t bytes = last - first;
            if (bytes > a.prefetch_bytes) bytes = a.prefetch_bytes;
            prefetch_l2_range(Wb + first, bytes, policy_evict_last());
        }
    }
    if (warp == 0) L2C_STAMP(3);
    grid_dep_wait();
    if (!a.late_trigger) grid_dep_launch();
    if (warp == 0) L2C_STAMP(1);

    // ---- after the wait: the input written by the previous kernel, then the
    // ring fill (its copies land while the codes are computed)
    if (MODE == M_QKV && a.amax && blockIdx.x == 0 && threadIdx.x == 0) *a.amax = 0ull;
    if (split && !eq) q8_pre_load<EPL, GM, NORM>(a, a.in, nullptr, nullptr, false, pre, Q8_WARPS);
    // residual: lane k fetches now the x of this warp's k-th row, for the epilogue
    float xres = 0.f;
    if (MODE == M_RESID && lane < nmine) xres = __ldcg(a.out + u0 + warp + lane * Q8_WARPS);
    if (warp == 0) L2C_STAMP(4);
    auto fill_ring = [&]() {
        if (lane == 0) {
            for (int k = 0; k < ns && k < nmine; k++) {
                mbar_arrive_expect_tx(&full[k], (uint32_t)L.unit_bytes);
                bulk_g2s(slots + (size_t)k * L.unit_bytes, unit_src(k), (uint32_t)L.unit_bytes, &full[k], pol);
            }
        }
    };
    if (split) {
        q8_pre_finish<EPL, GM, NORM>(a, pre, xq, xsc, red, fill_ring);
    } else {
        q8_quantize_input<NORM>(a, eq, es, xq, xsc, red);
        fill_ring();
    }
    if (warp == 0) L2C_STAMP(6);
    __syncthreads();
    if (warp == 0) L2C_STAMP(7);
    for (int g = threadIdx.x; g < K / gs; g += blockDim.x) sxd[g] = (double)xsc[g];
    __syncthreads();
    if (warp == 0) L2C_STAMP(2);

    // ---- stream this warp's units
    const int nchunk = K >> 4;   // 16-byte chunks per row
    const int cpg = gs >> 4;     // chunks per group
    const int iters = (nchunk + 31) >> 5;
    unsigned long long best = 0ull;
    for (int k = 0; k < nmine; k++) {
        const int s = k % ns;
        if (!mbar_wait_bounded(&full[s], (k / ns) & 1, a.err)) {
            // give up: let the copies already issued land before the CTA leaves
            for (int j = k + 1; j < nmine && j < k + ns; j++) mbar_wait_bounded(&full[j % ns], (j / ns) & 1, a.err);
            return;
        }
        const uint8_t* base = slots + (size_t)s * L.unit_bytes;
        double acc[UNIT];
        if (GS != 0) {
            q8_rows_dot64<GS == 0 ? 64 : GS, UNIT>(base, rb, xq, sxd, K, acc);
        } else {
#pragma unroll
            for (int r = 0; r < UNIT; r++) acc[r] = 0.0;
            for (int it = 0; it < iters; it++) {
                const int c = lane + 32 * it;
                const bool in = c < nchunk;
                int dsum[UNIT];
                int4 xv = in ? *reinterpret_cast<const int4*>(xq + 16 * c) : make_int4(0, 0, 0, 0);
#pragma unroll
                for (int r = 0; r < UNIT; r++) {
                    dsum[r] = 0;
                    if (in) {
                        const int4 wv = *reinterpret_cast<const int4*>(base + r * rb + 16 * c);
                        dsum[r] = __dp4a(wv.x, xv.x, dsum[r]);
                        dsum[r] = __dp4a(wv.y, xv.y, dsum[r]);
                        dsum[r] = __dp4a(wv.z, xv.z, dsum[r]);
                        dsum[r] = __dp4a(wv.w, xv.w, dsum[r]);
                    }
                }
                for (int o = 1; o < cpg; o <<= 1) {
#pragma unroll
                    for (int r = 0; r < UNIT; r++) dsum[r] += __shfl_xor_sync(0xffffffffu, dsum[r], o);
                }
                if (in && (c & (cpg - 1)) == 0) {
                    const int g = c / cpg;
#pragma unroll
                    for (int r = 0; r < UNIT; r++) {
                        const float* sw = reinterpret_cast<const float*>(base + r * rb + K);
                        acc[r] += (double)dsum[r] * (double)sw[g] * sxd[g];
                    }
                }
            }
        }
        // refill the slot with the unit ns ahead once every lane is done with it
        __syncwarp();
        if (a.late_trigger && k + ns == nmine) grid_dep_launch();  // this warp's last copy is in
        if (lane == 0 && k + ns < nmine) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive_expect_tx(&full[s], (uint32_t)L.unit_bytes);
            bulk_g2s(slots + (size_t)s * L.unit_bytes, unit_src(k + ns), (uint32_t)L.unit_bytes, &full[s], pol);
        }
#pragma unroll
        for (int r = 0; r < UNIT; r++) acc[r] = warp_sum(acc[r]);
        const int u = u0 + warp + k * Q8_WARPS;
        const float xo = MODE == M_RESID ? __shfl_sync(0xffffffffu, xres, k & 31) : 0.f;
        if (lane == 0) {
            if (MODE == M_QKV) {
                epi_qkv(a, u, (float)acc[0], (float)acc[UNIT - 1], pos, rope_cs);
            } else if (MODE == M_W13) {
                epi_w13(a, u, (float)acc[0], (float)acc[UNIT - 1]);
            } else if (MODE == M_RESID) {
                a.out[u] = (k < 32 ? xo : __ldcg(a.out + u)) + (float)acc[0];
            } else {
                const float v = (float)acc[0];
                a.out[u] = v;
                if (v != v) set_error(a.err, DERR_NAN);
                const unsigned long long key = argmax_key(v, u);
                best = key > best ? key : best;
            }
        }
    }
    if (a.late_trigger) grid_dep_launch();  // (repeat triggers are harmless)
    L2C_STAMP(8 + warp);
    if (MODE == M_CLS) {
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

// Exact int32 group dot products through the same dp4a chunk loop as the Q8_0
// GEMV: out[r][g] = sum_k qw[r][g*gs+k] * qx[g*gs+k].  One warp per row.
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
