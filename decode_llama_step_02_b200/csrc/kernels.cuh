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

// Unit u of the QKV matrix is the row pair (2u, 2u+1); v0/v1 its two outputs.
__device__ __forceinline__ void epi_qkv(const GemvArgs& a, int u, float v0, float v1, int pos) {
    int r = 2 * u;
    if (r < a.d) {
        float o0, o1;
        rope_pair(v0, v1, r % a.hs, pos, a.freq, o0, o1);
        a.out[r] = o0;
        a.out[r + 1] = o1;
    } else if (r < a.d + a.kvd) {
        int i = r - a.d;
        float o0, o1;
        rope_pair(v0, v1, i % a.hs, pos, a.freq, o0, o1);
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

// fp32 input into shared memory: RMSNorm (double) when norm_w is set.
// On layer 0 the input is the embedding row E[token] (fp32 or dequantized
// Q8_0: code * scale in fp32) and CTA 0 also stores it as the residual x.
template <bool Q8>
__device__ void load_input(const GemvArgs& a, int token, float* xs, double* red) {
    const int K = a.K;
    const float* in = a.in;
    const int8_t* eq = nullptr;
    const float* es = nullptr;
    if (a.emb) {
        if (Q8) {
            const uint8_t* rec = static_cast<const uint8_t*>(a.emb) + (size_t)token * a.ld;
            eq = reinterpret_cast<const int8_t*>(rec);
            es = reinterpret_cast<const float*>(rec + K);
        } else {
            in = static_cast<const float*>(a.emb) + (size_t)token * a.K;
        }
    }
    for (int i = threadIdx.x; i < K; i += blockDim.x) {
        float v = eq ? (float)eq[i] * es[i / a.gs] : in[i];
        xs[i] = v;
        if (a.emb && blockIdx.x == 0) a.x_resid[i] = v;
    }
    if (a.norm_w) {
        __syncthreads();
        double ss = 0.0;
        for (int i = threadIdx.x; i < K; i += blockDim.x) ss += (double)xs[i] * (double)xs[i];
        ss = block_sum(ss, red);
        double inv = 1.0 / sqrt(ss / (double)K + 1e-5);
        for (int i = threadIdx.x; i < K; i += blockDim.x)
            xs[i] = (float)((double)a.norm_w[i] * (inv * (double)xs[i]));
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
    for (; j < K4; j += 32) {
        float4 xv = xs[j];
#pragma unroll
        for (int r = 0; r < R; r++) {
            float4 wv = ld_stream_f4(reinterpret_cast<const float4*>(w + r * ldw) + j, pol);
            acc[r] = fmaf(wv.x, xv.x, acc[r]);
            acc[r] = fmaf(wv.y, xv.y, acc[r]);
            acc[r] = fmaf(wv.z, xv.z, acc[r]);
            acc[r] = fmaf(wv.w, xv.w, acc[r]);
        }
    }
#pragma unroll
    for (int r = 0; r < R; r++) out[r] = warp_sum(acc[r]);
}

constexpr int F32_THREADS = 512;

// Requires K % 4 == 0 (rows are 16-byte aligned).  Dynamic shared memory:
// K floats.  Each CTA owns a contiguous range of units (1 row, or a row pair
// for QKV/W13); its warps take the units round-robin.
template <int MODE>
__global__ void __launch_bounds__(F32_THREADS, 2) k_gemv_f32(const GemvArgs a) {
    extern __shared__ float4 smem_f4[];
    float* xs = reinterpret_cast<float*>(smem_f4);
    __shared__ double red[32];
    __shared__ unsigned long long best_s[32];
    constexpr int UNIT = (MODE == M_QKV || MODE == M_W13) ? 2 : 1;
    constexpr int U = (UNIT == 2) ? 4 : 8;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int units = a.rows / UNIT;
    const int u0 = (int)((long long)units * blockIdx.x / gridDim.x);
    const int u1 = (int)((long long)units * (blockIdx.x + 1) / gridDim.x);
    const float* W = static_cast<const float*>(a.W);
    const uint64_t pol = policy_evict_first();
    if (threadIdx.x == 0 && u1 > u0 && a.prefetch_bytes) {
        size_t bytes = (size_t)(u1 - u0) * UNIT * a.ld * sizeof(float);
        if (bytes > a.prefetch_bytes) bytes = a.prefetch_bytes;
        prefetch_l2_range(W + (size_t)u0 * UNIT * a.ld, bytes, policy_evict_last());
    }
    grid_dep_wait();
    grid_dep_launch();
    int token = 0, pos = 0;
    if (MODE == M_QKV) read_tp(a, token, pos);
    if (MODE == M_QKV && a.amax && blockIdx.x == 0 && threadIdx.x == 0) *a.amax = 0ull;
    load_input<false>(a, token, xs, red);
    __syncthreads();
    const int K4 = a.K >> 2;
    unsigned long long best = 0ull;
    for (int u = u0 + warp; u < u1; u += nwarps) {
        const float* wr = W + (size_t)u * UNIT * a.ld;
        float acc[UNIT];
        dot_rows_f32<UNIT, U>(wr, a.ld, K4, reinterpret_cast<const float4*>(xs), pol, acc);
        if (lane == 0) {
            if (MODE == M_QKV) {
                epi_qkv(a, u, acc[0], acc[UNIT - 1], pos);
            } else if (MODE == M_W13) {
                epi_w13(a, u, acc[0], acc[UNIT - 1]);
            } else if (MODE == M_RESID) {
                a.out[u] = a.out[u] + acc[0];
            } else {
                a.out[u] = acc[0];
                if (acc[0] != acc[0]) set_error(a.err, DERR_NAN);
                unsigned long long k = argmax_key(acc[0], u);
                best = k > best ? k : best;
            }
        }
    }
    if (MODE == M_CLS) {
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
__device__ __forceinline__ void quantize_group_warp(const float* x, int gs, int8_t* q, float* s) {
    const int lane = threadIdx.x & 31;
    float m = 0.f;
    for (int i = lane; i < gs; i += 32) m = fmaxf(m, fabsf(x[i]));
    m = warp_max(m);
    float scale = m / 127.0f;
    for (int i = lane; i < gs; i += 32) {
        float v = scale == 0.f ? 0.f : roundf(x[i] / scale);
        q[i] = (int8_t)(int)v;
    }
    if (lane == 0) *s = scale;
}

struct Q8Layout {
    // shared memory carve-up of k_gemv_q8
    int ns;            // ring stages
    int units_per_stage;
    size_t stage_bytes;
    int stage_fp32;    // 1: the input is normalised (or dequantized) into shared fp32 first
};

// One warp per unit (row or row pair) of each stage.  Warp `nwc` is the
// producer: lane 0 issues the bulk copies.  Dynamic shared memory:
//   ring [ns][stage_bytes] | x fp32 [K] (only with stage_fp32) | x codes [K]
//   | x scales [K/gs] | barriers
template <int MODE>
__global__ void __launch_bounds__(288, 1) k_gemv_q8(const GemvArgs a, const Q8Layout L) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int UNIT = (MODE == M_QKV || MODE == M_W13) ? 2 : 1;
    __shared__ double red[32];
    __shared__ unsigned long long best_s[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwc = (blockDim.x >> 5) - 1;  // consumer warps
    const int K = a.K, gs = a.gs;
    const size_t rb = a.ld;
    uint8_t* ring = smem;
    float* xs = reinterpret_cast<float*>(smem + (size_t)L.ns * L.stage_bytes);
    int8_t* xq = reinterpret_cast<int8_t*>(xs + (L.stage_fp32 ? K : 0));
    float* xsc = reinterpret_cast<float*>(xq + ((K + 15) & ~15));
    uint64_t* full = reinterpret_cast<uint64_t*>(
        (reinterpret_cast<uintptr_t>(xsc + K / gs) + 15) & ~uintptr_t(15));
    uint64_t* empty = full + L.ns;

    const int units = a.rows / UNIT;
    const int u0 = (int)((long long)units * blockIdx.x / gridDim.x);
    const int u1 = (int)((long long)units * (blockIdx.x + 1) / gridDim.x);
    const int nunits = u1 - u0;
    const int ups = L.units_per_stage;
    const int nstages = (nunits + ups - 1) / ups;
    const uint8_t* Wb = static_cast<const uint8_t*>(a.W) + (size_t)u0 * UNIT * rb;

    if (threadIdx.x == 0) {
        for (int s = 0; s < L.ns; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], nwc);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == nwc) {
        // ---------------- producer: weights do not depend on earlier kernels
        if (lane == 0 && nstages > 0) {
            const uint64_t pol = policy_evict_first();
            size_t total = (size_t)nunits * UNIT * rb;
            size_t ring_bytes = (size_t)L.ns * L.stage_bytes;
            if (a.prefetch_bytes && total > ring_bytes) {
                size_t pf = total - ring_bytes;
                if (pf > a.prefetch_bytes) pf = a.prefetch_bytes;
                prefetch_l2_range(Wb + ring_bytes, pf, policy_evict_last());
            }
            int issued = 0;
            bool ok = true;
            for (int i = 0; i < nstages; i++) {
                int s = i % L.ns;
                if (i >= L.ns && !mbar_wait_bounded(&empty[s], ((i / L.ns) - 1) & 1, a.err)) {
                    ok = false;
                    break;
                }
                int nu = min(ups, nunits - i * ups);
                uint32_t bytes = (uint32_t)((size_t)nu * UNIT * rb);
                mbar_arrive_expect_tx(&full[s], bytes);
                bulk_g2s(ring + (size_t)s * L.stage_bytes, Wb + (size_t)i * ups * UNIT * rb, bytes, &full[s], pol);
                issued = i + 1;
            }
            if (!ok) {
                // drain the copies still in flight before leaving (bounded)
                for (int i = max(0, issued - L.ns); i < issued; i++)
                    mbar_wait_bounded(&full[i % L.ns], (i / L.ns) & 1, a.err);
            }
        }
        return;
    }

    // ---------------- consumers
    grid_dep_wait();
    grid_dep_launch();
    int token = 0, pos = 0;
    if (MODE == M_QKV) read_tp(a, token, pos);
    if (MODE == M_QKV && a.amax && blockIdx.x == 0 && threadIdx.x == 0) *a.amax = 0ull;
    // input (RMSNorm in double) then Q8_0 quantization, one warp per group.
    {
        // load_input uses blockDim-strided loops; restrict to consumer threads
        const int nct = nwc * 32;
        const int8_t* eq = nullptr;
        const float* es = nullptr;
        if (a.emb) {
            const uint8_t* rec = static_cast<const uint8_t*>(a.emb) + (size_t)token * a.ld;
            eq = reinterpret_cast<const int8_t*>(rec);
            es = reinterpret_cast<const float*>(rec + K);
        }
        if (L.stage_fp32) {
            for (int i = threadIdx.x; i < K; i += nct) {
                float v = eq ? (float)eq[i] * es[i / gs] : a.in[i];
                xs[i] = v;
                if (eq && blockIdx.x == 0) a.x_resid[i] = v;
            }
            asm volatile("bar.sync 1, %0;" :: "r"(nct) : "memory");
        }
        if (L.stage_fp32 && a.norm_w) {
            double ss = 0.0;
            for (int i = threadIdx.x; i < K; i += nct) ss += (double)xs[i] * (double)xs[i];
            ss = warp_sum(ss);
            if (lane == 0) red[warp] = ss;
            asm volatile("bar.sync 1, %0;" :: "r"(nct) : "memory");
            double tot = 0.0;
            for (int i = 0; i < nwc; i++) tot += red[i];
            double inv = 1.0 / sqrt(tot / (double)K + 1e-5);
            for (int i = threadIdx.x; i < K; i += nct)
                xs[i] = (float)((double)a.norm_w[i] * (inv * (double)xs[i]));
            asm volatile("bar.sync 1, %0;" :: "r"(nct) : "memory");
        }
        const float* src = L.stage_fp32 ? xs : a.in;
        for (int g = warp; g < K / gs; g += nwc) quantize_group_warp(src + g * gs, gs, xq + g * gs, xsc + g);
        asm volatile("bar.sync 1, %0;" :: "r"(nct) : "memory");
    }

    const int nchunk = K >> 4;              // 16-byte chunks per row
    const int cpg = gs >> 4;                // chunks per group
    const int iters = (nchunk + 31) >> 5;
    unsigned long long best = 0ull;
    bool ok = true;
    for (int i = 0; i < nstages && ok; i++) {
        const int s = i % L.ns;
        if (!mbar_wait_bounded(&full[s], (i / L.ns) & 1, a.err)) { ok = false; break; }
        const int nu = min(ups, nunits - i * ups);
        if (warp < nu) {
            const int u = u0 + i * ups + warp;
            const uint8_t* base = ring + (size_t)s * L.stage_bytes + (size_t)warp * UNIT * rb;
            double accd[UNIT];
#pragma unroll
            for (int r = 0; r < UNIT; r++) {
                const uint8_t* rec = base + r * rb;
                const float* sw = reinterpret_cast<const float*>(rec + K);
                double acc = 0.0;
                for (int it = 0; it < iters; it++) {
                    const int c = lane + 32 * it;
                    int dsum = 0;
                    if (c < nchunk) {
                        int4 wv = *reinterpret_cast<const int4*>(rec + 16 * c);
                        int4 xv = *reinterpret_cast<const int4*>(xq + 16 * c);
                        dsum = __dp4a(wv.x, xv.x, dsum);
                        dsum = __dp4a(wv.y, xv.y, dsum);
                        dsum = __dp4a(wv.z, xv.z, dsum);
                        dsum = __dp4a(wv.w, xv.w, dsum);
                    }
                    for (int o = 1; o < cpg; o <<= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
                    if (c < nchunk && (c & (cpg - 1)) == 0) {
                        const int g = c / cpg;
                        acc += (double)dsum * (double)sw[g] * (double)xsc[g];
                    }
                }
                accd[r] = warp_sum(acc);
            }
            if (lane == 0) {
                if (MODE == M_QKV) {
                    epi_qkv(a, u, (float)accd[0], (float)accd[UNIT - 1], pos);
                } else if (MODE == M_W13) {
                    epi_w13(a, u, (float)accd[0], (float)accd[UNIT - 1]);
                } else if (MODE == M_RESID) {
                    a.out[u] = a.out[u] + (float)accd[0];
                } else {
                    float v = (float)accd[0];
                    a.out[u] = v;
                    if (v != v) set_error(a.err, DERR_NAN);
                    unsigned long long k = argmax_key(v, u);
                    best = k > best ? k : best;
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (MODE == M_CLS) {
        if (lane == 0) best_s[warp] = best;
        asm volatile("bar.sync 1, %0;" :: "r"(nwc * 32) : "memory");
        if (threadIdx.x == 0) {
            unsigned long long b = 0ull;
            for (int i = 0; i < nwc; i++) b = best_s[i] > b ? best_s[i] : b;
            if (b) atomicMax(a.amax, b);
        }
    }
}

// ------------------------------------------------------------- small kernels --

__global__ void k_set_tp(int* tp, int token, int pos) {
    tp[0] = token;
    tp[1] = pos;
}

// Greedy feedback between steps: token <- argmax of the step, pos += 1, and
// the token is appended to the output ring.
__global__ void k_advance(int* tp, const unsigned long long* amax, int* out_tokens, int* counter) {
    int tok = argmax_key_index(*amax);
    tp[0] = tok;
    tp[1] += 1;
    int i = *counter;
    out_tokens[i] = tok;
    *counter = i + 1;
}

__global__ void k_argmax_index(const unsigned long long* amax, int* out) { *out = argmax_key_index(*amax); }

// Block-reduced argmax over n values: per-thread best key, then one 64-bit
// atomicMax per block (first index among equal maxima).
__global__ void k_argmax(const float* x, int n, unsigned long long* key, int* err) {
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
__global__ void k_quantize(const float* x, long long ngroups, int gs, int8_t* q, float* s) {
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long g = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); g < ngroups; g += warps)
        quantize_group_warp(x + g * gs, gs, q + g * gs, s + g);
}

// Re-lays an fp32 matrix [rows][K] as Q8_0 row records [codes | scales | pad].
__global__ void k_quantize_rows(const float* W, long long rows, int K, int gs, uint8_t* out, size_t rb) {
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
__global__ void k_group_dots(const int8_t* qw, const int8_t* qx, int rows, int K, int gs, int* out) {
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
