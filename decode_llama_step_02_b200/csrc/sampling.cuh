// sampling.cuh - the token draw after the logits (sm_100a).
//
// A temperature divides the logits before the softmax ("LLM底层原理与工程实践"
// §3.2), temperature 0 is the greedy sample_argmax ("超精简LLM部署"
// 智能家居控制案例).  Reading taken where the pages stop: weights
// q_i = exp((z_i - max z) / T) in double; top-p keeps the smallest set of most
// probable tokens whose weight reaches topp * sum q (every token tied with the
// last one included); the caller's coin u in [0, 1) picks the first index, in
// index order, of the set at which the running weight exceeds u * (the set's
// weight) -- the last index of the set if rounding leaves none.
//
// One CTA per sequence, SAMPLE_THREADS threads, each owning a contiguous
// segment of the vocabulary (so that a block scan runs in index order):
//   1. max of the logits (and a NaN check),
//   2. the weights, stored in a scratch row, and their sum,
//   3. top-p: the set is {i : key(z_i) >= t} for the order-preserving 32-bit
//      key of the logit (q is increasing in z); t is found by a radix select
//      over the key, 8 bits a pass, on weighted histograms (double atomics in
//      shared memory), from the largest key down until the running weight
//      reaches topp * sum q,
//   4. the draw: an exclusive block scan of the set's weight per segment, and
//      the segment holding the crossing walks its elements.
// Sums are taken in a different order than a sequential loop: a decision can
// differ from one only where a running weight lies within rounding (~1e-16
// relative) of its threshold.
#pragma once
#include "common.cuh"

namespace l2c {

constexpr int SAMPLE_THREADS = 1024;

// Order-preserving key of a float: larger float, larger key.
__device__ __forceinline__ uint32_t f32_order_key(float v) {
    const uint32_t b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Block-wide sum of doubles (SAMPLE_THREADS threads); every thread gets it.
__device__ __forceinline__ double sample_block_sum(double v, double* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
#pragma unroll 4
    for (int i = 0; i < SAMPLE_THREADS / 32; i++) t += red[i];
    return t;
}

// grid (B), SAMPLE_THREADS threads.  Sequence b: logits z + b*n, weights
// scratch q + b*n, coin coins[b] (coin0 when coins is null), result out[b].
// temperature > 0.
__global__ void __launch_bounds__(SAMPLE_THREADS) k_sample(const float* z_all, int n, float temperature, float topp,
                                                          double coin0, const double* coins, double* q_all, int* out,
                                                          int* err) {
    __shared__ double hist[256];
    __shared__ double red[SAMPLE_THREADS / 32];
    __shared__ float fred[SAMPLE_THREADS / 32];
    __shared__ uint32_t digit_s;
    __shared__ double above_s;
    __shared__ int pick_s, last_s;
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float* z = z_all + (size_t)b * n;
    double* q = q_all + (size_t)b * n;
    const int i0 = (int)((long long)n * tid / SAMPLE_THREADS);
    const int i1 = (int)((long long)n * (tid + 1) / SAMPLE_THREADS);
    // 1. max (a NaN is reported and treated as absent)
    float mx = -INFINITY;
    bool nan = false;
    for (int i = i0; i < i1; i++) {
        const float v = z[i];
        nan |= v != v;
        mx = fmaxf(mx, v);
    }
    if (nan) set_error(err, DERR_NAN);
    mx = warp_max(mx);
    if (lane == 0) fred[warp] = mx;
    __syncthreads();
    mx = fred[0];
    for (int i = 1; i < SAMPLE_THREADS / 32; i++) mx = fmaxf(mx, fred[i]);
    // 2. weights and their sum
    double zs = 0.0;
    for (int i = i0; i < i1; i++) {
        const double w = exp(((double)z[i] - (double)mx) / (double)temperature);
        q[i] = w;
        zs += w;
    }
    const double Z = sample_block_sum(zs, red);
    // 3. top-p threshold on the logit key
    uint32_t tkey = 0;  // the set is {i : key_i >= tkey}
    double zset = Z;
    if (topp < 1.0f) {
        const double target = (double)topp * Z;
        uint32_t prefix = 0;
        double above = 0.0;  // weight of the keys above the current prefix
        for (int shift = 24; shift >= 0; shift -= 8) {
            if (tid < 256) hist[tid] = 0.0;
            __syncthreads();
            for (int i = i0; i < i1; i++) {
                const uint32_t k = f32_order_key(z[i]);
                if (shift == 24 || (k >> (shift + 8)) == prefix) atomicAdd(&hist[(k >> shift) & 255u], q[i]);
            }
            __syncthreads();
            if (tid == 0) {
                double cum = above;
                int d = 255;
                for (; d > 0; d--) {
                    if (cum + hist[d] >= target) break;
                    cum += hist[d];
                }
                digit_s = (uint32_t)d;
                above_s = cum;
            }
            __syncthreads();
            prefix = (prefix << 8) | digit_s;
            above = above_s;
        }
        tkey = prefix;
        // the set's weight: everything at or above the key
        double s = 0.0;
        for (int i = i0; i < i1; i++)
            if (f32_order_key(z[i]) >= tkey) s += q[i];
        zset = sample_block_sum(s, red);
    }
    // 4. the draw: exclusive scan of the set's weight over the segments
    double seg = 0.0;
    int seg_last = -1;
    for (int i = i0; i < i1; i++)
        if (f32_order_key(z[i]) >= tkey) {
            seg += q[i];
            seg_last = i;
        }
    double incl = seg;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    __syncthreads();  // red is free again
    if (lane == 31) red[warp] = incl;
    if (tid == 0) {
        pick_s = 0x7fffffff;
        last_s = -1;
    }
    __syncthreads();
    double wbase = 0.0;
    for (int w = 0; w < warp; w++) wbase += red[w];
    const double excl = wbase + incl - seg;
    const double target = (coins ? coins[b] : coin0) * zset;
    if (seg_last >= 0) {
        atomicMax(&last_s, seg_last);
        // a segment whose end passes the target holds a candidate: its first
        // element at which the running weight exceeds it; the first such
        // segment's candidate is the draw (the minimum over the candidates)
        if (excl + seg > target) {
            double cum = excl;
            for (int i = i0; i < i1; i++) {
                if (f32_order_key(z[i]) < tkey) continue;
                cum += q[i];
                if (cum > target) {
                    atomicMin(&pick_s, i);
                    break;
                }
            }
        }
    }
    __syncthreads();
    if (tid == 0) out[b] = pick_s != 0x7fffffff ? pick_s : last_s;
}

}  // namespace l2c
