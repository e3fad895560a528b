// kvcache.cuh - the int8 KV cache (sm_100a).
//
// Reading (the pages give no int8 KV cache; this variant is the library's):
// every K and V row, when stored, becomes Q8_0 groups of head_size values,
// one group per KV head, quantized with the quantize() rule of "超精简LLM部署"
// §1 INT8量化压缩 (scale = max|x| / 127 in fp32, code = round(x / scale) with
// the quotient in fp32 and halves away from zero; a zero group gets scale 0
// and codes 0), and attention reads code * scale (one fp32 multiply).
//
// Layout, per sequence and layer: codes [seq_len][kv_dim] int8 (the fp32
// cache's element order) and scales [seq_len][n_kv_heads] fp32.  The Q8_0
// step's attention reads these; the fp32 cache row is overwritten with the
// same code * scale values, so the fp32 step (which reads the fp32 cache)
// sees the same numbers.
#pragma once
#include "common.cuh"

namespace l2c {

struct Kv8Args {
    float* kc;          // fp32 K rows of row 0 of the range: row r at kc + r * kvd
    float* vc;
    int8_t* kq;         // codes, same element layout
    int8_t* vq;
    float* ks;          // scales: row r, head g at ks + r * n_kv_heads + g
    float* vs;
    int kvd, hs, n_kv_heads;
    const int* pos;     // non-null: one row, the one at *pos (the step's position)
    int seq_len;
};

// grid (rows, 2 * n_kv_heads): block (r, j) quantizes head j / 2 of the K
// (j even) or V (j odd) row r (or of row *pos) with one warp of 32 lanes,
// hs / 32 values or fewer per lane (hs <= 128).
// Launched with programmatic dependent launch in the step (it waits for the
// q/k/v kernel before reading the row), as a plain kernel elsewhere (the
// wait then returns at once).
__global__ void __launch_bounds__(32) k_kv8_rows(const Kv8Args a) {
    const int lane = threadIdx.x;
    const int g = blockIdx.y >> 1;
    const bool isv = blockIdx.y & 1;
    grid_dep_wait();
    grid_dep_launch();
    int r = blockIdx.x;
    if (a.pos) {
        r = *a.pos;
        if (r < 0 || r >= a.seq_len) return;  // flagged by the q/k/v kernel
    }
    float* x = (isv ? a.vc : a.kc) + (size_t)r * a.kvd + (size_t)g * a.hs;
    int8_t* q = (isv ? a.vq : a.kq) + (size_t)r * a.kvd + (size_t)g * a.hs;
    float* sc = (isv ? a.vs : a.ks) + (size_t)r * a.n_kv_heads + g;
    float v[4];
    float m = 0.f;
    bool nan = false;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const int i = lane + 32 * e;
        v[e] = i < a.hs ? x[i] : 0.f;
        m = fmaxf(m, fabsf(v[e]));
        nan |= !isfinite(v[e]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    // a non-finite element (which no code can hold) makes the group's scale
    // NaN, so that every read of the group is NaN
    const float scale = __any_sync(0xffffffffu, nan) ? __int_as_float(0x7fc00000) : m / 127.0f;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const int i = lane + 32 * e;
        if (i >= a.hs) break;
        const int code = scale != 0.f && scale == scale ? (int)roundf(v[e] / scale) : 0;
        q[i] = (int8_t)code;
        x[i] = __fmul_rn((float)code, scale);
    }
    if (lane == 0) *sc = scale;
}

}  // namespace l2c
