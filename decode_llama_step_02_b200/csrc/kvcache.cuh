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
// step's attention reads these, and stores the row at the step's position
// itself (kv8_store_head, in the CTA whose chunk ends there); the fp32 cache
// row is overwritten with the same code * scale values.  The kernel below
// stores rows in bulk: every row when the cache is enabled, and loaded rows.
#pragma once
#include "attention.cuh"

namespace l2c {

struct Kv8Args {
    float* kc;          // fp32 K rows of row 0 of the range: row r at kc + r * kvd
    float* vc;
    int8_t* kq;         // codes, same element layout
    int8_t* vq;
    float* ks;          // scales: row r, head g at ks + r * n_kv_heads + g
    float* vs;
    int kvd, hs, n_kv_heads;
};

// grid (rows, 2 * n_kv_heads): block (r, j) quantizes head j / 2 of the K
// (j even) or V (j odd) row r with one warp of 32 lanes (hs <= 128).
__global__ void __launch_bounds__(32) k_kv8_rows(const Kv8Args a) {
    const int g = blockIdx.y >> 1;
    const bool isv = blockIdx.y & 1;
    const int r = blockIdx.x;
    float* x = (isv ? a.vc : a.kc) + (size_t)r * a.kvd + (size_t)g * a.hs;
    int8_t* q = (isv ? a.vq : a.kq) + (size_t)r * a.kvd + (size_t)g * a.hs;
    float* sc = (isv ? a.vs : a.ks) + (size_t)r * a.n_kv_heads + g;
    kv8_store_head(x, q, sc, a.hs);
}

}  // namespace l2c
