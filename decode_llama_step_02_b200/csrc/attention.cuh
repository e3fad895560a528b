// attention.cuh - flash-decode grouped-query attention of one layer (sm_100a).
//
// Shared by the step kernels and by standalone entry points: it holds only
// templates and inline functions, so any translation unit may include it.
#pragma once
#include "common.cuh"

namespace l2c {

// Arguments of k_attention.  `part` and `count` are scratch: partial softmax
// state per (sequence, KV head, chunk) and one arrival counter per (sequence,
// KV head), which must be zero before a launch (the kernel leaves it zero).
struct AttnArgs {
    const float* q;      // [B][H*hs] (rotated)
    const float* kc;     // this layer's key cache of sequence 0: [S][kvd]; sequence b at + b*seq_stride
    const float* vc;
    size_t seq_stride;   // floats between sequences' caches
    float* out;          // [B][H*hs]
    const int* tp;       // {token, pos} per sequence, stride tp_stride ints
    int tp_stride;
    int H, Hkv, hs, kvd, seq_len;
    int chunk;           // positions per CTA
    int nchunks;         // gridDim.x
    void* part;          // partials [B][Hkv][nchunks][rep][hs+2] (Acc)
    int* count;          // [B][Hkv] arrival counters (zero between launches)
    int* err;
};

// grid (nchunks, Hkv, B), 128 threads.  CTA (c, g, b) handles positions
// [c*chunk, min((c+1)*chunk, pos+1)) of sequence b for the rep = H/Hkv query
// heads sharing KV head g (heads g*rep .. g*rep+rep-1: contiguous groups).
// Each active CTA writes (m, l, o) per head: the running max of the scaled
// scores, the sum of exp(s - m) and the unnormalised weighted V sum.  The
// last CTA to arrive for (b, g) merges the partials and writes the output.
template <typename Acc, int HS, int REP>
__global__ void __launch_bounds__(128) k_attention(const AttnArgs a) {
    constexpr int NT = 128;
    constexpr int TC = 64;                 // positions per sub-chunk held in shared memory
    constexpr int V4 = HS / 4;             // float4 per K/V row slice
    constexpr int PVL = (V4 + 31) / 32;    // float4 per lane in the weighted V sum
    __shared__ Acc qs[REP][HS];
    __shared__ Acc sc[TC][REP];
    __shared__ Acc red[4][REP];
    __shared__ Acc ostage[4][REP][HS];
    __shared__ int last_s;
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    grid_dep_wait();
    grid_dep_launch();
    int pos = a.tp[b * a.tp_stride + 1];
    if (pos < 0 || pos >= a.seq_len) pos = 0;  // the GEMV kernel has flagged it
    const int T = pos + 1;
    const int nact = (T + a.chunk - 1) / a.chunk;  // active chunks for this sequence
    if (c >= nact) return;
    const int t0 = c * a.chunk, t1 = min(T, t0 + a.chunk);
    const float* kc = a.kc + (size_t)b * a.seq_stride + (size_t)g * HS;
    const float* vc = a.vc + (size_t)b * a.seq_stride + (size_t)g * HS;
    const float* q = a.q + (size_t)b * a.H * HS + (size_t)g * REP * HS;
    for (int i = tid; i < REP * HS; i += NT) qs[i / HS][i % HS] = (Acc)q[i];
    const Acc scale = (Acc)1 / sqrt((Acc)HS);

    Acc m[REP], l[REP], o[REP][PVL][4];
#pragma unroll
    for (int h = 0; h < REP; h++) {
        m[h] = -INFINITY;
        l[h] = 0;
#pragma unroll
        for (int p = 0; p < PVL; p++) o[h][p][0] = o[h][p][1] = o[h][p][2] = o[h][p][3] = 0;
    }
    __syncthreads();

    for (int tb = t0; tb < t1; tb += TC) {
        const int n = min(TC, t1 - tb);
        // scores: one thread per position
        for (int t = tid; t < n; t += NT) {
            const float4* kr = reinterpret_cast<const float4*>(kc + (size_t)(tb + t) * a.kvd);
            Acc s[REP];
#pragma unroll
            for (int h = 0; h < REP; h++) s[h] = 0;
#pragma unroll 4
            for (int j = 0; j < V4; j++) {
                float4 kv = __ldg(kr + j);
#pragma unroll
                for (int h = 0; h < REP; h++) {
                    s[h] += (Acc)kv.x * qs[h][4 * j] + (Acc)kv.y * qs[h][4 * j + 1] +
                            (Acc)kv.z * qs[h][4 * j + 2] + (Acc)kv.w * qs[h][4 * j + 3];
                }
            }
#pragma unroll
            for (int h = 0; h < REP; h++) sc[t][h] = s[h] * scale;
        }
        __syncthreads();
        // max over the sub-chunk, new running max, weights p = exp(s - m_new)
        Acc mnew[REP], alpha[REP];
#pragma unroll
        for (int h = 0; h < REP; h++) {
            Acc mx = -INFINITY;
            for (int t = tid; t < n; t += NT) mx = max(mx, sc[t][h]);
            mx = warp_max(mx);
            if (lane == 0) red[warp][h] = mx;
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < REP; h++) {
            Acc mx = max(max(red[0][h], red[1][h]), max(red[2][h], red[3][h]));
            mnew[h] = max(m[h], mx);
            alpha[h] = exp(m[h] - mnew[h]);  // exp(-inf) = 0 on the first sub-chunk
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < REP; h++) {
            Acc ps = 0;
            for (int t = tid; t < n; t += NT) {
                Acc p = exp(sc[t][h] - mnew[h]);
                sc[t][h] = p;
                ps += p;
            }
            ps = warp_sum(ps);
            if (lane == 0) red[warp][h] = ps;
        }
        __syncthreads();
#pragma unroll
        for (int h = 0; h < REP; h++) {
            l[h] = l[h] * alpha[h] + (red[0][h] + red[1][h]) + (red[2][h] + red[3][h]);
            m[h] = mnew[h];
#pragma unroll
            for (int p = 0; p < PVL; p++) {
                o[h][p][0] *= alpha[h]; o[h][p][1] *= alpha[h];
                o[h][p][2] *= alpha[h]; o[h][p][3] *= alpha[h];
            }
        }
        // weighted V sum: warp per position, lane owns float4 slices of the row
        for (int t = warp; t < n; t += 4) {
            const float4* vr = reinterpret_cast<const float4*>(vc + (size_t)(tb + t) * a.kvd);
#pragma unroll
            for (int p = 0; p < PVL; p++) {
                const int j = lane + 32 * p;
                if (j < V4) {
                    float4 vv = __ldg(vr + j);
#pragma unroll
                    for (int h = 0; h < REP; h++) {
                        Acc w = sc[t][h];
                        o[h][p][0] += w * (Acc)vv.x; o[h][p][1] += w * (Acc)vv.y;
                        o[h][p][2] += w * (Acc)vv.z; o[h][p][3] += w * (Acc)vv.w;
                    }
                }
            }
        }
        __syncthreads();
    }
    // combine the four warps' weighted sums (same running max)
#pragma unroll
    for (int p = 0; p < PVL; p++) {
        const int j = lane + 32 * p;
        if (j < V4) {
#pragma unroll
            for (int h = 0; h < REP; h++) {
                ostage[warp][h][4 * j] = o[h][p][0]; ostage[warp][h][4 * j + 1] = o[h][p][1];
                ostage[warp][h][4 * j + 2] = o[h][p][2]; ostage[warp][h][4 * j + 3] = o[h][p][3];
            }
        }
    }
    __syncthreads();
    Acc* part = static_cast<Acc*>(a.part) +
                ((((size_t)b * a.Hkv + g) * a.nchunks + c) * REP) * (HS + 2);
    for (int i = tid; i < REP * HS; i += NT) {
        const int h = i / HS, e = i % HS;
        part[(size_t)h * (HS + 2) + e] = (ostage[0][h][e] + ostage[1][h][e]) + (ostage[2][h][e] + ostage[3][h][e]);
    }
    if (tid < REP) {
        part[(size_t)tid * (HS + 2) + HS] = m[tid];
        part[(size_t)tid * (HS + 2) + HS + 1] = l[tid];
    }
    __threadfence();
    __syncthreads();
    int* cnt = a.count + (size_t)b * a.Hkv + g;
    if (tid == 0) last_s = (atomicAdd(cnt, 1) == nact - 1);
    __syncthreads();
    if (!last_s) return;
    __threadfence();
    // merge the nact partials of (b, g): M = max m_c, L = sum l_c e^{m_c - M},
    // O = sum o_c e^{m_c - M}; output O / L.
    const Acc* p0 = static_cast<const Acc*>(a.part) + (((size_t)b * a.Hkv + g) * a.nchunks * REP) * (HS + 2);
    for (int i = tid; i < REP * HS; i += NT) {
        const int h = i / HS, e = i % HS;
        Acc M = -INFINITY;
        for (int k = 0; k < nact; k++) M = max(M, __ldcg(p0 + ((size_t)k * REP + h) * (HS + 2) + HS));
        Acc Ls = 0, Os = 0;
        for (int k = 0; k < nact; k++) {
            const Acc* pk = p0 + ((size_t)k * REP + h) * (HS + 2);
            Acc f = exp(__ldcg(pk + HS) - M);
            Ls += __ldcg(pk + HS + 1) * f;
            Os += __ldcg(pk + e) * f;
        }
        a.out[(size_t)b * a.H * HS + ((size_t)g * REP + h) * HS + e] = (float)(Os / Ls);
    }
    if (tid == 0) *cnt = 0;
}

typedef void (*AttnKernel)(const AttnArgs);

// The attention instantiation for a head size and GQA ratio (nullptr if none).
template <typename Acc>
inline AttnKernel attn_kernel_for(int hs, int rep) {
#define L2C_ATTN(HS_, REP_) \
    if (hs == HS_ && rep == REP_) return k_attention<Acc, HS_, REP_>;
    L2C_ATTN(8, 1) L2C_ATTN(8, 2) L2C_ATTN(8, 3) L2C_ATTN(8, 4)
    L2C_ATTN(16, 1) L2C_ATTN(16, 2) L2C_ATTN(16, 4)
    L2C_ATTN(32, 1) L2C_ATTN(32, 2) L2C_ATTN(32, 4)
    L2C_ATTN(48, 1) L2C_ATTN(48, 2) L2C_ATTN(48, 4)
    L2C_ATTN(64, 1) L2C_ATTN(64, 2) L2C_ATTN(64, 4) L2C_ATTN(64, 8)
    L2C_ATTN(96, 1) L2C_ATTN(96, 2) L2C_ATTN(96, 4)
    L2C_ATTN(128, 1) L2C_ATTN(128, 2) L2C_ATTN(128, 4) L2C_ATTN(128, 8)
#undef L2C_ATTN
    return nullptr;
}

}  // namespace l2c
