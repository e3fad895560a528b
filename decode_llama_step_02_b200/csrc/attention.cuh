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
    int nchunks;         // gridDim.x: the positions 0..pos are split into this many chunks
    void* part;          // partials [B][Hkv][nchunks][rep][hs+2] (Acc)
    int* count;          // [B][Hkv] arrival counters (zero between launches)
    int* err;
};

// Shared memory of one attention work item (four warps).
template <typename Acc, int HS, int REP>
struct AttnSmem {
    static constexpr int TC = 64;  // positions per sub-chunk held in shared memory
    Acc sc[TC][REP];
    Acc red[4][REP];
    Acc ostage[4][REP][HS];
    int last;
};

// One work item: chunk c of sequence b for the rep = H/Hkv query heads that
// share KV head g (heads g*rep .. g*rep+rep-1: contiguous groups), run by 128
// threads (tid 0..127) that synchronise through `sy`.  The positions 0..pos
// of sequence b are split into nchunks equal chunks (ceil((pos+1)/nchunks)
// each), so every K/V row is read once per group.  Within an item, sub-chunks
// of TC positions go through three passes: scores (one warp per position: the
// row slice is one coalesced 16-byte-per-lane load, the dots of a batch of
// positions one reduce-scatter), the sub-chunk max and exp(s - m), and the
// weighted V sum (one warp per position again).  Each active item writes (m, l, o) per head: the
// running max of the scaled scores, the sum of exp(s - m) and the unnormalised
// weighted V sum.  The last item to arrive for (b, g) merges the partials and
// writes the output.  With COH, q, K and V are read through L2 (ld.global.cg),
// so an item may follow, in the same launch, the kernel phase that wrote them;
// otherwise through the read-only path.
template <typename Acc, int HS, int REP, typename SY, bool PRE = false, bool COH = false>
__device__ __forceinline__ void attn_item(const AttnArgs& a, int c, int g, int b, int tid, const SY& sy,
                                          AttnSmem<Acc, HS, REP>& sm) {
    // q, K and V: read-only for this launch unless COH (then through L2, coherent
    // with writes of other CTAs earlier in the same launch)
    auto ld4 = [](const float4* p) { return COH ? __ldcg(p) : __ldg(p); };
    static_assert(HS % 4 == 0 && HS <= 128, "head size");
    constexpr int NT = 128, NW = 4;
    constexpr int TC = AttnSmem<Acc, HS, REP>::TC;
    constexpr int V4 = HS / 4;             // float4 per K/V row slice (<= 32: one per lane)
    constexpr int PB = 8;                  // positions a warp loads before reducing
    auto& sc = sm.sc;
    auto& red = sm.red;
    auto& ostage = sm.ostage;
    const int lane = tid & 31, warp = tid >> 5;

    int pos = a.tp[b * a.tp_stride + 1];
    if (pos < 0 || pos >= a.seq_len) pos = 0;  // the GEMV kernel has flagged it
    const int T = pos + 1;
    const int chunk = (T + a.nchunks - 1) / a.nchunks;
    const int nact = (T + chunk - 1) / chunk;  // active chunks for this sequence
    if (c >= nact) return;
    const int t0 = c * chunk, t1 = min(T, t0 + chunk);
    const float* kc = a.kc + (size_t)b * a.seq_stride + (size_t)g * HS;
    const float* vc = a.vc + (size_t)b * a.seq_stride + (size_t)g * HS;
    const float* q = a.q + (size_t)b * a.H * HS + (size_t)g * REP * HS;
    const bool lane_on = lane < V4;
    // this lane's four q values of every head, converted once
    Acc qr[REP][4];
#pragma unroll
    for (int h = 0; h < REP; h++) {
        float4 qv = lane_on ? ld4(reinterpret_cast<const float4*>(q + (size_t)h * HS + 4 * lane))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        qr[h][0] = (Acc)qv.x; qr[h][1] = (Acc)qv.y; qr[h][2] = (Acc)qv.z; qr[h][3] = (Acc)qv.w;
    }
    const Acc scale = (Acc)1 / sqrt((Acc)HS);

    Acc m[REP], l[REP], o[REP][4];
#pragma unroll
    for (int h = 0; h < REP; h++) {
        m[h] = -INFINITY;
        l[h] = 0;
        o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0;
    }

    // Sub-chunks of TC positions: warp w takes the NB batches of PB positions
    // starting at w*PB + j*NW*PB.
    constexpr int NB = TC / (NW * PB);
    // PRE = true requests a sub-chunk's rows at once; it costs registers, and at
    // 168 a thread only 3 CTAs fit an SM, so the 16-chunk grid needs two waves:
    // measured slower, hence one batch at a time by default
    constexpr bool VPRE = PRE && sizeof(Acc) == 4 && REP <= 2;
    constexpr bool KPRE = PRE && (sizeof(Acc) == 4 || REP <= 2);
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int tb = t0; tb < t1; tb += TC) {
        const int n = min(TC, t1 - tb);
        float4 kv[KPRE ? NB : 1][PB];
        float4 vv[VPRE ? NB : 1][PB];
        auto load_k = [&](int j, float4 (&dst)[PB]) {
            const int tq = warp * PB + j * NW * PB;
#pragma unroll
            for (int i = 0; i < PB; i++) {
                const bool on = lane_on && tq + i < n;
                dst[i] = on ? ld4(reinterpret_cast<const float4*>(kc + (size_t)(tb + tq + i) * a.kvd) + lane)
                            : zero4;
            }
        };
#pragma unroll
        for (int j = 0; j < NB; j++) {
            const int tq = warp * PB + j * NW * PB;
            if (KPRE) load_k(j, kv[KPRE ? j : 0]);
#pragma unroll
            for (int i = 0; i < PB; i++) {
                const bool on = lane_on && tq + i < n;
                if (VPRE)
                    vv[VPRE ? j : 0][i] =
                        on ? ld4(reinterpret_cast<const float4*>(vc + (size_t)(tb + tq + i) * a.kvd) + lane) : zero4;
            }
        }
        // scores: the PB sums of each head in one reduce-scatter (lane 4i ends
        // with position tq + i's total)
#pragma unroll
        for (int j = 0; j < NB; j++) {
            const int tq = warp * PB + j * NW * PB;
            if (tq < n) {  // warp-uniform
                if (!KPRE) load_k(j, kv[0]);
                const float4 (&kj)[PB] = kv[KPRE ? j : 0];
#pragma unroll
                for (int h = 0; h < REP; h++) {
                    Acc sp[PB];
#pragma unroll
                    for (int i = 0; i < PB; i++)
                        sp[i] = (Acc)kj[i].x * qr[h][0] + (Acc)kj[i].y * qr[h][1] +
                                (Acc)kj[i].z * qr[h][2] + (Acc)kj[i].w * qr[h][3];
                    const Acc s = warp_sum_scatter<PB>(sp);
                    const int i = lane >> 2;
                    if ((lane & 3) == 0 && tq + i < n) sc[tq + i][h] = s * scale;
                }
            }
        }
        sy.sync();
        // max over the sub-chunk, new running max, weights p = exp(s - m_new)
        Acc mnew[REP], alpha[REP];
#pragma unroll
        for (int h = 0; h < REP; h++) {
            Acc mx = -INFINITY;
            for (int t = tid; t < n; t += NT) mx = max(mx, sc[t][h]);
            mx = warp_max(mx);
            if (lane == 0) red[warp][h] = mx;
        }
        sy.sync();
#pragma unroll
        for (int h = 0; h < REP; h++) {
            Acc mx = max(max(red[0][h], red[1][h]), max(red[2][h], red[3][h]));
            mnew[h] = max(m[h], mx);
            alpha[h] = exp(m[h] - mnew[h]);  // exp(-inf) = 0 on the first sub-chunk
        }
        sy.sync();
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
        sy.sync();
#pragma unroll
        for (int h = 0; h < REP; h++) {
            l[h] = l[h] * alpha[h] + (red[0][h] + red[1][h]) + (red[2][h] + red[3][h]);
            m[h] = mnew[h];
            o[h][0] *= alpha[h]; o[h][1] *= alpha[h]; o[h][2] *= alpha[h]; o[h][3] *= alpha[h];
        }
        // weighted V sum: warp per position, lane owns one float4 slice of the row
#pragma unroll
        for (int j = 0; j < NB; j++) {
            const int tq = warp * PB + j * NW * PB;
            if (tq < n) {  // warp-uniform
                float4 vl[PB];
#pragma unroll
                for (int i = 0; i < PB; i++) {
                    if (VPRE) {
                        vl[i] = vv[VPRE ? j : 0][i];
                    } else {
                        const bool on = lane_on && tq + i < n;
                        vl[i] = on ? ld4(reinterpret_cast<const float4*>(vc + (size_t)(tb + tq + i) * a.kvd) + lane)
                                   : zero4;
                    }
                }
#pragma unroll
                for (int i = 0; i < PB; i++) {
                    if (tq + i < n) {
#pragma unroll
                        for (int h = 0; h < REP; h++) {
                            const Acc w = sc[tq + i][h];
                            o[h][0] += w * (Acc)vl[i].x; o[h][1] += w * (Acc)vl[i].y;
                            o[h][2] += w * (Acc)vl[i].z; o[h][3] += w * (Acc)vl[i].w;
                        }
                    }
                }
            }
        }
        sy.sync();
    }
    // combine the four warps' weighted sums (same running max)
    if (lane_on) {
#pragma unroll
        for (int h = 0; h < REP; h++) {
            ostage[warp][h][4 * lane] = o[h][0]; ostage[warp][h][4 * lane + 1] = o[h][1];
            ostage[warp][h][4 * lane + 2] = o[h][2]; ostage[warp][h][4 * lane + 3] = o[h][3];
        }
    }
    sy.sync();
    if (nact == 1) {  // the whole range in one item: O / L directly (the merge would scale by e^0 = 1)
        for (int i = tid; i < REP * HS; i += NT) {
            const int h = i / HS, e = i % HS;
            const Acc o_sum = (ostage[0][h][e] + ostage[1][h][e]) + (ostage[2][h][e] + ostage[3][h][e]);
            a.out[(size_t)b * a.H * HS + ((size_t)g * REP + h) * HS + e] = (float)(o_sum / l[h]);
        }
        return;
    }
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
    sy.sync();
    int* cnt = a.count + (size_t)b * a.Hkv + g;
    if (tid == 0) sm.last = (atomicAdd(cnt, 1) == nact - 1);
    sy.sync();
    if (!sm.last) return;
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

// grid (nchunks, Hkv, B), 128 threads: CTA (c, g, b) runs work item (c, g, b).
template <typename Acc, int HS, int REP>
__global__ void __launch_bounds__(128) k_attention(const AttnArgs a) {
    __shared__ AttnSmem<Acc, HS, REP> sm;
    grid_dep_wait();
    grid_dep_launch();
    attn_item<Acc, HS, REP>(a, blockIdx.x, blockIdx.y, blockIdx.z, threadIdx.x, SyncCTA(), sm);
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
