// attention.cuh - flash-decode grouped-query attention of one layer (sm_100a).
//
// Shared by the step kernels and by standalone entry points: it holds only
// templates and inline functions, so any translation unit may include it.
//
// Work item (chunk c, KV head g, sequence b): the positions [t0, t1) of the
// chunk, for the rep = H/Hkv query heads that share KV head g (heads
// g*rep .. g*rep+rep-1: contiguous groups), so every K/V row is read once per
// group.  One CTA per item: 8 warps in fp32 (K/V batches in registers), 4
// in double (K/V batches streamed into per-lane shared-memory rings with
// cp.async).  Each warp takes batches of positions in turn and runs an online
// softmax over them (scores from one reduce-scatter per head, running max,
// rescaled weighted V sum) while its next batches load; then the warps merge
// their states.  Rows before the current position do not depend on the
// kernel that precedes attention in the step, so a warp's first batches are
// read before the dependency wait when they do not contain a row the kernel
// before writes.
//
// Each active chunk writes its (o, m, l) per head; the last CTA to arrive for
// (b, g) (an atomic counter, no spin-wait) merges them:
// M = max m_c, L = sum l_c e^{m_c - M}, O = sum o_c e^{m_c - M}; out = O / L.
// A single active chunk writes O / L directly.
//
// Precision.  Acc = float accumulates in fp32 (the fp32 step).  Acc = double
// accumulates in double (the Q8_0 step, whose attention output is quantized,
// so it must round to the same fp32 values as a double reference): K and V
// elements are widened to double with integer operations instead of the
// conversion instruction, which issues on a narrow unit.  The widening keeps
// the float's bits and leaves its exponent unbiased, i.e. it yields x * 2^-896
// exactly, for every finite x including zeros and subnormals; scores and the
// weighted V sums are scaled back by 2^896 (exact) once per position / once
// at the end.  Products below 2^-126 in magnitude flush to zero there, far
// below the last bit of any sum they join.  A non-finite K or V element makes
// the output NaN.
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
    int nchunks;         // gridDim.x: the positions 0..pos are split into at most this many chunks
    int min_chunk;       // ... of at least this many positions each
    int shared_kv;       // 1: every entry reads one cache (the tokens of a prompt chunk, positions rising from
                         // entry 0's): rows from entry 0's position on come from the kernel before
    void* part;          // partials [B][Hkv][nchunks][rep][hs+2] (Acc)
    int* count;          // [B][Hkv] arrival counters (zero between launches)
    // int8 KV cache (the double kernel's KV8 form): this layer's codes of
    // sequence 0 ([S][kvd], sequence b at + b*seq_stride) and scales
    // ([S][Hkv], sequence b at + b*sc_seq_stride)
    const int8_t* kq;
    const int8_t* vq;
    const float* ks;
    const float* vs;
    size_t sc_seq_stride;
};

// x * 2^-896 as a double, exactly, for every finite float x (see above).
__device__ __forceinline__ double widen_scaled(float x) {
    const uint32_t b = __float_as_uint(x);
    const uint32_t hi = ((b & 0x7fffffffu) >> 3) | (b & 0x80000000u);
    return __hiloint2double((int)hi, (int)(b << 29));
}
constexpr double kTwo896 = 0x1p896;

// chk + v * 0 over the four elements: NaN once any element is infinite or
// NaN (the widening above would turn those into finite doubles), else chk.
__device__ __forceinline__ float nonfinite_fold(const float4 v, float chk) {
    chk = __fmaf_rn(v.x, 0.f, chk);
    chk = __fmaf_rn(v.y, 0.f, chk);
    chk = __fmaf_rn(v.z, 0.f, chk);
    return __fmaf_rn(v.w, 0.f, chk);
}

template <typename Acc>
__device__ __forceinline__ void widen4(const float4 v, Acc (&w)[4]) {
    if (sizeof(Acc) == 8) {
        w[0] = (Acc)widen_scaled(v.x); w[1] = (Acc)widen_scaled(v.y);
        w[2] = (Acc)widen_scaled(v.z); w[3] = (Acc)widen_scaled(v.w);
    } else {
        w[0] = (Acc)v.x; w[1] = (Acc)v.y; w[2] = (Acc)v.z; w[3] = (Acc)v.w;
    }
}

constexpr int ATTN_WARPS = 4;       // warps of a double-precision attention CTA
constexpr int ATTN_THREADS = 32 * ATTN_WARPS;
constexpr int ATTN_WARPS_F32 = 8;   // warps of an fp32 attention CTA (one CTA per SM: more loads in flight)

// Threads of an attention CTA of accumulator type Acc.
template <typename Acc>
constexpr int attn_threads() {
    return sizeof(Acc) == 8 ? ATTN_THREADS : 32 * ATTN_WARPS_F32;
}
constexpr int ATTN_NB = 3;  // batches in each lane's shared-memory ring

// Positions a warp loads at once (one batch): fewer when the query group is
// large, to bound the registers of the batch being computed.  In double,
// batches of 8 (two CTAs per SM with their 96 KB rings) measured faster than
// batches of 4 (four CTAs per SM) or 2 for MHA, and 4 faster than 2 or 1 at a
// GQA ratio of 4.
template <typename Acc, int REP>
struct AttnPB {
    static constexpr int value = sizeof(Acc) == 8 ? (REP >= 8 ? 2 : (REP >= 4 ? 4 : 8)) : (REP >= 3 ? 4 : 8);
};

// Dynamic shared memory of an attention CTA: per warp ATTN_NB batches of PB
// positions, K and V, one float4 per lane.
template <typename Acc, int REP>
constexpr int attn_ring_bytes() {
    return ATTN_WARPS * ATTN_NB * AttnPB<Acc, REP>::value * 2 * 32 * 16;
}

// 16-byte global -> shared asynchronous copy (cp.async, L2 evict-first); with
// on == false nothing is read and the destination is zero-filled.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool on, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(on ? 16 : 0), "l"(pol) : "memory");
}
// 4-byte form (int8 KV cache codes and scales)
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool on) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(smem_u32(dst)), "l"(src), "r"(on ? 4 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// One head's K or V row (hs <= 128 values at x) into the int8 KV cache with
// one warp: quantize() of "超精简LLM部署" §1 over the whole row (the group is the
// head), codes to q, the scale to *sc, and code * scale back over x.  A
// non-finite element makes the scale NaN (every read of the group is NaN).
__device__ __forceinline__ void kv8_store_head(float* x, int8_t* q, float* sc, int hs) {
    const int lane = threadIdx.x & 31;
    float v[4];
    float m = 0.f;
    bool bad = false;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const int i = lane + 32 * e;
        v[e] = i < hs ? x[i] : 0.f;
        m = fmaxf(m, fabsf(v[e]));
        bad |= !isfinite(v[e]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float scale = __any_sync(0xffffffffu, bad) ? __int_as_float(0x7fc00000) : m / 127.0f;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const int i = lane + 32 * e;
        if (i >= hs) break;
        const int code = scale != 0.f && scale == scale ? (int)roundf(v[e] / scale) : 0;
        q[i] = (int8_t)code;
        x[i] = __fmul_rn((float)code, scale);
    }
    if (lane == 0) *sc = scale;
}

// A ring entry of the int8 KV cache: .x holds four codes (little-endian), .y
// their head's scale; the values are code * scale (fp32 multiplies).
__device__ __forceinline__ float4 kv8_decode(const float4 e) {
    const uint32_t c = __float_as_uint(e.x);
    const float s = e.y;
    return make_float4(__fmul_rn((float)(int8_t)(c & 0xffu), s), __fmul_rn((float)(int8_t)((c >> 8) & 0xffu), s),
                       __fmul_rn((float)(int8_t)((c >> 16) & 0xffu), s), __fmul_rn((float)(int8_t)(c >> 24), s));
}
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

// The merge of a work item's NW warps and of the chunks of (b, g); every
// thread of the CTA calls it after its warp's online softmax is done.
template <typename Acc, int HS, int REP, int NW>
__device__ __forceinline__ void attn_finish(const AttnArgs& a, int c, int g, int b, int nact, const Acc (&m)[REP],
                                            const Acc (&l)[REP], const Acc (&o)[REP][4], Acc (*sm_m)[REP],
                                            Acc (*sm_l)[REP], Acc (*sm_o)[REP][HS], int* last_s) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool lane_on = lane < HS / 4;
    // merge the warps' states (a warp without positions has m = -inf, l = 0)
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < REP; h++) {
            sm_m[warp][h] = m[h];
            sm_l[warp][h] = l[h];
        }
    }
    if (lane_on) {
#pragma unroll
        for (int h = 0; h < REP; h++)
#pragma unroll
            for (int e = 0; e < 4; e++) sm_o[warp][h][4 * lane + e] = o[h][e];
    }
    __syncthreads();
    Acc* part = static_cast<Acc*>(a.part) + ((((size_t)b * a.Hkv + g) * a.nchunks + c) * REP) * (HS + 2);
    for (int i = tid; i < REP * HS; i += (32 * NW)) {
        const int h = i / HS, e = i % HS;
        Acc M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; w++) M = max(M, sm_m[w][h]);
        Acc L = 0, O = 0;
#pragma unroll
        for (int w = 0; w < NW; w++) {
            const Acc f = sm_m[w][h] == -INFINITY ? (Acc)0 : exp(sm_m[w][h] - M);
            L += sm_l[w][h] * f;
            O += sm_o[w][h][e] * f;
        }
        if (nact == 1) {
            a.out[(size_t)b * a.H * HS + ((size_t)g * REP + h) * HS + e] = (float)(O / L);
        } else {
            part[(size_t)h * (HS + 2) + e] = O;
            if (e == 0) {
                part[(size_t)h * (HS + 2) + HS] = M;
                part[(size_t)h * (HS + 2) + HS + 1] = L;
            }
        }
    }
    if (nact == 1) return;
    // the last CTA of (b, g) to arrive merges the chunks
    __threadfence();
    __syncthreads();
    int* cnt = a.count + (size_t)b * a.Hkv + g;
    if (tid == 0) *last_s = (atomicAdd(cnt, 1) == nact - 1);
    __syncthreads();
    if (!*last_s) return;
    __threadfence();
    const Acc* p0 = static_cast<const Acc*>(a.part) + (((size_t)b * a.Hkv + g) * a.nchunks * REP) * (HS + 2);
    for (int i = tid; i < REP * HS; i += (32 * NW)) {
        const int h = i / HS, e = i % HS;
        Acc M = -INFINITY, Ls = 0, Os = 0;
        auto term = [&](int k) {
            const Acc* pk = p0 + ((size_t)k * REP + h) * (HS + 2);
            const Acc f = exp(__ldcg(pk + HS) - M);
            Ls += __ldcg(pk + HS + 1) * f;
            Os += __ldcg(pk + e) * f;
        };
        if (sizeof(Acc) == 8) {
            // double: up to 4 CTAs per SM, so many chunks; unrolled, the chunks'
            // loads (independent of one another) are in flight together
#pragma unroll 8
            for (int k = 0; k < nact; k++) M = max(M, __ldcg(p0 + ((size_t)k * REP + h) * (HS + 2) + HS));
#pragma unroll 8
            for (int k = 0; k < nact; k++) term(k);
        } else {
            for (int k = 0; k < nact; k++) M = max(M, __ldcg(p0 + ((size_t)k * REP + h) * (HS + 2) + HS));
            for (int k = 0; k < nact; k++) term(k);
        }
        a.out[(size_t)b * a.H * HS + ((size_t)g * REP + h) * HS + e] = (float)(Os / Ls);
    }
    if (tid == 0) *cnt = 0;
}

// The online-softmax update of one warp with a batch of PB positions (n of
// them valid): K and V row slices of this lane (one float4 each).
template <typename Acc, int REP, int PB, typename KV>
__device__ __forceinline__ void attn_batch(int n, KV kv, const Acc (&qr)[REP][4], Acc scale, Acc (&m)[REP],
                                           Acc (&l)[REP], Acc (&o)[REP][4]) {
    float4 kr[PB];
#pragma unroll
    for (int i = 0; i < PB; i++) kr[i] = kv(i, 0);
#pragma unroll
    for (int h = 0; h < REP; h++) {
        Acc sp[PB];
#pragma unroll
        for (int i = 0; i < PB; i++) {
            Acc kw[4];
            widen4<Acc>(kr[i], kw);
            sp[i] = kw[0] * qr[h][0] + kw[1] * qr[h][1] + kw[2] * qr[h][2] + kw[3] * qr[h][3];
        }
        // lane l holds the score of position (l / (32/PB)) % PB of the batch:
        // the batch max comes from the lanes of the other positions, and each
        // lane takes the exponential of its own position only (one exp per
        // lane instead of PB), then the weights are broadcast
        const Acc tot = warp_sum_scatter<PB>(sp);
        const int mine = ((threadIdx.x & 31) / (32 / PB)) % PB;
        const Acc sc = mine < n ? tot * scale : (Acc)-INFINITY;
        Acc mx = sc;
#pragma unroll
        for (int sh = 32 / PB; sh < 32; sh <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, sh));
        const Acc mnew = max(m[h], mx);
        // exp(-inf) = 0 on the warp's first batch; an unchanged max scales by 1
        const Acc alpha = mnew == m[h] ? (Acc)1 : exp(m[h] - mnew);
        const Acc pm = exp(sc - mnew);  // masked positions: exp(-inf) = 0
        Acc ps = 0, w4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < PB; i++) {
            const Acc p = __shfl_sync(0xffffffffu, pm, i * (32 / PB));
            Acc vw[4];
            widen4<Acc>(kv(i, 1), vw);
            ps += p;
            w4[0] += p * vw[0]; w4[1] += p * vw[1]; w4[2] += p * vw[2]; w4[3] += p * vw[3];
        }
        l[h] = l[h] * alpha + ps;
        o[h][0] = o[h][0] * alpha + w4[0]; o[h][1] = o[h][1] * alpha + w4[1];
        o[h][2] = o[h][2] * alpha + w4[2]; o[h][3] = o[h][3] * alpha + w4[3];
        m[h] = mnew;
    }
}

// The work item of CTA (c, g, b): its chunk [t0, t1) and the number of
// active chunks of sequence b; false when this CTA has no positions.  Rows
// before `fresh` were written before the step (readable before the
// dependency wait): all rows before the entry's own position, or with a
// shared cache those before entry 0's position.
__device__ __forceinline__ bool attn_item(const AttnArgs& a, int c, int b, int& t0, int& t1, int& nact, int& pos,
                                          int& fresh) {
    pos = a.tp[b * a.tp_stride + 1];  // written before the step: readable before the wait
    if (pos < 0 || pos >= a.seq_len) pos = 0;  // the q/k/v kernel has flagged it
    fresh = pos;
    if (a.shared_kv) {
        const int p0 = a.tp[1];
        fresh = p0 < 0 ? 0 : (p0 < pos ? p0 : pos);
    }
    const int T = pos + 1;
    nact = (T + a.min_chunk - 1) / a.min_chunk;
    if (nact > a.nchunks) nact = a.nchunks;
    const int chunk = (T + nact - 1) / nact;
    nact = (T + chunk - 1) / chunk;
    if (c >= nact) return false;
    t0 = c * chunk;
    t1 = min(T, t0 + chunk);
    return true;
}

template <int REP>
struct AttnPBF {  // fp32 kernel: positions per batch
    static constexpr int value = REP >= 3 ? 4 : 8;
};

// fp32 attention, grid (nchunks, Hkv, B), 32 * ATTN_WARPS_F32 threads, no
// dynamic shared memory (the fp32 step's kernels keep the default L1 / shared
// split).  The chunk's positions go in batches of PB to the warps in turn; a lane
// holds one float4 of each K and V row slice (hs <= 128) in registers, and
// every warp keeps the next batch's 128-bit loads in flight while it computes
// the current one.
template <int HS, int REP>
__global__ void __launch_bounds__(32 * ATTN_WARPS_F32) k_attention_f32(const AttnArgs a) {
    constexpr int V4 = HS / 4;
    constexpr int PB = AttnPBF<REP>::value;
    static_assert(HS % 4 == 0 && HS <= 128, "head size");
    __shared__ float sm_m[ATTN_WARPS_F32][REP], sm_l[ATTN_WARPS_F32][REP];
    __shared__ float sm_o[ATTN_WARPS_F32][REP][HS];
    __shared__ int last_s;
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool lane_on = lane < V4;
    int t0, t1, nact, pos;
    int fresh;
    if (!attn_item(a, c, b, t0, t1, nact, pos, fresh)) return;
    const int nb = (t1 - t0 + PB - 1) / PB;
    const float* kc = a.kc + (size_t)b * a.seq_stride + (size_t)g * HS + 4 * lane;
    const float* vc = a.vc + (size_t)b * a.seq_stride + (size_t)g * HS + 4 * lane;
    const uint64_t pol = policy_evict_first();
    auto load = [&](int bi, float4 (&kr)[PB], float4 (&vr)[PB]) {
#pragma unroll
        for (int i = 0; i < PB; i++) {
            const int t = t0 + bi * PB + i;
            const bool on = lane_on && t < t1;
            kr[i] = on ? ld_stream_f4(reinterpret_cast<const float4*>(kc + (size_t)t * a.kvd), pol)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
            vr[i] = on ? ld_stream_f4(reinterpret_cast<const float4*>(vc + (size_t)t * a.kvd), pol)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    float4 ka[PB], va[PB], kb[PB], vb[PB];
    int bi = warp;
    // the warp's first batch, if all its rows precede `fresh` (rows from
    // there on come from the kernel before), is read before the wait
    const bool early = bi < nb && t0 + (bi + 1) * PB <= fresh;
    if (early) load(bi, ka, va);
    grid_dep_wait();
    grid_dep_launch();
    if (!early && bi < nb) load(bi, ka, va);
    const float* q = a.q + (size_t)b * a.H * HS + (size_t)g * REP * HS;
    float qr[REP][4];
#pragma unroll
    for (int h = 0; h < REP; h++) {
        const float4 qv = lane_on ? __ldg(reinterpret_cast<const float4*>(q + (size_t)h * HS) + lane)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        qr[h][0] = qv.x; qr[h][1] = qv.y; qr[h][2] = qv.z; qr[h][3] = qv.w;
    }
    const float scale = 1.0f / sqrtf((float)HS);
    float m[REP], l[REP], o[REP][4];
#pragma unroll
    for (int h = 0; h < REP; h++) {
        m[h] = -INFINITY;
        l[h] = 0.f;
        o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0.f;
    }
    // two register buffers: batch bi in (ka, va), the next one loading into (kb, vb)
    while (bi < nb) {
        if (bi + ATTN_WARPS_F32 < nb) load(bi + ATTN_WARPS_F32, kb, vb);
        attn_batch<float, REP, PB>(min(PB, t1 - (t0 + bi * PB)),
                                   [&](int i, int kv) { return kv ? va[i] : ka[i]; }, qr, scale, m, l, o);
        bi += ATTN_WARPS_F32;
        if (bi >= nb) break;
        if (bi + ATTN_WARPS_F32 < nb) load(bi + ATTN_WARPS_F32, ka, va);
        attn_batch<float, REP, PB>(min(PB, t1 - (t0 + bi * PB)),
                                   [&](int i, int kv) { return kv ? vb[i] : kb[i]; }, qr, scale, m, l, o);
        bi += ATTN_WARPS_F32;
    }
    attn_finish<float, HS, REP, ATTN_WARPS_F32>(a, c, g, b, nact, m, l, o, sm_m, sm_l, sm_o, &last_s);
}

// grid (nchunks, Hkv, B), ATTN_THREADS threads, attn_ring_bytes<Acc, REP>()
// bytes of dynamic shared memory: CTA (c, g, b) runs work item (c, g, b).
// The chunk's positions go in batches of PB to the ATTN_WARPS warps in turn; a lane
// owns one float4 of each K and V row slice (hs <= 128) and streams it into
// its own ring of ATTN_NB batches in shared memory with cp.async, so two
// batches are in flight while it computes a third, without holding them in
// registers (each lane reads back only what it copied: no synchronisation).
template <typename Acc, int HS, int REP, bool KV8 = false>
__global__ void __launch_bounds__(ATTN_THREADS) k_attention(const AttnArgs a) {
    constexpr bool DBL = sizeof(Acc) == 8;
    constexpr int V4 = HS / 4;  // float4 per row slice (<= 32: one per lane)
    constexpr int PB = AttnPB<Acc, REP>::value;
    static_assert(HS % 4 == 0 && HS <= 128, "head size");
    extern __shared__ __align__(16) float4 aring[];
    __shared__ Acc sm_m[ATTN_WARPS][REP], sm_l[ATTN_WARPS][REP];
    __shared__ Acc sm_o[ATTN_WARPS][REP][HS];
    __shared__ int last_s;
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool lane_on = lane < V4;
    int t0, t1, nact, pos;
    int fresh;
    if (!attn_item(a, c, b, t0, t1, nact, pos, fresh)) return;
    const int nb = (t1 - t0 + PB - 1) / PB;   // batches of the chunk; warp w takes w, w+4, ...
    const float* kc = a.kc + (size_t)b * a.seq_stride + (size_t)g * HS + 4 * (lane_on ? lane : 0);
    const float* vc = a.vc + (size_t)b * a.seq_stride + (size_t)g * HS + 4 * (lane_on ? lane : 0);
    const uint64_t pol = policy_evict_first();
    // KV8: this lane's four codes and its head's scale of each K / V row
    const int8_t* kq = KV8 ? a.kq + (size_t)b * a.seq_stride + (size_t)g * HS + 4 * (lane_on ? lane : 0) : nullptr;
    const int8_t* vq = KV8 ? a.vq + (size_t)b * a.seq_stride + (size_t)g * HS + 4 * (lane_on ? lane : 0) : nullptr;
    const float* ksc = KV8 ? a.ks + (size_t)b * a.sc_seq_stride + g : nullptr;
    const float* vsc = KV8 ? a.vs + (size_t)b * a.sc_seq_stride + g : nullptr;
    float4* ring = aring + (size_t)warp * ATTN_NB * PB * 2 * 32;
    // ring entry of (slot, position i, K or V) for this lane
    auto ent = [&](int slot, int i, int kv) -> float4* { return ring + ((slot * PB + i) * 2 + kv) * 32 + lane; };
    // its values (KV8: this lane's codes, decoded with the head's scale, which
    // lane 0 alone copies into its own entry)
    auto val = [&](int slot, int i, int kv) -> float4 {
        if (!KV8) return *ent(slot, i, kv);
        float4 e = *ent(slot, i, kv);
        e.y = (ring + ((slot * PB + i) * 2 + kv) * 32)->y;
        return kv8_decode(e);
    };
    // copies of the warp's jj-th batch into slot jj % ATTN_NB; always one commit group
    auto issue = [&](int jj) {
        const int bi = warp + ATTN_WARPS * jj;
        const int slot = jj % ATTN_NB;
#pragma unroll
        for (int i = 0; i < PB; i++) {
            const int t = t0 + bi * PB + i;
            const bool on = lane_on && bi < nb && t < t1;
            const size_t off = on ? (size_t)t * a.kvd : 0;
            if (KV8) {
                const bool pos_on = bi < nb && t < t1;
                const size_t so = pos_on ? (size_t)t * a.Hkv : 0;
                cp_async4(&ent(slot, i, 0)->x, kq + off, on);
                cp_async4(&ent(slot, i, 1)->x, vq + off, on);
                if (lane == 0) {
                    cp_async4(&ent(slot, i, 0)->y, ksc + so, pos_on);
                    cp_async4(&ent(slot, i, 1)->y, vsc + so, pos_on);
                }
            } else {
                cp_async16(ent(slot, i, 0), kc + off, on, pol);
                cp_async16(ent(slot, i, 1), vc + off, on, pol);
            }
        }
        cp_async_commit();
    };
    // a batch whose rows all precede `fresh` (rows from there on come from
    // the kernel before) may be copied before the dependency wait
    auto before_wait_ok = [&](int jj) { return t0 + (warp + ATTN_WARPS * jj + 1) * PB <= fresh; };
    int nissued = 0;
    while (nissued < ATTN_NB - 1 && before_wait_ok(nissued)) issue(nissued++);
    grid_dep_wait();
    grid_dep_launch();
    if (KV8 && t1 == pos + 1) {
        // this CTA's chunk holds the current position: its warp 0 stores the
        // K and V rows at pos of head g (written by the q/k/v kernel, fp32)
        // into the int8 cache, and the fp32 rows as code * scale, before any
        // warp copies that row (the copies of earlier rows are unaffected)
        if (warp == 0) {
            kv8_store_head(const_cast<float*>(a.kc) + (size_t)b * a.seq_stride + (size_t)pos * a.kvd + (size_t)g * HS,
                           const_cast<int8_t*>(a.kq) + (size_t)b * a.seq_stride + (size_t)pos * a.kvd + (size_t)g * HS,
                           const_cast<float*>(a.ks) + (size_t)b * a.sc_seq_stride + (size_t)pos * a.Hkv + g, HS);
            kv8_store_head(const_cast<float*>(a.vc) + (size_t)b * a.seq_stride + (size_t)pos * a.kvd + (size_t)g * HS,
                           const_cast<int8_t*>(a.vq) + (size_t)b * a.seq_stride + (size_t)pos * a.kvd + (size_t)g * HS,
                           const_cast<float*>(a.vs) + (size_t)b * a.sc_seq_stride + (size_t)pos * a.Hkv + g, HS);
            __threadfence();
        }
        __syncthreads();
    }
    while (nissued < ATTN_NB - 1) issue(nissued++);

    const float* q = a.q + (size_t)b * a.H * HS + (size_t)g * REP * HS;
    Acc qr[REP][4];
#pragma unroll
    for (int h = 0; h < REP; h++) {
        const float4 qv = lane_on ? __ldg(reinterpret_cast<const float4*>(q + (size_t)h * HS) + lane)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        qr[h][0] = (Acc)qv.x; qr[h][1] = (Acc)qv.y; qr[h][2] = (Acc)qv.z; qr[h][3] = (Acc)qv.w;
    }
    // score scale (the 2^896 of the widened K elements folded in)
    const Acc scale = DBL ? (Acc)(kTwo896 / sqrt((double)HS)) : (Acc)1 / sqrt((Acc)HS);
    Acc m[REP], l[REP], o[REP][4];
#pragma unroll
    for (int h = 0; h < REP; h++) {
        m[h] = -INFINITY;
        l[h] = 0;
        o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0;
    }
    // non-finite K/V elements (double path): x * 0 is NaN exactly for an
    // infinite or NaN x, so one FMA per element (on the FMA pipe, which this
    // kernel leaves idle) folds every element into chk
    float chk = 0.f;
    for (int jj = 0;; jj++) {
        const int bi = warp + ATTN_WARPS * jj;
        if (bi >= nb) break;
        cp_async_wait<ATTN_NB - 2>();  // batch jj has landed (this lane's copies)
        if (KV8) __syncwarp();         // ... and lane 0's scales, for every lane
        issue(jj + ATTN_NB - 1);       // into the slot read in the previous round
        const int slot = jj % ATTN_NB;
        if (DBL) {
#pragma unroll
            for (int i = 0; i < PB; i++) chk = nonfinite_fold(val(slot, i, 1), nonfinite_fold(val(slot, i, 0), chk));
        }
        attn_batch<Acc, REP, PB>(min(PB, t1 - (t0 + bi * PB)), [&](int i, int kv) { return val(slot, i, kv); }, qr,
                                 scale, m, l, o);
    }
    cp_async_wait<0>();  // no copy of this lane may land after the CTA leaves
    if (DBL) {
#pragma unroll
        for (int h = 0; h < REP; h++) {
            o[h][0] *= (Acc)kTwo896; o[h][1] *= (Acc)kTwo896; o[h][2] *= (Acc)kTwo896; o[h][3] *= (Acc)kTwo896;
        }
        if (__any_sync(0xffffffffu, chk != chk))
#pragma unroll
            for (int h = 0; h < REP; h++) o[h][0] = o[h][1] = o[h][2] = o[h][3] = (Acc)NAN;
    }
    attn_finish<Acc, HS, REP, ATTN_WARPS>(a, c, g, b, nact, m, l, o, sm_m, sm_l, sm_o, &last_s);
}

typedef void (*AttnKernel)(const AttnArgs);

// The attention instantiation for a head size and GQA ratio (nullptr if none):
// k_attention_f32 for Acc = float, k_attention<double> for Acc = double.
#define L2C_ATTN_SHAPES(X)                                                                  \
    X(8, 1) X(8, 2) X(8, 3) X(8, 4) X(16, 1) X(16, 2) X(16, 4) X(32, 1) X(32, 2) X(32, 4) \
    X(48, 1) X(48, 2) X(48, 4) X(64, 1) X(64, 2) X(64, 4) X(64, 8) X(96, 1) X(96, 2)      \
    X(96, 4) X(128, 1) X(128, 2) X(128, 4) X(128, 8)

template <typename Acc>
inline AttnKernel attn_kernel_for(int hs, int rep) {
#define L2C_ATTN_F(HS_, REP_) \
    if (hs == HS_ && rep == REP_) return k_attention_f32<HS_, REP_>;
#define L2C_ATTN_D(HS_, REP_) \
    if (hs == HS_ && rep == REP_) return k_attention<double, HS_, REP_>;
    if (sizeof(Acc) == 4) {
        L2C_ATTN_SHAPES(L2C_ATTN_F)
    } else {
        L2C_ATTN_SHAPES(L2C_ATTN_D)
    }
#undef L2C_ATTN_F
#undef L2C_ATTN_D
    return nullptr;
}

// The double kernel reading the int8 KV cache, for (hs, rep).
inline AttnKernel attn_kernel_kv8(int hs, int rep) {
#define L2C_ATTN_Q(HS_, REP_) \
    if (hs == HS_ && rep == REP_) return k_attention<double, HS_, REP_, true>;
    L2C_ATTN_SHAPES(L2C_ATTN_Q)
#undef L2C_ATTN_Q
    return nullptr;
}

// Dynamic shared memory of the attention instantiation for a GQA ratio (the
// fp32 kernel has none).
template <typename Acc>
inline int attn_smem_for(int rep) {
    if (sizeof(Acc) == 4) return 0;
    switch (rep) {
    case 1: return attn_ring_bytes<double, 1>();
    case 2: return attn_ring_bytes<double, 2>();
    case 3: return attn_ring_bytes<double, 3>();
    case 4: return attn_ring_bytes<double, 4>();
    default: return attn_ring_bytes<double, 8>();
    }
}

// The double attention kernels: their ring's shared-memory limit (above the
// default 48 KB for some), and all of the shared memory as carveout, as the
// Q8_0 kernels they run between ask for.
inline cudaError_t attn_set_smem_limits() {
    cudaError_t e = cudaSuccess;
#define L2C_ATTN_ATTR(HS_, REP_)                                                                                  \
    if ((e = cudaFuncSetAttribute(k_attention<double, HS_, REP_>, cudaFuncAttributeMaxDynamicSharedMemorySize,    \
                                  attn_ring_bytes<double, REP_>())) != cudaSuccess)                               \
        return e;                                                                                                 \
    if ((e = cudaFuncSetAttribute(k_attention<double, HS_, REP_>, cudaFuncAttributePreferredSharedMemoryCarveout, \
                                  (int)cudaSharedmemCarveoutMaxShared)) != cudaSuccess)                           \
        return e;
    L2C_ATTN_SHAPES(L2C_ATTN_ATTR)
#undef L2C_ATTN_ATTR
#define L2C_ATTN_ATTR_Q(HS_, REP_)                                                                                \
    if ((e = cudaFuncSetAttribute(k_attention<double, HS_, REP_, true>,                                           \
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, attn_ring_bytes<double, REP_>())) != \
        cudaSuccess)                                                                                              \
        return e;                                                                                                 \
    if ((e = cudaFuncSetAttribute(k_attention<double, HS_, REP_, true>,                                           \
                                  cudaFuncAttributePreferredSharedMemoryCarveout,                                 \
                                  (int)cudaSharedmemCarveoutMaxShared)) != cudaSuccess)                           \
        return e;
    L2C_ATTN_SHAPES(L2C_ATTN_ATTR_Q)
#undef L2C_ATTN_ATTR_Q
    return e;
}

}  // namespace l2c
