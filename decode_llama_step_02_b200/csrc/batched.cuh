// batched.cuh - the Q8_0 decode step for B independent sequences (sm_100a).
//
// With B sequences each matvec becomes a skinny GEMM Y[B][rows] = X[B][K] W^T.
// At B = 32 the int8 work is 32 multiply-adds per weight byte, more than dp4a
// sustains at HBM speed, so the group dot products run on the tensor cores:
// mma.sync m16n8k32 s8*s8 -> s32 gives the exact int32 dot of every
// (row, sequence, group), then ival * sw * sx is summed over groups in double,
// as in the single-sequence kernel.  Per layer:
//
//   prep<QKV>   per sequence: embedding row (layer 0), RMSNorm, quantize -> xq, xs
//   gemm<QKV>   q, RoPE, K/V cache write at each sequence's own position
//   attention   k_attention over (chunk, KV head, sequence), ragged positions
//   prep<Q>     quantize the attention output
//   gemm<RESID> x += Wo att
//   prep<QKV>   RMSNorm + quantize
//   gemm<W13>   hb = silu(W1 x) * (W3 x)
//   prep<Q>     quantize hb
//   gemm<RESID> x += W2 hb
// and prep + gemm<CLS> (logits and a per-sequence argmax) at the end.
#pragma once
#include "kernels.cuh"

namespace l2c {

constexpr int BMAX = 32;          // sequences per GEMM (n = 4 tiles of 8)
constexpr int BG_WARPS = 2;       // consumer warps per CTA, 16 rows each
constexpr int BG_ROWS = 16 * BG_WARPS;
constexpr int BPREP_SPLIT = 8;    // CTAs per sequence of the prep kernel (ranges of groups)

struct BPrepArgs {
    const float* in;        // [B][K] fp32 input (x, attention output or hb)
    size_t in_stride;       // floats between sequences
    const float* norm_w;    // RMSNorm gain or nullptr
    const uint8_t* emb;     // layer 0: embedding row records (codes | scales), else nullptr
    size_t emb_rb;          // record bytes
    float* x_resid;         // layer 0: receives the dequantized embedding rows [B][d]
    int K, gs;
    int8_t* xq;             // [B][kq_stride] codes
    double* xs;             // [B][ks_stride] scales, in double (exact copies of the fp32 scales)
    size_t kq_stride, ks_stride;
    const int* tp;          // [B][2] token, pos
    int vocab, seq_len;
    unsigned long long* amax;  // reset per sequence on layer 0
    int* err;
};

// CTA (b, y) of a (B, Y) grid: sequence b's input row and its RMSNorm sum (the
// whole row, in every CTA of the sequence), then the RMSNorm (double) and the
// Q8_0 codes of the y-th of Y equal ranges of the row's groups.
__global__ void __launch_bounds__(256) k_bprep(const BPrepArgs a) {
    extern __shared__ float bp_xs[];
    __shared__ double red[32];
    const int b = blockIdx.x;
    const int ngr = a.K / a.gs;
    const int g0 = (int)((long long)ngr * blockIdx.y / gridDim.y);
    const int g1 = (int)((long long)ngr * (blockIdx.y + 1) / gridDim.y);
    const int i0 = g0 * a.gs, i1 = g1 * a.gs;  // this CTA's elements
    grid_dep_wait();
    grid_dep_launch();
    const int K = a.K, gs = a.gs;
    const float* in = a.in + (size_t)b * a.in_stride;
    if (a.emb) {
        int token = a.tp[2 * b];
        if (token < 0 || token >= a.vocab) {
            if (threadIdx.x == 0) set_error(a.err, DERR_TOKEN);
            token = 0;
        }
        const uint8_t* rec = a.emb + (size_t)token * a.emb_rb;
        const int8_t* eq = reinterpret_cast<const int8_t*>(rec);
        const float* es = reinterpret_cast<const float*>(rec + K);
        for (int i = threadIdx.x; i < K; i += blockDim.x) {
            float v = (float)eq[i] * es[i / gs];
            bp_xs[i] = v;
            if (i >= i0 && i < i1) a.x_resid[(size_t)b * K + i] = v;
        }
        if (a.amax && threadIdx.x == 0 && blockIdx.y == 0) a.amax[b] = 0ull;
    } else if (a.norm_w) {
        for (int i = threadIdx.x; i < K; i += blockDim.x) bp_xs[i] = in[i];  // the whole row for the norm
    } else {
        for (int i = i0 + (int)threadIdx.x; i < i1; i += blockDim.x) bp_xs[i] = in[i];
    }
    __syncthreads();
    if (a.norm_w) {
        double ss = 0.0;
        for (int i = threadIdx.x; i < K; i += blockDim.x) ss += (double)bp_xs[i] * (double)bp_xs[i];
        ss = block_sum(ss, red);
        double inv = 1.0 / sqrt(ss / (double)K + 1e-5);
        for (int i = i0 + (int)threadIdx.x; i < i1; i += blockDim.x)
            bp_xs[i] = (float)((double)a.norm_w[i] * (inv * (double)bp_xs[i]));
        __syncthreads();
    }
    const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int8_t* q = a.xq + (size_t)b * a.kq_stride;
    double* s = a.xs + (size_t)b * a.ks_stride;
    for (int g = g0 + warp; g < g1; g += nw) {
        const float scale = quantize_group_warp(bp_xs + g * gs, gs, q + g * gs, nullptr);
        if ((threadIdx.x & 31) == 0) s[g] = (double)scale;
    }
}

struct BGemmArgs {
    const uint8_t* W;       // Q8_0 row records [rows][rb]
    size_t rb;
    int rows, K, gs, kc;    // kc: K bytes per stage (a multiple of 32 and of gs, dividing K; 4 groups'
                            // multiple unless kc == K)
    int B;                  // live sequences (<= BMAX); codes of the others are zero
    const int8_t* xq;       // [BMAX][kq_stride]
    const double* xs;       // [BMAX][ks_stride] activation scales in double
    size_t kq_stride, ks_stride;
    float* out;             // QKV: q [B][d]; RESID: x [B][d]; W13: hb [B][h]; CLS: logits [B][V]
    size_t out_stride;
    float* kc_base;         // QKV: this layer's key cache of sequence 0
    float* vc_base;
    size_t seq_stride;      // floats between sequences' caches
    const float* freq;
    int d, kvd, hs, seq_len;
    const int* tp;
    unsigned long long* amax;
    int* err;
    size_t prefetch_bytes;
};

__device__ __forceinline__ void mma_s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared memory per stage: weights [BG_ROWS][kc+16], weight scales
// [BG_ROWS][kc/gs] fp32, activations [BMAX][kc+16], activation scales
// [BMAX][kc/gs] double.
struct BLayout {
    int ns;
    int kcp;          // kc + 16 (row pitch in shared memory; spreads rows over banks)
    size_t w_off, ws_off, x_off, xs_off, stage_bytes;
};

__host__ __device__ inline BLayout make_blayout(int kc, int gs, int ns) {
    BLayout L;
    L.ns = ns;
    L.kcp = kc + 16;
    const size_t sc = ((size_t)(kc / gs) * 4 + 15) & ~size_t(15);
    const size_t scx = ((size_t)(kc / gs) * 8 + 15) & ~size_t(15);
    L.w_off = 0;
    L.ws_off = L.w_off + (size_t)BG_ROWS * L.kcp;
    L.x_off = L.ws_off + (size_t)BG_ROWS * sc;
    L.xs_off = L.x_off + (size_t)BMAX * L.kcp;
    L.stage_bytes = L.xs_off + (size_t)BMAX * scx;
    L.stage_bytes = (L.stage_bytes + 127) & ~size_t(127);
    return L;
}

// The epilogue of a batched GEMM CTA: its rows r0 .. r0+nrows-1 of every
// live sequence sit in `so` (fp32, rounded once).  Threads tid of nt (named
// barrier `bar`, nt threads) take (row unit, sequence) pairs:
//   QKV: RoPE of q and k, K/V cache write at each sequence's own position
//   W13: hb = silu(W1 x) * (W3 x) (interleaved rows)
//   RESID: out += v;  CLS: logits and a per-sequence argmax key.
template <int MODE>
__device__ __forceinline__ void bgemm_epilogue(const BGemmArgs& a, int r0, int nrows, const float (*so)[BMAX + 1],
                                               unsigned long long* best_s, int tid, int nt, int bar) {
    if (MODE == M_QKV || MODE == M_W13) {
        for (int i = tid; i < (nrows / 2) * a.B; i += nt) {
            const int up = i / a.B, b = i % a.B;
            const int r = r0 + 2 * up;
            const float v0 = so[2 * up][b], v1 = so[2 * up + 1][b];
            if (MODE == M_W13) {
                a.out[(size_t)b * a.out_stride + r / 2] = (float)(silu_d((double)v0) * (double)v1);
            } else {
                int pos = a.tp[2 * b + 1];
                if (pos < 0 || pos >= a.seq_len) pos = 0;  // flagged by the prep kernel
                if (r < a.d) {
                    float o0, o1;
                    rope_pair(v0, v1, r % a.hs, pos, a.freq, o0, o1);
                    a.out[(size_t)b * a.out_stride + r] = o0;
                    a.out[(size_t)b * a.out_stride + r + 1] = o1;
                } else if (r < a.d + a.kvd) {
                    const int j = r - a.d;
                    float o0, o1;
                    rope_pair(v0, v1, j % a.hs, pos, a.freq, o0, o1);
                    float* k = a.kc_base + (size_t)b * a.seq_stride + (size_t)pos * a.kvd;
                    k[j] = o0;
                    k[j + 1] = o1;
                } else {
                    const int j = r - a.d - a.kvd;
                    float* v = a.vc_base + (size_t)b * a.seq_stride + (size_t)pos * a.kvd;
                    v[j] = v0;
                    v[j + 1] = v1;
                }
            }
        }
    } else {
        for (int i = tid; i < nrows * a.B; i += nt) {
            const int rr = i / a.B, b = i % a.B;
            const float v = so[rr][b];
            float* o = a.out + (size_t)b * a.out_stride + r0 + rr;
            if (MODE == M_RESID) {
                *o = *o + v;
            } else {
                *o = v;
                if (v != v) set_error(a.err, DERR_NAN);
                atomicMax(&best_s[b], argmax_key(v, r0 + rr));
            }
        }
        if (MODE == M_CLS) {
            asm volatile("bar.sync %0, %1;" :: "r"(bar), "r"(nt) : "memory");
            if (tid < a.B && best_s[tid]) atomicMax(&a.amax[tid], best_s[tid]);
        }
    }
}

// grid = ceil(rows / BG_ROWS) CTAs of (BG_WARPS + 1) warps; the last warp is
// the producer (its 32 lanes issue the stage's bulk copies).
template <int MODE>
__global__ void __launch_bounds__(32 * (BG_WARPS + 1)) k_bgemm_q8(const BGemmArgs a, const BLayout L) {
    extern __shared__ __align__(128) uint8_t bsm[];
    __shared__ float stage_out[BG_ROWS][BMAX + 1];
    __shared__ unsigned long long best_s[BMAX];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r0 = blockIdx.x * BG_ROWS;
    const int nrows = min(BG_ROWS, a.rows - r0);
    const int nchunks = a.K / a.kc;
    const int gpc = a.kc / a.gs;                 // groups per chunk
    const size_t sc_bytes = (size_t)gpc * 4;     // scale bytes per row per chunk
    // copy sizes: multiples of 16 bytes (with one chunk, kc == K, the copy runs
    // into the padding of the weight record / of the activation scale row)
    const uint32_t wsc_copy = (uint32_t)((sc_bytes + 15) & ~size_t(15));
    const uint32_t xsc_copy = (uint32_t)((2 * sc_bytes + 15) & ~size_t(15));
    uint64_t* full = reinterpret_cast<uint64_t*>(bsm + (size_t)L.ns * L.stage_bytes);
    uint64_t* empty = full + L.ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < L.ns; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], BG_WARPS);
        }
        mbar_fence_init();
    }
    if (threadIdx.x < BMAX) best_s[threadIdx.x] = 0ull;
    __syncthreads();

    if (warp == BG_WARPS) {
        // ---------------- producer
        const uint64_t pol_w = policy_evict_first();
        const uint64_t pol_x = policy_evict_last();
        const uint8_t* Wb = a.W + (size_t)r0 * a.rb;
        if (lane == 0 && a.prefetch_bytes) {
            // the row block's records are contiguous: prefetch them into L2
            size_t bytes = (size_t)nrows * a.rb;
            if (bytes > a.prefetch_bytes) bytes = a.prefetch_bytes;
            prefetch_l2_range(Wb, bytes & ~size_t(15), policy_evict_last());
        }
        // activations come from the prep kernel: wait for it before copying them
        grid_dep_wait();
        const uint32_t bytes_stage = (uint32_t)((size_t)nrows * (a.kc + wsc_copy) + (size_t)BMAX * (a.kc + xsc_copy));
        bool ok = true;
        int issued = 0;
        for (int c = 0; c < nchunks && ok; c++) {
            const int s = c % L.ns;
            if (c >= L.ns) {
                bool w = true;
                if (lane == 0) w = mbar_wait_bounded(&empty[s], ((c / L.ns) - 1) & 1, a.err);
                w = __shfl_sync(0xffffffffu, w, 0);
                if (!w) { ok = false; break; }
            }
            uint8_t* st = bsm + (size_t)s * L.stage_bytes;
            if (lane == 0) mbar_arrive_expect_tx(&full[s], bytes_stage);
            __syncwarp();
            for (int r = lane; r < nrows; r += 32) {
                const uint8_t* rec = Wb + (size_t)r * a.rb;
                bulk_g2s(st + L.w_off + (size_t)r * L.kcp, rec + (size_t)c * a.kc, a.kc, &full[s], pol_w);
                bulk_g2s(st + L.ws_off + (size_t)r * wsc_copy, rec + a.K + (size_t)c * sc_bytes, wsc_copy, &full[s],
                         pol_w);
            }
            for (int b = lane; b < BMAX; b += 32) {
                bulk_g2s(st + L.x_off + (size_t)b * L.kcp, a.xq + (size_t)b * a.kq_stride + (size_t)c * a.kc, a.kc,
                         &full[s], pol_x);
                bulk_g2s(st + L.xs_off + (size_t)b * xsc_copy,
                         reinterpret_cast<const uint8_t*>(a.xs + (size_t)b * a.ks_stride) + (size_t)c * 2 * sc_bytes,
                         xsc_copy, &full[s], pol_x);
            }
            issued = c + 1;
        }
        if (!ok && lane == 0) {
            for (int c = max(0, issued - L.ns); c < issued; c++)
                mbar_wait_bounded(&full[c % L.ns], (c / L.ns) & 1, a.err);
        }
        return;
    }

    // ---------------- consumers: warp w owns rows r0 + 16w .. +15 of the block
    grid_dep_wait();
    grid_dep_launch();
    const int gid = lane >> 2, tig = lane & 3;
    const size_t scp = (sc_bytes + 15) & ~size_t(15);
    double acc[4][4];
#pragma unroll
    for (int n = 0; n < 4; n++) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0;
    const int wr0 = 16 * warp;   // first row of this warp in the block
    bool ok = true;
    for (int c = 0; c < nchunks; c++) {
        const int s = c % L.ns;
        if (!mbar_wait_bounded(&full[s], (c / L.ns) & 1, a.err)) { ok = false; break; }
        const uint8_t* st = bsm + (size_t)s * L.stage_bytes;
        const uint8_t* wt = st + L.w_off;
        const float* wsc = reinterpret_cast<const float*>(st + L.ws_off);
        const uint8_t* xt = st + L.x_off;
        const double* xsc = reinterpret_cast<const double*>(st + L.xs_off);
        const size_t scxp = ((2 * sc_bytes + 15) & ~size_t(15)) / 8;  // doubles per sequence
        if (wr0 < nrows) {
            for (int g = 0; g < gpc; g++) {
                int cc[4][4];
#pragma unroll
                for (int n = 0; n < 4; n++) cc[n][0] = cc[n][1] = cc[n][2] = cc[n][3] = 0;
                for (int ks = 0; ks < a.gs; ks += 32) {
                    const int k0 = g * a.gs + ks + 4 * tig;
                    uint32_t af[4];
                    af[0] = *reinterpret_cast<const uint32_t*>(wt + (size_t)(wr0 + gid) * L.kcp + k0);
                    af[1] = *reinterpret_cast<const uint32_t*>(wt + (size_t)(wr0 + gid + 8) * L.kcp + k0);
                    af[2] = *reinterpret_cast<const uint32_t*>(wt + (size_t)(wr0 + gid) * L.kcp + k0 + 16);
                    af[3] = *reinterpret_cast<const uint32_t*>(wt + (size_t)(wr0 + gid + 8) * L.kcp + k0 + 16);
#pragma unroll
                    for (int n = 0; n < 4; n++) {
                        const uint8_t* xr = xt + (size_t)(8 * n + gid) * L.kcp + k0;
                        uint32_t b0 = *reinterpret_cast<const uint32_t*>(xr);
                        uint32_t b1 = *reinterpret_cast<const uint32_t*>(xr + 16);
                        mma_s8(cc[n], af, b0, b1);
                    }
                }
                // scale the exact group dots: rows (gid, gid+8), sequences (2 tig, 2 tig + 1) of each tile
                const double sw0 = (double)wsc[(size_t)(wr0 + gid) * (scp / 4) + g];
                const double sw1 = (double)wsc[(size_t)(wr0 + gid + 8) * (scp / 4) + g];
#pragma unroll
                for (int n = 0; n < 4; n++) {
                    const double sx0 = xsc[(size_t)(8 * n + 2 * tig) * scxp + g];
                    const double sx1 = xsc[(size_t)(8 * n + 2 * tig + 1) * scxp + g];
                    acc[n][0] += i2d_exact(cc[n][0]) * sw0 * sx0;
                    acc[n][1] += i2d_exact(cc[n][1]) * sw0 * sx1;
                    acc[n][2] += i2d_exact(cc[n][2]) * sw1 * sx0;
                    acc[n][3] += i2d_exact(cc[n][3]) * sw1 * sx1;
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    // every consumer warp meets the others here, including one that gave up
    // on a wait (the error word is set): then all of them leave together
    const SyncNamed cons{1, 32 * BG_WARPS};
    if (cons.sync_or(!ok)) return;
    // results of this warp's rows -> shared staging (fp32, rounded once)
#pragma unroll
    for (int n = 0; n < 4; n++) {
        stage_out[wr0 + gid][8 * n + 2 * tig] = (float)acc[n][0];
        stage_out[wr0 + gid][8 * n + 2 * tig + 1] = (float)acc[n][1];
        stage_out[wr0 + gid + 8][8 * n + 2 * tig] = (float)acc[n][2];
        stage_out[wr0 + gid + 8][8 * n + 2 * tig + 1] = (float)acc[n][3];
    }
    cons.sync();
    bgemm_epilogue<MODE>(a, r0, nrows, stage_out, best_s, threadIdx.x, 32 * BG_WARPS, 1);
}


// ---------------------------------------------------------------- fp32 path --
//
// The fp32 batched step (B <= BMAX sequences, or the tokens of a prompt chunk)
// has the same shape with fp32 operands: prep_f32 writes each row's RMSNorm
// (or the embedding row) in fp32, and gemm_f32 multiplies in fp32 on the CUDA
// cores (FFMA: each weight element feeds B multiply-adds, so at B = 32 the
// GEMM is bound by the FMA pipes rather than by HBM), with the epilogues above.
// The attention output and hb feed their GEMMs directly (no norm).

constexpr int BF_ROWS = 32;               // weight rows per CTA
constexpr int BF_KT = 64;                 // K per stage
constexpr int BF_PITCH = BF_KT + 4;       // floats per shared row: conflict-free 16-byte reads
constexpr int BF_STAGES = 4;               // 70 KB: three CTAs per SM (measured best of 2..8)
constexpr int BF_THREADS = 64;
constexpr int BF_STAGE_FLOATS = (BF_ROWS + BMAX) * BF_PITCH;
constexpr int BF_SMEM = BF_STAGES * BF_STAGE_FLOATS * 4;

struct BPrepF32Args {
    const float* in;        // [B][in_stride] (x)
    size_t in_stride;
    const float* norm_w;    // RMSNorm gain
    const float* emb;       // layer 0: fp32 embedding table [vocab][K], else nullptr
    float* x_resid;         // layer 0: receives the embedding rows [B][K]
    float* out;             // [B][out_stride] normalized rows
    size_t out_stride;
    int K;
    const int* tp;
    int vocab;
    unsigned long long* amax;  // reset per sequence on layer 0
    int* err;
};

// CTA (b, y) of a (B, Y) grid: sequence b's row (the embedding row on layer
// 0), its RMSNorm sum over the whole row in every CTA of the sequence, then
// w * (inv * x) in double, rounded once, for the y-th of Y equal ranges.
__global__ void __launch_bounds__(256) k_bprep_f32(const BPrepF32Args a) {
    extern __shared__ float bpf_x[];
    __shared__ double red[32];
    const int b = blockIdx.x;
    const int K = a.K;
    const int i0 = (int)((long long)K * blockIdx.y / gridDim.y);
    const int i1 = (int)((long long)K * (blockIdx.y + 1) / gridDim.y);
    grid_dep_wait();
    grid_dep_launch();
    const float* in = a.in + (size_t)b * a.in_stride;
    if (a.emb) {
        int token = a.tp[2 * b];
        if (token < 0 || token >= a.vocab) {
            if (threadIdx.x == 0) set_error(a.err, DERR_TOKEN);
            token = 0;
        }
        in = a.emb + (size_t)token * K;
        if (a.amax && threadIdx.x == 0 && blockIdx.y == 0) a.amax[b] = 0ull;
    }
    for (int i = threadIdx.x; i < K; i += blockDim.x) {
        const float v = in[i];
        bpf_x[i] = v;
        if (a.emb && i >= i0 && i < i1) a.x_resid[(size_t)b * K + i] = v;
    }
    __syncthreads();
    double ss = 0.0;
    for (int i = threadIdx.x; i < K; i += blockDim.x) ss += (double)bpf_x[i] * (double)bpf_x[i];
    ss = block_sum(ss, red);
    const double inv = 1.0 / sqrt(ss / (double)K + 1e-5);
    float* out = a.out + (size_t)b * a.out_stride;
    for (int i = i0 + (int)threadIdx.x; i < i1; i += blockDim.x)
        out[i] = (float)((double)a.norm_w[i] * (inv * (double)bpf_x[i]));
}

// 16-byte global -> shared asynchronous copy; with on == false nothing is
// read and the destination is zero-filled.
__device__ __forceinline__ void bf_cp16(float* dst, const float* src, bool on, uint64_t pol) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;"
                 :: "r"(smem_u32(dst)), "l"(src), "r"(on ? 16 : 0), "l"(pol) : "memory");
}

// grid = ceil(rows / BF_ROWS) CTAs of BF_THREADS threads, BF_SMEM bytes of
// dynamic shared memory.  CTA i computes rows i*BF_ROWS .. +BF_ROWS-1 for
// every sequence: Y[b][r] = sum_k W[r][k] X[b][k] in fp32 FMAs.  Stages of
// BF_KT columns of W (this CTA's rows) and of X (all BMAX rows; rows >= B and
// columns >= K are zero-filled) stream through a BF_STAGES-deep cp.async
// ring.  Thread t computes rows t/8 + {0, 8, 16, 24} for sequences
// t%8 + {0, 8, 16, 24} in k order, reading 4 consecutive k of each at once
// (16-byte shared loads: a 4 x 4 tile does 64 FMAs per 8 loads, against 32
// per 6 for 2 x 4; the shared-memory pipe, four wavefronts per 16-byte warp
// load, is the limit).  a.W holds the fp32 rows (a.rb bytes apart); X is
// [B][x_stride].
template <int MODE>
__global__ void __launch_bounds__(BF_THREADS) k_bgemm_f32(const BGemmArgs a, const float* X, size_t x_stride) {
    extern __shared__ __align__(16) float fsm[];
    __shared__ float stage_out[BF_ROWS][BMAX + 1];
    __shared__ unsigned long long best_s[BMAX];
    const int tid = threadIdx.x;
    const int r0 = blockIdx.x * BF_ROWS;
    const int nrows = min(BF_ROWS, a.rows - r0);
    const int K = a.K;
    const int nkt = (K + BF_KT - 1) / BF_KT;
    const float* W = reinterpret_cast<const float*>(a.W) + (size_t)r0 * (a.rb / 4);
    const size_t ldw = a.rb / 4;
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_x = policy_evict_last();
    if (tid < BMAX) best_s[tid] = 0ull;
    if (tid == 0 && a.prefetch_bytes) {  // weights do not depend on earlier kernels
        size_t bytes = (size_t)nrows * a.rb;
        if (bytes > a.prefetch_bytes) bytes = a.prefetch_bytes;
        prefetch_l2_range(W, bytes & ~size_t(15), policy_evict_last());
    }
    grid_dep_wait();
    grid_dep_launch();
    auto load = [&](int t) {
        float* st = fsm + (size_t)(t % BF_STAGES) * BF_STAGE_FLOATS;
        const int k0 = t * BF_KT;
#pragma unroll
        for (int j = 0; j < (BF_ROWS * BF_KT / 4) / BF_THREADS; j++) {
            const int idx = tid + j * BF_THREADS;
            const int r = idx / (BF_KT / 4), c4 = idx % (BF_KT / 4);
            const int k = k0 + 4 * c4;
            const bool on = r < nrows && k < K;
            bf_cp16(st + r * BF_PITCH + 4 * c4, on ? W + (size_t)r * ldw + k : W, on, pol_w);
        }
#pragma unroll
        for (int j = 0; j < (BMAX * BF_KT / 4) / BF_THREADS; j++) {
            const int idx = tid + j * BF_THREADS;
            const int b = idx / (BF_KT / 4), c4 = idx % (BF_KT / 4);
            const int k = k0 + 4 * c4;
            const bool on = b < a.B && k < K;
            bf_cp16(st + (BF_ROWS + b) * BF_PITCH + 4 * c4, on ? X + (size_t)b * x_stride + k : X, on, pol_x);
        }
    };
#pragma unroll
    for (int t = 0; t < BF_STAGES - 1; t++) {
        if (t < nkt) load(t);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    const int sg = tid & 7, rp = tid >> 3;  // rows rp + 8i, sequences sg + 8j
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; i++) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    for (int t = 0; t < nkt; t++) {
        asm volatile("cp.async.wait_group %0;" :: "n"(BF_STAGES - 2) : "memory");
        __syncthreads();  // stage t landed for every thread; stage t-1 is free
        if (t + BF_STAGES - 1 < nkt) load(t + BF_STAGES - 1);
        asm volatile("cp.async.commit_group;" ::: "memory");
        const float* wt = fsm + (size_t)(t % BF_STAGES) * BF_STAGE_FLOATS;
        const float* xt = wt + BF_ROWS * BF_PITCH;
        // the stage's 16 steps of 4 columns, fully unrolled so that the shared
        // loads of later steps issue ahead of the FMAs of earlier ones
        const float* wr = wt + rp * BF_PITCH;
        const float* xr = xt + sg * BF_PITCH;
#pragma unroll
        for (int kk = 0; kk < BF_KT; kk += 4) {
            float4 wv[4], xv[4];
#pragma unroll
            for (int i = 0; i < 4; i++) wv[i] = *reinterpret_cast<const float4*>(wr + 8 * i * BF_PITCH + kk);
#pragma unroll
            for (int j = 0; j < 4; j++) xv[j] = *reinterpret_cast<const float4*>(xr + 8 * j * BF_PITCH + kk);
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    acc[i][j] = fmaf(wv[i].x, xv[j].x, acc[i][j]);
                    acc[i][j] = fmaf(wv[i].y, xv[j].y, acc[i][j]);
                    acc[i][j] = fmaf(wv[i].z, xv[j].z, acc[i][j]);
                    acc[i][j] = fmaf(wv[i].w, xv[j].w, acc[i][j]);
                }
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) stage_out[rp + 8 * i][sg + 8 * j] = acc[i][j];
    __syncthreads();
    bgemm_epilogue<MODE>(a, r0, nrows, stage_out, best_s, tid, BF_THREADS, 1);
}

}  // namespace l2c
