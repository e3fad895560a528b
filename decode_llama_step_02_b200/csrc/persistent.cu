// persistent.cu - the single-sequence Q8_0 decode step as one persistent
// kernel (sm_100a).
//
// The step is the same computation as the per-layer kernel sequence in
// kernels.cuh (llama2.c's forward(): embedding; per layer RMSNorm, q/k/v,
// RoPE, cache write, attention, wo + residual, RMSNorm, SwiGLU FFN +
// residual; final RMSNorm, classifier, argmax), with the same arithmetic and
// rounding points, but it runs as ONE launch of one CTA per SM:
//
//   * warps 8.. (the producers) stream, in order, every weight row unit this
//     CTA will use during the whole step -- its share of QKV, Wo, W13 and W2
//     of every layer, then of the classifier -- into a byte ring in shared
//     memory with 1-D bulk copies (TMA, no multicast), one mbarrier pair (full
//     / empty) per unit in flight; unit n goes to producer n % PS_PRODUCERS,
//     which owns a slice of the ring.  Weights do not depend on activations, so the
//     stream never waits for the computation except for ring space: while the
//     consumers sit at a grid barrier or quantize the next input, the next
//     matrix is already landing.
//   * warps 0..7 (the consumers) run the phases: quantize the phase input
//     (the same prologue as the GEMV kernels), then take the CTA's units
//     round-robin (unit n -> warp n mod 8), reduce each with dp4a into exact
//     int32 group sums scaled in double, release the ring space, and apply the
//     epilogue (RoPE + cache write, residual add, SwiGLU, logits + argmax).
//     Between phases a grid barrier makes the phase's outputs visible; after
//     QKV the consumers run the layer's attention as 2 x 148 four-warp work
//     items (the flash-decode items of attention.cuh).
//
// Grid barrier: an arrival counter that only grows during the launch (barrier
// i waits for i * gridDim.x arrivals); the last CTA to finish zeroes it.
// Every wait in the kernel (ring barriers, grid barrier) gives up after 2 s:
// it records DERR_TIMEOUT, raises abort_flag (which ends every other wait at
// once), lets the copies already issued land, and returns.  Activations
// written by other CTAs of the same launch are read with ld.global.cg.
#include "kernels.cuh"
#include "persistent.h"

// Development builds that define L2C_PSTEP_STAMPS record, per CTA and weight
// phase, global-timer stamps of the phase's milestones (barrier entry and
// exit, prologue end, unit loop end, attention end, the producer's first and
// last copy of the phase); l2c_dbg_pstamps copies them to the host.
#ifdef L2C_PSTEP_STAMPS
constexpr int PST_CTAS = 160, PST_PHASES = 132, PST_SLOTS = 12;
__device__ unsigned long long g_pstamps[PST_CTAS * PST_PHASES * PST_SLOTS];
#define PSTAMP(wp, k)                                                                               \
    do {                                                                                            \
        if (blockIdx.x < PST_CTAS && (wp) < PST_PHASES)                                             \
            g_pstamps[(blockIdx.x * PST_PHASES + (wp)) * PST_SLOTS + (k)] = global_timer_ns();     \
    } while (0)
#define PSTAMP_ADD(wp, k, v)                                                                        \
    do {                                                                                            \
        if (blockIdx.x < PST_CTAS && (wp) < PST_PHASES)                                             \
            atomicAdd(&g_pstamps[(blockIdx.x * PST_PHASES + (wp)) * PST_SLOTS + (k)], (unsigned long long)(v)); \
    } while (0)
#define PS_T0() const uint64_t pst_t0_ = global_timer_ns()
#define PS_DT() (global_timer_ns() - pst_t0_)
#else
#define PSTAMP_ADD(wp, k, v) \
    do {                     \
    } while (0)
#define PS_T0() \
    do {        \
    } while (0)
#define PS_DT() 0
#define PSTAMP(wp, k) \
    do {              \
    } while (0)
#endif

namespace l2c {

namespace {

constexpr uint64_t PS_WAIT_NS = 2000000000ull;

struct PPhase {
    const uint8_t* W;  // first record of the phase's matrix
    size_t rb;         // record bytes
    int rows, K, unit, mode;
};

// Weight phase wp of the step: 4 per layer (QKV, Wo, W13, W2), then the
// classifier.  A unit is PS_UNIT rows of width dim where the row count allows
// (else 2 or 1; QKV and W13 units are whole row pairs), one row of W2.
__device__ __forceinline__ int punit(int rows, int pair) {
    return rows % PS_UNIT == 0 ? PS_UNIT : (pair || rows % 2 == 0 ? 2 : 1);
}

__device__ __forceinline__ PPhase pphase(const PStepArgs& s, int wp) {
    PPhase p;
    if (wp == 4 * s.L) {
        p.W = s.Wcls; p.rb = s.rb_d; p.rows = s.V; p.K = s.d; p.unit = punit(s.V, 0); p.mode = M_CLS;
        return p;
    }
    const size_t l = (size_t)(wp >> 2), d = (size_t)s.d, h = (size_t)s.hdim, kvd = (size_t)s.kvd;
    switch (wp & 3) {
    case 0:
        p.rows = (int)(d + 2 * kvd); p.W = s.Wqkv + l * p.rows * s.rb_d; p.rb = s.rb_d;
        p.K = s.d; p.unit = punit(p.rows, 1); p.mode = M_QKV;
        break;
    case 1:
        p.rows = s.d; p.W = s.Wo + l * d * s.rb_d; p.rb = s.rb_d; p.K = s.d; p.unit = punit(s.d, 0); p.mode = M_RESID;
        break;
    case 2:
        p.rows = (int)(2 * h); p.W = s.W13 + l * 2 * h * s.rb_d; p.rb = s.rb_d;
        p.K = s.d; p.unit = punit(p.rows, 1); p.mode = M_W13;
        break;
    default:
        p.rows = s.d; p.W = s.W2 + l * d * s.rb_h; p.rb = s.rb_h; p.K = s.hdim; p.unit = 1; p.mode = M_RESID;
        break;
    }
    return p;
}

// This CTA's contiguous share [u0, u1) of `units`.
__device__ __forceinline__ void cta_range(int units, int& u0, int& u1) {
    u0 = (int)((long long)units * blockIdx.x / gridDim.x);
    u1 = (int)((long long)units * (blockIdx.x + 1) / gridDim.x);
}

__device__ __forceinline__ bool aborted(const PStepArgs& s) { return *(volatile const int*)s.abort_flag != 0; }

__device__ __forceinline__ void raise_abort(const PStepArgs& s) { atomicExch(s.abort_flag, 1); }

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid barrier number `idx` (1, 2, ...) of the launch, for the consumer
// threads of every CTA: each CTA adds 1 to a counter that only grows during
// the launch, then waits for idx * gridDim.x arrivals.  Returns false on every
// consumer thread of the CTA when the step is being abandoned.
__device__ bool grid_barrier(const PStepArgs& s, const SyncNamed& sy, int* flag, unsigned idx) {
    sy.sync();
    if (threadIdx.x == 0) {
        bool ok = !aborted(s);
        if (ok) {
            const unsigned target = idx * gridDim.x;
            __threadfence();  // the CTA's writes (ordered by the named barrier) before the arrival
            atomicAdd(s.bar, 1u);
            if (ld_relaxed_u32(s.bar) < target) {
                const uint64_t t0 = global_timer_ns();
                while (ld_relaxed_u32(s.bar) < target) {
                    if (aborted(s)) { ok = false; break; }
                    if (global_timer_ns() - t0 > PS_WAIT_NS) {
                        set_error(s.err, DERR_TIMEOUT);
                        raise_abort(s);
                        ok = false;
                        break;
                    }
                }
            }
            __threadfence();
        }
        *flag = ok ? 1 : 0;
    }
    sy.sync();
    return *flag != 0;
}

// End of the launch: the last CTA to get here zeroes the barrier counter for
// the next launch (every CTA has passed every barrier by then).
__device__ __forceinline__ void grid_barrier_retire(const PStepArgs& s) {
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(s.bar + 1, 1u) == gridDim.x - 1) {
            atomicExch(s.bar, 0u);
            atomicExch(s.bar + 1, 0u);
        }
    }
}

// Walks the units of one producer through the step: phase by phase, the
// units u of this CTA's share whose position in the CTA's sequence is
// congruent to pr modulo PS_PRODUCERS.
struct UnitCursor {
    int wp, u, u1, n;  // phase, unit, end of the phase's share, sequence position of u0
    PPhase ph;
    __device__ __forceinline__ void enter(const PStepArgs& s, int pr) {
        for (; wp <= 4 * s.L; wp++) {
            ph = pphase(s, wp);
            int u0;
            cta_range(ph.rows / ph.unit, u0, u1);
            u = u0 + ((pr - n) % PS_PRODUCERS + PS_PRODUCERS) % PS_PRODUCERS;
            n += u1 - u0;
            if (u < u1) return;
        }
    }
    __device__ __forceinline__ void start(const PStepArgs& s, int pr) {
        wp = 0;
        n = 0;
        enter(s, pr);
    }
    __device__ __forceinline__ bool done(const PStepArgs& s) const { return wp > 4 * s.L; }
    __device__ __forceinline__ uint32_t bytes() const { return (uint32_t)(ph.unit * ph.rb); }
    __device__ __forceinline__ const uint8_t* src() const { return ph.W + (size_t)u * ph.unit * ph.rb; }
    __device__ __forceinline__ void next(const PStepArgs& s, int pr) {
        u += PS_PRODUCERS;
        if (u >= u1) {
            wp++;
            enter(s, pr);
        }
    }
};

// Producer `pr`: lane 0 of warp PS_CONSUMERS + pr.  It issues the units n of
// the CTA's step sequence with n % PS_PRODUCERS == pr, in order, into its own
// slice of the ring (R bytes) with its own PS_PSLOTS barrier slots.  Units
// sit at increasing virtual byte positions (a unit never wraps: it skips to
// the next multiple of R instead); a unit may be issued once the slice holds
// no unreleased unit that its bytes would overwrite and fewer than PS_PSLOTS
// units are in flight.  Releases are awaited in issue order.  A second cursor
// runs up to s.pf_bytes ahead of the copies with L2 prefetches (evict-last),
// so HBM keeps streaming while the ring is full and the consumers are at a
// grid barrier or in a prologue; the copies then read L2.
__device__ void pstep_produce(const PStepArgs& s, int pr, uint8_t* ring, uint32_t R, uint32_t* meta,
                              unsigned long long* vstart, uint64_t* full, uint64_t* empty) {
    const uint64_t pol = policy_evict_first();
    const uint64_t pol_keep = policy_evict_last();
    const unsigned long long pf_limit = s.pf_bytes / PS_PRODUCERS;
    unsigned long long vhead = 0;  // virtual position of the next free byte
    uint32_t ohead = 0;            // vhead % R
    int m = 0, mrel = 0;           // this producer's units issued / known released
    unsigned long long copied = 0, fetched = 0;  // bytes copied to the ring / prefetched to L2
    UnitCursor c, f;
    c.start(s, pr);
    f.start(s, pr);
    bool ok = true;
    while (!c.done(s)) {
        [[maybe_unused]] const int wp = c.wp;
        // keep the L2 prefetch cursor up to pf_limit bytes ahead of the copies
        while (!f.done(s) && fetched < copied + pf_limit) {
            prefetch_l2_bulk(f.src(), f.bytes(), pol_keep);
            fetched += f.bytes();
            f.next(s, pr);
        }
        const uint32_t bytes = c.bytes();
        unsigned long long p = vhead;
        uint32_t off = ohead;
        if (off + bytes > R) {
            p += R - off;
            off = 0;
        }
        while (mrel < m && (m - mrel >= PS_PSLOTS || p + bytes - vstart[mrel % PS_PSLOTS] > R)) {
            PS_T0();
            if (!mbar_wait_bounded(&empty[mrel % PS_PSLOTS], (mrel / PS_PSLOTS) & 1, s.err, PS_WAIT_NS)) {
                ok = false;
                break;
            }
            PSTAMP_ADD(wp, 9, PS_DT());
            PSTAMP_ADD(wp, 10, 1);
            mrel++;
        }
        // the flag is a global load: look at it once every 64 units only
        if (!ok || ((m & 63) == 0 && aborted(s))) {
            ok = false;
            break;
        }
        // the consumers' reads of this space are ordered before the copy by
        // the empty barrier (arrive after the reads, wait before the copy)
        const int slot = m % PS_PSLOTS;
        vstart[slot] = p;
        meta[slot] = off;
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s(ring + off, c.src(), bytes, &full[slot], pol);
        vhead = p + bytes;
        ohead = off + bytes == R ? 0u : off + bytes;
        copied += bytes;
        m++;
        c.next(s, pr);
    }
    if (!ok) {
        raise_abort(s);
        // let every copy already issued land before the CTA can leave
        for (int j = mrel; j < m; j++) mbar_wait_bounded(&full[j % PS_PSLOTS], (j / PS_PSLOTS) & 1, s.err, PS_WAIT_NS);
    }
}

// Input codes of a phase, behind the phase's grid barrier: the activations
// (or, on layer 0, the embedding row) and the RMSNorm gain are loaded in one
// round trip into the registers of the split prologue (the batched loop when
// they do not fit).  Ends with the scales also in double (sxd).  Returns
// false when the step is being abandoned.
template <int EPL, bool NORM>
__device__ __forceinline__ bool p_prologue(const GemvArgs& a, const int8_t* eq, const float* es, unsigned bar_idx,
                                           const PStepArgs& s, const SyncNamed& sy, int* flag, int8_t* xq,
                                           float* xsc, double* sxd, double* red, int wp) {
    constexpr int GM = Q8PreGM<EPL, NORM>::value;
    // the register prologue loops over all GM slots: without RMSNorm (GM large)
    // it pays only when most of them are used
    const int per_warp = (a.K / (32 * EPL) + PS_CONSUMERS - 1) / PS_CONSUMERS;
    if (q8_pre_fits<EPL, GM>(a, PS_CONSUMERS) && (NORM || 2 * per_warp > GM)) {
        // (the gain is not held across the barrier: that costs spills)
        if (bar_idx && !grid_barrier(s, sy, flag, bar_idx)) return false;
        if (threadIdx.x == 0) PSTAMP(wp, 1);
        Q8Pre<EPL, GM, NORM> pre;
        if (NORM) q8_pre_load<EPL, GM, NORM>(a, nullptr, nullptr, nullptr, true, pre, PS_CONSUMERS);
        if (eq) q8_pre_load<EPL, GM, NORM>(a, nullptr, eq, es, false, pre, PS_CONSUMERS);
        if (!eq) q8_pre_load<EPL, GM, NORM>(a, a.in, nullptr, nullptr, false, pre, PS_CONSUMERS);
        q8_pre_finish<EPL, GM, NORM>(a, pre, xq, xsc, red, [] {}, sy);
    } else {
        if (bar_idx && !grid_barrier(s, sy, flag, bar_idx)) return false;
        if (threadIdx.x == 0) PSTAMP(wp, 1);
        q8_quantize_input<NORM>(a, eq, es, xq, xsc, red, sy);
    }
    sy.sync();
    for (int g = threadIdx.x; g < a.K / a.gs; g += sy.n) sxd[g] = (double)xsc[g];
    sy.sync();
    return true;
}

template <bool NORM>
__device__ __forceinline__ bool p_prologue_gs(const GemvArgs& a, const int8_t* eq, const float* es, unsigned bar_idx,
                                              const PStepArgs& s, const SyncNamed& sy, int* flag, int8_t* xq,
                                              float* xsc, double* sxd, double* red, int wp) {
    if (a.gs == 32) return p_prologue<1, NORM>(a, eq, es, bar_idx, s, sy, flag, xq, xsc, sxd, red, wp);
    if (a.gs == 64) return p_prologue<2, NORM>(a, eq, es, bar_idx, s, sy, flag, xq, xsc, sxd, red, wp);
    return p_prologue<4, NORM>(a, eq, es, bar_idx, s, sy, flag, xq, xsc, sxd, red, wp);
}

template <int UNIT>
__device__ __forceinline__ void pdot(const uint8_t* base, size_t rb, const int8_t* xq, const double* sxd, int K, int gs,
                                     double (&acc)[UNIT]) {
    if (gs == 32) q8_rows_dot64<32, UNIT>(base, rb, xq, sxd, K, acc);
    else if (gs == 64) q8_rows_dot64<64, UNIT>(base, rb, xq, sxd, K, acc);
    else q8_rows_dot64<128, UNIT>(base, rb, xq, sxd, K, acc);
}

template <int HS, int REP>
__global__ void __launch_bounds__(PS_THREADS, 1) k_step_q8(const PStepArgs s, const PLayout P) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ double red[PS_CONSUMERS];
    __shared__ unsigned long long best_s[PS_CONSUMERS];
    __shared__ double2 rope_cs[HS / 2];
    __shared__ int flag_s;
    uint8_t* ring = smem + P.ring;
    int8_t* xq = reinterpret_cast<int8_t*>(smem + P.xq);
    float* xsc = reinterpret_cast<float*>(smem + P.xsc);
    double* sxd = reinterpret_cast<double*>(smem + P.sxd);
    uint32_t* meta = reinterpret_cast<uint32_t*>(smem + P.meta);
    unsigned long long* vstart = reinterpret_cast<unsigned long long*>(smem + P.vstart);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + P.full);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + P.empty);
    AttnSmem<double, HS, REP>* asm2 = reinterpret_cast<AttnSmem<double, HS, REP>*>(smem + P.attn);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < PS_SLOTS; i++) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_fence_init();
    }
    // token and position (written before the launch), checked and clamped
    GemvArgs base = {};
    base.tp = s.tp; base.err = s.err; base.vocab = s.V; base.seq_len = s.S;
    base.d = s.d; base.kvd = s.kvd; base.hs = s.hs; base.gs = s.gs; base.freq = s.freq; base.amax = s.amax;
    int token = 0, pos = 0;
    read_tp(base, token, pos);
    rope_table(base, pos, rope_cs);  // one (cos, sin) pair per pair index, for every layer
    if (blockIdx.x == 0 && threadIdx.x == 0) *s.amax = 0ull;
    __syncthreads();

    const uint32_t Rp = (s.ring_bytes / PS_PRODUCERS) & ~127u;  // ring slice of one producer
    if (warp >= PS_CONSUMERS) {
        const int pr = warp - PS_CONSUMERS;
        if (lane == 0)
            pstep_produce(s, pr, ring + (size_t)pr * Rp, Rp, meta + pr * PS_PSLOTS, vstart + pr * PS_PSLOTS,
                          full + pr * PS_PSLOTS, empty + pr * PS_PSLOTS);
        return;
    }

    // ---- consumers
    const SyncNamed sy{1, 32 * PS_CONSUMERS};
    const int nwp = 4 * s.L + 1;
    const size_t d = (size_t)s.d, cache_layer = (size_t)s.S * s.kvd;
    int nbase = 0;
    unsigned nbar = 0;  // grid barriers passed
    bool dead = false;  // this warp gave up on a ring wait: it skips work until the next grid barrier
    for (int wp = 0; wp < nwp; wp++) {
        const PPhase ph = pphase(s, wp);
        const int l = wp >> 2;
        int u0, u1;
        cta_range(ph.rows / ph.unit, u0, u1);
        const int cnt = u1 - u0;
        GemvArgs a = base;
        a.rows = ph.rows; a.K = ph.K; a.ld = ph.rb;
        const int8_t* eq = nullptr;
        const float* es = nullptr;
        if (ph.mode == M_QKV) {
            a.in = s.x; a.norm_w = s.rms_att + l * d; a.out = s.q;
            a.kslot = s.kc + l * cache_layer; a.vslot = s.vc + l * cache_layer;
            if (l == 0) {
                a.emb = s.E; a.x_resid = s.x;
                eq = reinterpret_cast<const int8_t*>(s.E + (size_t)token * s.rb_d);
                es = reinterpret_cast<const float*>(s.E + (size_t)token * s.rb_d + s.d);
            }
        } else if (ph.mode == M_W13) {
            a.in = s.x; a.norm_w = s.rms_ffn + l * d; a.out = s.hb;
        } else if (ph.mode == M_CLS) {
            a.in = s.x; a.norm_w = s.rms_final; a.out = s.logits;
        } else {
            a.in = (wp & 3) == 1 ? s.att : s.hb; a.out = s.x;
        }
        if (threadIdx.x == 0) PSTAMP(wp, 0);
        // this phase's input codes (behind the phase's grid barrier, except on the first)
        const unsigned bidx = wp > 0 ? ++nbar : 0u;
        const bool ok = a.norm_w ? p_prologue_gs<true>(a, eq, es, bidx, s, sy, &flag_s, xq, xsc, sxd, red, wp)
                                 : p_prologue_gs<false>(a, eq, es, bidx, s, sy, &flag_s, xq, xsc, sxd, red, wp);
        if (!ok) return;
        dead = false;
        if (threadIdx.x == 0) PSTAMP(wp, 2);
        // residual phases: lane k * unit + r fetches now the current x of row r of
        // this warp's k-th unit
        float xres = 0.f;
        if (ph.mode == M_RESID) {
            const int k = lane / ph.unit, j = warp + PS_CONSUMERS * k;
            if (j < cnt) xres = __ldcg(a.out + (size_t)(u0 + j) * ph.unit + lane % ph.unit);
        }

        unsigned long long best = 0ull;
        for (int n = nbase + warp; n < nbase + cnt; n += PS_CONSUMERS) {
            const int pr = n % PS_PRODUCERS, m = n / PS_PRODUCERS;  // its producer, and its index there
            const int slot = pr * PS_PSLOTS + m % PS_PSLOTS;
            if (dead) continue;
            PS_T0();
            if (!mbar_wait_bounded(&full[slot], (m / PS_PSLOTS) & 1, s.err, PS_WAIT_NS)) {
                raise_abort(s);
                dead = true;
                continue;
            }
            if (lane == 0 && warp == 0) PSTAMP_ADD(wp, 8, PS_DT());
            const uint8_t* rec = ring + (size_t)pr * Rp + meta[slot];
            const int u = u0 + (n - nbase);
            // row totals: lane l holds the total of row l / stride of the unit
            const int stride = 32 / ph.unit;
            double tot;
            if (ph.unit == PS_UNIT) {
                double acc[PS_UNIT];
                pdot<PS_UNIT>(rec, ph.rb, xq, sxd, a.K, a.gs, acc);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);  // the unit's bytes are no longer read
                tot = warp_sum_scatter<PS_UNIT>(acc);
            } else if (ph.unit == 2) {
                double acc[2];
                pdot<2>(rec, ph.rb, xq, sxd, a.K, a.gs, acc);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
                tot = warp_sum_scatter<2>(acc);
            } else {
                double acc[1];
                pdot<1>(rec, ph.rb, xq, sxd, a.K, a.gs, acc);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
                tot = warp_sum_scatter<1>(acc);
            }
            const int r = lane / stride;            // the row this lane's total belongs to
            const bool owner = lane % stride == 0;  // one lane per row writes it
            const int row = u * ph.unit + r;
            if (ph.mode == M_QKV || ph.mode == M_W13) {
                const double odd = __shfl_down_sync(0xffffffffu, tot, stride);  // the pair's second row
                if (owner && (r & 1) == 0) {
                    if (ph.mode == M_QKV) epi_qkv(a, row >> 1, (float)tot, (float)odd, pos, rope_cs);
                    else epi_w13(a, row >> 1, (float)tot, (float)odd);
                }
            } else if (ph.mode == M_RESID) {
                // x of this row, fetched before the loop by lane k * unit + r
                const int k = (n - nbase) / PS_CONSUMERS;  // this warp's k-th unit
                const int src = k * ph.unit + r;
                float xo = __shfl_sync(0xffffffffu, xres, src & 31);
                if (owner) {
                    if (src >= 32) xo = __ldcg(a.out + row);
                    a.out[row] = xo + (float)tot;
                }
            } else if (owner) {
                const float v = (float)tot;
                a.out[row] = v;
                if (v != v) set_error(s.err, DERR_NAN);
                const unsigned long long key = argmax_key(v, row);
                best = key > best ? key : best;
            }
        }
        nbase += cnt;
        if (threadIdx.x == 0) PSTAMP(wp, 3);
        if (threadIdx.x == 32 * (PS_CONSUMERS - 1)) PSTAMP(wp, 5);

        if (ph.mode == M_CLS) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const unsigned long long b = __shfl_xor_sync(0xffffffffu, best, o);
                best = b > best ? b : best;
            }
            if (lane == 0) best_s[warp] = best;
            sy.sync();
            if (threadIdx.x == 0) {
                unsigned long long b = 0ull;
                for (int i = 0; i < PS_CONSUMERS; i++) b = best_s[i] > b ? best_s[i] : b;
                if (b) atomicMax(s.amax, b);
            }
        } else if (ph.mode == M_QKV) {
            // the layer's attention over positions 0..pos, two work items per CTA at a time
            if (!grid_barrier(s, sy, &flag_s, ++nbar)) return;
            dead = false;
            AttnArgs t;
            t.q = s.q; t.kc = s.kc + l * cache_layer; t.vc = s.vc + l * cache_layer; t.seq_stride = 0;
            t.out = s.att; t.tp = s.tp; t.tp_stride = 2;
            t.H = s.H; t.Hkv = s.Hkv; t.hs = s.hs; t.kvd = s.kvd; t.seq_len = s.S;
            t.nchunks = s.nchunks; t.part = s.part; t.count = s.count; t.err = s.err;
            // about one chunk per 32 positions, at most s.nchunks (a single chunk
            // writes its output directly, with no partials to merge)
            const int nch = min(s.nchunks, (pos + 32) / 32);
            t.nchunks = nch;
            const int half = warp >> 2;
            const SyncNamed hsy{2 + half, 128};
            const int items = nch * s.Hkv;
            for (int it = (int)blockIdx.x * 2 + half; it < items; it += 2 * (int)gridDim.x)
                attn_item<double, HS, REP, SyncNamed, false, true>(t, it % nch, it / nch, 0, threadIdx.x & 127,
                                                                   hsy, asm2[half]);
            if (threadIdx.x == 0) PSTAMP(wp, 4);
        }
    }
    grid_barrier_retire(s);
}

template <int HS, int REP>
constexpr size_t attn_pair_bytes() {
    return 2 * ((sizeof(AttnSmem<double, HS, REP>) + 15) & ~size_t(15));
}

#define L2C_PSTEP_CONFIGS(X) \
    X(8, 1) X(16, 1) X(16, 2) X(32, 1) X(32, 2) X(32, 4) X(48, 1) X(48, 2) \
    X(64, 1) X(64, 2) X(64, 4) X(64, 8) X(128, 1) X(128, 2) X(128, 4) X(128, 8)

}  // namespace

const void* pstep_kernel(int hs, int rep) {
#define L2C_PK(HS_, REP_) \
    if (hs == HS_ && rep == REP_) return reinterpret_cast<const void*>(&k_step_q8<HS_, REP_>);
    L2C_PSTEP_CONFIGS(L2C_PK)
#undef L2C_PK
    return nullptr;
}

static size_t attn_bytes_for(int hs, int rep) {
#define L2C_PA(HS_, REP_) \
    if (hs == HS_ && rep == REP_) return attn_pair_bytes<HS_, REP_>();
    L2C_PSTEP_CONFIGS(L2C_PA)
#undef L2C_PA
    return 0;
}

PLayout pstep_layout(uint32_t ring_bytes, int kmax, int gs, int hs, int rep) {
    auto up16 = [](size_t v) { return (v + 15) & ~size_t(15); };
    PLayout L = {};
    size_t o = 0;
    L.ring = (uint32_t)o; o = up16(o + ring_bytes);
    L.xq = (uint32_t)o; o = up16(o + (size_t)kmax);
    L.xsc = (uint32_t)o; o = up16(o + (size_t)(kmax / gs) * 4);
    L.sxd = (uint32_t)o; o = up16(o + (size_t)(kmax / gs) * 8);
    L.meta = (uint32_t)o; o = up16(o + PS_SLOTS * 4);
    L.vstart = (uint32_t)o; o = up16(o + PS_SLOTS * 8);
    L.full = (uint32_t)o; o = up16(o + PS_SLOTS * 8);
    L.empty = (uint32_t)o; o = up16(o + PS_SLOTS * 8);
    L.attn = (uint32_t)o; o = up16(o + attn_bytes_for(hs, rep));
    L.total = (uint32_t)o;
    return L;
}

cudaError_t pstep_static_smem(const void* kern, size_t* bytes) {
    cudaFuncAttributes at;
    cudaError_t e = cudaFuncGetAttributes(&at, kern);
    if (e == cudaSuccess) *bytes = at.sharedSizeBytes;
    return e;
}

#ifdef L2C_PSTEP_STAMPS
extern "C" __attribute__((visibility("default"))) int l2c_dbg_pstamps(void* host) {
    return (int)cudaMemcpyFromSymbol(host, g_pstamps, sizeof(g_pstamps));
}
extern "C" __attribute__((visibility("default"))) int l2c_dbg_pzero() {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_pstamps);
    if (e == cudaSuccess) e = cudaMemset(p, 0, sizeof(g_pstamps));
    return (int)e;
}
#endif

cudaError_t pstep_launch(const void* kern, int grid, const PStepArgs& a, const PLayout& L, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(PS_THREADS);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    PStepArgs av = a;
    PLayout lv = L;
    void* args[] = {&av, &lv};
    return cudaLaunchKernelExC(&cfg, kern, args);
}

}  // namespace l2c
