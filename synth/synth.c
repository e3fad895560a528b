/*
 * synth.c - seeded synthetic inputs for the Llama-2 decode step.
 *
 * This module produces the numbers that both the CPU oracle's tests and the
 * GPU harness feed to their implementations: model weights, prefilled KV
 * caches, token ids and positions.  It holds none of the decode step's
 * arithmetic; it only knows where each tensor sits in the weight blob so that
 * RMSNorm gains and matrix weights get the right distribution.
 *
 * Generator (counter based, so any element can be produced on its own):
 *   - SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014): the i-th output for key k is
 *     mix(k + (i + 1) * 0x9E3779B97F4A7C15), with Stafford's "Mix13" finaliser.
 *   - A key is derived from (seed, stream, sub) by chaining the same mixer.
 *     Streams: 0 = weight blob, 1 = KV prefill, 2 = token ids, 3 = positions.
 *   - Normal deviates: Box and Muller (1958).  Element i uses the pair of
 *     outputs (2*(i/2), 2*(i/2)+1) turned into u1 in (0,1] and u2 in [0,1)
 *     with 53 random bits each; r = sqrt(-2 ln u1), a = 2*pi*u2, and the even
 *     element takes r*cos(a), the odd one r*sin(a).  Everything is double and
 *     rounded once to float at the end: (float)(mu + sigma*z).
 *   - Uniform integers in [0, n): ((output >> 32) * n) >> 32.
 *
 * Weight blob layout (all fp32, no header; the order llama2.c's checkpoint
 * loader walks - "memory_map_weights" on the karpathy-notes Q&A page):
 *   E[V][d], w_att[L][d], Wq[L][d][d], Wk[L][kvd][d], Wv[L][kvd][d],
 *   Wo[L][d][d], w_ffn[L][d], W1[L][h][d], W2[L][d][h], W3[L][h][d],
 *   w_final[d], legacy freq_cis_real[S*hs/2], freq_cis_imag[S*hs/2] (zeros),
 *   and Wcls[V][d] only when the classifier is not tied to E.
 * Matrix weights and E/Wcls are N(0, wsigma); RMSNorm gains are
 * 1 + N(0, nsigma) (exactly 1 when nsigma == 0); the freq_cis regions are 0.
 * Element e of the blob always draws its z from counter e of stream 0.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t synth_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_key(uint64_t seed, uint32_t stream, uint64_t sub) {
    uint64_t k = synth_mix(seed + SYNTH_GOLDEN);
    k = synth_mix(k ^ ((uint64_t)stream * 0xD1B54A32D192ED03ULL));
    k = synth_mix(k ^ (sub * 0x8CB92BA72F3D8DD7ULL + 1ULL));
    return k;
}

uint64_t synth_u64(uint64_t key, uint64_t i) {
    return synth_mix(key + (i + 1ULL) * SYNTH_GOLDEN);
}

static inline double synth_z(uint64_t key, uint64_t i) {
    uint64_t pair = i >> 1;
    uint64_t a = synth_u64(key, 2 * pair), b = synth_u64(key, 2 * pair + 1);
    double u1 = (double)((a >> 11) + 1ULL) * 0x1.0p-53;  /* (0, 1] */
    double u2 = (double)(b >> 11) * 0x1.0p-53;           /* [0, 1) */
    double r = sqrt(-2.0 * log(u1));
    double ang = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(ang) : r * cos(ang);
}

/* z-values for counters [start, start+n) of `key`, as double. */
void synth_normal_f64(uint64_t key, uint64_t start, uint64_t n, double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)n; j++) out[j] = synth_z(key, start + (uint64_t)j);
}

/* Fills out[j] = (float)(mu + sigma * z(start + j)); pairs share one log and one sincos. */
void synth_normal_f32(uint64_t key, uint64_t start, uint64_t n, double mu, double sigma, float* out) {
    const int64_t CH = 1 << 16;
    int64_t nch = ((int64_t)n + CH - 1) / CH;
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t c = 0; c < nch; c++) {
        uint64_t j0 = (uint64_t)(c * CH), j1 = j0 + (uint64_t)CH;
        if (j1 > n) j1 = n;
        uint64_t j = j0;
        while (j < j1) {
            uint64_t i = start + j;
            if ((i & 1) == 0 && j + 1 < j1) {
                uint64_t pair = i >> 1;
                uint64_t a = synth_u64(key, 2 * pair), b = synth_u64(key, 2 * pair + 1);
                double u1 = (double)((a >> 11) + 1ULL) * 0x1.0p-53;
                double u2 = (double)(b >> 11) * 0x1.0p-53;
                double r = sqrt(-2.0 * log(u1));
                double ang = 6.283185307179586476925286766559 * u2;
                out[j] = (float)(mu + sigma * (r * cos(ang)));
                out[j + 1] = (float)(mu + sigma * (r * sin(ang)));
                j += 2;
            } else {
                out[j] = (float)(mu + sigma * synth_z(key, i));
                j += 1;
            }
        }
    }
}

/* Uniform integers in [0, n_range) for counters [start, start+n). */
void synth_uniform_int(uint64_t key, uint64_t start, uint64_t n, uint32_t n_range, int32_t* out) {
    for (uint64_t j = 0; j < n; j++) {
        uint64_t u = synth_u64(key, start + j) >> 32;
        out[j] = (int32_t)((u * (uint64_t)n_range) >> 32);
    }
}

/* ---- weight blob --------------------------------------------------------- */

/* cfg = {dim, hidden_dim, n_layers, n_heads, n_kv_heads, vocab_size, seq_len} */
uint64_t synth_blob_floats(const int32_t* cfg, int shared_weights) {
    uint64_t d = (uint64_t)cfg[0], h = (uint64_t)cfg[1], L = (uint64_t)cfg[2];
    uint64_t H = (uint64_t)cfg[3], Hkv = (uint64_t)cfg[4], V = (uint64_t)cfg[5], S = (uint64_t)cfg[6];
    uint64_t hs = d / H, kvd = Hkv * hs;
    uint64_t n = V * d + L * d + L * d * d + 2 * L * kvd * d + L * d * d + L * d
               + 3 * L * h * d + d + S * hs;
    if (!shared_weights) n += V * d;
    return n;
}

/* Region kinds: 0 = matrix weight, 1 = RMSNorm gain, 2 = zero (legacy freq_cis). */
static int synth_regions(const int32_t* cfg, int shared, uint64_t* ends, int* kinds) {
    uint64_t d = (uint64_t)cfg[0], h = (uint64_t)cfg[1], L = (uint64_t)cfg[2];
    uint64_t H = (uint64_t)cfg[3], Hkv = (uint64_t)cfg[4], V = (uint64_t)cfg[5], S = (uint64_t)cfg[6];
    uint64_t hs = d / H, kvd = Hkv * hs;
    uint64_t sizes[13] = {V * d, L * d, L * d * d, L * kvd * d, L * kvd * d, L * d * d, L * d,
                          L * h * d, L * d * h, L * h * d, d, S * hs, shared ? 0 : V * d};
    int kk[13] = {0, 1, 0, 0, 0, 0, 1, 0, 0, 0, 1, 2, 0};
    uint64_t acc = 0;
    for (int r = 0; r < 13; r++) { acc += sizes[r]; ends[r] = acc; kinds[r] = kk[r]; }
    return 13;
}

/* Writes blob elements [start, start+count) into out. */
int synth_blob(const int32_t* cfg, int shared_weights, uint64_t seed, double wsigma, double nsigma,
               uint64_t start, uint64_t count, float* out) {
    uint64_t ends[13]; int kinds[13];
    int nr = synth_regions(cfg, shared_weights, ends, kinds);
    uint64_t key = synth_key(seed, 0, 0);
    uint64_t e = start, stop = start + count, beg = 0;
    for (int r = 0; r < nr && e < stop; r++) {
        uint64_t rend = ends[r];
        if (e >= rend) { beg = rend; continue; }
        uint64_t seg_end = rend < stop ? rend : stop;
        uint64_t n = seg_end - e;
        float* o = out + (e - start);
        if (kinds[r] == 0) {
            synth_normal_f32(key, e, n, 0.0, wsigma, o);
        } else if (kinds[r] == 1) {
            if (nsigma == 0.0) { for (uint64_t j = 0; j < n; j++) o[j] = 1.0f; }
            else synth_normal_f32(key, e, n, 1.0, nsigma, o);
        } else {
            for (uint64_t j = 0; j < n; j++) o[j] = 0.0f;
        }
        e = seg_end;
        beg = rend;
    }
    (void)beg;
    return e == stop ? 0 : -1;
}

/* ---- KV prefill ---------------------------------------------------------- */

/* K and V values for sequence `seq`: element (l, t, c) of a cache laid out
 * [L][S][kvd] draws counter (l*S + t)*kvd + c of stream 1, sub 2*seq (K) and
 * 2*seq+1 (V).  Writes positions t in [0, n_pos) as [L][n_pos][kvd]. */
void synth_kv(uint64_t seed, uint64_t seq, int32_t n_layers, int32_t seq_len, int32_t kv_dim,
              int32_t n_pos, double sigma, float* k_out, float* v_out) {
    uint64_t kk = synth_key(seed, 1, 2 * seq), kv = synth_key(seed, 1, 2 * seq + 1);
    for (int32_t l = 0; l < n_layers; l++) {
        uint64_t c0 = ((uint64_t)l * (uint64_t)seq_len) * (uint64_t)kv_dim;
        uint64_t n = (uint64_t)n_pos * (uint64_t)kv_dim;
        uint64_t o0 = (uint64_t)l * n;
        if (k_out) synth_normal_f32(kk, c0, n, 0.0, sigma, k_out + o0);
        if (v_out) synth_normal_f32(kv, c0, n, 0.0, sigma, v_out + o0);
    }
}

/* token ids (stream 2) and positions (stream 3) */
void synth_tokens(uint64_t seed, uint64_t sub, uint64_t n, uint32_t vocab, int32_t* out) {
    synth_uniform_int(synth_key(seed, 2, sub), 0, n, vocab, out);
}

void synth_positions(uint64_t seed, uint64_t sub, uint64_t n, uint32_t n_range, int32_t* out) {
    synth_uniform_int(synth_key(seed, 3, sub), 0, n, n_range, out);
}
