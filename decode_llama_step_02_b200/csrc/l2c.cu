// l2c.cu - host runtime and C ABI of the decode-step library (see include/l2c.h).
//
// Device layout (all sizes 64-bit):
//   E [V][d]              embedding (also the classifier when tied)
//   rms_att, rms_ffn [L][d], rms_final [d]
//   Wqkv [L][d + 2 kvd][d]  Wq, Wk, Wv rows concatenated: one matvec per layer
//   Wo [L][d][d], W2 [L][d][h]
//   W13 [L][2h][d]        row 2i = W1 row i, row 2i+1 = W3 row i (SwiGLU pairs)
//   Wcls [V][d]           only when untied
//   Q8_0 copies: the same matrices as row records [K codes | K/gs scales | pad16]
//   KV caches [max_batch][L][S][kvd] fp32 for K and for V
// A step is captured once per variant as a CUDA graph; token and position
// live in device memory, so one graph serves every position.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "../../include/l2c.h"
#include "batched.cuh"
#include "kvcache.cuh"
#include "sampling.cuh"
#include "kernels.cuh"

using namespace l2c;

struct Q8Mat {
    uint8_t* p = nullptr;
    size_t rb = 0;  // record bytes per row
};

// Activations of a batched step over entries 0..B-1 (sequences of the
// handle, or the tokens of a prompt chunk) and where their KV caches are.
struct BatchBufs {
    float *x = nullptr, *q = nullptr, *att = nullptr, *hb = nullptr, *logits = nullptr;
    int* tp = nullptr;                   // [cap][2] token, pos
    unsigned long long* amax = nullptr;  // [cap] argmax keys
    void* part = nullptr;                // attention partials
    int* cnt = nullptr;                  // attention arrival counters [cap][Hkv] (zero between launches)
    size_t cache_off = 0;                // floats from sequence 0's cache to entry 0's
    size_t seq_stride = 0;               // floats between entries' caches (0: one cache shared by all)
};

struct l2c_ctx {
    l2c_config c{};
    int shared = 1, max_batch = 1;
    cudaStream_t stream = nullptr, cap = nullptr;
    int dev = 0, sms = 148;
    int d = 0, h = 0, L = 0, H = 0, Hkv = 0, hs = 0, kvd = 0, V = 0, S = 0, rep = 1;
    // fp32 weights
    float *E = nullptr, *rms_att = nullptr, *rms_ffn = nullptr, *rms_final = nullptr;
    float *Wqkv = nullptr, *Wo = nullptr, *W13 = nullptr, *W2 = nullptr, *Wcls = nullptr, *freq = nullptr;
    // Q8_0 weights
    int gs = 0;
    Q8Mat qE, qWqkv, qWo, qW13, qW2, qWcls;
    // Q4_0 weights (packed records; the embedding as Q8_0-layout records of 4-bit codes)
    int gs4 = 0;
    Q8Mat q4E, q4Wqkv, q4Wo, q4W13, q4W2, q4Wcls;
    // state
    float *kc = nullptr, *vc = nullptr;
    float *x = nullptr, *q = nullptr, *att = nullptr, *hb = nullptr, *logits = nullptr;
    int* tp = nullptr;  // [max_batch][2]
    unsigned long long* amax = nullptr;
    int* err = nullptr;
    int* gen_tokens = nullptr;  // [S]
    int* gen_count = nullptr;
    int* idx_out = nullptr;
    unsigned long long* key_scratch = nullptr;
    double* sample_q = nullptr;  // weights of l2c_sample, sample_n doubles (allocated on first use)
    size_t sample_n = 0;
    void* attn_part = nullptr;
    int* attn_cnt = nullptr;
    int attn_ctas = 0;          // fp32 attention CTAs to aim for (0: all that are resident at once)
    int attn_ctas_f64 = 0;      // double attention CTAs to aim for (0: all that are resident at once)
    int attn_occ_f32 = 1, attn_occ_f64 = 4;  // resident CTAs per SM of this shape's attention kernels
    int attn_min_chunk = 32;    // positions per attention chunk, at least
    int attn_nchunks_max = 1;   // chunks the partials buffer holds per (sequence, KV head)
    // graphs: [weight format: fp32, Q8_0, Q4_0][gen]
    cudaGraphExec_t graph[3][2] = {{nullptr, nullptr}, {nullptr, nullptr}, {nullptr, nullptr}};
    // batched Q8_0 step: quantized activations of every sequence, one graph per batch size
    int8_t* bxq = nullptr;
    double* bxs = nullptr;
    size_t bkq = 0, bks = 0;  // strides (bytes of codes, floats of scales) per sequence
    std::vector<cudaGraphExec_t> bgraph;  // Q8_0, index B (1..max_batch)
    std::vector<cudaGraphExec_t> bgraph_f32;  // fp32, index B
    // int8 KV cache (l2c_enable_kv8): codes [max_batch][L][S][kvd], scales [max_batch][L][S][Hkv]
    bool kv8 = false;
    int8_t *kq8 = nullptr, *vq8 = nullptr;
    float *ks8 = nullptr, *vs8 = nullptr;
    BatchBufs bb;            // the handle's sequences (x, q, ... above)
    BatchBufs pb;            // prompt chunks of l2c_prefill (allocated on first use, BMAX entries)
    float* xb = nullptr;     // fp32 batched step: normalized input rows [BMAX][xbs]
    size_t xbs = 0;
    size_t bgemm_smem = 64 << 10;         // dynamic shared memory a batched GEMM CTA may take
    int bgemm_stages = 3;                 // ring stages (deeper rings cost the second CTA per SM)
    // tuning
    size_t pf_f32 = 32 << 10, pf_q8 = 64 << 10;  // per CTA; larger leads measured slower in the step graph
    int f32_ctas_per_sm = 1;
    size_t q8_smem_budget = 220 << 10;  // dynamic shared memory of one Q8_0 GEMV CTA (its rings)
    int q8_early = 0;    // 1: Q8_0 GEMVs let the next kernel launch as soon as they start (else at their end)
    int q8_wide = 1;     // Q8_0 GEMVs take twice the rows per unit where the ring allows (launch_gemv)
    int q4_unit4 = 1;    // Q4_0 GEMVs take four times the rows per unit where the ring allows
    unsigned long long wait_ns = kWaitNs;  // limit of every bounded wait in the kernels
    int* stall = nullptr;  // test switch read by the Q8_0 q/k/v kernel of layer 0
    long long oom_after = -1;  // test switch: device allocations after this many fail
    bool pdl = true;     // programmatic dependent launch between the step's kernels
    int late_trigger = 2;  // bit 0 fp32, bit 1 Q8_0: GEMVs let the next kernel launch only near their end
    bool graphs = true;  // replay the step as a CUDA graph (off: plain launches)
    std::vector<void*> allocs;
    char msg[512] = {0};
    int status = L2C_OK;  // code of the last failure
};

// ------------------------------------------------------------------ helpers --

static int fail(l2c_ctx* h, int code, const char* fmt, ...) {
    if (h) {
        h->status = code;
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(h->msg, sizeof(h->msg), fmt, ap);
        va_end(ap);
    }
    return code;
}

#define CK(call)                                                                              \
    do {                                                                                      \
        cudaError_t e_ = (call);                                                              \
        if (e_ != cudaSuccess)                                                                \
            return fail(h, L2C_E_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));       \
    } while (0)

static int dalloc(l2c_ctx* h, void** p, size_t bytes) {
    if (bytes == 0) bytes = 16;
    if (h->oom_after >= 0 && (long long)h->allocs.size() >= h->oom_after) {
        *p = nullptr;
        return fail(h, L2C_E_OOM, "device allocation %zu refused by L2C_TEST_OOM_AFTER", h->allocs.size());
    }
    cudaError_t e = cudaMalloc(p, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(h, L2C_E_OOM, "cudaMalloc(%zu) failed: %s", bytes, cudaGetErrorString(e));
    }
    h->allocs.push_back(*p);
    return L2C_OK;
}

static size_t env_size(const char* name, size_t dflt) {
    const char* v = getenv(name);
    return v ? (size_t)strtoull(v, nullptr, 10) : dflt;
}

static bool is_device_ptr(const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

static bool g_pdl = true;  // launch attribute switch, set from the handle before each launch

template <typename Kern, typename... Args>
static cudaError_t launch(cudaStream_t s, bool pdl, Kern kernel, dim3 grid, dim3 block, size_t smem,
                          Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (pdl && g_pdl) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

extern "C" size_t l2c_blob_floats(const l2c_config* c, int shared_weights) {
    if (!c || c->n_heads <= 0) return 0;
    size_t d = (size_t)c->dim, hh = (size_t)c->hidden_dim, L = (size_t)c->n_layers;
    size_t hs = d / (size_t)c->n_heads, kvd = (size_t)c->n_kv_heads * hs;
    size_t V = (size_t)c->vocab_size, S = (size_t)c->seq_len;
    size_t n = V * d + L * d + 2 * L * d * d + 2 * L * kvd * d + L * d + 3 * L * hh * d + d + S * hs;
    return shared_weights ? n : n + V * d;
}

// ------------------------------------------------------------- step building --

struct GemvShape {
    int rows, K, unit;
};

// Kernels of the step, in order within a layer.
enum StepKernel : int { SK_QKV = 0, SK_ATTN = 1, SK_WO = 2, SK_W13 = 3, SK_W2 = 4, SK_CLS = 5 };

// Weight formats of the single-sequence step.
enum WeightFormat : int { WF_F32 = 0, WF_Q80 = 1, WF_Q40 = 2 };

template <int MODE>
static cudaError_t launch_gemv(l2c_ctx* h, int wf, GemvArgs a, int unit) {
    const int units = a.rows / unit;
    a.late_trigger = (h->late_trigger >> (wf != WF_F32 ? 1 : 0)) & 1;
    if (wf == WF_F32) {
        int grid = h->sms * h->f32_ctas_per_sm;
        if (grid > units) grid = units;
        a.prefetch_bytes = h->pf_f32;
        // K slices per row: the split that spreads the CTA's slices most evenly
        // over its 16 warps (slices of at least 512 floats)
        const int warps = F32_THREADS / 32;
        const int rows_max = unit * ((units + grid - 1) / grid);
        const double rows_avg = (double)a.rows / grid;
        int ks = 1;
        double best = 0.0;
        for (int k = 1; k <= 4; k *= 2) {
            if (a.K % (4 * k) || a.K / k < 1024) break;  // slices of at least one full load batch
            const int per_warp = (rows_max * k + warps - 1) / warps;
            const double eff = rows_avg * k / warps / per_warp;
            if (eff > best * 1.03) { best = eff; ks = k; }
        }
        const size_t smem = (size_t)a.K * 4 + (size_t)rows_max * ks * 4;
        return launch(h->cap, true, k_gemv_f32<MODE>, dim3(grid), dim3(F32_THREADS), smem, a, ks);
    }
    // ring slots per warp for units of u rows (0 if none fit the budget)
    auto slots_for = [&](int u) {
        const uint32_t ub = (uint32_t)((size_t)u * a.ld);
        const size_t fixed = q8_smem(0, ub, a.K, a.gs).total;
        const size_t per = (size_t)Q8_WARPS * (ub + 8);
        return h->q8_smem_budget > fixed ? (int)((h->q8_smem_budget - fixed) / per) : 0;
    };
    // Q8_0 with twice the rows per unit (UM = 2): where two ring slots of them fit, or
    // one and every warp still gets at least two units (measured on the 7B widths: q/k/v
    // 17.1 -> 14.4 us, W1/W3 20.5 -> 19.4, wo 8.8 -> 7.6, classifier 30.2 -> 26.6; W2 with
    // one slot and 1.7 units per warp 14.8 -> 15.9, so it keeps its single rows)
    bool wide = false;
    // Q4_0: rows per unit times 2, or 4 where two ring slots of those still fit (on the
    // 7B widths wo 6.9 -> 6.2 us and the classifier 23.5 -> 18.4; W1/W3 with one slot of
    // 8 rows measured no faster, so it keeps 4)
    int q4um = 2;
    if (wf == WF_Q40) {
        if (h->q4_unit4 && a.K % 64 == 0 && a.rows % (4 * unit) == 0 && slots_for(4 * unit) >= 2) q4um = 4;
        unit *= q4um;
    } else if (wf == WF_Q80 && h->q8_wide && a.K % 64 == 0 && (a.gs == 32 || a.gs == 64 || a.gs == 128) &&
               a.rows % (2 * unit) == 0) {
        const int ns_w = slots_for(2 * unit);
        const int units_w = a.rows / (2 * unit);
        const int warps = (h->sms < units_w ? h->sms : units_w) * Q8_WARPS;
        if (ns_w >= 2 || (ns_w == 1 && units_w >= 2 * warps)) {
            wide = true;
            unit *= 2;
        }
    }
    // units of UNIT rows, as many ring slots per warp as fit (2..8; the widened units: 1..8)
    const int units_q = a.rows / unit;
    const int grid = h->sms < units_q ? h->sms : units_q;
    Q8Ring R = {};
    R.unit_bytes = (uint32_t)((size_t)unit * a.ld);
    const int ns = slots_for(unit), ns_min = wide ? 1 : 2;
    R.ns = ns < ns_min ? ns_min : (ns > 8 ? 8 : ns);
    const size_t smem = q8_smem(R.ns, R.unit_bytes, a.K, a.gs).total;
    a.early = h->q8_early;
    a.prefetch_bytes = h->pf_q8;
    const dim3 g(grid), t(Q8_THREADS);
    if (wf == WF_Q40) {  // gs 32, 64 or 128 (l2c_enable_q40); K an odd multiple of 32 only with gs 32
        if (a.K % 64) return launch(h->cap, true, k_gemv_q8<MODE, 32, 1, 2>, g, t, smem, a, R);
        if (q4um == 4) {
            if (a.gs == 64) return launch(h->cap, true, k_gemv_q8<MODE, 64, 2, 4>, g, t, smem, a, R);
            if (a.gs == 32) return launch(h->cap, true, k_gemv_q8<MODE, 32, 2, 4>, g, t, smem, a, R);
            return launch(h->cap, true, k_gemv_q8<MODE, 128, 2, 4>, g, t, smem, a, R);
        }
        if (a.gs == 64) return launch(h->cap, true, k_gemv_q8<MODE, 64, 2, 2>, g, t, smem, a, R);
        if (a.gs == 32) return launch(h->cap, true, k_gemv_q8<MODE, 32, 2, 2>, g, t, smem, a, R);
        return launch(h->cap, true, k_gemv_q8<MODE, 128, 2, 2>, g, t, smem, a, R);
    }
    if (wide) {
        if (a.gs == 64) return launch(h->cap, true, k_gemv_q8<MODE, 64, 0, 2>, g, t, smem, a, R);
        if (a.gs == 32) return launch(h->cap, true, k_gemv_q8<MODE, 32, 0, 2>, g, t, smem, a, R);
        return launch(h->cap, true, k_gemv_q8<MODE, 128, 0, 2>, g, t, smem, a, R);
    }
    const bool k64 = a.K % 64 == 0;
    if (k64 && a.gs == 64) return launch(h->cap, true, k_gemv_q8<MODE, 64>, g, t, smem, a, R);
    if (k64 && a.gs == 32) return launch(h->cap, true, k_gemv_q8<MODE, 32>, g, t, smem, a, R);
    if (k64 && a.gs == 128) return launch(h->cap, true, k_gemv_q8<MODE, 128>, g, t, smem, a, R);
    return launch(h->cap, true, k_gemv_q8<MODE, 0>, g, t, smem, a, R);
}

// Every kernel of the Q8_0 step (and of the batched step) asks for the same
// shared-memory carveout, all of it, so that consecutive kernels never wait
// for an SM to be reconfigured between them (that would serialize the overlap
// of programmatic launches).  The fp32 step's kernels keep the default split:
// their streaming loads run faster with a large L1.
template <typename Kern>
static cudaError_t max_carveout(Kern k) {
    return cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
}

static int set_smem_limits(l2c_ctx* h) {
    int maxopt = 0;
    CK(cudaDeviceGetAttribute(&maxopt, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->dev));
    CK(cudaFuncSetAttribute(k_gemv_f32<M_QKV>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));
    CK(cudaFuncSetAttribute(k_gemv_f32<M_RESID>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));
    CK(cudaFuncSetAttribute(k_gemv_f32<M_W13>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));
    CK(cudaFuncSetAttribute(k_gemv_f32<M_CLS>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));
#define L2C_Q8_ATTR(GS_)                                                                                          \
    CK(cudaFuncSetAttribute(k_gemv_q8<M_QKV, GS_>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));   \
    CK(cudaFuncSetAttribute(k_gemv_q8<M_RESID, GS_>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096)); \
    CK(cudaFuncSetAttribute(k_gemv_q8<M_W13, GS_>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));   \
    CK(cudaFuncSetAttribute(k_gemv_q8<M_CLS, GS_>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));
    L2C_Q8_ATTR(0) L2C_Q8_ATTR(32) L2C_Q8_ATTR(64) L2C_Q8_ATTR(128)
#undef L2C_Q8_ATTR
#define L2C_Q4_ATTR(GS_, W4_, UM_)                                                                                           \
    CK(cudaFuncSetAttribute(k_gemv_q8<M_QKV, GS_, W4_, UM_>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));   \
    CK(cudaFuncSetAttribute(k_gemv_q8<M_RESID, GS_, W4_, UM_>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096)); \
    CK(cudaFuncSetAttribute(k_gemv_q8<M_W13, GS_, W4_, UM_>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));   \
    CK(cudaFuncSetAttribute(k_gemv_q8<M_CLS, GS_, W4_, UM_>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));   \
    CK(max_carveout(k_gemv_q8<M_QKV, GS_, W4_, UM_>));                                                                      \
    CK(max_carveout(k_gemv_q8<M_RESID, GS_, W4_, UM_>));                                                                    \
    CK(max_carveout(k_gemv_q8<M_W13, GS_, W4_, UM_>));                                                                      \
    CK(max_carveout(k_gemv_q8<M_CLS, GS_, W4_, UM_>));
    L2C_Q4_ATTR(32, 1, 2) L2C_Q4_ATTR(32, 2, 2) L2C_Q4_ATTR(64, 2, 2) L2C_Q4_ATTR(128, 2, 2)
    L2C_Q4_ATTR(32, 2, 4) L2C_Q4_ATTR(64, 2, 4) L2C_Q4_ATTR(128, 2, 4)
    L2C_Q4_ATTR(32, 0, 2) L2C_Q4_ATTR(64, 0, 2) L2C_Q4_ATTR(128, 0, 2)
#undef L2C_Q4_ATTR
    {
        cudaError_t e = attn_set_smem_limits();
        if (e != cudaSuccess) return fail(h, L2C_E_CUDA, "attention smem limit: %s", cudaGetErrorString(e));
    }
#define L2C_Q8_CARVE(GS_)                      \
    CK(max_carveout(k_gemv_q8<M_QKV, GS_>));   \
    CK(max_carveout(k_gemv_q8<M_RESID, GS_>)); \
    CK(max_carveout(k_gemv_q8<M_W13, GS_>));   \
    CK(max_carveout(k_gemv_q8<M_CLS, GS_>));
    L2C_Q8_CARVE(0) L2C_Q8_CARVE(32) L2C_Q8_CARVE(64) L2C_Q8_CARVE(128)
#undef L2C_Q8_CARVE
    CK(max_carveout(k_bgemm_q8<M_QKV>));
    CK(max_carveout(k_bgemm_q8<M_RESID>));
    CK(max_carveout(k_bgemm_q8<M_W13>));
    CK(max_carveout(k_bgemm_q8<M_CLS>));
    CK(max_carveout(k_bprep));
    h->bgemm_smem = (size_t)maxopt - 8192;
    CK(cudaFuncSetAttribute(k_bgemm_q8<M_QKV>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 8192));
    CK(cudaFuncSetAttribute(k_bgemm_q8<M_RESID>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 8192));
    CK(cudaFuncSetAttribute(k_bgemm_q8<M_W13>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 8192));
    CK(cudaFuncSetAttribute(k_bgemm_q8<M_CLS>, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 8192));
    CK(cudaFuncSetAttribute(k_bprep, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));
    CK(cudaFuncSetAttribute(k_bprep_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, maxopt - 4096));
    CK(max_carveout(k_bprep_f32));
    CK(cudaFuncSetAttribute(k_bgemm_f32<M_QKV>, cudaFuncAttributeMaxDynamicSharedMemorySize, BF_SMEM));
    CK(cudaFuncSetAttribute(k_bgemm_f32<M_RESID>, cudaFuncAttributeMaxDynamicSharedMemorySize, BF_SMEM));
    CK(cudaFuncSetAttribute(k_bgemm_f32<M_W13>, cudaFuncAttributeMaxDynamicSharedMemorySize, BF_SMEM));
    CK(cudaFuncSetAttribute(k_bgemm_f32<M_CLS>, cudaFuncAttributeMaxDynamicSharedMemorySize, BF_SMEM));
    CK(max_carveout(k_bgemm_f32<M_QKV>));
    CK(max_carveout(k_bgemm_f32<M_RESID>));
    CK(max_carveout(k_bgemm_f32<M_W13>));
    CK(max_carveout(k_bgemm_f32<M_CLS>));
    return L2C_OK;
}

// Attention chunks per (sequence, KV head) for a launch over B sequences: at
// most as many CTAs as are resident at once (the 7B shape: one 8-warp CTA per
// SM in fp32, four 4-warp CTAs per SM in double), each chunk at least
// attn_min_chunk positions.
static int attn_nchunks(const l2c_ctx* h, int B, bool dbl) {
    const int target = dbl ? (h->attn_ctas_f64 > 0 ? h->attn_ctas_f64 : h->attn_occ_f64 * h->sms)
                           : (h->attn_ctas > 0 ? h->attn_ctas : h->attn_occ_f32 * h->sms);
    // at most `target` CTAs, so that all of them are resident at once (a
    // second wave of a few CTAs would double the kernel's tail); but when that
    // leaves a single chunk per (sequence, KV head) (many sequences), the next
    // count up: one chunk serialises a whole sequence in one CTA
    const int per = h->Hkv * B;
    int nc = target / per;
    if (nc < 2) nc = (target + per - 1) / per;
    const int maxc = (h->S + h->attn_min_chunk - 1) / h->attn_min_chunk;
    if (nc > maxc) nc = maxc;
    return nc < 1 ? 1 : nc;
}

// Enqueues the attention of one layer over sequences 0..B-1 (grid z).
static cudaError_t launch_attention(l2c_ctx* h, cudaStream_t s, bool pdl, bool dbl, const float* q, const float* kc,
                                    const float* vc, size_t seq_stride, float* out, const int* tp, int B,
                                    void* part, int* cnt, bool shared_kv = false, bool kv8 = false) {
    AttnArgs t = {};
    t.q = q; t.kc = kc; t.vc = vc; t.seq_stride = seq_stride;
    t.out = out; t.tp = tp; t.tp_stride = 2;
    t.H = h->H; t.Hkv = h->Hkv; t.hs = h->hs; t.kvd = h->kvd; t.seq_len = h->S;
    t.nchunks = attn_nchunks(h, B, dbl);
    t.min_chunk = h->attn_min_chunk;
    t.part = part; t.count = cnt; t.shared_kv = shared_kv ? 1 : 0;
    AttnKernel ak = dbl ? attn_kernel_for<double>(h->hs, h->rep) : attn_kernel_for<float>(h->hs, h->rep);
    if (kv8 && dbl) {
        // the int8 cache of the same rows: codes at the same element offset,
        // scales at one per (row, KV head)
        const size_t eo = (size_t)(kc - h->kc);
        t.kq = h->kq8 + eo; t.vq = h->vq8 + eo;
        t.ks = h->ks8 + eo / h->hs; t.vs = h->vs8 + eo / h->hs;
        t.sc_seq_stride = seq_stride / h->hs;
        ak = attn_kernel_kv8(h->hs, h->rep);
    }
    const size_t smem = (size_t)(dbl ? attn_smem_for<double>(h->rep) : attn_smem_for<float>(h->rep));
    const int threads = dbl ? attn_threads<double>() : attn_threads<float>();
    return launch(s, pdl, ak, dim3(t.nchunks, h->Hkv, B), dim3(threads), smem, t);
}

// The int8 cache arguments for fp32 rows starting at kc / vc (rows of the
// handle's cache; the int8 rows sit at the same row index).
static Kv8Args kv8_args(l2c_ctx* h, float* kc, float* vc) {
    Kv8Args k8 = {};
    const size_t eo = (size_t)(kc - h->kc);
    k8.kc = kc; k8.vc = vc;
    k8.kq = h->kq8 + eo; k8.vq = h->vq8 + eo;
    k8.ks = h->ks8 + eo / h->hs; k8.vs = h->vs8 + eo / h->hs;
    k8.kvd = h->kvd; k8.hs = h->hs; k8.n_kv_heads = h->Hkv;
    return k8;
}

// Enqueues kernel `kind` of layer l (sequence seq) on stream s.
static int launch_step_kernel(l2c_ctx* h, cudaStream_t s, int kind, int wf, int l, int seq = 0) {
    const bool q80 = wf != WF_F32;  // quantized weights (Q8_0 or Q4_0)
    const bool w4 = wf == WF_Q40;
    const Q8Mat& mE = w4 ? h->q4E : h->qE;
    const Q8Mat& mQKV = w4 ? h->q4Wqkv : h->qWqkv;
    const Q8Mat& mO = w4 ? h->q4Wo : h->qWo;
    const Q8Mat& m13 = w4 ? h->q4W13 : h->qW13;
    const Q8Mat& m2 = w4 ? h->q4W2 : h->qW2;
    const Q8Mat& mCls = w4 ? h->q4Wcls : h->qWcls;
    g_pdl = h->pdl;
    const size_t d = h->d, kvd = h->kvd, hh = h->h, S = h->S;
    const size_t cache_off = (size_t)seq * h->L * S * kvd;
    float* kslot = h->kc + cache_off + (size_t)l * S * kvd;
    float* vslot = h->vc + cache_off + (size_t)l * S * kvd;
    float* x = h->x + (size_t)seq * d;
    float* q = h->q + (size_t)seq * d;
    float* att = h->att + (size_t)seq * d;
    float* hb = h->hb + (size_t)seq * hh;
    int* tp = h->tp + 2 * seq;
    unsigned long long* amax = h->amax + seq;
    cudaStream_t saved = h->cap;
    h->cap = s;  // launch_gemv enqueues on h->cap
    cudaError_t e = cudaSuccess;
    GemvArgs a = {};
    a.gs = w4 ? h->gs4 : h->gs; a.tp = tp; a.err = h->err; a.vocab = h->V; a.seq_len = h->S; a.wait_ns = h->wait_ns;
    a.d = (int)d; a.kvd = (int)kvd; a.hs = h->hs;
    switch (kind) {
    case SK_QKV:  // RMSNorm + q/k/v + RoPE + cache write
        a.rows = (int)(d + 2 * kvd);
        a.K = (int)d;
        if (q80) { a.W = mQKV.p + (size_t)l * a.rows * mQKV.rb; a.ld = mQKV.rb; }
        else { a.W = h->Wqkv + (size_t)l * a.rows * d; a.ld = d; }
        a.in = x;
        a.norm_w = h->rms_att + (size_t)l * d;
        if (l == 0) {
            a.emb = q80 ? (const void*)mE.p : (const void*)h->E;
            a.x_resid = x;
            a.amax = amax;
        }
        a.out = q;
        a.kslot = kslot;
        a.vslot = vslot;
        a.freq = h->freq;
        if (l == 0 && seq == 0) a.stall = h->stall;
        e = launch_gemv<M_QKV>(h, wf, a, 2);
        break;
    case SK_ATTN:  // with the int8 KV cache the attention also stores the row at pos
        e = launch_attention(h, s, true, q80, q, kslot, vslot, (size_t)h->L * S * kvd, att, tp, 1, h->attn_part,
                             h->attn_cnt + (size_t)seq * h->Hkv, false, h->kv8);
        break;
    case SK_WO:  // wo + residual
        a.rows = (int)d; a.K = (int)d;
        if (q80) { a.W = mO.p + (size_t)l * d * mO.rb; a.ld = mO.rb; }
        else { a.W = h->Wo + (size_t)l * d * d; a.ld = d; }
        a.in = att; a.out = x;
        e = launch_gemv<M_RESID>(h, wf, a, 1);
        break;
    case SK_W13:  // RMSNorm + W1/W3 + SwiGLU
        a.rows = (int)(2 * hh); a.K = (int)d;
        if (q80) { a.W = m13.p + (size_t)l * 2 * hh * m13.rb; a.ld = m13.rb; }
        else { a.W = h->W13 + (size_t)l * 2 * hh * d; a.ld = d; }
        a.in = x; a.norm_w = h->rms_ffn + (size_t)l * d; a.out = hb;
        e = launch_gemv<M_W13>(h, wf, a, 2);
        break;
    case SK_W2:  // W2 + residual
        a.rows = (int)d; a.K = (int)hh;
        if (q80) { a.W = m2.p + (size_t)l * d * m2.rb; a.ld = m2.rb; }
        else { a.W = h->W2 + (size_t)l * d * hh; a.ld = hh; }
        a.in = hb; a.out = x;
        e = launch_gemv<M_RESID>(h, wf, a, 1);
        break;
    default:  // final RMSNorm + classifier + argmax
        a.rows = h->V; a.K = (int)d;
        if (q80) { a.W = mCls.p; a.ld = mCls.rb; }
        else { a.W = h->Wcls; a.ld = d; }
        a.in = x; a.norm_w = h->rms_final; a.out = h->logits + (size_t)seq * h->V; a.amax = amax;
        e = launch_gemv<M_CLS>(h, wf, a, 1);
        break;
    }
    h->cap = saved;
    if (e != cudaSuccess) return fail(h, L2C_E_CUDA, "kernel %d launch: %s", kind, cudaGetErrorString(e));
    return L2C_OK;
}

// Enqueues one decode step of sequence 0 on h->cap (being captured).
static int enqueue_step(l2c_ctx* h, int wf) {
    int rc;
    for (int l = 0; l < h->L; l++)
        for (int k = SK_QKV; k <= SK_W2; k++)
            if ((rc = launch_step_kernel(h, h->cap, k, wf, l)) != L2C_OK) return rc;
    return launch_step_kernel(h, h->cap, SK_CLS, wf, 0);
}

// ------------------------------------------------------------- batched step --

// K bytes per GEMM stage: a multiple of 32 (the MMA k) and of 4*gs (16-byte
// scale copies) that divides K, at most 512; else the whole row in one stage
// (K a multiple of 32 up to 2048: its scale copies run into the records'
// padding).
static int batched_kc(int K, int gs) {
    int unit = 4 * gs > 32 ? 4 * gs : 32;
    for (int kc = 512 - 512 % unit; kc >= unit; kc -= unit)
        if (K % kc == 0) return kc;
    if (K % 32 == 0 && K % gs == 0 && K <= 2048) return K;
    return 0;
}

static int ensure_batched(l2c_ctx* h) {
    if (h->bxq) return L2C_OK;
    const size_t kmax = (size_t)(h->d > h->h ? h->d : h->h);
    h->bkq = (kmax + 15) & ~size_t(15);
    h->bks = ((kmax / h->gs) + 3) & ~size_t(3);
    int rc;
    if ((rc = dalloc(h, (void**)&h->bxq, (size_t)BMAX * h->bkq)) != L2C_OK) return rc;
    if ((rc = dalloc(h, (void**)&h->bxs, (size_t)BMAX * h->bks * 8)) != L2C_OK) return rc;
    CK(cudaMemsetAsync(h->bxq, 0, (size_t)BMAX * h->bkq, h->stream));
    CK(cudaMemsetAsync(h->bxs, 0, (size_t)BMAX * h->bks * 8, h->stream));
    return L2C_OK;
}

static int ensure_batched_f32(l2c_ctx* h) {
    if (h->xb) return L2C_OK;
    h->xbs = ((size_t)h->d + 3) & ~size_t(3);
    int rc;
    if ((rc = dalloc(h, (void**)&h->xb, (size_t)BMAX * h->xbs * 4)) != L2C_OK) return rc;
    CK(cudaMemsetAsync(h->xb, 0, (size_t)BMAX * h->xbs * 4, h->stream));
    return L2C_OK;
}

// The activations of l2c_prefill's prompt chunks (BMAX tokens each).
static int ensure_prefill(l2c_ctx* h) {
    if (h->pb.x) return L2C_OK;
    BatchBufs& p = h->pb;
    const size_t d = h->d, hh = h->h, V = h->V;
    const size_t part = (size_t)BMAX * h->Hkv * h->attn_nchunks_max * h->rep * (h->hs + 2) * sizeof(double);
    int rc;
    if ((rc = dalloc(h, (void**)&p.x, BMAX * d * 4)) != L2C_OK) return rc;
    if ((rc = dalloc(h, (void**)&p.q, BMAX * d * 4)) != L2C_OK) return rc;
    if ((rc = dalloc(h, (void**)&p.att, BMAX * d * 4)) != L2C_OK) return rc;
    if ((rc = dalloc(h, (void**)&p.hb, BMAX * hh * 4)) != L2C_OK) return rc;
    if ((rc = dalloc(h, (void**)&p.logits, BMAX * V * 4)) != L2C_OK) return rc;
    if ((rc = dalloc(h, (void**)&p.tp, BMAX * 2 * 4)) != L2C_OK) return rc;
    if ((rc = dalloc(h, (void**)&p.amax, BMAX * 8)) != L2C_OK) return rc;
    if ((rc = dalloc(h, &p.part, part)) != L2C_OK) return rc;
    if ((rc = dalloc(h, (void**)&p.cnt, (size_t)BMAX * h->Hkv * 4)) != L2C_OK) return rc;
    CK(cudaMemsetAsync(p.cnt, 0, (size_t)BMAX * h->Hkv * 4, h->stream));
    CK(cudaMemsetAsync(p.tp, 0, BMAX * 2 * 4, h->stream));
    return L2C_OK;
}

static int bprep(l2c_ctx* h, cudaStream_t s, int B, const BatchBufs& bb, const float* in, size_t in_stride, int K,
                 const float* norm, bool emb, unsigned long long* amax) {
    BPrepArgs p = {};
    p.in = in; p.in_stride = in_stride; p.norm_w = norm;
    p.emb = emb ? h->qE.p : nullptr; p.emb_rb = h->qE.rb; p.x_resid = bb.x;
    p.K = K; p.gs = h->gs; p.xq = h->bxq; p.xs = h->bxs; p.kq_stride = h->bkq; p.ks_stride = h->bks;
    p.tp = bb.tp; p.vocab = h->V; p.seq_len = h->S; p.amax = amax; p.err = h->err;
    CK(launch(s, true, k_bprep, dim3(B, BPREP_SPLIT), dim3(256), (size_t)K * 4, p));
    return L2C_OK;
}

// The epilogue fields of a batched GEMM over rows [row0, row0 + rows) of a
// layer-l matrix.
static BGemmArgs bgemm_args(l2c_ctx* h, int B, const BatchBufs& bb, int rows, int K, float* out, size_t out_stride,
                            int l) {
    BGemmArgs g = {};
    g.rows = rows; g.K = K; g.gs = h->gs; g.B = B;
    g.out = out; g.out_stride = out_stride;
    g.kc_base = h->kc + bb.cache_off + (size_t)l * h->S * h->kvd;
    g.vc_base = h->vc + bb.cache_off + (size_t)l * h->S * h->kvd;
    g.seq_stride = bb.seq_stride;
    g.freq = h->freq; g.d = h->d; g.kvd = h->kvd; g.hs = h->hs; g.seq_len = h->S;
    g.tp = bb.tp; g.amax = bb.amax; g.err = h->err;
    return g;
}

template <int MODE>
static int bgemm(l2c_ctx* h, cudaStream_t s, int B, const BatchBufs& bb, const Q8Mat& m, size_t row0, int rows,
                 int K, float* out, size_t out_stride, int l) {
    BGemmArgs g = bgemm_args(h, B, bb, rows, K, out, out_stride, l);
    g.W = m.p + row0 * m.rb; g.rb = m.rb; g.kc = batched_kc(K, h->gs);
    g.xq = h->bxq; g.xs = h->bxs; g.kq_stride = h->bkq; g.ks_stride = h->bks;
    g.prefetch_bytes = h->pf_q8;
    // ring stages: the depth sets the bytes in flight.  A grid of more CTAs
    // than SMs keeps bgemm_stages (two CTAs per SM then share the shared
    // memory); a grid of at most one CTA per SM takes as many as fit (up to 8)
    const int grid = (rows + BG_ROWS - 1) / BG_ROWS;
    BLayout L = make_blayout(g.kc, h->gs, 1);
    const int cap = grid <= h->sms ? 8 : h->bgemm_stages;
    int ns = (int)(h->bgemm_smem / (L.stage_bytes + 16));
    ns = ns < 2 ? 2 : (ns > cap ? cap : ns);
    L = make_blayout(g.kc, h->gs, ns);
    size_t smem = (size_t)L.ns * L.stage_bytes + 16 * (size_t)L.ns;
    CK(launch(s, true, k_bgemm_q8<MODE>, dim3(grid), dim3(32 * (BG_WARPS + 1)), smem, g, L));
    return L2C_OK;
}

// fp32: RMSNorm (or the layer-0 embedding row and its norm) of entries 0..B-1 -> h->xb.
static int bprep_f32(l2c_ctx* h, cudaStream_t s, int B, const BatchBufs& bb, const float* norm, bool emb,
                     unsigned long long* amax) {
    BPrepF32Args p = {};
    p.in = bb.x; p.in_stride = h->d; p.norm_w = norm;
    p.emb = emb ? h->E : nullptr; p.x_resid = bb.x;
    p.out = h->xb; p.out_stride = h->xbs; p.K = h->d;
    p.tp = bb.tp; p.vocab = h->V; p.amax = amax; p.err = h->err;
    CK(launch(s, true, k_bprep_f32, dim3(B, BPREP_SPLIT), dim3(256), (size_t)h->d * 4, p));
    return L2C_OK;
}

template <int MODE>
static int bgemm_f32(l2c_ctx* h, cudaStream_t s, int B, const BatchBufs& bb, const float* W, int rows, int K,
                     const float* X, size_t x_stride, float* out, size_t out_stride, int l) {
    BGemmArgs g = bgemm_args(h, B, bb, rows, K, out, out_stride, l);
    g.W = reinterpret_cast<const uint8_t*>(W); g.rb = (size_t)K * 4;
    g.prefetch_bytes = h->pf_f32;
    const int grid = (rows + BF_ROWS - 1) / BF_ROWS;
    CK(launch(s, true, k_bgemm_f32<MODE>, dim3(grid), dim3(BF_THREADS), (size_t)BF_SMEM, g, X, x_stride));
    return L2C_OK;
}

// One batched step of entries 0..B-1 of `bb` on stream s: Q8_0 (int8 tensor
// cores, double group sums) or fp32 (FFMA).  With shared_kv every entry
// reads and writes one cache (a prompt chunk).
static int enqueue_batch_step(l2c_ctx* h, cudaStream_t s, int B, const BatchBufs& bb, bool q80, bool shared_kv) {
    g_pdl = h->pdl;
    const size_t d = h->d, hh = h->h, kvd = h->kvd, S = h->S;
    int rc;
    for (int l = 0; l < h->L; l++) {
        const float* kl = h->kc + bb.cache_off + (size_t)l * S * kvd;
        const float* vl = h->vc + bb.cache_off + (size_t)l * S * kvd;
        if (q80) {
            if ((rc = bprep(h, s, B, bb, bb.x, d, (int)d, h->rms_att + (size_t)l * d, l == 0,
                            l == 0 ? bb.amax : nullptr)))
                return rc;
            if ((rc = bgemm<M_QKV>(h, s, B, bb, h->qWqkv, (size_t)l * (d + 2 * kvd), (int)(d + 2 * kvd), (int)d,
                                   bb.q, d, l)))
                return rc;
        } else {
            if ((rc = bprep_f32(h, s, B, bb, h->rms_att + (size_t)l * d, l == 0, l == 0 ? bb.amax : nullptr)))
                return rc;
            if ((rc = bgemm_f32<M_QKV>(h, s, B, bb, h->Wqkv + (size_t)l * (d + 2 * kvd) * d, (int)(d + 2 * kvd),
                                       (int)d, h->xb, h->xbs, bb.q, d, l)))
                return rc;
        }
        CK(launch_attention(h, s, true, q80, bb.q, kl, vl, bb.seq_stride, bb.att, bb.tp, B, bb.part, bb.cnt,
                            shared_kv));
        if (q80) {
            if ((rc = bprep(h, s, B, bb, bb.att, d, (int)d, nullptr, false, nullptr))) return rc;
            if ((rc = bgemm<M_RESID>(h, s, B, bb, h->qWo, (size_t)l * d, (int)d, (int)d, bb.x, d, l))) return rc;
            if ((rc = bprep(h, s, B, bb, bb.x, d, (int)d, h->rms_ffn + (size_t)l * d, false, nullptr))) return rc;
            if ((rc = bgemm<M_W13>(h, s, B, bb, h->qW13, (size_t)l * 2 * hh, (int)(2 * hh), (int)d, bb.hb, hh, l)))
                return rc;
            if ((rc = bprep(h, s, B, bb, bb.hb, hh, (int)hh, nullptr, false, nullptr))) return rc;
            if ((rc = bgemm<M_RESID>(h, s, B, bb, h->qW2, (size_t)l * d, (int)d, (int)hh, bb.x, d, l))) return rc;
        } else {
            if ((rc = bgemm_f32<M_RESID>(h, s, B, bb, h->Wo + (size_t)l * d * d, (int)d, (int)d, bb.att, d, bb.x, d,
                                         l)))
                return rc;
            if ((rc = bprep_f32(h, s, B, bb, h->rms_ffn + (size_t)l * d, false, nullptr))) return rc;
            if ((rc = bgemm_f32<M_W13>(h, s, B, bb, h->W13 + (size_t)l * 2 * hh * d, (int)(2 * hh), (int)d, h->xb,
                                       h->xbs, bb.hb, hh, l)))
                return rc;
            if ((rc = bgemm_f32<M_RESID>(h, s, B, bb, h->W2 + (size_t)l * d * hh, (int)d, (int)hh, bb.hb, hh, bb.x,
                                         d, l)))
                return rc;
        }
    }
    if (q80) {
        if ((rc = bprep(h, s, B, bb, bb.x, d, (int)d, h->rms_final, false, nullptr))) return rc;
        return bgemm<M_CLS>(h, s, B, bb, h->qWcls, 0, h->V, (int)d, bb.logits, (size_t)h->V, 0);
    }
    if ((rc = bprep_f32(h, s, B, bb, h->rms_final, false, nullptr))) return rc;
    return bgemm_f32<M_CLS>(h, s, B, bb, h->Wcls, h->V, (int)d, h->xb, h->xbs, bb.logits, (size_t)h->V, 0);
}

static int build_batch_graph(l2c_ctx* h, int B, bool q80) {
    std::vector<cudaGraphExec_t>& gv = q80 ? h->bgraph : h->bgraph_f32;
    if (gv.size() < (size_t)h->max_batch + 1) gv.assign((size_t)h->max_batch + 1, nullptr);
    if (gv[B]) return L2C_OK;
    CK(cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal));
    int rc = enqueue_batch_step(h, h->cap, B, h->bb, q80, false);
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamEndCapture(h->cap, &g);
    if (rc != L2C_OK) {
        if (g) cudaGraphDestroy(g);
        return rc;
    }
    if (e != cudaSuccess) return fail(h, L2C_E_CUDA, "batched capture failed: %s", cudaGetErrorString(e));
    e = cudaGraphInstantiate(&gv[B], g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return fail(h, L2C_E_CUDA, "batched graph instantiate: %s", cudaGetErrorString(e));
    return L2C_OK;
}

static int build_graph(l2c_ctx* h, int wf, bool gen) {
    if (h->graph[wf][gen]) return L2C_OK;
    CK(cudaStreamBeginCapture(h->cap, cudaStreamCaptureModeThreadLocal));
    int rc = enqueue_step(h, wf);
    if (rc == L2C_OK && gen) {
        cudaError_t e = launch(h->cap, false, k_advance, dim3(1), dim3(1), 0, h->tp,
                               (const unsigned long long*)h->amax, h->gen_tokens, h->gen_count);
        if (e != cudaSuccess) rc = fail(h, L2C_E_CUDA, "advance launch: %s", cudaGetErrorString(e));
    }
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamEndCapture(h->cap, &g);
    if (rc != L2C_OK) {
        if (g) cudaGraphDestroy(g);
        return rc;
    }
    if (e != cudaSuccess) return fail(h, L2C_E_CUDA, "capture failed: %s", cudaGetErrorString(e));
    e = cudaGraphInstantiate(&h->graph[wf][gen], g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return fail(h, L2C_E_CUDA, "graph instantiate: %s", cudaGetErrorString(e));
    return L2C_OK;
}

// ------------------------------------------------------------------ create --

static int copy_in(l2c_ctx* h, void* dst, const float* src, size_t n, cudaMemcpyKind kind) {
    CK(cudaMemcpyAsync(dst, src, n * sizeof(float), kind, h->stream));
    return L2C_OK;
}

// rows of `src` [rows][K] into every `stride`-th row of dst starting at row `first`
static int copy_rows_strided(l2c_ctx* h, float* dst, int first, int stride, const float* src, size_t rows,
                             size_t K, cudaMemcpyKind kind) {
    CK(cudaMemcpy2DAsync(dst + (size_t)first * K, (size_t)stride * K * sizeof(float), src, K * sizeof(float),
                         K * sizeof(float), rows, kind, h->stream));
    return L2C_OK;
}

static int check_config(l2c_ctx* h, const l2c_config* c) {
    if (c->dim <= 0 || c->hidden_dim <= 0 || c->n_layers <= 0 || c->n_heads <= 0 || c->n_kv_heads <= 0 ||
        c->vocab_size <= 0 || c->seq_len <= 0)
        return fail(h, L2C_E_ARG, "config fields must be positive");
    if (c->dim % c->n_heads || c->n_heads % c->n_kv_heads)
        return fail(h, L2C_E_ARG, "dim %% n_heads and n_heads %% n_kv_heads must be 0");
    int hs = c->dim / c->n_heads;
    if (hs % 2) return fail(h, L2C_E_ARG, "head_size must be even (RoPE rotates pairs)");
    if (c->dim % 4 || c->hidden_dim % 4) return fail(h, L2C_E_ARG, "dim and hidden_dim must be multiples of 4");
    if (!attn_kernel_for<float>(hs, c->n_heads / c->n_kv_heads))
        return fail(h, L2C_E_ARG, "unsupported head_size %d / GQA ratio %d", hs, c->n_heads / c->n_kv_heads);
    return L2C_OK;
}

extern "C" int l2c_create(const l2c_config* cfg, const float* blob, size_t blob_floats, int shared_weights,
                          int max_batch, void* cuda_stream, l2c_ctx** out) {
    if (!out) return L2C_E_ARG;
    *out = nullptr;
    if (!cfg || !blob || max_batch < 1) return L2C_E_ARG;
    l2c_ctx* h = new (std::nothrow) l2c_ctx();
    if (!h) return L2C_E_OOM;
    int rc = check_config(h, cfg);
    if (rc == L2C_OK && blob_floats != l2c_blob_floats(cfg, shared_weights))
        rc = fail(h, L2C_E_ARG, "blob has %zu floats, the config needs %zu", blob_floats,
                  l2c_blob_floats(cfg, shared_weights));
    if (rc != L2C_OK) {
        // keep the message reachable through a static handle-less error
        fprintf(stderr, "l2c_create: %s\n", h->msg);
        delete h;
        return rc;
    }
    h->c = *cfg;
    h->shared = shared_weights ? 1 : 0;
    h->max_batch = max_batch;
    h->stream = (cudaStream_t)cuda_stream;
    h->d = cfg->dim; h->h = cfg->hidden_dim; h->L = cfg->n_layers; h->H = cfg->n_heads;
    h->Hkv = cfg->n_kv_heads; h->hs = h->d / h->H; h->kvd = h->Hkv * h->hs; h->V = cfg->vocab_size;
    h->S = cfg->seq_len; h->rep = h->H / h->Hkv;
    h->pf_f32 = env_size("L2C_PREFETCH_F32", h->pf_f32);
    h->pf_q8 = env_size("L2C_PREFETCH_Q8", h->pf_q8);
    h->q8_smem_budget = env_size("L2C_Q8_SMEM", h->q8_smem_budget);
    h->f32_ctas_per_sm = (int)env_size("L2C_F32_CTAS_PER_SM", 1);
    h->pdl = env_size("L2C_NO_PDL", 0) == 0;
    h->late_trigger = (int)env_size("L2C_LATE_TRIGGER", (size_t)h->late_trigger);
    h->graphs = env_size("L2C_NO_GRAPH", 0) == 0;
    h->attn_ctas = (int)env_size("L2C_ATTN_CTAS", 0);
    h->attn_ctas_f64 = (int)env_size("L2C_ATTN_CTAS_F64", 0);
    h->attn_min_chunk = (int)env_size("L2C_ATTN_MIN_CHUNK", (size_t)h->attn_min_chunk);
    if (h->attn_min_chunk < 1) h->attn_min_chunk = 1;
    h->q8_early = (int)env_size("L2C_Q8_EARLY", (size_t)h->q8_early);
    h->q8_wide = (int)env_size("L2C_Q8_WIDE", (size_t)h->q8_wide);
    h->q4_unit4 = (int)env_size("L2C_Q4_UNIT4", (size_t)h->q4_unit4);
    h->bgemm_stages = (int)env_size("L2C_BGEMM_STAGES", (size_t)h->bgemm_stages);
    if (h->bgemm_stages < 2) h->bgemm_stages = 2;
    h->wait_ns = env_size("L2C_WAIT_NS", h->wait_ns);
    if (getenv("L2C_TEST_OOM_AFTER")) h->oom_after = (long long)env_size("L2C_TEST_OOM_AFTER", 0);
    auto bail = [&](int code) { l2c_destroy(h); return code; };
    if (cudaGetDevice(&h->dev) != cudaSuccess) return bail(fail(h, L2C_E_CUDA, "no CUDA device"));
    if (cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->dev) != cudaSuccess)
        return bail(L2C_E_CUDA);
    if (cudaStreamCreateWithFlags(&h->cap, cudaStreamNonBlocking) != cudaSuccess) return bail(L2C_E_CUDA);
    if ((rc = set_smem_limits(h)) != L2C_OK) return bail(rc);
    {  // resident attention CTAs per SM (the default chunk counts keep every CTA resident)
        int occ = 0;
        AttnKernel kf = attn_kernel_for<float>(h->hs, h->rep), kd = attn_kernel_for<double>(h->hs, h->rep);
        if (kf && cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kf, attn_threads<float>(), 0) == cudaSuccess &&
            occ > 0)
            h->attn_occ_f32 = occ;
        if (kd && cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kd, attn_threads<double>(),
                                                                attn_smem_for<double>(h->rep)) == cudaSuccess &&
            occ > 0)
            h->attn_occ_f64 = occ;
        cudaGetLastError();
    }

    const size_t d = h->d, hh = h->h, L = h->L, kvd = h->kvd, V = h->V, S = h->S, B = max_batch;
    const size_t rq = d + 2 * kvd;
#define ALLOC(ptr, bytes)                                                  \
    do {                                                                   \
        if ((rc = dalloc(h, (void**)&(ptr), (bytes))) != L2C_OK) return bail(rc); \
    } while (0)
    ALLOC(h->E, V * d * 4);
    ALLOC(h->rms_att, L * d * 4);
    ALLOC(h->rms_ffn, L * d * 4);
    ALLOC(h->rms_final, d * 4);
    ALLOC(h->Wqkv, L * rq * d * 4);
    ALLOC(h->Wo, L * d * d * 4);
    ALLOC(h->W13, L * 2 * hh * d * 4);
    ALLOC(h->W2, L * d * hh * 4);
    if (!h->shared) {
        ALLOC(h->Wcls, V * d * 4);
    } else {
        h->Wcls = h->E;
    }
    ALLOC(h->freq, (size_t)(h->hs / 2) * 4);
    ALLOC(h->kc, B * L * S * kvd * 4);
    ALLOC(h->vc, B * L * S * kvd * 4);
    ALLOC(h->x, B * d * 4);
    ALLOC(h->q, B * d * 4);
    ALLOC(h->att, B * d * 4);
    ALLOC(h->hb, B * hh * 4);
    ALLOC(h->logits, B * V * 4);
    ALLOC(h->tp, B * 2 * 4);
    ALLOC(h->amax, B * 8);
    ALLOC(h->err, 4);
    ALLOC(h->gen_tokens, (S + 1) * 4);
    ALLOC(h->gen_count, 4);
    ALLOC(h->idx_out, 4);
    ALLOC(h->key_scratch, 8);
    h->attn_nchunks_max = attn_nchunks(h, 1, true) > attn_nchunks(h, 1, false) ? attn_nchunks(h, 1, true)
                                                                                : attn_nchunks(h, 1, false);
    ALLOC(h->attn_part, B * (size_t)h->Hkv * h->attn_nchunks_max * h->rep * (h->hs + 2) * sizeof(double));
    ALLOC(h->stall, 4);
    ALLOC(h->attn_cnt, B * (size_t)h->Hkv * 4);
#undef ALLOC
    h->bb.x = h->x; h->bb.q = h->q; h->bb.att = h->att; h->bb.hb = h->hb; h->bb.logits = h->logits;
    h->bb.tp = h->tp; h->bb.amax = h->amax; h->bb.part = h->attn_part; h->bb.cnt = h->attn_cnt;
    h->bb.cache_off = 0;
    h->bb.seq_stride = L * S * kvd;
    // zero state
    if (cudaMemsetAsync(h->kc, 0, B * L * S * kvd * 4, h->stream) != cudaSuccess ||
        cudaMemsetAsync(h->vc, 0, B * L * S * kvd * 4, h->stream) != cudaSuccess ||
        cudaMemsetAsync(h->attn_cnt, 0, B * (size_t)h->Hkv * 4, h->stream) != cudaSuccess ||
        cudaMemsetAsync(h->err, 0, 4, h->stream) != cudaSuccess ||
        cudaMemsetAsync(h->stall, getenv("L2C_TEST_STALL") ? 1 : 0, 1, h->stream) != cudaSuccess ||
        cudaMemsetAsync(reinterpret_cast<char*>(h->stall) + 1, 0, 3, h->stream) != cudaSuccess ||
        cudaMemsetAsync(h->tp, 0, B * 2 * 4, h->stream) != cudaSuccess ||
        cudaMemsetAsync(h->x, 0, B * d * 4, h->stream) != cudaSuccess)
        return bail(fail(h, L2C_E_CUDA, "memset failed"));

    // weights in checkpoint order -> device layout
    const cudaMemcpyKind kind = is_device_ptr(blob) ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    const float* p = blob;
    const float *pE = p; p += V * d;
    const float *patt = p; p += L * d;
    const float *pq = p; p += L * d * d;
    const float *pk = p; p += L * kvd * d;
    const float *pv = p; p += L * kvd * d;
    const float *po = p; p += L * d * d;
    const float *pffn = p; p += L * d;
    const float *p1 = p; p += L * hh * d;
    const float *p2 = p; p += L * d * hh;
    const float *p3 = p; p += L * hh * d;
    const float *pfin = p; p += d;
    p += S * (size_t)h->hs;  // legacy freq_cis_real and freq_cis_imag, not used
    const float* pcls = h->shared ? nullptr : p;
    if ((rc = copy_in(h, h->E, pE, V * d, kind)) ||
        (rc = copy_in(h, h->rms_att, patt, L * d, kind)) ||
        (rc = copy_in(h, h->rms_ffn, pffn, L * d, kind)) ||
        (rc = copy_in(h, h->rms_final, pfin, d, kind)) ||
        (rc = copy_in(h, h->Wo, po, L * d * d, kind)) ||
        (rc = copy_in(h, h->W2, p2, L * d * hh, kind)))
        return bail(rc);
    if (pcls && (rc = copy_in(h, h->Wcls, pcls, V * d, kind))) return bail(rc);
    for (size_t l = 0; l < L; l++) {
        float* qkv = h->Wqkv + l * rq * d;
        if ((rc = copy_in(h, qkv, pq + l * d * d, d * d, kind)) ||
            (rc = copy_in(h, qkv + d * d, pk + l * kvd * d, kvd * d, kind)) ||
            (rc = copy_in(h, qkv + (d + kvd) * d, pv + l * kvd * d, kvd * d, kind)))
            return bail(rc);
        float* w13 = h->W13 + l * 2 * hh * d;
        if ((rc = copy_rows_strided(h, w13, 0, 2, p1 + l * hh * d, hh, d, kind)) ||
            (rc = copy_rows_strided(h, w13, 1, 2, p3 + l * hh * d, hh, d, kind)))
            return bail(rc);
    }
    // RoPE frequencies of the even in-head indices j: 1 / 10000^(j/hs), fp32
    // (the formula llama2.c evaluates inside forward; tabulated once here)
    std::vector<float> fr(h->hs / 2);
    for (int j = 0; j < h->hs; j += 2) fr[j / 2] = 1.0f / powf(10000.0f, (float)j / (float)h->hs);
    if (cudaMemcpyAsync(h->freq, fr.data(), fr.size() * 4, cudaMemcpyHostToDevice, h->stream) != cudaSuccess)
        return bail(fail(h, L2C_E_CUDA, "freq upload failed"));
    if (cudaStreamSynchronize(h->stream) != cudaSuccess)
        return bail(fail(h, L2C_E_CUDA, "upload failed: %s", cudaGetErrorString(cudaGetLastError())));
    *out = h;
    return L2C_OK;
}

// ---------------------------------------------------------------- Q8_0 set --

static size_t record_bytes(int K, int gs) {
    return (size_t)K + (((size_t)(K / gs) * 4 + 15) & ~size_t(15));
}

static int make_q8(l2c_ctx* h, Q8Mat& m, const float* W, size_t rows, int K) {
    m.rb = record_bytes(K, h->gs);
    int rc = dalloc(h, (void**)&m.p, rows * m.rb);
    if (rc) return rc;
    CK(cudaMemsetAsync(m.p, 0, rows * m.rb, h->stream));
    long long groups = (long long)rows * (K / h->gs);
    long long blocks = (groups + 7) / 8;
    int grid = (int)(blocks < 65535LL * 16 ? blocks : 65535LL * 16);
    k_quantize_rows<<<grid, 256, 0, h->stream>>>(W, (long long)rows, K, h->gs, m.p, m.rb);
    CK(cudaGetLastError());
    return L2C_OK;
}

extern "C" int l2c_enable_q80(l2c_ctx* h, int gs) {
    if (!h) return L2C_E_ARG;
    if (h->gs) return h->gs == gs ? L2C_OK : fail(h, L2C_E_STATE, "Q8_0 already enabled with gs=%d", h->gs);
    if (gs < 16 || gs > 256 || gs % 16 || h->d % gs || h->h % gs)
        return fail(h, L2C_E_ARG, "gs=%d must be a multiple of 16 in [16,256] dividing dim and hidden_dim", gs);
    h->gs = gs;
    const size_t d = h->d, hh = h->h, L = h->L, kvd = h->kvd, V = h->V;
    int rc;
    if ((rc = make_q8(h, h->qE, h->E, V, (int)d)) || (rc = make_q8(h, h->qWqkv, h->Wqkv, L * (d + 2 * kvd), (int)d)) ||
        (rc = make_q8(h, h->qWo, h->Wo, L * d, (int)d)) || (rc = make_q8(h, h->qW13, h->W13, L * 2 * hh, (int)d)) ||
        (rc = make_q8(h, h->qW2, h->W2, L * d, (int)hh))) {
        h->gs = 0;
        return rc;
    }
    if (h->shared) h->qWcls = h->qE;
    else if ((rc = make_q8(h, h->qWcls, h->Wcls, V, (int)d))) {
        h->gs = 0;
        return rc;
    }
    CK(cudaStreamSynchronize(h->stream));
    return L2C_OK;
}

// ---------------------------------------------------------------- Q4_0 set --

// Q4_0 records of an fp32 matrix [rows][K]: packed (the GEMV weights) or, for
// the embedding table, the Q8_0 record layout holding the 4-bit codes.
static int make_q4(l2c_ctx* h, Q8Mat& m, const float* W, size_t rows, int K, bool wide) {
    m.rb = wide ? record_bytes(K, h->gs4) : q4_record_bytes(K, h->gs4);
    int rc = dalloc(h, (void**)&m.p, rows * m.rb);
    if (rc) return rc;
    CK(cudaMemsetAsync(m.p, 0, rows * m.rb, h->stream));
    long long groups = (long long)rows * (K / h->gs4);  // warp tasks: at most one per group
    long long blocks = (groups + 7) / 8;
    int grid = (int)(blocks < 65535LL * 16 ? blocks : 65535LL * 16);
    // mode: 1 the Q8_0 layout (embedding); 2 the 64-value chunk layout; 0 the 32-value one
    const int mode = wide ? 1 : (K % 64 == 0 ? 2 : 0);
    k_quantize_rows_q4<<<grid, 256, 0, h->stream>>>(W, (long long)rows, K, h->gs4, m.p, m.rb, mode);
    CK(cudaGetLastError());
    return L2C_OK;
}

extern "C" int l2c_enable_q40(l2c_ctx* h, int gs) {
    if (!h) return L2C_E_ARG;
    if (h->gs4) return h->gs4 == gs ? L2C_OK : fail(h, L2C_E_STATE, "Q4_0 already enabled with gs=%d", h->gs4);
    if ((gs != 32 && gs != 64 && gs != 128) || h->d % gs || h->h % gs)
        return fail(h, L2C_E_ARG, "Q4_0: gs=%d must be 32, 64 or 128 and divide dim and hidden_dim", gs);
    if ((h->d + 2 * h->kvd) % 4 || h->V % 2)  // the 4-bit GEMV takes rows 4 (q/k/v) or 2 (classifier) at a time
        return fail(h, L2C_E_ARG, "Q4_0: dim + 2 * kv_dim must be a multiple of 4 and vocab_size even");
    h->gs4 = gs;
    const size_t d = h->d, hh = h->h, L = h->L, kvd = h->kvd, V = h->V;
    int rc;
    if ((rc = make_q4(h, h->q4E, h->E, V, (int)d, true)) ||
        (rc = make_q4(h, h->q4Wqkv, h->Wqkv, L * (d + 2 * kvd), (int)d, false)) ||
        (rc = make_q4(h, h->q4Wo, h->Wo, L * d, (int)d, false)) ||
        (rc = make_q4(h, h->q4W13, h->W13, L * 2 * hh, (int)d, false)) ||
        (rc = make_q4(h, h->q4W2, h->W2, L * d, (int)hh, false)) ||
        (rc = make_q4(h, h->q4Wcls, h->Wcls, V, (int)d, false))) {
        h->gs4 = 0;
        return rc;
    }
    CK(cudaStreamSynchronize(h->stream));
    return L2C_OK;
}

// ------------------------------------------------------------------ forward --

// Whether the weights of format wf are made, and the int8 KV cache (which
// serves the quantized steps) allows the step; 0 if so, else the failure code.
static int step_ready(l2c_ctx* h, int wf) {
    if (wf == WF_Q80 && !h->gs) return fail(h, L2C_E_STATE, "Q8_0 weights not made (l2c_enable_q80)");
    if (wf == WF_Q40 && !h->gs4) return fail(h, L2C_E_STATE, "Q4_0 weights not made (l2c_enable_q40)");
    if (wf == WF_F32 && h->kv8) return fail(h, L2C_E_STATE, "the int8 KV cache serves the quantized steps");
    return L2C_OK;
}

static const float* forward_impl(l2c_ctx* h, int token, int pos, int wf) {
    if (!h) return nullptr;
    if (token < 0 || token >= h->V) { fail(h, L2C_E_ARG, "token %d not in [0,%d)", token, h->V); return nullptr; }
    if (pos < 0 || pos >= h->S) { fail(h, L2C_E_ARG, "pos %d not in [0,%d)", pos, h->S); return nullptr; }
    if (step_ready(h, wf) != L2C_OK) return nullptr;
    if (h->graphs && build_graph(h, wf, false) != L2C_OK) return nullptr;
    k_set_tp<<<1, 1, 0, h->stream>>>(h->tp, token, pos);
    cudaError_t e = cudaSuccess;
    if (h->graphs) {
        e = cudaGraphLaunch(h->graph[wf][0], h->stream);
    } else {
        cudaStream_t saved = h->cap;
        h->cap = h->stream;
        int rc = enqueue_step(h, wf);
        h->cap = saved;
        if (rc != L2C_OK) return nullptr;
    }
    if (e != cudaSuccess) { fail(h, L2C_E_CUDA, "graph launch: %s", cudaGetErrorString(e)); return nullptr; }
    return h->logits;
}

extern "C" const float* l2c_forward(l2c_ctx* h, int token, int pos) { return forward_impl(h, token, pos, WF_F32); }
extern "C" const float* l2c_forward_q80(l2c_ctx* h, int token, int pos) { return forward_impl(h, token, pos, WF_Q80); }
extern "C" const float* l2c_forward_q40(l2c_ctx* h, int token, int pos) { return forward_impl(h, token, pos, WF_Q40); }

extern "C" int l2c_generate(l2c_ctx* h, int token0, int pos0, int steps, int q80, int32_t* tokens_out) {
    if (!h || !tokens_out || steps < 0) return L2C_E_ARG;
    if (q80 < WF_F32 || q80 > WF_Q40) return fail(h, L2C_E_ARG, "generate: weight format %d not in {0,1,2}", q80);
    if (token0 < 0 || token0 >= h->V) return fail(h, L2C_E_ARG, "token %d not in [0,%d)", token0, h->V);
    if (pos0 < 0 || pos0 + steps > h->S) return fail(h, L2C_E_ARG, "pos0 + steps exceeds seq_len");
    int rc = step_ready(h, q80);
    if (rc) return rc;
    if (steps == 0) return L2C_OK;
    rc = build_graph(h, q80, true);
    if (rc) return rc;
    k_set_tp<<<1, 1, 0, h->stream>>>(h->tp, token0, pos0);
    CK(cudaMemsetAsync(h->gen_count, 0, 4, h->stream));
    for (int t = 0; t < steps; t++) CK(cudaGraphLaunch(h->graph[q80][1], h->stream));
    CK(cudaMemcpyAsync(tokens_out, h->gen_tokens, (size_t)steps * 4, cudaMemcpyDeviceToHost, h->stream));
    return l2c_sync(h);
}

extern "C" int l2c_forward_batch(l2c_ctx* h, int B, const int32_t* tokens, const int32_t* pos, int q80,
                                 float* logits_out) {
    if (!h || !tokens || !pos || !logits_out || B < 1 || B > h->max_batch)
        return fail(h, L2C_E_ARG, "forward_batch: need 1 <= B <= max_batch and non-null arrays");
    if (q80 < 0 || q80 > 1) return fail(h, L2C_E_ARG, "forward_batch: q80 must be 0 or 1 (Q4_0 serves the single-sequence step)");
    if (q80 && !h->gs) return fail(h, L2C_E_STATE, "Q8_0 weights not made (l2c_enable_q80)");
    if (B > BMAX) return fail(h, L2C_E_ARG, "forward_batch: the batched step takes at most %d sequences", BMAX);
    if (h->kv8) return fail(h, L2C_E_STATE, "forward_batch: not with the int8 KV cache (l2c_enable_kv8)");
    const bool tok_dev = is_device_ptr(tokens), pos_dev = is_device_ptr(pos);
    if (!tok_dev && !pos_dev) {
        for (int b = 0; b < B; b++) {
            if (tokens[b] < 0 || tokens[b] >= h->V) return fail(h, L2C_E_ARG, "token[%d]=%d out of range", b, tokens[b]);
            if (pos[b] < 0 || pos[b] >= h->S) return fail(h, L2C_E_ARG, "pos[%d]=%d out of range", b, pos[b]);
        }
    }
    // (token, pos) pairs into the device words the kernels read; device-side
    // checks flag out-of-range values passed in device memory
    CK(cudaMemcpy2DAsync(h->tp, 8, tokens, 4, 4, (size_t)B,
                         tok_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice, h->stream));
    CK(cudaMemcpy2DAsync(h->tp + 1, 8, pos, 4, 4, (size_t)B,
                         pos_dev ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice, h->stream));
    int rc;
    if (q80) {
        if (batched_kc(h->d, h->gs) == 0 || batched_kc(h->h, h->gs) == 0 || h->gs % 32)
            return fail(h, L2C_E_ARG, "batched Q8_0 step needs gs a multiple of 32 and widths it tiles");
        if ((rc = ensure_batched(h))) return rc;
    } else if ((rc = ensure_batched_f32(h))) {
        return rc;
    }
    if (h->graphs) {
        if ((rc = build_batch_graph(h, B, q80 != 0))) return rc;
        CK(cudaGraphLaunch((q80 ? h->bgraph : h->bgraph_f32)[B], h->stream));
    } else if ((rc = enqueue_batch_step(h, h->stream, B, h->bb, q80 != 0, false))) {
        return rc;
    }
    CK(cudaMemcpyAsync(logits_out, h->logits, (size_t)B * h->V * 4, cudaMemcpyDeviceToDevice, h->stream));
    return L2C_OK;
}

extern "C" int l2c_prefill(l2c_ctx* h, int seq, int n, const int32_t* tokens, int pos0, int q80,
                           float* logits_last) {
    if (!h || !tokens || n < 1 || seq < 0 || seq >= h->max_batch || pos0 < 0 || (long long)pos0 + n > h->S)
        return fail(h, L2C_E_ARG, "prefill: need n >= 1, a sequence of the handle and pos0 + n <= seq_len");
    if (is_device_ptr(tokens)) return fail(h, L2C_E_ARG, "prefill: tokens must be host memory");
    for (int i = 0; i < n; i++)
        if (tokens[i] < 0 || tokens[i] >= h->V) return fail(h, L2C_E_ARG, "token[%d]=%d out of range", i, tokens[i]);
    if (q80 < 0 || q80 > 1) return fail(h, L2C_E_ARG, "prefill: q80 must be 0 or 1 (Q4_0 serves the single-sequence step)");
    if (q80 && !h->gs) return fail(h, L2C_E_STATE, "Q8_0 weights not made (l2c_enable_q80)");
    if (h->kv8) return fail(h, L2C_E_STATE, "prefill: not with the int8 KV cache (l2c_enable_kv8)");
    int rc;
    if (q80) {
        if (batched_kc(h->d, h->gs) == 0 || batched_kc(h->h, h->gs) == 0 || h->gs % 32)
            return fail(h, L2C_E_ARG, "Q8_0 prefill needs gs a multiple of 32 and widths the batched GEMM tiles");
        if ((rc = ensure_batched(h))) return rc;
    } else if ((rc = ensure_batched_f32(h))) {
        return rc;
    }
    if ((rc = ensure_prefill(h))) return rc;
    BatchBufs bb = h->pb;
    bb.cache_off = (size_t)seq * h->L * h->S * h->kvd;
    bb.seq_stride = 0;  // one cache: every token of a chunk reads and writes sequence seq's
    int tp[2 * BMAX];
    int last = 0;
    for (int c0 = 0; c0 < n; c0 += BMAX) {
        const int B = n - c0 < BMAX ? n - c0 : BMAX;
        for (int i = 0; i < B; i++) {
            tp[2 * i] = tokens[c0 + i];
            tp[2 * i + 1] = pos0 + c0 + i;
        }
        // a copy, not a kernel: the chunk's kernels start after every earlier
        // kernel has finished, so rows of earlier chunks are complete
        CK(cudaMemcpyAsync(bb.tp, tp, (size_t)B * 8, cudaMemcpyHostToDevice, h->stream));
        if ((rc = enqueue_batch_step(h, h->stream, B, bb, q80 != 0, true))) return rc;
        last = B - 1;
    }
    if (logits_last)
        CK(cudaMemcpyAsync(logits_last, bb.logits + (size_t)last * h->V, (size_t)h->V * 4, cudaMemcpyDeviceToDevice,
                           h->stream));
    return l2c_sync(h);
}

extern "C" int l2c_attention(l2c_ctx* h, const float* q, const float* k, const float* v, int pos, int precision,
                             float* out) {
    if (!h || !q || !k || !v || !out || pos < 0 || pos >= h->S || (precision != 0 && precision != 1))
        return fail(h, L2C_E_ARG, "attention: need pos in [0, seq_len) and precision 0 or 1");
    if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)out) & 15)
        return fail(h, L2C_E_ARG, "attention: buffers must be 16-byte aligned");
    k_set_tp<<<1, 1, 0, h->stream>>>(h->tp, 0, pos);
    CK(launch_attention(h, h->stream, false, precision != 0, q, k, v, 0, out, h->tp, 1, h->attn_part, h->attn_cnt));
    return L2C_OK;
}

extern "C" int l2c_time_kernel(l2c_ctx* h, int kind, int q80, int iters, float* avg_ms) {
    if (!h || kind < SK_QKV || kind > SK_CLS || iters < 1 || !avg_ms || q80 < WF_F32 || q80 > WF_Q40)
        return fail(h, L2C_E_ARG, "time_kernel: bad arguments");
    if (q80 == WF_Q80 && !h->gs) return fail(h, L2C_E_STATE, "Q8_0 weights not made (l2c_enable_q80)");
    if (q80 == WF_Q40 && !h->gs4) return fail(h, L2C_E_STATE, "Q4_0 weights not made (l2c_enable_q40)");
    cudaEvent_t e0, e1;
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));
    int rc = L2C_OK;
    cudaError_t er = cudaEventRecord(e0, h->stream);
    for (int i = 0; i < iters && rc == L2C_OK && er == cudaSuccess; i++) {
        rc = launch_step_kernel(h, h->stream, kind, q80, kind == SK_CLS ? 0 : i % h->L);
    }
    if (er == cudaSuccess) er = cudaEventRecord(e1, h->stream);
    if (er == cudaSuccess) er = cudaEventSynchronize(e1);
    float ms = 0.f;
    if (er == cudaSuccess) er = cudaEventElapsedTime(&ms, e0, e1);
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    if (rc != L2C_OK) return rc;
    if (er != cudaSuccess) return fail(h, L2C_E_CUDA, "time_kernel: %s", cudaGetErrorString(er));
    *avg_ms = ms / (float)iters;
    return l2c_sync(h);
}

// ------------------------------------------------------------------- misc --

extern "C" int l2c_argmax(l2c_ctx* h, const float* logits, int n, int* out_idx) {
    if (!h || !logits || n <= 0 || !out_idx) return L2C_E_ARG;
    CK(cudaMemsetAsync(h->key_scratch, 0, 8, h->stream));
    int grid = (n + 1023) / 1024;
    if (grid > h->sms) grid = h->sms;
    k_argmax<<<grid, 256, 0, h->stream>>>(logits, n, h->key_scratch, h->err);
    k_argmax_index<<<1, 1, 0, h->stream>>>(h->key_scratch, h->idx_out);
    CK(cudaGetLastError());
    int rc = l2c_sync(h);
    if (rc) return rc;
    CK(cudaMemcpy(out_idx, h->idx_out, 4, cudaMemcpyDeviceToHost));
    return L2C_OK;
}

extern "C" int l2c_sample(l2c_ctx* h, const float* logits, int n, float temperature, float topp, double coin,
                          int* out_idx) {
    if (!h || !logits || n <= 0 || !out_idx || !(temperature >= 0.0f) || !(topp > 0.0f) ||
        !(coin >= 0.0 && coin < 1.0))
        return fail(h, L2C_E_ARG, "sample: need n > 0, temperature >= 0, topp > 0 and a coin in [0, 1)");
    if (temperature == 0.0f) return l2c_argmax(h, logits, n, out_idx);
    if (h->sample_n < (size_t)n) {
        int rc;
        if ((rc = dalloc(h, (void**)&h->sample_q, (size_t)n * sizeof(double))) != L2C_OK) return rc;
        h->sample_n = (size_t)n;
    }
    k_sample<<<1, SAMPLE_THREADS, 0, h->stream>>>(logits, n, temperature, topp, coin, nullptr, h->sample_q, h->idx_out,
                                                  h->err);
    CK(cudaGetLastError());
    int rc = l2c_sync(h);
    if (rc) return rc;
    CK(cudaMemcpy(out_idx, h->idx_out, 4, cudaMemcpyDeviceToHost));
    return L2C_OK;
}

extern "C" int l2c_quantize_q80(l2c_ctx* h, const float* x, int64_t n, int gs, int8_t* q, float* s) {
    if (!h || !x || !q || !s || n < 0 || gs < 1 || gs > 1024 || n % gs)
        return fail(h, L2C_E_ARG, "quantize: need n %% gs == 0 and 1 <= gs <= 1024");
    if (n == 0) return L2C_OK;
    long long groups = n / gs;
    long long blocks = (groups + 7) / 8;
    int grid = (int)(blocks < 65535LL * 16 ? blocks : 65535LL * 16);
    k_quantize<<<grid, 256, 0, h->stream>>>(x, groups, gs, q, s);
    CK(cudaGetLastError());
    return L2C_OK;
}

extern "C" int l2c_q80_group_dots(l2c_ctx* h, const int8_t* qw, const int8_t* qx, int rows, int K, int gs,
                                  int32_t* out) {
    if (!h || !qw || !qx || !out || rows < 0 || K <= 0 || gs < 16 || gs > 512 || gs % 16 || K % gs)
        return fail(h, L2C_E_ARG, "group_dots: need K %% gs == 0 and gs a multiple of 16 in [16,512]");
    if (rows == 0) return L2C_OK;
    const bool hot = K % 64 == 0 && K <= 32768 && (gs == 32 || gs == 64 || gs == 128) &&
                     ((uintptr_t)qw & 15) == 0 && ((uintptr_t)qx & 15) == 0;
    const dim3 grid((rows + 7) / 8), block(256);
    if (hot && gs == 32) k_group_dots64<32><<<grid, block, (size_t)K, h->stream>>>(qw, qx, rows, K, out);
    else if (hot && gs == 64) k_group_dots64<64><<<grid, block, (size_t)K, h->stream>>>(qw, qx, rows, K, out);
    else if (hot && gs == 128) k_group_dots64<128><<<grid, block, (size_t)K, h->stream>>>(qw, qx, rows, K, out);
    else k_group_dots<<<grid, block, 0, h->stream>>>(qw, qx, rows, K, gs, out);
    CK(cudaGetLastError());
    return L2C_OK;
}

extern "C" int l2c_kv_load(l2c_ctx* h, int seq, int n_pos, const float* k, const float* v) {
    if (!h || seq < 0 || seq >= h->max_batch || n_pos < 0 || n_pos > h->S || (!k && !v))
        return fail(h, L2C_E_ARG, "kv_load: bad sequence or n_pos");
    if (n_pos == 0) return L2C_OK;
    const size_t kvd = h->kvd, S = h->S, L = h->L;
    const size_t base = (size_t)seq * L * S * kvd;
    const cudaMemcpyKind kk = k && is_device_ptr(k) ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    const cudaMemcpyKind kv = v && is_device_ptr(v) ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
    for (size_t l = 0; l < L; l++) {
        if (k) CK(cudaMemcpyAsync(h->kc + base + l * S * kvd, k + l * n_pos * kvd, n_pos * kvd * 4, kk, h->stream));
        if (v) CK(cudaMemcpyAsync(h->vc + base + l * S * kvd, v + l * n_pos * kvd, n_pos * kvd * 4, kv, h->stream));
        if (h->kv8) {  // the loaded rows into the int8 cache (both K and V, as a step stores them)
            Kv8Args k8 = kv8_args(h, h->kc + base + l * S * kvd, h->vc + base + l * S * kvd);
            k_kv8_rows<<<dim3((unsigned)n_pos, 2 * h->Hkv), 32, 0, h->stream>>>(k8);
            CK(cudaGetLastError());
        }
    }
    CK(cudaStreamSynchronize(h->stream));
    return L2C_OK;
}

extern "C" int l2c_enable_kv8(l2c_ctx* h, int on) {
    if (!h) return L2C_E_ARG;
    if (on && (h->hs % 4 || h->hs > 128 || !attn_kernel_kv8(h->hs, h->rep)))
        return fail(h, L2C_E_ARG, "int8 KV cache: head size %d / GQA ratio %d not built", h->hs, h->rep);
    if ((bool)on == h->kv8) return L2C_OK;
    int rc;
    if (on && !h->kq8) {
        const size_t rows = (size_t)h->max_batch * h->L * h->S;
        if ((rc = dalloc(h, (void**)&h->kq8, rows * h->kvd)) != L2C_OK) return rc;
        if ((rc = dalloc(h, (void**)&h->vq8, rows * h->kvd)) != L2C_OK) return rc;
        if ((rc = dalloc(h, (void**)&h->ks8, rows * h->Hkv * 4)) != L2C_OK) return rc;
        if ((rc = dalloc(h, (void**)&h->vs8, rows * h->Hkv * 4)) != L2C_OK) return rc;
    }
    if (on) {  // every row already in the cache into the int8 cache
        const size_t rows = (size_t)h->max_batch * h->L * h->S;
        for (size_t r0 = 0; r0 < rows; r0 += 65535) {
            const size_t n = rows - r0 < 65535 ? rows - r0 : 65535;
            Kv8Args k8 = kv8_args(h, h->kc + r0 * h->kvd, h->vc + r0 * h->kvd);
            k_kv8_rows<<<dim3((unsigned)n, 2 * h->Hkv), 32, 0, h->stream>>>(k8);
            CK(cudaGetLastError());
        }
    }
    // the step graphs were captured for the other cache
    for (int a = 0; a < 3; a++)
        for (int b = 0; b < 2; b++)
            if (h->graph[a][b]) {
                cudaGraphExecDestroy(h->graph[a][b]);
                h->graph[a][b] = nullptr;
            }
    h->kv8 = on != 0;
    return l2c_sync(h);
}

extern "C" int l2c_kv_read(l2c_ctx* h, int seq, int n_pos, float* k, float* v) {
    if (!h || seq < 0 || seq >= h->max_batch || n_pos < 0 || n_pos > h->S)
        return fail(h, L2C_E_ARG, "kv_read: bad sequence or n_pos");
    const size_t kvd = h->kvd, S = h->S, L = h->L;
    const size_t base = (size_t)seq * L * S * kvd;
    for (size_t l = 0; l < L && n_pos > 0; l++) {
        if (k) CK(cudaMemcpyAsync(k + l * n_pos * kvd, h->kc + base + l * S * kvd, n_pos * kvd * 4,
                                  cudaMemcpyDeviceToHost, h->stream));
        if (v) CK(cudaMemcpyAsync(v + l * n_pos * kvd, h->vc + base + l * S * kvd, n_pos * kvd * 4,
                                  cudaMemcpyDeviceToHost, h->stream));
    }
    return l2c_sync(h);
}

extern "C" int l2c_kv_reset(l2c_ctx* h, int seq) {
    if (!h || seq < -1 || seq >= h->max_batch) return fail(h, L2C_E_ARG, "kv_reset: bad sequence");
    const size_t n = (size_t)h->L * h->S * h->kvd;
    const size_t s0 = seq < 0 ? 0 : (size_t)seq, ns = seq < 0 ? (size_t)h->max_batch : 1;
    CK(cudaMemsetAsync(h->kc + s0 * n, 0, n * ns * 4, h->stream));
    CK(cudaMemsetAsync(h->vc + s0 * n, 0, n * ns * 4, h->stream));
    if (h->kq8) {  // codes 0, scales 0: the int8 cache reads 0 as well
        const size_t nsc = n / h->hs;
        CK(cudaMemsetAsync(h->kq8 + s0 * n, 0, n * ns, h->stream));
        CK(cudaMemsetAsync(h->vq8 + s0 * n, 0, n * ns, h->stream));
        CK(cudaMemsetAsync(h->ks8 + s0 * nsc, 0, nsc * ns * 4, h->stream));
        CK(cudaMemsetAsync(h->vs8 + s0 * nsc, 0, nsc * ns * 4, h->stream));
    }
    return L2C_OK;
}

extern "C" int l2c_sync(l2c_ctx* h) {
    if (!h) return L2C_E_ARG;
    CK(cudaStreamSynchronize(h->stream));
    int e = 0;
    CK(cudaMemcpy(&e, h->err, 4, cudaMemcpyDeviceToHost));
    if (e) {
        CK(cudaMemset(h->err, 0, 4));
        if (e & DERR_TIMEOUT) {  // an abandoned step can leave barriers and counters mid-way
            CK(cudaMemset(h->attn_cnt, 0, (size_t)h->max_batch * h->Hkv * 4));
        }
        return fail(h, L2C_E_DEVICE, "device error word 0x%x:%s%s%s%s", e, (e & DERR_TOKEN) ? " token" : "",
                    (e & DERR_POS) ? " pos" : "", (e & DERR_TIMEOUT) ? " wait-timeout" : "",
                    (e & DERR_NAN) ? " nan" : "");
    }
    return L2C_OK;
}

extern "C" void* l2c_stream(l2c_ctx* h) { return h ? (void*)h->stream : nullptr; }

extern "C" int l2c_last_status(l2c_ctx* h) { return h ? h->status : L2C_E_ARG; }

extern "C" int l2c_last_error(l2c_ctx* h, char* buf, int len) {
    if (!h) return 0;
    int n = (int)strlen(h->msg);
    if (buf && len > 0) {
        strncpy(buf, h->msg, (size_t)len - 1);
        buf[len - 1] = 0;
    }
    return n;
}

extern "C" void l2c_destroy(l2c_ctx* h) {
    if (!h) return;
    if (h->stream || h->cap) cudaDeviceSynchronize();
    for (int a = 0; a < 2; a++)
        for (int b = 0; b < 2; b++)
            if (h->graph[a][b]) cudaGraphExecDestroy(h->graph[a][b]);
    for (cudaGraphExec_t g : h->bgraph_f32)
        if (g) cudaGraphExecDestroy(g);
    for (cudaGraphExec_t g : h->bgraph)
        if (g) cudaGraphExecDestroy(g);
    for (void* p : h->allocs) cudaFree(p);
    if (h->cap) cudaStreamDestroy(h->cap);
    delete h;
}
