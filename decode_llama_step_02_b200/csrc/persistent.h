// persistent.h - host interface of the persistent Q8_0 decode-step kernel.
//
// One launch runs a whole single-sequence Q8_0 decode step (every layer and
// the classifier) on one CTA per SM.  Declarations only; the kernel and its
// launch helpers live in persistent.cu.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace l2c {

// Everything one step reads and writes.  Q8_0 matrices are row records
// [K int8 codes | K/gs fp32 scales | pad to 16 B]; rb_d and rb_h are the
// record sizes of rows of width dim and hidden_dim.
struct PStepArgs {
    const uint8_t* Wqkv;  // [L][dim + 2 kv_dim] records (Wq; Wk; Wv rows)
    const uint8_t* Wo;    // [L][dim]
    const uint8_t* W13;   // [L][2 hidden]: row 2i = W1 row i, row 2i+1 = W3 row i
    const uint8_t* W2;    // [L][dim], records of width hidden
    const uint8_t* Wcls;  // [vocab]
    const uint8_t* E;     // [vocab] token embedding records
    size_t rb_d, rb_h;
    const float* rms_att;    // [L][dim]
    const float* rms_ffn;    // [L][dim]
    const float* rms_final;  // [dim]
    const float* freq;       // RoPE pair frequencies [hs/2]
    float* x;                // residual stream [dim]
    float* q;                // [dim]
    float* att;              // attention output [dim]
    float* hb;               // [hidden]
    float* logits;           // [vocab]
    float* kc;               // key cache of the sequence [L][seq_len][kv_dim]
    float* vc;               // value cache
    int d, hdim, L, H, Hkv, hs, kvd, V, S, gs;
    const int* tp;               // {token, pos}
    unsigned long long* amax;    // argmax key of the logits
    int* err;                    // device error word
    int* abort_flag;             // set when a bounded wait gives up; every wait then returns
    unsigned* bar;               // {barrier arrivals, CTAs finished}: zero before a launch, left zero
    void* part;                  // attention partials [Hkv][nchunks][rep][hs + 2] doubles
    int* count;                  // [Hkv] attention arrival counters (zero between uses)
    int nchunks;                 // attention chunks per KV head
    uint32_t ring_bytes;         // weight ring size in shared memory
    uint64_t pf_bytes;           // how far (bytes per CTA) L2 prefetches run ahead of the ring copies
};

// Byte offsets inside the kernel's dynamic shared memory.
struct PLayout {
    uint32_t ring, xq, xsc, sxd, meta, vstart, full, empty, attn, total;
};

#ifndef L2C_PS_PRODUCERS
#define L2C_PS_PRODUCERS 4
#endif
constexpr int PS_CONSUMERS = 8;                   // consumer warps
constexpr int PS_PRODUCERS = L2C_PS_PRODUCERS;    // producer warps, each with its own slice of the ring
constexpr int PS_THREADS = 32 * (PS_CONSUMERS + PS_PRODUCERS);
constexpr int PS_SLOTS = 64;                      // ring units in flight at most (all producers)
constexpr int PS_UNIT = 4;                        // rows per unit of the dim-wide matrices
constexpr int PS_PSLOTS = PS_SLOTS / PS_PRODUCERS;  // per producer

// The kernel for head size hs and GQA ratio rep, or nullptr if there is none.
const void* pstep_kernel(int hs, int rep);

// Dynamic shared memory of the kernel apart from the ring (input codes and
// scales for rows of width up to kmax, ring bookkeeping, attention work space).
PLayout pstep_layout(uint32_t ring_bytes, int kmax, int gs, int hs, int rep);

// Static shared memory of a kernel returned by pstep_kernel.
cudaError_t pstep_static_smem(const void* kern, size_t* bytes);

// Cooperative launch of `grid` CTAs (all resident at once) on stream s.
cudaError_t pstep_launch(const void* kern, int grid, const PStepArgs& a, const PLayout& L, cudaStream_t s);

}  // namespace l2c
