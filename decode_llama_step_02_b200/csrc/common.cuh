// common.cuh - device helpers shared by the decode-step kernels (sm_100a).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace l2c {

// ---- device error word (read by the host after a step) --------------------
enum : int {
    DERR_TOKEN = 1,       // token id outside [0, vocab)
    DERR_POS = 2,         // position outside [0, seq_len)
    DERR_TIMEOUT = 4,     // a bounded wait on a shared-memory barrier gave up
    DERR_NAN = 8,         // argmax met a NaN logit
};

__device__ __forceinline__ void set_error(int* err, int code) { atomicOr(err, code); }

// ---- programmatic dependent launch ----------------------------------------
// Everything a kernel reads that an earlier kernel of the step writes must be
// read after grid_dep_wait(); weights may be fetched before it.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

// ---- streaming loads ---------------------------------------------------------
// Weights are read once per step: bypass L1 and mark the L2 lines evict-first
// so that bytes prefetched for the next kernel stay resident.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ float4 ld_stream_f4(const float4* p, uint64_t pol) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.f32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

// L2 prefetch of a contiguous byte range (untiled bulk prefetch, no multicast).
// addr and bytes must be multiples of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void* addr, uint32_t bytes, uint64_t pol) {
    asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;"
                 :: "l"(addr), "r"(bytes), "l"(pol) : "memory");
}

// Prefetch [p, p+bytes) in pieces of at most 64 KB (the instruction takes a
// 32-bit size; smaller pieces also spread over the L2 slices).
__device__ __forceinline__ void prefetch_l2_range(const void* p, size_t bytes, uint64_t pol) {
    const char* c = static_cast<const char*>(p);
    while (bytes >= 16) {
        uint32_t n = bytes > 65536 ? 65536u : (uint32_t)(bytes & ~size_t(15));
        prefetch_l2_bulk(c, n, pol);
        c += n;
        bytes -= n;
    }
}

// ---- shared-memory barriers and bulk copies (1-D TMA, no multicast) ---------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Shared-memory counters handed between warps of a CTA (release / acquire).
__device__ __forceinline__ void st_release_cta(int* p, int v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta(const int* p) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}

// Default limit of every barrier wait (2 s of %globaltimer).
constexpr unsigned long long kWaitNs = 2000000000ull;

// Waits for the barrier phase with the given parity.  Gives up after
// `limit_ns` of wall time (records DERR_TIMEOUT) or, without recording, as
// soon as *abort (a CTA-shared flag, may be null) is set; returns false then.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err,
                                                  unsigned long long limit_ns = kWaitNs,
                                                  volatile int* abort = nullptr) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (abort && *abort) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            set_error(err, DERR_TIMEOUT);
            return false;
        }
    }
}

// Global -> shared bulk copy completing on `bar` (bytes and both addresses are
// multiples of 16).  No multicast: the source is always this GPU's memory.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        :: "r"(smem_u32(dst_smem)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// ---- CTA-wide synchronisation policies ------------------------------------------
// Helpers that a whole group of threads runs together take one of these: the
// full CTA (barrier 0), or the first n threads of the CTA on a named barrier
// (a kernel whose producer warp does not take part).
struct SyncCTA {
    __device__ __forceinline__ void sync() const { __syncthreads(); }
    __device__ __forceinline__ int nthreads() const { return blockDim.x; }
};
struct SyncNamed {
    int id, n;  // barrier 1..15, thread count (a multiple of 32)
    __device__ __forceinline__ void sync() const { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
    __device__ __forceinline__ int nthreads() const { return n; }
    // A barrier that also returns whether any participating thread passed true.
    __device__ __forceinline__ bool sync_or(bool v) const {
        uint32_t r;
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.ne.u32 p, %1, 0;\n\t"
            "bar.red.or.pred q, %2, %3, p;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(r) : "r"((uint32_t)v), "r"(id), "r"(n) : "memory");
        return r != 0;
    }
};

// ---- exact int32 -> double on the FP64 pipe ------------------------------------
// 2^52 + 2^31 + v is a double whose low word is the bits of v + 2^31: build it
// and subtract 2^52 + 2^31 (one DADD, exact).  Same value as the conversion
// instruction, which issues on a narrow unit on this part.
__device__ __forceinline__ double i2d_exact(int v) {
    return __hiloint2double(0x43300000, (int)((unsigned)v ^ 0x80000000u)) - 4503601774854144.0;
}

// ---- reductions --------------------------------------------------------------
template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename T>
__device__ __forceinline__ T warp_max(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Sums each of v[0..N-1] over the warp (N = 1, 2, 4 or 8); lane l ends with
// the total of v[(l / (32 / N)) % N].  A reduce-scatter: at each of the first
// log2(N) steps (offsets 16, 8, ...) a lane keeps half of its values and adds
// its partner's copies of them, then a butterfly finishes; each total comes
// from the same additions in the same order as warp_sum applied to that value
// alone, in 5 shuffle rounds of one value instead of 5 of N.
template <int N, typename T>
__device__ __forceinline__ T warp_sum_scatter(const T (&v)[N]) {
    static_assert(N == 1 || N == 2 || N == 4 || N == 8, "N");
    const int lane = threadIdx.x & 31;
    T w[N];
#pragma unroll
    for (int j = 0; j < N; j++) w[j] = v[j];
    int o = 16;
#pragma unroll
    for (int m = N; m > 1; m >>= 1, o >>= 1) {
        const bool up = lane & o;
#pragma unroll
        for (int j = 0; j < m / 2; j++) {
            const T keep = up ? w[j + m / 2] : w[j];
            const T send = up ? w[j] : w[j + m / 2];
            w[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    T t = w[0];
#pragma unroll
    for (; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    return t;
}

// Block-wide sum; `red` must hold one T per warp.  All threads get the result.
template <typename T>
__device__ __forceinline__ T block_sum(T v, T* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    T s = T(0);
    for (int i = 0; i < nw; i++) s += red[i];
    return s;
}

// ---- argmax key ---------------------------------------------------------------
// Orders floats as unsigned integers; the low word prefers the lowest index on
// ties, so one 64-bit atomicMax yields (max value, first index).
__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
    uint32_t b = __float_as_uint(v);
    uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)ord << 32) | (unsigned long long)(0xffffffffu - (uint32_t)idx);
}

__device__ __forceinline__ int argmax_key_index(unsigned long long k) {
    return (int)(0xffffffffu - (uint32_t)(k & 0xffffffffu));
}

}  // namespace l2c
