// attention_noalloc.cu - grouped-query attention that allocates no memory.
//
// Some callers cannot allocate device memory: their process has handed the
// GPU's memory to another allocator up front (a framework's pool or a serving
// engine that reserves HBM at start-up, where a stray cudaMalloc would fail
// or break the owner's accounting), or they run on a latency-critical path
// where cudaMalloc and cudaFree may synchronize the device.  Such callers also
// cannot create an l2c handle, which owns weights, caches and scratch.  For
// them, l2c_attention_noalloc runs the attention kernel of l2c_attention on
// buffers the caller owns.  The kernel's scratch (partial softmax state per
// KV head and position chunk, arrival counters and the position word) lives
// in a file-scope __device__ array of fixed size instead of a handle's
// allocation.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/l2c.h"
#include "attention.cuh"

using namespace l2c;

namespace {

// The fixed scratch: 4 MiB, held by every GPU that loads the library until
// the process exits.  Layout: [0, 256) the position word, [256, 256 +
// 4*n_kv_heads) arrival counters (rounded up to 256 B), then the partial
// (o, m, l) records of every (KV head, chunk, query head).
constexpr size_t kScratchBytes = size_t(4) << 20;
constexpr int kChunk = 64;      // positions per chunk (the handle picks its own split)
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_attn_scratch[kScratchBytes];

// cuCtxGetCurrent / cuCtxGetId, reached through the runtime's driver entry
// points (the library links no driver library).
typedef int (*CtxGetCurrentFn)(void** ctx);
typedef int (*CtxGetIdFn)(void* ctx, unsigned long long* id);

struct Slot {
    void* addr = nullptr;
    unsigned long long ctx_id = 0;
};

std::mutex g_setup_mutex;
Slot g_slot[kMaxDevices];
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;

int current_context_id(unsigned long long* id) {
    if (!g_ctx_current || !g_ctx_id) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
            return L2C_E_CUDA;
        g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        g_ctx_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    void* ctx = nullptr;
    if (g_ctx_current(&ctx) != 0 || !ctx || g_ctx_id(ctx, id) != 0) return L2C_E_CUDA;
    return L2C_OK;
}

// The device address of g_attn_scratch in the current context.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// (cudaGetSymbolAddress) with the device current, once per device and
// context: a context ID is never reused, so after a device reset (which
// loads the module again, at a new address) the lookup runs again.  The
// attention kernels' shared-memory limit is set at the same time.
int scratch_on_current_device(unsigned char** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return L2C_E_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return L2C_E_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    unsigned long long id = 0;
    if (current_context_id(&id) != L2C_OK) return L2C_E_CUDA;
    Slot& s = g_slot[dev];
    if (!s.addr || s.ctx_id != id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || !p) return L2C_E_CUDA;
        if (attn_set_smem_limits() != cudaSuccess) return L2C_E_CUDA;
        s.addr = p;
        s.ctx_id = id;
    }
    *out = static_cast<unsigned char*>(s.addr);
    return L2C_OK;
}

// Writes the position word and clears the arrival counters (they must start
// at zero; the array keeps whatever the previous call left).
__global__ void k_noalloc_prepare(int* tp, int pos, int* counters, int n) {
    if (threadIdx.x == 0) {
        tp[0] = 0;
        tp[1] = pos;
    }
    for (int i = threadIdx.x; i < n; i += blockDim.x) counters[i] = 0;
}

}  // namespace

extern "C" int l2c_attention_noalloc(const float* q_dev, const float* k_dev, const float* v_dev, int n_heads,
                                     int n_kv_heads, int head_size, int pos, int precision, float* out_dev,
                                     void* cuda_stream) {
    if (!q_dev || !k_dev || !v_dev || !out_dev || n_heads <= 0 || n_kv_heads <= 0 || head_size <= 0 || pos < 0 ||
        n_heads % n_kv_heads || (precision != 0 && precision != 1))
        return L2C_E_ARG;
    if (((uintptr_t)q_dev | (uintptr_t)k_dev | (uintptr_t)v_dev | (uintptr_t)out_dev) & 15) return L2C_E_ARG;
    const int rep = n_heads / n_kv_heads;
    AttnKernel ak = precision ? attn_kernel_for<double>(head_size, rep) : attn_kernel_for<float>(head_size, rep);
    if (!ak) return L2C_E_ARG;
    const int nchunks = pos / kChunk + 1;
    const size_t acc = precision ? sizeof(double) : sizeof(float);
    const size_t cnt_bytes = ((size_t)n_kv_heads * sizeof(int) + 255) & ~size_t(255);
    const size_t part_bytes = (size_t)n_kv_heads * nchunks * rep * (head_size + 2) * acc;
    if (256 + cnt_bytes + part_bytes > kScratchBytes) return L2C_E_SCRATCH;
    unsigned char* scratch = nullptr;
    int rc = scratch_on_current_device(&scratch);
    if (rc != L2C_OK) return rc;
    int* tp = reinterpret_cast<int*>(scratch);
    int* counters = reinterpret_cast<int*>(scratch + 256);
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    k_noalloc_prepare<<<1, 256, 0, s>>>(tp, pos, counters, n_kv_heads);
    if (cudaGetLastError() != cudaSuccess) return L2C_E_CUDA;
    AttnArgs t = {};
    t.q = q_dev; t.kc = k_dev; t.vc = v_dev; t.seq_stride = 0;
    t.out = out_dev; t.tp = tp; t.tp_stride = 2;
    t.H = n_heads; t.Hkv = n_kv_heads; t.hs = head_size; t.kvd = n_kv_heads * head_size; t.seq_len = pos + 1;
    t.nchunks = nchunks;
    t.min_chunk = kChunk;
    t.part = scratch + 256 + cnt_bytes; t.count = counters;
    const int smem = precision ? attn_smem_for<double>(rep) : attn_smem_for<float>(rep);
    const int threads = precision ? attn_threads<double>() : attn_threads<float>();
    ak<<<dim3(nchunks, n_kv_heads, 1), threads, smem, s>>>(t);
    if (cudaGetLastError() != cudaSuccess) return L2C_E_CUDA;
    return L2C_OK;
}
