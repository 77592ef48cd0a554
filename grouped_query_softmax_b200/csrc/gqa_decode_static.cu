// gqa_attn_decode_static: decode for callers that cannot allocate device memory.
//
// gqa_attn_decode needs a caller-provided workspace for its split-KV partial
// results. Some callers cannot provide one at call time: for example a plugin whose
// enqueue function runs inside an inference engine that owns every byte of device
// memory, or a latency-critical decode loop that forbids cudaMalloc because it can
// synchronise the device and take an unpredictable amount of time. This entry point
// takes the same arguments minus the workspace and uses a fixed scratch array
// compiled into the library instead. It allocates nothing, ever.
//
// The scratch is one file-scope device array of kStaticScratchBytes. Every GPU on
// which the library is loaded holds it until the process exits. All calls on a
// device share it and it keeps whatever the last call left there; decode writes
// every partial it later reads within the same call, so nothing needs clearing.
// Two calls whose kernels can overlap on the GPU (different streams, or the same
// stream used from several host threads without ordering) race on the scratch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/gqa.h"

namespace {

constexpr size_t kStaticScratchBytes = 16u << 20;  // 16 MiB per device
constexpr int kCacheSlots = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The address of a __device__ array belongs to a CUDA context, not to a device: a
// context created after cudaDeviceReset, or a caller's own (non-primary) context, holds
// its copy elsewhere. Addresses are therefore cached by the ID of the context that was
// current when they were looked up; the driver never gives two contexts of one process
// the same ID, so a cached entry can never be used in another context.
struct ScratchCache {
    std::mutex mutex;
    CtxGetCurrentFn get_current = nullptr;
    CtxGetIdFn get_id = nullptr;
    bool resolved = false;
    unsigned long long ids[kCacheSlots] = {};
    void* addrs[kCacheSlots] = {};
    int used = 0, next = 0;
};
ScratchCache g_cache;

template <class Fn>
Fn driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

// ID of the context current on this thread. When no context is current yet, the
// runtime binds the device's primary context on its next call; the symbol lookup is
// such a call, so it is made first and the context read again.
bool current_context_id(unsigned long long* id) {
    CUcontext ctx = nullptr;
    if (g_cache.get_current(&ctx) != CUDA_SUCCESS) return false;
    if (ctx == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return false;
        if (g_cache.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    }
    return g_cache.get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context. The first call in a
// context (normally once per device: the runtime's primary context) looks it up with
// cudaGetSymbolAddress, since the array's host-side name is only a stand-in, and caches
// it; later calls in that context read the cache.
gqa_status scratch_address(void** out) {
    std::lock_guard<std::mutex> lock(g_cache.mutex);
    if (!g_cache.resolved) {
        g_cache.get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
        g_cache.get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
        g_cache.resolved = true;
    }
    if (!g_cache.get_current || !g_cache.get_id) return GQA_ERR_CUDA;
    unsigned long long id = 0;
    if (!current_context_id(&id)) return GQA_ERR_CUDA;
    for (int i = 0; i < g_cache.used; ++i)
        if (g_cache.ids[i] == id) {
            *out = g_cache.addrs[i];
            return GQA_OK;
        }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return GQA_ERR_CUDA;
    const int slot = g_cache.used < kCacheSlots ? g_cache.used++ : g_cache.next;
    if (g_cache.used == kCacheSlots) g_cache.next = (slot + 1) % kCacheSlots;
    g_cache.ids[slot] = id;
    g_cache.addrs[slot] = p;
    *out = p;
    return GQA_OK;
}

}  // namespace

extern "C" gqa_status gqa_attn_decode_static(const void* q, const void* k_cache,
                                             const void* v_cache, void* o, int B, int Hq, int Hkv,
                                             int Tk, int D, long long k_sb, long long k_sh,
                                             long long v_sb, long long v_sh, float softmax_scale,
                                             int num_splits, void* stream) {
    if (gqa_attn_decode_num_splits(B, Hq, Hkv, Tk, D, num_splits) <= 0)  // invalid sizes:
        return gqa_attn_decode(q, k_cache, v_cache, o, B, Hq, Hkv, Tk, D, k_sb, k_sh, v_sb, v_sh,
                               softmax_scale, num_splits, nullptr, 0, stream);  // reports them
    const size_t need = gqa_attn_decode_workspace_bytes(B, Hq, Hkv, Tk, D, num_splits);
    if (need > kStaticScratchBytes) return GQA_ERR_WORKSPACE;  // problem too large for the fixed scratch
    void* scratch = nullptr;
    const gqa_status st = scratch_address(&scratch);  // one-time set-up on the first call per context
    if (st != GQA_OK) return st;
    return gqa_attn_decode(q, k_cache, v_cache, o, B, Hq, Hkv, Tk, D, k_sb, k_sh, v_sb, v_sh,
                           softmax_scale, num_splits, scratch, kStaticScratchBytes, stream);
}
