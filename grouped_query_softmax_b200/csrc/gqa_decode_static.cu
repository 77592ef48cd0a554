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
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/gqa.h"

namespace {

constexpr size_t kStaticScratchBytes = 16u << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device. The first call on a
// device looks it up with cudaGetSymbolAddress (the host-side name of the array is a
// stand-in, not a device address) and caches it for later calls.
gqa_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return GQA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
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
    const gqa_status st = scratch_address(&scratch);  // one-time set-up on the first call per device
    if (st != GQA_OK) return st;
    return gqa_attn_decode(q, k_cache, v_cache, o, B, Hq, Hkv, Tk, D, k_sb, k_sh, v_sb, v_sh,
                           softmax_scale, num_splits, scratch, kStaticScratchBytes, stream);
}
