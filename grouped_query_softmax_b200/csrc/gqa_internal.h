// Internal interface between the C ABI (gqa_api.cpp) and the kernel translation
// unit (gqa_kernels.cu). Not installed, not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gqa {

struct FwdLaunch {
    CUtensorMap tm_q, tm_k, tm_v;
    int B, Hq, Hkv, Tq, Tk, D;
    int window;  // 0: causal; > 0: sliding window of that many positions
    float scale;
    void* o;
    float* lse;
};

struct DecLaunch {
    CUtensorMap tm_k, tm_v;
    int B, Hq, Hkv, Tq, Tk, D;
    int window;
    int splits, blk_per_split, blk_first, n_blk;
    float scale;
    const void* q;
    void* o;
    float* ws_o;
    float* ws_lse;
};

// Each returns cudaSuccess or the launch error; nothing is synchronised.
cudaError_t launch_fwd(const FwdLaunch& a, cudaStream_t stream);
cudaError_t launch_decode(const DecLaunch& a, cudaStream_t stream);
cudaError_t launch_selftest_wait(unsigned long long timeout_ns, cudaStream_t stream);

// Read and clear the device error word of the current device (after a stream sync).
cudaError_t read_and_clear_device_error(uint32_t* value);

// Bound on every device-side wait of the production kernels.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

// Rows per fwd sub-tile and keys per tile, shared with the host planner.
constexpr int kTileRows = 128;
constexpr int kTileKeys = 128;

}  // namespace gqa
