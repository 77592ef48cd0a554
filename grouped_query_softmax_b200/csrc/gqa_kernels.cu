// Kernel translation unit: every device kernel of libgqa and its launcher.
// Keeping them in one unit lets them share one device error word without
// relocatable device code.
#include <cuda_runtime.h>

#include <algorithm>

#include "bwd_sm100.cuh"
#include "decode_sm100.cuh"
#include "fwd_sm100.cuh"
#include "gqa_internal.h"

namespace gqa {

// Bit flags (kDevErr*) set by the kernels; see gqa_get_device_error().
static_assert(kDevErrWaitTimeout == kErrBitWaitTimeout && kDevErrBadSeqlens == kErrBitBadSeqlens,
              "device and host disagree on the error bits");
__device__ uint32_t g_device_error = 0;

static uint32_t* device_error_ptr() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    return static_cast<uint32_t*>(p);
}

template <int D>
static cudaError_t launch_fwd_d(const FwdLaunch& a, cudaStream_t stream) {
    FwdParams p{};
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Tq = a.Tq;
    p.Tk = a.Tk;
    p.G = a.Hq / a.Hkv;
    p.n_qt = (a.Tq + kFwdRows - 1) / kFwdRows;
    p.unit_flags = (p.G % 2 == 0) ? kUnitPairHeads : 0;
    // A suffix at least as long as its prefix has row levels of similar length, so units go
    // head by head: the levels of one head then read its K/V from L2 rather than from HBM
    // once per level (the K/V of all heads can exceed L2, as with many MHA heads)
    if (a.Tk - a.Tq >= a.Tq) p.unit_flags |= kUnitHeadMajor;
    long long units;
    if (p.unit_flags & kUnitPairHeads) {
        p.per_level = a.B * a.Hkv * (p.G / 2);
        units = (long long)p.per_level * p.n_qt;
    } else {
        p.per_level = a.B * a.Hq;
        units = (long long)p.per_level * ((p.n_qt + 1) / 2);
    }
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.window = a.window;
    p.o = static_cast<__nv_bfloat16*>(a.o);
    p.lse = a.lse;
    p.err = device_error_ptr();
    p.timeout_ns = kWaitTimeoutNs;
    if (!p.err) return cudaErrorUnknown;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    FwdSplitPlan sp;
    p.split_slices = 0;
    p.split_whole = 0;
    p.split_group = 1;
    if (a.split_slices > 0) {
        // the caller sized its workspace with the same plan on the same device
        sp = fwd_split_plan(a.B, a.Hq, a.Hkv, a.Tq, a.Tk, a.window, sms);
        if (sp.slices != a.split_slices || !a.part || units != sp.whole + sp.split) return cudaErrorInvalidValue;
        p.split_whole = (int)sp.whole;
        p.split_slices = sp.slices;
        p.split_group = sp.group;
        p.part = a.part;
        p.part_lse = reinterpret_cast<float*>(reinterpret_cast<char*>(a.part) + fwd_split_lse_offset(sp.rows, D));
    }
    if (units <= 0 || units > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.units = (int)units;
    const int smem = FwdSmem<D>::kBytes;
    e = cudaFuncSetAttribute(gqa_fwd_sm100_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // The in-kernel register split (setmaxnreg) needs exactly the launch allocation it
    // was sized for; never launch a build where that does not hold.
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, gqa_fwd_sm100_kernel<D, false>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kFwdLaunchRegs) return cudaErrorInvalidConfiguration;
    // persistent: one CTA per SM (shared memory and TMEM allow exactly one); a split launch
    // has one CTA per SM exactly, as its plan assumes
    const unsigned grid = p.split_slices > 0 ? (unsigned)sms : (unsigned)std::min<long long>(units, sms > 0 ? sms : 1);
    gqa_fwd_sm100_kernel<D, false><<<grid, kFwdThreads, smem, stream>>>(a.tm_q, a.tm_k, a.tm_v, p,
                                                                         FwdVarlenParams{});
    e = cudaGetLastError();
    if (e != cudaSuccess || p.split_slices <= 0) return e;
    // merge the pieces of the split units (stream order makes their partials visible)
    const long long warps = sp.split * 2 * (kFwdRows / 32) * (D / 32);
    const long long blocks = (warps + kCombineWarps - 1) / kCombineWarps;
    gqa_fwd_split_combine_kernel<D><<<(unsigned)blocks, kCombineWarps * 32, 0, stream>>>(p, warps);
    return cudaGetLastError();
}

cudaError_t launch_fwd(const FwdLaunch& a, cudaStream_t stream) {
    return a.D == 128 ? launch_fwd_d<128>(a, stream) : launch_fwd_d<64>(a, stream);
}

template <int D>
static cudaError_t launch_fwd_varlen_d(const FwdVarlenLaunch& a, cudaStream_t stream) {
    FwdParams p{};
    p.B = a.S;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.G = a.Hq / a.Hkv;
    p.unit_flags = (p.G % 2 == 0) ? kUnitPairHeads : 0;
    FwdVarlenParams vp{};
    const long long n_cand = fwd_varlen_candidates(a.S, a.Hq, a.Hkv, a.max_q, &vp.n_lvl, &vp.n_h);
    if (n_cand <= 0 || n_cand > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.window = a.window;
    p.o = static_cast<__nv_bfloat16*>(a.o);
    p.lse = a.lse;
    p.err = device_error_ptr();
    p.timeout_ns = kWaitTimeoutNs;
    if (!p.err) return cudaErrorUnknown;
    vp.cu_q = a.cu_q;
    vp.cu_k = a.cu_k;
    vp.len_q = a.len_q;
    vp.len_k = a.len_k;
    vp.rows_q = a.rows_q;
    vp.rows_k = a.rows_k;
    vp.unit_count = a.ws;
    vp.unit_list = a.ws + kPlanHeaderInts;
    vp.fetch = a.ws + 1;
    vp.dynamic = a.S <= kPlanMaxDynamicSeqs;
    vp.o_sb = a.o_sb;
    vp.o_sh = a.o_sh;
    vp.o_st = a.o_st;
    vp.table = a.table;
    vp.max_pages = a.max_pages;
    vp.page_size = a.page_size;
    vp.box_rows = a.page_size > 0 && a.page_size < kFwdKeys ? a.page_size : kFwdKeys;
    vp.num_pages = a.num_pages;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int smem = FwdSmem<D>::kBytes;
    e = cudaFuncSetAttribute(gqa_fwd_sm100_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, gqa_fwd_sm100_kernel<D, true>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kFwdLaunchRegs) return cudaErrorInvalidConfiguration;
    gqa_fwd_varlen_plan_kernel<<<1, kPlanThreads, 0, stream>>>(p, vp, a.S, a.max_q, n_cand, a.ws);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)std::min<long long>(n_cand, sms > 0 ? sms : 1);
    gqa_fwd_sm100_kernel<D, true><<<grid, kFwdThreads, smem, stream>>>(a.tm_q, a.tm_k, a.tm_v, p, vp);
    return cudaGetLastError();
}

cudaError_t launch_fwd_varlen(const FwdVarlenLaunch& a, cudaStream_t stream) {
    return a.D == 128 ? launch_fwd_varlen_d<128>(a, stream) : launch_fwd_varlen_d<64>(a, stream);
}

static_assert(kPlanHeaderInts * sizeof(int) == kPlanHeaderBytes, "plan workspace header");

template <int D, bool kVarlen>
static cudaError_t launch_decode_d(const DecLaunch& a, cudaStream_t stream) {
    DecParams p{};
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Tq = a.Tq;
    p.Tk = a.Tk;
    p.G = a.Hq / a.Hkv;
    p.n_hc = (p.G * a.Tq + kDecRows - 1) / kDecRows;
    p.splits = a.splits;
    p.blk_per_split = a.blk_per_split;
    p.blk_first = a.blk_first;
    p.n_blk = a.n_blk;
    p.window = a.window;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.q = static_cast<const __nv_bfloat16*>(a.q);
    p.o = static_cast<__nv_bfloat16*>(a.o);
    p.ws_o = a.ws_o;
    p.ws_lse = a.ws_lse;
    p.err = device_error_ptr();
    p.timeout_ns = kWaitTimeoutNs;
    if (!p.err) return cudaErrorUnknown;
    p.seqlens = a.seqlens;
    p.table = a.table;
    p.max_pages = a.max_pages;
    p.page_size = a.page_size;
    p.box_rows = a.page_size > 0 && a.page_size < kDecKeys ? a.page_size : kDecKeys;
    p.num_pages = a.num_pages;
    p.capacity = a.capacity;
    const int smem = DecSmem<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(gqa_decode_sm100_kernel<D, kVarlen>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)a.splits, (unsigned)(a.Hkv * p.n_hc), (unsigned)a.B);
    gqa_decode_sm100_kernel<D, kVarlen><<<grid, kDecThreads, smem, stream>>>(a.tm_k, a.tm_v, p);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.splits == 1) return e;
    const int rows = a.B * a.Hq * a.Tq;
    gqa_decode_combine_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(
        a.ws_o, a.ws_lse, static_cast<__nv_bfloat16*>(a.o), rows, a.splits);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecLaunch& a, cudaStream_t stream) {
    if (a.seqlens != nullptr)
        return a.D == 128 ? launch_decode_d<128, true>(a, stream) : launch_decode_d<64, true>(a, stream);
    return a.D == 128 ? launch_decode_d<128, false>(a, stream) : launch_decode_d<64, false>(a, stream);
}

template <int D, bool kWindow>
static cudaError_t launch_bwd_d(const BwdLaunch& a, cudaStream_t stream) {
    BwdParams p{};
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hkv = a.Hkv;
    p.Tq = a.Tq;
    p.Tk = a.Tk;
    p.G = a.Hq / a.Hkv;
    p.n_kb = (a.Tk + kBwdKeys - 1) / kBwdKeys;
    p.chunk = bwd_chunk(a.B * a.Hkv, p.G, a.Tq, D);
    p.n_qt = (a.Tq + kBwdRows - 1) / kBwdRows;
    p.tq_pad = p.n_qt * kBwdRows;
    p.window = a.window;
    p.scale = a.scale;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.lse2 = a.lse2;
    p.dvec = a.dvec;
    p.dq_acc = a.dq_acc;
    p.dk = static_cast<__nv_bfloat16*>(a.dk);
    p.dv = static_cast<__nv_bfloat16*>(a.dv);
    p.err = device_error_ptr();
    p.timeout_ns = kWaitTimeoutNs;
    if (!p.err) return cudaErrorUnknown;
    const int smem = BwdSmem<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(gqa_bwd_sm100_kernel<D, kWindow>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, gqa_bwd_sm100_kernel<D, kWindow>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kBwdLaunchRegs) return cudaErrorInvalidConfiguration;  // the register split needs it
    const long long rows = (long long)a.B * a.Hq * p.tq_pad;
    constexpr int kPrepRows = 256 / (D / 8);
    gqa_bwd_prep_kernel<D><<<(unsigned)((rows + kPrepRows - 1) / kPrepRows), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.lse, a.lse2, a.dvec,
        a.dq_acc, a.B * a.Hq, a.Tq, p.tq_pad);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const dim3 grid((unsigned)(p.n_kb * a.B * a.Hkv));
    gqa_bwd_sm100_kernel<D, kWindow><<<grid, kBwdThreads, smem, stream>>>(a.tm_q, a.tm_k, a.tm_v, a.tm_do, a.tm_dq, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long n8 = (long long)a.B * a.Hq * a.Tq * a.D / 8;
    gqa_bwd_dq_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, stream>>>(a.dq_acc, static_cast<__nv_bfloat16*>(a.dq),
                                                                        n8);
    return cudaGetLastError();
}

cudaError_t launch_bwd(const BwdLaunch& a, cudaStream_t stream) {
    if (a.window > 0) return a.D == 128 ? launch_bwd_d<128, true>(a, stream) : launch_bwd_d<64, true>(a, stream);
    return a.D == 128 ? launch_bwd_d<128, false>(a, stream) : launch_bwd_d<64, false>(a, stream);
}

// One CTA, one thread: wait on an mbarrier that never completes, bounded by
// timeout_ns, through the same routine the production kernels use.
__global__ void gqa_selftest_wait_kernel(uint32_t* err, unsigned long long timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 never completes: nothing arrives on the barrier
        (void)mbar_wait_bounded(smem_u32(&bar), 0, &abort_flag, err, timeout_ns);
    }
}

cudaError_t launch_selftest_wait(unsigned long long timeout_ns, cudaStream_t stream) {
    uint32_t* err = device_error_ptr();
    if (!err) return cudaErrorUnknown;
    gqa_selftest_wait_kernel<<<1, 32, 0, stream>>>(err, timeout_ns);
    return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(uint32_t* value) {
    uint32_t zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    if (*value) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(uint32_t));
    return e;
}

}  // namespace gqa
