// C ABI of libgqa (declared in include/gqa.h): argument checks, TMA descriptor
// encoding, split planning and dispatch to the kernel launchers. No device memory is
// allocated here and no state is kept between calls.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <mutex>

#include "../../include/gqa.h"
#include "../../include/gqa_testing.h"
#include "gqa_internal.h"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A [B, H, T, D] bf16 view with free (b, h, t) strides (d contiguous), tiled as boxes of
// box_rows rows x 64 columns (128 bytes) with the 128-byte swizzle. Strides in elements.
gqa_status make_map(CUtensorMap* map, const void* base, int B, int H, int T, int D,
                    long long s_b, long long s_h, long long s_t = -1, int box_rows = gqa::kTileRows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return GQA_ERR_CUDA;
    if (s_t < 0) s_t = D;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)s_t * 2, (cuuint64_t)s_h * 2, (cuuint64_t)s_b * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)box_rows, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_UNSUPPORTED;
}

// The fp32 dQ buffer [BH, Tq, D] as a 3-D map (D, Tq, BH) with [128 rows][32 columns]
// boxes in the 128-byte swizzle, for bulk reductions from shared memory. Rows past Tq of a
// (b, head) plane fall outside the map and are never written.
gqa_status make_dq_map(CUtensorMap* map, void* base, int BH, int Tq, int D) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return GQA_ERR_CUDA;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Tq, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)Tq * D * 4};
    cuuint32_t box[3] = {32, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_UNSUPPORTED;
}

// Strides of a dimension of extent 1 are never used; give TMA a harmless legal value.
long long effective_stride(long long s, int extent, long long fallback) {
    return extent == 1 ? fallback : s;
}

gqa_status check_kv_strides(int B, int Hkv, int Tk, int D, long long& sb, long long& sh) {
    const long long plane = (long long)Tk * D;
    sh = effective_stride(sh, Hkv, plane);
    sb = effective_stride(sb, B, plane * Hkv);
    if (sb <= 0 || sh <= 0) return GQA_ERR_INVALID_ARGUMENT;
    if ((sb & 7) || (sh & 7)) return GQA_ERR_INVALID_ARGUMENT;  // 16-byte TMA strides
    if (sb * 2 >= (1LL << 40) || sh * 2 >= (1LL << 40)) return GQA_ERR_UNSUPPORTED;
    return GQA_OK;
}

// Strides of a gqa_layout over extents (B, H, rows): used ones must be positive
// multiples of 8 elements (16-byte TMA strides), rows at least D apart; unused ones
// (extent 1) get a harmless legal value.
gqa_status check_layout(const gqa_layout* l, int B, int H, int rows, int D, long long& sb,
                        long long& sh, long long& st) {
    if (l == nullptr) return GQA_ERR_INVALID_ARGUMENT;
    st = effective_stride(l->st, rows, D);
    sh = effective_stride(l->sh, H, st * rows);
    sb = effective_stride(l->sb, B, sh * H);
    if (st < D || sh <= 0 || sb <= 0) return GQA_ERR_INVALID_ARGUMENT;
    if ((st & 7) || (sh & 7) || (sb & 7)) return GQA_ERR_INVALID_ARGUMENT;
    if (st * 2 >= (1LL << 40) || sh * 2 >= (1LL << 40) || sb * 2 >= (1LL << 40)) return GQA_ERR_UNSUPPORTED;
    return GQA_OK;
}

gqa_status check_common(int B, int Hq, int Hkv, int Tq, int Tk, int D) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || Tk <= 0 || D <= 0) return GQA_ERR_INVALID_ARGUMENT;
    if (Hq % Hkv != 0 || Tq > Tk) return GQA_ERR_INVALID_ARGUMENT;
    if (D != 64 && D != 128) return GQA_ERR_UNSUPPORTED;
    // flat element offsets of q and o must fit in 63 bits; grid and TMA limits below
    if ((long long)B * Hq > (1LL << 30)) return GQA_ERR_UNSUPPORTED;
    return GQA_OK;
}

int device_sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    return sms;
}

constexpr int kMaxDecodeRows = 16;  // query rows per head the decode path takes (T_q)
constexpr int kVarlenWaves = 8;     // automatic split target of gqa_attn_decode_varlen

struct SplitPlan {
    int splits, blk_per_split, blk_first, n_blk;
};

// Key blocks [blk_first, n_blk) hold every key some query row can see: with a window
// the rows of a chunk (positions Tk-Tq .. Tk-1) see nothing before Tk - Tq - window + 1.
// `waves`: CTAs per SM the automatic choice aims for. Sequences of different lengths
// (the varlen call) make CTAs of different lengths; more, shorter CTAs even out the
// last wave.
SplitPlan plan_splits(int B, int Hq, int Hkv, int Tq, int Tk, int window, int requested, int waves = 4) {
    SplitPlan sp{};
    sp.n_blk = (Tk + gqa::kTileKeys - 1) / gqa::kTileKeys;
    const int key_lo = window > 0 ? std::max(0, Tk - Tq - window + 1) : 0;
    sp.blk_first = key_lo / gqa::kTileKeys;
    const int n_range = sp.n_blk - sp.blk_first;
    const int G = Hq / Hkv;
    const long long units = (long long)B * Hkv * ((G * Tq + 15) / 16);
    int want = requested;
    if (want <= 0) {
        // about `waves` waves of one CTA per SM, each split at least 8 tiles (1024 keys)
        const long long target = (long long)waves * device_sm_count();
        want = (int)std::min<long long>((target + units - 1) / units, 1 << 20);
        want = std::min(want, std::max(1, n_range / 8));
    }
    want = std::max(1, std::min(want, n_range));
    sp.blk_per_split = (n_range + want - 1) / want;
    sp.splits = (n_range + sp.blk_per_split - 1) / sp.blk_per_split;  // no empty split
    return sp;
}

size_t ws_lse_offset(int splits, long long rows, int D) {
    const size_t o_bytes = (size_t)splits * rows * D * sizeof(float);
    return (o_bytes + 255) & ~(size_t)255;
}

size_t ws_bytes_for(const SplitPlan& sp, long long rows, int D) {
    if (sp.splits == 1) return 0;
    return ws_lse_offset(sp.splits, rows, D) + (size_t)sp.splits * rows * sizeof(float);
}

gqa_status check_decode(int B, int Hq, int Hkv, int Tq, int Tk, int D, int window) {
    gqa_status st = check_common(B, Hq, Hkv, Tq, Tk, D);
    if (st != GQA_OK) return st;
    if (window < 0) return GQA_ERR_INVALID_ARGUMENT;
    if (Tq > kMaxDecodeRows) return GQA_ERR_UNSUPPORTED;  // longer chunks: gqa_attn_fwd_ex
    return GQA_OK;
}

gqa_status current_sms(int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQA_ERR_CUDA;
    if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return GQA_ERR_CUDA;
    return GQA_OK;
}

// gqa_attn_fwd_ex, and with allow_split gqa_attn_fwd_split (a workspace for the parts of a
// split launch, when the plan splits).
gqa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                    int Tq, int Tk, int D, long long k_sb, long long k_sh, long long v_sb, long long v_sh,
                    float softmax_scale, int window, void* workspace, size_t workspace_bytes, bool allow_split,
                    void* stream) {
    gqa_status st = check_common(B, Hq, Hkv, Tq, Tk, D);
    if (st != GQA_OK) return st;
    if (window < 0) return GQA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return GQA_ERR_INVALID_ARGUMENT;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GQA_ERR_INVALID_ARGUMENT;
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return GQA_ERR_INVALID_ARGUMENT;
    if ((st = check_kv_strides(B, Hkv, Tk, D, k_sb, k_sh)) != GQA_OK) return st;
    if ((st = check_kv_strides(B, Hkv, Tk, D, v_sb, v_sh)) != GQA_OK) return st;

    gqa::FwdLaunch a{};
    a.window = window >= Tk ? 0 : window;  // a window covering every key is plain causal
    a.split_slices = 0;
    if (allow_split) {
        int sms = 0;
        if ((st = current_sms(&sms)) != GQA_OK) return st;
        const gqa::FwdSplitPlan sp = gqa::fwd_split_plan(B, Hq, Hkv, Tq, Tk, a.window, sms);
        const size_t need = gqa::fwd_split_workspace_bytes(sp, D);
        if (need > 0) {
            if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < need)
                return GQA_ERR_WORKSPACE;
            a.split_slices = sp.slices;
            a.part = static_cast<float*>(workspace);
        }
    }
    const long long q_sh = (long long)Tq * D;
    if ((st = make_map(&a.tm_q, q, B, Hq, Tq, D, q_sh * Hq, q_sh)) != GQA_OK) return st;
    if ((st = make_map(&a.tm_k, k, B, Hkv, Tk, D, k_sb, k_sh)) != GQA_OK) return st;
    if ((st = make_map(&a.tm_v, v, B, Hkv, Tk, D, v_sb, v_sh)) != GQA_OK) return st;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Tq = Tq; a.Tk = Tk; a.D = D;
    a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
    a.o = o;
    a.lse = lse;
    return gqa::launch_fwd(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* gqa_status_string(gqa_status s) {
    switch (s) {
        case GQA_OK: return "GQA_OK";
        case GQA_ERR_INVALID_ARGUMENT: return "GQA_ERR_INVALID_ARGUMENT";
        case GQA_ERR_UNSUPPORTED: return "GQA_ERR_UNSUPPORTED";
        case GQA_ERR_WORKSPACE: return "GQA_ERR_WORKSPACE";
        case GQA_ERR_CUDA: return "GQA_ERR_CUDA";
        case GQA_ERR_TIMEOUT: return "GQA_ERR_TIMEOUT";
    }
    return "GQA_ERR_UNKNOWN";
}

gqa_status gqa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Tq, int Tk, int D, long long k_sb, long long k_sh,
                        long long v_sb, long long v_sh, float softmax_scale, void* stream) {
    return gqa_attn_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh,
                           softmax_scale, 0, stream);
}

gqa_status gqa_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int Hq, int Hkv, int Tq, int Tk, int D, long long k_sb, long long k_sh,
                           long long v_sb, long long v_sh, float softmax_scale, int window,
                           void* stream) {
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh, softmax_scale, window,
                    nullptr, 0, false, stream);
}

size_t gqa_attn_fwd_split_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int D, int window) {
    if (check_common(B, Hq, Hkv, Tq, Tk, D) != GQA_OK || window < 0) return 0;
    int sms = 0;
    if (current_sms(&sms) != GQA_OK) return 0;
    return gqa::fwd_split_workspace_bytes(
        gqa::fwd_split_plan(B, Hq, Hkv, Tq, Tk, window >= Tk ? 0 : window, sms), D);
}

gqa_status gqa_attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                              int Hkv, int Tq, int Tk, int D, long long k_sb, long long k_sh, long long v_sb,
                              long long v_sh, float softmax_scale, int window, void* workspace,
                              size_t workspace_bytes, void* stream) {
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, k_sb, k_sh, v_sb, v_sh, softmax_scale, window,
                    workspace, workspace_bytes, true, stream);
}

int gqa_attn_decode_ex_num_splits(int B, int Hq, int Hkv, int Tq, int Tk, int D, int window,
                                  int num_splits) {
    if (check_decode(B, Hq, Hkv, Tq, Tk, D, window) != GQA_OK) return 0;
    return plan_splits(B, Hq, Hkv, Tq, Tk, window, num_splits).splits;
}

size_t gqa_attn_decode_ex_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int D, int window,
                                          int num_splits) {
    if (check_decode(B, Hq, Hkv, Tq, Tk, D, window) != GQA_OK) return 0;
    return ws_bytes_for(plan_splits(B, Hq, Hkv, Tq, Tk, window, num_splits), (long long)B * Hq * Tq, D);
}

gqa_status gqa_attn_decode_ex(const void* q, const void* k_cache, const void* v_cache, void* o, int B,
                              int Hq, int Hkv, int Tq, int Tk, int D, long long k_sb, long long k_sh,
                              long long v_sb, long long v_sh, float softmax_scale, int window,
                              int num_splits, void* workspace, size_t workspace_bytes, void* stream) {
    gqa_status st = check_decode(B, Hq, Hkv, Tq, Tk, D, window);
    if (st != GQA_OK) return st;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return GQA_ERR_INVALID_ARGUMENT;
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return GQA_ERR_INVALID_ARGUMENT;
    if ((st = check_kv_strides(B, Hkv, Tk, D, k_sb, k_sh)) != GQA_OK) return st;
    if ((st = check_kv_strides(B, Hkv, Tk, D, v_sb, v_sh)) != GQA_OK) return st;
    if (window >= Tk) window = 0;  // a window covering every key is plain causal
    const SplitPlan sp = plan_splits(B, Hq, Hkv, Tq, Tk, window, num_splits);
    const long long rows = (long long)B * Hq * Tq;
    gqa::DecLaunch a{};
    if (sp.splits > 1) {
        const size_t need = ws_bytes_for(sp, rows, D);
        if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return GQA_ERR_WORKSPACE;
        a.ws_o = static_cast<float*>(workspace);
        a.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws_lse_offset(sp.splits, rows, D));
    }
    if ((st = make_map(&a.tm_k, k_cache, B, Hkv, Tk, D, k_sb, k_sh)) != GQA_OK) return st;
    if ((st = make_map(&a.tm_v, v_cache, B, Hkv, Tk, D, v_sb, v_sh)) != GQA_OK) return st;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Tq = Tq; a.Tk = Tk; a.D = D;
    a.window = window;
    a.splits = sp.splits;
    a.blk_per_split = sp.blk_per_split;
    a.blk_first = sp.blk_first;
    a.n_blk = sp.n_blk;
    a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
    a.q = q;
    a.o = o;
    return gqa::launch_decode(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

int gqa_attn_decode_num_splits(int B, int Hq, int Hkv, int Tk, int D, int num_splits) {
    return gqa_attn_decode_ex_num_splits(B, Hq, Hkv, 1, Tk, D, 0, num_splits);
}

size_t gqa_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Tk, int D, int num_splits) {
    return gqa_attn_decode_ex_workspace_bytes(B, Hq, Hkv, 1, Tk, D, 0, num_splits);
}

gqa_status gqa_attn_decode(const void* q, const void* k_cache, const void* v_cache, void* o, int B,
                           int Hq, int Hkv, int Tk, int D, long long k_sb, long long k_sh,
                           long long v_sb, long long v_sh, float softmax_scale, int num_splits,
                           void* workspace, size_t workspace_bytes, void* stream) {
    return gqa_attn_decode_ex(q, k_cache, v_cache, o, B, Hq, Hkv, 1, Tk, D, k_sb, k_sh, v_sb, v_sh,
                              softmax_scale, 0, num_splits, workspace, workspace_bytes, stream);
}

size_t gqa_attn_fwd_varlen_workspace_bytes(int S, int Hq, int Hkv, int max_seqlen_q) {
    if (S <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_seqlen_q <= 0) return 0;
    int n_lvl = 0, n_h = 0;
    const long long n = gqa::fwd_varlen_candidates(S, Hq, Hkv, max_seqlen_q, &n_lvl, &n_h);
    if (n <= 0 || n > 0x7fffffffLL - 64) return 0;
    return gqa::fwd_varlen_workspace_bytes(n);
}

namespace {

// Shared by the contiguous and the paged variable-length forward. table non-null: the keys
// are paged (rows_k = the key capacity, max_pages * page_size; the k/v layouts and maps cover
// the pool of num_pages pages).
gqa_status fwd_varlen_impl(const void* q, const void* k, const void* v, void* o, float* lse,
                           const int* cu_seqlens_q, const int* cu_seqlens_k, const int* seqlens_q,
                           const int* seqlens_k, const int* table, int page_size, int num_pages, int max_pages,
                           int S, int Hq, int Hkv, int D, int rows_q, int rows_k, int max_seqlen_q,
                           const gqa_layout* q_layout, const gqa_layout* k_layout, const gqa_layout* v_layout,
                           const gqa_layout* o_layout, float softmax_scale, int window, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (S <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || rows_q <= 0 || rows_k <= 0 || max_seqlen_q <= 0)
        return GQA_ERR_INVALID_ARGUMENT;
    if (Hq % Hkv != 0 || window < 0) return GQA_ERR_INVALID_ARGUMENT;
    if (D != 64 && D != 128) return GQA_ERR_UNSUPPORTED;
    if ((cu_seqlens_q && seqlens_q) || (cu_seqlens_k && seqlens_k)) return GQA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return GQA_ERR_INVALID_ARGUMENT;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GQA_ERR_INVALID_ARGUMENT;
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return GQA_ERR_INVALID_ARGUMENT;
    const int bq = cu_seqlens_q ? 1 : S;  // batch extent of each side
    const int bk = table ? num_pages : (cu_seqlens_k ? 1 : S);
    const int kv_rows = table ? page_size : rows_k;  // rows of one k/v batch plane (a page)
    gqa::FwdVarlenLaunch a{};
    long long ls[3][3];  // (sb, sh, st) of q, k, v
    gqa_status e;
    if ((e = check_layout(q_layout, bq, Hq, rows_q, D, ls[0][0], ls[0][1], ls[0][2])) != GQA_OK) return e;
    if ((e = check_layout(k_layout, bk, Hkv, kv_rows, D, ls[1][0], ls[1][1], ls[1][2])) != GQA_OK) return e;
    if ((e = check_layout(v_layout, bk, Hkv, kv_rows, D, ls[2][0], ls[2][1], ls[2][2])) != GQA_OK) return e;
    if ((e = check_layout(o_layout, bq, Hq, rows_q, D, a.o_sb, a.o_sh, a.o_st)) != GQA_OK) return e;
    const size_t need = gqa_attn_fwd_varlen_workspace_bytes(S, Hq, Hkv, max_seqlen_q);
    if (need == 0) return GQA_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return GQA_ERR_WORKSPACE;
    if ((e = make_map(&a.tm_q, q, bq, Hq, rows_q, D, ls[0][0], ls[0][1], ls[0][2])) != GQA_OK) return e;
    const int box = table && page_size < gqa::kTileKeys ? page_size : gqa::kTileKeys;
    if ((e = make_map(&a.tm_k, k, bk, Hkv, kv_rows, D, ls[1][0], ls[1][1], ls[1][2], box)) != GQA_OK) return e;
    if ((e = make_map(&a.tm_v, v, bk, Hkv, kv_rows, D, ls[2][0], ls[2][1], ls[2][2], box)) != GQA_OK) return e;
    a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D;
    a.rows_q = rows_q; a.rows_k = rows_k; a.max_q = max_seqlen_q;
    a.window = window;
    a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
    a.cu_q = cu_seqlens_q; a.cu_k = cu_seqlens_k;
    a.len_q = seqlens_q; a.len_k = seqlens_k;
    a.o = o;
    a.lse = lse;
    a.ws = static_cast<int*>(workspace);
    a.table = table;
    a.page_size = page_size;
    a.num_pages = num_pages;
    a.max_pages = max_pages;
    return gqa::launch_fwd_varlen(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // namespace

gqa_status gqa_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                               const int* cu_seqlens_q, const int* cu_seqlens_k, const int* seqlens_q,
                               const int* seqlens_k, int S, int Hq, int Hkv, int D, int rows_q,
                               int rows_k, int max_seqlen_q, const gqa_layout* q_layout,
                               const gqa_layout* k_layout, const gqa_layout* v_layout,
                               const gqa_layout* o_layout, float softmax_scale, int window,
                               void* workspace, size_t workspace_bytes, void* stream) {
    return fwd_varlen_impl(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, seqlens_q, seqlens_k, nullptr, 0, 0, 0, S,
                           Hq, Hkv, D, rows_q, rows_k, max_seqlen_q, q_layout, k_layout, v_layout, o_layout,
                           softmax_scale, window, workspace, workspace_bytes, stream);
}

gqa_status gqa_attn_fwd_varlen_paged(const void* q, const void* k_pool, const void* v_pool, void* o, float* lse,
                                     const int* cu_seqlens_q, const int* seqlens_q, const int* seqlens_k,
                                     const int* block_table, int page_size, int num_pages, int max_pages, int S,
                                     int Hq, int Hkv, int D, int rows_q, int max_seqlen_q,
                                     const gqa_layout* q_layout, const gqa_layout* k_layout,
                                     const gqa_layout* v_layout, const gqa_layout* o_layout, float softmax_scale,
                                     int window, void* workspace, size_t workspace_bytes, void* stream) {
    if (!seqlens_k || !block_table) return GQA_ERR_INVALID_ARGUMENT;
    const bool page_ok = page_size >= 16 && page_size % 16 == 0 &&
                         (page_size % gqa::kTileKeys == 0 || gqa::kTileKeys % page_size == 0);
    if (!page_ok || num_pages <= 0 || max_pages <= 0) return GQA_ERR_INVALID_ARGUMENT;
    if ((long long)max_pages * page_size > 0x7fffffffLL) return GQA_ERR_UNSUPPORTED;
    return fwd_varlen_impl(q, k_pool, v_pool, o, lse, cu_seqlens_q, nullptr, seqlens_q, seqlens_k, block_table,
                           page_size, num_pages, max_pages, S, Hq, Hkv, D, rows_q, max_pages * page_size,
                           max_seqlen_q, q_layout, k_layout, v_layout, o_layout, softmax_scale, window, workspace,
                           workspace_bytes, stream);
}

int gqa_attn_decode_varlen_num_splits(int B, int Hq, int Hkv, int Tq, int max_seqlen_k, int D, int window,
                                      int num_splits) {
    if (check_decode(B, Hq, Hkv, Tq, max_seqlen_k, D, window) != GQA_OK) return 0;
    return plan_splits(B, Hq, Hkv, Tq, max_seqlen_k, window >= max_seqlen_k ? 0 : window, num_splits,
                       kVarlenWaves).splits;
}

size_t gqa_attn_decode_varlen_workspace_bytes(int B, int Hq, int Hkv, int Tq, int max_seqlen_k, int D,
                                              int window, int num_splits) {
    if (check_decode(B, Hq, Hkv, Tq, max_seqlen_k, D, window) != GQA_OK) return 0;
    return ws_bytes_for(plan_splits(B, Hq, Hkv, Tq, max_seqlen_k, window >= max_seqlen_k ? 0 : window,
                                    num_splits, kVarlenWaves),
                        (long long)B * Hq * Tq, D);
}

gqa_status gqa_attn_decode_varlen(const void* q, const void* k_cache, const void* v_cache, void* o,
                                  const int* seqlens_k, const int* block_table, int page_size,
                                  int num_pages, int max_pages, int B, int Hq, int Hkv, int Tq,
                                  int max_seqlen_k, int D, const gqa_layout* k_layout,
                                  const gqa_layout* v_layout, float softmax_scale, int window,
                                  int num_splits, void* workspace, size_t workspace_bytes, void* stream) {
    gqa_status st = check_decode(B, Hq, Hkv, Tq, max_seqlen_k, D, window);
    if (st != GQA_OK) return st;
    if (!seqlens_k) return GQA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
        return GQA_ERR_INVALID_ARGUMENT;
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return GQA_ERR_INVALID_ARGUMENT;
    gqa::DecLaunch a{};
    long long lk[3], lv[3];  // (sb, sh, st)
    int capacity = max_seqlen_k, box = gqa::kTileKeys;
    const int b_ext = block_table ? num_pages : B, rows_ext = block_table ? page_size : max_seqlen_k;
    if (block_table) {
        const bool page_ok = page_size >= 16 && page_size % 16 == 0 &&
                             (page_size % gqa::kTileKeys == 0 || gqa::kTileKeys % page_size == 0);
        if (!page_ok || num_pages <= 0 || max_pages <= 0) return GQA_ERR_INVALID_ARGUMENT;
        box = page_size < gqa::kTileKeys ? page_size : gqa::kTileKeys;
        capacity = (long long)max_pages * page_size < max_seqlen_k ? max_pages * page_size : max_seqlen_k;
    } else {
        page_size = num_pages = max_pages = 0;
    }
    if ((st = check_layout(k_layout, b_ext, Hkv, rows_ext, D, lk[0], lk[1], lk[2])) != GQA_OK) return st;
    if ((st = check_layout(v_layout, b_ext, Hkv, rows_ext, D, lv[0], lv[1], lv[2])) != GQA_OK) return st;
    // The split count is planned for the longest sequence; each sequence shares its
    // own blocks over those splits on the device.
    const SplitPlan sp = plan_splits(B, Hq, Hkv, Tq, max_seqlen_k, window >= max_seqlen_k ? 0 : window,
                                     num_splits, kVarlenWaves);
    const long long rows = (long long)B * Hq * Tq;
    if (sp.splits > 1) {
        const size_t need = ws_bytes_for(sp, rows, D);
        if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return GQA_ERR_WORKSPACE;
        a.ws_o = static_cast<float*>(workspace);
        a.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws_lse_offset(sp.splits, rows, D));
    }
    if ((st = make_map(&a.tm_k, k_cache, b_ext, Hkv, rows_ext, D, lk[0], lk[1], lk[2], box)) != GQA_OK) return st;
    if ((st = make_map(&a.tm_v, v_cache, b_ext, Hkv, rows_ext, D, lv[0], lv[1], lv[2], box)) != GQA_OK) return st;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Tq = Tq; a.Tk = max_seqlen_k; a.D = D;
    a.window = window;
    a.splits = sp.splits;
    a.blk_per_split = sp.blk_per_split;
    a.blk_first = sp.blk_first;
    a.n_blk = sp.n_blk;
    a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
    a.q = q;
    a.o = o;
    a.seqlens = seqlens_k;
    a.table = block_table;
    a.max_pages = max_pages;
    a.page_size = page_size;
    a.num_pages = num_pages;
    a.capacity = capacity;
    return gqa::launch_decode(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

size_t gqa_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int D) {
    if (check_common(B, Hq, Hkv, Tq, Tk, D) != GQA_OK) return 0;
    size_t dq_bytes, vec_bytes;
    gqa::bwd_workspace_layout(B, Hq, Tq, D, &dq_bytes, &vec_bytes);
    return dq_bytes + 2 * vec_bytes;
}

gqa_status gqa_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Tq, int Tk,
                        int D, long long k_sb, long long k_sh, long long v_sb, long long v_sh,
                        float softmax_scale, int window, void* workspace, size_t workspace_bytes,
                        void* stream) {
    gqa_status st = check_common(B, Hq, Hkv, Tq, Tk, D);
    if (st != GQA_OK) return st;
    if (window < 0) return GQA_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || !aligned16(lse))
        return GQA_ERR_INVALID_ARGUMENT;
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return GQA_ERR_INVALID_ARGUMENT;
    if ((st = check_kv_strides(B, Hkv, Tk, D, k_sb, k_sh)) != GQA_OK) return st;
    if ((st = check_kv_strides(B, Hkv, Tk, D, v_sb, v_sh)) != GQA_OK) return st;
    if ((long long)B * Hkv > 65535 || (Tk + 127) / 128 > 0x7fffffff) return GQA_ERR_UNSUPPORTED;  // grid y, x
    size_t dq_bytes, vec_bytes;
    gqa::bwd_workspace_layout(B, Hq, Tq, D, &dq_bytes, &vec_bytes);
    if (!workspace || workspace_bytes < dq_bytes + 2 * vec_bytes || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return GQA_ERR_WORKSPACE;
    gqa::BwdLaunch a{};
    const long long q_sh = (long long)Tq * D;
    if ((st = make_map(&a.tm_q, q, B, Hq, Tq, D, q_sh * Hq, q_sh)) != GQA_OK) return st;
    if ((st = make_map(&a.tm_do, dout, B, Hq, Tq, D, q_sh * Hq, q_sh)) != GQA_OK) return st;
    if ((st = make_map(&a.tm_k, k, B, Hkv, Tk, D, k_sb, k_sh)) != GQA_OK) return st;
    if ((st = make_map(&a.tm_v, v, B, Hkv, Tk, D, v_sb, v_sh)) != GQA_OK) return st;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Tq = Tq; a.Tk = Tk; a.D = D;
    a.window = window >= Tk ? 0 : window;  // a window covering every key is plain causal
    a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
    a.o = o; a.dout = dout; a.lse = lse;
    a.dq = dq; a.dk = dk; a.dv = dv;
    char* ws = static_cast<char*>(workspace);
    a.dq_acc = reinterpret_cast<float*>(ws);
    if ((st = make_dq_map(&a.tm_dq, a.dq_acc, B * Hq, Tq, D)) != GQA_OK) return st;
    a.lse2 = reinterpret_cast<float*>(ws + dq_bytes);
    a.dvec = reinterpret_cast<float*>(ws + dq_bytes + vec_bytes);
    return gqa::launch_bwd(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

gqa_status gqa_get_device_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GQA_ERR_CUDA;
    uint32_t v = 0;
    if (gqa::read_and_clear_device_error(&v) != cudaSuccess) return GQA_ERR_CUDA;
    if (v & gqa::kErrBitWaitTimeout) return GQA_ERR_TIMEOUT;
    if (v & gqa::kErrBitBadSeqlens) return GQA_ERR_INVALID_ARGUMENT;
    return GQA_OK;
}

gqa_status gqa_testing_fwd_split_plan(int B, int Hq, int Hkv, int Tq, int Tk, int D, int window, int sms,
                                      int* out_slices, long long* out_whole, long long* out_split, long long* out_units) {
    if (!out_slices || !out_whole || !out_split || !out_units || sms < 1 || window < 0) return GQA_ERR_INVALID_ARGUMENT;
    if (check_common(B, Hq, Hkv, Tq, Tk, D) != GQA_OK) return GQA_ERR_INVALID_ARGUMENT;
    const gqa::FwdSplitPlan sp = gqa::fwd_split_plan(B, Hq, Hkv, Tq, Tk, window >= Tk ? 0 : window, sms);
    *out_slices = sp.slices;
    *out_whole = sp.whole;
    *out_split = sp.split;
    *out_units = gqa::fwd_units(B, Hq, Hkv, Tq);
    return GQA_OK;
}

gqa_status gqa_testing_bwd_order(int n_kb, int n_bg, int G, int Tq, int D, int* out_chunk, int* out_bg, int* out_j) {
    if (n_kb <= 0 || n_bg <= 0 || G <= 0 || Tq <= 0 || D <= 0 || !out_chunk || !out_bg || !out_j)
        return GQA_ERR_INVALID_ARGUMENT;
    const int chunk = gqa::bwd_chunk(n_bg, G, Tq, D);
    *out_chunk = chunk;
    for (int L = 0; L < n_kb * n_bg; ++L) gqa::bwd_block_coords(L, n_kb, n_bg, chunk, &out_bg[L], &out_j[L]);
    return GQA_OK;
}

gqa_status gqa_selftest_bounded_wait(unsigned long long timeout_ns, void* stream) {
    if (timeout_ns < 1000ull || timeout_ns > 10000000000ull) return GQA_ERR_INVALID_ARGUMENT;
    return gqa::launch_selftest_wait(timeout_ns, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? GQA_OK
               : GQA_ERR_CUDA;
}

}  // extern "C"
