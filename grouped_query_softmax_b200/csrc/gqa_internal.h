// Internal interface between the C ABI (gqa_api.cpp) and the kernel translation
// unit (gqa_kernels.cu). Not installed, not part of the ABI.
#pragma once

#include <algorithm>

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
    // split launch (fwd_split_plan): the last units' key tiles dealt out over
    // split_slices slices, whose fp32 partials go to `part` and are merged by a second
    // kernel; split_slices = 0: none
    int split_slices;
    float* part;
};

// Work units of a dense forward launch: pairs of 128-row sub-tiles (heads a, a+1 of one
// group when the group size is even, else rows r and r + 128 of one head).
inline long long fwd_units(int B, int Hq, int Hkv, int Tq) {
    const int G = Hq / Hkv;
    const int n_qt = (Tq + 127) / 128;
    return G % 2 == 0 ? (long long)B * Hkv * (G / 2) * n_qt : (long long)B * Hq * ((n_qt + 1) / 2);
}

// Split plan of a dense forward launch on `sms` persistent CTAs. Only plain causal suffix
// launches whose cached prefix is at least as long as the suffix qualify: their units all
// have about n key tiles (n = the last row's), so a last wave of r = units mod sms units
// would leave sms - r CTAs idle for most of a unit. The full waves run whole; the last r
// units' key tiles are dealt out as `slices` equal runs of consecutive tiles, one per CTA,
// cut at unit boundaries into pieces whose fp32 partial rows a second kernel merges. Units
// come in groups of `group` (the row levels of one KV head, listed together); when the whole
// units fill whole groups, each run covers the same keys of every unit of a group on
// `group` CTAs at once, and slices is a multiple of group. Bounds: r <= slices <= min(sms,
// r n / 2, 29 r): at least two tiles a run, at most 29 runs a unit. Estimated makespan in
// key tiles: full x n + r n / slices + c per piece of the busiest slice (two unless slices
// is a multiple of r, when no run crosses a unit boundary), c = kFwdSplitPartCost for a
// piece's fixed cost (its Q load, pipeline fill, fp32 partial rows and share of the merge).
// The best slice count is used when it beats the unsplit (full + 1) x n by the factor
// kFwdSplitGain. Partial rows: slices x 2 pieces x 2 sub-tiles x 128 rows.
struct FwdSplitPlan {
    int slices = 0;      // 0: no split
    int group = 1;       // units per group of the slice lanes
    long long whole = 0; // units run whole (they come first in the unit list)
    long long split = 0; // units cut into pieces
    long long rows = 0;  // partial rows in the workspace
};
constexpr double kFwdSplitPartCost = 5.0;
constexpr double kFwdSplitGain = 0.95;
constexpr int kFwdSplitMaxPerUnit = 29;
inline double fwd_split_cost(long long n, long long full, long long r, long long slices) {
    return (double)full * n + (double)(r * n) / slices + kFwdSplitPartCost * (slices % r == 0 ? 1 : 2);
}
inline FwdSplitPlan fwd_split_plan(int B, int Hq, int Hkv, int Tq, int Tk, int window, int sms) {
    FwdSplitPlan sp;
    const long long units = fwd_units(B, Hq, Hkv, Tq);
    sp.whole = units;
    if (window > 0 || Tk - Tq < Tq || sms <= 0 || units <= 0) return sp;
    const long long n = (Tk - 1) / 128 + 1;  // key tiles of a unit's last row
    const long long full = units / sms, r = units % sms;
    if (r == 0 || n < 4) return sp;
    // these launches list units head by head: the row levels of one head (pair) together
    const int G = Hq / Hkv;
    const int n_qt = (Tq + 127) / 128;
    long long group = G % 2 == 0 ? n_qt : (n_qt + 1) / 2;
    if ((full * sms) % group != 0) group = 1;
    const long long top = std::min<long long>(std::min<long long>(sms, r * n / 2), r * kFwdSplitMaxPerUnit);
    const double base = (double)(full + 1) * n;
    double best = base;
    long long best_s = 0;
    for (long long s = (r + group - 1) / group * group; s <= top; s += group) {
        const double cost = fwd_split_cost(n, full, r, s);
        if (cost < best) {
            best = cost;
            best_s = s;
        }
    }
    if (best_s == 0 || best > kFwdSplitGain * base) return sp;
    sp.slices = (int)best_s;
    sp.group = (int)group;
    sp.whole = full * sms;
    sp.split = r;
    sp.rows = best_s * 2 * 2 * 128;
    return sp;
}
// Workspace of a split launch: fp32 partial O rows [rows, D], then their log2-domain
// log-sum-exp [rows] (each 256-byte aligned).
inline size_t fwd_split_lse_offset(long long rows, int D) {
    return ((size_t)rows * D * sizeof(float) + 255) & ~(size_t)255;
}
inline size_t fwd_split_workspace_bytes(const FwdSplitPlan& sp, int D) {
    if (sp.slices <= 0) return 0;
    return fwd_split_lse_offset(sp.rows, D) + (size_t)sp.rows * sizeof(float);
}

// Sequences of different lengths (gqa_attn_fwd_varlen). Exactly one of cu_* / len_*
// describes each side (both null: every sequence owns all rows of its batch).
struct FwdVarlenLaunch {
    CUtensorMap tm_q, tm_k, tm_v;
    int S, Hq, Hkv, D;
    int rows_q, rows_k, max_q;
    int window;
    float scale;
    const int* cu_q;
    const int* cu_k;
    const int* len_q;
    const int* len_k;
    void* o;
    long long o_sb, o_sh, o_st;  // elements
    float* lse;
    int* ws;  // plan workspace (fwd_varlen_workspace_bytes)
    // paged keys (gqa_attn_fwd_varlen_paged); table null = contiguous keys
    const int* table;
    int max_pages, page_size, num_pages;
};

// Candidate units of a variable-length forward: S x row levels x head slots. A unit
// is a head pair (even group size) or a pair of 128-row tiles of one head.
inline long long fwd_varlen_candidates(int S, int Hq, int Hkv, int max_q, int* n_lvl, int* n_h) {
    const int G = Hq / Hkv;
    const bool pair_heads = G % 2 == 0;
    const int n_qt = (max_q + 127) / 128;
    *n_lvl = pair_heads ? n_qt : (n_qt + 1) / 2;
    *n_h = pair_heads ? Hq / 2 : Hq;
    return (long long)S * *n_lvl * *n_h;
}

constexpr size_t kPlanHeaderBytes = 256;
inline size_t fwd_varlen_workspace_bytes(long long candidates) {
    return kPlanHeaderBytes + (size_t)candidates * sizeof(int);
}

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
    // per-sequence lengths (gqa_attn_decode_varlen); seqlens null = the dense path
    const int* seqlens;
    const int* table;
    int max_pages, page_size, num_pages, capacity;
};

// Backward (gqa_attn_bwd). The workspace holds the fp32 dQ buffer, then LSE * log2(e)
// and <dO, O> per query row padded to whole 128-row tiles.
struct BwdLaunch {
    CUtensorMap tm_q, tm_k, tm_v, tm_do, tm_dq;  // tm_dq: the fp32 dQ buffer, for bulk reductions
    int B, Hq, Hkv, Tq, Tk, D;
    int window;
    float scale;
    const void* o;
    const void* dout;
    const float* lse;
    void* dq;
    void* dk;
    void* dv;
    float* dq_acc;
    float* lse2;
    float* dvec;
};

// Backward launch order. Key block j of a (batch, KV head) pair walks the query tiles from
// about j on, so low j carries the most work. The pairs are taken in chunks of `chunk`;
// inside a chunk every pair's block 0 is launched first, then every pair's block 1, and so
// on (longest first, which keeps the last wave short). A chunk's fp32 dQ rows, which all its
// key blocks add into, are the L2 working set: `chunk` is the largest divisor of the number
// of pairs whose dQ rows fit in kBwdChunkDqBytes.
constexpr double kBwdChunkDqBytes = 72.0 * 1024 * 1024;
inline int bwd_chunk(int n_bg, int G, int Tq, int D) {
    const double per_pair = (double)G * Tq * D * sizeof(float);
    int best = 1;
    for (int c = 2; c <= n_bg; ++c)
        if (n_bg % c == 0 && c * per_pair <= kBwdChunkDqBytes) best = c;
    return best;
}
// (pair, key block) of linear block index L, for n_kb key blocks per pair.
__host__ __device__ inline void bwd_block_coords(int L, int n_kb, int n_bg, int chunk, int* bg, int* j) {
    const int per_chunk = chunk * n_kb;
    const int c = L / per_chunk;
    const int r = L - c * per_chunk;
    const int width = n_bg - c * chunk < chunk ? n_bg - c * chunk : chunk;
    *j = r / width;
    *bg = c * chunk + (r - *j * width);
}

inline size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }
inline void bwd_workspace_layout(int B, int Hq, int Tq, int D, size_t* dq_bytes, size_t* vec_bytes) {
    const size_t tq_pad = (size_t)(Tq + 127) / 128 * 128;
    *dq_bytes = round256((size_t)B * Hq * Tq * D * sizeof(float));
    *vec_bytes = round256((size_t)B * Hq * tq_pad * sizeof(float));
}

// Each returns cudaSuccess or the launch error; nothing is synchronised.
cudaError_t launch_fwd(const FwdLaunch& a, cudaStream_t stream);
cudaError_t launch_fwd_varlen(const FwdVarlenLaunch& a, cudaStream_t stream);
cudaError_t launch_decode(const DecLaunch& a, cudaStream_t stream);
cudaError_t launch_bwd(const BwdLaunch& a, cudaStream_t stream);
cudaError_t launch_selftest_wait(unsigned long long timeout_ns, cudaStream_t stream);

// Read and clear the device error word of the current device (after a stream sync).
cudaError_t read_and_clear_device_error(uint32_t* value);

// Bits of the device error word (set by the kernels, read by gqa_get_device_error).
constexpr uint32_t kErrBitWaitTimeout = 1u;   // a bounded wait ran out
constexpr uint32_t kErrBitBadSeqlens = 2u;    // sequence bounds outside their tensors

// Bound on every device-side wait of the production kernels.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

// Rows per fwd sub-tile and keys per tile, shared with the host planner.
constexpr int kTileRows = 128;
constexpr int kTileKeys = 128;

}  // namespace gqa
