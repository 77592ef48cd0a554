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
    // split launch (fwd_split_plan): the last units' key tiles in split_k parts, whose
    // fp32 partials go to `part` and are merged by a second kernel; split_k <= 1: none
    int split_k;
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
// have about the same number of key tiles n, so a last wave of r = units mod sms units
// leaves sms - r CTAs idle for a whole unit. Those r units are cut into k parts of about
// n / k tiles (at least 2), which the persistent CTAs take after the whole units; k (at
// most 8) minimises the estimated makespan (whole waves x n + part waves x (n / k + c),
// c = kFwdSplitPartCost tiles standing for a part's fixed cost: its Q load, pipeline fill,
// fp32 partial rows and share of the merge) and is used only if that estimate beats no
// split by 10 %. Partial rows: split units x k x 2 sub-tiles x 128 rows.
struct FwdSplitPlan {
    int k = 1;           // parts per split unit (1: no split)
    long long whole = 0; // units run whole (they come first in the unit list)
    long long split = 0; // units cut into k parts
    long long rows = 0;  // partial rows written to the workspace
};
constexpr int kFwdSplitMaxParts = 8;
// Fixed cost of a part, in key tiles: the MHA suffix workload (256 units of 64 tiles on 148
// SMs) measured 2.5 % slower split in 4 than whole, which puts it near 5 tiles.
constexpr double kFwdSplitPartCost = 5.0;
inline FwdSplitPlan fwd_split_plan(int B, int Hq, int Hkv, int Tq, int Tk, int window, int sms) {
    FwdSplitPlan sp;
    const long long units = fwd_units(B, Hq, Hkv, Tq);
    sp.whole = units;
    if (window > 0 || Tk - Tq < Tq || sms <= 0 || units <= 0) return sp;
    const long long n = (Tk - 1) / 128 + 1;  // key tiles of a unit's last row
    const long long full = units / sms, r = units % sms;
    if (r == 0) return sp;
    const double base = (double)(full + 1) * n;
    double best = base;
    int best_k = 1;
    for (int k = 2; k <= kFwdSplitMaxParts && n / k >= 2; ++k) {
        const long long part_waves = (r * k + sms - 1) / sms;
        const double cost = (double)full * n + (double)part_waves * ((double)n / k + kFwdSplitPartCost);
        if (cost < best) {
            best = cost;
            best_k = k;
        }
    }
    if (best_k == 1 || best > 0.9 * base) return sp;
    sp.k = best_k;
    sp.whole = units - r;
    sp.split = r;
    sp.rows = r * best_k * 2 * 128;
    return sp;
}
// Workspace of a split launch: fp32 partial O rows [rows, D], then their log2-domain
// log-sum-exp [rows] (each 256-byte aligned).
inline size_t fwd_split_lse_offset(long long rows, int D) {
    return ((size_t)rows * D * sizeof(float) + 255) & ~(size_t)255;
}
inline size_t fwd_split_workspace_bytes(const FwdSplitPlan& sp, int D) {
    if (sp.k <= 1) return 0;
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
