// Causal grouped-query attention forward (prefill and suffix chunks) for sm_100a.
//
// Computes o_a = softmax(Q_a K_{g(a)}^T * scale + M) V_{g(a)}, g(a) = a / (H_q/H_kv)
// ("注意力家族", section 统一记号), with the causal mask M placing query row i at
// absolute position (T_k - T_q) + i ("注意力家族", sections 最小语义实现 and
// Mask 与增量位置). Execution follows the tiled exact-attention idea ("A Visual
// Guide to Attention", section "Sources and execution"; "长上下文与高效注意力", the
// FlashAttention entry): tiles of Q, K and V are staged on chip and merged with an
// online softmax so the T_q x T_k score matrix never reaches HBM.
//
// B200 mapping: a work unit is two 128-row query sub-tiles that share every K/V tile;
// units are ordered longest first and a persistent CTA per SM strides over them, so
// the next unit's Q load and Q K^T products overlap the current unit's epilogue.
//   * warp 0      : TMA producer. Loads both Q sub-tiles of a unit, then K_0, V_0, K_1, V_1 ...
//                   of KV head g(a) into a ring of 128-key slots (128-byte swizzle).
//                   K/V are addressed per KV head; nothing is replicated.
//   * warp 1      : tcgen05 issuer (one thread). S_s = Q_s K_j^T into TMEM (fp32),
//                   O_s += P_s V_j with P read from TMEM. Completion is signalled with
//                   tcgen05.commit on mbarriers.
//   * warp 2      : TMEM allocation (512 columns: S_0, S_1, O_0, O_1).
//   * warps 4..11 : two softmax warpgroups, one per sub-tile; thread r owns row r
//                   (TMEM lane r), so row max and row sum need no shuffles. P is
//                   rounded to bf16 and written over the first half of S in TMEM.
//                   The running max is refreshed only when it grows by more than
//                   2^8 (in the log2 domain), so O is rescaled rarely; the final
//                   O / l and the log-sum-exp are exact whatever max was kept. The
//                   epilogue stages each warp's bf16 rows in shared memory and
//                   stores them as whole row segments.
// Causal tile skipping: a sub-tile visits KV tiles 0 .. floor((off + last_row)/128)
// only, and applies the mask only on tiles that cross its diagonal.
#pragma once

#include "sm100_ptx.cuh"

namespace gqa {

constexpr int kFwdRows = 128;     // query rows per sub-tile (= TMEM lanes)
constexpr int kFwdKeys = 128;     // keys per KV tile
constexpr int kFwdThreads = 384;  // 12 warps = 3 warpgroups
// Register split (setmaxnreg): the launch gives 384 threads x kFwdLaunchRegs; the
// producer/MMA warpgroup drops to kFwdCtlRegs so the two softmax warpgroups can hold
// a full 128-column score row without spilling. 128 * (104 + 200 + 200) = 384 * 168.
constexpr int kFwdLaunchRegs = 168;
constexpr int kFwdCtlRegs = 104;
constexpr int kFwdSoftmaxRegs = 200;
static_assert(128 * (kFwdCtlRegs + 2 * kFwdSoftmaxRegs) <= kFwdThreads * kFwdLaunchRegs,
              "register split exceeds the launch allocation");
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 2^8 between refreshes

// Readers of a published unit in a dynamic-fetch launch: the MMA thread, the eight softmax
// warps and the ragged-tile cleaner warp.
constexpr int kUnitReaders = 10;

constexpr int kUnitPairHeads = 1;
constexpr int kUnitHeadMajor = 2;

struct FwdParams {
    int B, Hq, Hkv, Tq, Tk, G;
    int n_qt;        // ceil(Tq / 128)
    int unit_flags;  // kUnitPairHeads: sub-tiles are heads (a, a+1) of one group on the same
                     //   rows, else rows (r, r+128) of one head
                     // kUnitHeadMajor: units listed head by head (all row levels of one head
                     //   together), else level by level, longest rows first
    int per_level;   // work units per row level
    int units;       // total work units (grid-strided by the persistent CTAs)
    float scale_log2;
    int window;      // > 0: each query sees only its `window` most recent positions
    __nv_bfloat16* o;
    float* lse;  // nullable
    uint32_t* err;
    unsigned long long timeout_ns;
    // split launches (split_slices > 0): the first split_whole units run whole, the other
    // units - split_whole are cut into key-tile pieces over split_slices slices (entries
    // split_whole + 2 * slice + piece), in split_group lanes of units that share K/V; pieces
    // write fp32 O / l rows to part and their log2-domain log-sum-exp to part_lse
    int split_whole, split_slices, split_group;
    float* part;
    float* part_lse;
};

// Sequences of different lengths (the kVarlen instantiation only). A kernel parameter
// of its own: growing FwdParams past ~112 bytes made the dense kernel spill.
struct FwdVarlenParams {
    const int* cu_q;  // packed queries: sequence s owns rows cu_q[s] .. cu_q[s+1]-1 (batch 0)
    const int* cu_k;  // packed keys, likewise
    const int* len_q; // padded queries (cu_q null): sequence s is batch s, rows 0 .. len_q[s]-1
    const int* len_k; // padded keys; a null length array means every sequence has all rows
    int rows_q, rows_k;  // row extent of the q/o and k/v tensors
    int n_lvl, n_h;      // candidate unit c = (s * n_lvl + level) * n_h + head slot
    const int* unit_list;   // present units (written by the plan kernel)
    const int* unit_count;  // their number
    // dynamic != 0: the list is sequence-major and the persistent CTAs take its entries in
    // order through the counter *fetch (zeroed by the plan kernel) instead of a fixed stride
    int* fetch;
    int dynamic;
    long long o_sb, o_sh, o_st;  // element strides of o (batch, head, row); d is contiguous
    // paged keys (table non-null): key t of sequence s is row t % page_size of pool page
    // table[s * max_pages + t / page_size]; the k/v tensor maps cover the pool
    const int* table;
    int max_pages, page_size, box_rows, num_pages;
};

// Where one sequence's rows are: batch index, first row and length of each side.
struct SeqGeo {
    int b_q, r_q, len_q;
    int b_k, r_k, len_k;
};

template <int D>
struct FwdSmem {
    static constexpr int kChunks = D / 64;             // 64-element (128-byte) column chunks
    static constexpr int kChunkBytes = 128 * 128;      // 128 rows x 128 bytes
    static constexpr int kTileBytes = kChunks * kChunkBytes;
    static constexpr int kStages = D == 128 ? 4 : 8;   // ring slots, each one K or one V tile
    static constexpr int kQOff = 0;
    static constexpr int kRingOff = 2 * kTileBytes;
    // output staging: each softmax warp's 32 rows x 64 columns of bf16 (128 bytes a row), so
    // the epilogue's global stores go out as whole row segments
    static constexpr int kStageWarpBytes = 32 * 128;
    static constexpr int kStageOff = kRingOff + kStages * kTileBytes;
    static constexpr int kCtlOff = kStageOff + 8 * kStageWarpBytes;
    struct Ctl {
        uint64_t q_full;
        uint64_t q_empty;
        uint64_t full[kStages];
        uint64_t empty[kStages];
        uint64_t land[kStages];  // ragged last V tile of a sequence: lands here, is cleaned, then full
        uint64_t s_full[2];
        uint64_t p_full[2];
        uint64_t o_full[2];
        uint64_t o_empty[2];
        uint64_t drain;
        uint64_t unit_full[4];   // dynamic unit fetch: the producer publishes the CTA's k-th unit
        uint64_t unit_empty[4];  // in slot k % 4; its readers release the slot
        int unit_ring[4];
        int split_entry[2];      // split launch: this CTA's pieces (fwd_split_entry), -1: none
        uint32_t tmem_base;
        uint32_t abort;
    };
    static constexpr int kBytes = kCtlOff + (int)sizeof(Ctl) + 1024;  // + alignment slack
    static_assert(kBytes <= 232448, "shared memory above the 227 KB a CTA may have");
};

struct SubTile {
    int head;         // query head a
    int row0;         // first query row of the sub-tile
    int j_begin;      // first KV tile to visit (> 0 only inside a sliding window)
    int n_kv;         // KV tiles end (exclusive); the sub-tile visits [j_begin, n_kv) (n_kv 0 = absent)
    int masked_from;  // first KV tile that crosses the causal diagonal
    int lo_masked_end;  // KV tiles below this cross the lower edge of the window
};

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// Key-tile bounds of one sub-tile whose rows sit at positions off + row0 ...
__device__ __forceinline__ void fwd_fill_subtile(SubTile& st, int len_q, int off, int window) {
    st.j_begin = 0;
    st.lo_masked_end = 0;
    if (st.row0 >= len_q) {
        st.n_kv = 0;
        st.masked_from = 0;
        return;
    }
    const int last = min(st.row0 + kFwdRows - 1, len_q - 1);
    st.n_kv = (off + last) / kFwdKeys + 1;
    st.masked_from = (off + st.row0 + 1) / kFwdKeys;
    if (window > 0) {
        // row positions P0..P1 see keys (P - w, P]: tiles before the first row's
        // window are skipped, tiles before the last row's window start are masked
        const int lo_first = off + st.row0 - window + 1;
        const int lo_last = off + last - window + 1;
        st.j_begin = lo_first > 0 ? lo_first / kFwdKeys : 0;
        st.lo_masked_end = lo_last > 0 ? (lo_last + kFwdKeys - 1) / kFwdKeys : 0;
    }
}

__device__ __forceinline__ void fwd_decode_unit(const FwdParams& p, int u, int& b, int& g,
                                                SubTile (&st)[2]) {
    const int off = p.Tk - p.Tq;
    const bool pair = (p.unit_flags & kUnitPairHeads) != 0;
    int level, rest;
    if (p.unit_flags & kUnitHeadMajor) {
        // the row levels of one head (pair) run side by side and share its K/V through L2
        const int n_lvl = pair ? p.n_qt : (p.n_qt + 1) >> 1;
        rest = u / n_lvl;
        level = u - rest * n_lvl;
    } else {
        level = u / p.per_level;
        rest = u - level * p.per_level;
    }
    if (pair) {
        const int half_g = p.G >> 1;
        const int rt = p.n_qt - 1 - level;  // longest rows first
        b = rest / (p.Hkv * half_g);
        const int hp = rest - b * (p.Hkv * half_g);
        st[0].head = 2 * hp;
        st[1].head = 2 * hp + 1;
        st[0].row0 = st[1].row0 = rt * kFwdRows;
    } else {
        const int n_rb = (p.n_qt + 1) >> 1;
        const int rb = n_rb - 1 - level;
        b = rest / p.Hq;
        const int a = rest - b * p.Hq;
        st[0].head = st[1].head = a;
        st[0].row0 = rb * 2 * kFwdRows;
        st[1].row0 = st[0].row0 + kFwdRows;
    }
    g = st[0].head / p.G;
    fwd_fill_subtile(st[0], p.Tq, off, p.window);
    fwd_fill_subtile(st[1], p.Tq, off, p.window);
}

// a b / c for non-negative a, b and positive c, in 32-bit arithmetic when it fits.
__device__ __forceinline__ long long fwd_muldiv(long long a, long long b, long long c) {
    const long long x = a * b;
    if (x <= 0x7fffffffLL && c <= 0x7fffffffLL) return (long long)((uint32_t)x / (uint32_t)c);
    return x / c;
}

// Split launches. The S = units - split_whole last units form S / L groups of L consecutive
// units (the row levels of one KV head, which share its K/V; L = split_group); each group is
// laid out as N ticks (N = key tiles of the launch's last row, a bound on every unit's tiles)
// and the S / L groups end to end as T = (S / L) N ticks, dealt out as m = split_slices / L
// equal runs. Slice i = j L + lane takes run j of the unit in lane `lane` of each group it
// reaches, so the L CTAs of one run read the same keys of one head at the same time (L2
// hits). S / L <= m: a run crosses at most one group boundary. Piece 0 of slice i lies in the
// group holding the run's first tick, piece 1 (when the run crosses) in the next group. A
// piece covering ticks [a, b) of a unit with n key tiles takes tiles [a n / N, b n / N), so
// adjacent pieces tile every unit exactly.
__device__ __forceinline__ bool fwd_split_piece(const FwdParams& p, int slot, int& su, int& a, int& b) {
    const int L = p.split_group;
    const int m = p.split_slices / L;
    const long long N = (p.Tk - 1) / kFwdKeys + 1;
    const long long T = (long long)((p.units - p.split_whole) / L) * N;
    const int i = slot >> 1;
    const int j = i / L, lane = i - j * L;
    const long long lo = fwd_muldiv(T, j, m), hi = fwd_muldiv(T, j + 1, m);
    const long long g0 = fwd_muldiv(lo, 1, N);
    long long gr;
    if (slot & 1) {
        const long long start = (g0 + 1) * N;
        if (hi <= start) return false;
        gr = g0 + 1;
        a = 0;
        b = (int)(hi - start);
    } else {
        if (hi <= lo) return false;
        gr = g0;
        a = (int)(lo - g0 * N);
        b = (int)(min(hi, (g0 + 1) * N) - g0 * N);
    }
    su = (int)(gr * L + lane);
    return true;
}

// Keep key tiles [n a / N, n b / N) of a unit whose longest sub-tile has n tiles; each
// sub-tile keeps the tiles of its own range inside them (none: n_kv = 0).
__device__ __forceinline__ void fwd_clamp_ticks(SubTile (&st)[2], int a, int b, int N) {
    const long long n_max = max(st[0].n_kv, st[1].n_kv);
    const int j0 = (int)fwd_muldiv(n_max, a, N), j1 = (int)fwd_muldiv(n_max, b, N);
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        if (st[s].n_kv == 0) continue;
        st[s].j_begin = max(st[s].j_begin, j0);
        st[s].n_kv = min(st[s].n_kv, j1);
        if (st[s].j_begin >= st[s].n_kv) st[s].n_kv = 0;
    }
}

// Unit u of a dense launch: a whole unit, or (u >= split_whole in a split launch) a piece;
// an absent piece comes back with no tiles. Returns the split slot (-1: a whole unit).
__device__ __forceinline__ int fwd_dense_unit(const FwdParams& p, int u, int& b, int& g, SubTile (&st)[2]) {
    if (p.split_slices <= 0 || u < p.split_whole) {
        fwd_decode_unit(p, u, b, g, st);
        return -1;
    }
    const int slot = u - p.split_whole;
    int su = 0, ta = 0, tb = 0;
    const bool has = fwd_split_piece(p, slot, su, ta, tb);
    fwd_decode_unit(p, p.split_whole + su, b, g, st);
    if (has)
        fwd_clamp_ticks(st, ta, tb, (p.Tk - 1) / kFwdKeys + 1);
    else
        st[0].n_kv = st[1].n_kv = 0;
    return slot;
}

// One sequence side: batch index, first row and length.
__device__ __forceinline__ void fwd_seq_side(const int* cu, const int* len, int rows, int s, int& b,
                                             int& r, int& l) {
    if (cu != nullptr) {
        r = __ldg(cu + s);
        l = __ldg(cu + s + 1) - r;
        b = 0;
    } else {
        r = 0;
        l = len != nullptr ? __ldg(len + s) : rows;
        b = s;
    }
}

// Candidate unit c of a variable-length launch: sequence s, row level, head slot.
__device__ __forceinline__ void fwd_varlen_unit(const FwdParams& p, const FwdVarlenParams& vp, int c,
                                                SeqGeo& geo, int& g, SubTile (&st)[2]) {
    const int hidx = c % vp.n_h;
    const int t = c / vp.n_h;
    const int lvl = t % vp.n_lvl;
    const int s = t / vp.n_lvl;
    fwd_seq_side(vp.cu_q, vp.len_q, vp.rows_q, s, geo.b_q, geo.r_q, geo.len_q);
    fwd_seq_side(vp.cu_k, vp.len_k, vp.rows_k, s, geo.b_k, geo.r_k, geo.len_k);
    if (p.unit_flags & kUnitPairHeads) {
        st[0].head = 2 * hidx;
        st[1].head = 2 * hidx + 1;
        st[0].row0 = st[1].row0 = lvl * kFwdRows;
    } else {
        st[0].head = st[1].head = hidx;
        st[0].row0 = lvl * 2 * kFwdRows;
        st[1].row0 = st[0].row0 + kFwdRows;
    }
    g = st[0].head / p.G;
    const int off = geo.len_k - geo.len_q;
    fwd_fill_subtile(st[0], geo.len_q, off, p.window);
    fwd_fill_subtile(st[1], geo.len_q, off, p.window);
}

// KV tiles a unit's sub-tiles visit in total (0 = nothing to compute).
__device__ __forceinline__ int fwd_unit_work(const SubTile (&st)[2]) {
    int w = 0;
#pragma unroll
    for (int s = 0; s < 2; ++s)
        if (st[s].n_kv > 0) w += st[s].n_kv - st[s].j_begin;
    return w;
}

// Unit u of the launch, as the geometry of its sequence and its two sub-tiles.
template <bool kVarlen>
__device__ __forceinline__ void fwd_unit(const FwdParams& p, const FwdVarlenParams& vp, int u,
                                         SeqGeo& geo, int& g, SubTile (&st)[2]) {
    if constexpr (kVarlen) {
        fwd_varlen_unit(p, vp, __ldg(vp.unit_list + u), geo, g, st);
    } else {
        int b;
        fwd_dense_unit(p, u, b, g, st);
        geo.b_q = geo.b_k = b;
        geo.r_q = geo.r_k = 0;
        geo.len_q = p.Tq;
        geo.len_k = p.Tk;
    }
}

// k-th unit of persistent CTA i out of n: a boustrophedon walk over the longest-first
// unit list (i, 2n-1-i, 2n+i, ...), so each CTA's total work is nearly equal.
__device__ __forceinline__ int snake_unit(int k, int i, int n) {
    return k * n + ((k & 1) ? (n - 1 - i) : i);
}

// The k-th entry of persistent CTA i of n in a split launch: its split_whole / n whole units
// on the boustrophedon walk, then the pieces of slice i that hold key tiles (-1: none left).
__device__ __forceinline__ int fwd_split_entry(const FwdParams& p, int k, int i, int n) {
    const int full = p.split_whole / n;
    if (k < full) return snake_unit(k, i, n);
    if (i >= p.split_slices) return -1;
    int want = k - full;
    for (int piece = 0; piece < 2; ++piece) {
        const int u = p.split_whole + 2 * i + piece;
        int b, g;
        SubTile st[2];
        fwd_dense_unit(p, u, b, g, st);
        if (fwd_unit_work(st) > 0 && want-- == 0) return u;
    }
    return -1;
}

// The k-th unit of a persistent CTA as a list index, -1 when the CTA has no more, -2 when a
// bounded wait gave up. Static launches stride over the list (snake_unit); dynamic ones take
// the next free entry with an atomic counter, and the producer publishes it in a 4-slot ring
// that every other role reads (fwd_read_unit) and releases.
template <class Ctl>
__device__ __forceinline__ int fwd_publish_unit(Ctl* ctl, int* fetch, int units, int k, volatile uint32_t* abort_flag,
                                                uint32_t* err, unsigned long long timeout_ns) {
    const int slot = k & 3;
    if (k >= 4 && !mbar_wait_bounded(smem_u32(&ctl->unit_empty[slot]), ((k >> 2) - 1) & 1u, abort_flag, err,
                                     timeout_ns))
        return -2;
    const int idx = atomicAdd(fetch, 1);
    const int u = idx < units ? idx : -1;
    reinterpret_cast<volatile int*>(ctl->unit_ring)[slot] = u;
    mbar_arrive(smem_u32(&ctl->unit_full[slot]));  // release: the ring entry is visible to its readers
    return u;
}
// Read the k-th published unit (every lane of the calling warp reads it); lane 0 releases the
// slot for the warp (one_thread: the caller is a single thread and releases it itself).
template <class Ctl>
__device__ __forceinline__ int fwd_read_unit(Ctl* ctl, int k, bool one_thread, volatile uint32_t* abort_flag,
                                             uint32_t* err, unsigned long long timeout_ns) {
    const int slot = k & 3;
    if (!mbar_wait_bounded(smem_u32(&ctl->unit_full[slot]), (k >> 2) & 1u, abort_flag, err, timeout_ns)) return -2;
    const int u = reinterpret_cast<volatile int*>(ctl->unit_ring)[slot];
    if (one_thread) {
        mbar_arrive(smem_u32(&ctl->unit_empty[slot]));
    } else {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&ctl->unit_empty[slot]));
    }
    return u;
}

template <int D, bool kVarlen>
__global__ void __launch_bounds__(kFwdThreads, 1)
    gqa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const FwdParams p,
                         const FwdVarlenParams vp) {
    using L = FwdSmem<D>;
    using Ctl = typename L::Ctl;
    constexpr int kStages = L::kStages;
    constexpr int kTileBytes = L::kTileBytes;
    constexpr int kChunkBytes = L::kChunkBytes;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    const uint32_t sQ = sbase + L::kQOff;
    const uint32_t sRing = sbase + L::kRingOff;
    const uint32_t sStage = sbase + L::kStageOff;
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + L::kCtlOff);
    volatile uint32_t* abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Persistent CTA: units blockIdx.x, blockIdx.x + gridDim.x, ... (units are ordered
    // longest first, so this striding spreads the causal work evenly over the SMs).
    const int cta = blockIdx.x;
    const int ncta = gridDim.x;
    // variable-length launches read the unit count the plan kernel wrote
    const int units = kVarlen ? *reinterpret_cast<const volatile int*>(vp.unit_count) : p.units;
    const bool dyn = kVarlen && vp.dynamic != 0;
    // static launches: the k-th unit of this CTA on the boustrophedon walk (-1: none left)
    auto static_unit = [&](int k) -> int {
        if (!kVarlen && p.split_slices > 0) {
            const int full = p.split_whole / ncta;
            if (k < full) return snake_unit(k, cta, ncta);
            return k - full < 2 ? ctl->split_entry[k - full] : -1;
        }
        if (k * ncta >= units) return -1;
        const int u = snake_unit(k, cta, ncta);
        return u < units ? u : -1;
    };

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&ctl->q_full), 1);
        mbar_init(smem_u32(&ctl->q_empty), 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(smem_u32(&ctl->full[i]), 1);
            mbar_init(smem_u32(&ctl->empty[i]), 1);
            mbar_init(smem_u32(&ctl->land[i]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&ctl->s_full[s]), 1);
            mbar_init(smem_u32(&ctl->p_full[s]), kFwdRows);
            mbar_init(smem_u32(&ctl->o_full[s]), 1);
            mbar_init(smem_u32(&ctl->o_empty[s]), kFwdRows);
        }
        mbar_init(smem_u32(&ctl->drain), 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(smem_u32(&ctl->unit_full[i]), 1);
            mbar_init(smem_u32(&ctl->unit_empty[i]), kUnitReaders);
        }
        ctl->abort = 0;
        if (!kVarlen && p.split_slices > 0) {
            const int full = p.split_whole / ncta;
            ctl->split_entry[0] = fwd_split_entry(p, full, cta, ncta);
            ctl->split_entry[1] = fwd_split_entry(p, full + 1, cta, ncta);
        }
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(&ctl->tmem_base), 512);
        tmem_relinquish();
    }
    if (threadIdx.x == 32) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    if (warp < 4) setmaxnreg_dec<kFwdCtlRegs>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued[kStages];
            uint32_t landed[kStages];  // copies that completed on land[] (ragged V tiles)
            bool last_land[kStages];
            for (int i = 0; i < kStages; ++i) {
                issued[i] = landed[i] = 0;
                last_land[i] = false;
            }
            uint32_t q_loads = 0;
            const uint32_t qbar = smem_u32(&ctl->q_full);
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int u = dyn ? fwd_publish_unit(ctl, vp.fetch, units, k, abort_flag, p.err, p.timeout_ns)
                                  : static_unit(k);
                if (u == -2) ok = false;
                if (u < 0) break;
                int g;
                SeqGeo geo;
                SubTile st[2];
                fwd_unit<kVarlen>(p, vp, u, geo, g, st);
                const int n_max = max(st[0].n_kv, st[1].n_kv);
                const int jb = st[1].n_kv > 0 ? min(st[0].j_begin, st[1].j_begin) : st[0].j_begin;
                // the previous unit's Q K^T products must be done before Q is replaced
                if (q_loads > 0 && !(ok = mbar_wait_bounded(smem_u32(&ctl->q_empty), (q_loads - 1) & 1u,
                                                            abort_flag, p.err, p.timeout_ns)))
                    break;
                const int nq = st[1].n_kv > 0 ? 2 : 1;
                mbar_arrive_expect_tx(qbar, nq * kTileBytes);
                for (int s = 0; s < nq; ++s)
                    for (int c = 0; c < L::kChunks; ++c)
                        tma_load_4d(sQ + s * kTileBytes + c * kChunkBytes, &tm_q, qbar, c * 64,
                                    geo.r_q + st[s].row0, st[s].head, geo.b_q);
                ++q_loads;
                for (int j = jb; j < n_max && ok; ++j) {
                    for (int t = 0; t < 2; ++t) {
                        if (!(ok = mbar_wait_bounded(smem_u32(&ctl->empty[stage]), phase ^ 1u, abort_flag,
                                                     p.err, p.timeout_ns)))
                            break;
                        // A V tile that runs past its sequence's last key may hold another
                        // sequence's rows or padding (even NaN); it lands on land[] and warp 3
                        // zeroes those rows before it signals full[] (P is 0 there, 0 * NaN is not).
                        const bool ragged = kVarlen && t == 1 && (j + 1) * kFwdKeys > geo.len_k;
                        const uint32_t fbar = smem_u32(ragged ? &ctl->land[stage] : &ctl->full[stage]);
                        mbar_arrive_expect_tx(fbar, kTileBytes);
                        const CUtensorMap* map = t ? &tm_v : &tm_k;
                        if (kVarlen && vp.table != nullptr) {
                            // one box per page (or per 128 keys of a large page); keys past the
                            // sequence read an out-of-range page, i.e. zeros
                            const int n_box = kFwdKeys / vp.box_rows;
                            for (int bi = 0; bi < n_box; ++bi) {
                                const int key0 = j * kFwdKeys + bi * vp.box_rows;
                                const int page = key0 < geo.len_k
                                                     ? __ldg(vp.table + (size_t)geo.b_k * vp.max_pages + key0 / vp.page_size)
                                                     : vp.num_pages;
                                const uint32_t dst = sRing + stage * kTileBytes + bi * vp.box_rows * 128;
                                for (int c = 0; c < L::kChunks; ++c)
                                    tma_load_4d(dst + c * kChunkBytes, map, fbar, c * 64, key0 % vp.page_size, g, page);
                            }
                        } else {
                            for (int c = 0; c < L::kChunks; ++c)
                                tma_load_4d(sRing + stage * kTileBytes + c * kChunkBytes, map, fbar, c * 64,
                                            geo.r_k + j * kFwdKeys, g, geo.b_k);
                        }
                        ++issued[stage];
                        if constexpr (kVarlen) {
                            last_land[stage] = ragged;
                            if (ragged) ++landed[stage];
                        }
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
            if (*abort_flag) {
                // let every copy this thread started land before the CTA exits
                if (q_loads) mbar_wait_drain(qbar, (q_loads - 1) & 1u, p.timeout_ns);
                for (int i = 0; i < kStages; ++i) {
                    if (kVarlen && last_land[i])
                        mbar_wait_drain(smem_u32(&ctl->land[i]), (landed[i] - 1u) & 1u, p.timeout_ns);
                    else if (issued[i])
                        mbar_wait_drain(smem_u32(&ctl->full[i]), (issued[i] - 1u) & 1u, p.timeout_ns);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ tcgen05 issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16(kFwdRows, kFwdKeys, 0, 0);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(kFwdRows, D, 0, 1);
            const uint32_t tS[2] = {tmem + 0u, tmem + 128u};
            const uint32_t tO[2] = {tmem + 256u, tmem + 256u + (uint32_t)D};
            // descriptors advance by constants (their start-address field is in 16-byte units)
            const uint64_t desc_q[2] = {umma_desc_sw128(sQ, 16, 1024), umma_desc_sw128(sQ + kTileBytes, 16, 1024)};
            int stage = 0;
            uint32_t phase = 0;
            uint32_t pph[2] = {0u, 0u};
            uint32_t o_uses[2] = {0u, 0u};  // units whose O_s epilogue must drain first
            uint32_t q_uses = 0;
            bool ok = true;

            auto acquire = [&](int& slot) -> bool {
                slot = stage;
                if (!mbar_wait_bounded(smem_u32(&ctl->full[stage]), phase, abort_flag, p.err,
                                       p.timeout_ns))
                    return false;
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
                tc_fence_after_sync();
                return true;
            };
            // S_s = Q_s K^T: M=128 rows, N=128 keys, K=D in steps of 16 (32 bytes of a
            // 128-byte swizzled row; the next 64 columns live in the next chunk).
            auto issue_qk = [&](int s, int kslot) {
                const uint64_t a0 = desc_q[s];
                const uint64_t b0 = umma_desc_sw128(sRing + kslot * kTileBytes, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t koff = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
                    tc_mma_ss(tS[s], a0 + koff, b0 + koff, idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            // O_s += P_s V: M=128 rows, N=D, K=128 keys in steps of 16. P (bf16, two per
            // column) sits in the first 64 columns of S_s; V is N-contiguous (d), with
            // the 64-column chunks LBO apart and 8-key groups 1024 bytes apart.
            auto issue_pv = [&](int s, int vslot, bool accumulate) {
                const uint64_t b0 = umma_desc_sw128(sRing + vslot * kTileBytes, kChunkBytes, 1024);
#pragma unroll
                for (int kk = 0; kk < kFwdKeys / 16; ++kk)
                    tc_mma_ts(tO[s], tS[s] + kk * 8, b0 + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                              (accumulate || kk > 0) ? 1u : 0u);
            };

            for (int k = 0; ok; ++k) {
                const int u = dyn ? fwd_read_unit(ctl, k, true, abort_flag, p.err, p.timeout_ns) : static_unit(k);
                if (u == -2) ok = false;
                if (u < 0) break;
                int g;
                SeqGeo geo;
                SubTile st[2];
                fwd_unit<kVarlen>(p, vp, u, geo, g, st);
                const int n_max = max(st[0].n_kv, st[1].n_kv);
                // KV tiles jb .. n_max-1; sub-tile s uses tiles st[s].j_begin .. st[s].n_kv-1
                const int jb = st[1].n_kv > 0 ? min(st[0].j_begin, st[1].j_begin) : st[0].j_begin;
                auto in_range = [&](int s, int jj) { return jj >= st[s].j_begin && jj < st[s].n_kv; };
                if (!(ok = mbar_wait_bounded(smem_u32(&ctl->q_full), q_uses & 1u, abort_flag, p.err,
                                             p.timeout_ns)))
                    break;
                ++q_uses;
                int kslot;
                if (!(ok = acquire(kslot))) break;
                for (int s = 0; s < 2; ++s)
                    if (in_range(s, jb)) {
                        issue_qk(s, kslot);
                        tc_commit(smem_u32(&ctl->s_full[s]));
                    }
                tc_commit(smem_u32(&ctl->empty[kslot]));
                if (n_max - jb == 1) tc_commit(smem_u32(&ctl->q_empty));
                for (int j = jb; j < n_max && ok; ++j) {
                    int vslot;
                    if (!(ok = acquire(vslot))) break;
                    const bool next = j + 1 < n_max;
                    // take the next K slot now, so each Q K^T follows its P V on the tensor
                    // pipe with no gap
                    int knext = -1;
                    if (next && !(ok = acquire(knext))) break;
                    for (int s = 0; s < 2 && ok; ++s) {
                        if (in_range(s, j)) {
                            if (!(ok = mbar_wait_bounded(smem_u32(&ctl->p_full[s]), pph[s], abort_flag,
                                                         p.err, p.timeout_ns)))
                                break;
                            pph[s] ^= 1u;
                            if (j == st[s].j_begin && o_uses[s] > 0) {
                                // the previous unit's epilogue must have read O_s
                                if (!(ok = mbar_wait_bounded(smem_u32(&ctl->o_empty[s]), (o_uses[s] - 1) & 1u,
                                                             abort_flag, p.err, p.timeout_ns)))
                                    break;
                            }
                            tc_fence_after_sync();
                            issue_pv(s, vslot, j > st[s].j_begin);
                            if (j == st[s].n_kv - 1) {
                                tc_commit(smem_u32(&ctl->o_full[s]));
                                ++o_uses[s];
                            }
                        }
                        if (s == 1) tc_commit(smem_u32(&ctl->empty[vslot]));
                        if (next) {
                            if (in_range(s, j + 1)) {
                                issue_qk(s, knext);
                                tc_commit(smem_u32(&ctl->s_full[s]));
                            }
                        }
                    }
                    if (ok && next) {
                        tc_commit(smem_u32(&ctl->empty[knext]));
                        if (j + 2 == n_max) tc_commit(smem_u32(&ctl->q_empty));  // last Q K^T issued
                    }
                }
            }
            if (*abort_flag) {
                // wait for the MMAs already issued before TMEM is released
                tc_commit(smem_u32(&ctl->drain));
                mbar_wait_drain(smem_u32(&ctl->drain), 0, p.timeout_ns);
            }
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ ragged-tile cleaner
        // Walks the same units and ring slots as the producer. For each V tile that runs
        // past its sequence's last key it waits for the copy on land[], zeroes the rows
        // past that key and releases the slot to the MMA issuer through full[].
        if constexpr (kVarlen) {
            int stage = 0;
            uint32_t land_uses[kStages];
            for (int i = 0; i < kStages; ++i) land_uses[i] = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int u = dyn ? fwd_read_unit(ctl, k, false, abort_flag, p.err, p.timeout_ns) : static_unit(k);
                if (u == -2) ok = false;
                if (u < 0) break;
                int g;
                SeqGeo geo;
                SubTile st[2];
                fwd_unit<kVarlen>(p, vp, u, geo, g, st);
                const int n_max = max(st[0].n_kv, st[1].n_kv);
                const int jb = st[1].n_kv > 0 ? min(st[0].j_begin, st[1].j_begin) : st[0].j_begin;
                for (int j = jb; j < n_max && ok; ++j) {
                    const int vstage = stage + 1 == kStages ? 0 : stage + 1;  // K at stage, V next
                    if ((j + 1) * kFwdKeys > geo.len_k) {
                        const uint32_t lbar = smem_u32(&ctl->land[vstage]);
                        bool got = true;
                        if (lane == 0)
                            got = mbar_wait_bounded(lbar, land_uses[vstage] & 1u, abort_flag, p.err,
                                                    p.timeout_ns);
                        got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
                        ++land_uses[vstage];
                        if (!got) {
                            ok = false;
                            break;
                        }
                        // rows keep .. 127 of every 128-byte column chunk (swizzle only
                        // permutes 16-byte units inside a row, so whole rows are zeroed)
                        const int keep = geo.len_k - j * kFwdKeys;  // 1 .. 127
                        const int n16 = (kFwdKeys - keep) * 8;      // 16-byte units per chunk
                        const uint32_t tile = sRing + vstage * kTileBytes + keep * 128;
                        for (int c = 0; c < L::kChunks; ++c)
                            for (int i = lane; i < n16; i += 32)
                                st_shared_v4(tile + c * kChunkBytes + i * 16, 0u, 0u, 0u, 0u);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&ctl->full[vstage]));
                    }
                    stage = vstage + 1 == kStages ? 0 : vstage + 1;
                }
            }
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax warpgroups
        setmaxnreg_inc<kFwdSoftmaxRegs>();
        const int s = (warp - 4) >> 2;
        const int quad = warp & 3;         // TMEM lane quadrant this warp may access
        const int r = quad * 32 + lane;    // row within the sub-tile
        const uint32_t lane_sel = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + lane_sel + (uint32_t)(s * 128);
        const uint32_t tO = tmem + lane_sel + 256u + (uint32_t)(s * D);
        const float sl2 = p.scale_log2;
        if (!kVarlen && cta < p.split_slices) {
            // this CTA's partial rows start as "no key": a piece (or sub-tile) that holds no
            // tile leaves them so, and the merge kernel skips them (the epilogue below, in this
            // same thread, overwrites the rows it computes)
            for (int i = 0; i < 2; ++i) p.part_lse[((size_t)(2 * cta + i) * 2 + s) * kFwdRows + r] = -INFINITY;
        }
        uint32_t sph = 0, oph = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int u = dyn ? fwd_read_unit(ctl, k, false, abort_flag, p.err, p.timeout_ns) : static_unit(k);
            if (u == -2) ok = false;
            if (u < 0) break;
            int g;
            SeqGeo geo;
            SubTile st[2];
            fwd_unit<kVarlen>(p, vp, u, geo, g, st);
            const SubTile me = st[s];
            if (me.n_kv == 0) continue;
            const int off = geo.len_k - geo.len_q;
            const int pos = off + me.row0 + r;  // absolute position of this query row
            const int lo = pos - p.window + 1;  // first key inside the window (window > 0)
            float m = -INFINITY;  // running max of scaled scores (log2 units)
            float l = 0.f;        // running sum of exp2(score - m)
            for (int j = me.j_begin; j < me.n_kv; ++j) {
                if (!(ok = mbar_wait_bounded(smem_u32(&ctl->s_full[s]), sph, abort_flag, p.err,
                                             p.timeout_ns)))
                    break;
                sph ^= 1u;
                tc_fence_after_sync();
                uint32_t sr[4][32];
                tmem_ld32(tS + 0, sr[0]);
                tmem_ld32(tS + 32, sr[1]);
                tc_wait_ld();
                reg_fence32(sr[0]);
                reg_fence32(sr[1]);
                tmem_ld32(tS + 64, sr[2]);
                tmem_ld32(tS + 96, sr[3]);
                const bool diag = j >= me.masked_from || j < me.lo_masked_end;
                // row max: eight independent chains of 3-input max, then a small tree; the
                // first 64 columns are reduced while the last 64 are still loading
                float mx[8];
#pragma unroll
                for (int qd = 0; qd < 8; ++qd) mx[qd] = -INFINITY;
                if (!diag) {
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int qd = 0; qd < 8; ++qd) {
                            mx[qd] = max3f(mx[qd], __uint_as_float(sr[c][4 * qd]), __uint_as_float(sr[c][4 * qd + 1]));
                            mx[qd] = max3f(mx[qd], __uint_as_float(sr[c][4 * qd + 2]), __uint_as_float(sr[c][4 * qd + 3]));
                        }
                }
                tc_wait_ld();
                reg_fence32(sr[2]);
                reg_fence32(sr[3]);
                if (diag) {
                    if (j >= me.masked_from) {
                        // the causal diagonal (sub-tile uniform): columns > lim are in the future
                        const int lim = pos - j * kFwdKeys;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (c * 32 + e > lim) sr[c][e] = __float_as_uint(-INFINITY);
                    }
                    if (j < me.lo_masked_end) {
                        // the window's lower edge (sub-tile uniform): columns < lim_lo are before it
                        const int lim_lo = lo - j * kFwdKeys;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (c * 32 + e < lim_lo) sr[c][e] = __float_as_uint(-INFINITY);
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (!diag && c < 2) continue;  // already reduced
#pragma unroll
                    for (int qd = 0; qd < 8; ++qd) {
                        mx[qd] = max3f(mx[qd], __uint_as_float(sr[c][4 * qd]), __uint_as_float(sr[c][4 * qd + 1]));
                        mx[qd] = max3f(mx[qd], __uint_as_float(sr[c][4 * qd + 2]), __uint_as_float(sr[c][4 * qd + 3]));
                    }
                }
                const float tmax = fmaxf(max3f(mx[0], mx[1], mx[2]),
                                         max3f(max3f(mx[3], mx[4], mx[5]), mx[6], mx[7]));
                const float m_new = fmaxf(m, tmax * sl2);
                const bool refresh = m_new > m + kRescaleThreshold;
                // warp-uniform branch, rarely taken after a unit's first tile: the MUFU op for
                // alpha stays off the common path (it would queue behind the exponentials)
                float alpha = 1.f;  // < 2^-8 where this row's max moved, else exactly 1
                if (__any_sync(0xffffffffu, refresh)) {
                    alpha = refresh ? ex2_approx(m - m_new) : 1.f;
                    l *= alpha;
                    m = refresh ? m_new : m;
                }
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                const uint64_t sl2x2 = f2_pack(sl2, sl2);
                const uint64_t negm2 = f2_pack(neg_m, neg_m);
                uint64_t lacc[4] = {0ull, 0ull, 0ull, 0ull};
                // p = 2^(s * scale * log2(e) - m), two columns per packed instruction
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint64_t x = f2_fma(
                            f2_pack(__uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1])), sl2x2, negm2);
                        float x0, x1;
                        f2_unpack(x, x0, x1);
                        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                        lacc[e & 3] = f2_add(lacc[e & 3], f2_pack(p0, p1));
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(tS + c * 16, pk);
                }

                {
                    const uint64_t s01 = f2_add(f2_add(lacc[0], lacc[1]), f2_add(lacc[2], lacc[3]));
                    float a0, a1;
                    f2_unpack(s01, a0, a1);
                    l += a0 + a1;
                }
                if (__any_sync(0xffffffffu, alpha != 1.f) && j > me.j_begin) {
                    // O_s has absorbed all earlier P V products (their completion is ordered
                    // before S_j's commit) and this tile's P V waits for p_full below: rescale
                    // this row in place, after the exponentials, when S no longer holds
                    // registers, so all column chunks load behind one wait
                    uint32_t orr[D / 32][32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, orr[c]);
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        reg_fence32(orr[c]);
#pragma unroll
                        for (int e = 0; e < 32; ++e) orr[c][e] = __float_as_uint(__uint_as_float(orr[c][e]) * alpha);
                        tmem_st32(tO + c * 32, orr[c]);
                    }
                }
                tc_wait_st();
                tc_fence_before_sync();
                mbar_arrive(smem_u32(&ctl->p_full[s]));
            }
            if (!ok || !(ok = mbar_wait_bounded(smem_u32(&ctl->o_full[s]), oph, abort_flag, p.err,
                                                p.timeout_ns)))
                break;
            oph ^= 1u;
            tc_fence_after_sync();
            if (!kVarlen && p.split_slices > 0 && u >= p.split_whole) {
                // a piece of a split unit: fp32 O / l and the log2-domain log-sum-exp of this
                // row over the piece's keys (a row that saw none writes zeros and -inf); the
                // combine kernel merges the pieces
                // rows chunk-major (float4 chunk e of row r at e * 128 + r): a warp's store
                // of one chunk of its 32 rows is one contiguous 512-byte run
                const size_t pblk = (size_t)(u - p.split_whole) * 2 + s;
                const size_t prow = pblk * kFwdRows + r;
                const bool any = l > 0.f;
                const float inv_l = any ? 1.f / l : 0.f;
                float4* dst = reinterpret_cast<float4*>(p.part + pblk * kFwdRows * D) + r;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t orr[32];
                    tmem_ld32(tO + c * 32, orr);
                    tc_wait_ld();
                    reg_fence32(orr);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[(c * 8 + e) * kFwdRows] = make_float4(__uint_as_float(orr[4 * e]) * inv_l, __uint_as_float(orr[4 * e + 1]) * inv_l,
                                                     __uint_as_float(orr[4 * e + 2]) * inv_l, __uint_as_float(orr[4 * e + 3]) * inv_l);
                }
                tc_fence_before_sync();
                mbar_arrive(smem_u32(&ctl->o_empty[s]));
                p.part_lse[prow] = any ? m + __log2f(l) : -INFINITY;
                continue;
            }
            const int row = me.row0 + r;
            const bool row_ok = row < geo.len_q;
            const float inv_l = 1.f / l;
            // row 0 of this warp's 32 output rows, and the row stride (elements)
            __nv_bfloat16* out0;
            long long ost;
            if constexpr (kVarlen) {
                out0 = p.o + geo.b_q * vp.o_sb + me.head * vp.o_sh + (long long)(geo.r_q + me.row0 + quad * 32) * vp.o_st;
                ost = vp.o_st;
            } else {
                out0 = p.o + (((size_t)geo.b_q * p.Hq + me.head) * (size_t)p.Tq + (size_t)(me.row0 + quad * 32)) * D;
                ost = D;
            }
            const int rows_left = geo.len_q - me.row0 - quad * 32;  // of the warp's rows, those that exist
            const uint32_t stg = sStage + (uint32_t)(warp - 4) * L::kStageWarpBytes;
            // 64 columns at a time: O / l as bf16 into the warp's staging rows (16-byte chunk q of
            // row t at chunk q ^ (t & 7), so 8 consecutive rows fill all banks), then back out as
            // whole 128-byte row segments, 4 rows per store instruction
#pragma unroll 1
            for (int h = 0; h < D / 64; ++h) {
                uint32_t pw[32];
                {
                    uint32_t orr[2][32];
                    tmem_ld32(tO + h * 64, orr[0]);
                    tmem_ld32(tO + h * 64 + 32, orr[1]);
                    tc_wait_ld();
                    reg_fence32(orr[0]);
                    reg_fence32(orr[1]);
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pw[c2 * 16 + e] = pack_bf16x2(__uint_as_float(orr[c2][2 * e]) * inv_l,
                                                          __uint_as_float(orr[c2][2 * e + 1]) * inv_l);
                }
                if (h == D / 64 - 1) {
                    // O_s has been read: the next unit's first P V may overwrite it
                    tc_fence_before_sync();
                    mbar_arrive(smem_u32(&ctl->o_empty[s]));
                }
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    st_shared_v4(stg + lane * 128 + ((q ^ (lane & 7)) << 4), pw[4 * q], pw[4 * q + 1], pw[4 * q + 2],
                                 pw[4 * q + 3]);
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int t = i * 4 + (lane >> 3), q = lane & 7;
                    const uint4 v = ld_shared_v4(stg + t * 128 + ((q ^ (t & 7)) << 4));
                    if (t < rows_left) *reinterpret_cast<uint4*>(out0 + (long long)t * ost + h * 64 + q * 8) = v;
                }
                __syncwarp();
            }
            if (p.lse != nullptr && row_ok) {
                const size_t li = kVarlen ? ((size_t)geo.b_q * p.Hq + me.head) * (size_t)vp.rows_q + geo.r_q + row
                                          : ((size_t)geo.b_q * p.Hq + me.head) * (size_t)p.Tq + row;
                p.lse[li] = (m + __log2f(l)) * 0.69314718055994530942f;
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}


// ---------------------------------------------------------------- split-launch merge
// Row r of sub-tile s of split unit su has one partial row per slice that reaches the unit:
// fp32 O / l over the piece's keys (stored chunk-major: float4 chunk e of row r of a (slot,
// sub-tile) block at e * 128 + r) and the log2-domain log-sum-exp of those keys (-inf when the
// piece held none of this row's keys, or no tile of the sub-tile, or is absent: the forward
// kernel writes -inf first). With M the largest and w_q = 2^(lse_q - M), the row is
// O = sum_q w_q O_q / sum_q w_q with log-sum-exp M + log2(sum_q w_q): the merge of the
// split-KV decode partials, summed in slice order, so the result is fixed.
// One warp per 32 rows x 32 columns of one (unit, sub-tile), a lane per row: lane t first
// finds the slot of candidate run c0 + t, then every load of a chunk for the warp's rows is one
// 512-byte run.
constexpr int kCombineWarps = 8;

template <int D>
__global__ void __launch_bounds__(kCombineWarps * 32)
    gqa_fwd_split_combine_kernel(const FwdParams p, long long n_warps) {
    const long long w = (long long)blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
    if (w >= n_warps) return;  // n_warps = split units x 2 sub-tiles x 4 row quarters x D / 32
    constexpr int kColGroups = D / 32;
    const int lane = threadIdx.x & 31;
    const int cc = (int)(w % kColGroups);
    const long long wr = w / kColGroups;
    const int su = (int)(wr >> 3);
    const int s = (int)(wr >> 2) & 1;
    const int r = (int)(wr & 3) * 32 + lane;
    int b, g;
    SubTile st[2];
    fwd_decode_unit(p, p.split_whole + su, b, g, st);
    const SubTile me = s ? st[1] : st[0];
    if (me.n_kv == 0 || me.row0 + (r & ~31) >= p.Tq) return;  // no such sub-tile, or rows past T_q
    // runs c0 .. c1-1 of this unit's lane reach its group's ticks [x0, x1): c0 is the last
    // one starting at or before x0, c1 the first one starting at or after x1
    const int L = p.split_group;
    const int m = p.split_slices / L;
    const int gr = su / L, ln = su - gr * L;
    const long long N = (p.Tk - 1) / kFwdKeys + 1;
    const long long T = (long long)((p.units - p.split_whole) / L) * N;
    const long long x0 = gr * N, x1 = x0 + N;
    const int c0 = (int)fwd_muldiv((x0 + 1) * m - 1, 1, T);
    const int c1 = (int)min((long long)m, fwd_muldiv(x1 * m + T - 1, 1, T));
    auto slot_of = [&](int c) { return 2 * (c * L + ln) + (fwd_muldiv(T, c, m) < x0 ? 1 : 0); };
    float M = -INFINITY;
    for (int cb = c0; cb < c1; cb += 32) {
        const int mine = cb + lane < c1 ? slot_of(cb + lane) : 0;
        const int n = min(32, c1 - cb);
        for (int t = 0; t < n; ++t) {
            const size_t blk = (size_t)__shfl_sync(0xffffffffu, mine, t) * 2 + s;
            M = fmaxf(M, p.part_lse[blk * kFwdRows + r]);
        }
    }
    const int row = me.row0 + r;
    float wsum = 0.f;
    __nv_bfloat16* out = p.o + (((size_t)b * p.Hq + me.head) * (size_t)p.Tq + row) * D;
    {
        float acc[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[e] = 0.f;
        for (int cb = c0; cb < c1; cb += 32) {
            const int mine = cb + lane < c1 ? slot_of(cb + lane) : 0;
            const int n = min(32, c1 - cb);
            for (int t = 0; t < n; ++t) {
                const size_t blk = (size_t)__shfl_sync(0xffffffffu, mine, t) * 2 + s;
                const float lq = p.part_lse[blk * kFwdRows + r];
                const float wq = lq == -INFINITY ? 0.f : ex2_approx(lq - M);
                wsum += wq;
                const float4* src = reinterpret_cast<const float4*>(p.part + blk * kFwdRows * D) + r;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float4 v = src[(cc * 8 + e) * kFwdRows];
                    acc[4 * e] += wq * v.x;
                    acc[4 * e + 1] += wq * v.y;
                    acc[4 * e + 2] += wq * v.z;
                    acc[4 * e + 3] += wq * v.w;
                }
            }
        }
        if (row < p.Tq) {
            const float inv = 1.f / wsum;  // > 0: every row sees at least one key in some piece
            uint4 v4[4];
            uint32_t* pw = reinterpret_cast<uint32_t*>(v4);
#pragma unroll
            for (int e = 0; e < 16; ++e) pw[e] = pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
            uint4* dst = reinterpret_cast<uint4*>(out + cc * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = v4[e];
        }
    }
    if (p.lse != nullptr && cc == 0 && row < p.Tq)
        p.lse[((size_t)b * p.Hq + me.head) * (size_t)p.Tq + row] = (M + __log2f(wsum)) * 0.69314718055994530942f;
}

// ---------------------------------------------------------------- variable-length plan
// One CTA. Checks every sequence's bounds against the tensors, then lists the units
// that have work, ordered by decreasing KV-tile count (a counting sort over buckets),
// so the persistent kernel's boustrophedon walk keeps its balance when sequences
// differ in length. Workspace: ws[0] = unit count, units from ws[kPlanHeaderInts].
// A sequence outside its tensor (or with more queries than keys) sets
// kDevErrBadSeqlens and an empty list: nothing is computed, nothing is written.
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 4 * kPlanThreads;
constexpr int kPlanHeaderInts = 64;  // 256 bytes: ws[0] = unit count, ws[1] = fetch counter
// Launches of up to this many sequences list their units sequence-major (longest sequence
// first, each sequence's longest row levels first) for dynamic fetching: the units a CTA
// takes next then belong to the few sequences in flight, whose K/V stays in L2.
constexpr int kPlanMaxDynamicSeqs = kPlanThreads;

__global__ void __launch_bounds__(kPlanThreads, 1)
    gqa_fwd_varlen_plan_kernel(const FwdParams p, const FwdVarlenParams vp, int S, int max_q,
                               long long n_cand, int* ws) {
    __shared__ int hist[kPlanBuckets];
    __shared__ int warp_sum[32];
    __shared__ int bad;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    for (int i = tid; i < kPlanBuckets; i += kPlanThreads) hist[i] = 0;
    if (tid == 0) bad = 0;
    __syncthreads();
    for (int s = tid; s < S; s += kPlanThreads) {
        int bq, rq, lq, bk, rk, lk;
        fwd_seq_side(vp.cu_q, vp.len_q, vp.rows_q, s, bq, rq, lq);
        fwd_seq_side(vp.cu_k, vp.len_k, vp.rows_k, s, bk, rk, lk);
        const bool ok = rq >= 0 && lq >= 0 && (long long)rq + lq <= vp.rows_q && rk >= 0 && lk >= 0 &&
                        (long long)rk + lk <= vp.rows_k && lq <= lk && lq <= max_q;
        if (!ok) bad = 1;
    }
    __syncthreads();
    if (bad) {
        if (tid == 0) {
            ws[0] = 0;
            ws[1] = 0;
            atomicOr(p.err, kDevErrBadSeqlens);
        }
        return;
    }
    if (vp.dynamic) {
        // sequence-major list: rank the sequences by key count (longest first, ties by index),
        // give each its units' range by a scan over ranks, then write its units with the
        // longest row levels first. One thread per sequence (S <= kPlanMaxDynamicSeqs).
        int* key = hist;                     // [S] key counts
        int* cnt_by_rank = hist + kPlanThreads;
        const bool pair = (p.unit_flags & kUnitPairHeads) != 0;
        const int rows_per_lvl = pair ? kFwdRows : 2 * kFwdRows;
        int lq = 0, lk = 0, cnt = 0, rank = 0;
        if (tid < S) {
            int bq, rq, bk, rk;
            fwd_seq_side(vp.cu_q, vp.len_q, vp.rows_q, tid, bq, rq, lq);
            fwd_seq_side(vp.cu_k, vp.len_k, vp.rows_k, tid, bk, rk, lk);
            cnt = (lq + rows_per_lvl - 1) / rows_per_lvl * vp.n_h;
            key[tid] = lk;
        }
        __syncthreads();
        if (tid < S) {
            for (int o = 0; o < S; ++o) rank += key[o] > lk || (key[o] == lk && o < tid);
            cnt_by_rank[rank] = cnt;
        }
        __syncthreads();
        // exclusive scan of the counts over ranks: rank r starts after ranks 0 .. r-1
        int v = tid < S ? cnt_by_rank[tid] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_sum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int x = warp_sum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            warp_sum[lane] = x;
        }
        __syncthreads();
        incl += warp > 0 ? warp_sum[warp - 1] : 0;
        const int total = warp_sum[31];
        __syncthreads();
        cnt_by_rank[tid] = incl - v;  // exclusive offset of rank tid
        __syncthreads();
        if (tid < S && cnt > 0) {
            int* list = ws + kPlanHeaderInts + cnt_by_rank[rank];
            const int n_lvl_s = cnt / vp.n_h;
            for (int lvl = n_lvl_s - 1; lvl >= 0; --lvl)
                for (int h = 0; h < vp.n_h; ++h) *list++ = (tid * vp.n_lvl + lvl) * vp.n_h + h;
        }
        if (tid == 0) {
            ws[0] = total;
            ws[1] = 0;
        }
        return;
    }
    for (long long c = tid; c < n_cand; c += kPlanThreads) {
        SeqGeo geo;
        int g;
        SubTile st[2];
        fwd_varlen_unit(p, vp, (int)c, geo, g, st);
        const int w = fwd_unit_work(st);
        if (w > 0) atomicAdd(&hist[min(w, kPlanBuckets - 1)], 1);
    }
    __syncthreads();
    // bucket b starts after every unit in buckets above it: thread t owns buckets
    // 4t .. 4t+3; an ascending block scan of the per-thread totals gives the rest
    int cnt[4], mine = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        cnt[e] = hist[4 * tid + e];
        mine += cnt[e];
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int x = warp_sum[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        warp_sum[lane] = x;
    }
    __syncthreads();
    incl += warp > 0 ? warp_sum[warp - 1] : 0;
    const int total = warp_sum[31];
    int cursor = total - incl;  // units in buckets owned by higher threads
#pragma unroll
    for (int e = 3; e >= 0; --e) {
        hist[4 * tid + e] = cursor;
        cursor += cnt[e];
    }
    __syncthreads();
    int* list = ws + kPlanHeaderInts;
    for (long long c = tid; c < n_cand; c += kPlanThreads) {
        SeqGeo geo;
        int g;
        SubTile st[2];
        fwd_varlen_unit(p, vp, (int)c, geo, g, st);
        const int w = fwd_unit_work(st);
        if (w > 0) list[atomicAdd(&hist[min(w, kPlanBuckets - 1)], 1)] = (int)c;
    }
    if (tid == 0) {
        ws[0] = total;
        ws[1] = 0;
    }
}

}  // namespace gqa
