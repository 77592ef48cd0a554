// Decode over a bf16 KV cache (T_q = 1, or a short chunk of T_q <= 16 new queries):
// split-KV partials + log-sum-exp combine.
//
// Query row i of head a sits at position T_k - T_q + i and sees keys up to it (for
// T_q = 1 every cached key) -- "注意力家族", section 最小语义实现: the suffix case;
// with a window it sees only its `window` most recent positions. Decode is
// bound by the bytes of K/V it must stream ("注意力家族", section KV Cache 成本: the
// cache is read again at every decode step; "Attention Architecture Evolution",
// section Full Attention: decode is limited by memory bandwidth), so the kernel
// reads every K/V byte of a KV head exactly once for all H_q/H_kv query heads that
// share it ("A Visual Guide to Attention", section "How many KV heads?").
//
// Work unit = (split of the key axis, KV head g, batch b, chunk of 16 query rows of
// group g, the G heads' T_q rows packed together). One producer warp streams 128-key K and V tiles with TMA (128-byte
// swizzle) through a ring deep enough to keep >= 128 KB in flight per SM. Four
// consumer warps each take 32 keys of every tile and keep their own running
// (max, sum, O); scores and P.V use warp-level bf16 tensor-core MMAs with the query
// heads as the M dimension; row maxima and sums combine across the four lanes of a
// row with warp shuffles. At the end the four warps merge through shared memory and
// the CTA writes either the final bf16 row (one split) or a normalised fp32 partial
// plus its log2-domain log-sum-exp (several splits), which gqa_decode_combine merges
// in fixed split order.
#pragma once

#include "sm100_ptx.cuh"

namespace gqa {

constexpr int kDecKeys = 128;     // keys per streamed tile
constexpr int kDecRows = 16;      // query rows per CTA (one m16 tile)
constexpr int kDecConsumers = 4;  // consumer warps
constexpr int kDecThreads = 32 * (1 + kDecConsumers);

struct DecParams {
    int B, Hq, Hkv, Tq, Tk, G;
    int n_hc;        // chunks of 16 query rows per group (a group has G * Tq rows)
    int splits;      // key-axis splits
    int blk_per_split;
    int blk_first;   // first key block any row can see
    int n_blk;       // ceil(Tk / 128)
    int window;      // > 0: each row sees only its `window` most recent positions
    float scale_log2;
    const __nv_bfloat16* q;  // [B, Hq, Tq, D]
    __nv_bfloat16* o;        // [B, Hq, Tq, D] (written when splits == 1)
    float* ws_o;             // [splits, B * Hq * Tq, D] normalised partial outputs
    float* ws_lse;           // [splits, B * Hq * Tq] log2-domain log-sum-exp
    uint32_t* err;
    unsigned long long timeout_ns;
    // ---- per-sequence cache lengths (the kVarlen instantiation only)
    const int* seqlens;  // [B] cached keys of each sequence (its Tq queries are the last Tq)
    const int* table;    // [B, max_pages] pool page of each page of a sequence, or null
    int max_pages;       // block-table row length
    int page_size;       // keys per page (16, 32, 64 or a multiple of 128)
    int box_rows;        // rows per TMA box: min(page_size, 128)
    int num_pages;       // pages in the pool; page coordinates past it read as zeros
    int capacity;        // most keys a sequence may hold
};

template <int D>
struct DecSmem {
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkBytes = kDecKeys * 128;
    static constexpr int kTileBytes = kChunks * kChunkBytes;   // one K or V tile
    static constexpr int kStageBytes = 2 * kTileBytes;         // K + V
    static constexpr int kStages = D == 128 ? 3 : 6;
    static constexpr int kCtlOff = kStages * kStageBytes;
    struct Ctl {
        uint64_t full[kStages];
        uint64_t empty[kStages];
        uint32_t abort;
    };
    // merge area (reuses the ring once streaming is done): per warp m,l[16] + O[16][D]
    static constexpr int kMergeBytes = kDecConsumers * (2 * kDecRows + kDecRows * D) * 4;
    static_assert(kMergeBytes <= kCtlOff, "merge area must fit in the ring");
    static constexpr int kBytes = kCtlOff + (int)sizeof(Ctl) + 1024;
};

// Byte offset of 16-byte unit (row, col8) inside a 128-byte-swizzled tile of 128-byte rows.
__device__ __forceinline__ uint32_t sw128_off(int row, int d) {
    const int chunk = d >> 6;
    const int unit = ((d & 63) >> 3) ^ (row & 7);
    return (uint32_t)(chunk * (kDecKeys * 128) + row * 128 + unit * 16);
}

// bf16 pair (keys k, k+1; k in the low half) with the keys at or past `end` zeroed.
__device__ __forceinline__ uint32_t clear_past(uint32_t pair, int k, int end) {
    return k >= end ? 0u : (k + 1 >= end ? (pair & 0xFFFFu) : pair);
}

template <int D, bool kVarlen>
__global__ void __launch_bounds__(kDecThreads, 1)
    gqa_decode_sm100_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const DecParams p) {
    using L = DecSmem<D>;
    using Ctl = typename L::Ctl;
    constexpr int kStages = L::kStages;
    constexpr int NT = D / 8;  // n8 tiles of the output row

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + L::kCtlOff);
    volatile uint32_t* abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int g = blockIdx.y / p.n_hc;
    const int hc = blockIdx.y - g * p.n_hc;
    const int b = blockIdx.z;
    int Tk = p.Tk, blk0, blk1;
    if constexpr (kVarlen) {
        // this sequence's own length: its key blocks are shared out over the splits
        Tk = __ldg(p.seqlens + b);
        if (Tk < p.Tq || Tk > p.capacity) {  // uniform over the CTA: nothing waits yet
            if (threadIdx.x == 0) atomicOr(p.err, kDevErrBadSeqlens);
            return;
        }
        const int n_blk = (Tk + kDecKeys - 1) / kDecKeys;
        const int key_lo = p.window > 0 ? max(0, Tk - p.Tq - p.window + 1) : 0;
        const int first = key_lo / kDecKeys;
        const int per = (n_blk - first + p.splits - 1) / p.splits;
        blk0 = first + split * per;
        blk1 = min(blk0 + per, n_blk);
    } else {
        blk0 = p.blk_first + split * p.blk_per_split;
        blk1 = min(blk0 + p.blk_per_split, p.n_blk);
    }
    const int t_end = min(blk1 * kDecKeys, Tk);
    // Query rows of group g: the G heads' Tq rows each, contiguous in q ((a, i) order).
    const int group_rows = p.G * p.Tq;
    const int rbase = hc * kDecRows;                            // first row of this CTA
    const int nrows = min(kDecRows, group_rows - rbase);        // valid rows in the chunk
    const size_t row0 = ((size_t)b * p.Hq + (size_t)g * p.G) * p.Tq + rbase;  // flat row id
    // rows see keys up to their own position (Tk - Tq + i) and, in a window, from
    // position - window + 1; tiles touching either bound are masked element-wise
    const int pos_min = Tk - p.Tq;
    const int lo_max = p.window > 0 ? Tk - p.window : -1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(smem_u32(&ctl->full[i]), 1);
            mbar_init(smem_u32(&ctl->empty[i]), kDecConsumers);
        }
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == 32) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    __syncthreads();

    float* mrg = reinterpret_cast<float*>(smem);  // merge area, valid after the loop

    if (warp == 0 && kVarlen) {
        // Whole warp: lanes look up the pool pages of a tile's boxes, lane 0 issues.
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued[kStages];
        for (int i = 0; i < kStages; ++i) issued[i] = 0;
        const bool paged = p.table != nullptr;
        const int n_box = paged ? kDecKeys / p.box_rows : 1;
        for (int blk = blk0; blk < blk1; ++blk) {
            int page = b, row = blk * kDecKeys;  // contiguous cache: batch b, rows from blk*128
            if (paged && lane < n_box) {
                const int key0 = blk * kDecKeys + lane * p.box_rows;
                row = key0 % p.page_size;
                page = key0 < Tk ? __ldg(p.table + (size_t)b * p.max_pages + key0 / p.page_size)
                                 : p.num_pages;  // past the sequence: an out-of-range page reads zeros
            }
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait_bounded(smem_u32(&ctl->empty[stage]), phase ^ 1u, abort_flag, p.err,
                                       p.timeout_ns);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
            const uint32_t fbar = smem_u32(&ctl->full[stage]);
            const uint32_t sK = sbase + stage * L::kStageBytes;
            if (lane == 0) mbar_arrive_expect_tx(fbar, L::kStageBytes);
            __syncwarp();
            // lane bi issues the copies of box bi (small pages need many boxes per tile)
            if (lane < n_box) {
                const uint32_t dst = sK + lane * p.box_rows * 128;
                for (int c = 0; c < L::kChunks; ++c) {
                    tma_load_4d(dst + c * L::kChunkBytes, &tm_k, fbar, c * 64, row, g, page);
                    tma_load_4d(dst + L::kTileBytes + c * L::kChunkBytes, &tm_v, fbar, c * 64, row, g, page);
                }
            }
            ++issued[stage];
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (lane == 0 && *abort_flag)
            for (int i = 0; i < kStages; ++i)
                if (issued[i])
                    mbar_wait_drain(smem_u32(&ctl->full[i]), (issued[i] - 1u) & 1u, p.timeout_ns);
        __syncthreads();  // pairs with the consumers' barrier before the merge
        __syncthreads();
    } else if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued[kStages];
            for (int i = 0; i < kStages; ++i) issued[i] = 0;
            for (int blk = blk0; blk < blk1; ++blk) {
                if (!mbar_wait_bounded(smem_u32(&ctl->empty[stage]), phase ^ 1u, abort_flag, p.err,
                                       p.timeout_ns))
                    break;
                const uint32_t fbar = smem_u32(&ctl->full[stage]);
                mbar_arrive_expect_tx(fbar, L::kStageBytes);
                const uint32_t sK = sbase + stage * L::kStageBytes;
                for (int c = 0; c < L::kChunks; ++c) {
                    tma_load_4d(sK + c * L::kChunkBytes, &tm_k, fbar, c * 64, blk * kDecKeys, g, b);
                    tma_load_4d(sK + L::kTileBytes + c * L::kChunkBytes, &tm_v, fbar, c * 64,
                                blk * kDecKeys, g, b);
                }
                ++issued[stage];
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (*abort_flag)
                for (int i = 0; i < kStages; ++i)
                    if (issued[i])
                        mbar_wait_drain(smem_u32(&ctl->full[i]), (issued[i] - 1u) & 1u, p.timeout_ns);
        }
        __syncthreads();  // pairs with the consumers' barrier before the merge
        __syncthreads();
    } else {
        const int cw = warp - 1;  // consumer index: keys [cw*32, cw*32+32) of every tile
        const int r_lo = lane >> 2;
        const int c2 = (lane & 3) * 2;
        // Q fragments (A operand, rows = query rows). Rows beyond the group are zero.
        uint32_t qa[D / 16][4];
        // absolute positions of this thread's two rows, and the first key they see
        int rpos[2], rlo[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int rr = rbase + r_lo + 8 * h;
            rpos[h] = Tk - p.Tq + rr % p.Tq;
            rlo[h] = p.window > 0 ? rpos[h] - p.window + 1 : -1;
        }
        {
            const __nv_bfloat16* q0 = p.q + row0 * D;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int row = r_lo + (e & 1) * 8;
                    const int col = ks * 16 + c2 + (e >> 1) * 8;
                    qa[ks][e] = row < nrows
                                    ? *reinterpret_cast<const uint32_t*>(q0 + (size_t)row * D + col)
                                    : 0u;
                }
            }
        }
        float m[2] = {-INFINITY, -INFINITY};  // rows r_lo and r_lo + 8, log2 units
        float l[2] = {0.f, 0.f};              // this thread's share of the row sums
        float oacc[NT][4];
#pragma unroll
        for (int i = 0; i < NT; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;

        int stage = 0;
        uint32_t phase = 0;
        const float sl2 = p.scale_log2;
        for (int blk = blk0; blk < blk1; ++blk) {
            if (!mbar_wait_bounded(smem_u32(&ctl->full[stage]), phase, abort_flag, p.err, p.timeout_ns))
                break;
            const uint32_t sK = sbase + stage * L::kStageBytes;
            const uint32_t sV = sK + L::kTileBytes;
            // ---- S = Q K^T for this warp's 32 keys: 4 n8 tiles
            float sacc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int mi = lane >> 3, rr = lane & 7;
                    const int key = cw * 32 + np * 16 + (mi >> 1) * 8 + rr;
                    const int d = ks * 16 + (mi & 1) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(sK + sw128_off(key, d), b0, b1, b2, b3);
                    mma_bf16_16816(sacc[np * 2], qa[ks], b0, b1);
                    mma_bf16_16816(sacc[np * 2 + 1], qa[ks], b2, b3);
                }
            }
            // keys past the split's end, after the row's position or before its window
            if (blk * kDecKeys + kDecKeys > min(t_end, pos_min + 1) || blk * kDecKeys < lo_max) {
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = blk * kDecKeys + cw * 32 + nt * 8 + c2 + (e & 1);
                        const int h = e >> 1;
                        if (key >= t_end || key > rpos[h] || key < rlo[h]) sacc[nt][e] = -INFINITY;
                    }
            }
            // ---- online softmax, one row half at a time
            uint32_t pa[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float mx = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) mx = fmaxf(mx, fmaxf(sacc[nt][2 * h], sacc[nt][2 * h + 1]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_new = fmaxf(m[h], mx * sl2);
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                const float alpha = ex2_approx(m[h] - m_use);
                m[h] = m_new;
                l[h] *= alpha;
#pragma unroll
                for (int i = 0; i < NT; ++i) {
                    oacc[i][2 * h] *= alpha;
                    oacc[i][2 * h + 1] *= alpha;
                }
                float pv[4][2];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    pv[nt][0] = ex2_approx(fmaf(sacc[nt][2 * h], sl2, -m_use));
                    pv[nt][1] = ex2_approx(fmaf(sacc[nt][2 * h + 1], sl2, -m_use));
                    l[h] += pv[nt][0] + pv[nt][1];
                }
                // A fragment of P for k-steps of 16 keys: (row half h) -> regs 0/2 or 1/3
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                    pa[k2][h] = pack_bf16x2(pv[2 * k2][0], pv[2 * k2][1]);
                    pa[k2][h + 2] = pack_bf16x2(pv[2 * k2 + 1][0], pv[2 * k2 + 1][1]);
                }
            }
            // ---- O += P V for this warp's 32 keys
            // Keys past the sequence's end (rest of a page, padding of a contiguous
            // cache) hold arbitrary bits; P is 0 there, but 0 * NaN is not, so their
            // V values are cleared in registers on the sequence's last tile.
            const bool tail = kVarlen && blk * kDecKeys + kDecKeys > Tk;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
#pragma unroll
                for (int dp = 0; dp < D / 16; ++dp) {
                    const int mi = lane >> 3, rr = lane & 7;
                    const int key = cw * 32 + k2 * 16 + (mi & 1) * 8 + rr;
                    const int d = dp * 16 + (mi >> 1) * 8;
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(sV + sw128_off(key, d), b0, b1, b2, b3);
                    if (tail) {
                        // this thread holds keys kb, kb+1 (b0, b2) and kb+8, kb+9 (b1, b3),
                        // the lower key in the low half
                        const int kb = blk * kDecKeys + cw * 32 + k2 * 16 + c2;
                        b0 = clear_past(b0, kb, Tk);
                        b2 = clear_past(b2, kb, Tk);
                        b1 = clear_past(b1, kb + 8, Tk);
                        b3 = clear_past(b3, kb + 8, Tk);
                    }
                    mma_bf16_16816(oacc[dp * 2], pa[k2], b0, b1);
                    mma_bf16_16816(oacc[dp * 2 + 1], pa[k2], b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->empty[stage]));
            if (++stage == kStages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        // full row sums: the four lanes of a row hold disjoint key columns
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
            l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
        }
        __syncthreads();  // every stage consumed and every copy landed: reuse the ring
        float* wm = mrg + cw * (2 * kDecRows + kDecRows * D);
        float* wl = wm + kDecRows;
        float* wo = wl + kDecRows;
        if ((lane & 3) == 0) {
            wm[r_lo] = m[0];
            wm[r_lo + 8] = m[1];
            wl[r_lo] = l[0];
            wl[r_lo + 8] = l[1];
        }
#pragma unroll
        for (int i = 0; i < NT; ++i) {
            const int col = i * 8 + c2;
            wo[r_lo * D + col] = oacc[i][0];
            wo[r_lo * D + col + 1] = oacc[i][1];
            wo[(r_lo + 8) * D + col] = oacc[i][2];
            wo[(r_lo + 8) * D + col + 1] = oacc[i][3];
        }
        __syncthreads();
        // ---- merge the four warps' partial softmax states; 128 threads over (row, d)
        const int t = threadIdx.x - 32;
        const float* base = mrg;
        const int stride_w = 2 * kDecRows + kDecRows * D;
        for (int idx = t; idx < nrows * D; idx += 32 * kDecConsumers) {
            const int row = idx / D;
            const int d = idx - row * D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kDecConsumers; ++w) M = fmaxf(M, base[w * stride_w + row]);
            const float Mu = M == -INFINITY ? 0.f : M;
            float lsum = 0.f, acc = 0.f;
#pragma unroll
            for (int w = 0; w < kDecConsumers; ++w) {
                const float* bw = base + w * stride_w;
                const float sc = ex2_approx(bw[row] - Mu);
                lsum += bw[kDecRows + row] * sc;
                acc += bw[2 * kDecRows + row * D + d] * sc;
            }
            const size_t frow = row0 + row;   // flat row id in [B * Hq * Tq]
            // a row can see no key of this split (window, or keys past its position):
            // its partial is 0 with log-sum-exp -inf, which the merge weighs by 0
            const float val = lsum > 0.f ? acc / lsum : 0.f;
            if (p.splits == 1) {
                p.o[frow * D + d] = __float2bfloat16_rn(val);
            } else {
                const size_t prow = (size_t)split * ((size_t)p.B * p.Hq * p.Tq) + frow;
                p.ws_o[prow * D + d] = val;
                if (d == 0) p.ws_lse[prow] = lsum > 0.f ? M + __log2f(lsum) : -INFINITY;
            }
        }
    }
}

// Merge split partials: o = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M), M = max_s lse_s,
// in fixed split order. One warp per (b, a) row.
template <int D>
__global__ void __launch_bounds__(256) gqa_decode_combine_kernel(const float* __restrict__ ws_o,
                                                                 const float* __restrict__ ws_lse,
                                                                 __nv_bfloat16* __restrict__ o,
                                                                 int rows, int splits) {
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int E = D / 32;  // elements per lane
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, ws_lse[(size_t)s * rows + row]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    float wsum = 0.f;
    for (int s = 0; s < splits; ++s) {
        const float w = ex2_approx(ws_lse[(size_t)s * rows + row] - Mu);
        wsum += w;
        const float* src = ws_o + ((size_t)s * rows + row) * D + lane * E;
        if constexpr (E == 4) {
            const float4 v = *reinterpret_cast<const float4*>(src);
            acc[0] += w * v.x;
            acc[1] += w * v.y;
            acc[2] += w * v.z;
            acc[3] += w * v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2*>(src);
            acc[0] += w * v.x;
            acc[1] += w * v.y;
        }
    }
    const float inv = 1.f / wsum;
    __nv_bfloat16* dst = o + (size_t)row * D + lane * E;
    if constexpr (E == 4) {
        uint2 pk;
        pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2*>(dst) = pk;
    } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
}

}  // namespace gqa
