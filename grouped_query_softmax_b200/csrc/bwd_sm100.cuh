// Causal grouped-query attention backward for sm_100a: dQ, dK, dV.
//
// The gradients of o_a = softmax(Q_a K_g^T * scale + M) V_g ("注意力家族", section
// 统一记号) for an output gradient dO, with P_ij the softmax weights of row i:
//   dV_j = sum_i P_ij dO_i,  dP_ij = <dO_i, v_j>,  dS_ij = P_ij (dP_ij - D_i),
//   D_i = sum_j P_ij dP_ij = <dO_i, O_i>,  dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,
// with a KV head's dK and dV summed over the G query heads that read it. As in the
// FlashAttention backward ("长上下文与高效注意力：研究账本", section FlashAttention: the backward
// recomputes, adding FLOPs) P is recomputed from Q, K and the forward's log-sum-exp; the
// T_q x T_k matrices never reach HBM.
//
// B200 mapping. A CTA owns one 128-key block j of one KV head g of one batch b and walks
// every (query head a of the group, 128-row query tile i) that sees those keys, so dK and
// dV accumulate in TMEM for the whole group without atomics. Per step, with K_j and V_j
// resident in shared memory:
//   S^T  = K_j Q_i^T      (tcgen05, TMEM; lanes = keys)
//   P^T  = 2^(S^T scale log2e - LSE_i log2e), causal (and window) mask on the edge tiles (bf16, in place)
//   dP^T = V_j dO_i^T     (TMEM)
//   dV  += P^T dO_i       (A from TMEM)
//   dS^T = P^T (dP^T - D_i)  -> shared memory, bf16, [keys][rows]
//   dK  += dS^T Q_i       (A = dS^T, K-major)
//   dQ_i = dS K_j         (A = the same buffer read M-major), added into an fp32 dQ buffer
// Warps: 0 TMA producer (K_j, V_j once; Q_i through a 2-slot ring, dO_i through one slot
// released right after dV; each step's LSE and D vectors by bulk copy), 1 tcgen05 issuer,
// 2 TMEM allocation, 4-7 the P / dS warpgroup (thread t owns key row t and keeps its 128
// probabilities in registers), 8-11 the dQ warpgroup (thread t owns query row t of the dQ
// tile; it stages 64 columns at a time in shared memory and one thread adds them to the
// fp32 buffer with a TMA bulk reduction) and, at the end, the dK and dV epilogue.
// TMEM (512 columns at D = 128): S^T | dP^T, later dQ | dV | dK.
#pragma once

#include "gqa_internal.h"
#include "sm100_ptx.cuh"

namespace gqa {

constexpr int kBwdKeys = 128;     // keys per CTA
constexpr int kBwdRows = 128;     // query rows per step
constexpr int kBwdThreads = 384;
// Register split (setmaxnreg): 384 x 168 at launch = 128 x (136 + 240 + 128).
constexpr int kBwdLaunchRegs = 168;
constexpr int kBwdCtlRegs = 136;
constexpr int kBwdPRegs = 240;
constexpr int kBwdDqRegs = 128;
static_assert(128 * (kBwdCtlRegs + kBwdPRegs + kBwdDqRegs) <= kBwdThreads * kBwdLaunchRegs,
              "register split exceeds the launch allocation");

struct BwdParams {
    int B, Hq, Hkv, Tq, Tk, G;
    int n_kb;       // key blocks per (batch, KV head)
    int chunk;      // launch order: (batch, KV head) pairs per chunk (bwd_block_coords)
    int n_qt;       // ceil(Tq / 128)
    int tq_pad;     // n_qt * 128: row stride of lse2 and dvec
    float scale;
    float scale_log2;     // scale * log2(e)
    const float* lse2;    // [B, Hq, tq_pad]: -(the forward's LSE) * log2(e); -inf past Tq
    const float* dvec;    // [B, Hq, tq_pad]: <dO_i, O_i>; 0 past Tq
    float* dq_acc;        // [B, Hq, Tq, D] fp32, zeroed by the prep kernel
    __nv_bfloat16* dk;    // [B, Hkv, Tk, D]
    __nv_bfloat16* dv;    // [B, Hkv, Tk, D]
    uint32_t* err;
    unsigned long long timeout_ns;
    int window;     // > 0: each query sees only its `window` most recent positions
};

template <int D>
struct BwdSmem {
    static constexpr int kChunks = D / 64;
    static constexpr int kChunkBytes = 128 * 128;          // 128 rows x 128 bytes
    static constexpr int kTileBytes = kChunks * kChunkBytes;  // one [128][D] bf16 tile
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kTileBytes;
    static constexpr int kQOff = 2 * kTileBytes;           // 2 slots of Q_i
    static constexpr int kDoOff = 4 * kTileBytes;          // 1 slot of dO_i
    static constexpr int kDsOff = 5 * kTileBytes;          // dS^T [128 keys][128 rows] bf16
    static constexpr int kDsBytes = 2 * kChunkBytes;
    static constexpr int kStageOff = kDsOff + kDsBytes;    // dQ staging: [128 rows][64 fp32], two boxes
    static constexpr int kStageBytes = 2 * kChunkBytes;    // of [128][32] in the 128-byte swizzle
    static constexpr int kLseOff = kStageOff + kStageBytes;  // LSE_i log2(e) of the current step
    static constexpr int kDvecOff = kLseOff + 4 * kBwdRows;  // D_i of the current step
    static constexpr int kCtlOff = kDvecOff + 4 * kBwdRows;
    struct Ctl {
        uint64_t kv_full;
        uint64_t q_full[2];
        uint64_t q_empty[2];
        uint64_t do_full, do_empty;
        uint64_t lse_full, dvec_full;
        uint64_t s_full, p_full, dp_full, ds_full, ds_empty, dq_full, dq_empty, dkdv_full;
        uint64_t stage_full, stage_free;
        uint64_t drain;
        uint32_t tmem_base;
        uint32_t abort;
    };
    static constexpr int kBytes = kCtlOff + (int)sizeof(Ctl) + 1024;
};

// First 128-row query tile with a row that sees key block j (row r sees key k iff
// k <= Tk - Tq + r).
__device__ __forceinline__ int bwd_first_tile(int j, int Tq, int Tk) {
    const int r = j * kBwdKeys - (Tk - Tq);
    return r > 0 ? r / kBwdRows : 0;
}

// One past the last query tile with a row that sees key block j: with a window w, row r
// (position Tk - Tq + r) sees keys down to position - w + 1 only.
__device__ __forceinline__ int bwd_end_tile(int j, int Tq, int Tk, int n_qt, int window) {
    if (window <= 0) return n_qt;
    const int r_last = j * kBwdKeys + kBwdKeys - 1 + window - 1 - (Tk - Tq);  // last row seeing the block
    if (r_last < 0) return 0;
    return min(n_qt, r_last / kBwdRows + 1);
}

template <int D, bool kWindow>
__global__ void __launch_bounds__(kBwdThreads, 1)
    gqa_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                         const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
    using L = BwdSmem<D>;
    using Ctl = typename L::Ctl;
    constexpr int kTileBytes = L::kTileBytes;
    constexpr int kChunkBytes = L::kChunkBytes;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw_addr + pad;
    const uint32_t sK = sbase + L::kKOff;
    const uint32_t sV = sbase + L::kVOff;
    const uint32_t sQ0 = sbase + L::kQOff;
    const uint32_t sDO = sbase + L::kDoOff;
    const uint32_t sDS = sbase + L::kDsOff;
    const uint32_t sStage = sbase + L::kStageOff;
    const uint32_t sLse = sbase + L::kLseOff;
    const uint32_t sDvec = sbase + L::kDvecOff;
    const float* nlse_s = reinterpret_cast<const float*>(smem + L::kLseOff);  // -LSE_i log2(e)
    const float* dvec_s = reinterpret_cast<const float*>(smem + L::kDvecOff);
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + L::kCtlOff);
    volatile uint32_t* abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Launch order: chunks of (b, g) pairs whose dQ rows stay in L2 while their key blocks
    // add into them; inside a chunk, low j first (most work).
    int j, bg;  // key block, b * Hkv + g
    bwd_block_coords((int)blockIdx.x, p.n_kb, p.B * p.Hkv, p.chunk, &bg, &j);
    const int b = bg / p.Hkv;
    const int g = bg - b * p.Hkv;
    const int off = p.Tk - p.Tq;
    const int i0 = bwd_first_tile(j, p.Tq, p.Tk);
    const int i1 = kWindow ? bwd_end_tile(j, p.Tq, p.Tk, p.n_qt, p.window) : p.n_qt;
    // (query tile, head) steps, tile-major; 0 when no query sees the block (inside a window)
    const int items = i1 > i0 ? p.G * (i1 - i0) : 0;

    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&ctl->kv_full), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&ctl->q_full[s]), 1);
            mbar_init(smem_u32(&ctl->q_empty[s]), 1);
        }
        mbar_init(smem_u32(&ctl->do_full), 1);
        mbar_init(smem_u32(&ctl->do_empty), 1);
        mbar_init(smem_u32(&ctl->stage_full), 128);
        mbar_init(smem_u32(&ctl->stage_free), 1);
        mbar_init(smem_u32(&ctl->lse_full), 1);
        mbar_init(smem_u32(&ctl->dvec_full), 1);
        mbar_init(smem_u32(&ctl->s_full), 1);
        mbar_init(smem_u32(&ctl->p_full), 128);
        mbar_init(smem_u32(&ctl->dp_full), 1);
        mbar_init(smem_u32(&ctl->ds_full), 128);
        mbar_init(smem_u32(&ctl->ds_empty), 1);
        mbar_init(smem_u32(&ctl->dq_full), 1);
        mbar_init(smem_u32(&ctl->dq_empty), 128);
        mbar_init(smem_u32(&ctl->dkdv_full), 1);
        mbar_init(smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
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
        prefetch_tensormap(&tm_do);
        prefetch_tensormap(&tm_dq);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t tS = tmem;                    // S^T, P^T (bf16 in the first 64 columns)
    const uint32_t tDP = tmem + 128u;            // dP^T, then dQ
    const uint32_t tDV = tmem + 256u;            // dV (D columns)
    const uint32_t tDK = tmem + 256u + (uint32_t)D;  // dK (D columns)

    if (warp < 4) setmaxnreg_dec<kBwdCtlRegs>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            const uint32_t kvbar = smem_u32(&ctl->kv_full);
            mbar_arrive_expect_tx(kvbar, 2 * kTileBytes);
            for (int c = 0; c < L::kChunks; ++c) {
                tma_load_4d(sK + c * kChunkBytes, &tm_k, kvbar, c * 64, j * kBwdKeys, g, b);
                tma_load_4d(sV + c * kChunkBytes, &tm_v, kvbar, c * 64, j * kBwdKeys, g, b);
            }
            uint32_t q_issued[2] = {0u, 0u};
            uint32_t lse_issued = 0, do_issued = 0, dvec_issued = 0;
            const uint32_t lbar = smem_u32(&ctl->lse_full), dbar = smem_u32(&ctl->dvec_full);
            const uint32_t obar = smem_u32(&ctl->do_full);
            for (int w = 0; w < items && ok; ++w) {
                const int slot = w & 1;
                const int i = i0 + w / p.G;
                const int a = g * p.G + (w - (w / p.G) * p.G);
                // Q_i: two slots (the next step's S^T is issued while this step still needs Q_i)
                if (w >= 2 && !(ok = mbar_wait_bounded(smem_u32(&ctl->q_empty[slot]), ((w >> 1) - 1) & 1u,
                                                       abort_flag, p.err, p.timeout_ns)))
                    break;
                const uint32_t qbar = smem_u32(&ctl->q_full[slot]);
                mbar_arrive_expect_tx(qbar, kTileBytes);
                for (int c = 0; c < L::kChunks; ++c)
                    tma_load_4d(sQ0 + slot * kTileBytes + c * kChunkBytes, &tm_q, qbar, c * 64, i * kBwdRows, a, b);
                ++q_issued[slot];
                // LSE once the previous step's P is done with it, dO once the previous dV has
                // read it, D once the previous step's dS is done (one slot each)
                const size_t vrow = ((size_t)b * p.Hq + a) * p.tq_pad + (size_t)i * kBwdRows;
                if (w > 0 && !(ok = mbar_wait_bounded(smem_u32(&ctl->p_full), (w - 1) & 1u, abort_flag, p.err,
                                                      p.timeout_ns)))
                    break;
                mbar_arrive_expect_tx(lbar, 4 * kBwdRows);
                bulk_load(sLse, p.lse2 + vrow, 4 * kBwdRows, lbar);
                ++lse_issued;
                if (w > 0 && !(ok = mbar_wait_bounded(smem_u32(&ctl->do_empty), (w - 1) & 1u, abort_flag, p.err,
                                                      p.timeout_ns)))
                    break;
                mbar_arrive_expect_tx(obar, kTileBytes);
                for (int c = 0; c < L::kChunks; ++c)
                    tma_load_4d(sDO + c * kChunkBytes, &tm_do, obar, c * 64, i * kBwdRows, a, b);
                ++do_issued;
                if (w > 0 && !(ok = mbar_wait_bounded(smem_u32(&ctl->ds_full), (w - 1) & 1u, abort_flag, p.err,
                                                      p.timeout_ns)))
                    break;
                mbar_arrive_expect_tx(dbar, 4 * kBwdRows);
                bulk_load(sDvec, p.dvec + vrow, 4 * kBwdRows, dbar);
                ++dvec_issued;
            }
            if (*abort_flag) {
                mbar_wait_drain(kvbar, 0, p.timeout_ns);
                for (int s = 0; s < 2; ++s)
                    if (q_issued[s]) mbar_wait_drain(smem_u32(&ctl->q_full[s]), (q_issued[s] - 1u) & 1u, p.timeout_ns);
                if (lse_issued) mbar_wait_drain(lbar, (lse_issued - 1u) & 1u, p.timeout_ns);
                if (do_issued) mbar_wait_drain(obar, (do_issued - 1u) & 1u, p.timeout_ns);
                if (dvec_issued) mbar_wait_drain(dbar, (dvec_issued - 1u) & 1u, p.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ tcgen05 issuer
        if (lane == 0) {
            constexpr uint32_t idesc_t = umma_idesc_bf16(kBwdKeys, kBwdRows, 0, 0);  // S^T, dP^T
            constexpr uint32_t idesc_kv = umma_idesc_bf16(kBwdKeys, D, 0, 1);       // dV, dK
            constexpr uint32_t idesc_q = umma_idesc_bf16(kBwdRows, D, 1, 1);        // dQ
            const uint64_t dK_kmaj = umma_desc_sw128(sK, 16, 1024);
            const uint64_t dV_kmaj = umma_desc_sw128(sV, 16, 1024);
            const uint64_t dK_nmaj = umma_desc_sw128(sK, kChunkBytes, 1024);
            const uint64_t dS_kmaj = umma_desc_sw128(sDS, 16, 1024);
            const uint64_t dS_mmaj = umma_desc_sw128(sDS, kChunkBytes, 1024);
            // S^T = K_j Q_i^T of step w: M = 128 keys, N = 128 rows, K = D in steps of 16
            auto issue_s = [&](int w) -> bool {
                if (!mbar_wait_bounded(smem_u32(&ctl->q_full[w & 1]), (w >> 1) & 1u, abort_flag, p.err,
                                       p.timeout_ns))
                    return false;
                tc_fence_after_sync();
                const uint64_t dQ_kmaj = umma_desc_sw128(sQ0 + (w & 1) * kTileBytes, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ko = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
                    tc_mma_ss(tS, dK_kmaj + ko, dQ_kmaj + ko, idesc_t, kk > 0 ? 1u : 0u);
                }
                tc_commit(smem_u32(&ctl->s_full));
                return true;
            };
            bool ok = mbar_wait_bounded(smem_u32(&ctl->kv_full), 0, abort_flag, p.err, p.timeout_ns);
            tc_fence_after_sync();
            if (ok && items > 0) ok = issue_s(0);
            const uint64_t dDO_kmaj = umma_desc_sw128(sDO, 16, 1024);
            const uint64_t dDO_nmaj = umma_desc_sw128(sDO, kChunkBytes, 1024);
            for (int w = 0; w < items && ok; ++w) {
                const int slot = w & 1;
                const uint32_t ph = w & 1;
                const uint64_t dQ_nmaj = umma_desc_sw128(sQ0 + slot * kTileBytes, kChunkBytes, 1024);
                // dP^T = V_j dO_i^T into the dQ columns, once dO_i has landed and the previous
                // dQ has been read
                if (!(ok = mbar_wait_bounded(smem_u32(&ctl->do_full), ph, abort_flag, p.err, p.timeout_ns))) break;
                if (w > 0 && !(ok = mbar_wait_bounded(smem_u32(&ctl->dq_empty), (w - 1) & 1u, abort_flag, p.err,
                                                      p.timeout_ns)))
                    break;
                tc_fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ko = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
                    tc_mma_ss(tDP, dV_kmaj + ko, dDO_kmaj + ko, idesc_t, kk > 0 ? 1u : 0u);
                }
                tc_commit(smem_u32(&ctl->dp_full));
                // dV += P^T dO_i: A = P^T (bf16 pairs in TMEM), K = 128 query rows
                if (!(ok = mbar_wait_bounded(smem_u32(&ctl->p_full), ph, abort_flag, p.err, p.timeout_ns))) break;
                tc_fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kBwdRows / 16; ++kk)
                    tc_mma_ts(tDV, tS + kk * 8, dDO_nmaj + (uint64_t)((kk * 2048) >> 4), idesc_kv,
                              (w > 0 || kk > 0) ? 1u : 0u);
                tc_commit(smem_u32(&ctl->do_empty));  // dV is dO_i's last reader
                // the next step's S^T now: it runs while this step's dS is formed (the tensor
                // pipe executes in order, so dV has read P^T before S^T overwrites it)
                if (w + 1 < items && !(ok = issue_s(w + 1))) break;
                // dQ_i = dS K_j and dK += dS^T Q_i, once dS^T is in shared memory
                if (!(ok = mbar_wait_bounded(smem_u32(&ctl->ds_full), ph, abort_flag, p.err, p.timeout_ns))) break;
                tc_fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kBwdKeys / 16; ++kk)
                    tc_mma_ss(tDP, dS_mmaj + (uint64_t)((kk * 2048) >> 4), dK_nmaj + (uint64_t)((kk * 2048) >> 4),
                              idesc_q, kk > 0 ? 1u : 0u);
                tc_commit(smem_u32(&ctl->dq_full));  // dQ first: its read-out overlaps dK
#pragma unroll
                for (int kk = 0; kk < kBwdRows / 16; ++kk) {
                    const uint64_t ko = (uint64_t)(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
                    tc_mma_ss(tDK, dS_kmaj + ko, dQ_nmaj + (uint64_t)((kk * 2048) >> 4), idesc_kv,
                              (w > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(smem_u32(&ctl->ds_empty));
                tc_commit(smem_u32(&ctl->q_empty[slot]));
            }
            if (ok) tc_commit(smem_u32(&ctl->dkdv_full));
            if (*abort_flag) {
                tc_commit(smem_u32(&ctl->drain));
                mbar_wait_drain(smem_u32(&ctl->drain), 0, p.timeout_ns);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ P and dS
        setmaxnreg_inc<kBwdPRegs>();
        const int t = (warp - 4) * 32 + lane;              // key row = TMEM lane
        const uint32_t lane_sel = (uint32_t)((warp & 3) * 32) << 16;
        const int kabs = j * kBwdKeys + t;                 // this thread's key position
        bool ok = true;
        for (int w = 0; w < items && ok; ++w) {
            const uint32_t ph = w & 1;
            const int i = i0 + w / p.G;
            const int a = g * p.G + (w - (w / p.G) * p.G);
            (void)a;
            // column c (query row i*128 + c) sees this key iff lim <= c < lim + window
            const int lim = kabs - (off + i * kBwdRows);
            const int lim_hi = kWindow ? lim + p.window : 0;
            const bool diag = j * kBwdKeys + kBwdKeys - 1 > off + i * kBwdRows ||
                              (kWindow && off + i * kBwdRows + kBwdRows - p.window > j * kBwdKeys);
            if (!(ok = mbar_wait_bounded(smem_u32(&ctl->lse_full), ph, abort_flag, p.err, p.timeout_ns))) break;
            if (!(ok = mbar_wait_bounded(smem_u32(&ctl->s_full), ph, abort_flag, p.err, p.timeout_ns))) break;
            tc_fence_after_sync();
            // P^T row in fp32 pairs (kept for dS); the next 32-column chunk of S^T is loaded
            // while this one is exponentiated
            uint64_t pr[64];
            uint32_t sb[2][32];
            const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
            tmem_ld32(tS + lane_sel, sb[0]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                tc_wait_ld();
                reg_fence32(sb[c & 1]);
                if (c + 1 < 4) tmem_ld32(tS + lane_sel + (c + 1) * 32, sb[(c + 1) & 1]);
                const uint32_t* sr = sb[c & 1];
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 l4 = *reinterpret_cast<const float4*>(nlse_s + c * 32 + e);
#pragma unroll
                    for (int u = 0; u < 4; u += 2) {
                        const int col = c * 32 + e + u;
                        const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[e + u]), __uint_as_float(sr[e + u + 1])),
                                                  sl2, u ? f2_pack(l4.z, l4.w) : f2_pack(l4.x, l4.y));
                        float x0, x1;
                        f2_unpack(x, x0, x1);
                        x0 = ex2_approx(x0);
                        x1 = ex2_approx(x1);
                        if (diag && (col < lim || (kWindow && col >= lim_hi))) x0 = 0.f;
                        if (diag && (col + 1 < lim || (kWindow && col + 1 >= lim_hi))) x1 = 0.f;
                        pr[col / 2] = f2_pack(x0, x1);
                        pk[(e + u) / 2] = pack_bf16x2(x0, x1);
                    }
                }
                tmem_st16(tS + lane_sel + c * 16, pk);
            }
            tc_wait_st();
            tc_fence_before_sync();
            mbar_arrive(smem_u32(&ctl->p_full));
            // dS^T = P^T (dP^T - D_i), rounded to bf16, into the [keys][rows] tile
            if (!(ok = mbar_wait_bounded(smem_u32(&ctl->dp_full), ph, abort_flag, p.err, p.timeout_ns))) break;
            if (!(ok = mbar_wait_bounded(smem_u32(&ctl->dvec_full), ph, abort_flag, p.err, p.timeout_ns))) break;
            if (w > 0 && !(ok = mbar_wait_bounded(smem_u32(&ctl->ds_empty), (w - 1) & 1u, abort_flag, p.err,
                                                  p.timeout_ns)))
                break;
            tc_fence_after_sync();
            tmem_ld32(tDP + lane_sel, sb[0]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                tc_wait_ld();
                reg_fence32(sb[c & 1]);
                if (c + 1 < 4) tmem_ld32(tDP + lane_sel + (c + 1) * 32, sb[(c + 1) & 1]);
                const uint32_t* dr = sb[c & 1];
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 d4 = *reinterpret_cast<const float4*>(dvec_s + c * 32 + e);
                    const uint64_t ds0 = f2_mul(pr[(c * 32 + e) / 2],
                                                f2_sub(f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])),
                                                       f2_pack(d4.x, d4.y)));
                    const uint64_t ds1 = f2_mul(pr[(c * 32 + e) / 2 + 1],
                                                f2_sub(f2_pack(__uint_as_float(dr[e + 2]), __uint_as_float(dr[e + 3])),
                                                       f2_pack(d4.z, d4.w)));
                    float a0, a1, a2, a3;
                    f2_unpack(ds0, a0, a1);
                    f2_unpack(ds1, a2, a3);
                    pk[e / 2] = pack_bf16x2(a0, a1);
                    pk[e / 2 + 1] = pack_bf16x2(a2, a3);
                }
                // row t, query columns c*32 .. c*32+31: four 16-byte units of chunk c/2
                const uint32_t rowb = sDS + (uint32_t)((c >> 1) * kChunkBytes + t * 128);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int unit = ((c & 1) * 4 + u) ^ (t & 7);
                    st_shared_v4(rowb + unit * 16, pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            mbar_arrive(smem_u32(&ctl->ds_full));
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ dQ, then dK and dV
        setmaxnreg_dec<kBwdDqRegs>();
        const int t = (warp - 8) * 32 + lane;
        const uint32_t lane_sel = (uint32_t)((warp & 3) * 32) << 16;
        bool ok = true;
        uint32_t rounds = 0;   // staging rounds so far (64 dQ columns each)
        bool pending = false;  // thread 0: a bulk reduction whose shared-memory read is not yet released
        // thread 0 waits until its last reduction has read the staging tile and frees the tile;
        // it does so only right before the tile is needed again, so the TMEM columns of dQ
        // are handed back to the MMA without waiting for the reduction
        auto release = [&]() {
            if (t == 0 && pending) {
                bulk_wait_read_all();
                mbar_arrive(smem_u32(&ctl->stage_free));
                pending = false;
            }
        };
        for (int w = 0; w < items && ok; ++w) {
            const int i = i0 + w / p.G;
            const int a = g * p.G + (w - (w / p.G) * p.G);
            if (!(ok = mbar_wait_bounded(smem_u32(&ctl->dq_full), w & 1u, abort_flag, p.err, p.timeout_ns))) break;
            tc_fence_after_sync();
#pragma unroll 1
            for (int h = 0; h < D / 64 && ok; ++h) {
                uint32_t r0[32], r1[32];
                tmem_ld32(tDP + lane_sel + h * 64, r0);
                tmem_ld32(tDP + lane_sel + h * 64 + 32, r1);
                tc_wait_ld();
                reg_fence32(r0);
                reg_fence32(r1);
                if (h == D / 64 - 1) {
                    // every dQ column has been read: the next dP^T may overwrite them
                    tc_fence_before_sync();
                    mbar_arrive(smem_u32(&ctl->dq_empty));
                }
                // the previous round's bulk reduction has finished reading the staging tile
                release();
                if (rounds > 0 && !(ok = mbar_wait_bounded(smem_u32(&ctl->stage_free), (rounds - 1) & 1u, abort_flag,
                                                           p.err, p.timeout_ns)))
                    break;
                // row t of two [128][32] fp32 boxes, 16-byte units in the 128-byte swizzle
#pragma unroll
                for (int bx = 0; bx < 2; ++bx) {
                    const uint32_t* rr = bx ? r1 : r0;
                    const uint32_t rowb = sStage + bx * kChunkBytes + t * 128;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        st_shared_v4(rowb + ((u ^ (t & 7)) * 16),
                                     __float_as_uint(__uint_as_float(rr[4 * u]) * p.scale),
                                     __float_as_uint(__uint_as_float(rr[4 * u + 1]) * p.scale),
                                     __float_as_uint(__uint_as_float(rr[4 * u + 2]) * p.scale),
                                     __float_as_uint(__uint_as_float(rr[4 * u + 3]) * p.scale));
                }
                fence_proxy_async_smem();
                mbar_arrive(smem_u32(&ctl->stage_full));
                if (t == 0) {
                    // one thread adds the staged tile into the fp32 dQ buffer (rows past Tq
                    // fall outside the tensor map and are dropped)
                    if (!(ok = mbar_wait_bounded(smem_u32(&ctl->stage_full), rounds & 1u, abort_flag, p.err,
                                                 p.timeout_ns)))
                        break;
                    const int plane = b * p.Hq + a;
                    tma_reduce_add_3d(&tm_dq, sStage, h * 64, i * kBwdRows, plane);
                    tma_reduce_add_3d(&tm_dq, sStage + kChunkBytes, h * 64 + 32, i * kBwdRows, plane);
                    bulk_commit_group();
                    pending = true;
                }
                ++rounds;
            }
        }
        if (t == 0) bulk_wait_all();  // every reduction into dQ has completed
        if (kWindow && ok && items == 0) {
            // no query sees this key block (it lies before every row's window): zero gradients
            const int key = j * kBwdKeys + t;
            if (key < p.Tk) {
                const size_t orow = ((size_t)b * p.Hkv + g) * p.Tk + key;
                uint4* k4 = reinterpret_cast<uint4*>(p.dk + orow * D);
                uint4* v4 = reinterpret_cast<uint4*>(p.dv + orow * D);
#pragma unroll
                for (int e = 0; e < D / 8; ++e) k4[e] = v4[e] = make_uint4(0u, 0u, 0u, 0u);
            }
        } else if (ok && mbar_wait_bounded(smem_u32(&ctl->dkdv_full), 0, abort_flag, p.err, p.timeout_ns)) {
            tc_fence_after_sync();
            const int key = j * kBwdKeys + t;
            const size_t orow = ((size_t)b * p.Hkv + g) * p.Tk + key;
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const uint32_t tacc = which ? tDV : tDK;
                const float mul = which ? 1.f : p.scale;
                __nv_bfloat16* out = (which ? p.dv : p.dk) + orow * D;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(tacc + lane_sel + c * 32, r);
                    tc_wait_ld();
                    reg_fence32(r);
                    uint4 v4[4];
                    uint32_t* pw = reinterpret_cast<uint32_t*>(v4);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pw[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
                    if (key < p.Tk) {
                        uint4* d4 = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e) d4[e] = v4[e];
                    }
                }
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

// D_i = <dO_i, O_i> and -LSE_i * log2(e) per query row (padded to whole 128-row tiles with
// 0 and -inf), and the fp32 dQ buffer zeroed. D / 8 lanes per row, 16-byte accesses.
template <int D>
__global__ void __launch_bounds__(256) gqa_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                           const __nv_bfloat16* __restrict__ dout,
                                                           const float* __restrict__ lse, float* __restrict__ lse2,
                                                           float* __restrict__ dvec, float* __restrict__ dq_acc,
                                                           int BH, int Tq, int tq_pad) {
    constexpr int kLanes = D / 8;            // lanes per row (16 or 8), 8 elements each
    constexpr int kRows = 256 / kLanes;      // rows per block
    const int sub = threadIdx.x % kLanes;
    const long long gw = (long long)blockIdx.x * kRows + threadIdx.x / kLanes;
    if (gw >= (long long)BH * tq_pad) return;  // whole row groups leave together
    const long long bh = gw / tq_pad;
    const int r = (int)(gw - bh * tq_pad);
    if (r >= Tq) {
        if (sub == 0) {
            lse2[gw] = -INFINITY;  // P = 2^(s - inf) = 0 for rows past Tq
            dvec[gw] = 0.f;
        }
        return;
    }
    const size_t base = ((size_t)bh * Tq + r) * D + sub * 8;
    const uint4 ov = *reinterpret_cast<const uint4*>(o + base);
    const uint4 dv = *reinterpret_cast<const uint4*>(dout + base);
    const uint32_t* ow = reinterpret_cast<const uint32_t*>(&ov);
    const uint32_t* dw = reinterpret_cast<const uint32_t*>(&dv);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(dw[e] << 16), acc);
        acc = fmaf(__uint_as_float(ow[e] & 0xFFFF0000u), __uint_as_float(dw[e] & 0xFFFF0000u), acc);
    }
    // only this row's lanes take part (other rows of the warp may have left)
    const unsigned group = (kLanes == 32 ? 0xffffffffu : ((1u << kLanes) - 1u)) << ((threadIdx.x & 31) & ~(kLanes - 1));
#pragma unroll
    for (int s = kLanes / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(group, acc, s);
    float4* z = reinterpret_cast<float4*>(dq_acc + base);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (sub == 0) {
        dvec[gw] = acc;
        lse2[gw] = -lse[bh * Tq + r] * 1.4426950408889634f;
    }
}

// dQ (bf16) from the fp32 buffer, 8 elements per thread.
__global__ void __launch_bounds__(256) gqa_bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                         __nv_bfloat16* __restrict__ dq, long long n8) {
    const long long idx = (long long)blockIdx.x * 256 + threadIdx.x;
    if (idx >= n8) return;
    const float4 a = reinterpret_cast<const float4*>(dq_acc)[2 * idx];
    const float4 c = reinterpret_cast<const float4*>(dq_acc)[2 * idx + 1];
    uint4 o;
    o.x = pack_bf16x2(a.x, a.y);
    o.y = pack_bf16x2(a.z, a.w);
    o.z = pack_bf16x2(c.x, c.y);
    o.w = pack_bf16x2(c.z, c.w);
    reinterpret_cast<uint4*>(dq)[idx] = o;
}

}  // namespace gqa
