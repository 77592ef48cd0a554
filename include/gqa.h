/*
 * gqa.h -- C ABI of libgqa: causal grouped-query softmax attention on B200 (sm_100a).
 *
 * The operation (one definition covers MHA, GQA and MQA):
 *
 *   o_a = softmax( Q_a K_{g(a)}^T * scale + M ) V_{g(a)},   g(a) = floor(a / (H_q / H_kv))
 *
 *   -- "注意力家族" (wineandchord.com, attention variants), section 统一记号 (the o_a
 *      equation) and section 最小语义实现 (interface q:[B,H_q,T_q,D], k,v:[B,H_kv,T_k,D];
 *      consecutive H_q/H_kv query heads map to one KV head; H_q % H_kv == 0 and
 *      T_q <= T_k are required; scale 1/sqrt(D); the result has q's dtype).
 *   -- "Attention Architecture Evolution", section GQA (group(i) = floor(i/(Hq/Hkv))).
 *
 * M is the causal mask with the suffix offset: query row i (0 <= i < T_q) sits at
 * absolute position (T_k - T_q) + i and sees keys j <= (T_k - T_q) + i, its own
 * position included ("注意力家族", sections 最小语义实现 and Mask 与增量位置; "A Visual
 * Guide to Attention", section "Which positions are visible?"). There is no
 * non-causal mode.
 *
 * Types and precision: Q, K, V and O are bf16; products accumulate in fp32; the
 * softmax runs in fp32 and its probabilities are rounded to bf16 before the product
 * with V (the pages' reference rounds the fp32 probabilities to the input dtype
 * before "@ v"); O is rounded to bf16 round-to-nearest-even.
 *
 * Memory: every pointer is a DEVICE pointer owned by the caller, except the operands of
 * gqa_attn_fwd_host, which live in host memory. The library never allocates device
 * memory and keeps no per-call state; K and V are addressed per KV
 * head and are never replicated per query head. All calls are asynchronous on
 * `stream` (a cudaStream_t; NULL = the legacy default stream) and return as soon as
 * the kernels are enqueued. Calls are thread-safe and re-entrant.
 *
 * Errors: argument checks run on the host before anything is enqueued; a call that
 * returns an error has launched nothing. Launch failures return GQA_ERR_CUDA.
 * Device-side waits are bounded; a wait that runs out sets a device error word
 * that gqa_get_device_error() reports as GQA_ERR_TIMEOUT. Sequence bounds that
 * live on the device (the *_varlen calls) are checked there and reported the same
 * way, as GQA_ERR_INVALID_ARGUMENT.
 */
#ifndef GQA_H_
#define GQA_H_

#include <stddef.h>

/* Symbols of the C ABI are the only ones the shared library exports. */
#if defined(__GNUC__)
#define GQA_API __attribute__((visibility("default")))
#else
#define GQA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gqa_status {
    GQA_OK = 0,
    GQA_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, bad size or stride, Hq % Hkv, Tq > Tk */
    GQA_ERR_UNSUPPORTED = 2,      /* D not in {64, 128}, sizes beyond grid or TMA limits */
    GQA_ERR_WORKSPACE = 3,        /* decode workspace missing or smaller than required */
    GQA_ERR_CUDA = 4,             /* a CUDA runtime/driver call or a kernel launch failed */
    GQA_ERR_TIMEOUT = 5           /* a bounded device-side wait ran out (reported later) */
} gqa_status;

/*
 * Prefill and suffix chunks (1 <= T_q <= T_k).
 *
 *   q    bf16 [B, Hq, Tq, D], contiguous; 16-byte aligned.
 *   k    bf16; element (b, h, t, d) at k + b*k_sb + h*k_sh + t*D + d (elements).
 *        Rows are packed (row stride D); batch/head strides are free, so a cache
 *        pre-allocated to a capacity T_cap >= T_k is read as its [:T_k] slice.
 *        16-byte aligned; k_sb and k_sh multiples of 8 elements.
 *   v    bf16; same addressing with v_sb, v_sh.
 *   o    bf16 [B, Hq, Tq, D], contiguous; written. Must not overlap the inputs.
 *   lse  fp32 [B, Hq, Tq] or NULL; if given, receives the natural-log
 *        log-sum-exp of each row's scaled, masked scores.
 *   softmax_scale  <= 0 selects 1/sqrt(D).
 *   D    64 or 128.
 */
GQA_API gqa_status gqa_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int Hq, int Hkv, int Tq, int Tk, int D,
                        long long k_sb, long long k_sh, long long v_sb, long long v_sh,
                        float softmax_scale, void* stream);

/*
 * gqa_attn_fwd with a sliding window: window > 0 restricts the query at position p to
 * its `window` most recent positions, keys j with p - window < j <= p (itself
 * included) -- "A Visual Guide to Attention", section "Which positions are visible?"
 * (sliding-window attention; GQA combined with it as in Mistral 7B, section "Read the
 * data path"). KV tiles wholly outside every row's window are never loaded.
 * window = 0 is plain causal attention; window < 0 is GQA_ERR_INVALID_ARGUMENT.
 */
GQA_API gqa_status gqa_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                                   int B, int Hq, int Hkv, int Tq, int Tk, int D,
                                   long long k_sb, long long k_sh, long long v_sb, long long v_sh,
                                   float softmax_scale, int window, void* stream);

/*
 * gqa_attn_fwd_ex with a caller workspace that lets the library split the keys of some work
 * units over several CTAs. The operation is the same o_a definition ("注意力家族", section
 * 统一记号, with the causal suffix mask of its section 最小语义实现); only the order in which
 * the keys of a row are summed changes, so results agree with gqa_attn_fwd_ex within rounding
 * (not bit for bit).
 *
 * Which launches split: plain causal suffix calls (window = 0) whose cached prefix is at
 * least as long as the suffix (T_k - T_q >= T_q). Their work units (pairs of 128-row query
 * tiles) all need about the same number of key tiles, so when their count is not a multiple
 * of the number of SMs the last wave of the persistent kernel leaves SMs idle. The full waves
 * then run whole, and the key tiles of the last wave's units, laid end to end, are dealt out
 * in equal runs of consecutive tiles, one run per SM; a run is cut at unit boundaries into
 * pieces, each piece writes its rows' fp32 partial output and log-sum-exp to the workspace,
 * and a second kernel merges them by log-sum-exp (the same merge as decode's split-KV
 * partials). The tile splitting that "A Visual Guide to Attention", section "Sources and
 * execution", describes for one row is here spread over CTAs.
 *
 *   workspace, workspace_bytes  device memory of at least
 *            gqa_attn_fwd_split_workspace_bytes(B, Hq, Hkv, Tq, Tk, D, window) bytes (same
 *            arguments, same current device), 256-byte aligned, caller-owned. Its contents on
 *            entry are ignored; it must not be shared by calls that can overlap on the GPU.
 *            When that size is 0 the launch does not split and workspace may be NULL.
 *            A missing, misaligned or smaller workspace is GQA_ERR_WORKSPACE.
 * Other arguments and errors as gqa_attn_fwd_ex.
 */
GQA_API size_t gqa_attn_fwd_split_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int D, int window);
GQA_API gqa_status gqa_attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse,
                                      int B, int Hq, int Hkv, int Tq, int Tk, int D,
                                      long long k_sb, long long k_sh, long long v_sb, long long v_sh,
                                      float softmax_scale, int window, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * gqa_attn_fwd_ex for operands in HOST memory, for callers whose tensors are not yet on the
 * device. The pages define the operation only; moving operands is a library convenience.
 *
 * The query rows are cut into chunks of whole 128-row tiles, at most 8. Chunk c (rows
 * [r0, r1)) is computed as the suffix call over keys [0, T_k - T_q + r1), the keys its rows
 * see, so each query sits at the same position and gets the same result as in the one-shot
 * call, bit for bit. Each key crosses to the device once, just before the first chunk that
 * needs it. Copies in, the kernel and copies out run on three streams, so chunk c + 1's
 * inputs and chunk c - 1's output move while chunk c is computed.
 *
 *   q, o     bf16 [B, Hq, Tq, D], contiguous host memory. Pinned memory (cudaHostAlloc or
 *            cudaHostRegister) lets the copies overlap the kernels. With pageable memory the
 *            results are the same, but the copies serialise.
 *   k, v     bf16 [B, Hkv, Tk, D], contiguous host memory.
 *   lse      NULL, or fp32 [B, Hq, Tq] host memory (as gqa_attn_fwd).
 *   window   as gqa_attn_fwd_ex.
 *   workspace  device memory of at least gqa_attn_fwd_host_workspace_bytes(...) bytes,
 *            256-byte aligned. It holds K, V and two query/output slots. Its contents on
 *            entry are ignored. It must not be used by other work that can overlap the call.
 *   stream   the call is ordered on this stream. It starts after the work already enqueued
 *            there. Work enqueued after it starts once every row of o (and lse) is in host
 *            memory. The call returns without waiting, and the host buffers must stay
 *            valid and unchanged until the stream gets there.
 *
 * Errors:
 *   - Checked before anything is enqueued. GQA_ERR_INVALID_ARGUMENT for a null q, k, v or o,
 *     a non-positive size, Hq % Hkv != 0, T_q > T_k, window < 0, an lse that is not 4-byte
 *     aligned, or a non-finite scale. GQA_ERR_UNSUPPORTED for D outside {64, 128}. Host
 *     pointers need no alignment.
 *   - A missing, misaligned or short workspace returns GQA_ERR_WORKSPACE.
 *   - GQA_ERR_CUDA means that a stream, event, copy or launch call failed. Part of the
 *     work may then already be enqueued: synchronise the device before reusing o or the
 *     workspace.
 */
GQA_API size_t gqa_attn_fwd_host_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int D);
GQA_API gqa_status gqa_attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                                     int B, int Hq, int Hkv, int Tq, int Tk, int D, float softmax_scale,
                                     int window, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode (T_q = 1): the query of each (b, a) sits at position T_k - 1 and sees all
 * T_k cached keys ("注意力家族", section 最小语义实现: the suffix case with one
 * query). The KV cache is split into num_splits key ranges; each range yields a
 * partial result (fp32 output and log-sum-exp) and a second kernel merges them in
 * fixed split order, so the result is deterministic.
 *
 *   q        bf16 [B, Hq, 1, D], contiguous; 16-byte aligned.
 *   k_cache, v_cache  addressed as k/v of gqa_attn_fwd, first T_k rows read.
 *   o        bf16 [B, Hq, 1, D], contiguous; written.
 *   num_splits  0 = choose automatically; otherwise the requested split count
 *            (clamped to [1, ceil(T_k / 128)]).
 *   workspace   device buffer of at least gqa_attn_decode_workspace_bytes(...)
 *            bytes (same arguments), 256-byte aligned; may be NULL when that size
 *            is 0 (a single split writes o directly). Its contents on entry are
 *            ignored; it must not be shared by calls that can overlap on the GPU.
 */
GQA_API size_t gqa_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Tk, int D, int num_splits);

GQA_API gqa_status gqa_attn_decode(const void* q, const void* k_cache, const void* v_cache, void* o,
                           int B, int Hq, int Hkv, int Tk, int D,
                           long long k_sb, long long k_sh, long long v_sb, long long v_sh,
                           float softmax_scale, int num_splits,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode for callers that cannot allocate device memory at call time (for example a
 * plugin running inside an engine that owns all device memory, or a decode loop that
 * forbids cudaMalloc because it may synchronise the device). The pages have no
 * counterpart: this is a library convenience around gqa_attn_decode.
 *
 * Same arguments and results as gqa_attn_decode without the workspace. The split-KV
 * partials live in a 16 MiB scratch array compiled into the library: one per device
 * that loads the library, held until the process exits. A call whose partials need
 * more (gqa_attn_decode_workspace_bytes(...) > 16 MiB) returns GQA_ERR_WORKSPACE and
 * launches nothing; num_splits = 1 needs no scratch. Allocates nothing.
 * The scratch's device address belongs to a CUDA context. The first call in each
 * context (normally once per device, in the runtime's primary context) does a one-time
 * set-up: it looks that address up and caches it under the context's ID. Make that
 * first call before any stream capture. A context created later, for example after
 * cudaDeviceReset, or a caller's own context, has another ID and gets its own set-up,
 * so a cached address is never used outside the context it came from. All calls in a
 * context share the scratch and it keeps the last call's contents (nothing needs
 * clearing: every partial is written before it is read); calls whose kernels can
 * overlap on the GPU race on it.
 */
GQA_API gqa_status gqa_attn_decode_static(const void* q, const void* k_cache, const void* v_cache,
                                          void* o, int B, int Hq, int Hkv, int Tk, int D,
                                          long long k_sb, long long k_sh, long long v_sb,
                                          long long v_sh, float softmax_scale, int num_splits,
                                          void* stream);

/*
 * Decode of a short chunk of new queries, optionally in a sliding window: T_q in
 * [1, 16] query rows per head at positions T_k - T_q .. T_k - 1 (speculative or
 * verification chunks; "注意力家族", section 最小语义实现 -- the suffix case with
 * query positions starting at T_k - T_q), each seeing keys up to its own position and,
 * if window > 0, only its `window` most recent positions. The G * T_q rows of a KV
 * head are packed into the same tensor-core tiles, so the cache is still read once
 * per KV head.
 *
 *   q, o   bf16 [B, Hq, Tq, D], contiguous. Other arguments as gqa_attn_decode.
 *   T_q > 16 returns GQA_ERR_UNSUPPORTED (use gqa_attn_fwd_ex); window < 0 returns
 *   GQA_ERR_INVALID_ARGUMENT. The workspace is sized by
 *   gqa_attn_decode_ex_workspace_bytes with the same arguments.
 * gqa_attn_decode(...) is gqa_attn_decode_ex(..., Tq = 1, ..., window = 0, ...).
 */
GQA_API size_t gqa_attn_decode_ex_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int D,
                                                  int window, int num_splits);
GQA_API int gqa_attn_decode_ex_num_splits(int B, int Hq, int Hkv, int Tq, int Tk, int D, int window,
                                          int num_splits);
GQA_API gqa_status gqa_attn_decode_ex(const void* q, const void* k_cache, const void* v_cache,
                                      void* o, int B, int Hq, int Hkv, int Tq, int Tk, int D,
                                      long long k_sb, long long k_sh, long long v_sb, long long v_sh,
                                      float softmax_scale, int window, int num_splits,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* The split count gqa_attn_decode will use for these arguments (num_splits 0 = auto). */
GQA_API int gqa_attn_decode_num_splits(int B, int Hq, int Hkv, int Tk, int D, int num_splits);

/*
 * Element strides of one bf16 operand: element (b, h, t, d) is at
 * base + b*sb + h*sh + t*st + d (elements; d is contiguous). Every stride used must
 * be a positive multiple of 8 elements (16 bytes, a TMA requirement) and st >= D.
 * A stride along an axis of extent 1 is not used.
 *   head-major  [H, rows, D]:     sh = rows*D, st = D
 *   token-major [rows, H, D]:     sh = D,      st = H*D   (serving engines' packed layout)
 *   padded      [B, H, rows, D]:  sb = H*rows*D, sh = rows*D, st = D
 *   paged pool  [pages, page, H, D]: sb = page*H*D, sh = D, st = H*D (b = pool page)
 */
typedef struct gqa_layout {
    long long sb, sh, st;
} gqa_layout;

/*
 * Sequences of different lengths: S independent causal problems in one call. The
 * pages ask an attention implementation for padding masks and packed segments, for
 * query lengths that differ from the cache length, and for masks built from each
 * sequence's own positions, not from the tensors' shapes ("注意力家族", section
 * Mask 与增量位置); "Attention Architecture Evolution", section GDN, names the packed
 * boundaries cu_seqlens. Sequence s has L_q(s) query rows at positions
 * L_k(s) - L_q(s) .. L_k(s) - 1 of its own L_k(s) keys; no row sees another sequence's
 * keys or any padding.
 *
 * Each side, queries (q, o, lse) and keys (k, v), is either
 *   packed  cu_seqlens_x non-NULL: int32 [S + 1] on the device, non-decreasing;
 *           sequence s owns rows cu[s] .. cu[s+1]-1 of a tensor with rows_x rows and
 *           no batch axis; or
 *   padded  cu_seqlens_x NULL: sequence s is batch s of an [S, H, rows_x, D] tensor
 *           and owns its rows 0 .. seqlens_x[s]-1 (seqlens_x int32 [S] on the device;
 *           NULL = all rows_x rows).
 * Giving both cu_seqlens_x and seqlens_x for one side is GQA_ERR_INVALID_ARGUMENT.
 *
 *   q, k, v, o    bf16 device pointers, 16-byte aligned, addressed through the
 *                 layouts (see gqa_layout); o is written on the rows of sequences
 *                 only and must not overlap the inputs.
 *   lse           fp32 or NULL: the natural-log log-sum-exp of row t of head h of
 *                 batch b at lse[(b*Hq + h)*rows_q + t] (b = 0 for packed queries).
 *   max_seqlen_q  >= every L_q(s); sizes the work decomposition and the workspace.
 *   window        0 = causal; > 0 = sliding window, as for gqa_attn_fwd_ex.
 *   workspace     device, >= gqa_attn_fwd_varlen_workspace_bytes(S, Hq, Hkv,
 *                 max_seqlen_q) bytes, 256-byte aligned; contents on entry ignored;
 *                 not shared by calls that can overlap on the GPU.
 * Sequence bounds live on the device and are checked there (no host sync): if any
 * sequence reaches past its tensor's rows or has L_q > L_k or L_q > max_seqlen_q,
 * the call computes and writes nothing, and the next gqa_get_device_error()
 * returns GQA_ERR_INVALID_ARGUMENT. Empty sequences (L_q = 0) are allowed.
 * Work: a small planning kernel lists the (sequence, rows, heads) units that have
 * work, longest first; the attention kernel then runs over that list.
 */
GQA_API size_t gqa_attn_fwd_varlen_workspace_bytes(int S, int Hq, int Hkv, int max_seqlen_q);
GQA_API gqa_status gqa_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                                       float* lse, const int* cu_seqlens_q, const int* cu_seqlens_k,
                                       const int* seqlens_q, const int* seqlens_k, int S, int Hq,
                                       int Hkv, int D, int rows_q, int rows_k, int max_seqlen_q,
                                       const gqa_layout* q_layout, const gqa_layout* k_layout,
                                       const gqa_layout* v_layout, const gqa_layout* o_layout,
                                       float softmax_scale, int window, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * gqa_attn_fwd_varlen over a paged key/value cache (chunked prefill reading the same pages
 * the decode steps use). Queries are packed (cu_seqlens_q) or padded (seqlens_q), as for
 * gqa_attn_fwd_varlen. Sequence s holds seqlens_k[s] keys (int32 [S] on the device,
 * required); key t of sequence s is row t % page_size of pool page
 * block_table[s * max_pages + t / page_size] (int32 [S, max_pages] on the device).
 *   k_pool, v_pool  bf16 pools of num_pages pages, element (page, h, r, d) at
 *                   page*sb + h*sh + r*st + d (k_layout / v_layout).
 *   page_size       16, 32, 64 or a multiple of 128.
 * Every seqlens_k[s] must lie within max_pages * page_size (checked on the device, reported
 * like the other bounds). Table entries past a sequence's last page are never read; a page
 * number outside [0, num_pages) reads zeros; key rows past a sequence's length (the rest of
 * its last page) may hold any bits. Other arguments as for gqa_attn_fwd_varlen; the
 * workspace is sized by gqa_attn_fwd_varlen_workspace_bytes.
 */
GQA_API gqa_status gqa_attn_fwd_varlen_paged(const void* q, const void* k_pool, const void* v_pool, void* o,
                                             float* lse, const int* cu_seqlens_q, const int* seqlens_q,
                                             const int* seqlens_k, const int* block_table, int page_size,
                                             int num_pages, int max_pages, int S, int Hq, int Hkv, int D,
                                             int rows_q, int max_seqlen_q, const gqa_layout* q_layout,
                                             const gqa_layout* k_layout, const gqa_layout* v_layout,
                                             const gqa_layout* o_layout, float softmax_scale, int window,
                                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode over a cache whose sequences have different lengths, contiguous or paged.
 * Sequence b holds L(b) = seqlens_k[b] keys; its T_q new queries are the last T_q of
 * them (positions L(b) - T_q .. L(b) - 1), as for gqa_attn_decode_ex. Each sequence's
 * key blocks are shared out over the splits, so short sequences are not charged for
 * the longest one's blocks.
 *
 *   q, o        bf16 [B, Hq, Tq, D], contiguous; 1 <= Tq <= 16.
 *   seqlens_k   int32 [B] on the device.
 *   block_table NULL: contiguous cache; k/v element (b, h, t, d) at the layout's
 *               b*sb + h*sh + t*st + d, rows 0 .. max_seqlen_k-1 of each sequence.
 *               Non-NULL: paged cache; int32 [B, max_pages] on the device. Position t
 *               of sequence b is row t % page_size of pool page
 *               block_table[b*max_pages + t/page_size]; pool element (page, h, r, d)
 *               at page*sb + h*sh + r*st + d, num_pages pages. page_size must be 16,
 *               32, 64 or a multiple of 128. Table entries past a sequence's last page
 *               are never read; a page number outside [0, num_pages) reads zeros.
 *   max_seqlen_k  >= every L(b); sizes the split plan (and, for a contiguous cache,
 *               the rows the cache must hold).
 *   window, num_splits, workspace   as for gqa_attn_decode_ex, but sized by
 *               gqa_attn_decode_varlen_workspace_bytes with the same arguments: the
 *               automatic split count (num_splits = 0) aims at twice as many CTAs as
 *               gqa_attn_decode_ex does, because sequences of different lengths make
 *               CTAs of different lengths and more, shorter ones even out the last wave.
 * Every L(b) must lie in [Tq, capacity], capacity = max_seqlen_k for a contiguous
 * cache and min(max_seqlen_k, max_pages*page_size) for a paged one. It is checked on
 * the device: a sequence outside that range gets no output and the next
 * gqa_get_device_error() returns GQA_ERR_INVALID_ARGUMENT. Keys past L(b) (the rest
 * of a page, a contiguous cache's unused rows) may hold any bits, NaN included.
 */
GQA_API size_t gqa_attn_decode_varlen_workspace_bytes(int B, int Hq, int Hkv, int Tq, int max_seqlen_k,
                                                      int D, int window, int num_splits);
GQA_API int gqa_attn_decode_varlen_num_splits(int B, int Hq, int Hkv, int Tq, int max_seqlen_k, int D,
                                              int window, int num_splits);
GQA_API gqa_status gqa_attn_decode_varlen(const void* q, const void* k_cache, const void* v_cache,
                                          void* o, const int* seqlens_k, const int* block_table,
                                          int page_size, int num_pages, int max_pages, int B, int Hq,
                                          int Hkv, int Tq, int max_seqlen_k, int D,
                                          const gqa_layout* k_layout, const gqa_layout* v_layout,
                                          float softmax_scale, int window, int num_splits,
                                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward pass: dQ, dK and dV of gqa_attn_fwd for an output gradient dO (training).
 * With P the softmax weights of each row over its visible keys and D_i = <dO_i, O_i>:
 *   dV_j = sum_i P_ij dO_i,   dS_ij = P_ij (<dO_i, v_j> - D_i),
 *   dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i,
 * the derivative of the o_a definition ("注意力家族", section 统一记号); a KV head's dK and
 * dV sum over the H_q/H_kv query heads that read it. As in the FlashAttention backward
 * ("长上下文与高效注意力：研究账本", section FlashAttention: the backward recomputes, which
 * adds FLOPs), P is recomputed from q, k and the forward's log-sum-exp.
 *
 *   q, o, dout  bf16 [B, Hq, Tq, D], contiguous: the forward's inputs and output, and dO.
 *   k, v        as for gqa_attn_fwd (first Tk rows, free batch/head strides).
 *   lse         fp32 [B, Hq, Tq]: the natural-log LSE gqa_attn_fwd returned for o.
 *   dq          bf16 [B, Hq, Tq, D], contiguous; written.
 *   dk, dv      bf16 [B, Hkv, Tk, D], contiguous; written (the gradient of the [:Tk] slice).
 *   workspace   device, >= gqa_attn_bwd_workspace_bytes(...) bytes, 256-byte aligned
 *               (an fp32 copy of dQ plus two fp32 values per query row); contents on
 *               entry ignored; not shared by calls that can overlap on the GPU.
 *   window      0 = causal; > 0 = the sliding window of gqa_attn_fwd_ex (the forward
 *               that produced o and lse must have used the same window).
 * dQ is accumulated with fp32 bulk additions in arrival order, so its last bits can differ
 * from run to run; dK and dV are deterministic. Keys that no query sees (before every
 * row's window) get zero gradients.
 */
GQA_API size_t gqa_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int D);
GQA_API gqa_status gqa_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                                const void* dout, const float* lse, void* dq, void* dk, void* dv,
                                int B, int Hq, int Hkv, int Tq, int Tk, int D, long long k_sb,
                                long long k_sh, long long v_sb, long long v_sh, float softmax_scale,
                                int window, void* workspace, size_t workspace_bytes, void* stream);

/* A static, human-readable name for a status code. */
GQA_API const char* gqa_status_string(gqa_status s);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device. Returns GQA_ERR_TIMEOUT if a bounded wait in any kernel of this
 * library ran out since the last call, else GQA_ERR_INVALID_ARGUMENT if a
 * variable-length call found sequence bounds outside its tensors (see
 * gqa_attn_fwd_varlen, gqa_attn_decode_varlen), GQA_ERR_CUDA if the stream reports
 * a CUDA error, else GQA_OK.
 */
GQA_API gqa_status gqa_get_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GQA_H_ */
