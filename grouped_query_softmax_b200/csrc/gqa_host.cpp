// gqa_attn_fwd_host: the prefill/suffix call for operands in host memory, streamed through a
// device workspace so that copies in, attention and copies out overlap.
//
// The query rows are cut into chunks of whole 128-row tiles. Chunk c (rows [r0, r1)) is the
// suffix call of the same operation over the keys [0, T_k - T_q + r1): its queries sit at the
// same absolute positions and see the same keys as in the one-shot call, so the result is the
// one-shot result (the kernel's per-row arithmetic does not depend on which other rows share
// the launch). The keys a chunk needs beyond the previous chunk's are copied just before it,
// so the cache arrives incrementally and each key crosses PCIe once.
//
// Three streams: copies in on one, the kernel on the caller's stream, copies out on a third.
// Query and output tiles alternate between two workspace slots; the copy into a slot waits
// until the kernel two chunks back has read it, and that kernel's successor in the slot
// waits until its output has been copied out.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "../../include/gqa.h"
#include "../../include/gqa_testing.h"

namespace {

constexpr int kHostChunks = 8;         // at most this many query-row chunks
constexpr int kHostMinChunkRows = 256;  // and at least this many rows per chunk

struct HostPlan {
    int chunk_rows;  // rows per chunk (a multiple of 128, the last chunk may be shorter)
    int chunks;
    size_t k_bytes, q_slot_bytes, lse_slot_bytes;
    size_t off_v, off_q[2], off_o[2], off_lse[2], total;
};

size_t round_up256(size_t x) { return (x + 255) & ~(size_t)255; }

HostPlan plan_host(int B, int Hq, int Hkv, int Tq, int Tk, int D) {
    HostPlan p{};
    int rows = (Tq + kHostChunks - 1) / kHostChunks;
    rows = (rows + 127) / 128 * 128;
    if (rows < kHostMinChunkRows) rows = kHostMinChunkRows;
    if (rows > Tq) rows = Tq;
    p.chunk_rows = rows;
    p.chunks = (Tq + rows - 1) / rows;
    p.k_bytes = round_up256((size_t)B * Hkv * Tk * D * 2);
    p.q_slot_bytes = round_up256((size_t)B * Hq * rows * D * 2);
    p.lse_slot_bytes = round_up256((size_t)B * Hq * rows * sizeof(float));
    size_t at = p.k_bytes;  // K first, then V
    p.off_v = at;
    at += p.k_bytes;
    for (int s = 0; s < 2; ++s) {
        p.off_q[s] = at;
        at += p.q_slot_bytes;
        p.off_o[s] = at;
        at += p.q_slot_bytes;
        p.off_lse[s] = at;
        at += p.lse_slot_bytes;
    }
    p.total = at;
    return p;
}

// Query rows of chunk c (the last chunk may be shorter).
int chunk_rows_of(const HostPlan& pl, int c, int Tq) {
    const int r0 = c * pl.chunk_rows;
    return (Tq - r0 < pl.chunk_rows) ? Tq - r0 : pl.chunk_rows;
}

gqa_status check_host_args(const void* q, const void* k, const void* v, const void* o, const float* lse, int B,
                           int Hq, int Hkv, int Tq, int Tk, int D, float scale, int window) {
    if (!q || !k || !v || !o) return GQA_ERR_INVALID_ARGUMENT;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || Tk <= 0 || D <= 0) return GQA_ERR_INVALID_ARGUMENT;
    if (Hq % Hkv != 0 || Tq > Tk || window < 0) return GQA_ERR_INVALID_ARGUMENT;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GQA_ERR_INVALID_ARGUMENT;
    if (!(scale == scale) || std::isinf(scale)) return GQA_ERR_INVALID_ARGUMENT;
    if (D != 64 && D != 128) return GQA_ERR_UNSUPPORTED;
    if ((long long)B * Hq > (1LL << 30)) return GQA_ERR_UNSUPPORTED;
    return GQA_OK;
}

// A run of `bytes` bytes from each of `planes` (b, h) planes: one 2-D copy whose "rows" are
// the planes, each side advancing by its own pitch from one plane to the next.
cudaError_t copy_rows(void* dst, size_t dst_pitch, const void* src, size_t src_pitch, size_t bytes, size_t planes,
                      cudaMemcpyKind kind, cudaStream_t s) {
    return cudaMemcpy2DAsync(dst, dst_pitch, src, src_pitch, bytes, planes, kind, s);
}

// Chunk before whose kernel gqa_attn_fwd_host stops with an error (-1: never); set only
// through gqa_testing_fwd_host_fail_at, to test the error path.
std::atomic<int> g_fail_at_chunk{-1};

}  // namespace

extern "C" {

size_t gqa_attn_fwd_host_workspace_bytes(int B, int Hq, int Hkv, int Tq, int Tk, int D) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || Tk <= 0 || (D != 64 && D != 128) || Hq % Hkv != 0 || Tq > Tk)
        return 0;
    return plan_host(B, Hq, Hkv, Tq, Tk, D).total;
}

gqa_status gqa_testing_fwd_host_fail_at(int chunk) {
    if (chunk < -1 || chunk >= kHostChunks) return GQA_ERR_INVALID_ARGUMENT;
    g_fail_at_chunk.store(chunk, std::memory_order_relaxed);
    return GQA_OK;
}

gqa_status gqa_testing_fwd_host_plan(int B, int Hq, int Hkv, int Tq, int Tk, int D, int* out_chunks, int* out_row0,
                                     int* out_rows, int* out_keys) {
    if (!out_chunks || !out_row0 || !out_rows || !out_keys) return GQA_ERR_INVALID_ARGUMENT;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || Tk <= 0 || Hq % Hkv != 0 || Tq > Tk)
        return GQA_ERR_INVALID_ARGUMENT;
    if (D != 64 && D != 128) return GQA_ERR_INVALID_ARGUMENT;
    const HostPlan pl = plan_host(B, Hq, Hkv, Tq, Tk, D);
    *out_chunks = pl.chunks;
    for (int c = 0; c < pl.chunks; ++c) {
        out_row0[c] = c * pl.chunk_rows;
        out_rows[c] = chunk_rows_of(pl, c, Tq);
        out_keys[c] = Tk - Tq + out_row0[c] + out_rows[c];
    }
    return GQA_OK;
}

gqa_status gqa_attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                             int Hkv, int Tq, int Tk, int D, float softmax_scale, int window, void* workspace,
                             size_t workspace_bytes, void* stream) {
    gqa_status st = check_host_args(q, k, v, o, lse, B, Hq, Hkv, Tq, Tk, D, softmax_scale, window);
    if (st != GQA_OK) return st;
    const HostPlan pl = plan_host(B, Hq, Hkv, Tq, Tk, D);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GQA_ERR_WORKSPACE;
    if (workspace_bytes < pl.total) return GQA_ERR_WORKSPACE;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* k_dev = ws;
    uint8_t* v_dev = ws + pl.off_v;
    const cudaStream_t s_main = static_cast<cudaStream_t>(stream);
    const int off = Tk - Tq;
    const size_t row_b = (size_t)D * 2;  // bytes of one bf16 row
    const size_t q_planes = (size_t)B * Hq, kv_planes = (size_t)B * Hkv;

    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev_start = nullptr;
    cudaEvent_t ev_in[kHostChunks] = {}, ev_comp[kHostChunks] = {}, ev_out[kHostChunks] = {};
    cudaError_t e = cudaSuccess;
    gqa_status result = GQA_OK;
    auto ok = [&](cudaError_t x) {
        if (x != cudaSuccess && e == cudaSuccess) e = x;
        return e == cudaSuccess;
    };
    if (!ok(cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking)) ||
        !ok(cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking)) ||
        !ok(cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming)))
        goto done;
    for (int c = 0; c < pl.chunks; ++c)
        if (!ok(cudaEventCreateWithFlags(&ev_in[c], cudaEventDisableTiming)) ||
            !ok(cudaEventCreateWithFlags(&ev_comp[c], cudaEventDisableTiming)) ||
            !ok(cudaEventCreateWithFlags(&ev_out[c], cudaEventDisableTiming)))
            goto done;
    // everything the caller enqueued before this call (for example earlier use of the
    // workspace) comes first
    if (!ok(cudaEventRecord(ev_start, s_main)) || !ok(cudaStreamWaitEvent(s_in, ev_start, 0)) ||
        !ok(cudaStreamWaitEvent(s_out, ev_start, 0)))
        goto done;
    {
        int keys_in = 0;  // key rows already on the device
        for (int c = 0; c < pl.chunks; ++c) {
            const int slot = c & 1;
            const int r0 = c * pl.chunk_rows;
            const int rows = chunk_rows_of(pl, c, Tq);
            const int keys = off + r0 + rows;  // keys this chunk's last row sees
            uint8_t* q_slot = ws + pl.off_q[slot];
            uint8_t* o_slot = ws + pl.off_o[slot];
            float* lse_slot = reinterpret_cast<float*>(ws + pl.off_lse[slot]);
            // copies in: this chunk's query rows once the kernel two chunks back has read the
            // slot, and the keys it needs beyond those already copied
            if (c >= 2 && !ok(cudaStreamWaitEvent(s_in, ev_comp[c - 2], 0))) goto done;
            if (!ok(copy_rows(q_slot, rows * row_b, static_cast<const uint8_t*>(q) + (size_t)r0 * row_b,
                              (size_t)Tq * row_b, rows * row_b, q_planes, cudaMemcpyHostToDevice, s_in)))
                goto done;
            if (keys > keys_in) {
                const size_t kb = (size_t)(keys - keys_in) * row_b, at = (size_t)keys_in * row_b;
                if (!ok(copy_rows(k_dev + at, (size_t)Tk * row_b, static_cast<const uint8_t*>(k) + at,
                                  (size_t)Tk * row_b, kb, kv_planes, cudaMemcpyHostToDevice, s_in)) ||
                    !ok(copy_rows(v_dev + at, (size_t)Tk * row_b, static_cast<const uint8_t*>(v) + at,
                                  (size_t)Tk * row_b, kb, kv_planes, cudaMemcpyHostToDevice, s_in)))
                    goto done;
                keys_in = keys;
            }
            if (!ok(cudaEventRecord(ev_in[c], s_in))) goto done;
            // attention on the chunk: a suffix call over the first `keys` keys; the output
            // slot must have been copied out (chunk c - 2)
            if (!ok(cudaStreamWaitEvent(s_main, ev_in[c], 0))) goto done;
            if (c >= 2 && !ok(cudaStreamWaitEvent(s_main, ev_out[c - 2], 0))) goto done;
            if (c == g_fail_at_chunk.load(std::memory_order_relaxed)) {  // testing hook only
                result = GQA_ERR_UNSUPPORTED;
                goto done;
            }
            st = gqa_attn_fwd_ex(q_slot, k_dev, v_dev, o_slot, lse ? lse_slot : nullptr, B, Hq, Hkv, rows, keys, D,
                                 (long long)Hkv * Tk * D, (long long)Tk * D, (long long)Hkv * Tk * D,
                                 (long long)Tk * D, softmax_scale, window, s_main);
            if (st != GQA_OK) {
                result = st;
                goto done;
            }
            if (!ok(cudaEventRecord(ev_comp[c], s_main))) goto done;
            // copies out
            if (!ok(cudaStreamWaitEvent(s_out, ev_comp[c], 0))) goto done;
            if (!ok(copy_rows(static_cast<uint8_t*>(o) + (size_t)r0 * row_b, (size_t)Tq * row_b, o_slot,
                              rows * row_b, rows * row_b, q_planes, cudaMemcpyDeviceToHost, s_out)))
                goto done;
            if (lse && !ok(copy_rows(lse + r0, (size_t)Tq * sizeof(float), lse_slot, rows * sizeof(float),
                                     rows * sizeof(float), q_planes, cudaMemcpyDeviceToHost, s_out)))
                goto done;
            if (!ok(cudaEventRecord(ev_out[c], s_out))) goto done;
        }
        // the caller's stream continues once every output row is in host memory
        if (!ok(cudaStreamWaitEvent(s_main, ev_out[pl.chunks - 1], 0))) goto done;
    }
done:
    if ((result != GQA_OK || e != cudaSuccess) && s_in && s_out) {
        // an error after some chunks were queued: copies already on the internal streams may
        // still read the caller's inputs or write its outputs; the call returns only after
        // they have finished, so the caller may free or reuse its host buffers at once
        cudaStreamSynchronize(s_in);
        cudaStreamSynchronize(s_out);
    }
    // streams and events are released once their work completes
    for (int c = 0; c < kHostChunks; ++c) {
        if (ev_in[c]) cudaEventDestroy(ev_in[c]);
        if (ev_comp[c]) cudaEventDestroy(ev_comp[c]);
        if (ev_out[c]) cudaEventDestroy(ev_out[c]);
    }
    if (ev_start) cudaEventDestroy(ev_start);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
    if (result != GQA_OK) return result;
    return e == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

}  // extern "C"
