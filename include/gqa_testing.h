/*
 * gqa_testing.h -- test hooks of libgqa (not needed by ordinary callers).
 *
 * The pages define nothing here; these entry points exist so the library's own
 * failure handling can be tested on a GPU without faulting, trapping or hanging it.
 */
#ifndef GQA_TESTING_H_
#define GQA_TESTING_H_

#include "gqa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Enqueues a one-CTA kernel whose only wait is on an mbarrier that nothing ever
 * arrives at, bounded by timeout_ns of device wall time (%globaltimer). When the
 * bound runs out the kernel records GQA_ERR_TIMEOUT in the device error word (the
 * same word and the same bounded-wait routine every kernel of the library uses) and
 * returns normally; the CUDA context stays usable. A following
 * gqa_get_device_error() returns GQA_ERR_TIMEOUT once. timeout_ns must be in
 * [1000, 10^10]; returns GQA_ERR_INVALID_ARGUMENT otherwise.
 */
GQA_API gqa_status gqa_selftest_bounded_wait(unsigned long long timeout_ns, void* stream);

/*
 * The launch order of the backward kernel's CTAs, for host-side tests. For n_kb key blocks
 * of 128 keys per (batch, KV head) pair, n_bg pairs, G query heads per KV head, T_q query
 * rows and head dimension D, writes *out_chunk (pairs per launch chunk) and, for every
 * linear CTA index L < n_kb * n_bg, out_bg[L] and out_j[L]: the pair and the key block that
 * CTA processes. The arrays are caller-owned host memory of n_kb * n_bg ints each. Touches
 * no GPU. Returns GQA_ERR_INVALID_ARGUMENT for a non-positive size or a null pointer.
 */
GQA_API gqa_status gqa_testing_bwd_order(int n_kb, int n_bg, int G, int Tq, int D, int* out_chunk, int* out_bg,
                                         int* out_j);

/*
 * The chunk plan of gqa_attn_fwd_host, for host-side tests. For the given sizes writes
 * *out_chunks (at most 8) and, for each chunk c, out_row0[c], out_rows[c] (its query rows are
 * out_row0[c] .. out_row0[c] + out_rows[c] - 1) and out_keys[c] (the number of leading key
 * rows its suffix call reads). The three arrays are caller-owned host memory of 8 ints each.
 * Touches no GPU. Returns GQA_ERR_INVALID_ARGUMENT for sizes gqa_attn_fwd_host rejects or a
 * null pointer.
 */
GQA_API gqa_status gqa_testing_fwd_host_plan(int B, int Hq, int Hkv, int Tq, int Tk, int D, int* out_chunks,
                                             int* out_row0, int* out_rows, int* out_keys);

/*
 * Makes every later gqa_attn_fwd_host call stop with GQA_ERR_UNSUPPORTED just before the
 * kernel of chunk `chunk` (0 <= chunk < 8), after the earlier chunks' kernels and copies
 * were queued, so that tests can check the error path: such a call returns only once the
 * copies it queued have finished. -1 switches the hook off (the default). Process-wide;
 * touches no GPU. Returns GQA_ERR_INVALID_ARGUMENT for other values.
 */
GQA_API gqa_status gqa_testing_fwd_host_fail_at(int chunk);

/*
 * The split plan of gqa_attn_fwd_split for a device with `sms` SMs, for host-side tests:
 * *out_slices runs of key tiles the last units are dealt out in (0 = no split), *out_whole
 * units run whole, *out_split units cut into pieces, *out_units = all units. Touches no GPU.
 * Returns
 * GQA_ERR_INVALID_ARGUMENT for sizes gqa_attn_fwd_ex rejects, sms < 1 or a null pointer.
 */
GQA_API gqa_status gqa_testing_fwd_split_plan(int B, int Hq, int Hkv, int Tq, int Tk, int D, int window, int sms,
                                              int* out_slices, long long* out_whole, long long* out_split,
                                              long long* out_units);

#ifdef __cplusplus
}
#endif

#endif /* GQA_TESTING_H_ */
