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

#ifdef __cplusplus
}
#endif

#endif /* GQA_TESTING_H_ */
