/*
 * gdr2_testing.h -- test support for the Gated Delta Rule-2 library.
 *
 * Not part of the operator. It lets a test exercise the failure-detection
 * path of the tensor-core kernels on a real GPU without faulting, trapping or
 * hanging it.
 */
#ifndef GDR2_TESTING_H_
#define GDR2_TESTING_H_

#include <stdint.h>

#include "gdr2.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * gdr2_selftest_bounded_wait -- launches one CTA that waits on a shared-memory
 * barrier nothing ever arrives on, through the same bounded wait the chunk
 * kernel uses, but with a limit of `timeout_us` microseconds (1..2000000)
 * instead of about one second. When the limit passes, the CTA records the
 * timeout in the device error word and returns normally, so the context stays
 * usable; gdr2_check_device_error then reports GDR2_ERR_DEVICE_TIMEOUT once.
 * Asynchronous on `stream`. Returns GDR2_ERR_INVALID_ARG for a limit outside
 * the range, GDR2_ERR_CUDA if the launch fails.
 */
gdr2_status gdr2_selftest_bounded_wait(uint32_t timeout_us, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDR2_TESTING_H_ */
