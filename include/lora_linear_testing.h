/*
 * lora_linear_testing.h — test hooks of liblora_linear.so.  Not part of the layer's
 * interface; used by the failure-detection tests.
 */
#ifndef LORA_LINEAR_TESTING_H
#define LORA_LINEAR_TESTING_H

#include <stdint.h>

#include "lora_linear.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Enqueues one small kernel that waits, with the same bounded wait the forward and
 * backward kernels use, on a barrier that nothing ever completes.  After `limit_ns`
 * nanoseconds (1 <= limit_ns <= 1e10) the wait gives up, the kernel sets the timeout
 * bit of the status word at the head of `workspace` (device, zero-filled, at least
 * 256 bytes) and returns normally, leaving the CUDA context usable.  A following
 * lora_device_status(workspace, stream) then returns LORA_ERR_DEVICE_TIMEOUT.
 * No fault, trap or hang is involved.
 */
lora_status_t lora_testing_bounded_wait(void* workspace, uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_LINEAR_TESTING_H */
