/*
 * lora_linear_profiling.h — measurement hooks of liblora_linear.so, used by the
 * benchmark.  They time and count the library's own kernels; they change nothing
 * that the kernels compute.
 */
#ifndef LORA_LINEAR_PROFILING_H
#define LORA_LINEAR_PROFILING_H

#include <stdint.h>

#include "lora_linear.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LORA_KERNEL_FWD_GEMM = 0,   /* Y = X·Wᵀ + (s·XA)·Bᵀ (tcgen05 GEMM, bf16 or 4-bit weight) */
  LORA_KERNEL_BWD_GEMM = 1,   /* dX = dY·W + (s·dY·B)·A (tcgen05 GEMM, bf16 or 4-bit weight) */
  LORA_KERNEL_COUNT = 2
} lora_kernel_id_t;

/*
 * on != 0: every later forward/backward call records a pair of CUDA events on its
 * stream around each launch of the GEMM kernels above (host-side event objects are
 * created per launch and released by lora_timing_read).  on == 0: stop recording.
 */
lora_status_t lora_timing_enable(int32_t on);

/*
 * Waits for the recorded events of `kernel`, returns the summed device time in
 * milliseconds and the number of launches recorded, and forgets them.
 */
lora_status_t lora_timing_read(int32_t kernel, double* total_ms, int64_t* launches);

/* Number of kernels this library has launched in this process so far (all kinds). */
int64_t lora_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LORA_LINEAR_PROFILING_H */
