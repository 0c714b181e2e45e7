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

/*
 * Schedule of the Y or dX GEMM of lora_linear_fwd / lora_linear_bwd for an output of
 * M × Nout over a reduction of length Kred, LoRA rank r (0..128; the rank of the GEMM's
 * LoRA fill) and a weight of format `fmt` (a lora_wfmt_t): the number of output tiles the
 * stream-K schedule shares out among the CTA pairs as pieces, 0 when every tile is
 * computed whole, -1 for an invalid format or rank.  A pure function of its arguments
 * (lora_workspace_bytes includes the schedule's fp32 slots); lets tests check that a case
 * takes the stream-K path.
 */
int32_t lora_testing_gemm_streamk(int64_t M, int64_t Nout, int64_t Kred, int32_t r, int32_t fmt);

/*
 * Which passes over X run on the TMA-fed stream (the kernel of the one-pass dY·B / dYᵀ·XA
 * products in a single-product mode) rather than the cp.async passes, for M tokens, K
 * input features and LoRA rank r (the grouped layers' G·r): bit 0 the forward's X·Aᵀ,
 * bit 1 the backward's Xᵀ·(s·dY·B) for dA; -1 for invalid sizes.  A pure function of
 * its arguments; lets tests check that a case takes those paths.
 */
int32_t lora_testing_xpass_tma(int64_t M, int64_t K, int32_t r);

/*
 * Blocking of the one-pass kernel over a [M, C] activation at rank r: mode 0 both
 * products (dY·B and dYᵀ·XA), 1 the row product only (X·Aᵀ), 2 the column product only.
 * Writes {a, b, row_tiles, col_tiles} to out4 (host memory, 4 int32): an a × b grid of
 * blocks of row_tiles × 64 rows by col_tiles × 256 columns.  Returns 1 when the kernel is
 * used for these sizes, 0 when the cp.async passes are (out4 then holds zeros), -1 for
 * invalid arguments.  A pure function of its arguments.
 */
int32_t lora_testing_dual_blocking(int64_t M, int64_t C, int32_t r, int32_t mode, int32_t* out4);

/*
 * Launches the tensor-core rank-r row projection (X·Aᵀ at rank r, 16 < r <= 128, r % 8 == 0)
 * over P [rows, red] (device bf16, row-major) and A [r, red] (device bf16) with one output
 * tile more than `rows` holds: that tile starts at row 128·ceil(rows/128), past the last
 * row.  Its TMA loads lie wholly outside P, so the hardware fills them with zeros, and its
 * epilogue writes no row at or past `rows`; nothing out of range is read or written.  The
 * regular build computes the real tiles into part (device fp32, at least part_bytes =
 * splits·rows·r·4 bytes for the pass's split count, which this call checks) and returns
 * LORA_OK from lora_device_status; the checked build (-DLORA_CHECKED=1) also rejects the
 * extra tile before its first copy, so lora_device_status(workspace, stream) then returns
 * LORA_ERR_DEVICE_BOUNDS.  workspace: device, zero-filled, at least 256 bytes.  Lets the
 * tests see the checked build's bounds test fire.
 */
/* Split count of the tensor-core rank-r pass for an output of `rows` rows over a
 * reduction of length `red` at rank r (a pure function of the three); -1 for invalid
 * sizes. */
int32_t lora_testing_tcproj_splits(int64_t rows, int64_t red, int32_t r);

lora_status_t lora_testing_tcproj_extra_tile(const void* P, const void* A, int64_t rows, int64_t red, int32_t r,
                                             float* part, size_t part_bytes, void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LORA_LINEAR_TESTING_H */
