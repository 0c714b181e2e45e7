/*
 * lora_linear.h — C ABI of liblora_linear.so: forward and hand-derived backward of a
 * LoRA-adapted linear layer over a frozen weight (bf16, 4-bit blockwise, or 8-bit int8 /
 * fp8 e4m3 with per-row scales), for NVIDIA B200 (sm_100a).
 *
 * The operation.  A linear layer with frozen weight W:[N,K] and a trainable rank-r
 * adapter A:[r,K], B:[N,r] scaled by s = alpha/r:
 *
 *     Y  = X·Wᵀ + s·(X·Aᵀ)·Bᵀ
 *     dX = dY·W + s·(dY·B)·A        dB = s·dYᵀ·(X·Aᵀ)        dA = s·(dY·B)ᵀ·X
 *
 * The fused quantized-weight LoRA product and its replaced backward are described in
 * "Rev vs unsloth" (fused quantized-LoRA paragraph) and "Unsloth vs The Stack v2"
 * (LoRA kernel and quantized fine-tuning paragraphs); the hand derivation and the
 * skinny-first bracketing, which never forms the N×K matrix B·A, in "Unsloth vs
 * PyTorch: The ONLY Video You Need to Understand the Difference" (transcript
 * 0:43-2:11).  W is frozen, so there is no dW.
 *
 * Conventions for every entry point:
 *   - Shapes follow PyTorch Linear: X:[M,K], W:[N,K], A:[r,K], B:[N,r], Y:[M,N].  All
 *     matrices are dense row-major with no padding (row pitch = columns × element size).
 *   - bf16 means IEEE bfloat16 bit patterns (uint16).  Accumulation is fp32; every
 *     bf16 output is the round-to-nearest-even of its fp32 value.
 *   - Pointers named "device" must point to memory of the current CUDA device; the
 *     library reads them on the GPU.  Pointers marked "host" are read on the CPU.
 *   - Ownership: the caller owns every buffer.  The library allocates no memory; the
 *     scratch it needs is the caller's workspace (lora_workspace_bytes()).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and return after enqueueing.  Arguments are validated on the host before
 *     anything is enqueued; on a validation error nothing is enqueued.
 *   - Device pointers must be 16-byte aligned (LORA_ERR_ALIGNMENT otherwise).
 *   - Results are deterministic: the same inputs give the same bits on every call.
 *   - lora_linear_fwd / lora_linear_bwd (and the grouped, feed-forward and cross-entropy
 *     calls) only enqueue kernels on `stream`, so a CUDA stream capture records them; the
 *     first call on a device sets kernel attributes and looks up a driver entry point
 *     and must come before any capture.  A replay reads and writes the buffers given at
 *     capture time.
 *   - Limits: 8 <= r <= 128 with r % 8 == 0; N % 8 == 0 and K % 8 == 0 (bf16 weight),
 *     K % 64 == 0 (4-bit weight) or K % 16 == 0 (8-bit weights); M >= 0 (M == 0 is an empty batch);
 *     s finite.  Sizes outside these give LORA_ERR_UNSUPPORTED (r, alignment of sizes)
 *     or LORA_ERR_INVALID_ARG (negative or zero N/K, non-finite s, NULL pointers).
 */
#ifndef LORA_LINEAR_H
#define LORA_LINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LORA_OK = 0,
  LORA_ERR_INVALID_ARG = 1,     /* NULL pointer, bad size, non-finite s, bad enum */
  LORA_ERR_ALIGNMENT = 2,       /* a device pointer is not 16-byte aligned */
  LORA_ERR_UNSUPPORTED = 3,     /* sizes outside the limits above */
  LORA_ERR_WORKSPACE = 4,       /* workspace NULL or smaller than lora_workspace_bytes() */
  LORA_ERR_CUDA = 5,            /* a CUDA runtime/driver call failed (launch error etc.) */
  LORA_ERR_DEVICE_TIMEOUT = 6,  /* a kernel gave up a bounded wait (read with lora_device_status) */
  LORA_ERR_SCRATCH_LIMIT = 7,   /* lora_linear_fwd_noalloc: problem too large for its fixed scratch */
  LORA_ERR_DEVICE_BOUNDS = 8    /* checked build only: a kernel found a tile or copy origin out of range
                                   and skipped it (read with lora_device_status) */
} lora_status_t;

typedef enum {
  LORA_W_BF16 = 0,     /* data: bf16 [N,K] */
  LORA_W_BLOCK4 = 1,   /* data: uint8 [N,K/2] codes; absmax: fp16 [N*K/64]; codebook: fp32 [16] */
  LORA_W_INT8 = 2,     /* data: int8 [N,K]; absmax: fp32 [N] row scales */
  LORA_W_FP8_E4M3 = 3  /* data: fp8 e4m3 [N,K]; absmax: fp32 [N] row scales */
} lora_wfmt_t;

/*
 * Frozen weight, logical shape [N,K], row-major.  All pointers are device pointers.
 *
 * LORA_W_BF16:   data = bf16 [N,K]; absmax and codebook are ignored (may be NULL).
 * LORA_W_BLOCK4: the 4-bit blockwise format ("Rev vs unsloth", fused quantized-LoRA
 *   paragraph: 4-bit frozen weights; "Unsloth vs The Stack v2", quantized fine-tuning
 *   paragraph).  data = uint8 [N, K/2]: byte j of row n holds element 2j in its low
 *   nibble and element 2j+1 in its high nibble (4-bit codes).  absmax = IEEE fp16
 *   [N*K/64]: scale of block b = elements [64b, 64b+64) of the row-major flattened
 *   weight (K % 64 == 0, so a block never straddles two rows).  codebook = fp32 [16]
 *   levels.  Element value = bf16_rn(fp32_rn(codebook[code] * float(absmax[block]))),
 *   computed as an fp32 multiply (never fused into an FMA) followed by a
 *   round-to-nearest-even conversion to bf16.
 * LORA_W_INT8 / LORA_W_FP8_E4M3: the 8-bit frozen weights ("Rev vs unsloth", fused
 *   quantized-LoRA paragraph: int4, int8 and fp8 weights; "Unsloth vs The Stack v2",
 *   quantized fine-tuning paragraph: 4-bit and 8-bit).  data = one byte per element,
 *   [N,K] row-major: a two's-complement int8, or an fp8 e4m3 (1 sign, 4 exponent bits
 *   with bias 7, 3 mantissa bits, no infinities; 0x7F and 0xFF are NaN).  absmax = fp32
 *   [N]: the scale of weight row n.  Element value =
 *   bf16_rn(fp32_rn(value(code) * absmax[n])), the multiply never fused into an FMA.
 *   codebook is ignored (may be NULL).
 */
typedef struct {
  int32_t fmt;            /* lora_wfmt_t */
  int32_t reserved;       /* must be 0 */
  int64_t N, K;
  const void* data;
  const void* absmax;
  const float* codebook;
} lora_weight_t;

/*
 * Bytes of device workspace the forward and backward need for these sizes (the same
 * buffer serves both).  The workspace must be zero-filled once before its first use
 * (it holds the device status word read by lora_device_status()); afterwards calls
 * leave that word alone unless a kernel reports an error.  Returns 0 for invalid sizes.
 * It holds the rank-r operand s·XA or s·dY·B, the fp32 split partials of the rank-r
 * passes and, for sizes whose output tiles would leave the GPU's CTA pairs idle in the
 * last wave, the fp32 slots of the GEMM's stream-K schedule (up to 2·74 tiles of
 * 512 × 256 fp32, 77.6 MB, for a quantized weight).
 */
size_t lora_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r, int32_t fmt);

/*
 * Forward.  Computes XA = X·Aᵀ (saved for the backward) and Y = X·Wᵀ + s·XA·Bᵀ.
 *   X  : device bf16 [M,K]          A : device bf16 [r,K]        B : device bf16 [N,r]
 *   Y  : device bf16 [M,N] (out)    XA: device bf16 [M,r] (out; pass it to the backward)
 *   workspace: device, ws_bytes >= lora_workspace_bytes(M, N, K, r, W->fmt).
 * Y and XA must not overlap any input.  M == 0 enqueues nothing.
 */
lora_status_t lora_linear_fwd(const void* X, int64_t M, const lora_weight_t* W,
                              const void* A, const void* B, int32_t r, float s,
                              void* Y, void* XA,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * Backward with W frozen.  Computes
 *   dX = dY·W + s·(dY·B)·A   (skipped when dX == NULL, e.g. for a first layer)
 *   dB = s·dYᵀ·XA            dA = s·(dY·B)ᵀ·X
 *   dY : device bf16 [M,N]   X : device bf16 [M,K]   XA : device bf16 [M,r] (from the forward)
 *   dX : device bf16 [M,K] (out, or NULL)   dA : device bf16 [r,K] (out)   dB : device bf16 [N,r] (out)
 * With M == 0, dA and dB are set to zero.  Outputs must not overlap inputs.
 */
lora_status_t lora_linear_bwd(const void* dY, const void* X, const void* XA, int64_t M,
                              const lora_weight_t* W, const void* A, const void* B,
                              int32_t r, float s,
                              void* dX, void* dA, void* dB,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * Adapter gradients in fp32, for data-parallel training.  When the tokens of a batch are
 * split over several GPUs (data parallelism over M), dA and dB are sums over tokens and
 * therefore sums over the GPUs' partial results; summing those partials in bf16 would
 * round every rank's gradient and the sum again.  With flags = LORA_GRADS_F32 the
 * backward writes dA [G·r, K] and dB [N, r] as fp32 (the same sums, scaled by s, without
 * the final rounding); the caller sums them over ranks (e.g. one NCCL all-reduce of a
 * buffer holding both) and rounds the sum once with lora_round_bf16.  On one GPU,
 * lora_round_bf16 of these fp32 gradients gives lora_linear_bwd's bf16 gradients bit for
 * bit.  flags = 0 is exactly lora_linear_bwd; other bits give LORA_ERR_INVALID_ARG.
 * Everything else (arguments, workspace, dX) is as for lora_linear_bwd.  The data-parallel
 * layout — each rank holds the frozen weight and the adapter and processes its own
 * tokens, the adapter gradients being the one exchange step — follows the distributed
 * training paragraph of "Unsloth vs The Stack v2" (a data-parallel wrapper with a custom
 * all-reduce), which names no precision for the exchange; fp32 is this library's choice.
 */
#define LORA_GRADS_F32 1u
lora_status_t lora_linear_bwd_ex(const void* dY, const void* X, const void* XA, int64_t M,
                                 const lora_weight_t* W, const void* A, const void* B,
                                 int32_t r, float s,
                                 void* dX, void* dA, void* dB, uint32_t flags,
                                 void* workspace, size_t ws_bytes, void* stream);

/*
 * dst = bf16_rn(src) for n elements: src fp32 (device), dst bf16 (device, out; must not
 * overlap src).  The one rounding of adapter gradients summed over ranks in fp32.
 * n == 0 enqueues nothing; n < 0 gives LORA_ERR_INVALID_ARG.
 */
lora_status_t lora_round_bf16(const float* src, void* dst, int64_t n, void* stream);

/*
 * Grouped projections sharing one input — e.g. the q, k and v projections of an
 * attention block, whose six adapter derivatives (dA and dB of each) "Unsloth vs
 * PyTorch: The ONLY Video You Need to Understand the Difference" counts at transcript
 * 1:14-1:24.  G projections g = 0..G-1 with weights W_g:[N_g,K], adapters A_g:[r,K],
 * B_g:[N_g,r] and a common scale s read the same X:
 *
 *     Y_g = X·W_gᵀ + s·(X·A_gᵀ)·B_gᵀ
 *     dX  = Σ_g (dY_g·W_g + s·(dY_g·B_g)·A_g)     dB_g = s·dY_gᵀ·(X·A_gᵀ)     dA_g = s·(dY_g·B_g)ᵀ·X
 *
 * computed as one layer: X is read once for all X·A_gᵀ, one GEMM produces every Y_g, and
 * one GEMM produces dX with the G adapter terms summed inside it.  The caller stacks the
 * projections along rows: W (lora_weight_t) = [W_0; W_1; ...] of N = ΣN_g rows;
 * A = [A_0; A_1; ...] bf16 [G·r, K]; B = [B_0; B_1; ...] bf16 [N, r]; Y, dY: [M, N]
 * (projection g in columns [N_0+...+N_{g-1}, +N_g)); XA: bf16 [M, G·r] (X·A_gᵀ in
 * columns [g·r, g·r+r)); dA: [G·r, K]; dB: [N, r].
 * Limits: 1 <= G <= LORA_MAX_SEGMENTS, G·r <= 128, N_g % 8 == 0, and every projection
 * but the last starts and ends on a multiple of 256 rows (LORA_ERR_UNSUPPORTED
 * otherwise); ΣN_g must equal W->N (LORA_ERR_INVALID_ARG).  The workspace is
 * lora_grouped_workspace_bytes(M, N, K, r, G, fmt).  G = 1 is exactly lora_linear_fwd /
 * lora_linear_bwd.
 */
#define LORA_MAX_SEGMENTS 8
typedef struct {
  int32_t count;                       /* G */
  int32_t reserved;                    /* must be 0 */
  int64_t rows[LORA_MAX_SEGMENTS];     /* N_g; entries past count are ignored */
} lora_segments_t;

size_t lora_grouped_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r, int32_t nseg, int32_t fmt);

lora_status_t lora_grouped_fwd(const void* X, int64_t M, const lora_weight_t* W, const lora_segments_t* segs,
                               const void* A, const void* B, int32_t r, float s,
                               void* Y, void* XA,
                               void* workspace, size_t ws_bytes, void* stream);

lora_status_t lora_grouped_bwd(const void* dY, const void* X, const void* XA, int64_t M,
                               const lora_weight_t* W, const lora_segments_t* segs,
                               const void* A, const void* B, int32_t r, float s,
                               void* dX, void* dA, void* dB,
                               void* workspace, size_t ws_bytes, void* stream);

/* As lora_grouped_bwd; flags = LORA_GRADS_F32 writes dA and dB as fp32 (see
 * lora_linear_bwd_ex). */
lora_status_t lora_grouped_bwd_ex(const void* dY, const void* X, const void* XA, int64_t M,
                                  const lora_weight_t* W, const lora_segments_t* segs,
                                  const void* A, const void* B, int32_t r, float s,
                                  void* dX, void* dA, void* dB, uint32_t flags,
                                  void* workspace, size_t ws_bytes, void* stream);

/*
 * Feed-forward block with LoRA on all three projections and SwiGLU gating ("Unsloth"
 * wiki entry, Theory: the fused SwiGLU block and the hand-derived LoRA backward; "Unsloth
 * vs PyTorch: The ONLY Video You Need to Understand the Difference", transcript
 * 2:11-2:22, the feed-forward blocks).  With model width D, hidden width I, rank r and
 * scale s:
 *
 *     G = X·W_gᵀ + s·(X·A_gᵀ)·B_gᵀ      U = X·W_uᵀ + s·(X·A_uᵀ)·B_uᵀ        [M, I]
 *     H = silu(G)·U,  silu(g) = g/(1+e^-g)                                   [M, I]
 *     Z = H·W_dᵀ + s·(H·A_dᵀ)·B_dᵀ                                           [M, D]
 *
 * Backward, by hand: dH = dZ·W_d + s·(dZ·B_d)·A_d; with σ = sigmoid(G),
 * dG = dH·U·σ·(1 + G·(1-σ)) and dU = dH·G·σ; then each of gate and up as a LoRA linear
 * of X with dX = dX_gate + dX_up.
 *
 * The forward's gate and up GEMMs run as one GEMM whose epilogue applies SwiGLU (each
 * output tile holds matching gate and up columns), writing H and the saved G, U; the
 * backward's dH GEMM applies SwiGLU's derivative in its epilogue, turning the saved
 * G, U into dG, dU in place, so dH is never written.
 *
 * Layout: gate_up is the gate weight stacked over the up weight, [2I, D] (a 4-bit
 * gate_up stacks codes and absmax the same way); down is [D, I].  A_gate_up bf16
 * [2r, D] = [A_g; A_u]; B_gate_up bf16 [2I, r] = [B_g; B_u]; A_down bf16 [r, I];
 * B_down bf16 [D, r].  GU bf16 [M, 2I] holds G in columns [0, I) and U in [I, 2I);
 * XA_gate_up bf16 [M, 2r] = [X·A_gᵀ | X·A_uᵀ]; XA_down bf16 [M, r] = H·A_dᵀ.
 * Both weights have the same format.  Limits: D % 8 == 0 and I % 8 == 0 (% 64 for
 * 4-bit), 8 <= r <= 64 with r % 8 == 0 (else LORA_ERR_UNSUPPORTED).  The workspace is
 * lora_mlp_workspace_bytes(M, D, I, r, fmt).
 */
typedef struct {
  lora_weight_t gate_up;   /* [2I, D] */
  lora_weight_t down;      /* [D, I] */
  const void* A_gate_up;   /* bf16 [2r, D] */
  const void* B_gate_up;   /* bf16 [2I, r] */
  const void* A_down;      /* bf16 [r, I] */
  const void* B_down;      /* bf16 [D, r] */
} lora_mlp_t;

size_t lora_mlp_workspace_bytes(int64_t M, int64_t D, int64_t I, int32_t r, int32_t fmt);

/* Forward.  Writes Z [M, D] and, for the backward, GU [M, 2I], H [M, I], XA_gate_up
 * [M, 2r] and XA_down [M, r] (all bf16, device). */
lora_status_t lora_mlp_fwd(const void* X, int64_t M, const lora_mlp_t* mlp, int32_t r, float s,
                           void* Z, void* GU, void* H, void* XA_gate_up, void* XA_down,
                           void* workspace, size_t ws_bytes, void* stream);

/* Backward.  GU holds the forward's G and U on entry and dG, dU (same columns) on
 * return.  Writes dX [M, D] (skipped when NULL), dA_gate_up [2r, D], dB_gate_up [2I, r],
 * dA_down [r, I], dB_down [D, r] (bf16, device).  M = 0 zeroes the adapter gradients. */
lora_status_t lora_mlp_bwd(const void* dZ, const void* X, void* GU, const void* H, const void* XA_gate_up,
                           const void* XA_down, int64_t M, const lora_mlp_t* mlp, int32_t r, float s,
                           void* dX, void* dA_gate_up, void* dB_gate_up, void* dA_down, void* dB_down,
                           void* workspace, size_t ws_bytes, void* stream);

/* As lora_mlp_bwd; flags = LORA_GRADS_F32 writes the four adapter gradients as fp32 (see
 * lora_linear_bwd_ex). */
lora_status_t lora_mlp_bwd_ex(const void* dZ, const void* X, void* GU, const void* H, const void* XA_gate_up,
                              const void* XA_down, int64_t M, const lora_mlp_t* mlp, int32_t r, float s,
                              void* dX, void* dA_gate_up, void* dB_gate_up, void* dA_down, void* dB_down,
                              uint32_t flags, void* workspace, size_t ws_bytes, void* stream);

/*
 * Cross-entropy over a frozen LM head without the [M, V] logits ("Unsloth" wiki entry,
 * Theory: chunked cross-entropy never materialises the logits; "Unsloth vs PyTorch: The
 * ONLY Video You Need to Understand the Difference", transcript 3:06-3:51: the loss
 * computed slice by slice, each slice thrown away, the slice size picked from the memory
 * left).  With hidden states X [M, D] (bf16), head W [V, D] (LORA_W_BF16 only,
 * LORA_ERR_UNSUPPORTED otherwise) and labels y [M] (device int32):
 *
 *     z = X·Wᵀ          lse_m = log Σ_v exp(z_mv)          loss_m = lse_m - z_{m,y_m}
 *     dX = (softmax(z) - onehot(y))·diag(dloss)·W  (row m scaled by dloss_m)
 *
 * Rows with y_m == ignore_index have loss 0 and no gradient; a label outside [0, V) that
 * is not ignore_index gives a NaN loss (its gradient is unspecified).
 *
 * lora_ce_fwd writes loss [M] and lse [M] (fp32, device; lse is the backward's input);
 * it needs lora_ce_workspace_bytes(M, D, V, 0) bytes or more of workspace.
 * lora_ce_bwd recomputes the logits slice by slice: the slice is the largest multiple
 * of 256 vocabulary rows whose bf16 dlogits [M, slice] fit in the workspace beside an
 * fp32 [M, D] running sum of dX, so a larger workspace means fewer, wider slices
 * (lora_ce_workspace_bytes(M, D, V, slice) gives the size for a chosen slice; fewer
 * than 256 columns' room is LORA_ERR_WORKSPACE).  dX: bf16 [M, D] (device, out);
 * dloss: fp32 [M] (device), e.g. 1/(number of rows not ignored) for a mean loss.
 * W is frozen: there is no dW.  Limits as for the layer: D % 8 == 0, V % 8 == 0.
 */
size_t lora_ce_workspace_bytes(int64_t M, int64_t D, int64_t V, int64_t slice);

lora_status_t lora_ce_fwd(const void* X, int64_t M, const lora_weight_t* W, const int32_t* labels,
                          int32_t ignore_index, float* loss, float* lse,
                          void* workspace, size_t ws_bytes, void* stream);

lora_status_t lora_ce_bwd(const void* X, int64_t M, const lora_weight_t* W, const int32_t* labels,
                          int32_t ignore_index, const float* lse, const float* dloss, void* dX,
                          void* workspace, size_t ws_bytes, void* stream);

/*
 * Standalone dequantization of a weight of any format to bf16 [N,K] (device, out),
 * element by element as defined for lora_weight_t (bit-exact; a bf16 weight is copied).
 * W_out must not overlap the weight's arrays.
 */
lora_status_t lora_dequant(const lora_weight_t* W, void* W_out, void* stream);

/*
 * Standalone dequantization of a LORA_W_BLOCK4 weight to bf16 [N,K] (device, out),
 * element by element as defined for lora_weight_t.  Bit-exact.  Not used by the
 * forward/backward, which dequantize tiles in shared memory and never write a
 * dequantized weight to device memory.
 */
lora_status_t dequant_blockwise4(const lora_weight_t* Wq, void* W_out, void* stream);

/*
 * Merge the adapter into the weight: W_out = W + s·B·A, bf16 [N,K] (device, out),
 * accumulated in fp32 ("Rev vs unsloth", GGUF export paragraph: merging LoRA adapters
 * into base weights; "Unsloth vs The Stack v2", merge paragraph).  W may be bf16
 * (W_out may then alias W->data exactly) or 4-bit / 8-bit (dequantized first, element by
 * element as in lora_dequant).  A: device bf16 [r,K]; B: device bf16 [N,r].
 */
lora_status_t lora_merge(const lora_weight_t* W, const void* A, const void* B, int32_t r,
                         float s, void* W_out, void* stream);

/*
 * Forward without any memory allocation and without a caller-provided workspace.
 * (The pages describe no such call; it exists for callers of this library.)
 *
 * Who needs it: callers that are handed only their input and output buffers and may
 * not obtain any other device memory — for example a plugin running inside a host
 * framework whose memory is entirely owned by that framework's pool allocator, or
 * latency-critical code that must not call cudaMalloc/cudaFree because those calls
 * can synchronize the whole device and may fail under a fixed memory budget.
 *
 * Computes what lora_linear_fwd computes, with two differences of schedule, both because
 * the larger partial-sum buffers they need do not fit the fixed scratch: X·Aᵀ always
 * runs as the split pass over K whose partial sums are added in order (lora_linear_fwd
 * takes a one-pass TMA-fed kernel for r <= 16 at most sizes), and every output tile of
 * the GEMM is computed whole (lora_linear_fwd takes the stream-K schedule for some small
 * outputs).  Both change only the order of fp32 additions, so XA and Y agree with
 * lora_linear_fwd's within the parity tolerance, not necessarily bit for bit.  Its
 * scratch (s·XA and the split partial sums of X·Aᵀ) is one fixed array of
 * LORA_NOALLOC_SCRATCH_BYTES bytes that is part of the library image: every GPU that
 * loads the library holds that array until the process exits.
 * The call allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *
 *   - Size limit: the scratch a problem needs is 2·M·r bytes for s·XA plus 4·S·M·r
 *     bytes of partial sums (S = number of K splits, which shrinks as M grows), each
 *     rounded up to 256 bytes.  It fits in LORA_NOALLOC_SCRATCH_BYTES = 16 MiB whenever
 *     6·M·r + 76000·r <= 16 MiB, e.g. up to about 160 000 tokens at r = 16 and about
 *     9 000 tokens at r = 128.  A larger problem gets LORA_ERR_SCRATCH_LIMIT and
 *     nothing is enqueued.  Other arguments are validated as for lora_linear_fwd.
 *   - First call on each device: it looks up the device address of the array on that
 *     device (the current device) and caches it for the current CUDA context; a
 *     context created anew (after cudaDeviceReset) gets the lookup again on its first
 *     call.  Make that first call before any stream capture begins on the device.
 *   - Shared state: all calls in the process share the one array per device, and the
 *     array keeps whatever the last call left in it.  Every scratch byte a call reads
 *     is written earlier by the same call, so nothing needs clearing between calls.
 *     Calls whose work overlaps on the GPU (different streams, or different host
 *     threads without ordering) race on the array and corrupt each other's results:
 *     order them on one stream or synchronize between them.
 *   - A device-side wait that runs out ends the kernels (no hang) but is not reported:
 *     there is no workspace to hold the status word.
 */
#define LORA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
lora_status_t lora_linear_fwd_noalloc(const void* X, int64_t M, const lora_weight_t* W,
                                      const void* A, const void* B, int32_t r, float s,
                                      void* Y, void* XA, void* stream);

/*
 * Reads and clears the device status word in `workspace` (synchronizes `stream`).
 * Returns LORA_OK, or LORA_ERR_DEVICE_TIMEOUT if a kernel of an earlier call gave up a
 * bounded wait (its outputs are then undefined), or LORA_ERR_DEVICE_BOUNDS if a kernel of
 * the checked build (compiled with -DLORA_CHECKED=1) found a tile or TMA box origin out of
 * range and skipped that copy (outputs undefined; the regular build does not test), or
 * LORA_ERR_CUDA.
 */
lora_status_t lora_device_status(void* workspace, void* stream);

/* Static message for a status code (never NULL). */
const char* lora_status_string(int32_t status);

/* Library version as major*10000 + minor*100 + patch. */
int32_t lora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LORA_LINEAR_H */
