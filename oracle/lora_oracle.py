"""Plain fp64 CPU oracle for the LoRA-adapted linear layer.

TEST INFRASTRUCTURE ONLY.  This module is what the CUDA library is checked against.
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import it; the library (``qlora_linear_b200``) never does, and this module
imports nothing from the library.

What it computes (the method is exact, so the oracle is the plain definition):

* Forward of a linear layer with a frozen weight ``W:[N,K]`` and a rank-``r``
  adapter ``A:[r,K]``, ``B:[N,r]`` scaled by ``s = alpha/r``::

      XA = X·Aᵀ                  [M,r]
      Y  = X·Wᵀ + s·XA·Bᵀ        [M,N]

  The adapter product is bracketed skinny-first, so the ``N×K`` matrix ``B·A`` is
  never built ("Unsloth vs PyTorch: The ONLY Video You Need to Understand the
  Difference", transcript 1:35-2:00, on associativity and the skinny adapter).
* Backward with ``W`` frozen (no ``dW``), derived by hand rather than by autograd
  (same page, transcript 0:43-1:35; "Unsloth" wiki entry, Theory, second bullet)::

      dYB = dY·B                 [M,r]
      dX  = dY·W + s·dYB·A       [M,K]
      dB  = s·dYᵀ·XA             [N,r]
      dA  = s·dYBᵀ·X             [r,K]

* The 4-bit blockwise weight ("Rev vs unsloth", fused quantized-LoRA paragraph;
  "Unsloth vs The Stack v2", quantized fine-tuning paragraph): packed codes
  ``[N, K/2]`` (element ``2j`` in the low nibble, ``2j+1`` in the high nibble),
  one fp16 absmax per 64 contiguous elements of the row-major weight and a
  16-entry float32 codebook.  One element dequantizes to
  ``bf16_rn(fp32_rn(codebook[code] * absmax))``.
* The feed-forward block (gate and up LoRA linears, ``H = silu(G)·U``, down LoRA
  linear) and its chain-rule backward, see :func:`lora_mlp_forward`.
* The 8-bit weights ("Rev vs unsloth", fused quantized-LoRA paragraph: int8 and fp8;
  "Unsloth vs The Stack v2", quantized fine-tuning paragraph: 8-bit): one int8 or fp8
  e4m3 byte per element and one fp32 scale per weight row; an element dequantizes to
  ``bf16_rn(fp32_rn(value(code) * scale[row]))``.
* Cross-entropy over a frozen LM head and its gradient in the hidden states, see
  :func:`cross_entropy`.
* Merge of the adapter into the weight ("Rev vs unsloth", GGUF export paragraph;
  "Unsloth vs The Stack v2", merge paragraph): ``W' = W + s·B·A``.

Everything runs in fp64 on the exact values of the bf16 / fp16 / fp32 inputs;
matrix products use numpy's fp64 ``matmul`` as a library primitive, with no
blocking or reordering beyond the formulas above.

Parity pins: every function here is pinned by a CPU test against something other
than itself (brute force on tiny integer inputs, associativity and merge
invariants, the B = 0 and W = 0 special cases, finite differences, an exhaustive
codebook round trip).  No function is left unpinned.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# storage types -> fp64 (exact widening)
# ----------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly (bf16 is the top half of fp32)."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def fp16_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE half bit patterns (uint16) -> float64, exactly."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (8 significant bits, ties to even); uint16 bits.

    Written from the definition: split ``x = m·2^e`` with ``0.5 <= |m| < 1``, keep
    ``round_half_even(m·2^8)`` and rescale.  Valid for zero and normal values, which
    is the whole domain this oracle meets (products of fp32 codebook levels and
    normal fp16 scales); subnormal inputs are rejected.
    """
    v = np.asarray(x, dtype=np.float32).astype(np.float64)
    if not np.all(np.isfinite(v)):
        raise ValueError("bf16_round_bits: non-finite input")
    tiny = np.abs(v) < np.float64(np.finfo(np.float32).tiny)
    if np.any(tiny & (v != 0)):
        raise ValueError("bf16_round_bits: subnormal input")
    m, e = np.frexp(v)
    q = np.rint(m * 256.0)  # numpy rint rounds half to even
    r = np.ldexp(q, e - 8)
    r32 = r.astype(np.float32)  # exact: r has <= 8 significant bits
    if not np.all(np.isfinite(r32)):
        raise ValueError("bf16_round_bits: overflow")
    return (r32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------------------
# 4-bit blockwise format
# ----------------------------------------------------------------------------

BLOCK = 64


def _unpack_codes(codes: np.ndarray, N: int, K: int) -> np.ndarray:
    """[N, K/2] packed bytes -> [N, K] codes; element 2j is the low nibble of byte j."""
    c = np.asarray(codes, dtype=np.uint8).reshape(N, K // 2)
    out = np.empty((N, K), dtype=np.uint8)
    out[:, 0::2] = c & 0x0F
    out[:, 1::2] = c >> 4
    return out


def dequant_blockwise4(codes: np.ndarray, absmax: np.ndarray, codebook: np.ndarray,
                       N: int, K: int) -> np.ndarray:
    """Dequantize the 4-bit blockwise weight to bf16 bit patterns ``[N, K]``.

    Element ``(n, k)`` has code ``c`` and lies in block ``b = (n*K + k) // 64`` of the
    row-major weight; its value is ``bf16_rn(fp32_rn(codebook[c] * absmax[b]))``.
    The fp64 product of an fp32 level and an fp16 scale is exact, so rounding it to
    float32 gives the correctly rounded fp32 product.
    """
    if K % BLOCK:
        raise ValueError("K must be a multiple of 64")
    c = _unpack_codes(codes, N, K)
    level = np.asarray(codebook, dtype=np.float32).astype(np.float64)[c]
    scale = fp16_to_f64(np.asarray(absmax).reshape(-1)[: N * K // BLOCK]).reshape(N, K // BLOCK)
    prod = level * np.repeat(scale, BLOCK, axis=1)
    return bf16_round_bits(prod.astype(np.float32))


def nearest_codes(values: np.ndarray, scales: np.ndarray, codebook: np.ndarray) -> np.ndarray:
    """Code of the nearest level for each value of each block.

    ``values`` is ``[nblocks, 64]``, ``scales`` (fp64) is ``[nblocks]``.  Each value
    takes ``argmin_i |v/scale - codebook[i]|``, ties to the lower index; a block
    whose scale is zero takes code 7 everywhere.
    """
    v = np.asarray(values, dtype=np.float64)
    scale = np.asarray(scales, dtype=np.float64)
    cb = np.asarray(codebook, dtype=np.float32).astype(np.float64)
    safe = np.where(scale > 0, scale, 1.0)
    dist = np.abs(v[..., None] / safe[:, None, None] - cb)
    code = np.argmin(dist, axis=-1).astype(np.uint8)  # first minimum = lower index
    code[scale == 0] = 7
    return code


def quantize_blockwise4(W: np.ndarray, codebook: np.ndarray):
    """Quantize an ``[N, K]`` weight to the 4-bit blockwise format.

    Per block of 64 contiguous elements: ``scale = fp16_rn(max |w|)`` and each
    element takes its nearest level (:func:`nearest_codes`).
    Returns ``(codes uint8 [N, K/2], absmax uint16 [N*K/64])``.
    """
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 64")
    blocks = W.reshape(N * K // BLOCK, BLOCK)
    scale16 = np.max(np.abs(blocks), axis=1).astype(np.float16)
    code = nearest_codes(blocks, scale16.astype(np.float64), codebook).reshape(N, K)
    packed = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)
    return packed, scale16.view(np.uint16)


# ----------------------------------------------------------------------------
# 8-bit formats: int8 or fp8 e4m3 codes, one fp32 scale per weight row
# ----------------------------------------------------------------------------


def int8_value(codes: np.ndarray) -> np.ndarray:
    """Two's-complement value of each byte."""
    return np.asarray(codes, dtype=np.uint8).view(np.int8).astype(np.float64)


def e4m3_value(codes: np.ndarray) -> np.ndarray:
    """Value of each fp8 e4m3 byte: sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
    exponent field 0 is subnormal (``m/8 · 2^-6``); exponent 15 with mantissa 7 is NaN
    and there are no infinities, so the largest finite value is ``1.75 · 2^8 = 448``."""
    b = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & ((b & 7) == 7), np.nan, mag)
    return sign * mag


def code8_value(codes: np.ndarray, fmt: str) -> np.ndarray:
    return int8_value(codes) if fmt == "int8" else e4m3_value(codes)


def dequant_rowwise8(codes: np.ndarray, row_scale: np.ndarray, fmt: str) -> np.ndarray:
    """Dequantize 8-bit codes ``[N, K]`` with fp32 row scales ``[N]`` to bf16 bit patterns:
    element ``(n, k)`` is ``bf16_rn(fp32_rn(value(code) · scale[n]))``.  value(code) has at
    most 8 significant bits and the scale 24, so the fp64 product is exact and its
    float32 cast is the correctly rounded fp32 product."""
    v = code8_value(codes, fmt)
    sc = np.asarray(row_scale, dtype=np.float32).astype(np.float64)
    return bf16_round_bits((v * sc[:, None]).astype(np.float32))


def e4m3_finite_values() -> np.ndarray:
    """The 254 finite e4m3 values by code (codes 0x7F and 0xFF left out)."""
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    return codes, e4m3_value(codes)


def e4m3_nearest(x: np.ndarray) -> np.ndarray:
    """Code of the e4m3 value nearest to each x (|x| <= 448), ties to the code with an even
    mantissa; the sign of zero follows x."""
    x = np.asarray(x, dtype=np.float64)
    codes, vals = e4m3_finite_values()
    pos = vals >= 0
    pc, pv = codes[pos & (codes < 0x80)], vals[pos & (codes < 0x80)]  # +0 .. 448
    a = np.abs(x)
    d = np.abs(a[..., None] - pv)
    best = d.min(axis=-1, keepdims=True)
    tie = d == best
    # among equally near codes take the even one (at most two candidates)
    even = tie & ((pc & 1) == 0)
    pick = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(tie, axis=-1))
    c = pc[pick].astype(np.uint8)
    return np.where(np.signbit(x), c | 0x80, c).astype(np.uint8)


def quantize_rowwise8(W: np.ndarray, fmt: str):
    """Quantize ``[N, K]`` to 8-bit codes with one fp32 scale per row:
    int8: ``scale = fp32(max|w| / 127)``, ``code = clip(rint(w/scale), -127, 127)``;
    fp8:  ``scale = fp32(max|w| / 448)``, ``code = e4m3_nearest(w/scale)``.
    A zero row takes scale 0 and code 0.  Returns ``(codes uint8 [N, K], scale float32 [N])``."""
    W = np.asarray(W, dtype=np.float64)
    top = 127.0 if fmt == "int8" else 448.0
    scale = (np.max(np.abs(W), axis=1) / top).astype(np.float32)
    safe = np.where(scale > 0, scale.astype(np.float64), 1.0)
    q = W / safe[:, None]
    if fmt == "int8":
        codes = np.clip(np.rint(q), -127, 127).astype(np.int8).view(np.uint8)
    else:
        codes = e4m3_nearest(np.clip(q, -448.0, 448.0))
    codes[scale == 0] = 0
    return codes, scale


def weight_f64(inputs: dict) -> np.ndarray:
    """The frozen weight of an input dict as fp64 ``[N, K]`` (dequantized if 4- or 8-bit)."""
    if inputs.get("W") is not None:
        return bf16_to_f64(inputs["W"])
    case = inputs["case"]
    if case.fmt in ("int8", "fp8"):
        return bf16_to_f64(dequant_rowwise8(inputs["codes"], inputs["row_scale"], case.fmt))
    bits = dequant_blockwise4(inputs["codes"], inputs["absmax"], inputs["codebook"], case.N, case.K)
    return bf16_to_f64(bits)


# ----------------------------------------------------------------------------
# the layer
# ----------------------------------------------------------------------------


def lora_forward(X: np.ndarray, W: np.ndarray, A: np.ndarray, B: np.ndarray, s: float):
    """Forward: returns ``(Y, XA)`` with ``XA = X·Aᵀ`` and ``Y = X·Wᵀ + s·XA·Bᵀ`` (fp64)."""
    X, W, A, B = (np.asarray(t, dtype=np.float64) for t in (X, W, A, B))
    XA = X @ A.T
    Y = X @ W.T + s * (XA @ B.T)
    return Y, XA


def lora_backward(dY: np.ndarray, X: np.ndarray, W: np.ndarray, A: np.ndarray,
                  B: np.ndarray, s: float) -> dict:
    """Backward with frozen ``W``: returns dict with ``dX, dA, dB`` and the skinny
    intermediates ``XA = X·Aᵀ``, ``dYB = dY·B`` (all fp64)."""
    dY, X, W, A, B = (np.asarray(t, dtype=np.float64) for t in (dY, X, W, A, B))
    XA = X @ A.T
    dYB = dY @ B
    dX = dY @ W + s * (dYB @ A)
    dB = s * (dY.T @ XA)
    dA = s * (dYB.T @ X)
    return {"dX": dX, "dA": dA, "dB": dB, "XA": XA, "dYB": dYB}


def lora_forward_rows(X_rows: np.ndarray, W: np.ndarray, A: np.ndarray, B: np.ndarray,
                      s: float):
    """Rows of ``(Y, XA)`` for a subset of the tokens (each output row depends only on
    its own input row)."""
    return lora_forward(X_rows, W, A, B, s)


def lora_backward_rows(dY_rows: np.ndarray, W: np.ndarray, A: np.ndarray, B: np.ndarray,
                       s: float) -> np.ndarray:
    """Rows of ``dX`` for a subset of the tokens: ``dX[m] = dY[m]·W + s·(dY[m]·B)·A``."""
    dY_rows, W, A, B = (np.asarray(t, dtype=np.float64) for t in (dY_rows, W, A, B))
    return dY_rows @ W + s * ((dY_rows @ B) @ A)


def lora_merge(W: np.ndarray, A: np.ndarray, B: np.ndarray, s: float) -> np.ndarray:
    """Merged weight ``W' = W + s·B·A`` (fp64, ``[N, K]``)."""
    W, A, B = (np.asarray(t, dtype=np.float64) for t in (W, A, B))
    return W + s * (B @ A)


def lora_adapter_grads_sampled(dY_bits: np.ndarray, X_bits: np.ndarray, A: np.ndarray, B: np.ndarray, s: float,
                               n_idx: np.ndarray, k_idx: np.ndarray, chunk_rows: int = 2048):
    """Selected rows of ``dB = s·dYᵀ·XA`` and columns of ``dA = s·dYBᵀ·X`` for large
    problems, accumulating over the tokens in chunks of ``chunk_rows`` so that only a
    chunk of ``X``/``dY`` is held in fp64 at a time.

    ``dY_bits`` [M,N] and ``X_bits`` [M,K] are bf16 bit patterns; ``A`` [r,K] and ``B``
    [N,r] are fp64.  Returns ``(dB[n_idx, :], dA[:, k_idx])``.  Each output element is
    the same sum over m as in :func:`lora_backward`, split into consecutive chunks.
    """
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    M = dY_bits.shape[0]
    r = A.shape[0]
    dB = np.zeros((len(n_idx), r))
    dA = np.zeros((r, len(k_idx)))
    for m0 in range(0, M, chunk_rows):
        Xc = bf16_to_f64(X_bits[m0:m0 + chunk_rows])
        dYc = bf16_to_f64(dY_bits[m0:m0 + chunk_rows])
        XAc = Xc @ A.T
        dYBc = dYc @ B
        dB += dYc[:, n_idx].T @ XAc
        dA += dYBc.T @ Xc[:, k_idx]
    return s * dB, s * dA


# ----------------------------------------------------------------------------
# several LoRA linears sharing one input (e.g. the q, k, v projections)
# ----------------------------------------------------------------------------


def lora_grouped_forward(X: np.ndarray, Ws: list, As: list, Bs: list, s: float):
    """G LoRA linears that read the same X (the attention block's q, k and v projections,
    whose six adapter derivatives "Unsloth vs PyTorch: The ONLY Video You Need to
    Understand the Difference" counts at transcript 1:14-1:24).  Returns
    ``(Y, XA)``: Y is the G outputs side by side ``[M, ΣN_g]``, XA the G skinny products
    side by side ``[M, G·r]``; each part is :func:`lora_forward` of its projection."""
    outs = [lora_forward(X, W, A, B, s) for W, A, B in zip(Ws, As, Bs)]
    return np.concatenate([y for y, _ in outs], axis=1), np.concatenate([xa for _, xa in outs], axis=1)


def lora_grouped_backward(dY: np.ndarray, X: np.ndarray, Ws: list, As: list, Bs: list, s: float) -> dict:
    """Backward of :func:`lora_grouped_forward`: ``dY`` is ``[M, ΣN_g]``.  dX is the sum
    of the G projections' dX (X feeds all of them); dA and dB are per projection,
    stacked: dA ``[G·r, K]``, dB ``[ΣN_g, r]``; dYB ``[M, G·r]``."""
    dY = np.asarray(dY, dtype=np.float64)
    offs = np.cumsum([0] + [np.asarray(W).shape[0] for W in Ws])
    parts = [lora_backward(dY[:, offs[g]:offs[g + 1]], X, Ws[g], As[g], Bs[g], s) for g in range(len(Ws))]
    dX = parts[0]["dX"].copy()
    for q in parts[1:]:
        dX += q["dX"]
    return {"dX": dX, "dA": np.concatenate([q["dA"] for q in parts], axis=0),
            "dB": np.concatenate([q["dB"] for q in parts], axis=0),
            "dYB": np.concatenate([q["dYB"] for q in parts], axis=1),
            "XA": np.concatenate([q["XA"] for q in parts], axis=1)}


# ----------------------------------------------------------------------------
# the feed-forward block: gate and up LoRA linears, SwiGLU, down LoRA linear
# ----------------------------------------------------------------------------


def sigmoid(g: np.ndarray) -> np.ndarray:
    """The logistic function 1/(1+e^-g), evaluated without overflow on either side."""
    g = np.asarray(g, dtype=np.float64)
    e = np.exp(-np.abs(g))
    return np.where(g >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def swiglu_forward(G: np.ndarray, U: np.ndarray) -> np.ndarray:
    """SwiGLU gating of the feed-forward block: ``H = silu(G)·U`` element by element,
    with ``silu(g) = g·sigmoid(g)`` (the "SwiGLU block" that the "Unsloth" wiki entry,
    Theory, first bullet, lists among the fused kernels; Llama's feed-forward)."""
    G = np.asarray(G, dtype=np.float64)
    return G * sigmoid(G) * np.asarray(U, dtype=np.float64)


def swiglu_backward(dH: np.ndarray, G: np.ndarray, U: np.ndarray):
    """Hand-derived derivatives of ``H = silu(G)·U``: with ``σ = sigmoid(G)``,
    ``silu'(g) = σ·(1 + g·(1-σ))``, so ``dG = dH·U·σ·(1 + G·(1-σ))`` and
    ``dU = dH·G·σ``."""
    G = np.asarray(G, dtype=np.float64)
    U = np.asarray(U, dtype=np.float64)
    dH = np.asarray(dH, dtype=np.float64)
    sg = sigmoid(G)
    return dH * U * sg * (1.0 + G * (1.0 - sg)), dH * G * sg


def lora_mlp_forward(X: np.ndarray, W_gu: np.ndarray, A_gu: np.ndarray, B_gu: np.ndarray,
                     W_d: np.ndarray, A_d: np.ndarray, B_d: np.ndarray, s: float) -> dict:
    """Feed-forward block with LoRA on all three projections ("Unsloth" wiki entry, Theory:
    fused SwiGLU block and hand-derived LoRA backward; "Unsloth vs PyTorch: The ONLY Video
    You Need to Understand the Difference", transcript 2:11-2:22, the feed-forward blocks).

    ``W_gu:[2I,D]`` is the gate weight stacked over the up weight, ``A_gu:[2r,D]`` and
    ``B_gu:[2I,r]`` their adapters stacked the same way; ``W_d:[D,I]``, ``A_d:[r,I]``,
    ``B_d:[D,r]`` the down projection.  ``G`` and ``U`` are the gate and up LoRA
    linears of X, ``H = silu(G)·U`` and ``Z`` the down LoRA linear of H."""
    I2 = np.asarray(W_gu).shape[0]
    I = I2 // 2
    r = np.asarray(A_gu).shape[0] // 2
    G, XA_g = lora_forward(X, W_gu[:I], A_gu[:r], B_gu[:I], s)
    U, XA_u = lora_forward(X, W_gu[I:], A_gu[r:], B_gu[I:], s)
    H = swiglu_forward(G, U)
    Z, XA_d = lora_forward(H, W_d, A_d, B_d, s)
    return {"Z": Z, "H": H, "G": G, "U": U, "XA_gu": np.concatenate([XA_g, XA_u], axis=1), "XA_d": XA_d}


def lora_mlp_backward(dZ: np.ndarray, X: np.ndarray, W_gu: np.ndarray, A_gu: np.ndarray, B_gu: np.ndarray,
                      W_d: np.ndarray, A_d: np.ndarray, B_d: np.ndarray, s: float) -> dict:
    """Backward of :func:`lora_mlp_forward` by the chain rule, one step at a time: the down
    projection's backward gives ``dH`` (its dX) and the down adapter's gradients; SwiGLU's
    derivative gives ``dG``, ``dU``; the gate and up projections' backward gives their
    adapter gradients (stacked like the forward's) and ``dX = dX_gate + dX_up``."""
    I = np.asarray(W_gu).shape[0] // 2
    r = np.asarray(A_gu).shape[0] // 2
    f = lora_mlp_forward(X, W_gu, A_gu, B_gu, W_d, A_d, B_d, s)
    gd = lora_backward(dZ, f["H"], W_d, A_d, B_d, s)
    dH = gd["dX"]
    dG, dU = swiglu_backward(dH, f["G"], f["U"])
    gg = lora_backward(dG, X, W_gu[:I], A_gu[:r], B_gu[:I], s)
    gu = lora_backward(dU, X, W_gu[I:], A_gu[r:], B_gu[I:], s)
    return {"dX": gg["dX"] + gu["dX"], "dA_gu": np.concatenate([gg["dA"], gu["dA"]], axis=0),
            "dB_gu": np.concatenate([gg["dB"], gu["dB"]], axis=0), "dA_d": gd["dA"], "dB_d": gd["dB"],
            "dH": dH, "dG": dG, "dU": dU, "fwd": f}


# ----------------------------------------------------------------------------
# cross-entropy over a frozen LM head
# ----------------------------------------------------------------------------


def cross_entropy(X: np.ndarray, W: np.ndarray, labels: np.ndarray, ignore_index: int, dloss=None):
    """Cross-entropy of the logits ``z = X·Wᵀ`` ("Unsloth" wiki entry, Theory: chunked
    cross-entropy; "Unsloth vs PyTorch: The ONLY Video You Need to Understand the
    Difference", transcript 3:06-3:51), the plain definition on the full logits:
    ``lse_m = log Σ_v exp(z_mv)`` (evaluated as ``max + log Σ exp(z - max)``),
    ``loss_m = lse_m - z_{m,y_m}`` and, when ``dloss`` is given,
    ``dX = (softmax(z) - onehot(y))·diag(dloss)·W``.  Rows whose label is ``ignore_index``
    have loss 0 and zero gradient.  Returns ``(loss, lse, dX or None)``."""
    X = np.asarray(X, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    y = np.asarray(labels, dtype=np.int64)
    z = X @ W.T
    zmax = z.max(axis=1, keepdims=True)
    lse = (zmax + np.log(np.sum(np.exp(z - zmax), axis=1, keepdims=True)))[:, 0]
    keep = y != ignore_index
    ysafe = np.where(keep, y, 0)
    loss = np.where(keep, lse - z[np.arange(len(y)), ysafe], 0.0)
    dX = None
    if dloss is not None:
        P = np.exp(z - lse[:, None])
        P[np.arange(len(y)), ysafe] -= 1.0
        P *= np.where(keep, np.asarray(dloss, dtype=np.float64), 0.0)[:, None]
        dX = P @ W
    return loss, lse, dX


def cross_entropy_rows_bits(X_rows_bits: np.ndarray, W_bits: np.ndarray, labels: np.ndarray, ignore_index: int,
                            dloss=None, chunk: int = 8192):
    """:func:`cross_entropy` for a few rows against a large bf16 head ``W_bits [V, D]``:
    the logits of the rows are built in full (fp64), converting the head to fp64
    ``chunk`` vocabulary rows at a time for the matrix products only."""
    X = bf16_to_f64(X_rows_bits)
    V = W_bits.shape[0]
    z = np.empty((X.shape[0], V))
    for v0 in range(0, V, chunk):
        z[:, v0:v0 + chunk] = X @ bf16_to_f64(W_bits[v0:v0 + chunk]).T
    y = np.asarray(labels, dtype=np.int64)
    zmax = z.max(axis=1, keepdims=True)
    lse = (zmax + np.log(np.sum(np.exp(z - zmax), axis=1, keepdims=True)))[:, 0]
    keep = y != ignore_index
    ysafe = np.where(keep, y, 0)
    loss = np.where(keep, lse - z[np.arange(len(y)), ysafe], 0.0)
    dX = None
    if dloss is not None:
        P = np.exp(z - lse[:, None])
        P[np.arange(len(y)), ysafe] -= 1.0
        P *= np.where(keep, np.asarray(dloss, dtype=np.float64), 0.0)[:, None]
        dX = np.zeros((X.shape[0], W_bits.shape[1]))
        for v0 in range(0, V, chunk):
            dX += P[:, v0:v0 + chunk] @ bf16_to_f64(W_bits[v0:v0 + chunk])
    return loss, lse, dX
