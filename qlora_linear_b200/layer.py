"""A LoRA linear layer object over the C ABI: holds the frozen weight and the adapter
on the device, allocates outputs with torch and calls the library's forward and
hand-derived backward."""
from __future__ import annotations

import torch

from . import binding as _b


class LoraLinear:
    """Y = X·Wᵀ + s·(X·Aᵀ)·Bᵀ with W frozen (bf16 or 4-bit blockwise), s = alpha/r.

    ``W`` is a :class:`LoraWeight`; ``A`` bf16 [r, K] and ``B`` bf16 [N, r] are device
    tensors.  ``forward`` returns ``(Y, XA)``; keep ``XA`` for ``backward``.
    """

    def __init__(self, W: "_b.LoraWeight", A: torch.Tensor, B: torch.Tensor, alpha: float):
        self.W, self.A, self.B = W, A, B
        self.r = int(A.shape[0])
        self.s = float(alpha) / float(self.r)
        self._ws = None
        self._ws_M = -1

    def workspace(self, M: int) -> torch.Tensor:
        if self._ws is None or self._ws_M < M:
            self._ws = _b.alloc_workspace(M, self.W.N, self.W.K, self.r, self.W.fmt, device=self.A.device)
            self._ws_M = M
        return self._ws

    def forward(self, X: torch.Tensor, Y: torch.Tensor | None = None, XA: torch.Tensor | None = None, stream=None):
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, self.W.N), dtype=torch.bfloat16, device=X.device)
        if XA is None:
            XA = torch.empty((M, self.r), dtype=torch.bfloat16, device=X.device)
        _b.lora_linear_fwd(X, M, self.W, self.A, self.B, self.r, self.s, Y, XA, self.workspace(M), stream=stream)
        return Y, XA

    def backward(self, dY: torch.Tensor, X: torch.Tensor, XA: torch.Tensor, need_dX: bool = True, out=None,
                 stream=None):
        M = dY.shape[0]
        dev = dY.device
        if out is None:
            dX = torch.empty((M, self.W.K), dtype=torch.bfloat16, device=dev) if need_dX else None
            dA = torch.empty((self.r, self.W.K), dtype=torch.bfloat16, device=dev)
            dB = torch.empty((self.W.N, self.r), dtype=torch.bfloat16, device=dev)
        else:
            dX, dA, dB = out
        _b.lora_linear_bwd(dY, X, XA, M, self.W, self.A, self.B, self.r, self.s, dX, dA, dB, self.workspace(M),
                           stream=stream)
        return dX, dA, dB


class LoraGroupedLinear:
    """G LoRA linears reading the same X (e.g. q, k, v), run as one layer.

    ``W`` is a :class:`LoraWeight` over the stacked weights ``[ΣN_g, K]``; ``A`` bf16
    ``[G·r, K]`` and ``B`` bf16 ``[ΣN_g, r]`` stack the adapters; ``rows`` lists N_g.
    ``forward`` returns ``(Y, XA)`` with Y ``[M, ΣN_g]`` and XA ``[M, G·r]``;
    ``backward`` returns ``(dX, dA, dB)`` with dA ``[G·r, K]`` and dB ``[ΣN_g, r]``.
    """

    def __init__(self, W: "_b.LoraWeight", rows, A: torch.Tensor, B: torch.Tensor, alpha: float):
        self.W, self.rows, self.A, self.B = W, [int(n) for n in rows], A, B
        self.G = len(self.rows)
        self.r = int(A.shape[0]) // self.G
        self.s = float(alpha) / float(self.r)
        self._ws = None
        self._ws_M = -1

    def workspace(self, M: int) -> torch.Tensor:
        if self._ws is None or self._ws_M < M:
            n = _b.grouped_workspace_bytes(M, self.W.N, self.W.K, self.r, self.G, self.W.fmt)
            if n == 0:
                raise _b.LoraError(_b.LORA_ERR_UNSUPPORTED, "grouped_workspace_bytes")
            self._ws = torch.zeros(n, dtype=torch.uint8, device=self.A.device)
            self._ws_M = M
        return self._ws

    def forward(self, X: torch.Tensor, Y=None, XA=None, stream=None):
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, self.W.N), dtype=torch.bfloat16, device=X.device)
        if XA is None:
            XA = torch.empty((M, self.G * self.r), dtype=torch.bfloat16, device=X.device)
        _b.lora_grouped_fwd(X, M, self.W, self.rows, self.A, self.B, self.r, self.s, Y, XA, self.workspace(M),
                            stream=stream)
        return Y, XA

    def backward(self, dY: torch.Tensor, X: torch.Tensor, XA: torch.Tensor, need_dX: bool = True, out=None,
                 stream=None):
        M = dY.shape[0]
        dev = dY.device
        if out is None:
            dX = torch.empty((M, self.W.K), dtype=torch.bfloat16, device=dev) if need_dX else None
            dA = torch.empty((self.G * self.r, self.W.K), dtype=torch.bfloat16, device=dev)
            dB = torch.empty((self.W.N, self.r), dtype=torch.bfloat16, device=dev)
        else:
            dX, dA, dB = out
        _b.lora_grouped_bwd(dY, X, XA, M, self.W, self.rows, self.A, self.B, self.r, self.s, dX, dA, dB,
                            self.workspace(M), stream=stream)
        return dX, dA, dB
