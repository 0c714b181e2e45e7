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
                 stream=None, grads_f32: bool = False):
        """dX, dA, dB.  ``grads_f32``: dA and dB are fp32 (unrounded), for a sum over
        data-parallel ranks before the one rounding to bf16."""
        M = dY.shape[0]
        dev = dY.device
        gt = torch.float32 if grads_f32 else torch.bfloat16
        if out is None:
            dX = torch.empty((M, self.W.K), dtype=torch.bfloat16, device=dev) if need_dX else None
            dA = torch.empty((self.r, self.W.K), dtype=gt, device=dev)
            dB = torch.empty((self.W.N, self.r), dtype=gt, device=dev)
        else:
            dX, dA, dB = out
        _b.lora_linear_bwd_ex(dY, X, XA, M, self.W, self.A, self.B, self.r, self.s, dX, dA, dB,
                              _b.LORA_GRADS_F32 if grads_f32 else 0, self.workspace(M), stream=stream)
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
                 stream=None, grads_f32: bool = False):
        M = dY.shape[0]
        dev = dY.device
        gt = torch.float32 if grads_f32 else torch.bfloat16
        if out is None:
            dX = torch.empty((M, self.W.K), dtype=torch.bfloat16, device=dev) if need_dX else None
            dA = torch.empty((self.G * self.r, self.W.K), dtype=gt, device=dev)
            dB = torch.empty((self.W.N, self.r), dtype=gt, device=dev)
        else:
            dX, dA, dB = out
        _b.lora_grouped_bwd_ex(dY, X, XA, M, self.W, self.rows, self.A, self.B, self.r, self.s, dX, dA, dB,
                               _b.LORA_GRADS_F32 if grads_f32 else 0, self.workspace(M), stream=stream)
        return dX, dA, dB


class LoraMLP:
    """SwiGLU feed-forward block with LoRA on gate, up and down projections.

    ``gate_up`` is a :class:`LoraWeight` of shape ``[2I, D]`` (gate rows over up rows),
    ``down`` one of ``[D, I]``; ``A_gate_up [2r, D]``, ``B_gate_up [2I, r]``,
    ``A_down [r, I]``, ``B_down [D, r]`` are bf16 tensors.  ``forward`` returns ``Z`` and
    the tensors ``backward`` needs (``saved``: GU, H, XA_gate_up, XA_down); ``backward``
    overwrites ``saved["GU"]`` with ``[dG | dU]`` and returns
    ``(dX, dA_gate_up, dB_gate_up, dA_down, dB_down)``.
    """

    def __init__(self, gate_up: "_b.LoraWeight", down: "_b.LoraWeight", A_gate_up: torch.Tensor,
                 B_gate_up: torch.Tensor, A_down: torch.Tensor, B_down: torch.Tensor, alpha: float):
        self.gate_up, self.down = gate_up, down
        self.A_gate_up, self.B_gate_up, self.A_down, self.B_down = A_gate_up, B_gate_up, A_down, B_down
        self.D, self.I = gate_up.K, down.K
        self.r = int(A_down.shape[0])
        self.s = float(alpha) / float(self.r)
        self._ws = None
        self._ws_M = -1

    def c_struct(self):
        return _b.mlp_struct(self.gate_up, self.down, self.A_gate_up, self.B_gate_up, self.A_down, self.B_down)

    def workspace(self, M: int) -> torch.Tensor:
        if self._ws is None or self._ws_M < M:
            n = _b.mlp_workspace_bytes(M, self.D, self.I, self.r, self.gate_up.fmt)
            if n == 0:
                raise _b.LoraError(_b.LORA_ERR_UNSUPPORTED, "mlp_workspace_bytes")
            self._ws = torch.zeros(n, dtype=torch.uint8, device=self.A_down.device)
            self._ws_M = M
        return self._ws

    def alloc_saved(self, M: int, device) -> dict:
        bf = torch.bfloat16
        return {"GU": torch.empty((M, 2 * self.I), dtype=bf, device=device),
                "H": torch.empty((M, self.I), dtype=bf, device=device),
                "XA_gate_up": torch.empty((M, 2 * self.r), dtype=bf, device=device),
                "XA_down": torch.empty((M, self.r), dtype=bf, device=device)}

    def forward(self, X: torch.Tensor, Z=None, saved=None, stream=None):
        M = X.shape[0]
        if Z is None:
            Z = torch.empty((M, self.D), dtype=torch.bfloat16, device=X.device)
        if saved is None:
            saved = self.alloc_saved(M, X.device)
        _b.lora_mlp_fwd(X, M, self.c_struct(), self.r, self.s, Z, saved["GU"], saved["H"], saved["XA_gate_up"],
                        saved["XA_down"], self.workspace(M), stream=stream)
        return Z, saved

    def backward(self, dZ: torch.Tensor, X: torch.Tensor, saved: dict, need_dX: bool = True, out=None, stream=None,
                 grads_f32: bool = False):
        M = dZ.shape[0]
        dev = dZ.device
        bf = torch.bfloat16
        gt = torch.float32 if grads_f32 else bf
        if out is None:
            out = (torch.empty((M, self.D), dtype=bf, device=dev) if need_dX else None,
                   torch.empty((2 * self.r, self.D), dtype=gt, device=dev),
                   torch.empty((2 * self.I, self.r), dtype=gt, device=dev),
                   torch.empty((self.r, self.I), dtype=gt, device=dev),
                   torch.empty((self.D, self.r), dtype=gt, device=dev))
        dX, dAgu, dBgu, dAd, dBd = out
        _b.lora_mlp_bwd_ex(dZ, X, saved["GU"], saved["H"], saved["XA_gate_up"], saved["XA_down"], M,
                           self.c_struct(), self.r, self.s, dX, dAgu, dBgu, dAd, dBd,
                           _b.LORA_GRADS_F32 if grads_f32 else 0, self.workspace(M), stream=stream)
        return out


class LoraCrossEntropy:
    """Cross-entropy over a frozen bf16 LM head ``W [V, D]`` (a :class:`LoraWeight`), per
    row, without the ``[M, V]`` logits.  ``slice_`` (vocabulary rows per backward slice,
    0 = all) sizes the workspace; the backward takes the widest slice the workspace holds."""

    def __init__(self, W: "_b.LoraWeight", ignore_index: int = -100, slice_: int = 8192):
        self.W, self.ignore_index, self.slice = W, int(ignore_index), int(slice_)
        self._ws = None
        self._ws_M = -1

    def workspace(self, M: int) -> torch.Tensor:
        if self._ws is None or self._ws_M < M:
            n = _b.ce_workspace_bytes(M, self.W.K, self.W.N, self.slice)
            if n == 0:
                raise _b.LoraError(_b.LORA_ERR_UNSUPPORTED, "ce_workspace_bytes")
            self._ws = torch.zeros(n, dtype=torch.uint8, device=self.W.data.device)
            self._ws_M = M
        return self._ws

    def forward(self, X: torch.Tensor, labels: torch.Tensor, stream=None):
        M = X.shape[0]
        loss = torch.empty(M, dtype=torch.float32, device=X.device)
        lse = torch.empty(M, dtype=torch.float32, device=X.device)
        _b.lora_ce_fwd(X, M, self.W, labels, self.ignore_index, loss, lse, self.workspace(M), stream=stream)
        return loss, lse

    def backward(self, X: torch.Tensor, labels: torch.Tensor, lse: torch.Tensor, dloss: torch.Tensor, dX=None,
                 stream=None):
        M = X.shape[0]
        if dX is None:
            dX = torch.empty((M, self.W.K), dtype=torch.bfloat16, device=X.device)
        _b.lora_ce_bwd(X, M, self.W, labels, self.ignore_index, lse, dloss, dX, self.workspace(M), stream=stream)
        return dX
