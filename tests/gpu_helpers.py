"""Helpers shared by the GPU tests: upload seeded inputs, run the library, compare
with the oracle under the stated tolerance."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

# Parity bar for floating-point outputs (bf16 outputs, fp32 accumulation):
# relative Frobenius error <= 1e-2 and, element by element, |err| <= 5e-2 * rms(ref).
REL_FRO = 1e-2
ELEM_RMS = 5e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def dev_f16_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return O.bf16_to_f64(host_bits(t))


def make_weight(q, inp):
    case = inp["case"]
    if case.fmt == "bf16":
        w = dev_bf16(inp["W"])
        return q.LoraWeight(case.N, case.K, w), (w,)
    if case.fmt in ("int8", "fp8"):
        codes = dev_u8(inp["codes"])
        sc = torch.from_numpy(inp["row_scale"]).cuda()
        fmt = q.LORA_W_INT8 if case.fmt == "int8" else q.LORA_W_FP8_E4M3
        return q.LoraWeight(case.N, case.K, codes, sc, None, fmt), (codes, sc)
    codes = dev_u8(inp["codes"])
    absmax = dev_f16_bits(inp["absmax"])
    cb = torch.from_numpy(inp["codebook"]).cuda()
    return q.LoraWeight(case.N, case.K, codes, absmax, cb), (codes, absmax, cb)


def nan_canary(shape) -> torch.Tensor:
    """A bf16 output buffer filled with NaN: an element the kernels never write stays NaN
    and fails the parity check (which rejects non-finite values)."""
    return torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")


def run_layer(q, inp, need_dX=True):
    """Forward and backward of one case through the library, every output buffer
    NaN-filled first; returns device tensors."""
    case = inp["case"]
    W, keep = make_weight(q, inp)
    X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    layer = q.LoraLinear(W, A, B, case.alpha)
    M, N, K, r = case.M, case.N, case.K, case.r
    Y, XA = layer.forward(X, Y=nan_canary((M, N)), XA=nan_canary((M, r)))
    dX, dA, dB = layer.backward(dY, X, XA, out=(nan_canary((M, K)) if need_dX else None, nan_canary((r, K)),
                                                nan_canary((N, r))))
    torch.cuda.synchronize()
    st = q.lora_device_status(layer.workspace(case.M))
    assert st == q.LORA_OK, q.status_string(st)
    return {"Y": Y, "XA": XA, "dX": dX, "dA": dA, "dB": dB, "layer": layer, "keep": keep,
            "X": X, "dY": dY}


def check(name: str, got: np.ndarray, ref: np.ndarray, rel_elem: float = 0.0):
    """Parity bar.  ``rel_elem`` adds ``rel_elem·|ref|`` to the per-element bound for
    outputs whose own bf16 storage rounding (2^-8 relative) and that of the bf16 values
    they are computed from are not covered by ``ELEM_RMS·rms``: heavy-tailed products
    such as SwiGLU's derivatives, whose largest elements lie over 12·rms."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    err = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / nref if nref > 0 else np.linalg.norm(err)
    rms = nref / np.sqrt(ref.size) if ref.size else 0.0
    emax = np.max(np.abs(err)) if err.size else 0.0
    assert rel <= REL_FRO, f"{name}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    if rel_elem == 0.0:
        assert emax <= ELEM_RMS * rms + 1e-30, f"{name}: max |err| {emax:.3e} > {ELEM_RMS}*rms {rms:.3e}"
    else:
        excess = np.abs(err) - (ELEM_RMS * rms + rel_elem * np.abs(ref))
        worst = float(np.max(excess)) if excess.size else 0.0
        assert worst <= 1e-30, f"{name}: an element exceeds {ELEM_RMS}*rms + {rel_elem:.4f}*|ref| by {worst:.3e}"
    return rel, emax / rms if rms > 0 else 0.0
