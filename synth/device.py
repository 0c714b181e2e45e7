"""Seeded synthetic inputs drawn directly on a CUDA device (for the benchmark, whose
inputs are too large to draw quickly on the host).  Same value recipe as
``synth.inputs`` (see its docstring), drawn with torch's device generator; values are
rounded to bf16 / fp16 by torch's round-to-nearest-even casts and nothing else happens
to them here."""
from __future__ import annotations

import math

import torch

from .inputs import RMS_FP8, RMS_INT8, LoraCase, codebook_levels

_TID = {"X": 1, "W": 2, "A": 3, "B": 4, "dY": 5, "codes": 6, "absmax": 7}


def _gen(device, seed: int, tid: int, rank: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tid * 7919 + rank * 104_729) % (2 ** 63))
    return g


def _normal_bf16(shape, std, device, g):
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def make_case_device(case: LoraCase, device, rank: int = 0, want=("X", "W", "A", "B", "dY")) -> dict:
    M, N, K, r = case.M, case.N, case.K, case.r
    ds = case.data_seed if case.data_seed is not None else case.seed
    xs = case.x_seed if case.x_seed is not None else ds
    out: dict = {"case": case}
    if "X" in want:
        out["X"] = _normal_bf16((M, K), 1.0, device, _gen(device, xs, _TID["X"], rank))
    if "W" in want:
        if case.fmt == "bf16":
            out["W"] = _normal_bf16((N, K), 1.0 / math.sqrt(K), device, _gen(device, ds, _TID["W"], rank))
        elif case.fmt in ("int8", "fp8"):
            g = _gen(device, ds, _TID["codes"], rank)
            if case.fmt == "int8":
                out["codes"] = torch.randint(-127, 128, (N, K), generator=g, device=device,
                                             dtype=torch.int16).to(torch.int8).view(torch.uint8)
                rms = RMS_INT8
            else:
                sign = torch.randint(0, 2, (N, K), generator=g, device=device, dtype=torch.uint8)
                expo = torch.randint(1, 15, (N, K), generator=g, device=device, dtype=torch.uint8)
                mant = torch.randint(0, 8, (N, K), generator=g, device=device, dtype=torch.uint8)
                out["codes"] = (sign << 7) | (expo << 3) | mant
                rms = RMS_FP8
            g = _gen(device, ds, _TID["absmax"], rank)
            u = torch.rand(N, generator=g, device=device, dtype=torch.float32)
            out["row_scale"] = (0.8 + 0.4 * u) / (rms * math.sqrt(K))
        else:
            g = _gen(device, ds, _TID["codes"], rank)
            out["codes"] = torch.randint(0, 256, (N, K // 2), generator=g, device=device, dtype=torch.uint8)
            g = _gen(device, ds, _TID["absmax"], rank)
            u = torch.rand(N * K // 64, generator=g, device=device, dtype=torch.float32)
            out["absmax"] = ((1.2 + 0.8 * u) / math.sqrt(K)).to(torch.float16)
            out["codebook"] = torch.from_numpy(codebook_levels()).to(device)
    if "A" in want:
        a = 1.0 / math.sqrt(K)
        g = _gen(device, case.seed, _TID["A"], rank)
        out["A"] = (torch.rand((case.G * r, K), generator=g, device=device, dtype=torch.float32) * (2 * a) - a).to(torch.bfloat16)
    if "B" in want:
        out["B"] = _normal_bf16((N, r), 0.1, device, _gen(device, case.seed, _TID["B"], rank))
    if "dY" in want:
        out["dY"] = _normal_bf16((M, N), 1.0, device, _gen(device, ds, _TID["dY"], rank))
    return out
