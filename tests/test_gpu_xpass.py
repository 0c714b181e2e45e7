"""GPU parity of the two passes over X on the TMA-fed stream (the one-pass dY kernel in a
single-product mode): the forward's XA = X·Aᵀ and the backward's dA = (s·dY·B)ᵀ·X.  Each
case is checked to take those paths (the library's own choice) and compared in full with
the fp64 oracle, with token counts and input widths that leave ragged 64-row and 256-column
tiles, ranks 8 and 16, and a grouped layer whose stacked rank is 16."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import LoraCase, make_case, make_grouped_case
from tests.gpu_helpers import check, dev_bf16, host_f64, run_layer

pytestmark = pytest.mark.gpu

CASES = [
    # M, N, K, r, fmt, the passes that run on the TMA stream (bit 0 XA, bit 1 dA)
    (2000, 520, 4160, 8, "bf16", 3),
    (6000, 264, 2112, 16, "bf16", 3),
    (5000, 512, 4160, 16, "block4", 2),
    (8100, 256, 1088, 16, "bf16", 1),
]


@pytest.mark.parametrize("M,N,K,r,fmt,paths", CASES)
def test_xpass_tma_layer(lib, M, N, K, r, fmt, paths):
    assert lib.lora_testing_xpass_tma(M, K, r) == paths
    case = LoraCase(f"xpass_{M}_{N}_{K}_{r}_{fmt}", M, N, K, r, 2.0 * r, fmt, 7500 + M + r)
    inp = make_case(case)
    out = run_layer(lib, inp)
    W = O.weight_f64(inp)
    X, A, B, dY = (O.bf16_to_f64(inp[k]) for k in ("X", "A", "B", "dY"))
    Y, XA = O.lora_forward(X, W, A, B, case.s)
    g = O.lora_backward(dY, X, W, A, B, case.s)
    check("Y", host_f64(out["Y"]), Y)
    check("XA", host_f64(out["XA"]), XA)
    check("dX", host_f64(out["dX"]), g["dX"])
    check("dA", host_f64(out["dA"]), g["dA"])
    check("dB", host_f64(out["dB"]), g["dB"])


def test_xpass_tma_grouped(lib):
    """Two projections of rank 8 share X: both passes over X run at the stacked rank 16."""
    M, rows, K, r = 6000, [256, 264], 2112, 8
    assert lib.lora_testing_xpass_tma(M, K, 2 * r) == 3
    case = LoraCase("xpass_grouped", M, sum(rows), K, r, 2.0 * r, "bf16", 7600)
    inp = make_grouped_case(case, rows)
    W = lib.LoraWeight(case.N, case.K, dev_bf16(inp["W"]))
    X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    layer = lib.LoraGroupedLinear(W, rows, A, B, case.alpha)
    Y, XA = layer.forward(X)
    dX, dA, dB = layer.backward(dY, X, XA)
    torch.cuda.synchronize()
    assert lib.lora_device_status(layer.workspace(M)) == lib.LORA_OK
    Wall = O.weight_f64(inp)
    Aall, Ball = O.bf16_to_f64(inp["A"]), O.bf16_to_f64(inp["B"])
    offs = np.cumsum([0] + rows)
    Ws = [Wall[offs[g]:offs[g + 1]] for g in range(len(rows))]
    As = [Aall[g * r:(g + 1) * r] for g in range(len(rows))]
    Bs = [Ball[offs[g]:offs[g + 1]] for g in range(len(rows))]
    Xf, dYf = O.bf16_to_f64(inp["X"]), O.bf16_to_f64(inp["dY"])
    Yr, XAr = O.lora_grouped_forward(Xf, Ws, As, Bs, case.s)
    g = O.lora_grouped_backward(dYf, Xf, Ws, As, Bs, case.s)
    check("Y", host_f64(Y), Yr)
    check("XA", host_f64(XA), XAr)
    check("dX", host_f64(dX), g["dX"])
    check("dA", host_f64(dA), g["dA"])
    check("dB", host_f64(dB), g["dB"])
