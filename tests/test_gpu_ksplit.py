"""GPU parity of the GEMMs' split reduction: outputs with fewer tiles than the GPU has CTA
pairs cut each tile's reduction into ranges computed by different pairs into fp32
partials, added in split order by a second kernel.  Each case here is checked to take that
path (the library's own split choice) and compared in full with the fp64 oracle, with
ragged row counts, both LoRA fill widths of the quantized kernel (r <= 64 and r = 128),
every weight format and the grouped layer; a repeated call must give the same bits."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import LoraCase, make_case, make_grouped_case
from tests.gpu_helpers import check, dev_bf16, host_bits, host_f64, run_layer

pytestmark = pytest.mark.gpu

FMT = {"bf16": 0, "block4": 1, "int8": 2, "fp8": 3}

CASES = [
    # M, N, K, r, fmt
    (300, 2048, 4160, 16, "block4"),   # 4 splits of 65 fills forward, one ragged 512-row tile
    (300, 2048, 4096, 128, "block4"),  # two LoRA fills in split 0
    (100, 1024, 8256, 8, "bf16"),      # 4 splits of 65 fills forward, the last fill half empty
    (300, 2048, 4096, 32, "bf16"),     # 4 splits forward, none backward
    (200, 2048, 4096, 16, "int8"),
    (513, 1024, 4096, 64, "fp8"),      # two 512-row tiles, the second one row high
]


@pytest.mark.parametrize("M,N,K,r,fmt", CASES)
def test_ksplit_layer(lib, M, N, K, r, fmt):
    fwd_split = lib.lora_testing_gemm_ksplit(M, N, K, FMT[fmt])
    bwd_split = lib.lora_testing_gemm_ksplit(M, K, N, FMT[fmt])
    assert max(fwd_split, bwd_split) > 1, (fwd_split, bwd_split)
    case = LoraCase(f"ksplit_{M}_{N}_{K}_{r}_{fmt}", M, N, K, r, 2.0 * r, fmt, 7100 + M + r)
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
    # the partials are added in a fixed order: a second call gives the same bits
    layer = out["layer"]
    Y2, XA2 = layer.forward(out["X"])
    dX2, _, _ = layer.backward(out["dY"], out["X"], XA2)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(Y2), host_bits(out["Y"]))
    assert np.array_equal(host_bits(dX2), host_bits(out["dX"]))


def test_ksplit_grouped(lib):
    """Grouped projections at a small batch: the LoRA fill of split 0 picks each output
    tile's projection."""
    M, rows, K, r = 200, [1024, 512, 520], 4096, 16
    N = sum(rows)
    assert lib.lora_testing_gemm_ksplit(M, N, K, 0) > 1
    case = LoraCase("ksplit_grouped", M, N, K, r, 2.0 * r, "bf16", 7300)
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
