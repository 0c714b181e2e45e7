"""GPU parity of the GEMMs' stream-K schedule.  When an output's tiles do not fill the
GPU's CTA pairs evenly, every pair runs the same number of whole tiles and then an equal
share of the fills of the remaining tiles; pieces of tiles accumulate into fp32 slots that
a second kernel adds in pair order.  Each case here is checked to take that path (the
library's own schedule choice) and compared in full with the fp64 oracle: ragged row
counts, both kernels, every weight format, the quantized kernel's two LoRA fills at
r = 128, the grouped layer, and a repeated call giving the same bits.  The full-size
tests cover the schedule with whole-tile waves before the pieces (the QLoRA dX GEMM and
the rank sweep's 512-token shapes)."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import CONFIGS, LoraCase, make_case, make_grouped_case
from tests.gpu_helpers import check, dev_bf16, host_bits, host_f64, run_layer

pytestmark = pytest.mark.gpu

FMT = {"bf16": 0, "block4": 1, "int8": 2, "fp8": 3}

CASES = [
    # M, N, K, r, fmt
    (300, 2048, 8256, 16, "block4"),    # forward: 8 tiles of 129 + 1 fills shared by 74 pairs
    (300, 4096, 8192, 128, "block4"),   # forward and backward, two LoRA fills per tile
    (1100, 6400, 2048, 16, "block4"),   # backward: three row tiles, the last 76 rows high
    (300, 2048, 8192, 32, "bf16"),      # forward
    (250, 19200, 2048, 8, "bf16"),      # backward: dX reduces over 19200 (150 fills a tile)
    (200, 2048, 8192, 16, "int8"),
    (513, 1024, 8192, 64, "fp8"),       # two row tiles, the second one row high
]


@pytest.mark.parametrize("M,N,K,r,fmt", CASES)
def test_streamk_layer(lib, M, N, K, r, fmt):
    fwd = lib.lora_testing_gemm_streamk(M, N, K, r, FMT[fmt])
    bwd = lib.lora_testing_gemm_streamk(M, K, N, r, FMT[fmt])
    assert max(fwd, bwd) > 0, (fwd, bwd)
    case = LoraCase(f"streamk_{M}_{N}_{K}_{r}_{fmt}", M, N, K, r, 2.0 * r, fmt, 7100 + M + r)
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
    # the pieces are added in a fixed order: a second call gives the same bits
    layer = out["layer"]
    Y2, XA2 = layer.forward(out["X"])
    dX2, _, _ = layer.backward(out["dY"], out["X"], XA2)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(Y2), host_bits(out["Y"]))
    assert np.array_equal(host_bits(dX2), host_bits(out["dX"]))


def test_streamk_grouped(lib):
    """Grouped projections at a small batch: each piece's LoRA fills pick its tile's
    projection."""
    M, rows, K, r = 300, [2048, 1024, 1032], 8192, 16
    N = sum(rows)
    assert lib.lora_testing_gemm_streamk(M, N, K, r, 0) > 0
    case = LoraCase("streamk_grouped", M, N, K, r, 2.0 * r, "bf16", 7300)
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


def test_full_size_configs_take_streamk_with_whole_waves_first(lib):
    """The full-size parity tests run these through the schedule whose pairs first take
    whole tiles (waves of 74) and then the pieces: the QLoRA dX GEMM and the rank sweep."""
    c3 = CONFIGS["c3"][0]
    tiles = (c3.M + 511) // 512 * ((c3.K + 255) // 256)
    assert 0 < lib.lora_testing_gemm_streamk(c3.M, c3.K, c3.N, c3.r, FMT["block4"]) < tiles - 74
    c4 = [c for c in CONFIGS["c4"] if c.M == 512 and c.N == 28672 and c.fmt == "bf16" and c.r == 16][0]
    tiles = (c4.M + 255) // 256 * ((c4.N + 255) // 256)
    assert 0 < lib.lora_testing_gemm_streamk(c4.M, c4.N, c4.K, c4.r, FMT["bf16"]) < tiles - 74
