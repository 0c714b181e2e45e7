"""GPU parity of the one-pass dY·B / dYᵀ·XA kernel (rank r <= 16): the backward's two
rank-r products that read dY come from a single TMA-fed pass over dY.  Shapes are chosen so
that the pass is taken with several row and column blocks and ragged tails in M and in the
columns of dY; results are checked against the fp64 oracle element by element."""
import pytest
import torch

import oracle as O
from synth import LoraCase, make_case
from tests.gpu_helpers import check, dev_bf16, host_f64, make_weight, run_layer

pytestmark = pytest.mark.gpu

# M, N, K, r, fmt: M and N ragged against the 64 × 256 tiles, several blocks each way
DUAL = [
    (2000, 1800, 256, 16, "bf16"),
    (4000, 3000, 200, 8, "bf16"),
    (4000, 3000, 192, 16, "block4"),
    (3000, 2000, 136, 16, "bf16"),
]


def _check_all(inp, out):
    case = inp["case"]
    W = O.weight_f64(inp)
    X, A, B, dY = (O.bf16_to_f64(inp[k]) for k in ("X", "A", "B", "dY"))
    Y, XA = O.lora_forward(X, W, A, B, case.s)
    g = O.lora_backward(dY, X, W, A, B, case.s)
    check("Y", host_f64(out["Y"]), Y)
    check("dX", host_f64(out["dX"]), g["dX"])
    check("dA", host_f64(out["dA"]), g["dA"])
    check("dB", host_f64(out["dB"]), g["dB"])


@pytest.mark.parametrize("M,N,K,r,fmt", DUAL)
def test_dual_pass_parity(lib, M, N, K, r, fmt):
    case = LoraCase(f"dual_{M}_{N}_{K}_{r}_{fmt}", M, N, K, r, 2.0 * r, fmt, 7000 + M + N + K + r)
    inp = make_case(case)
    _check_all(inp, run_layer(lib, inp))


def test_dual_pass_is_taken(lib):
    """The backward of a dual-shaped case launches one pass over dY plus its two
    finalizes instead of two passes and two finalizes: 6 launches with dX, not 7."""
    case = LoraCase("dual_count", 2000, 1800, 256, 16, 32.0, "bf16", 7100)
    inp = make_case(case)
    W, keep = make_weight(lib, inp)
    X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    layer = lib.LoraLinear(W, A, B, case.alpha)
    Y, XA = layer.forward(X)
    n0 = lib.lora_launch_count()
    layer.backward(dY, X, XA)
    torch.cuda.synchronize()
    assert lib.lora_launch_count() - n0 == 6
    # a rank above 16 keeps the two separate passes
    case = LoraCase("sep_count", 2000, 1800, 256, 24, 48.0, "bf16", 7101)
    inp = make_case(case)
    W, keep = make_weight(lib, inp)
    X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    layer = lib.LoraLinear(W, A, B, case.alpha)
    Y, XA = layer.forward(X)
    n0 = lib.lora_launch_count()
    layer.backward(dY, X, XA)
    torch.cuda.synchronize()
    assert lib.lora_launch_count() - n0 == 7


def test_dual_pass_deterministic(lib):
    case = LoraCase("dual_det", 4000, 3000, 200, 16, 32.0, "bf16", 7200)
    inp = make_case(case)
    a = run_layer(lib, inp)
    b = run_layer(lib, inp)
    for k in ("dX", "dA", "dB"):
        assert torch.equal(a[k].view(torch.int16), b[k].view(torch.int16)), k

