"""fp32 adapter gradients (LORA_GRADS_F32) on the GPU, through the C ABI: rounded once
with lora_round_bf16 they equal the plain backward's bf16 gradients bit for bit (one GPU
is a data-parallel group of one), and unrounded they meet the oracle at the bar.  Covers
the layer, the grouped layer, the feed-forward block, the exchange buffer of the
data-parallel path and the rounding kernel itself."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import LoraCase, MlpCase, make_case, make_grouped_case, make_mlp_case
from tests.gpu_helpers import check, dev_bf16, host_bits, make_weight

pytestmark = pytest.mark.gpu


def _bits(t):
    return host_bits(t)


def _rounded(q, g32):
    out = torch.empty(g32.shape, dtype=torch.bfloat16, device=g32.device)
    q.lora_round_bf16(g32, out)
    return out


def _f32_close(name, got32, ref):
    """fp32 dA: no rounding of the output; its one rounded operand is the bf16 s·dY·B
    (2^-9 relative per element), which stays within 1e-2·rms."""
    got = got32.double().cpu().numpy()
    err = got - ref
    rms = np.linalg.norm(ref) / np.sqrt(ref.size)
    assert np.max(np.abs(err)) <= 1e-2 * rms, (name, float(np.max(np.abs(err)) / rms))


@pytest.mark.parametrize("M,N,K,r,fmt", [(300, 264, 192, 16, "bf16"), (129, 512, 256, 64, "block4"),
                                         (1000, 768, 320, 8, "int8"), (4096, 1024, 1024, 16, "bf16")])
def test_layer_f32_grads_round_to_plain_bits(lib, M, N, K, r, fmt):
    case = LoraCase(f"g32_{M}_{N}_{K}_{r}_{fmt}", M, N, K, r, 2.0 * r, fmt, 8100 + M + r)
    inp = make_case(case)
    W, keep = make_weight(lib, inp)
    X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    layer = lib.LoraLinear(W, A, B, case.alpha)
    Y, XA = layer.forward(X)
    dX, dA, dB = layer.backward(dY, X, XA)
    dX2, dA32, dB32 = layer.backward(dY, X, XA, grads_f32=True)
    torch.cuda.synchronize()
    assert lib.lora_device_status(layer.workspace(M)) == lib.LORA_OK
    assert dA32.dtype == torch.float32 and dB32.dtype == torch.float32
    assert np.array_equal(_bits(dX), _bits(dX2))
    assert np.array_equal(_bits(_rounded(lib, dA32)), _bits(dA))
    assert np.array_equal(_bits(_rounded(lib, dB32)), _bits(dB))
    Wf = O.weight_f64(inp)
    ref = O.lora_backward(O.bf16_to_f64(inp["dY"]), O.bf16_to_f64(inp["X"]), Wf, O.bf16_to_f64(inp["A"]),
                          O.bf16_to_f64(inp["B"]), case.s)
    # dB is computed from the bf16 XA of the forward (the oracle keeps XA exact): the plain
    # bar; dA to 1e-2·rms
    _f32_close("dA", dA32, ref["dA"])
    check("dB", dB32.double().cpu().numpy(), ref["dB"])


def test_grouped_f32_grads_round_to_plain_bits(lib):
    rows = [256, 256, 128]
    case = LoraCase("g32_grouped", 333, 640, 256, 16, 32.0, "bf16", 8200)
    inp = make_grouped_case(case, rows)
    W = lib.LoraWeight(case.N, case.K, dev_bf16(inp["W"]))
    X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    layer = lib.LoraGroupedLinear(W, rows, A, B, case.alpha)
    Y, XA = layer.forward(X)
    _, dA, dB = layer.backward(dY, X, XA)
    _, dA32, dB32 = layer.backward(dY, X, XA, grads_f32=True)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(_rounded(lib, dA32)), _bits(dA))
    assert np.array_equal(_bits(_rounded(lib, dB32)), _bits(dB))


@pytest.mark.parametrize("fmt", ["bf16", "block4"])
def test_mlp_f32_grads_round_to_plain_bits(lib, fmt):
    case = MlpCase(f"g32_mlp_{fmt}", 200, 192, 256, 16, 32.0, fmt, 8300)
    inp = make_mlp_case(case)
    Wgu, k1 = make_weight(lib, inp["gate_up"])
    Wd, k2 = make_weight(lib, inp["down"])
    X, Agu, Bgu, Ad, Bd, dZ = (dev_bf16(inp[k]) for k in ("X", "A_gu", "B_gu", "A_d", "B_d", "dZ"))
    mlp = lib.LoraMLP(Wgu, Wd, Agu, Bgu, Ad, Bd, case.alpha)
    plain, f32 = [], []
    for grads_f32, sink in ((False, plain), (True, f32)):
        Z, saved = mlp.forward(X)  # the backward overwrites the saved G, U: run the forward again
        sink.extend(mlp.backward(dZ, X, saved, grads_f32=grads_f32))
    torch.cuda.synchronize()
    assert lib.lora_device_status(mlp.workspace(case.M)) == lib.LORA_OK
    assert np.array_equal(_bits(plain[0]), _bits(f32[0]))  # dX
    for i in range(1, 5):
        assert f32[i].dtype == torch.float32
        assert np.array_equal(_bits(_rounded(lib, f32[i])), _bits(plain[i])), i


def test_exchange_buffer_on_one_gpu(lib):
    """The data-parallel step of a group of one: the backward writes into the exchange
    buffer's views, the all-reduce is a no-op, the rounding gives the plain bits."""
    from qlora_linear_b200 import AdapterGradExchange
    case = LoraCase("g32_ex", 512, 384, 256, 16, 32.0, "bf16", 8400)
    inp = make_case(case)
    W, keep = make_weight(lib, inp)
    X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    layer = lib.LoraLinear(W, A, B, case.alpha)
    Y, XA = layer.forward(X)
    dX, dA, dB = layer.backward(dY, X, XA)
    ex = AdapterGradExchange([dA.shape, dB.shape], "cuda")
    ex.flat.fill_(float("nan"))  # every element must be written by the backward
    layer.backward(dY, X, XA, out=(torch.empty_like(dX), ex.views[0], ex.views[1]), grads_f32=True)
    ex.allreduce()
    oA, oB = torch.empty_like(dA), torch.empty_like(dB)
    ex.round_into([oA, oB])
    torch.cuda.synchronize()
    assert np.array_equal(_bits(oA), _bits(dA)) and np.array_equal(_bits(oB), _bits(dB))


def test_round_bf16_is_nearest_even(lib):
    # normal values: exact, below and above half an ulp, ties to even of both parities,
    # a carry into the exponent, and a wide random sweep of magnitudes (against the
    # oracle's rounding, written from the definition)
    normal = np.array([1.0, 1.0 + 2 ** -9, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20,
                       -(1.0 + 2 ** -8), 2.0 - 2 ** -9, 3.0e38, 2 ** -126 * 1.5, 65504.0, -1.2345e-3],
                      dtype=np.float32)
    rng = np.random.default_rng(7)
    normal = np.concatenate([normal, (rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000))
                             .astype(np.float32)])
    # zeros, subnormals and infinities: against torch's round-to-nearest-even cast on the host
    special = np.array([0.0, -0.0, 1e-40, -3e-39, np.inf, -np.inf], dtype=np.float32)
    v = np.concatenate([normal, special])
    src = torch.from_numpy(v).cuda()
    out = torch.empty(v.size, dtype=torch.bfloat16, device="cuda")
    lib.lora_round_bf16(src, out)
    nan = torch.tensor([float("nan")], device="cuda")
    nan_out = torch.empty(1, dtype=torch.bfloat16, device="cuda")
    lib.lora_round_bf16(nan, nan_out)
    torch.cuda.synchronize()
    got = _bits(out)
    assert np.array_equal(got[:normal.size], O.bf16_round_bits(normal))
    ref_special = torch.from_numpy(special).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got[normal.size:], ref_special)
    assert torch.isnan(nan_out.float()).all()
