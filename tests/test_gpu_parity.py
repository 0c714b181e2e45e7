"""GPU parity: the CUDA library (called through its C ABI) against the fp64 oracle on
seeded inputs.  Floating-point outputs must meet the parity bar in gpu_helpers
(relative Frobenius <= 1e-2, per element <= 5e-2·rms); the 4-bit dequantization must
match bit for bit."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import LoraCase, make_case
from synth.inputs import codebook_levels
from tests.gpu_helpers import (check, dev_bf16, dev_f16_bits, dev_u8, host_bits, host_f64, make_weight,
                               run_layer)

pytestmark = pytest.mark.gpu


def _full_check(inp, out, need_dX=True):
    case = inp["case"]
    W = O.weight_f64(inp)
    X, A, B, dY = (O.bf16_to_f64(inp[k]) for k in ("X", "A", "B", "dY"))
    Y, XA = O.lora_forward(X, W, A, B, case.s)
    g = O.lora_backward(dY, X, W, A, B, case.s)
    check("Y", host_f64(out["Y"]), Y)
    check("XA", host_f64(out["XA"]), XA)
    if need_dX:
        check("dX", host_f64(out["dX"]), g["dX"])
    check("dA", host_f64(out["dA"]), g["dA"])
    check("dB", host_f64(out["dB"]), g["dB"])


# ---------------------------------------------------------------- 4-bit dequant, bit-exact
@pytest.mark.parametrize("N,K", [(8, 64), (520, 320), (4096, 1024)])
def test_dequant_blockwise4_bit_exact(lib, N, K):
    rng = np.random.default_rng(N * 7 + K)
    codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    scales = rng.uniform(1e-4, 100.0, N * K // 64).astype(np.float16).view(np.uint16)
    for cb in (codebook_levels(), rng.standard_normal(16).astype(np.float32) * 3):
        W = lib.LoraWeight(N, K, dev_u8(codes), dev_f16_bits(scales), torch.from_numpy(cb).cuda())
        out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        lib.dequant_blockwise4(W, out)
        torch.cuda.synchronize()
        want = O.dequant_blockwise4(codes, scales, cb, N, K)
        assert np.array_equal(host_bits(out), want)


# ---------------------------------------------------------------- merge
@pytest.mark.parametrize("fmt,N,K,r", [("bf16", 264, 328, 24), ("block4", 520, 384, 128), ("bf16", 8, 8, 8)])
def test_merge(lib, fmt, N, K, r):
    case = LoraCase(f"merge_{fmt}", 1, N, K, r, 3.0 * r, fmt, 99)
    inp = make_case(case, want=("W", "A", "B"))
    W, keep = make_weight(lib, inp)
    A, B = dev_bf16(inp["A"]), dev_bf16(inp["B"])
    out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    lib.lora_merge(W, A, B, r, case.s, out)
    torch.cuda.synchronize()
    ref = O.lora_merge(O.weight_f64(inp), O.bf16_to_f64(inp["A"]), O.bf16_to_f64(inp["B"]), case.s)
    got = host_f64(out)
    # one rounding to bf16 of an fp32 sum: within one bf16 ulp of the exact value
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= ulp)
    # B = 0 gives the weight back bit for bit, also in place for a bf16 weight
    B0 = torch.zeros_like(B)
    lib.lora_merge(W, A, B0, r, case.s, out)
    torch.cuda.synchronize()
    wbits = inp["W"] if fmt == "bf16" else O.dequant_blockwise4(inp["codes"], inp["absmax"], inp["codebook"], N, K)
    assert np.array_equal(host_bits(out), wbits)
    if fmt == "bf16":
        w = keep[0].clone()
        Wt = lib.LoraWeight(N, K, w)
        lib.lora_merge(Wt, A, B, r, case.s, w)
        lib.lora_merge(W, A, B, r, case.s, out)
        torch.cuda.synchronize()
        assert torch.equal(w.view(torch.int16), out.view(torch.int16))


# ---------------------------------------------------------------- the layer, small and ragged
def test_c0_tiny_full(lib):
    from synth import CONFIGS
    inp = make_case(CONFIGS["c0"][0])
    _full_check(inp, run_layer(lib, inp))


RAGGED = [
    # M, N, K, r, fmt — several tiles of 128×256 plus a ragged tail in M, N and K
    (300, 520, 200, 8, "bf16"),
    (300, 520, 200, 24, "bf16"),
    (129, 264, 136, 72, "bf16"),
    (257, 776, 328, 128, "bf16"),
    (1, 8, 8, 8, "bf16"),
    (7, 16, 72, 40, "bf16"),
    (300, 520, 192, 16, "block4"),
    (257, 776, 320, 128, "block4"),
    (1, 8, 64, 8, "block4"),
    (130, 264, 128, 56, "block4"),
]


@pytest.mark.parametrize("M,N,K,r,fmt", RAGGED)
def test_ragged_shapes(lib, M, N, K, r, fmt):
    case = LoraCase(f"ragged_{M}_{N}_{K}_{r}_{fmt}", M, N, K, r, 2.0 * r + 1.0, fmt, 1000 + M + N + K + r)
    inp = make_case(case)
    _full_check(inp, run_layer(lib, inp))


def test_block4_matches_bf16_of_dequantized_weight(lib):
    """The fused 4-bit GEMM sees exactly the dequantized bf16 weight: same tiles, same
    accumulation order, so Y and dX agree bit for bit with the bf16 path on dequant(W)."""
    case = LoraCase("fused_vs_deq", 300, 520, 320, 16, 32.0, "block4", 4242)
    inp = make_case(case)
    out4 = run_layer(lib, inp)
    inp16 = dict(inp)
    inp16["W"] = O.dequant_blockwise4(inp["codes"], inp["absmax"], inp["codebook"], case.N, case.K)
    inp16["case"] = LoraCase("fused_vs_deq16", 300, 520, 320, 16, 32.0, "bf16", 4242)
    out16 = run_layer(lib, inp16)
    for k in ("Y", "dX", "dA", "dB", "XA"):
        assert torch.equal(out4[k].view(torch.int16), out16[k].view(torch.int16)), k


def test_b_zero_and_w_zero(lib):
    case = LoraCase("special", 200, 264, 128, 16, 32.0, "bf16", 555)
    inp = make_case(case)
    inp["B"] = np.zeros_like(inp["B"])
    out = run_layer(lib, inp)
    _full_check(inp, out)
    assert not torch.any(out["dA"].float() != 0)  # dA = s·(dY·B)ᵀ·X vanishes exactly
    inp = make_case(case)
    inp["W"] = np.zeros_like(inp["W"])
    _full_check(inp, run_layer(lib, inp))


def test_empty_batch(lib):
    case = LoraCase("empty", 0, 264, 128, 16, 32.0, "bf16", 556)
    inp = make_case(case, want=("W", "A", "B"))
    W, keep = make_weight(lib, inp)
    A, B = dev_bf16(inp["A"]), dev_bf16(inp["B"])
    layer = lib.LoraLinear(W, A, B, case.alpha)
    X = torch.empty((0, case.K), dtype=torch.bfloat16, device="cuda")
    Y, XA = layer.forward(X)
    assert Y.shape == (0, case.N) and XA.shape == (0, case.r)
    dA = torch.full((case.r, case.K), 7.0, dtype=torch.bfloat16, device="cuda")
    dB = torch.full((case.N, case.r), 7.0, dtype=torch.bfloat16, device="cuda")
    dY = torch.empty((0, case.N), dtype=torch.bfloat16, device="cuda")
    layer.backward(dY, X, XA, need_dX=True, out=(torch.empty((0, case.K), dtype=torch.bfloat16, device="cuda"), dA, dB))
    torch.cuda.synchronize()
    assert not torch.any(dA.float() != 0) and not torch.any(dB.float() != 0)


def test_backward_without_dX(lib):
    case = LoraCase("nodx", 300, 264, 200, 16, 32.0, "bf16", 557)
    inp = make_case(case)
    _full_check(inp, run_layer(lib, inp, need_dX=False), need_dX=False)


def test_deterministic(lib):
    case = LoraCase("det", 1000, 1032, 1096, 40, 80.0, "bf16", 558)
    inp = make_case(case)
    a = run_layer(lib, inp)
    b = run_layer(lib, inp)
    for k in ("Y", "XA", "dX", "dA", "dB"):
        assert torch.equal(a[k].view(torch.int16), b[k].view(torch.int16)), k


def test_bounded_wait_reports_timeout_and_context_survives(lib):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert lib.lora_device_status(ws) == lib.LORA_OK
    assert lib.lora_testing_bounded_wait(ws, 20_000_000) == lib.LORA_OK  # 20 ms
    torch.cuda.synchronize()
    assert lib.lora_device_status(ws) == lib.LORA_ERR_DEVICE_TIMEOUT
    assert lib.lora_device_status(ws) == lib.LORA_OK  # read-and-clear
    # the context is still usable
    case = LoraCase("after_timeout", 64, 256, 64, 8, 16.0, "bf16", 559)
    inp = make_case(case)
    _full_check(inp, run_layer(lib, inp))
