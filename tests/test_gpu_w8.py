"""GPU parity of the 8-bit frozen weights (int8 and fp8 e4m3 codes with fp32 row
scales): standalone dequantization bit for bit, the layer, the feed-forward block and
the merge against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import LoraCase, MlpCase, make_case, make_mlp_case
from tests.gpu_helpers import check, dev_bf16, dev_u8, host_bits, host_f64, make_weight, run_layer

pytestmark = pytest.mark.gpu
FMTS = ["int8", "fp8"]


def _fmt(lib, fmt):
    return lib.LORA_W_INT8 if fmt == "int8" else lib.LORA_W_FP8_E4M3


@pytest.mark.parametrize("fmt", FMTS)
def test_dequant8_every_code_bit_exact(lib, fmt):
    """Each of 256 rows holds every byte value (shifted per row), with its own scale."""
    N, K = 256, 512
    base = np.arange(K, dtype=np.int64)
    codes = ((base[None, :] + 37 * np.arange(N)[:, None]) % 256).astype(np.uint8)
    rng = np.random.default_rng(3)
    scale = (rng.random(N) * 0.05 + 1e-3).astype(np.float32)
    scale[5] = 0.0
    W = lib.LoraWeight(N, K, dev_u8(codes), torch.from_numpy(scale).cuda(), None, _fmt(lib, fmt))
    out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    lib.lora_dequant(W, out)
    torch.cuda.synchronize()
    # the fp8 NaN codes (0x7F, 0xFF) lie outside the oracle's domain: compare every other
    # element bit for bit and check that those two give NaN
    nan_code = ((codes & 0x7F) == 0x7F) if fmt == "fp8" else np.zeros_like(codes, dtype=bool)
    ref = O.dequant_rowwise8(np.where(nan_code, 0, codes).astype(np.uint8), scale, fmt)
    got = host_bits(out)
    assert np.array_equal(got[~nan_code], ref[~nan_code])
    assert np.all(np.isnan(O.bf16_to_f64(got[nan_code])))
    assert nan_code.sum() == (2 * N * K // 256 if fmt == "fp8" else 0)


RAGGED = [
    # M, N, K, r
    (300, 520, 208, 16),
    (129, 264, 144, 72),
    (257, 776, 320, 128),
    (1, 8, 16, 8),
    (7, 16, 80, 40),
]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K,r", RAGGED)
def test_w8_layer_ragged(lib, fmt, M, N, K, r):
    case = LoraCase(f"w8_{fmt}_{M}_{N}_{K}_{r}", M, N, K, r, 2.0 * r, fmt, 8000 + M + N + K + r)
    inp = make_case(case)
    out = run_layer(lib, inp)
    W = O.weight_f64(inp)
    X, A, B, dY = (O.bf16_to_f64(inp[k]) for k in ("X", "A", "B", "dY"))
    Y, XA = O.lora_forward(X, W, A, B, case.s)
    g = O.lora_backward(dY, X, W, A, B, case.s)
    check("Y", host_f64(out["Y"]), Y)
    check("XA", host_f64(out["XA"]), XA)
    for k in ("dX", "dA", "dB"):
        check(k, host_f64(out[k]), g[k])


@pytest.mark.parametrize("fmt", FMTS)
def test_w8_layer_equals_bf16_layer_of_its_dequantized_weight(lib, fmt):
    """The GEMM expands the same bf16 values the standalone dequantization writes, into
    the same tiles, so the 8-bit layer and the bf16 layer on lora_dequant(W) agree bit
    for bit."""
    case = LoraCase(f"w8eq_{fmt}", 513, 776, 528, 16, 32.0, fmt, 8100)
    inp = make_case(case)
    out8 = run_layer(lib, inp)
    Wq = out8["layer"].W
    Wbf = torch.empty((case.N, case.K), dtype=torch.bfloat16, device="cuda")
    lib.lora_dequant(Wq, Wbf)
    layer = lib.LoraLinear(lib.LoraWeight(case.N, case.K, Wbf), out8["layer"].A, out8["layer"].B, case.alpha)
    Y, XA = layer.forward(out8["X"])
    dX, dA, dB = layer.backward(out8["dY"], out8["X"], XA)
    torch.cuda.synchronize()
    for k, v in (("Y", Y), ("XA", XA), ("dX", dX), ("dA", dA), ("dB", dB)):
        assert torch.equal(out8[k].view(torch.int16), v.view(torch.int16)), k


@pytest.mark.parametrize("fmt", FMTS)
def test_w8_merge(lib, fmt):
    N, K, r = 264, 208, 24
    case = LoraCase(f"merge8_{fmt}", 1, N, K, r, 3.0 * r, fmt, 8200)
    inp = make_case(case, want=("W", "A", "B"))
    W, keep = make_weight(lib, inp)
    A, B = dev_bf16(inp["A"]), dev_bf16(inp["B"])
    out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    lib.lora_merge(W, A, B, r, case.s, out)
    torch.cuda.synchronize()
    ref = O.lora_merge(O.weight_f64(inp), O.bf16_to_f64(inp["A"]), O.bf16_to_f64(inp["B"]), case.s)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(host_f64(out) - ref) <= ulp)
    lib.lora_merge(W, A, torch.zeros_like(B), r, case.s, out)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(out), O.dequant_rowwise8(inp["codes"], inp["row_scale"], fmt))


@pytest.mark.parametrize("fmt", FMTS)
def test_w8_mlp_block(lib, fmt):
    from tests.test_gpu_mlp import REL_SWIGLU, SWIGLU_KEYS, _oracle_weights, _run
    case = MlpCase(f"mlp8_{fmt}", 200, 256, 384, 16, 32.0, fmt, 8300)
    inp = make_mlp_case(case)
    fwd, bwd, _ = _run(lib, inp)
    Wgu, Agu, Bgu, Wd, Ad, Bd = _oracle_weights(inp)
    g = O.lora_mlp_backward(O.bf16_to_f64(inp["dZ"]), O.bf16_to_f64(inp["X"]), Wgu, Agu, Bgu, Wd, Ad, Bd, case.s)
    for k in ("Z", "G", "U", "H"):
        check(k, host_f64(fwd[k]), g["fwd"][k], rel_elem=REL_SWIGLU if k in SWIGLU_KEYS else 0.0)
    for k in ("dX", "dA_gu", "dB_gu", "dA_d", "dB_d", "dG", "dU"):
        check(k, host_f64(bwd[k]), g[k], rel_elem=REL_SWIGLU if k in SWIGLU_KEYS else 0.0)


@pytest.mark.slow
@pytest.mark.parametrize("fmt", FMTS)
def test_w8_full_size(lib, fmt):
    """The 4096 -> 14336 projection at M = 8192 with an 8-bit weight: sampled outputs."""
    case = LoraCase(f"w8full_{fmt}", 8192, 14336, 4096, 16, 32.0, fmt, 8400 + (fmt == "fp8"))
    inp = make_case(case)
    out = run_layer(lib, inp)
    rng = np.random.default_rng(case.seed)

    def sample(n):
        return np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=46, replace=False)]))

    rows, n_idx, k_idx = sample(case.M), sample(case.N), sample(case.K)
    W = O.weight_f64(inp)
    A, B = O.bf16_to_f64(inp["A"]), O.bf16_to_f64(inp["B"])
    Yr, XAr = O.lora_forward_rows(O.bf16_to_f64(inp["X"][rows]), W, A, B, case.s)
    dXr = O.lora_backward_rows(O.bf16_to_f64(inp["dY"][rows]), W, A, B, case.s)
    dB_s, dA_s = O.lora_adapter_grads_sampled(inp["dY"], inp["X"], A, B, case.s, n_idx, k_idx)
    t = torch.from_numpy(rows).cuda()
    check("Y", host_f64(out["Y"].index_select(0, t)), Yr)
    check("XA", host_f64(out["XA"].index_select(0, t)), XAr)
    check("dX", host_f64(out["dX"].index_select(0, t)), dXr)
    check("dB", host_f64(out["dB"].index_select(0, torch.from_numpy(n_idx).cuda())), dB_s)
    check("dA", host_f64(out["dA"].index_select(1, torch.from_numpy(k_idx).cuda())), dA_s)


@pytest.mark.parametrize("fmt", ["bf16", "block4"])
def test_lora_dequant_other_formats(lib, fmt):
    """lora_dequant copies a bf16 weight and expands a 4-bit one exactly like
    dequant_blockwise4; an output overlapping the stored weight is refused."""
    case = LoraCase(f"dq_{fmt}", 1, 264, 320, 8, 16.0, fmt, 8500)
    inp = make_case(case, want=("W",))
    W, keep = make_weight(lib, inp)
    out = torch.empty((case.N, case.K), dtype=torch.bfloat16, device="cuda")
    lib.lora_dequant(W, out)
    torch.cuda.synchronize()
    ref = inp["W"] if fmt == "bf16" else O.dequant_blockwise4(inp["codes"], inp["absmax"], inp["codebook"], case.N,
                                                                case.K)
    assert np.array_equal(host_bits(out), ref)
    if fmt == "bf16":
        with pytest.raises(lib.LoraError):
            lib.lora_dequant(W, keep[0])
