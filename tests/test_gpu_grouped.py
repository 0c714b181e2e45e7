"""GPU parity of grouped projections sharing X (fused q/k/v) against the oracle's
grouped forward/backward, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import LoraCase, make_grouped_case
from tests.gpu_helpers import check, dev_bf16, dev_f16_bits, dev_u8, host_f64

pytestmark = pytest.mark.gpu


def _run(lib, inp, case):
    rows = inp["rows"]
    if case.fmt == "bf16":
        W = lib.LoraWeight(case.N, case.K, dev_bf16(inp["W"]))
    else:
        W = lib.LoraWeight(case.N, case.K, dev_u8(inp["codes"]), dev_f16_bits(inp["absmax"]),
                           torch.from_numpy(inp["codebook"]).cuda())
    X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    layer = lib.LoraGroupedLinear(W, rows, A, B, case.alpha)
    Y, XA = layer.forward(X)
    dX, dA, dB = layer.backward(dY, X, XA)
    torch.cuda.synchronize()
    assert lib.lora_device_status(layer.workspace(case.M)) == lib.LORA_OK
    return {"Y": Y, "XA": XA, "dX": dX, "dA": dA, "dB": dB, "W": W}


def _split(inp, case):
    rows = inp["rows"]
    Wall = O.weight_f64(inp)
    Aall, Ball = O.bf16_to_f64(inp["A"]), O.bf16_to_f64(inp["B"])
    offs = np.cumsum([0] + rows)
    Ws = [Wall[offs[g]:offs[g + 1]] for g in range(len(rows))]
    As = [Aall[g * case.r:(g + 1) * case.r] for g in range(len(rows))]
    Bs = [Ball[offs[g]:offs[g + 1]] for g in range(len(rows))]
    return Ws, As, Bs


GROUPS = [
    # M, rows, K, r, fmt
    (300, [512, 256, 264], 200, 16, "bf16"),
    (257, [256, 256], 328, 24, "bf16"),
    (129, [768, 256, 256, 256], 136, 8, "bf16"),
    (300, [512, 256, 256], 192, 32, "block4"),
    (64, [256, 8], 64, 40, "bf16"),
    # large enough for the one-pass dY·B / dYᵀ·XA kernel on every segment, the last ragged
    (3000, [1024, 512, 776], 136, 8, "bf16"),
]


@pytest.mark.parametrize("M,rows,K,r,fmt", GROUPS)
def test_grouped_small(lib, M, rows, K, r, fmt):
    case = LoraCase(f"grouped_{M}_{len(rows)}_{r}_{fmt}", M, sum(rows), K, r, 2.0 * r, fmt, 5000 + M + K + r)
    inp = make_grouped_case(case, rows)
    out = _run(lib, inp, case)
    Ws, As, Bs = _split(inp, case)
    X, dY = O.bf16_to_f64(inp["X"]), O.bf16_to_f64(inp["dY"])
    Y, XA = O.lora_grouped_forward(X, Ws, As, Bs, case.s)
    g = O.lora_grouped_backward(dY, X, Ws, As, Bs, case.s)
    check("Y", host_f64(out["Y"]), Y)
    check("XA", host_f64(out["XA"]), XA)
    check("dX", host_f64(out["dX"]), g["dX"])
    check("dA", host_f64(out["dA"]), g["dA"])
    check("dB", host_f64(out["dB"]), g["dB"])


def test_single_projection_group_matches_plain_layer(lib):
    """G = 1 through the grouped entry points gives the plain layer's bits."""
    case = LoraCase("g1", 300, 520, 200, 16, 32.0, "bf16", 5100)
    inp = make_grouped_case(case, [520])
    out = _run(lib, inp, case)
    W = out["W"]
    X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
    layer = lib.LoraLinear(W, A, B, case.alpha)
    Y, XA = layer.forward(X)
    dX, dA, dB = layer.backward(dY, X, XA)
    torch.cuda.synchronize()
    for k, v in (("Y", Y), ("XA", XA), ("dX", dX), ("dA", dA), ("dB", dB)):
        assert torch.equal(out[k].view(torch.int16), v.view(torch.int16)), k


@pytest.mark.slow
@pytest.mark.parametrize("fmt", ["bf16", "block4"])
def test_llama8b_qkv_full_size(lib, fmt):
    """Llama-8B attention q/k/v (grouped-query: q 4096, k 1024, v 1024 rows) at
    M = 8192 tokens, K = 4096, r = 16: sampled rows/columns against the oracle."""
    rows = [4096, 1024, 1024]
    case = LoraCase(f"qkv_{fmt}", 8192, sum(rows), 4096, 16, 32.0, fmt, 5200 + (fmt == "block4"))
    inp = make_grouped_case(case, rows)
    out = _run(lib, inp, case)
    Ws, As, Bs = _split(inp, case)
    rng = np.random.default_rng(7)
    ridx = np.unique(np.concatenate([[0, case.M - 1], rng.choice(case.M, 40, replace=False)]))
    X = O.bf16_to_f64(inp["X"][ridx])
    dY = O.bf16_to_f64(inp["dY"][ridx])
    Y, XA = O.lora_grouped_forward(X, Ws, As, Bs, case.s)
    # dX rows depend only on the same rows of dY; dA, dB sum over every token, so
    # they are checked on sampled rows/columns, accumulated over the tokens in chunks
    g_rows = O.lora_grouped_backward(dY, X, Ws, As, Bs, case.s)
    t = torch.from_numpy(ridx).cuda()
    check("Y", host_f64(out["Y"].index_select(0, t)), Y)
    check("XA", host_f64(out["XA"].index_select(0, t)), XA)
    check("dX", host_f64(out["dX"].index_select(0, t)), g_rows["dX"])
    k_idx = np.unique(np.concatenate([[0, case.K - 1], rng.choice(case.K, 48, replace=False)]))
    dA_dev = host_f64(out["dA"])
    dB_dev = host_f64(out["dB"])
    off = 0
    for g, n in enumerate(rows):
        n_idx = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 48, replace=False)]))
        dB_ref, dA_ref = O.lora_adapter_grads_sampled(inp["dY"][:, off:off + n], inp["X"], As[g], Bs[g], case.s,
                                                      n_idx, k_idx)
        check(f"dB[{g}]", dB_dev[off + n_idx], dB_ref)
        check(f"dA[{g}]", dA_dev[g * case.r:(g + 1) * case.r][:, k_idx], dA_ref)
        off += n
