"""GPU parity of the SwiGLU feed-forward block (LoRA on gate, up and down) against the
oracle's chain-rule forward/backward, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import MlpCase, make_mlp_case
from tests.gpu_helpers import check, dev_bf16, host_f64, make_weight

pytestmark = pytest.mark.gpu

# G, U, H, dG, dU are stored in bf16 and computed from bf16 G and U: per element the bar
# also allows one bf16 rounding (2^-8 relative) for each of G, U and the stored result.
REL_SWIGLU = 3 * 2.0 ** -8
SWIGLU_KEYS = ("G", "U", "H", "dG", "dU")


def _check(k, got, ref):
    check(k, got, ref, rel_elem=REL_SWIGLU if k in SWIGLU_KEYS else 0.0)


def _oracle_weights(inp):
    return (O.weight_f64(inp["gate_up"]), O.bf16_to_f64(inp["A_gu"]), O.bf16_to_f64(inp["B_gu"]),
            O.weight_f64(inp["down"]), O.bf16_to_f64(inp["A_d"]), O.bf16_to_f64(inp["B_d"]))


def _run(q, inp):
    case = inp["case"]
    Wgu, keep1 = make_weight(q, inp["gate_up"])
    Wd, keep2 = make_weight(q, inp["down"])
    X, Agu, Bgu, Ad, Bd, dZ = (dev_bf16(inp[k]) for k in ("X", "A_gu", "B_gu", "A_d", "B_d", "dZ"))
    mlp = q.LoraMLP(Wgu, Wd, Agu, Bgu, Ad, Bd, case.alpha)
    Z, saved = mlp.forward(X)
    torch.cuda.synchronize()
    fwd = {"Z": Z.clone(), "G": saved["GU"][:, :case.I].clone(), "U": saved["GU"][:, case.I:].clone(),
           "H": saved["H"].clone(), "XA_gu": saved["XA_gate_up"].clone(), "XA_d": saved["XA_down"].clone()}
    dX, dAgu, dBgu, dAd, dBd = mlp.backward(dZ, X, saved)
    torch.cuda.synchronize()
    assert q.lora_device_status(mlp.workspace(case.M)) == q.LORA_OK
    bwd = {"dX": dX, "dA_gu": dAgu, "dB_gu": dBgu, "dA_d": dAd, "dB_d": dBd,
           "dG": saved["GU"][:, :case.I], "dU": saved["GU"][:, case.I:]}
    return fwd, bwd, (keep1, keep2, mlp, X, dZ)


SMALL = [
    # M, D, I, r, fmt
    (300, 200, 264, 16, "bf16"),
    (129, 136, 520, 8, "bf16"),
    (257, 328, 384, 40, "bf16"),
    (300, 192, 256, 16, "block4"),
    (64, 256, 448, 64, "block4"),
    (17, 64, 8, 8, "bf16"),
]


@pytest.mark.parametrize("M,D,I,r,fmt", SMALL)
def test_mlp_small(lib, M, D, I, r, fmt):  # noqa: E741
    case = MlpCase(f"mlp_{M}_{D}_{I}_{r}_{fmt}", M, D, I, r, 2.0 * r, fmt, 6000 + M + D + I + r)
    inp = make_mlp_case(case)
    fwd, bwd, _ = _run(lib, inp)
    Wgu, Agu, Bgu, Wd, Ad, Bd = _oracle_weights(inp)
    X, dZ = O.bf16_to_f64(inp["X"]), O.bf16_to_f64(inp["dZ"])
    g = O.lora_mlp_backward(dZ, X, Wgu, Agu, Bgu, Wd, Ad, Bd, case.s)
    f = g["fwd"]
    for k in ("Z", "G", "U", "H", "XA_gu", "XA_d"):
        _check(k, host_f64(fwd[k]), f[k])
    for k in ("dX", "dA_gu", "dB_gu", "dA_d", "dB_d", "dG", "dU"):
        _check(k, host_f64(bwd[k]), g[k])


def test_mlp_no_dX_and_empty_batch(lib):
    case = MlpCase("mlp_nodx", 96, 128, 256, 16, 32.0, "bf16", 6100)
    inp = make_mlp_case(case)
    Wgu, keep1 = make_weight(lib, inp["gate_up"])
    Wd, keep2 = make_weight(lib, inp["down"])
    X, Agu, Bgu, Ad, Bd, dZ = (dev_bf16(inp[k]) for k in ("X", "A_gu", "B_gu", "A_d", "B_d", "dZ"))
    mlp = lib.LoraMLP(Wgu, Wd, Agu, Bgu, Ad, Bd, case.alpha)
    Z, saved = mlp.forward(X)
    ref = {k: v.clone() for k, v in saved.items()}
    out_a = mlp.backward(dZ, X, saved, need_dX=False)
    saved2 = {k: v.clone() for k, v in ref.items()}
    out_b = mlp.backward(dZ, X, saved2, need_dX=True)
    torch.cuda.synchronize()
    assert out_a[0] is None
    for a, b in zip(out_a[1:], out_b[1:]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))   # same bits without dX
    # empty batch: adapter gradients are zero
    E = torch.empty((0, case.D), dtype=torch.bfloat16, device="cuda")
    Z0, s0 = mlp.forward(E)
    grads = mlp.backward(torch.empty((0, case.D), dtype=torch.bfloat16, device="cuda"), E, s0)
    torch.cuda.synchronize()
    for t in grads[1:]:
        assert t.numel() > 0 and not torch.any(t.float() != 0)


def test_mlp_deterministic(lib):
    case = MlpCase("mlp_det", 513, 256, 512, 16, 32.0, "bf16", 6200)
    inp = make_mlp_case(case)
    a_f, a_b, _ = _run(lib, inp)
    b_f, b_b, _ = _run(lib, inp)
    for d1, d2 in ((a_f, b_f), (a_b, b_b)):
        for k in d1:
            assert torch.equal(d1[k].view(torch.int16), d2[k].view(torch.int16)), k


@pytest.mark.slow
def test_mlp_mid_size_adapter_gradients(lib):
    """Several tiles in every direction with a ragged token count; every output whole."""
    case = MlpCase("mlp_mid", 1500, 1024, 2048, 16, 32.0, "bf16", 6300)
    inp = make_mlp_case(case)
    fwd, bwd, _ = _run(lib, inp)
    Wgu, Agu, Bgu, Wd, Ad, Bd = _oracle_weights(inp)
    X, dZ = O.bf16_to_f64(inp["X"]), O.bf16_to_f64(inp["dZ"])
    g = O.lora_mlp_backward(dZ, X, Wgu, Agu, Bgu, Wd, Ad, Bd, case.s)
    for k in ("Z", "H", "G", "U"):
        _check(k, host_f64(fwd[k]), g["fwd"][k])
    for k in ("dX", "dA_gu", "dB_gu", "dA_d", "dB_d", "dG", "dU"):
        _check(k, host_f64(bwd[k]), g[k])


@pytest.mark.slow
@pytest.mark.parametrize("fmt", ["bf16", "block4"])
def test_mlp_llama8b_rows(lib, fmt):
    """Llama-8B feed-forward (D = 4096, I = 14336, r = 16) at M = 4096 tokens: every output
    that depends on single tokens (Z, G, U, H, dG, dU, dX) checked on sampled tokens."""
    case = MlpCase(f"mlp_llama8b_{fmt}", 4096, 4096, 14336, 16, 32.0, fmt, 6400 + (fmt == "block4"))
    inp = make_mlp_case(case)
    fwd, bwd, _ = _run(lib, inp)
    Wgu, Agu, Bgu, Wd, Ad, Bd = _oracle_weights(inp)
    rng = np.random.default_rng(11)
    ridx = np.unique(np.concatenate([[0, case.M - 1], rng.choice(case.M, 24, replace=False)]))
    X, dZ = O.bf16_to_f64(inp["X"][ridx]), O.bf16_to_f64(inp["dZ"][ridx])
    g = O.lora_mlp_backward(dZ, X, Wgu, Agu, Bgu, Wd, Ad, Bd, case.s)
    t = torch.from_numpy(ridx).cuda()
    for k in ("Z", "H", "G", "U"):
        _check(k, host_f64(fwd[k].index_select(0, t)), g["fwd"][k])
    for k in ("dX", "dG", "dU"):
        _check(k, host_f64(bwd[k].index_select(0, t)), g[k])
