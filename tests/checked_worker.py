"""Worker of tests/test_gpu_checked.py, run in a subprocess on the library that
LORA_LIB_PATH names (the binding loads one library per process).

    python tests/checked_worker.py all     the ragged parity shapes, a grouped and a
                                           feed-forward case, then the out-of-range tile
    python tests/checked_worker.py tile    the out-of-range tile only

Prints one JSON line: the library loaded, the cases that met the parity bar with status
LORA_OK and every output written (NaN canaries), and the status after the tile probe.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def out_of_range_tile(q, torch):
    """The tensor-core rank-r pass with one output tile past the last row."""
    rows, red, r = 300, 520, 72
    P = torch.randn((rows, red), device="cuda").to(torch.bfloat16)
    A = torch.randn((r, red), device="cuda").to(torch.bfloat16)
    splits = q.lora_testing_tcproj_splits(rows, red, r)
    part = torch.zeros(splits * rows * r, dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    st = q.lora_testing_tcproj_extra_tile(P, A, rows, red, r, part, ws)
    torch.cuda.synchronize()
    dev = q.lora_device_status(ws)
    # the real tiles of the regular build: the split partials sum to P·Aᵀ
    ref = P.float() @ A.float().T
    got = part.view(splits, rows, r).sum(0)
    err = float(((got - ref).norm() / ref.norm()).item())
    return {"launch": st, "device_status": dev, "rel_err": err}


def main(what):
    import numpy as np  # noqa: F401
    import torch

    import qlora_linear_b200 as q
    res = {"lib": os.path.basename(q.LIB_PATH)}
    if what == "all":
        import oracle as O
        from synth import LoraCase, MlpCase, make_case, make_grouped_case, make_mlp_case
        from tests.gpu_helpers import check, dev_bf16, host_f64, make_weight, nan_canary, run_layer
        from tests.test_gpu_parity import RAGGED, _full_check
        ok = []
        for (M, N, K, r, fmt) in RAGGED:
            case = LoraCase(f"checked_{M}_{N}_{K}_{r}_{fmt}", M, N, K, r, 2.0 * r + 1.0, fmt, 1000 + M + N + K + r)
            inp = make_case(case)
            _full_check(inp, run_layer(q, inp))  # status LORA_OK is asserted inside
            ok.append(case.name)
        # grouped projections (ragged last projection, G·r = 48 on the tensor-core passes)
        rows = [256, 256, 136]
        case = LoraCase("checked_grouped", 300, sum(rows), 200, 16, 32.0, "bf16", 2024)
        inp = make_grouped_case(case, rows)
        W = q.LoraWeight(case.N, case.K, dev_bf16(inp["W"]))
        X, A, B, dY = (dev_bf16(inp[k]) for k in ("X", "A", "B", "dY"))
        layer = q.LoraGroupedLinear(W, rows, A, B, case.alpha)
        Y, XA = layer.forward(X, Y=nan_canary((case.M, case.N)), XA=nan_canary((case.M, 3 * case.r)))
        dX, dA, dB = layer.backward(dY, X, XA, out=(nan_canary((case.M, case.K)), nan_canary((3 * case.r, case.K)),
                                                    nan_canary((case.N, case.r))))
        torch.cuda.synchronize()
        assert q.lora_device_status(layer.workspace(case.M)) == q.LORA_OK
        Wf = O.weight_f64(inp)
        offs = np.cumsum([0] + rows)
        Ws = [Wf[offs[g]:offs[g + 1]] for g in range(3)]
        Af, Bf = O.bf16_to_f64(inp["A"]), O.bf16_to_f64(inp["B"])
        As = [Af[g * case.r:(g + 1) * case.r] for g in range(3)]
        Bs = [Bf[offs[g]:offs[g + 1]] for g in range(3)]
        Xf, dYf = O.bf16_to_f64(inp["X"]), O.bf16_to_f64(inp["dY"])
        fwd = O.lora_grouped_forward(Xf, Ws, As, Bs, case.s)
        bwd = O.lora_grouped_backward(dYf, Xf, Ws, As, Bs, case.s)
        check("grouped Y", host_f64(Y), fwd[0])
        check("grouped dX", host_f64(dX), bwd["dX"])
        check("grouped dA", host_f64(dA), bwd["dA"])
        check("grouped dB", host_f64(dB), bwd["dB"])
        ok.append(case.name)
        # the feed-forward block, 4-bit weights, rank 40 (2r = 80 on the tensor-core passes)
        mc = MlpCase("checked_mlp", 130, 192, 256, 40, 80.0, "block4", 2025)
        mi = make_mlp_case(mc)
        Wgu, k1 = make_weight(q, mi["gate_up"])
        Wd, k2 = make_weight(q, mi["down"])
        Xm, Agu, Bgu, Ad, Bd, dZ = (dev_bf16(mi[k]) for k in ("X", "A_gu", "B_gu", "A_d", "B_d", "dZ"))
        mlp = q.LoraMLP(Wgu, Wd, Agu, Bgu, Ad, Bd, mc.alpha)
        Z, saved = mlp.forward(Xm, Z=nan_canary((mc.M, mc.D)))
        grads = mlp.backward(dZ, Xm, saved, out=(nan_canary((mc.M, mc.D)), nan_canary((2 * mc.r, mc.D)),
                                                 nan_canary((2 * mc.I, mc.r)), nan_canary((mc.r, mc.I)),
                                                 nan_canary((mc.D, mc.r))))
        torch.cuda.synchronize()
        assert q.lora_device_status(mlp.workspace(mc.M)) == q.LORA_OK
        for t in (Z,) + tuple(grads):
            assert torch.isfinite(t.float()).all()
        ok.append(mc.name)
        res["ok"] = ok
    res["tile"] = out_of_range_tile(q, torch)
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main(sys.argv[1] if len(sys.argv) > 1 else "all")
