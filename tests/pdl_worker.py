"""Worker of tests/test_gpu_pdl.py, run in a subprocess (the library reads LORA_PDL once
per process): forward and backward of a few layer shapes and one feed-forward block,
printing one JSON line with a SHA-256 of every output's bits per case and whether the
layer kernels were launched with programmatic dependent launch."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

CASES = [
    # M, N, K, r, fmt: stream-K pieces, both kernels, every weight format, rank passes on
    # both kinds of kernel (r <= 16 TMA passes, r > 16 tensor-core passes)
    (300, 2048, 8192, 32, "bf16"),
    (1000, 768, 320, 8, "bf16"),
    (300, 2048, 8256, 16, "block4"),
    (1100, 6400, 2048, 16, "block4"),
    (200, 2048, 8192, 16, "int8"),
    (513, 1024, 8192, 64, "fp8"),
]


def main():
    import torch

    import qlora_linear_b200 as q
    from synth import LoraCase, MlpCase, make_case, make_mlp_case
    from tests.gpu_helpers import dev_bf16, host_bits, make_weight, run_layer

    def digest(tensors):
        h = hashlib.sha256()
        for t in tensors:
            h.update(host_bits(t).tobytes())
        return h.hexdigest()

    res = {"pdl": os.environ.get("LORA_PDL", "1") != "0", "cases": {}}
    for (M, N, K, r, fmt) in CASES:
        case = LoraCase(f"pdl_{M}_{N}_{K}_{r}_{fmt}", M, N, K, r, 2.0 * r, fmt, 9100 + M + N + K + r)
        out = run_layer(q, make_case(case))  # asserts status LORA_OK
        res["cases"][case.name] = digest([out[k] for k in ("Y", "XA", "dX", "dA", "dB")])
    case = MlpCase("pdl_mlp", 200, 192, 256, 16, 32.0, "block4", 9300)
    inp = make_mlp_case(case)
    Wgu, k1 = make_weight(q, inp["gate_up"])
    Wd, k2 = make_weight(q, inp["down"])
    X, Agu, Bgu, Ad, Bd, dZ = (dev_bf16(inp[k]) for k in ("X", "A_gu", "B_gu", "A_d", "B_d", "dZ"))
    mlp = q.LoraMLP(Wgu, Wd, Agu, Bgu, Ad, Bd, case.alpha)
    Z, saved = mlp.forward(X)
    grads = mlp.backward(dZ, X, saved)
    torch.cuda.synchronize()
    assert q.lora_device_status(mlp.workspace(case.M)) == q.LORA_OK
    res["cases"][case.name] = digest([Z, *grads])
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
