"""Writes the golden fixtures in this folder.  Calls only ``oracle/`` (and the seeded
input generator in ``synth/``); no value here comes from the CUDA library.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from synth import LoraCase, make_case  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))

CASES = [
    LoraCase("golden_bf16", 4, 16, 64, 8, 16.0, "bf16", 777),
    LoraCase("golden_block4", 4, 16, 128, 8, 12.0, "block4", 778),
]


def hexlist(a):
    return [float(v).hex() for v in np.asarray(a, dtype=np.float64).reshape(-1)]


def main():
    for case in CASES:
        inp = make_case(case)
        W = O.weight_f64(inp)
        X, A, B, dY = (O.bf16_to_f64(inp[k]) for k in ("X", "A", "B", "dY"))
        Y, XA = O.lora_forward(X, W, A, B, case.s)
        g = O.lora_backward(dY, X, W, A, B, case.s)
        doc = {
            "what": "oracle outputs of the LoRA-adapted linear layer on seeded inputs",
            "source": ("forward Y = X·Wᵀ + s·(X·Aᵀ)·Bᵀ and hand-derived backward; 'Unsloth vs "
                       "PyTorch: The ONLY Video You Need to Understand the Difference', transcript "
                       "0:43-2:00; 4-bit format: 'Rev vs unsloth', fused quantized-LoRA paragraph"),
            "written_by": "tests/golden/make_golden.py (oracle only)",
            "case": {k: getattr(case, k) for k in ("name", "M", "N", "K", "r", "alpha", "fmt", "seed")},
            "Y": hexlist(Y), "XA": hexlist(XA), "dX": hexlist(g["dX"]),
            "dA": hexlist(g["dA"]), "dB": hexlist(g["dB"]),
        }
        if case.fmt == "block4":
            doc["W_bf16_bits"] = [int(v) for v in O.dequant_blockwise4(
                inp["codes"], inp["absmax"], inp["codebook"], case.N, case.K).reshape(-1)]
        with open(os.path.join(HERE, case.name + ".json"), "w") as f:
            json.dump(doc, f, indent=0)
            f.write("\n")


if __name__ == "__main__":
    main()
