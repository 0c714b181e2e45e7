"""The oracle still reproduces its committed golden fixtures (tests/golden/*.json),
which were written by tests/golden/make_golden.py from the oracle alone."""
import json
import os

import numpy as np
import pytest

import oracle as O
from synth import LoraCase, make_case

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("name", ["golden_bf16", "golden_block4"])
def test_oracle_reproduces_golden(name):
    with open(os.path.join(HERE, name + ".json")) as f:
        doc = json.load(f)
    case = LoraCase(**doc["case"])
    inp = make_case(case)
    W = O.weight_f64(inp)
    X, A, B, dY = (O.bf16_to_f64(inp[k]) for k in ("X", "A", "B", "dY"))
    Y, XA = O.lora_forward(X, W, A, B, case.s)
    g = O.lora_backward(dY, X, W, A, B, case.s)
    for key, val in (("Y", Y), ("XA", XA), ("dX", g["dX"]), ("dA", g["dA"]), ("dB", g["dB"])):
        want = np.array([float.fromhex(h) for h in doc[key]])
        np.testing.assert_allclose(val.reshape(-1), want, rtol=1e-12, atol=1e-12, err_msg=key)
    if case.fmt == "block4":
        bits = O.dequant_blockwise4(inp["codes"], inp["absmax"], inp["codebook"], case.N, case.K)
        assert np.array_equal(bits.reshape(-1), np.array(doc["W_bf16_bits"], dtype=np.uint16))
