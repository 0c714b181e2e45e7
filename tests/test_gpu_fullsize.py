"""GPU parity at the full sizes of every configuration (the sizes the benchmark runs),
through the same C ABI calls and launch configurations.

The oracle computes sampled outputs one by one: Y, XA and dX on sampled token rows,
dB on sampled output rows and dA on sampled input columns (each an exact sum over all
M tokens, accumulated chunk by chunk).  Each sampled set must meet the parity bar.
"""
import functools

import numpy as np
import pytest
import torch

import oracle as O
from synth import CONFIGS, make_case
from tests.gpu_helpers import check, host_f64, run_layer

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

CASES = CONFIGS["c1"] + CONFIGS["c2"] + CONFIGS["c3"] + CONFIGS["c4"]


@functools.lru_cache(maxsize=1)
def _shared_inputs(key):
    case = key[0]
    return make_case(case, want=("X", "W", "dY"))


def _inputs(case):
    # X, W and dY depend only on the data seeds and sizes (shared by the ranks of a
    # sweep shape); A and B are drawn per case
    ds = case.data_seed if case.data_seed is not None else case.seed
    xs = case.x_seed if case.x_seed is not None else ds
    shared_key = (case.__class__(name="shared", M=case.M, N=case.N, K=case.K, r=8, alpha=16.0, fmt=case.fmt,
                                 seed=ds, x_seed=xs, data_seed=ds),)
    inp = dict(_shared_inputs(shared_key))
    inp.update({k: v for k, v in make_case(case, want=("A", "B")).items() if k in ("A", "B")})
    inp["case"] = case
    return inp


def _sample(rng, n, k=46):
    idx = np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=min(k, n), replace=False)]))
    return idx


@pytest.mark.parametrize("case", CASES, ids=[c.name for c in CASES])
def test_full_size_parity(lib, case):
    inp = _inputs(case)
    out = run_layer(lib, inp)
    rng = np.random.default_rng(case.seed)
    rows = _sample(rng, case.M)
    n_idx = _sample(rng, case.N)
    k_idx = _sample(rng, case.K)
    W = O.weight_f64(inp)
    A, B = O.bf16_to_f64(inp["A"]), O.bf16_to_f64(inp["B"])
    Yr, XAr = O.lora_forward_rows(O.bf16_to_f64(inp["X"][rows]), W, A, B, case.s)
    dXr = O.lora_backward_rows(O.bf16_to_f64(inp["dY"][rows]), W, A, B, case.s)
    dB_s, dA_s = O.lora_adapter_grads_sampled(inp["dY"], inp["X"], A, B, case.s, n_idx, k_idx)
    ridx = torch.from_numpy(rows).cuda()
    check("Y", host_f64(out["Y"].index_select(0, ridx)), Yr)
    check("XA", host_f64(out["XA"].index_select(0, ridx)), XAr)
    check("dX", host_f64(out["dX"].index_select(0, ridx)), dXr)
    check("dB", host_f64(out["dB"].index_select(0, torch.from_numpy(n_idx).cuda())), dB_s)
    check("dA", host_f64(out["dA"].index_select(1, torch.from_numpy(k_idx).cuda())), dA_s)
    del out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("fmt", ["bf16", "block4"])
def test_large_token_count(lib, fmt):
    """2^17 tokens through a 1024 x 1024 projection: row offsets, tile counts and the split
    partials of the token reductions at a size far past the configurations."""
    from synth import LoraCase
    case = LoraCase(f"large_M_{fmt}", 131072, 1024, 1024, 16, 32.0, fmt, 4242 + (fmt == "block4"))
    inp = make_case(case)
    out = run_layer(lib, inp)
    rng = np.random.default_rng(case.seed)
    rows = _sample(rng, case.M)
    n_idx = _sample(rng, case.N)
    k_idx = _sample(rng, case.K)
    W = O.weight_f64(inp)
    A, B = O.bf16_to_f64(inp["A"]), O.bf16_to_f64(inp["B"])
    Yr, XAr = O.lora_forward_rows(O.bf16_to_f64(inp["X"][rows]), W, A, B, case.s)
    dXr = O.lora_backward_rows(O.bf16_to_f64(inp["dY"][rows]), W, A, B, case.s)
    dB_s, dA_s = O.lora_adapter_grads_sampled(inp["dY"], inp["X"], A, B, case.s, n_idx, k_idx)
    ridx = torch.from_numpy(rows).cuda()
    check("Y", host_f64(out["Y"].index_select(0, ridx)), Yr)
    check("XA", host_f64(out["XA"].index_select(0, ridx)), XAr)
    check("dX", host_f64(out["dX"].index_select(0, ridx)), dXr)
    check("dB", host_f64(out["dB"].index_select(0, torch.from_numpy(n_idx).cuda())), dB_s)
    check("dA", host_f64(out["dA"].index_select(1, torch.from_numpy(k_idx).cuda())), dA_s)
