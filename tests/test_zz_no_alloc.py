"""The forward entry point that allocates nothing (lora_linear_fwd_noalloc).

Some callers are handed only their input and output buffers and may not obtain any
other device memory (a plugin inside a framework that owns all device memory through
its pool allocator, or latency-critical code that must not call cudaMalloc/cudaFree,
which can synchronize the device and can fail under a fixed budget).  For them the
library keeps the forward's scratch in a fixed array of its own.  These tests call
that entry point through the C ABI and compare it with the ordinary forward.

This file is collected last on purpose, so that a run stopping at its first failure
has already run every other test.
"""
import ctypes

import pytest
import torch

from synth import LoraCase, make_case
from tests.gpu_helpers import check, dev_bf16, host_f64, make_weight


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # validation happens on the host before any device work: fake aligned addresses suffice
    import qlora_linear_b200 as q
    from qlora_linear_b200.binding import lora_weight_t
    P = 0x10000
    W = lora_weight_t(0, 0, 4096, 4096, P, P, P)
    fn = q.lib().lora_linear_fwd_noalloc
    assert fn(P, 30000, ctypes.byref(W), P, P, 128, 2.0, P, P, None) == q.LORA_ERR_SCRATCH_LIMIT
    assert fn(P, 400000, ctypes.byref(W), P, P, 16, 2.0, P, P, None) == q.LORA_ERR_SCRATCH_LIMIT
    assert fn(P, 256, ctypes.byref(W), P, P, 12, 2.0, P, P, None) == q.LORA_ERR_UNSUPPORTED
    assert fn(P, 256, None, P, P, 16, 2.0, P, P, None) == q.LORA_ERR_INVALID_ARG
    assert fn(0, 0, ctypes.byref(W), P, P, 16, 2.0, 0, 0, None) == q.LORA_OK  # empty batch
    assert "scratch" in q.status_string(q.LORA_ERR_SCRATCH_LIMIT)


def _forward_both_ways(q, case):
    inp = make_case(case, want=("X", "W", "A", "B"))
    W, keep = make_weight(q, inp)
    X, A, B = dev_bf16(inp["X"]), dev_bf16(inp["A"]), dev_bf16(inp["B"])
    M, N, r = case.M, case.N, case.r
    Y0 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    XA0 = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    ws = q.alloc_workspace(M, N, case.K, r, W.fmt)
    q.lora_linear_fwd(X, M, W, A, B, r, case.s, Y0, XA0, ws)
    Y1 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    XA1 = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device="cuda")
    w = W.c_struct()
    st = q.lib().lora_linear_fwd_noalloc(X.data_ptr(), M, ctypes.byref(w), A.data_ptr(), B.data_ptr(), r,
                                         ctypes.c_float(case.s), Y1.data_ptr(), XA1.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == q.LORA_OK, q.status_string(st)
    torch.cuda.synchronize()
    return (Y0, XA0), (Y1, XA1)


@pytest.mark.gpu
def test_noalloc_forward_matches_forward_on_consecutive_calls(lib):
    cases = [
        LoraCase("noalloc_a", 1000, 1032, 1096, 40, 80.0, "bf16", 9001),
        LoraCase("noalloc_b", 300, 520, 192, 16, 32.0, "block4", 9002),
        LoraCase("noalloc_a_again", 1000, 1032, 1096, 40, 80.0, "bf16", 9001),
    ]
    first = None
    for case in cases:
        (Y0, XA0), (Y1, XA1) = _forward_both_ways(lib, case)
        check(f"{case.name} Y", host_f64(Y1), host_f64(Y0))
        check(f"{case.name} XA", host_f64(XA1), host_f64(XA0))
        if first is None:
            first = Y1
        elif case.name == "noalloc_a_again":
            # the scratch left behind by the previous call does not leak into this one
            assert torch.equal(Y1.view(torch.int16), first.view(torch.int16))
