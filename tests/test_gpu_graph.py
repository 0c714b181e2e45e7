"""The layer's forward and backward captured once into a CUDA graph and replayed: after the
first call on the device (kernel attributes, driver entry point), the entry points only
enqueue work on the caller's stream, so a capture records the whole step.  A replay on new
data written into the captured input buffers must give the bits an ordinary call gives on
the same data.  Shapes that take the stream-K schedule and the TMA-fed passes over X."""
import numpy as np
import pytest
import torch

from synth import LoraCase, make_case
from tests.gpu_helpers import dev_bf16, host_bits, make_weight

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["bf16", "block4"])
def test_layer_step_replays_from_a_cuda_graph(lib, fmt):
    M, N, K, r = 512, 4096, 8192, 16
    F = {"bf16": 0, "block4": 1}[fmt]
    assert lib.lora_testing_gemm_streamk(M, N, K, r, F) > 0 or lib.lora_testing_gemm_streamk(M, K, N, r, F) > 0
    assert lib.lora_testing_xpass_tma(M, K, r) & 1
    case = LoraCase(f"graph_{fmt}", M, N, K, r, 2.0 * r, fmt, 7900)
    inp = make_case(case)
    W, keep = make_weight(lib, inp)
    A, B = dev_bf16(inp["A"]), dev_bf16(inp["B"])
    layer = lib.LoraLinear(W, A, B, case.alpha)
    X, dY = dev_bf16(inp["X"]), dev_bf16(inp["dY"])
    # second data set for the replay
    g2 = torch.Generator(device="cuda")
    g2.manual_seed(11)
    X2 = torch.randn(X.shape, generator=g2, device="cuda").to(torch.bfloat16)
    dY2 = torch.randn(dY.shape, generator=g2, device="cuda").to(torch.bfloat16)

    # ordinary calls on the second data set (the first calls also initialise the device)
    Ye, XAe = layer.forward(X2)
    dXe, dAe, dBe = layer.backward(dY2, X2, XAe)
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer.forward(X)  # a call on the capture stream before capturing
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        Y, XA = layer.forward(X)
        dX, dA, dB = layer.backward(dY, X, XA)
    X.copy_(X2)
    dY.copy_(dY2)
    graph.replay()
    torch.cuda.synchronize()
    assert lib.lora_device_status(layer.workspace(M)) == lib.LORA_OK
    for name, got, want in (("Y", Y, Ye), ("XA", XA, XAe), ("dX", dX, dXe), ("dA", dA, dAe), ("dB", dB, dBe)):
        assert np.array_equal(host_bits(got), host_bits(want)), name
    # a second replay after changing the inputs again follows them
    X.copy_(dev_bf16(inp["X"]))
    dY.copy_(dev_bf16(inp["dY"]))
    graph.replay()
    Yo, XAo = layer.forward(dev_bf16(inp["X"]))
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(Y), host_bits(Yo))
    del graph
