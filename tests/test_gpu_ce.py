"""GPU parity of the cross-entropy over an LM head (no [M, V] logits) against the
oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import CeCase, make_ce_case
from tests.gpu_helpers import check, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

# loss and lse are fp32 sums of exactly represented bf16 products and of exponentials
# (relative error ~1e-6); 1e-3 absolute is far above that and far below any formula slip
LOSS_ATOL = 1e-3


def _run(lib, inp, slice_=0, ws_bytes=None):
    case = inp["case"]
    W = lib.LoraWeight(case.V, case.D, dev_bf16(inp["W"]))
    X = dev_bf16(inp["X"])
    labels = torch.from_numpy(inp["labels"]).cuda()
    dloss = torch.from_numpy(inp["dloss"]).cuda()
    ce = lib.LoraCrossEntropy(W, case.ignore_index, slice_)
    if ws_bytes is not None:
        ce._ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
        ce._ws_M = case.M
    loss, lse = ce.forward(X, labels)
    dX = ce.backward(X, labels, lse, dloss)
    torch.cuda.synchronize()
    assert lib.lora_device_status(ce.workspace(case.M)) == lib.LORA_OK
    return loss, lse, dX


def _compare(case, inp, loss, lse, dX, rows=None):
    if rows is None:
        ref = O.cross_entropy(O.bf16_to_f64(inp["X"]), O.bf16_to_f64(inp["W"]), inp["labels"], case.ignore_index,
                              inp["dloss"])
        sel = slice(None)
    else:
        ref = O.cross_entropy_rows_bits(inp["X"][rows], inp["W"], inp["labels"][rows], case.ignore_index,
                                        inp["dloss"][rows])
        sel = torch.from_numpy(rows).cuda()
    got_loss = loss[sel].double().cpu().numpy()
    got_lse = lse[sel].double().cpu().numpy()
    assert np.max(np.abs(got_loss - ref[0])) <= LOSS_ATOL
    assert np.max(np.abs(got_lse - ref[1])) <= LOSS_ATOL
    got_dX = host_f64(dX[sel] if rows is None else dX.index_select(0, sel))
    check("dX", got_dX, ref[2])
    ign = (inp["labels"] if rows is None else inp["labels"][rows]) == case.ignore_index
    assert np.all(got_loss[ign] == 0) and np.all(got_dX[ign] == 0)


@pytest.mark.parametrize("M,D,V", [(300, 200, 1000), (129, 64, 264), (1, 8, 8), (513, 328, 4096)])
def test_ce_small(lib, M, D, V):
    case = CeCase(f"ce_{M}_{D}_{V}", M, D, V, 9000 + M + D + V)
    inp = make_ce_case(case)
    _compare(case, inp, *_run(lib, inp))


def test_ce_slices_from_workspace(lib):
    """A workspace with room for 256 vocabulary columns gives four slices for V = 1000;
    a large one gives one; both match the oracle and each other closely."""
    case = CeCase("ce_slices", 300, 200, 1000, 9100)
    inp = make_ce_case(case)
    small = lib.ce_workspace_bytes(case.M, case.D, case.V, 256)
    one = _run(lib, inp, slice_=0)
    four = _run(lib, inp, ws_bytes=small)
    _compare(case, inp, *four)
    assert torch.equal(one[0], four[0]) and torch.equal(one[1], four[1])  # the forward does not slice
    check("dX slices", host_f64(four[2]), host_f64(one[2]))


def test_ce_empty_batch(lib):
    case = CeCase("ce_empty", 0, 64, 256, 9200)
    W = lib.LoraWeight(case.V, case.D, torch.zeros((case.V, case.D), dtype=torch.bfloat16, device="cuda"))
    ce = lib.LoraCrossEntropy(W)
    E = torch.empty((0, case.D), dtype=torch.bfloat16, device="cuda")
    lab = torch.empty(0, dtype=torch.int32, device="cuda")
    loss, lse = ce.forward(E, lab)
    dX = ce.backward(E, lab, lse, torch.empty(0, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert loss.numel() == 0 and dX.numel() == 0


@pytest.mark.slow
def test_ce_llama3_vocab(lib):
    """Llama-3 vocabulary (V = 128256) over D = 4096 hidden states, M = 2048 rows:
    loss, lse and dX on sampled rows (the backward in 16384-column slices)."""
    case = CeCase("ce_llama3", 2048, 4096, 128256, 9300)
    inp = make_ce_case(case)
    loss, lse, dX = _run(lib, inp, slice_=16384)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, case.M - 1], rng.choice(case.M, 22, replace=False)]))
    _compare(case, inp, loss, lse, dX, rows=rows)
