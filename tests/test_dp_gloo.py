"""Data-parallel path on CPU with two gloo ranks: per-rank adapter gradients of each
rank's token shard, summed with the same all-reduce helper the benchmark uses, equal
the gradients of the whole batch; Y and dX rows are those of the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from synth import LoraCase, make_case


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, M_total, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from qlora_linear_b200.dp import allreduce_adapter_grads, token_shard
        case = LoraCase("dp", M_total, 40, 48, 8, 16.0, "bf16", 4321)
        inp = make_case(case)
        X, W, A, B, dY = (O.bf16_to_f64(inp[k]) for k in ("X", "W", "A", "B", "dY"))
        lo, hi = token_shard(M_total, rank, world)
        g = O.lora_backward(dY[lo:hi], X[lo:hi], W, A, B, case.s)
        dA = torch.from_numpy(g["dA"].copy())
        dB = torch.from_numpy(g["dB"].copy())
        allreduce_adapter_grads(dA, dB)
        full = O.lora_backward(dY, X, W, A, B, case.s)
        ok = (np.allclose(dA.numpy(), full["dA"], rtol=1e-12, atol=1e-12)
              and np.allclose(dB.numpy(), full["dB"], rtol=1e-12, atol=1e-12)
              and np.allclose(g["dX"], full["dX"][lo:hi], rtol=1e-12, atol=1e-12))
        q.put((rank, bool(ok), lo, hi))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M_total", [64, 37])
def test_two_rank_gloo_adapter_grads_sum_to_full_batch(M_total):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, M_total, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert all(ok for _, ok, _, _ in res)
    # the shards tile the batch exactly
    assert res[0][2] == 0 and res[0][3] == res[1][2] and res[1][3] == M_total


def test_token_shard_covers_every_token_once():
    from qlora_linear_b200.dp import token_shard
    for M in (0, 1, 7, 64, 1001):
        for world in (1, 2, 3, 8):
            spans = [token_shard(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            assert max(b - a for a, b in spans) - min(b - a for a, b in spans) <= 1


def _cpu_round(src: torch.Tensor, dst: torch.Tensor) -> None:
    # the rounding the library's lora_round_bf16 applies (nearest even), on the host
    dst.copy_(src.to(torch.bfloat16))


def _worker_f32(rank, world, port, M_total, q):
    """One rank of the fp32 exchange: the rank's adapter gradients as the library emits
    them with LORA_GRADS_F32 (fp32 values of s·Σ over the rank's tokens; here the exact
    sums rounded to fp32), written into the exchange buffer, summed over ranks with one
    all-reduce and rounded to bf16 once."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from qlora_linear_b200.dp import AdapterGradExchange, token_shard
        case = LoraCase("dp32", M_total, 64, 48, 8, 16.0, "bf16", 98765)
        inp = make_case(case)
        X, W, A, B, dY = (O.bf16_to_f64(inp[k]) for k in ("X", "W", "A", "B", "dY"))
        lo, hi = token_shard(M_total, rank, world)
        g = O.lora_backward(dY[lo:hi], X[lo:hi], W, A, B, case.s)
        ex = AdapterGradExchange([g["dA"].shape, g["dB"].shape], "cpu", round_fn=_cpu_round)
        ex.views[0].copy_(torch.from_numpy(g["dA"].astype(np.float32)))
        ex.views[1].copy_(torch.from_numpy(g["dB"].astype(np.float32)))
        ex.allreduce()
        dA = torch.empty(g["dA"].shape, dtype=torch.bfloat16)
        dB = torch.empty(g["dB"].shape, dtype=torch.bfloat16)
        ex.round_into([dA, dB])
        full = O.lora_backward(dY, X, W, A, B, case.s)
        res = {}
        for name, got in (("dA", dA), ("dB", dB)):
            got = got.to(torch.float64).numpy()
            ref = full[name]
            err = got - ref
            rms = np.linalg.norm(ref) / np.sqrt(ref.size)
            res[name] = (float(np.linalg.norm(err) / np.linalg.norm(ref)), float(np.max(np.abs(err)) / rms),
                         # one rounding: within half a bf16 ulp (2^-8 relative) plus fp32 noise
                         bool(np.all(np.abs(err) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * rms)))
        # the whole buffer went through one collective: every rank holds the same bits
        digest = torch.tensor([float(ex.flat.double().sum())])
        gathered = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, digest.double())
        same = all(float(t) == float(gathered[0]) for t in gathered)
        q.put((rank, res, same))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,M_total", [(2, 64), (2, 37), (4, 61)])
def test_gloo_fp32_exchange_rounds_once_and_meets_the_bar(world, M_total):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_f32, args=(r, world, port, M_total, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, r, same in res:
        assert same, "ranks disagree after the all-reduce"
        for name, (rel, emax, one_rounding) in r.items():
            assert rel <= 1e-2 and emax <= 5e-2, (rank, name, rel, emax)
            assert one_rounding, (rank, name)


def test_exchange_buffer_layout():
    from qlora_linear_b200.dp import AdapterGradExchange
    ex = AdapterGradExchange([(8, 40), (48, 8), (3, 5)], "cpu", round_fn=_cpu_round)
    starts = [v.data_ptr() - ex.flat.data_ptr() for v in ex.views]
    assert starts == [0, 320 * 4, (320 + 384) * 4]
    assert all(s % 16 == 0 for s in starts)
    assert [tuple(v.shape) for v in ex.views] == [(8, 40), (48, 8), (3, 5)]
    with pytest.raises(ValueError):
        ex.round_into([torch.empty((8, 40), dtype=torch.bfloat16)])
