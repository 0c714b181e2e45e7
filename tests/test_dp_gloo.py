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
