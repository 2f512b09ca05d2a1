"""Data-parallel exchange of the adapter gradients, on CPU ranks (gloo).

Two processes each take a contiguous shard of the tokens, form the shard's
dA and dB with the oracle (the fp64 statement of the layer), round them to
bf16 as the layer's outputs are, and exchange them through
nf4_base_lora_b200.dp.  Because dA and dB are sums over tokens, the exchanged
result must match the oracle's gradients of the whole batch within the
layer's tolerance, and be the same on every rank.  A shard may be empty (fewer
tokens than ranks): it contributes zero gradients.  No GPU is used."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import workloads
from parity import assert_close

WORLD = 2


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _grads_worker(rank, world, port, m):
    from nf4_base_lora_b200 import dp
    _init(rank, world, port)
    try:
        c = workloads.linear_case(256, 192, m, 8, alpha=16.0)
        b, e = dp.token_shard(m, world, rank)
        dA_s, dB_s = oracle.lora_grads(c.A, c.B, c.X[b:e], c.dY[b:e], c.scaling)
        dA = torch.from_numpy(dA_s).to(torch.bfloat16).contiguous()
        dB = torch.from_numpy(dB_s).to(torch.bfloat16).contiguous()
        ex = dp.LoraGradExchange([dA, dB])
        assert ex.numel == dA.numel() + dB.numel()
        ex()
        dA_ref, dB_ref = oracle.lora_grads(c.A, c.B, c.X, c.dY, c.scaling)
        assert_close(dA, dA_ref, "dA (exchanged, rank %d)" % rank)
        assert_close(dB, dB_ref, "dB (exchanged, rank %d)" % rank)
        # the same bits on every rank
        mine = torch.cat([dA.float().reshape(-1), dB.float().reshape(-1)])
        got = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(got, mine)
        for t in got:
            assert torch.equal(t, mine)
    finally:
        dist.destroy_process_group()


def _exact_worker(rank, world, port):
    from nf4_base_lora_b200 import dp
    _init(rank, world, port)
    try:
        a = torch.arange(12, dtype=torch.float32).reshape(3, 4) * (rank + 1)
        b = torch.full((5,), float(rank), dtype=torch.float32)
        h = torch.tensor([0.5, -2.0], dtype=torch.bfloat16) * (rank + 1)
        dp.LoraGradExchange([a, b, h])()
        tot = sum(range(1, world + 1))
        assert torch.equal(a, torch.arange(12, dtype=torch.float32).reshape(3, 4) * tot)
        assert torch.equal(b, torch.full((5,), float(sum(range(world))), dtype=torch.float32))
        assert torch.equal(h, torch.tensor([0.5 * tot, -2.0 * tot], dtype=torch.bfloat16))
        c = torch.full((4,), float(2 * (rank + 1)), dtype=torch.float32)
        dp.LoraGradExchange([c])(average=True)
        assert torch.equal(c, torch.full((4,), float(world + 1), dtype=torch.float32))
        assert dp.max_over_ranks(rank + 1.5, torch.device("cpu")) == world + 0.5
    finally:
        dist.destroy_process_group()


def test_token_shard_partition():
    from nf4_base_lora_b200 import dp
    for m in (0, 1, 2, 7, 16, 37, 8192):
        for world in (1, 2, 3, 8):
            spans = [dp.token_shard(m, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == m
            for (b0, e0), (b1, _) in zip(spans, spans[1:]):
                assert e0 == b1
            sizes = [e - b for b, e in spans]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    with pytest.raises(ValueError):
        dp.token_shard(4, 2, 2)
    with pytest.raises(ValueError):
        dp.token_shard(-1, 2, 0)


@pytest.mark.parametrize("m", [37, 1])
def test_exchange_gives_full_batch_gradients(m):
    """m = 37: shards of 19 and 18 tokens; m = 1: the second rank's shard is empty."""
    mp.spawn(_grads_worker, args=(WORLD, _free_port(), m), nprocs=WORLD, join=True)


def test_exchange_exact_sum_and_mean():
    mp.spawn(_exact_worker, args=(WORLD, _free_port()), nprocs=WORLD, join=True)


def test_exchange_rejects_bad_inputs():
    from nf4_base_lora_b200 import dp
    with pytest.raises(ValueError):
        dp.LoraGradExchange([])
    with pytest.raises(ValueError):
        dp.LoraGradExchange([torch.zeros(4, dtype=torch.float16)])
    with pytest.raises(ValueError):
        dp.LoraGradExchange([torch.zeros(4, 4).t()])


def _overlap_worker(rank, world, port):
    """Per-module buckets exchanged one by one (on CPU the exchange runs at
    launch): the same sums as one exchange of everything, on every rank."""
    from nf4_base_lora_b200 import dp
    _init(rank, world, port)
    try:
        c = workloads.linear_case(128, 192, 23, 8, alpha=16.0)
        b, e = dp.token_shard(23, world, rank)
        grads = []
        for i in range(3):                       # three modules, scaled copies of one case
            dA_s, dB_s = oracle.lora_grads(c.A, c.B, c.X[b:e], c.dY[b:e], c.scaling * (i + 1))
            grads.append([torch.from_numpy(dA_s).to(torch.bfloat16).contiguous(),
                          torch.from_numpy(dB_s).to(torch.bfloat16).contiguous()])
        whole = [t.clone() for g in grads for t in g]
        dp.LoraGradExchange(whole)()
        ex = dp.OverlappedGradExchange(grads)
        assert not ex.cuda and len(ex.buckets) == 3
        for i in reversed(range(3)):             # the backward visits the modules last to first
            ex.launch(i)
        ex.finish()
        for got, ref in zip([t for g in grads for t in g], whole):
            assert torch.equal(got, ref)
    finally:
        dist.destroy_process_group()


def test_overlapped_exchange_matches_single_exchange():
    mp.spawn(_overlap_worker, args=(WORLD, _free_port()), nprocs=WORLD, join=True)


def test_overlapped_exchange_rejects_bad_inputs():
    from nf4_base_lora_b200 import dp
    with pytest.raises(ValueError):
        dp.OverlappedGradExchange([])
    with pytest.raises(ValueError):
        dp.OverlappedGradExchange([[torch.zeros(4, dtype=torch.float16)]])
