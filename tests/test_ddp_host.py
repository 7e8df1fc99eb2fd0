"""Host logic of the data-parallel gradient exchange (gpt_decoder_lm_b200/
ddp.py and gpt_grad_buckets), on CPU: the bucket plan covers the gradient
arena exactly once in backward order, and the bucket-by-bucket all-reduce
gives every rank the mean over ranks, run as two gloo ranks.  For the
sharded optimiser (ZeRO-1): the shards (gpt_zero1_shard) partition the
arena, the bucket plan cut at the shard bounds gives every element one
owner, and the reduce-to-owner / in-place all-gather pattern gives every
rank the full result, run as three gloo ranks (a ragged last shard)."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from gpt_decoder_lm_b200 import binding as gb
from gpt_decoder_lm_b200 import ddp
from gpt_decoder_lm_b200 import workloads as W


@pytest.fixture(scope="module", autouse=True)
def lib():
    import __graft_entry__
    __graft_entry__.build()
    return gb.lib()


@pytest.mark.parametrize("w,over", [(W.GPT2_124M, {}), (W.GPT2_XL, {}), (W.MICRO, {}), (W.CHAR, {"decay_1d": 1})],
                         ids=["gpt2_124m", "gpt2_xl", "micro", "char_decay_1d"])
def test_bucket_plan_covers_the_arena_once(w, over):
    cfg = gb.make_config(w, **over)
    r = gb.grad_buckets(cfg)
    spans = sorted((o, c) for o, c, _ in r)
    pos = 0
    for o, c in spans:          # contiguous, no overlap, from 0
        assert o == pos and c > 0
        pos += c
    assert pos >= gb.param_count(cfg)            # the arena holds every parameter (plus alignment and padding)
    assert pos % 64 == 0
    buckets = [b for _, _, b in r]
    assert buckets == sorted(buckets)             # listed in backward order
    assert set(buckets) == set(range(w.n_layer + 1))
    plan = ddp.bucket_plan(cfg)
    assert [b for b, _ in plan] == list(range(w.n_layer + 1))
    if w.variant == "gpt2" and not over.get("decay_1d"):
        # a layer: its four matrices (12 d^2, 64-aligned) and its eight vectors (13 d) as two runs
        d = w.n_embd
        for b, ranges in plan[:-1]:
            assert len(ranges) == 2
            assert sorted(c for _, c in ranges)[-1] == 12 * d * d


def _rank(rank, world, port, out, sizes):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = gb.make_config(W.CHAR.with_(n_layer=3))
        plan = ddp.bucket_plan(cfg)
        n = sum(c for _, ranges in plan for _, c in ranges)
        g = torch.arange(n, dtype=torch.float32) * (rank + 1) + 0.25 * rank
        for _, ranges in plan:   # the order every rank follows
            ddp.exchange_bucket(g, ranges, None, world)
        want = torch.arange(n, dtype=torch.float32) * 1.5 + 0.125
        out[rank] = float((g - want).abs().max())
        sizes[rank] = n
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_bucket_exchange_gives_the_mean_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out, sizes = mgr.dict(), mgr.dict()
    port = socket.socket()
    port.bind(("127.0.0.1", 0))
    p = port.getsockname()[1]
    port.close()
    procs = [ctx.Process(target=_rank, args=(r, 2, p, out, sizes)) for r in range(2)]
    for q in procs:
        q.start()
    for q in procs:
        q.join(180)
        assert q.exitcode == 0
    assert sizes[0] == sizes[1]
    assert out[0] <= 1e-3 and out[1] <= 1e-3   # fp32 mean of values up to ~1e7: a few ulps


@pytest.mark.parametrize("w", [W.GPT2_124M, W.GPT2_XL, W.CHAR, W.MICRO], ids=["gpt2_124m", "gpt2_xl", "char", "micro"])
def test_zero1_shards_partition_the_arena(w):
    cfg = gb.make_config(w)
    plan = ddp.bucket_plan(cfg)
    n = sum(c for _, ranges in plan for _, c in ranges)
    for world in (1, 2, 3, 4, 7, 8, 64):
        shards = [gb.zero1_shard(cfg, world, r) for r in range(world)]
        stride = shards[0][2]
        assert stride % 64 == 0 and all(s[2] == stride for s in shards)
        assert world * stride <= n + 4096          # an in-place all-gather fits the arenas' slack
        pos = 0
        for off, cnt, _ in shards:
            assert off == min(pos, n) and cnt >= 0 and cnt % 4 == 0
            pos += cnt
        assert pos == n
        owner = np.full(n, -1)
        for bucket, parts in ddp.shard_parts(plan, stride, world):
            for r, off, cnt in parts:
                assert cnt > 0
                so, sc, _ = shards[r]
                assert so <= off and off + cnt <= so + sc   # a part lies inside its owner's shard
                assert (owner[off:off + cnt] == -1).all()
                owner[off:off + cnt] = r
        assert (owner >= 0).all()
    for bad in ((0, 0), (65, 0), (2, 2), (2, -1)):
        with pytest.raises(gb.GptError):
            gb.zero1_shard(cfg, *bad)


def _zero_rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = gb.make_config(W.CHAR.with_(n_layer=3))
        plan = ddp.bucket_plan(cfg)
        n = sum(c for _, ranges in plan for _, c in ranges)
        off, cnt, stride = gb.zero1_shard(cfg, world, rank)
        base = (torch.arange(n) % 4099).to(torch.float32)   # small integers: every sum exact
        g = base * (rank + 1)                       # sum over ranks: base * 6
        for _, parts in ddp.shard_parts(plan, stride, world):
            ddp.reduce_parts(g, parts)
        own_ok = bool(torch.equal(g[off:off + cnt], base[off:off + cnt] * 6))
        # the "update" of the own shard, then the in-place all-gather over a slack-padded arena
        w = torch.full((n + 4096,), float("nan"))
        w[off:off + cnt] = g[off:off + cnt] * 0.5
        ddp.all_gather_shards(w, stride, world, rank)
        out[rank] = (own_ok, bool(torch.equal(w[:n], base * 3)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_zero1_exchange_over_three_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = socket.socket()
    port.bind(("127.0.0.1", 0))
    p = port.getsockname()[1]
    port.close()
    procs = [ctx.Process(target=_zero_rank, args=(r, 3, p, out)) for r in range(3)]
    for q in procs:
        q.start()
    for q in procs:
        q.join(180)
        assert q.exitcode == 0
    assert all(out[r] == (True, True) for r in range(3)), dict(out)
