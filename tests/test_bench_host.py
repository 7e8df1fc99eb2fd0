"""Host logic of bench.py on CPU: the max-over-ranks reduction used for the
multi-replica timing, run as two gloo ranks; FLOP accounting closed forms."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
from gpt_decoder_lm_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        v = bench.reduce_max(10.0 + 5.0 * rank, torch.device("cpu"))
        out[rank] = v
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 15.0


def test_reduce_max_without_group_is_identity():
    import torch
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5


def test_flop_accounting():
    w = W.GPT2_124M
    # 6N + 12 L d T with N excluding the position embedding (855.2 MFLOP/token)
    assert abs(bench.flops_per_token(w) - 855_166_464) < 1
    d, L, V, M = 768, 12, 50257, 12 * 1024
    assert bench.gemm_flops_per_step(w) == 3 * 5 * 2 * M * (L * 12 * d * d + V * d)


def test_decode_bytes_accounting():
    # GPT-2 124M: 12 layers x 12 d^2 bf16 weights + the padded tied head, plus
    # keys and values (2 x d bf16 per position, layer and row) up to pos
    w = W.GPT2_124M
    weights = 2 * (12 * 12 * 768 * 768 + 50304 * 768)
    assert bench.decode_bytes_per_step(w, 0) == weights + 2 * 2 * 768 * 1 * 12 * 12
    assert bench.decode_bytes_per_step(w, 95.0) == weights + 2 * 2 * 768 * 96 * 12 * 12
    assert abs(bench.decode_bytes_per_step(w, 96.0) - 290_045_952) < 1  # the bench line's per_step_bytes
