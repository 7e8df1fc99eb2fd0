"""The data-parallel step (gpt_decoder_lm_b200/ddp.py: accumulate, bucketed
NCCL all-reduce overlapped on a second stream, clip + AdamW) on a one-rank
NCCL group: the exchange is then the identity, so the step must equal
gpt_train_step bit for bit (losses, norms, weights), eager and replayed.
This checks the split of the step, the bucket events and the stream
ordering on the GPU; the mean over several ranks is checked on CPU with two
gloo ranks (tests/test_ddp_host.py).

The sharded optimiser (ZeroTrainer, ZeRO-1) is checked the same way on one
rank, and with two ranks emulated on one GPU: two models take the two ranks'
batches, the reduce-to-owner and the all-gathers are done with tensor copies
between their arenas, each model runs gpt_grad_sumsq_shard /
gpt_clip_adamw_shard on its own shard, and the result must equal, bit for
bit, a third model that takes the mean gradient and the whole-arena
gpt_clip_adamw_step (the data-parallel step)."""

import os
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import torch.distributed as dist  # noqa: E402

from gpt_decoder_lm_b200 import binding as gb  # noqa: E402
from gpt_decoder_lm_b200 import ddp  # noqa: E402
from gpt_decoder_lm_b200 import workloads as W  # noqa: E402


@pytest.fixture(scope="module")
def group():
    import datetime
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    yield None
    dist.destroy_process_group()


def _weights(m):
    P = m.get(gb.GPT_PARAM)
    return np.concatenate([P[k].ravel() for k in sorted(P)])


@pytest.mark.parametrize("wname", ["char", "dropout"])
def test_one_rank_data_parallel_step_equals_train_step(group, wname):
    w, over = {"char": (W.CHAR, dict(n_layer=2, batch_size=4, block_size=128, grad_accum=2)),
               "dropout": (W.DROPOUT_512, dict(n_layer=2, batch_size=2, block_size=256, grad_accum=2,
                                               token_dtype=gb.GPT_TOK_I32))}[wname]
    sd = torch.from_numpy(W.token_stream(w, n=1 << 16).astype(np.int32)).cuda()
    res = []
    for use_ddp in (False, True):
        m = gb.Model(gb.make_config(w, **over), seed=w.weight_seed)
        tr = ddp.DataParallelTrainer(m) if use_ddp else None
        out = []
        for step in range(1, 6):
            lr = gb.lr_cosine(w.lr, step - 1, 2, 6)
            out.append(tr.step(sd, w.data_seed, lr, step) if use_ddp else m.train_step(sd, w.data_seed, lr, step))
        res.append((out, _weights(m)))
        assert m.flags() == 0
        m.close()
    (l0, w0), (l1, w1) = res
    assert l0 == l1
    assert np.array_equal(w0, w1)


def test_one_rank_data_parallel_host_batches(group):
    w = W.CHAR
    over = dict(n_layer=2, batch_size=4, block_size=128, grad_accum=2)
    res = []
    for use_ddp in (False, True):
        m = gb.Model(gb.make_config(w, **over), seed=w.weight_seed)
        tr = ddp.DataParallelTrainer(m) if use_ddp else None
        out = []
        for step in range(1, 5):
            idx, tgt = W.random_batch(w, 50 + step, 8, 128)
            idx, tgt = np.ascontiguousarray(idx, np.int32), np.ascontiguousarray(tgt, np.int32)
            out.append(tr.step_host(idx, tgt, 1e-3, step) if use_ddp else m.train_step_host(idx, tgt, 1e-3, step))
        res.append((out, _weights(m)))
        m.close()
    assert res[0][0] == res[1][0]
    assert np.array_equal(res[0][1], res[1][1])


@pytest.mark.parametrize("wname", ["char", "dropout"])
def test_one_rank_zero1_step_equals_train_step(group, wname):
    w, over = {"char": (W.CHAR, dict(n_layer=2, batch_size=4, block_size=128, grad_accum=2)),
               "dropout": (W.DROPOUT_512, dict(n_layer=2, batch_size=2, block_size=256, grad_accum=2,
                                               token_dtype=gb.GPT_TOK_I32))}[wname]
    sd = torch.from_numpy(W.token_stream(w, n=1 << 16).astype(np.int32)).cuda()
    res = []
    for use_zero in (False, True):
        m = gb.Model(gb.make_config(w, **over), seed=w.weight_seed)
        tr = ddp.ZeroTrainer(m) if use_zero else None
        out = []
        for step in range(1, 6):
            lr = gb.lr_cosine(w.lr, step - 1, 2, 6)
            out.append(tr.step(sd, w.data_seed, lr, step) if use_zero else m.train_step(sd, w.data_seed, lr, step))
        res.append((out, _weights(m)))
        assert m.flags() == 0
        m.close()
    (l0, w0), (l1, w1) = res
    assert l0 == l1
    assert np.array_equal(w0, w1)


def test_two_ranks_zero1_emulated_equal_the_data_parallel_step():
    w = W.CHAR
    over = dict(n_layer=2, batch_size=4, block_size=128, grad_accum=2)
    cfg = gb.make_config(w, **over)
    world = 2
    # the two ranks hold the moments of their own shard only (zero_world 2)
    A, B = (gb.Model(gb.make_config(w, zero_world=world, zero_rank=r, **over), seed=w.weight_seed)
            for r in range(world))
    C = gb.Model(cfg, seed=w.weight_seed)
    ar = [A.state_arenas(), B.state_arenas()]
    ref = C.state_arenas()
    n = ref["n"]
    shards = [gb.zero1_shard(cfg, world, r) for r in range(world)]
    stride = shards[0][2]
    parts = [p for _, ps in ddp.shard_parts(ddp.bucket_plan(cfg), stride, world) for p in ps]
    partials = [torch.zeros(gb.NORM_PARTIALS, dtype=torch.float64, device="cuda") for _ in range(world)]
    for step in range(1, 4):
        lr = 1e-3 * step
        batches = [W.random_batch(w, 100 * step + r, 8, 128) for r in range(world)]
        for mdl, (idx, tgt) in zip((A, B), batches):
            mdl.train_step_host_accumulate(idx, tgt, step)
        C.train_step_host_accumulate(*batches[0], step)
        torch.cuda.synchronize()
        gA, gB = ar[0]["grad"], ar[1]["grad"]
        ref["grad"][:n].copy_((gA[:n] + gB[:n]) * 0.5)           # the data-parallel mean
        for r, off, cnt in parts:                                  # the sum reduced to each part's owner
            ar[r]["grad"][off:off + cnt] += ar[1 - r]["grad"][off:off + cnt]
        for r, mdl in enumerate((A, B)):
            mdl.grad_sumsq_shard(shards[r][0], shards[r][1], partials[r])
        gathered = torch.cat(partials)
        norms = [mdl.clip_adamw_shard(lr, step, shards[r][0], shards[r][1], 1.0 / world, gathered)
                 for r, mdl in enumerate((A, B))]
        for name in ("param", "param_bf16"):                       # the all-gathers
            for r in range(world):
                off, cnt, _ = shards[r]
                ar[1 - r][name][off:off + cnt].copy_(ar[r][name][off:off + cnt])
        norm_ref = C.clip_adamw_step(lr, step)
        torch.cuda.synchronize()
        # every rank sums the same gathered partials: one norm; the data-parallel
        # step sums another partition of the same squares (fp64), which rounds to
        # the same fp32 norm unless a last-bit tie falls differently
        assert norms[0] == norms[1]
        assert abs(norms[0] - norm_ref) <= 1e-6 * norm_ref
        same = (lambda a, b: torch.equal(a, b)) if norms[0] == norm_ref else \
            (lambda a, b: torch.allclose(a.float(), b.float(), rtol=1e-5 if a.dtype == torch.float32 else 8e-3,
                                         atol=1e-7))
        for r in range(world):
            assert not ar[r]["grad"][:n].any()                     # the whole arena cleared
            for name in ("param", "param_bf16"):
                assert same(ar[r][name][:n], ref[name][:n]), (step, r, name)
            off, cnt, _ = shards[r]
            for name in ("adam_m", "adam_v"):                      # each owner's moments (compact)
                assert same(ar[r][name][:cnt], ref[name][off:off + cnt]), (step, r, name)
    for mdl in (A, B, C):
        assert mdl.flags() == 0
        mdl.close()


def test_sharded_moments_model_limits():
    """A model whose config shards the moments (zero_world 2) holds its own
    shard of them only: the whole-arena optimiser calls and the moment
    accessors refuse, the shard call accepts its own shard alone, and the
    workspace is smaller by the other shard's moments."""
    w = W.CHAR
    over = dict(n_layer=2, batch_size=4, block_size=128, grad_accum=2)
    full = gb.make_config(w, **over)
    cfg = gb.make_config(w, zero_world=2, zero_rank=1, **over)
    off, cnt, stride = gb.zero1_shard(cfg, 2, 1)
    n = gb.Model(full, seed=1).state_arenas()["n"]
    assert gb.workspace_bytes(full) - gb.workspace_bytes(cfg) >= 8 * (n + 4096 - stride) - 512
    m = gb.Model(cfg, seed=w.weight_seed)
    sd = torch.from_numpy(W.token_stream(w, n=1 << 16).astype(np.int32)).cuda()
    for call in (lambda: m.train_step(sd, w.data_seed, 1e-3, 1), lambda: m.clip_adamw_step(1e-3, 1),
                 lambda: m.get(gb.GPT_ADAM_M)):
        with pytest.raises(gb.GptError) as e:
            call()
        assert e.value.name == "GPT_ERR_UNSUPPORTED"
    m.train_step_accumulate(sd, w.data_seed, 1, sync=True)
    parts = torch.zeros(gb.NORM_PARTIALS, dtype=torch.float64, device="cuda")
    m.grad_sumsq_shard(off, cnt, parts)
    with pytest.raises(gb.GptError) as e:
        m.clip_adamw_shard(1e-3, 1, 0, cnt, 0.5, parts)
    assert e.value.name == "GPT_ERR_INVALID_ARG"
    assert m.clip_adamw_shard(1e-3, 1, off, cnt, 0.5, parts) > 0
    assert m.flags() == 0
    m.close()


def test_zero1_empty_shard_rank():
    """A rank past the end of a small arena (64 shards of the micro model's
    4k-element arena) owns nothing: its shard calls run on an empty range,
    clear its gradients and leave its weights as they were."""
    w = W.MICRO
    world, rank = 64, 63
    cfg = gb.make_config(w, zero_world=world, zero_rank=rank)
    off, cnt, stride = gb.zero1_shard(cfg, world, rank)
    assert cnt == 0
    m = gb.Model(cfg, seed=w.weight_seed)
    ar = m.state_arenas()
    n = ar["n"]
    w0 = ar["param"][:n].clone()
    idx, tgt = W.random_batch(w, 5, w.batch_size * w.grad_accum, w.block_size)
    m.train_step_host_accumulate(idx, tgt, 1)
    parts = torch.full((gb.NORM_PARTIALS,), 7.0, dtype=torch.float64, device="cuda")
    m.grad_sumsq_shard(off, cnt, parts)
    assert not parts.any()                       # an empty shard: zero partial sums
    gathered = torch.zeros(world * gb.NORM_PARTIALS, dtype=torch.float64, device="cuda")
    assert m.clip_adamw_shard(1e-3, 1, off, cnt, 1.0 / world, gathered) == 0.0
    assert not ar["grad"][:n].any()
    assert torch.equal(ar["param"][:n], w0)
    assert m.flags() == 0
    m.close()
