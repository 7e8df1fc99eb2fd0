"""The data-parallel step (gpt_decoder_lm_b200/ddp.py: accumulate, bucketed
NCCL all-reduce overlapped on a second stream, clip + AdamW) on a one-rank
NCCL group: the exchange is then the identity, so the step must equal
gpt_train_step bit for bit (losses, norms, weights), eager and replayed.
This checks the split of the step, the bucket events and the stream
ordering on the GPU; the mean over several ranks is checked on CPU with two
gloo ranks (tests/test_ddp_host.py)."""

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
