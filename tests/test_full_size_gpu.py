"""Parity at the dimensions the bench times: GPT-2 124M (12 layers, d 768,
12 heads, T 1024, vocab 50257 padded to 50304) and GPT-2 XL's layer shape
(d 1600, 25 heads, 4d 6400, T 1024, vocab 50257; two of its 48 layers so
that the float64 oracle finishes).

The oracle cannot run twelve (or eight) full windows, so each micro-batch
holds ONE window repeated over the batch rows: the batch's mean loss and its
gradient equal that window's, a property that holds at any size.  The GPU
therefore runs the full-size kernels (M = 12 x 1024 or 8 x 1024 rows, the
launch shapes of the bench) while the oracle runs B = 1.  Two micro-batches
(grad_accum 2) go through gpt_train_step_host, the bench's end-to-end entry
point, so gradient accumulation, the deferred per-step reductions, the
global norm, clipping and AdamW all run at full size.

After the first optimiser step the AdamW moments hold the step's gradient:
m = (1 - beta1) c g and v = (1 - beta2) (c g)^2 with c the clip factor.  So
the step's gradients are read back as m / ((1 - beta1) c) and compared with
the oracle's per tensor (bf16 tolerance, rel-L2 2e-2); v is checked to come
from the same g; the updated weights are checked against the AdamW formula
applied in float64 to the GPU's own moments (rel-L2 1e-6 per tensor).  The
final weights are not compared against the oracle's own AdamW step: at the
first step Adam moves every element by about lr times the SIGN of its
gradient, so elements whose gradient is within bf16 rounding of zero may
move either way (several results are correct there)."""

import functools

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import oracle  # noqa: E402
from gpt_decoder_lm_b200 import binding as gb  # noqa: E402
from gpt_decoder_lm_b200 import workloads as W  # noqa: E402
from tests.helpers import oracle_config, rel_l2  # noqa: E402

GA = 2
LR = 6e-4
WINDOW_SEEDS = (901, 902)


def _workload(name):
    if name == "gpt2_124m":
        return W.GPT2_124M.with_(token_dtype="int32"), {}
    # GPT-2 XL's layer shape at two layers
    return W.GPT2_XL.with_(token_dtype="int32", n_layer=2), {}


def _windows(w):
    return [W.random_batch(w, s, 1, w.block_size) for s in WINDOW_SEEDS]


@functools.lru_cache(maxsize=2)
def _oracle_step(name):
    """The oracle's step on the B = 1 windows: per-window loss, logits
    statistics of window 0, the summed gradients and their norm."""
    w, _ = _workload(name)
    oc = oracle_config(w).with_(batch_size=1, grad_accum=GA)
    P = oracle.init_params(oc, w.weight_seed)
    G, losses = None, []
    lse0 = am0 = gap0 = None
    for i, (idx, tgt) in enumerate(_windows(w)):
        loss, g, cache = oracle.loss_and_grads(oc, P, idx.astype(np.int64), tgt.astype(np.int64), None, 1.0 / GA)
        losses.append(loss)
        if i == 0:
            z = cache["z"].reshape(-1, w.vocab_size)
            zmax = z.max(axis=1)
            lse0 = zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=1))
            top2 = np.partition(z, -2, axis=1)[:, -2:]
            gap0 = np.abs(top2[:, 1] - top2[:, 0])
            am0 = oracle.argmax_rows(z)
        del cache
        if G is None:
            G = g
        else:
            for k in G:
                G[k] += g[k]
    return losses, G, oracle.global_grad_norm(G), lse0, am0, gap0, oc


def _repeat(a, B):
    return np.ascontiguousarray(np.repeat(a, B, axis=0), np.int32)


def _check_full_size_step(name, recompute):
    w, over = _workload(name)
    cfg = gb.make_config(w, grad_accum=GA, recompute=recompute, **over)
    m = gb.Model(cfg, seed=w.weight_seed)
    B, T = cfg.batch_size, cfg.block_size
    losses, OG, onorm, lse0, am0, gap0, oc = _oracle_step(name)
    wins = _windows(w)

    # forward alone on micro-batch 0: loss, per-row LSE and argmax of the
    # 50257-way logits (rows of the repeated window must agree with each other)
    idx0, tgt0 = (_repeat(a, B) for a in wins[0])
    loss0 = m.forward_loss(torch.from_numpy(idx0).cuda(), torch.from_numpy(tgt0).cuda())
    assert abs(loss0 - losses[0]) <= 2e-3, (loss0, losses[0])
    lse = m.lse().reshape(B, T).astype(np.float64)
    assert np.abs(lse - lse[0]).max() <= 1e-5
    assert np.abs(lse[0] - lse0).max() <= 1e-2, np.abs(lse[0] - lse0).max()
    am = m.argmax().reshape(B, T)
    assert np.array_equal(am, np.broadcast_to(am[0], am.shape))
    robust = gap0 > 0.05
    assert robust.mean() > 0.5
    assert np.array_equal(am[0][robust], am0[robust])

    # one optimiser step of two accumulated micro-batches through the
    # host-batch entry point
    W0 = {k: v.astype(np.float64) for k, v in m.get(gb.GPT_PARAM).items()}
    h_idx = np.ascontiguousarray(np.stack([_repeat(a[0], B) for a in wins]))
    h_tgt = np.ascontiguousarray(np.stack([_repeat(a[1], B) for a in wins]))
    loss, norm = m.train_step_host(h_idx, h_tgt, LR, 1)
    assert abs(loss - np.mean(losses)) <= 2e-3, (loss, np.mean(losses))
    assert abs(norm - onorm) <= 2e-2 * onorm, (norm, onorm)
    assert m.flags() == 0

    b1, b2, eps, wd = oc.beta1, oc.beta2, oc.eps, oc.weight_decay
    c = min(1.0, oc.grad_clip / (norm + 1e-6)) if oc.grad_clip > 0 else 1.0
    Mm = {k: v.astype(np.float64) for k, v in m.get(gb.GPT_ADAM_M).items()}
    Vv = {k: v.astype(np.float64) for k, v in m.get(gb.GPT_ADAM_V).items()}
    W1 = {k: v.astype(np.float64) for k, v in m.get(gb.GPT_PARAM).items()}
    assert set(Mm) == set(OG)
    bad = {}
    for k in OG:
        g = Mm[k] / ((1.0 - b1) * c)
        if np.linalg.norm(OG[k]) > 0:
            e = rel_l2(g, OG[k])
            if e > 2e-2:
                bad[k] = e
        # v and m come from the same clipped gradient
        assert rel_l2(Vv[k], (1.0 - b2) * (c * g) ** 2) <= 1e-5, k
    assert not bad, sorted(bad.items(), key=lambda kv: -kv[1])[:8]
    specs = {s.name: s for s in oracle.gpt_oracle.tensor_specs(oc)}
    bc1, bc2 = 1.0 - b1, 1.0 - b2
    for k in W1:
        w0 = W0[k] * ((1.0 - LR * wd) if specs[k].decayed_by_default else 1.0)
        want = w0 - LR * (Mm[k] / bc1) / (np.sqrt(Vv[k] / bc2) + eps)
        assert rel_l2(W1[k], want) <= 1e-6, (k, rel_l2(W1[k], want))
    m.close()


def test_gpt2_124m_full_dims_train_step():
    _check_full_size_step("gpt2_124m", 0)


@pytest.mark.parametrize("recompute", [0, 1], ids=["stored", "recompute"])
def test_gpt2_xl_layer_shape_train_step(recompute):
    _check_full_size_step("gpt2_xl_2l", recompute)


def test_embedding_routing_full_micro_batch():
    # the 12 x 1024 routing sort of the bench's micro-batch: a stable sort of
    # the positions by token id, compared with the definition bit for bit
    w = W.GPT2_124M.with_(token_dtype="int32")
    cfg = gb.make_config(w, n_layer=1, grad_accum=1)
    m = gb.Model(cfg, seed=w.weight_seed)
    idx, tgt = W.random_batch(w, 77, cfg.batch_size, cfg.block_size)
    m.forward_loss(torch.from_numpy(idx).cuda(), torch.from_numpy(tgt).cuda())
    m.backward()
    n, tok, pos = m.embed_routing()
    flat = idx.reshape(-1)
    order = np.lexsort((np.arange(flat.size), flat))
    assert np.array_equal(tok, flat[order])
    assert np.array_equal(pos, order)
    assert n == np.unique(flat).size
    m.close()


@pytest.mark.parametrize("B,T", [(3, 1000), (24, 1024), (32, 1024)], ids=["ragged", "global24k", "max32k"])
def test_embedding_routing_sizes(B, T):
    # the radix routing sort at a ragged size (a partial last round of 1024
    # keys) and past the shared-memory ping-pong (2 M keys above 190 KB: the
    # second key array is the output array), up to the largest micro-batch a
    # config allows (32,768 tokens); a one-layer model of the GPT-2 vocabulary
    w = W.GPT2_124M.with_(token_dtype="int32")
    cfg = gb.make_config(w, n_layer=1, n_head=1, n_embd=64, batch_size=B, block_size=T, grad_accum=1)
    m = gb.Model(cfg, seed=w.weight_seed)
    idx, tgt = W.random_batch(w, 91 + B, B, T)
    m.forward_loss(torch.from_numpy(idx).cuda(), torch.from_numpy(tgt).cuda())
    m.backward()
    n, tok, pos = m.embed_routing()
    flat = idx.reshape(-1)
    order = np.lexsort((np.arange(flat.size), flat))
    assert np.array_equal(tok, flat[order])
    assert np.array_equal(pos, order)
    assert n == np.unique(flat).size
    m.close()
