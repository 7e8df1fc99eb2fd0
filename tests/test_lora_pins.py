"""Pins of the LoRA oracle (oracle/lora.py) against facts outside it: the
closed-form parameter count, the base model at B = 0, the low-rank branch
written out directly, finite differences of the loss, and the closed form of
the first AdamW step over the trainable set."""

import numpy as np
import pytest

from oracle import gpt_oracle as O
from oracle import lora as LR

TINY = O.Config(vocab_size=11, n_layer=2, n_head=2, n_embd=16, block_size=8, batch_size=2, init_std=0.3,
                weight_decay=0.1, grad_clip=1.0)


def _batch(cfg, seed):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, cfg.vocab_size, (cfg.batch_size, cfg.block_size))
    tgt = rng.integers(0, cfg.vocab_size, (cfg.batch_size, cfg.block_size))
    return idx, tgt


def test_param_count_closed_form():
    # per adapted block: A r x d plus B d x r; GPT-2 124M with r = 8 on q and v:
    # 12 layers x 2 blocks x 2 x 8 x 768
    gpt2 = O.Config(vocab_size=50257, n_layer=12, n_head=12, n_embd=768, block_size=1024)
    assert LR.lora_param_count(gpt2, LR.LoraConfig(r=8)) == 294912
    assert LR.lora_param_count(gpt2, LR.LoraConfig(r=16, targets=("q",))) == 12 * 2 * 16 * 768


def test_zero_B_is_the_base_model():
    lc = LR.LoraConfig(r=4, alpha=16)
    P = O.init_params(TINY, 1)
    Lp = LR.init_lora(TINY, lc, 2)
    idx, tgt = _batch(TINY, 3)
    base, _, _ = O.loss_and_grads(TINY, P, idx, tgt)
    loss, GL, _ = LR.loss_and_grads(TINY, P, Lp, lc, idx, tgt)
    assert loss == base
    for _, _, na, nb in LR.lora_names(TINY, lc):
        assert not GL[na].any()          # dL/dA = s B^T G vanishes with B = 0
        assert np.abs(GL[nb]).max() > 0  # while B receives a gradient


def test_low_rank_branch_written_out():
    # q and v of layer 0 equal a W0^T + b + s (a A^T) B^T computed directly
    # from the norm output; k is the base projection
    lc = LR.LoraConfig(r=3, alpha=6)
    P = O.init_params(TINY, 1)
    Lp = LR.init_lora(TINY, lc, 5, b_std=0.2)
    idx, _ = _batch(TINY, 7)
    _, cache = O.forward(TINY, LR.merged_params(TINY, P, Lp, lc), idx, None)
    lc0 = cache["layers"][0]
    a = lc0["a"]
    d, H = TINY.n_embd, TINY.n_head
    W = P["h.0.attn.c_attn.weight"]
    b = P["h.0.attn.c_attn.bias"]
    s = 6 / 3

    def heads(x):
        return x.reshape(TINY.batch_size, TINY.block_size, H, d // H).transpose(0, 2, 1, 3)

    q = a @ W[:d].T + b[:d] + s * (a @ Lp["h.0.attn.lora_q.A"].T) @ Lp["h.0.attn.lora_q.B"].T
    k = a @ W[d:2 * d].T + b[d:2 * d]
    v = a @ W[2 * d:].T + b[2 * d:] + s * (a @ Lp["h.0.attn.lora_v.A"].T) @ Lp["h.0.attn.lora_v.B"].T
    np.testing.assert_allclose(lc0["q"], heads(q), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lc0["k"], heads(k), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lc0["v"], heads(v), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("variant", ["gpt2", "micro"])
def test_gradients_match_finite_differences(variant):
    cfg = TINY.with_(variant=variant)
    lc = LR.LoraConfig(r=2, alpha=4)
    P = O.init_params(cfg, 11)
    Lp = LR.init_lora(cfg, lc, 12, b_std=0.3)
    idx, tgt = _batch(cfg, 13)
    _, GL, _ = LR.loss_and_grads(cfg, P, Lp, lc, idx, tgt)
    rng = np.random.default_rng(14)
    eps = 1e-6
    for name in sorted(Lp):
        for _ in range(4):
            i = tuple(int(rng.integers(0, n)) for n in Lp[name].shape)
            old = Lp[name][i]
            Lp[name][i] = old + eps
            lp, _, _ = LR.loss_and_grads(cfg, P, Lp, lc, idx, tgt)
            Lp[name][i] = old - eps
            lm, _, _ = LR.loss_and_grads(cfg, P, Lp, lc, idx, tgt)
            Lp[name][i] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - GL[name][i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, GL[name][i])


def test_train_step_freezes_base_and_takes_the_first_adamw_step():
    cfg = TINY.with_(grad_accum=2)
    lc = LR.LoraConfig(r=2, alpha=16)
    P = O.init_params(cfg, 21)
    P0 = {k: v.copy() for k, v in P.items()}
    Lp = LR.init_lora(cfg, lc, 22, b_std=0.1)
    L0 = {k: v.copy() for k, v in Lp.items()}
    stream = np.random.default_rng(23).integers(0, cfg.vocab_size, 4096)
    lr, step = 1e-2, 1
    # the step's summed gradient, computed before the update
    GL = None
    for mu in range(cfg.grad_accum):
        idx, tgt = O.gather_batch(stream, cfg.block_size, 5, step, mu, cfg.batch_size)
        _, g, _ = LR.loss_and_grads(cfg, P, Lp, lc, idx, tgt, None, 1.0 / cfg.grad_accum)
        GL = g if GL is None else {k: GL[k] + g[k] for k in GL}
    norm = np.sqrt(sum((g * g).sum() for g in GL.values()))
    c = min(1.0, cfg.grad_clip / (norm + 1e-6))
    _, got_norm = LR.train_step(cfg, P, Lp, lc, LR.LoraAdamState(), stream, 5, lr, step)
    assert got_norm == pytest.approx(norm, rel=1e-12)
    for k in P:
        assert np.array_equal(P[k], P0[k]), k
    # step 1: m_hat = g, v_hat = g^2, so the update is g / (|g| + eps) per element
    for k in Lp:
        g = c * GL[k]
        want = L0[k] * (1 - lr * cfg.weight_decay) - lr * g / (np.abs(g) + cfg.eps)
        np.testing.assert_allclose(Lp[k], want, rtol=1e-12, atol=1e-15)
