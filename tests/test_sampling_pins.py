"""Pins of the evaluation / sampling oracle (oracle/sampling.py) against
closed forms and exact properties of inverse-CDF sampling: greedy and
top_k = 1 reduce to the arg-max; uniform logits give floor(u V); over a
uniform grid of M draws every token's frequency is its (kept,
renormalised) probability to within 1/M; the nucleus of a hand-computed
distribution; temperature scaling; the evaluation loss of uniform logits is
ln V; generation of one token is one draw from the last position."""

import math

import numpy as np
import pytest

import oracle
from oracle import sampling as S


def grid_freq(z, temperature, top_k, top_p, M=20000):
    u = (np.arange(M) + 0.5) / M
    toks = np.array([S.sample_row(z, temperature, top_k, top_p, x) for x in u])
    return np.bincount(toks, minlength=len(z)) / M


def softmax(y):
    e = np.exp(y - y.max())
    return e / e.sum()


def test_greedy_and_top1_are_argmax():
    rng = np.random.default_rng(0)
    z = rng.standard_normal(97)
    z[40] = z.max() + 1.0
    for u in (0.0, 0.3, 0.999):
        assert S.sample_row(z, 0.0, 0, 1.0, u) == 40
        assert S.sample_row(z, 0.8, 1, 1.0, u) == 40
        assert S.sample_row(z, 1.3, 0, 1e-9, u) == 40
    z2 = np.zeros(10)
    z2[[3, 7]] = 5.0
    assert S.sample_row(z2, 0.0, 0, 1.0, 0.5) == 3  # lowest index among tied maxima


def test_uniform_logits_inverse_cdf():
    V = 50
    z = np.full(V, 0.25)
    for u in (0.001, 0.0101, 0.37, 0.6543, 0.999):
        assert S.sample_row(z, 1.0, 0, 1.0, u) == math.floor(u * V)


@pytest.mark.parametrize("temperature", [1.0, 0.5, 2.0])
def test_frequencies_are_softmax(temperature):
    rng = np.random.default_rng(1)
    z = rng.standard_normal(30) * 2
    f = grid_freq(z, temperature, 0, 1.0)
    np.testing.assert_allclose(f, softmax(z / temperature), atol=1.0 / 20000 + 1e-12)


def test_top_k_renormalises_the_k_largest():
    rng = np.random.default_rng(2)
    z = rng.standard_normal(40)
    k = 5
    top = np.argsort(-z)[:k]
    f = grid_freq(z, 0.7, k, 1.0)
    expect = np.zeros_like(z)
    expect[top] = softmax(z[top] / 0.7)
    np.testing.assert_allclose(f, expect, atol=1.0 / 20000 + 1e-12)
    # ties at the k-th value are kept
    z3 = np.array([3.0, 1.0, 2.0, 2.0, 0.0])
    f3 = grid_freq(z3, 1.0, 2, 1.0)
    assert f3[1] == 0 and f3[4] == 0 and f3[2] > 0 and f3[3] > 0


def test_nucleus_closed_form():
    z = np.log(np.array([0.2, 0.5, 0.3]))
    # cumulative mass in probability order: 0.5, 0.8, 1.0
    np.testing.assert_allclose(grid_freq(z, 1.0, 0, 0.7), [0.0, 0.625, 0.375], atol=1e-4)
    np.testing.assert_allclose(grid_freq(z, 1.0, 0, 0.85), [0.2, 0.5, 0.3], atol=1e-4)
    np.testing.assert_allclose(grid_freq(z, 1.0, 0, 0.5), [0.0, 1.0, 0.0], atol=1e-12)
    # top-k first, then the nucleus of the renormalised two
    np.testing.assert_allclose(grid_freq(z, 1.0, 2, 0.6), [0.0, 1.0, 0.0], atol=1e-12)


def _tiny():
    cfg = oracle.Config(vocab_size=11, n_layer=2, n_head=2, n_embd=8, block_size=8, batch_size=2, grad_accum=1)
    return cfg, oracle.init_params(cfg, 5)


def test_eval_loss_of_uniform_logits_is_log_v():
    cfg, P = _tiny()
    P["wte"][:] = 0.0  # tied head: every logit 0
    stream = np.random.default_rng(3).integers(0, cfg.vocab_size, 200)
    assert abs(S.eval_loss(cfg, P, stream, 9, 3) - math.log(cfg.vocab_size)) < 1e-12


def test_eval_loss_is_the_mean_of_batch_losses():
    cfg, P = _tiny()
    stream = np.random.default_rng(4).integers(0, cfg.vocab_size, 300)
    ls = []
    for i in range(4):
        idx, tgt = oracle.gather_batch(stream, cfg.block_size, 7, i + 1, 0, cfg.batch_size)
        ls.append(oracle.forward(cfg, P, idx, tgt)[0])
    assert abs(S.eval_loss(cfg, P, stream, 7, 4) - np.mean(ls)) < 1e-15


def test_generate_one_token_is_one_draw_and_keeps_the_prompt():
    cfg, P = _tiny()
    prompt = np.array([[1, 2, 3], [4, 5, 6]])
    U = np.array([[0.3, 0.8]])
    out = S.generate(cfg, P, prompt, 1, 0.9, 4, 0.95, U)
    assert np.array_equal(out[:, :3], prompt)
    z = oracle.forward(cfg, P, prompt, None)[1]["z"][:, -1, :]
    assert list(out[:, 3]) == [S.sample_row(z[b], 0.9, 4, 0.95, U[0, b]) for b in range(2)]
    # greedy continuation is the arg-max chain
    g = S.generate(cfg, P, prompt, 3, 0.0, 0, 1.0, np.zeros((3, 2)))
    seq = prompt
    for _ in range(3):
        z = oracle.forward(cfg, P, seq, None)[1]["z"][:, -1, :]
        seq = np.concatenate([seq, np.argmax(z, -1)[:, None]], axis=1)
    assert np.array_equal(g, seq)
