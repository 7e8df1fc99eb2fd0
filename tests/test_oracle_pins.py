"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties one part of the oracle to something other than itself: a
number a page prints, a closed form, an invariant, a special case that
reduces to a textbook routine, or central finite differences.
"""

import math
import os

import numpy as np
import pytest
from scipy import stats

import oracle
from gpt_decoder_lm_b200 import workloads as W
from tests.helpers import oracle_config, rel_l2

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            out[parts[0]] = parts[1:]
    return out


TINY = oracle.Config(vocab_size=11, n_layer=2, n_head=2, n_embd=8, block_size=6, batch_size=2,
                     init_std=0.3, weight_decay=0.1, grad_clip=1.0)


# ---------------------------------------------------------------- counts


def test_param_count_micro_matches_page():
    g = _golden("page_values.txt")
    cfg = oracle_config(W.MICRO)
    assert oracle.param_count(cfg) == int(g["micro_param_count"][0]) == 4192
    assert oracle.param_count_closed_form(cfg) == 4192


@pytest.mark.parametrize("w", list(W.ALL.values()), ids=list(W.ALL))
def test_param_count_closed_form(w):
    cfg = oracle_config(w)
    assert oracle.param_count(cfg) == oracle.param_count_closed_form(cfg)
    gcfg = cfg.with_(variant="gpt2")
    V, d, T, L = w.vocab_size, w.n_embd, w.block_size, w.n_layer
    assert oracle.param_count(gcfg) == V * d + T * d + L * (12 * d * d + 13 * d) + 2 * d


def test_param_count_known_sizes():
    # GPT-2 124M-sized model (vocab 50257, block 1024): 124,439,808 parameters
    # with the position embedding; GPT-2 XL: 1,557,611,200.
    assert oracle.param_count(oracle_config(W.GPT2_124M)) == 124_439_808
    assert oracle.param_count(oracle_config(W.GPT2_XL)) == 1_557_611_200
    assert oracle.param_count(oracle_config(W.MICRO).with_(variant="gpt2")) == 4000


def test_head_dim_page():
    g = _golden("page_values.txt")["head_dim_runlog"]
    cfg = oracle.Config(vocab_size=10, n_layer=1, n_head=int(g[1]), n_embd=int(g[0]), block_size=4)
    assert cfg.head_dim == int(g[2])


# ---------------------------------------------------------------- generators


def test_splitmix64_known_answers():
    with open(os.path.join(GOLDEN, "splitmix64_seed0.txt")) as f:
        want = [int(l, 16) for l in f if l.strip() and not l.startswith("#")]
    gamma = np.uint64(0x9E3779B97F4A7C15)
    with np.errstate(over="ignore"):
        got = [int(oracle.sm64(np.uint64(k) * gamma)) for k in range(len(want))]
    assert got == want


def test_init_is_gaussian_with_std():
    cfg = oracle_config(W.CHAR)
    spec = oracle.tensor_specs(cfg)[2 + 2]  # h.0.attn.c_attn.weight
    assert spec.name == "h.0.attn.c_attn.weight"
    w = oracle.init_tensor(cfg, 1337, 4, spec).ravel()
    assert w.dtype == np.float64
    assert np.array_equal(w, w.astype(np.float32).astype(np.float64))
    assert abs(w.mean()) < 4 * 0.02 / math.sqrt(w.size)
    assert abs(w.std() / 0.02 - 1) < 0.01
    assert stats.kstest(w / 0.02, "norm").pvalue > 1e-3
    # different tensors / seeds give unrelated values
    w2 = oracle.init_tensor(cfg, 1337, 6, oracle.tensor_specs(cfg)[6]).ravel()
    assert abs(np.corrcoef(w[: w2.size], w2[: w.size])[0, 1]) < 0.02


def test_init_constants():
    cfg = oracle_config(W.CHAR)
    P = oracle.init_params(cfg, 7)
    assert np.all(P["h.0.ln_1.weight"] == 1) and np.all(P["h.0.ln_1.bias"] == 0)
    assert np.all(P["h.3.mlp.c_fc.bias"] == 0) and np.all(P["ln_f.weight"] == 1)


def test_batch_gather_windows():
    stream = np.arange(1000, dtype=np.int64) % 97
    idx, tgt = oracle.gather_batch(stream, 16, 5, step=3, micro=1, batch_size=64)
    ix = oracle.batch_offsets(1000, 16, 5, 3, 1, 64)
    assert ix.min() >= 0 and ix.max() <= 1000 - 16 - 1 + 1
    assert np.array_equal(tgt[:, :-1], idx[:, 1:])
    for b in range(64):
        assert np.array_equal(idx[b], stream[ix[b]: ix[b] + 16])
        assert np.array_equal(tgt[b], stream[ix[b] + 1: ix[b] + 17])
    # offsets are uniform over [0, N - T)
    many = np.concatenate([oracle.batch_offsets(1 << 20, 1024, 9, s, 0, 512) for s in range(40)])
    assert stats.kstest(many / ((1 << 20) - 1024), "uniform").pvalue > 1e-3
    assert not np.array_equal(oracle.batch_offsets(1000, 16, 5, 3, 1, 8), oracle.batch_offsets(1000, 16, 5, 3, 2, 8))


def test_dropout_mask_rate():
    n = 1 << 18
    e = np.arange(n, dtype=np.uint64)
    keep = oracle.dropout_keep(1339, 7, 3, 2, e, 0.1)
    frac = keep.mean()
    assert abs(frac - 0.9) < 4 * math.sqrt(0.09 / n)
    assert oracle.dropout_keep(1339, 7, 3, 2, e, 0.0).all()
    assert not np.array_equal(keep, oracle.dropout_keep(1339, 7, 3, 1, e, 0.1))


# ---------------------------------------------------------------- forward


def test_uniform_logits_give_ln_vocab():
    cfg = oracle_config(W.CHAR).with_(batch_size=2, block_size=32)
    P = oracle.init_params(cfg, 1)
    P["wte"][:] = 0.0
    idx, tgt = W.random_batch(W.CHAR, 3, 2, 32)
    loss, cache = oracle.forward(cfg, P, idx, tgt)
    assert abs(loss - math.log(65)) < 1e-12


@pytest.mark.parametrize("w,expect", [(W.MICRO, 3.347), (W.CHAR, 4.251)], ids=["micro", "char"])
def test_initial_loss_near_ln_vocab(w, expect):
    # E[loss] ~ ln V + Var(logit)/2 with Var(logit) = d * std^2 (unit-variance
    # normalised features against N(0, std^2) head rows).
    cfg = oracle_config(w)
    B = min(w.batch_size, 8)
    P = oracle.init_params(cfg, w.weight_seed)
    idx, tgt = W.random_batch(w, 11, B, w.block_size)
    loss, _ = oracle.forward(cfg, P, idx, tgt)
    analytic = math.log(w.vocab_size) + w.n_embd * w.init_std ** 2 / 2
    assert abs(analytic - expect) < 1e-3
    assert abs(loss - analytic) < 0.15


def test_initial_loss_gpt2_vocab_matches_run_log():
    g = _golden("page_values.txt")["initial_loss_gpt2_vocab"]
    w = W.GPT2_124M
    cfg = oracle_config(w).with_(n_layer=2, block_size=128)
    P = oracle.init_params(cfg, w.weight_seed)
    idx, tgt = W.random_batch(w.with_(block_size=128), 5, 1, 128)
    loss, _ = oracle.forward(cfg, P, idx, tgt)
    assert abs(loss - float(g[0])) < float(g[1])
    assert abs(loss - (math.log(50257) + 768 * 0.02 ** 2 / 2)) < 0.15


def test_softmax_rows_sum_to_one():
    cfg = TINY
    P = oracle.init_params(cfg, 3)
    idx = np.array([[1, 2, 3, 4, 5, 6], [0, 0, 10, 9, 8, 7]])
    loss, cache = oracle.forward(cfg, P, idx, idx)
    for lc in cache["layers"]:
        assert np.allclose(lc["p"].sum(-1), 1.0, atol=1e-12, rtol=0)
        assert np.all(np.triu(lc["p"][0, 0], 1) == 0)
    pz = np.exp(cache["z"] - cache["lse"][..., None])
    assert np.allclose(pz.sum(-1), 1.0, atol=1e-12, rtol=0)


def test_causality():
    cfg = TINY
    P = oracle.init_params(cfg, 4)
    idx = np.array([[1, 2, 3, 4, 5, 6], [0, 0, 10, 9, 8, 7]])
    _, c1 = oracle.forward(cfg, P, idx, None)
    for t in range(5):
        idx2 = idx.copy()
        idx2[:, t + 1:] = (idx2[:, t + 1:] + 3) % 11
        _, c2 = oracle.forward(cfg, P, idx2, None)
        np.testing.assert_allclose(c2["z"][:, : t + 1], c1["z"][:, : t + 1], rtol=0, atol=1e-13)
        assert not np.allclose(c2["z"][:, t + 1:], c1["z"][:, t + 1:])


def test_single_position_attention_is_value_projection():
    cfg = TINY.with_(block_size=1)
    P = oracle.init_params(cfg, 5)
    idx = np.array([[3], [7]])
    _, cache = oracle.forward(cfg, P, idx, None)
    lc = cache["layers"][0]
    np.testing.assert_allclose(lc["o"].reshape(2, 8), lc["v"].transpose(0, 2, 1, 3).reshape(2, 8), atol=1e-15)


def test_layernorm_and_activations_textbook():
    cfg = TINY
    x = np.full((3, 8), 2.5)
    w = np.linspace(0.5, 1.5, 8)
    b = np.linspace(-1, 1, 8)
    y, _ = oracle.gpt_oracle._norm_fwd(cfg, x, w, b)
    np.testing.assert_allclose(y, np.broadcast_to(b, y.shape), atol=1e-12)
    # textbook LayerNorm on a random row: zero mean / unit (biased) variance
    r = np.random.default_rng(0).normal(size=(4, 8)) * 3 + 1
    y, _ = oracle.gpt_oracle._norm_fwd(cfg, r, np.ones(8), np.zeros(8))
    np.testing.assert_allclose(y.mean(-1), 0, atol=1e-12)
    np.testing.assert_allclose((y ** 2).mean(-1), r.var(-1) / (r.var(-1) + 1e-5), rtol=1e-12)
    # GELU(x) = x Phi(x): GELU(0) = 0, GELU(1) = Phi(1) (standard normal table 0.841344746...)
    h = np.array([0.0, 1.0, -1.0])
    g = oracle.gpt_oracle._act_fwd(cfg, h)
    np.testing.assert_allclose(g, [0.0, stats.norm.cdf(1.0), -stats.norm.cdf(-1.0)], atol=1e-15)
    assert abs(g[1] - 0.8413447460685429) < 1e-15
    m = cfg.with_(variant="micro")
    np.testing.assert_array_equal(oracle.gpt_oracle._act_fwd(m, h), [0.0, 1.0, 0.0])
    y, _ = oracle.gpt_oracle._norm_fwd(m, r, None, None)
    np.testing.assert_allclose((y ** 2).mean(-1), (r ** 2).mean(-1) / ((r ** 2).mean(-1) + 1e-5), rtol=1e-12)


# ---------------------------------------------------------------- backward


def _fd_check(cfg, P, idx, tgt, drop=None, h=1e-5, tol=1e-6):
    _, G, _ = oracle.loss_and_grads(cfg, P, idx, tgt, drop)
    for name, w in P.items():
        fd = np.zeros_like(w)
        flat = w.reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + h
            lp, _ = oracle.forward(cfg, P, idx, tgt, drop, keep_cache=False)
            flat[i] = old - h
            lm, _ = oracle.forward(cfg, P, idx, tgt, drop, keep_cache=False)
            flat[i] = old
            fd.reshape(-1)[i] = (lp - lm) / (2 * h)
        err = rel_l2(G[name], fd)
        assert err < tol, (name, err)


def test_backward_finite_differences_gpt2():
    cfg = TINY
    P = oracle.init_params(cfg, 21)
    for k in P:                              # move norms/biases off their init values
        if P[k].ndim == 1:
            P[k] += np.random.default_rng(len(k)).normal(scale=0.2, size=P[k].shape)
    idx = np.array([[1, 2, 3, 4, 5, 6], [0, 0, 10, 9, 8, 7]])
    tgt = np.array([[2, 3, 4, 5, 6, 1], [0, 10, 9, 8, 7, 3]])
    _fd_check(cfg, P, idx, tgt)


def test_backward_finite_differences_dropout():
    cfg = TINY.with_(dropout=0.25, dropout_seed=99)
    P = oracle.init_params(cfg, 22)
    idx = np.array([[1, 2, 3, 4, 5, 6], [0, 0, 10, 9, 8, 7]])
    tgt = np.array([[2, 3, 4, 5, 6, 1], [0, 10, 9, 8, 7, 3]])
    _fd_check(cfg, P, idx, tgt, drop=oracle.gpt_oracle.DropCtx(99, 3))


def test_backward_finite_differences_micro():
    w = W.MICRO
    cfg = oracle_config(w).with_(batch_size=2)
    P = oracle.init_params(cfg, 5)
    idx, tgt = W.random_batch(w, 8, 2, 16)
    # ReLU has a kink at 0: the step must stay well inside the distance of every
    # pre-activation from it (smallest |h| here is ~1.7e-5).
    _, cache = oracle.forward(cfg, P, idx, tgt)
    step = 1e-7
    assert np.abs(cache["layers"][0]["h"]).min() > 20 * step * np.abs(cache["layers"][0]["a2"]).max()
    _fd_check(cfg, P, idx, tgt, h=step)


def test_grad_accumulation_equals_concatenated_batch():
    cfg = TINY
    P = oracle.init_params(cfg, 30)
    rng = np.random.default_rng(1)
    i1, t1, i2, t2 = (rng.integers(0, 11, size=(2, 6)) for _ in range(4))
    _, g1, _ = oracle.loss_and_grads(cfg, P, i1, t1, loss_scale=0.5)
    _, g2, _ = oracle.loss_and_grads(cfg, P, i2, t2, loss_scale=0.5)
    _, g, _ = oracle.loss_and_grads(cfg.with_(batch_size=4), P, np.concatenate([i1, i2]), np.concatenate([t1, t2]))
    for k in g:
        np.testing.assert_allclose(g1[k] + g2[k], g[k], rtol=1e-10, atol=1e-14)


# ---------------------------------------------------------------- optimizer / schedule


def test_adam_first_step_closed_form():
    g = _golden("page_values.txt")["adam_micro"]
    b1, b2, eps, lr = map(float, g)
    cfg = TINY.with_(beta1=b1, beta2=b2, eps=eps, weight_decay=0.0, grad_clip=0.0)
    P = oracle.init_params(cfg, 1)
    P0 = {k: v.copy() for k, v in P.items()}
    G = {k: np.random.default_rng(i).normal(size=v.shape) * 1e-3 for i, (k, v) in enumerate(P.items())}
    oracle.clip_adamw(cfg, P, G, oracle.AdamState(), lr, 1)
    for k in P:
        np.testing.assert_allclose(P[k] - P0[k], -lr * G[k] / (np.abs(G[k]) + eps), rtol=1e-12, atol=1e-18)


def test_adamw_decay_and_clip():
    b1, b2, wd = map(float, _golden("page_values.txt")["adamw_runlog"])
    cfg = TINY.with_(beta1=b1, beta2=b2, weight_decay=wd, grad_clip=1.0)
    P = oracle.init_params(cfg, 2)
    for k in P:
        P[k] = P[k] + 0.5
    P0 = {k: v.copy() for k, v in P.items()}
    zero = {k: np.zeros_like(v) for k, v in P.items()}
    oracle.clip_adamw(cfg, P, zero, oracle.AdamState(), 1e-2, 1)
    for k in P:     # zero gradient: only the decoupled decay acts, on matrices only
        want = P0[k] * (1 - 1e-2 * wd) if P0[k].ndim == 2 else P0[k]
        np.testing.assert_allclose(P[k], want, rtol=1e-15)
    # clipping: a gradient of norm 10 is scaled to norm 1 (up to the 1e-6 guard)
    G = {k: np.full_like(v, 1.0) for k, v in P.items()}
    n = oracle.global_grad_norm(G)
    G = {k: v * (10.0 / n) for k, v in G.items()}
    norm = oracle.clip_adamw(cfg, P, G, oracle.AdamState(), 1e-3, 1)
    assert abs(norm - 10.0) < 1e-12
    c = min(1.0, 1.0 / (norm + 1e-6))
    assert abs(c * norm - 1.0) < 1e-6


def test_adam_constant_gradient_second_step():
    cfg = TINY.with_(weight_decay=0.0, grad_clip=0.0)
    P = oracle.init_params(cfg, 3)
    G = {k: np.full_like(v, 0.01) for k, v in P.items()}
    S = oracle.AdamState()
    oracle.clip_adamw(cfg, P, {k: v.copy() for k, v in G.items()}, S, 1e-3, 1)
    P1 = {k: v.copy() for k, v in P.items()}
    oracle.clip_adamw(cfg, P, {k: v.copy() for k, v in G.items()}, S, 1e-3, 2)
    for k in P:     # bias-corrected moments equal g and g^2 exactly
        np.testing.assert_allclose(P[k] - P1[k], -1e-3 * 0.01 / (0.01 + cfg.eps), rtol=1e-9)


def test_lr_schedules():
    lr, w, mx = 6e-4, 100, 1100
    assert oracle.lr_cosine(lr, 0, w, mx) == 0.0
    assert abs(oracle.lr_cosine(lr, w, w, mx) - lr) < 1e-18
    assert abs(oracle.lr_cosine(lr, w // 2, w, mx) - lr / 2) < 1e-18
    assert abs(oracle.lr_cosine(lr, (w + mx) // 2, w, mx) - lr / 2) < 1e-15
    assert abs(oracle.lr_cosine(lr, mx, w, mx)) < 1e-18
    assert oracle.lr_linear(1e-2, 0, 100) == 1e-2 and oracle.lr_linear(1e-2, 100, 100) == 0.0
    assert abs(oracle.lr_linear(1e-2, 25, 100) - 7.5e-3) < 1e-18


def test_resume_equals_uninterrupted():
    w = W.MICRO
    cfg = oracle_config(w).with_(batch_size=2)
    stream = W.token_stream(w, n=4096).astype(np.int64)

    def run(P, S, steps):
        for s in steps:
            oracle.train_step(cfg, P, S, stream, w.data_seed, oracle.lr_linear(w.lr, s - 1, 10), s)

    Pa, Sa = oracle.init_params(cfg, 1), oracle.AdamState()
    run(Pa, Sa, range(1, 11))
    Pb, Sb = oracle.init_params(cfg, 1), oracle.AdamState()
    run(Pb, Sb, range(1, 6))
    Pc = {k: v.copy() for k, v in Pb.items()}
    Sc = oracle.AdamState({k: v.copy() for k, v in Sb.m.items()}, {k: v.copy() for k, v in Sb.v.items()})
    run(Pc, Sc, range(6, 11))
    for k in Pa:
        assert np.array_equal(Pa[k], Pc[k])


def test_argmax_ties_lowest_index():
    z = np.array([[1.0, 3.0, 3.0, 0.0], [5.0, 5.0, 5.0, 5.0]])
    assert list(oracle.argmax_rows(z)) == [1, 0]


def test_attention_uniform_scores_is_causal_mean():
    # q = 0 makes every allowed score equal: output i is the mean of v_0..v_i
    rng = np.random.default_rng(3)
    v = rng.standard_normal((2, 3, 7, 4))
    k = rng.standard_normal((2, 3, 7, 4))
    q = np.zeros_like(k)
    o, p, lse = oracle.attention_fwd(q, k, v)
    want = np.cumsum(v, axis=2) / np.arange(1, 8)[None, None, :, None]
    np.testing.assert_allclose(o, want, atol=1e-14)
    np.testing.assert_allclose(lse, np.log(np.arange(1, 8))[None, None, :].repeat(2, 0).repeat(3, 1), atol=1e-14)


def test_attention_backward_finite_differences():
    rng = np.random.default_rng(4)
    q, k, v, w = (rng.standard_normal((1, 2, 5, 4)) for _ in range(4))
    keep = rng.random((1, 2, 5, 5)) > 0.3
    o, p, _ = oracle.attention_fwd(q, k, v, keep, 0.3)
    dq, dk, dv = oracle.attention_bwd(q, k, v, p, w, keep, 0.3)
    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        fd = np.zeros_like(x)
        for i in np.ndindex(x.shape):
            old = x[i]
            x[i] = old + h
            lp = (oracle.attention_fwd(q, k, v, keep, 0.3)[0] * w).sum()
            x[i] = old - h
            lm = (oracle.attention_fwd(q, k, v, keep, 0.3)[0] * w).sum()
            x[i] = old
            fd[i] = (lp - lm) / (2 * h)
        assert rel_l2(g, fd) < 1e-7
