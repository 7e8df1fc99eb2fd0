"""Autoregressive generation with the key / value cache (gpt_generate)
against the cache-free oracle (oracle/sampling.py).

Every generated token is checked in the context the GPU produced: the
oracle's logits of that prefix (a full forward, no cache) decide the draw.
Greedy tokens must be the oracle's arg-max wherever its top-2 gap exceeds
the logit error bound of the precision (bf16: 0.05, fp32: 1e-4), and
otherwise within that bound of the maximum.  Sampled tokens must equal the
oracle's draw at the same uniform wherever the decision is robust to logit
perturbations of that size; everywhere else they must be kept tokens."""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a GPU", allow_module_level=True)

import oracle  # noqa: E402
from oracle import sampling as S  # noqa: E402
from gpt_decoder_lm_b200 import binding as gb  # noqa: E402
from gpt_decoder_lm_b200 import workloads as W  # noqa: E402
from tests.helpers import oracle_config  # noqa: E402


def setup(w, **over):
    cfg = gb.make_config(w, **over)
    m = gb.Model(cfg, seed=w.weight_seed)
    oc = oracle_config(w).with_(**over)
    return m, cfg, oracle.init_params(oc, w.weight_seed), oc


def generate(m, cfg, T0, n_new, temperature, top_k, top_p, seed):
    rng = np.random.default_rng(seed)
    B = cfg.batch_size
    prompt = rng.integers(0, cfg.vocab_size, (B, T0)).astype(np.int32)
    U = rng.random((n_new, B)).astype(np.float32)
    out = torch.full((B, T0 + n_new), -1, dtype=torch.int32, device="cuda")
    m.generate(torch.from_numpy(prompt).cuda(), n_new, temperature, top_k, top_p, torch.from_numpy(U).cuda(), out)
    seq = out.cpu().numpy().astype(np.int64)
    assert np.array_equal(seq[:, :T0], prompt)
    assert ((seq >= 0) & (seq < cfg.vocab_size)).all()
    return seq, U.astype(np.float64)


def oracle_logits(oc, P, prefix):
    return oracle.forward(oc, P, prefix, None)[1]["z"][:, -1, :]


@pytest.mark.parametrize("wname,precision,tol", [("char", "bf16", 0.05), ("char", "fp32", 1e-4),
                                                  ("micro", "fp32", 1e-4), ("micro64", "bf16", 0.05),
                                                  ("char12", "bf16", 0.05)])
def test_greedy_generation_matches_oracle(wname, precision, tol):
    w = (W.CHAR if wname.startswith("char") else W.MICRO).with_(precision=precision)
    # micro64: the RMSNorm variant wide enough for the decoding GEMM that computes the norm itself;
    # char12: 12 rows, the two-tile (9-16 row) decoding GEMM with the LayerNorm computed inside it,
    # as GPT-2 124M decoding at batch 12 runs it
    over = {"char": dict(n_layer=2, batch_size=4, block_size=128), "micro": {},
            "micro64": dict(n_layer=2, n_embd=64, n_head=4),
            "char12": dict(n_layer=2, batch_size=12, block_size=128)}[wname]
    m, cfg, P, oc = setup(w, **over)
    T0, n_new = (9, 20) if wname.startswith("char") else (4, 12)
    seq, _ = generate(m, cfg, T0, n_new, 0.0, 0, 1.0, seed=1)
    exact = 0
    for s in range(n_new):
        z = oracle_logits(oc, P, seq[:, :T0 + s])
        for b in range(cfg.batch_size):
            tok = seq[b, T0 + s]
            top2 = np.sort(z[b])[-2:]
            if top2[1] - top2[0] > tol:
                assert tok == np.argmax(z[b]), (s, b, tok, np.argmax(z[b]))
                exact += 1
            else:
                assert z[b, tok] >= z[b].max() - tol, (s, b)
    assert exact >= n_new * cfg.batch_size // 2
    m.close()


def robust_draw(z, temperature, top_k, top_p, u, eps):
    """The oracle's draw when logit errors up to eps cannot change it (the
    top-k membership, the nucleus and the inverse-CDF position all keep a
    margin; probabilities move by about eps / temperature relative), else
    None."""
    ref = S.sample_row(z, temperature, top_k, top_p, u)
    zs = np.sort(z)[::-1]
    if 0 < top_k < len(z) and zs[top_k - 1] - zs[top_k] <= 2 * eps:
        return None
    d = eps / temperature
    p = S._kept_probs(z, temperature, top_k, top_p)
    c = np.cumsum(p) / p.sum()
    if np.min(np.abs(c - u)) < 2 * d:
        return None
    if top_p < 1.0:
        for pp in (top_p - 2 * d, top_p + 2 * d):
            if S.sample_row(z, temperature, top_k, min(max(pp, 0.0), 1.0), u) != ref:
                return None
    return ref


@pytest.mark.parametrize("precision,eps", [("bf16", 0.1), ("fp32", 1e-4)])
def test_sampled_generation_matches_oracle(precision, eps):
    # a wider initialisation than training's (logits of standard deviation ~6)
    # so that enough draws are decided robustly under bf16 logit errors
    w = W.CHAR.with_(precision=precision, init_std=0.3)
    m, cfg, P, oc = setup(w, n_layer=2, batch_size=4, block_size=128)
    T0, n_new, temperature, top_k, top_p = 5, 24, 1.0, 5, 0.95
    seq, U = generate(m, cfg, T0, n_new, temperature, top_k, top_p, seed=2)
    exact = 0
    for s in range(n_new):
        z = oracle_logits(oc, P, seq[:, :T0 + s])
        for b in range(cfg.batch_size):
            tok = seq[b, T0 + s]
            ref = robust_draw(z[b], temperature, top_k, top_p, U[s, b], eps)
            if ref is not None:
                assert tok == ref, (s, b, tok, ref)
                exact += 1
            else:
                loose = S._kept_probs(z[b] + 0.0, temperature, min(top_k + 5, len(z[b]) - 1), 1.0)
                assert loose[tok] > 0, (s, b, tok)
    assert exact >= n_new * cfg.batch_size // 8, exact
    m.close()


def test_generate_errors():
    w = W.CHAR
    m, cfg, _, _ = setup(w, n_layer=1, batch_size=2, block_size=64)
    prompt = torch.zeros((2, 60), dtype=torch.int32, device="cuda")
    U = torch.zeros((10, 2), device="cuda")
    out = torch.empty((2, 70), dtype=torch.int32, device="cuda")
    with pytest.raises(gb.GptError) as e:
        m.generate(prompt, 10, 1.0, 0, 1.0, U, out)  # 60 + 10 > block_size
    assert e.value.name == "GPT_ERR_INVALID_ARG"
    prompt = torch.full((2, 4), cfg.vocab_size + 3, dtype=torch.int32, device="cuda")
    with pytest.raises(gb.GptError) as e:
        m.generate(prompt, 2, 1.0, 0, 1.0, U, out)
    assert e.value.name == "GPT_ERR_TOKEN_RANGE"
    m.close()


def test_generate_graph_replay_matches_eager():
    """A repeated call shape replays a CUDA graph of the whole call (the first
    call is eager, the second captured); replays read the prompt and uniforms
    in place, so new contents give the eager result for those contents."""
    w = W.CHAR.with_(precision="bf16", init_std=0.3)
    over = dict(n_layer=2, batch_size=4, block_size=128)
    m_graph, cfg, _, _ = setup(w, **over)
    m_eager, _, _, _ = setup(w, **over)
    m_eager.set_graphs(False)
    B, T0, n_new = cfg.batch_size, 7, 16
    prompt = torch.zeros((B, T0), dtype=torch.int32, device="cuda")
    U = torch.zeros((n_new, B), device="cuda")
    out_g = torch.full((B, T0 + n_new), -1, dtype=torch.int32, device="cuda")
    out_e = torch.full_like(out_g, -1)
    rng = np.random.default_rng(5)
    for call in range(5):
        prompt.copy_(torch.from_numpy(rng.integers(0, cfg.vocab_size, (B, T0)).astype(np.int32)))
        U.copy_(torch.from_numpy(rng.random((n_new, B)).astype(np.float32)))
        m_graph.generate(prompt, n_new, 1.0, 5, 0.95, U, out_g)
        m_eager.generate(prompt, n_new, 1.0, 5, 0.95, U, out_e)
        assert torch.equal(out_g, out_e), call
    # the token-range check still reports from a replayed graph
    prompt.fill_(cfg.vocab_size + 1)
    with pytest.raises(gb.GptError) as e:
        m_graph.generate(prompt, n_new, 1.0, 5, 0.95, U, out_g)
    assert e.value.name == "GPT_ERR_TOKEN_RANGE"
    # a new call shape starts over (eager, capture, replay) and stays exact
    p3 = torch.zeros((B, 3), dtype=torch.int32, device="cuda")
    short_g = torch.full((B, 3 + n_new), -1, dtype=torch.int32, device="cuda")
    short_e = torch.full_like(short_g, -1)
    for call in range(4):
        p3.copy_(torch.from_numpy(rng.integers(0, cfg.vocab_size, (B, 3)).astype(np.int32)))
        U.copy_(torch.from_numpy(rng.random((n_new, B)).astype(np.float32)))
        m_graph.generate(p3, n_new, 0.7, 0, 0.9, U, short_g)
        m_eager.generate(p3, n_new, 0.7, 0, 0.9, U, short_e)
        assert torch.equal(short_g, short_e), call
    m_graph.close()
    m_eager.close()
