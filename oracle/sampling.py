"""Float64 oracle of evaluation and sampling (generation) for the GPT-2 model
of gpt_oracle.

TEST INFRASTRUCTURE ONLY (tests and the smoke check).  The product library
never imports it, and it imports nothing from the product package.

Sources (section names are the pages' own):

* "nanoGPT README" (translated, oa0.com), section "采样 / 推理": sample.py
  draws num_samples continuations of max_new_tokens tokens from a prompt,
  with a temperature and top_k; train.py's estimate_loss averages the loss
  of eval_iters batches of the val split.
* "微型 GPT 从零构建：核心训练循环、分词与单 GPU 高效推理" (blog.hotdry.top),
  section "单 GPU 高效推理：采样 + KV Cache": autoregressive sampling,
  logits / temperature -> softmax -> draw from the probabilities; top_k;
  top_p (nucleus) among the listed optimisations; the KV cache appends one
  token's keys and values per step instead of recomputing the past.

Readings where the pages are silent (also listed in the design notes):

* temperature <= 0 means greedy decoding: the arg-max, lowest index on ties.
* top_k keeps every token whose logit is >= the k-th largest logit (ties at
  the threshold are kept), k <= 0 or k >= V keeps all.  It is applied to the
  logits before the temperature (the same set for any temperature > 0).
* top_p (after top_k and the softmax): the nucleus is the smallest set of
  most probable tokens whose probability mass reaches top_p; with the
  boundary probability tau of that set, every token with probability >= tau
  is kept (ties kept).  top_p >= 1 keeps all.
* The draw is the inverse CDF of the kept, renormalised probabilities in
  token-index order at a uniform u in [0, 1) given by the caller: the first
  token whose cumulative mass exceeds u times the kept mass.
* Evaluation windows come from the same gather as training (gather_batch)
  with step = i + 1 and micro-batch 0 for the i-th batch.
"""

from __future__ import annotations

from typing import Dict

import numpy as np

from . import gpt_oracle as go

__all__ = ["eval_loss", "sample_row", "sample_rows", "generate"]


def eval_loss(cfg: go.Config, P: Dict[str, np.ndarray], stream: np.ndarray, data_seed: int, n_batches: int) -> float:
    """Mean over n_batches evaluation batches of the batch's mean token loss
    (estimate_loss in train.py, README section "采样 / 推理" neighbourhood)."""
    losses = []
    for i in range(n_batches):
        idx, tgt = go.gather_batch(stream, cfg.block_size, data_seed, i + 1, 0, cfg.batch_size)
        loss, _ = go.forward(cfg, P, idx, tgt, None, keep_cache=False)
        losses.append(loss)
    return float(np.mean(losses))


def _kept_probs(z: np.ndarray, temperature: float, top_k: int, top_p: float) -> np.ndarray:
    """Unnormalised probabilities of the kept tokens (0 elsewhere)."""
    z = np.asarray(z, dtype=np.float64)
    V = z.shape[0]
    keep = np.ones(V, dtype=bool)
    if 0 < top_k < V:
        thr = np.sort(z)[V - top_k]  # the k-th largest value
        keep = z >= thr
    y = np.where(keep, z / temperature, -np.inf)
    p = np.exp(y - y.max())
    if top_p < 1.0:
        q = p / p.sum()
        order = np.argsort(-q, kind="stable")
        cum = np.cumsum(q[order])
        n = int(np.searchsorted(cum, top_p, side="left"))  # first prefix whose mass reaches top_p
        n = min(n, V - 1)
        tau = q[order][n]
        p = np.where(q >= tau, p, 0.0)
    return p


def sample_row(z: np.ndarray, temperature: float, top_k: int, top_p: float, u: float) -> int:
    """One draw from one row of logits (microGPT "单 GPU 高效推理" pipeline:
    logits / temperature -> top-k -> softmax -> top-p -> multinomial)."""
    z = np.asarray(z, dtype=np.float64)
    if temperature <= 0:
        return int(np.argmax(z))
    p = _kept_probs(z, temperature, top_k, top_p)
    c = np.cumsum(p)
    target = u * c[-1]
    i = int(np.searchsorted(c, target, side="right"))  # first index with c[i] > target
    if i >= len(c):
        i = int(np.nonzero(p)[0][-1])
    return i


def sample_rows(Z: np.ndarray, temperature: float, top_k: int, top_p: float, U: np.ndarray) -> np.ndarray:
    return np.array([sample_row(Z[r], temperature, top_k, top_p, float(U[r])) for r in range(Z.shape[0])],
                    dtype=np.int64)


def generate(cfg: go.Config, P: Dict[str, np.ndarray], prompt: np.ndarray, n_new: int, temperature: float,
             top_k: int, top_p: float, U: np.ndarray) -> np.ndarray:
    """Autoregressive continuation of prompt [B, T0] by n_new tokens (README
    sample.py); U [n_new, B] holds the uniforms of the draws.  The oracle has
    no cache: every step runs the full forward over the sequence so far, the
    definition a KV cache must reproduce.  T0 + n_new <= block_size."""
    seq = np.asarray(prompt, dtype=np.int64).copy()
    assert seq.shape[1] + n_new <= cfg.block_size
    for s in range(n_new):
        _, cache = go.forward(cfg, P, seq, None, None, keep_cache=False)
        z = cache["z"][:, -1, :]
        nxt = sample_rows(z, temperature, top_k, top_p, U[s])
        seq = np.concatenate([seq, nxt[:, None]], axis=1)
    return seq
