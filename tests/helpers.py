"""Test helpers: map a workload preset onto the oracle's Config."""

import numpy as np

import oracle
from gpt_decoder_lm_b200.workloads import Workload


def oracle_config(w: Workload, **kw) -> "oracle.Config":
    c = oracle.Config(
        vocab_size=w.vocab_size, n_layer=w.n_layer, n_head=w.n_head, n_embd=w.n_embd,
        block_size=w.block_size, batch_size=w.batch_size, grad_accum=w.grad_accum,
        variant=w.variant, init_std=w.init_std, dropout=w.dropout, beta1=w.beta1,
        beta2=w.beta2, eps=w.eps, weight_decay=w.weight_decay, grad_clip=w.grad_clip,
        dropout_seed=w.dropout_seed)
    return c.with_(**kw) if kw else c


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))
