"""Seeded synthetic workloads shared by the tests, the smoke check and the bench.

This module holds inputs only: the five workload presets (sizes,
hyper-parameters, seeds) and the token streams that stand in for the
datasets the nanoGPT pages train on (tinyshakespeare, OpenWebText, the
names list), which are not available here.  It contains none of the
training step's arithmetic and imports neither the CUDA library nor the
oracle.

Streams are i.i.d. Zipf(s) over the vocabulary (p_k proportional to
k^-s for rank k = 1..V, token id k - 1), drawn by inverse CDF from a
numpy PCG64 generator; the microGPT-sized case uses uniform ids.
"""

from __future__ import annotations

from dataclasses import dataclass, asdict
from typing import Dict

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    vocab_size: int
    n_layer: int
    n_head: int
    n_embd: int
    block_size: int
    batch_size: int
    grad_accum: int
    precision: str          # "fp32" or "bf16"
    variant: str            # "gpt2" or "micro"
    init_std: float
    dropout: float
    lr: float
    beta1: float
    beta2: float
    eps: float
    weight_decay: float
    grad_clip: float
    token_dtype: str        # "int32" or "uint16"
    zipf_s: float           # 0 -> uniform ids
    stream_len: int
    stream_seed: int = 1337
    data_seed: int = 1338
    weight_seed: int = 1337
    dropout_seed: int = 1339
    warmup: int = 2
    max_iters: int = 10

    def as_dict(self) -> Dict:
        return asdict(self)

    def with_(self, **kw) -> "Workload":
        d = asdict(self)
        d.update(kw)
        return Workload(**d)

    @property
    def tokens_per_step(self) -> int:
        return self.batch_size * self.block_size * self.grad_accum


# microGPT-sized model, one fp32 step (vocab 27, 1 layer, 4 heads, d 16, block 16, batch 8).
MICRO = Workload("micro_fp32", 27, 1, 4, 16, 16, 8, 1, "fp32", "micro", 0.08, 0.0,
                 1e-2, 0.85, 0.99, 1e-8, 0.0, 0.0, "int32", 0.0, 1 << 16)
# char-level Shakespeare-shaped model (vocab 65, 6 layers, 6 heads, d 384, block 256, batch 64).
CHAR = Workload("char_bf16", 65, 6, 6, 384, 256, 64, 1, "bf16", "gpt2", 0.02, 0.0,
                1e-3, 0.9, 0.99, 1e-8, 0.1, 1.0, "int32", 1.2, 1 << 20)
# GPT-2 124M (vocab 50257, 12 layers, 12 heads, d 768, block 1024, micro-batch 12, grad-accum 5).
GPT2_124M = Workload("gpt2_124m_bf16", 50257, 12, 12, 768, 1024, 12, 5, "bf16", "gpt2", 0.02, 0.0,
                     6e-4, 0.9, 0.95, 1e-8, 0.1, 1.0, "uint16", 1.1, 1 << 25)
# 12 layers, 8 heads, d 512, block 512, batch 12, dropout 0.1.
DROPOUT_512 = Workload("gpt_12l_512d_dropout_bf16", 50257, 12, 8, 512, 512, 12, 1, "bf16", "gpt2", 0.02, 0.1,
                       6e-4, 0.9, 0.95, 1e-8, 0.1, 1.0, "uint16", 1.1, 1 << 25)
# GPT-2 XL 1558M (vocab 50257, 48 layers, 25 heads, d 1600, block 1024, micro-batch 8).
GPT2_XL = Workload("gpt2_xl_1558m_bf16", 50257, 48, 25, 1600, 1024, 8, 1, "bf16", "gpt2", 0.02, 0.0,
                   6e-5, 0.9, 0.95, 1e-8, 0.1, 1.0, "uint16", 1.1, 1 << 25)

ALL = {w.name: w for w in (MICRO, CHAR, GPT2_124M, DROPOUT_512, GPT2_XL)}


def token_stream(w: Workload, n: int | None = None, seed: int | None = None) -> np.ndarray:
    """The seeded synthetic token stream of workload ``w`` (host array)."""
    n = w.stream_len if n is None else n
    rng = np.random.default_rng(w.stream_seed if seed is None else seed)
    V = w.vocab_size
    if w.zipf_s <= 0:
        ids = rng.integers(0, V, size=n, dtype=np.int64)
    else:
        ranks = np.arange(1, V + 1, dtype=np.float64)
        p = ranks ** (-w.zipf_s)
        cdf = np.cumsum(p)
        cdf /= cdf[-1]
        ids = np.searchsorted(cdf, rng.random(n), side="right")
        ids = np.minimum(ids, V - 1)
    dt = np.uint16 if w.token_dtype == "uint16" else np.int32
    return ids.astype(dt)


def random_batch(w: Workload, seed: int, batch_size: int | None = None, block_size: int | None = None):
    """An (idx, tgt) pair of int32 [B, T] arrays drawn directly from the stream law."""
    B = w.batch_size if batch_size is None else batch_size
    T = w.block_size if block_size is None else block_size
    s = token_stream(w, n=B * (T + 1), seed=seed).astype(np.int32).reshape(B, T + 1)
    return np.ascontiguousarray(s[:, :T]), np.ascontiguousarray(s[:, 1:])
