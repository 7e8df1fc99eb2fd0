"""Float64 oracle of a LoRA fine-tuning step for the GPT-2 model of gpt_oracle.

TEST INFRASTRUCTURE ONLY (tests and the smoke check).  The product library
never imports it, and it imports nothing from the product package.

Source: "使用 nanoGPT 构建中型 GPT 微调管道：自定义 PyTorch 循环、LoRA 集成与
多 GPU 分布式训练" (blog.hotdry.top), the paragraph on LoRA integration: the
pretrained weight W0 stays frozen and a low-rank update B A (rank r much
smaller than the matrix sides, typically 8-64) is trained in its place, so a
layer computes h = W0 x + B A x; lora_alpha = 16 is the scaling factor; the
adapted modules are the query and value projections; only the LoRA matrices
are optimised; at inference B A can be merged into W0.

Readings where the page is silent (also listed in the design notes):

* The scaling is s = lora_alpha / r, applied to the low-rank branch:
  h = W0 x + s * B (A x), with A [r, d_in] and B [d_out, r].
* nanoGPT fuses Q, K and V into one projection (c_attn, rows 0..d-1 for q,
  d..2d-1 for k, 2d..3d-1 for v); "q_proj" and "v_proj" are those row blocks.
* B starts at zero, so the adapted model starts as the base model; A is
  drawn by the caller (here: any seeded values).
* Every base tensor is frozen (embeddings, norms and biases included).  The
  optimiser is the base step's clip + AdamW with its hyper-parameters, over
  the LoRA tensors only: the global-norm clip sees only their gradients, and
  both LoRA matrices are 2-D, so weight decay applies to them.
* The page's "dropout=0.1" is the model's own dropout (the sites of the
  base model); there is no separate dropout on the low-rank branch.

Because h = (W0 + s B A) x exactly, the adapted model is the base model with
the merged weight W0 + s B A in the q and v row blocks.  The oracle uses that
identity as its definition of the forward, and the chain rule through it for
the gradients: with G = dL/dW of the merged block,
dL/dB = s G A^T and dL/dA = s B^T G.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np

from . import gpt_oracle as O

TARGET_ROWS = {"q": 0, "k": 1, "v": 2}  # row block of c_attn (times n_embd)


@dataclass
class LoraConfig:
    r: int = 8
    alpha: float = 16.0
    targets: Tuple[str, ...] = ("q", "v")

    @property
    def scale(self) -> float:
        return self.alpha / self.r


def lora_names(cfg: O.Config, lc: LoraConfig):
    """(layer, target, name of A, name of B) of every adapted block."""
    out = []
    for l in range(cfg.n_layer):
        for t in lc.targets:
            out.append((l, t, f"h.{l}.attn.lora_{t}.A", f"h.{l}.attn.lora_{t}.B"))
    return out


def lora_param_count(cfg: O.Config, lc: LoraConfig) -> int:
    """Trainable parameters: per adapted block r*d (A) + d*r (B)."""
    return sum(2 * lc.r * cfg.n_embd for _ in lora_names(cfg, lc))


def init_lora(cfg: O.Config, lc: LoraConfig, seed: int, a_std: Optional[float] = None,
              b_std: float = 0.0) -> Dict[str, np.ndarray]:
    """A ~ N(0, a_std^2) (default 1/sqrt(d)), B ~ N(0, b_std^2) (default 0:
    the adapted model starts as the base model)."""
    rng = np.random.default_rng(seed)
    d = cfg.n_embd
    a_std = 1.0 / np.sqrt(d) if a_std is None else a_std
    Lp = {}
    for _, _, na, nb in lora_names(cfg, lc):
        Lp[na] = rng.standard_normal((lc.r, d)) * a_std
        Lp[nb] = rng.standard_normal((d, lc.r)) * b_std if b_std > 0 else np.zeros((d, lc.r))
    return Lp


def _block(l: int, t: str, d: int):
    rb = TARGET_ROWS[t] * d
    return f"h.{l}.attn.c_attn.weight", slice(rb, rb + d)


def merged_params(cfg: O.Config, P: Dict[str, np.ndarray], Lp: Dict[str, np.ndarray],
                  lc: LoraConfig) -> Dict[str, np.ndarray]:
    """The base parameters with W0 + s B A in every adapted row block."""
    M = {k: v for k, v in P.items()}
    d = cfg.n_embd
    for l, t, na, nb in lora_names(cfg, lc):
        name, rows = _block(l, t, d)
        if M[name] is P[name]:
            M[name] = P[name].copy()
        M[name][rows] += lc.scale * (Lp[nb] @ Lp[na])
    return M


def loss_and_grads(cfg: O.Config, P, Lp, lc: LoraConfig, idx, tgt, drop: Optional[O.DropCtx] = None,
                   loss_scale: float = 1.0):
    """Loss of one micro-batch and the gradients of loss_scale * loss with
    respect to the LoRA tensors (the base tensors are frozen)."""
    Pm = merged_params(cfg, P, Lp, lc)
    loss, G, cache = O.loss_and_grads(cfg, Pm, idx, tgt, drop, loss_scale)
    d = cfg.n_embd
    GL = {}
    for l, t, na, nb in lora_names(cfg, lc):
        name, rows = _block(l, t, d)
        Gb = G[name][rows]                       # dL/d(merged block) [d, d]
        GL[nb] = lc.scale * Gb @ Lp[na].T        # [d, r]
        GL[na] = lc.scale * Lp[nb].T @ Gb        # [r, d]
    return loss, GL, cache


@dataclass
class LoraAdamState:
    m: Dict[str, np.ndarray] = field(default_factory=dict)
    v: Dict[str, np.ndarray] = field(default_factory=dict)


def clip_adamw(cfg: O.Config, Lp: Dict[str, np.ndarray], GL: Dict[str, np.ndarray], S: LoraAdamState,
               lr: float, step: int) -> float:
    """The base step's clip + AdamW (run log section 2.1 hyper-parameters)
    over the LoRA tensors only; every LoRA tensor is 2-D, hence decayed."""
    norm = O.global_grad_norm(GL)
    c = 1.0
    if cfg.grad_clip > 0:
        c = min(1.0, cfg.grad_clip / (norm + 1e-6))
    b1, b2 = cfg.beta1, cfg.beta2
    bc1 = 1.0 - b1 ** step
    bc2 = 1.0 - b2 ** step
    for name, w in Lp.items():
        g = GL[name] * c
        if name not in S.m:
            S.m[name] = np.zeros_like(w)
            S.v[name] = np.zeros_like(w)
        if cfg.weight_decay != 0.0:
            w *= (1.0 - lr * cfg.weight_decay)
        S.m[name] = b1 * S.m[name] + (1.0 - b1) * g
        S.v[name] = b2 * S.v[name] + (1.0 - b2) * g * g
        w -= lr * (S.m[name] / bc1) / (np.sqrt(S.v[name] / bc2) + cfg.eps)
    return norm


def train_step(cfg: O.Config, P, Lp, lc: LoraConfig, S: LoraAdamState, stream: np.ndarray, data_seed: int,
               lr: float, step: int):
    """grad_accum micro-batches of the base step's batch gather and dropout,
    LoRA gradients summed (each loss divided by grad_accum), then clip +
    AdamW on the LoRA tensors.  P is not modified.  Returns (mean loss,
    LoRA gradient norm before clipping)."""
    GL = None
    losses = []
    for mu in range(cfg.grad_accum):
        idx, tgt = O.gather_batch(stream, cfg.block_size, data_seed, step, mu, cfg.batch_size)
        drop = O.DropCtx(cfg.dropout_seed, step * cfg.grad_accum + mu) if cfg.dropout > 0 else None
        loss, g, _ = loss_and_grads(cfg, P, Lp, lc, idx, tgt, drop, 1.0 / cfg.grad_accum)
        losses.append(loss)
        if GL is None:
            GL = g
        else:
            for k in GL:
                GL[k] += g[k]
    norm = clip_adamw(cfg, Lp, GL, S, lr, step)
    return float(np.mean(losses)), norm
