"""Float64 oracle of one nanoGPT-style GPT-2 causal-LM training step.

TEST INFRASTRUCTURE ONLY (tests, the smoke check and the bench's CPU
baseline).  The product library never imports it, and it imports nothing
from the product package.

Sources (the web pages this method is taken from; section names are the
pages' own):

* "nanoGPT README" (translated, oa0.com) -- model.py/train.py structure,
  GPT-2 124M reproduction, section "复现 GPT-2".
* "从零实现GPT训练与推理：基于nanoGPT的实战指南" (adg.csdn.net) -- section 6
  "性能优化技巧" prints ``get_lr`` (warmup + cosine), bf16 and grad accumulation.
* "nanoGPT run log" (wmrh.cn) -- section 1.3 (train.bin windows of block_size),
  section 2.1 (config table: beta1 0.9, beta2 0.95, weight decay 0.1, dropout),
  section 2.2 (head_dim = n_embd / n_head), section 2.3 (parameter count made of
  token embedding, attention 4d^2, MLP, layer norms), section 3.1 (gradient
  accumulation sums micro-batch gradients), section 3.3 (initial loss near
  ln(vocab)), section 4.5 (fixed seeds).
* "微型 GPT 从零构建：核心训练循环、分词与单 GPU 高效推理" (blog.hotdry.top),
  section "模型核心" (embedding + position embedding, blocks of
  attention + MLP, RMSNorm without bias, ReLU in place of GeLU, 4192
  parameters at embd 16 / head 4, Gaussian(0, 0.08) init) and section
  "核心训练循环" (loss = mean of -log p(target); backward by the chain rule;
  Adam beta1 0.85, beta2 0.99, eps 1e-8; lr decays linearly to 0;
  clip_grad 1.0).

Readings taken where the pages are silent (each one is also listed in the
design notes of the repository):

* LayerNorm: biased variance, eps 1e-5, weight 1 / bias 0 at init.
* RMSNorm (micro variant): y = x / sqrt(mean(x^2) + 1e-5), no parameters,
  placed where the GPT-2 variant has its LayerNorms (ln_1, ln_2, ln_f).
* GELU is the exact erf form x * Phi(x).
* Loss: mean over all B*T positions; with grad accumulation each
  micro-batch loss is divided by the number of micro-batches.
* Clip: global L2 norm over all gradients, coefficient
  min(1, clip / (norm + 1e-6)); off when clip <= 0.
* AdamW: decoupled decay w <- w * (1 - lr * wd) before the Adam update,
  applied to tensors with two or more dimensions only unless ``decay_1d``.
* Random numbers (weight init, batch offsets, dropout masks) come from the
  SplitMix64 generator of Steele, Lea and Flood (2014), used as a
  counter-based hash; Gaussians by the Box-Muller transform (1958).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional, Tuple

import numpy as np

try:  # the erf used by the exact GELU; scipy is a plain library routine
    from scipy.special import erf as _erf
except Exception:  # pragma: no cover - scipy is in the image
    _erf = np.vectorize(math.erf)

__all__ = [
    "Config", "TensorSpec", "tensor_specs", "param_count", "param_count_closed_form",
    "sm64", "init_tensor", "init_params", "batch_offsets", "gather_batch",
    "dropout_keep", "attention_fwd", "attention_bwd", "forward", "backward", "loss_and_grads", "global_grad_norm",
    "clip_adamw", "AdamState", "train_step", "lr_cosine", "lr_linear", "argmax_rows",
]

# --------------------------------------------------------------------------
# configuration and parameter layout
# --------------------------------------------------------------------------


@dataclass
class Config:
    """Hyper-parameters of one model and its optimiser.

    Names follow the nanoGPT config files quoted in the practical guide's
    section 3 (n_layer, n_head, n_embd, block_size, batch_size) and the run
    log's section 2.1 table (dropout, learning rate, weight decay, betas).
    """

    vocab_size: int
    n_layer: int
    n_head: int
    n_embd: int
    block_size: int
    batch_size: int = 1
    grad_accum: int = 1
    variant: str = "gpt2"          # "gpt2" (LayerNorm, biases, GELU, tied) or "micro"
    init_std: float = 0.02
    dropout: float = 0.0
    beta1: float = 0.9
    beta2: float = 0.95
    eps: float = 1e-8
    weight_decay: float = 0.1
    grad_clip: float = 1.0
    decay_1d: bool = False
    dropout_seed: int = 0
    norm_eps: float = 1e-5

    @property
    def head_dim(self) -> int:
        # run log section 2.2: each head has n_embd / n_head dimensions
        return self.n_embd // self.n_head

    def with_(self, **kw) -> "Config":
        return replace(self, **kw)


@dataclass
class TensorSpec:
    name: str
    shape: Tuple[int, ...]
    init: str  # "normal", "ones" or "zeros"

    @property
    def decayed_by_default(self) -> bool:
        return len(self.shape) >= 2


def tensor_specs(cfg: Config) -> List[TensorSpec]:
    """The model's tensors in their canonical order.

    The order fixes the tensor index used by the weight-init generator.
    gpt2 variant: token and position embeddings, per block ln_1, the fused
    QKV projection (c_attn), the attention output projection (c_proj),
    ln_2, the 4x MLP (c_fc, c_proj), then ln_f; the lm_head is tied to wte.
    micro variant (microGPT, section "模型核心"): no biases, no norm
    parameters, untied lm_head at the end.
    """
    V, d, T, L = cfg.vocab_size, cfg.n_embd, cfg.block_size, cfg.n_layer
    gpt2 = cfg.variant == "gpt2"
    s = [TensorSpec("wte", (V, d), "normal"), TensorSpec("wpe", (T, d), "normal")]
    for l in range(L):
        p = f"h.{l}."
        if gpt2:
            s += [TensorSpec(p + "ln_1.weight", (d,), "ones"), TensorSpec(p + "ln_1.bias", (d,), "zeros")]
        s.append(TensorSpec(p + "attn.c_attn.weight", (3 * d, d), "normal"))
        if gpt2:
            s.append(TensorSpec(p + "attn.c_attn.bias", (3 * d,), "zeros"))
        s.append(TensorSpec(p + "attn.c_proj.weight", (d, d), "normal"))
        if gpt2:
            s.append(TensorSpec(p + "attn.c_proj.bias", (d,), "zeros"))
            s += [TensorSpec(p + "ln_2.weight", (d,), "ones"), TensorSpec(p + "ln_2.bias", (d,), "zeros")]
        s.append(TensorSpec(p + "mlp.c_fc.weight", (4 * d, d), "normal"))
        if gpt2:
            s.append(TensorSpec(p + "mlp.c_fc.bias", (4 * d,), "zeros"))
        s.append(TensorSpec(p + "mlp.c_proj.weight", (d, 4 * d), "normal"))
        if gpt2:
            s.append(TensorSpec(p + "mlp.c_proj.bias", (d,), "zeros"))
    if gpt2:
        s += [TensorSpec("ln_f.weight", (d,), "ones"), TensorSpec("ln_f.bias", (d,), "zeros")]
    else:
        s.append(TensorSpec("lm_head.weight", (V, d), "normal"))
    return s


def param_count(cfg: Config) -> int:
    """Sum of tensor sizes (what nanoGPT prints as 'number of parameters')."""
    return int(sum(int(np.prod(t.shape)) for t in tensor_specs(cfg)))


def param_count_closed_form(cfg: Config) -> int:
    """Closed form of the parameter count.

    Run log section 2.3 breaks the count into the token embedding
    (vocab * d), the attention (4 d^2 weights) and the MLP per layer and the
    layer norms.  Written out for the gpt2 variant with biases:
    V d + T d + L (12 d^2 + 13 d) + 2 d.  The micro variant (no biases, no
    norm parameters, untied head) is 2 V d + T d + 12 L d^2, which gives the
    4192 of the microGPT page at vocab 27, d 16, block 16, one layer.
    """
    V, d, T, L = cfg.vocab_size, cfg.n_embd, cfg.block_size, cfg.n_layer
    if cfg.variant == "gpt2":
        return V * d + T * d + L * (12 * d * d + 13 * d) + 2 * d
    return 2 * V * d + T * d + 12 * L * d * d


# --------------------------------------------------------------------------
# SplitMix64 as a counter-based generator (Steele, Lea & Flood 2014)
# --------------------------------------------------------------------------

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)


def sm64(x) -> np.ndarray:
    """SplitMix64 output for generator state ``x`` (before its increment).

    The generator adds the golden-ratio gamma to its state and passes the
    result through the variant-13 mixer: xor-shift 30, multiply, xor-shift
    27, multiply, xor-shift 31 (all modulo 2^64).
    """
    with np.errstate(over="ignore"):
        z = np.asarray(x, dtype=np.uint64) + _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _MIX1
        z = (z ^ (z >> np.uint64(27))) * _MIX2
        return z ^ (z >> np.uint64(31))


def _u64(v: int) -> np.ndarray:
    return np.asarray(v & 0xFFFFFFFFFFFFFFFF, dtype=np.uint64)


def init_tensor(cfg: Config, seed: int, index: int, spec: TensorSpec) -> np.ndarray:
    """Initial values of tensor number ``index`` (fp32-rounded, held in fp64).

    microGPT page, section "模型核心": weights ~ Gaussian(0, std) with std
    0.08 for the tiny model and 0.02-0.1 by size; biases start at 0 and norm
    gains at 1.  Element e of the tensor (row-major) draws two 64-bit words
    from key k = sm64(seed ^ sm64(index)):  b1 = sm64(k ^ 2e),
    b2 = sm64(k ^ (2e + 1)); u1 = ((b1 >> 11) + 1) / 2^53 in (0, 1],
    u2 = (b2 >> 11) / 2^53 in [0, 1); z = sqrt(-2 ln u1) cos(2 pi u2).
    """
    n = int(np.prod(spec.shape))
    if spec.init == "ones":
        return np.ones(spec.shape)
    if spec.init == "zeros":
        return np.zeros(spec.shape)
    k = sm64(_u64(seed) ^ sm64(_u64(index)))
    e2 = np.arange(n, dtype=np.uint64) * np.uint64(2)
    b1 = sm64(k ^ e2)
    b2 = sm64(k ^ (e2 + np.uint64(1)))
    u1 = ((b1 >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (b2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    w = (cfg.init_std * z).astype(np.float32).astype(np.float64)
    return w.reshape(spec.shape)


def init_params(cfg: Config, seed: int) -> Dict[str, np.ndarray]:
    return {t.name: init_tensor(cfg, seed, i, t) for i, t in enumerate(tensor_specs(cfg))}


# --------------------------------------------------------------------------
# get_batch: random windows of the token stream
# --------------------------------------------------------------------------


def batch_offsets(n_stream: int, block_size: int, data_seed: int, step: int, micro: int,
                  batch_size: int) -> np.ndarray:
    """Window starts for one micro-batch.

    Run log section 1.3 / README: train.bin is a flat token stream and a
    batch is batch_size random windows of block_size tokens; the target is
    the window shifted by one (practical guide / microGPT "核心训练循环":
    predict the next token).  Start b of micro-batch (step, micro) is
    sm64(data_seed ^ sm64(step << 40 ^ micro << 20 ^ b)) mod (n_stream - block_size),
    so that the last target index is at most n_stream - 1.
    """
    b = np.arange(batch_size, dtype=np.uint64)
    key = (_u64(step) << np.uint64(40)) ^ (_u64(micro) << np.uint64(20)) ^ b
    r = sm64(_u64(data_seed) ^ sm64(key))
    return (r % np.uint64(n_stream - block_size)).astype(np.int64)


def gather_batch(stream: np.ndarray, block_size: int, data_seed: int, step: int, micro: int,
                 batch_size: int) -> Tuple[np.ndarray, np.ndarray]:
    ix = batch_offsets(len(stream), block_size, data_seed, step, micro, batch_size)
    rows = ix[:, None] + np.arange(block_size)[None, :]
    s = np.asarray(stream).astype(np.int64)
    return s[rows], s[rows + 1]


# --------------------------------------------------------------------------
# dropout mask (counter hash)
# --------------------------------------------------------------------------


def dropout_keep(seed: int, counter: int, layer: int, site: int, elems: np.ndarray, p: float) -> np.ndarray:
    """Inverted-dropout keep mask.

    The run log (section 2.1/2.2) turns dropout 0.1 on; the pages do not say
    where, so the GPT-2 sites are used: 0 = embedding output (layer index =
    n_layer), 1 = attention probabilities, 2 = attention projection output,
    3 = MLP projection output.  counter = step * grad_accum + micro.
    keep iff (sm64(k ^ elem) >> 32) >= floor(p * 2^32) with
    k = sm64(seed ^ sm64(counter << 32 ^ layer << 8 ^ site)).
    """
    thr = np.uint64(int(math.floor(p * 4294967296.0)))
    tag = (_u64(counter) << np.uint64(32)) ^ (_u64(layer) << np.uint64(8)) ^ _u64(site)
    k = sm64(_u64(seed) ^ sm64(tag))
    u = sm64(k ^ np.asarray(elems, dtype=np.uint64)) >> np.uint64(32)
    return u >= thr


# --------------------------------------------------------------------------
# forward
# --------------------------------------------------------------------------


def _norm_fwd(cfg: Config, x: np.ndarray, w: Optional[np.ndarray], b: Optional[np.ndarray]):
    """LayerNorm (gpt2) or parameter-free RMSNorm (micro) over the last axis."""
    if cfg.variant == "gpt2":
        mu = x.mean(axis=-1, keepdims=True)
        var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)   # biased variance
        rstd = 1.0 / np.sqrt(var + cfg.norm_eps)
        xhat = (x - mu) * rstd
        return xhat * w + b, (xhat, rstd)
    ms = (x * x).mean(axis=-1, keepdims=True)
    r = 1.0 / np.sqrt(ms + cfg.norm_eps)
    return x * r, (x, r)


def _norm_bwd(cfg: Config, dy: np.ndarray, cache, w: Optional[np.ndarray]):
    """Returns (dx, dw, db); dw/db are None for RMSNorm."""
    if cfg.variant == "gpt2":
        xhat, rstd = cache
        dw = (dy * xhat).reshape(-1, dy.shape[-1]).sum(axis=0)
        db = dy.reshape(-1, dy.shape[-1]).sum(axis=0)
        g = dy * w
        dx = rstd * (g - g.mean(axis=-1, keepdims=True) - xhat * (g * xhat).mean(axis=-1, keepdims=True))
        return dx, dw, db
    x, r = cache
    dx = r * dy - (r ** 3) * x * (dy * x).mean(axis=-1, keepdims=True)
    return dx, None, None


def _act_fwd(cfg: Config, h: np.ndarray) -> np.ndarray:
    if cfg.variant == "gpt2":
        return h * 0.5 * (1.0 + _erf(h / math.sqrt(2.0)))      # x * Phi(x)
    return np.maximum(h, 0.0)                                   # microGPT: ReLU


def _act_bwd(cfg: Config, h: np.ndarray) -> np.ndarray:
    if cfg.variant == "gpt2":
        phi = np.exp(-0.5 * h * h) / math.sqrt(2.0 * math.pi)
        return 0.5 * (1.0 + _erf(h / math.sqrt(2.0))) + h * phi
    return (h > 0.0).astype(np.float64)


def _logsumexp_rows(z: np.ndarray) -> np.ndarray:
    m = z.max(axis=-1, keepdims=True)
    return (m + np.log(np.exp(z - m).sum(axis=-1, keepdims=True)))[..., 0]


@dataclass
class DropCtx:
    seed: int
    counter: int


def attention_fwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, keep: Optional[np.ndarray] = None,
                  p_drop: float = 0.0):
    """Causal scaled dot-product attention of [B, H, T, hd] inputs (README /
    microGPT "模型核心": scores q k^T / sqrt(head_dim), future keys masked,
    softmax, weighted sum of V).  Dropout (``keep`` mask, [B, H, T, T]) acts
    on the probabilities.  Returns (o, p, lse) with lse the natural-log
    log-sum-exp of each row of scaled scores."""
    T, hd = q.shape[-2], q.shape[-1]
    s = (q @ k.transpose(0, 1, 3, 2)) / math.sqrt(hd)
    causal = np.tril(np.ones((T, T), dtype=bool))
    s = np.where(causal, s, -np.inf)
    mx = s.max(axis=-1, keepdims=True)
    e = np.exp(s - mx)
    z = e.sum(axis=-1, keepdims=True)
    pr = e / z
    lse = (mx + np.log(z))[..., 0]
    pd = pr * keep / (1.0 - p_drop) if keep is not None else pr
    return pd @ v, pr, lse


def attention_bwd(q, k, v, pr, do, keep: Optional[np.ndarray] = None, p_drop: float = 0.0):
    """Gradients (dq, dk, dv) of attention_fwd: dV = P~^T dO, dP = dO V^T
    (times the dropout mask), dS = P * (dP - rowsum(dP * P)),
    dQ = dS K / sqrt(hd), dK = dS^T Q / sqrt(hd)."""
    hd = q.shape[-1]
    inv_keep = 1.0 / (1.0 - p_drop) if keep is not None else 1.0
    pd = pr * keep * inv_keep if keep is not None else pr
    dv = pd.transpose(0, 1, 3, 2) @ do
    dpd = do @ v.transpose(0, 1, 3, 2)
    dp = dpd * keep * inv_keep if keep is not None else dpd
    ds = pr * (dp - (dp * pr).sum(axis=-1, keepdims=True))
    dq = (ds @ k) / math.sqrt(hd)
    dk = (ds.transpose(0, 1, 3, 2) @ q) / math.sqrt(hd)
    return dq, dk, dv


def forward(cfg: Config, P: Dict[str, np.ndarray], idx: np.ndarray, tgt: Optional[np.ndarray],
            drop: Optional[DropCtx] = None, keep_cache: bool = True):
    """Loss of one micro-batch (mean over its B*T positions) and the cache.

    Structure per the README / practical guide (model.py) and the microGPT
    page ("模型核心"): x = wte[idx] + wpe[pos]; per block
    x += attn(norm_1(x)); x += mlp(norm_2(x)); z = norm_f(x) @ W_head^T.
    Attention: QKV projection, scores q k^T / sqrt(head_dim) with future
    positions masked, softmax, weighted sum of V, output projection.
    MLP: fc (4 d) -> GELU (ReLU in micro) -> proj.
    Loss (microGPT "核心训练循环"): mean of -log softmax(z)[target].
    """
    B, T = idx.shape
    d, H, L = cfg.n_embd, cfg.n_head, cfg.n_layer
    hd = d // H
    gpt2 = cfg.variant == "gpt2"
    p_drop = cfg.dropout if drop is not None else 0.0
    inv_keep = 1.0 / (1.0 - p_drop) if p_drop > 0 else 1.0
    cache = {"idx": idx, "tgt": tgt, "B": B, "T": T, "drop": drop, "layers": []}

    def _mask(layer: int, site: int, shape) -> Optional[np.ndarray]:
        if p_drop <= 0:
            return None
        n = int(np.prod(shape))
        return dropout_keep(drop.seed, drop.counter, layer, site, np.arange(n, dtype=np.uint64), p_drop).reshape(shape)

    x = P["wte"][idx] + P["wpe"][:T][None, :, :]
    m0 = _mask(L, 0, x.shape)
    if m0 is not None:
        x = x * m0 * inv_keep
    cache["m0"] = m0
    for l in range(L):
        pre = f"h.{l}."
        lc = {"x_in": x}
        a, lc["n1"] = _norm_fwd(cfg, x, P.get(pre + "ln_1.weight"), P.get(pre + "ln_1.bias"))
        qkv = a @ P[pre + "attn.c_attn.weight"].T
        if gpt2:
            qkv = qkv + P[pre + "attn.c_attn.bias"]
        q, k, v = np.split(qkv, 3, axis=-1)
        q = q.reshape(B, T, H, hd).transpose(0, 2, 1, 3)
        k = k.reshape(B, T, H, hd).transpose(0, 2, 1, 3)
        v = v.reshape(B, T, H, hd).transpose(0, 2, 1, 3)
        m1 = _mask(l, 1, (B, H, T, T))
        o, pr, _ = attention_fwd(q, k, v, m1, p_drop)
        o = o.transpose(0, 2, 1, 3).reshape(B, T, d)
        y = o @ P[pre + "attn.c_proj.weight"].T
        if gpt2:
            y = y + P[pre + "attn.c_proj.bias"]
        m2 = _mask(l, 2, y.shape)
        if m2 is not None:
            y = y * m2 * inv_keep
        x = x + y
        lc.update(a=a, q=q, k=k, v=v, p=pr, m1=m1, o=o, m2=m2, x_mid=x)
        a2, lc["n2"] = _norm_fwd(cfg, x, P.get(pre + "ln_2.weight"), P.get(pre + "ln_2.bias"))
        h = a2 @ P[pre + "mlp.c_fc.weight"].T
        if gpt2:
            h = h + P[pre + "mlp.c_fc.bias"]
        g = _act_fwd(cfg, h)
        y = g @ P[pre + "mlp.c_proj.weight"].T
        if gpt2:
            y = y + P[pre + "mlp.c_proj.bias"]
        m3 = _mask(l, 3, y.shape)
        if m3 is not None:
            y = y * m3 * inv_keep
        x = x + y
        lc.update(a2=a2, h=h, g=g, m3=m3)
        cache["layers"].append(lc)
    xf, cache["nf"] = _norm_fwd(cfg, x, P.get("ln_f.weight"), P.get("ln_f.bias"))
    w_head = P["wte"] if gpt2 else P["lm_head.weight"]
    z = xf @ w_head.T                                       # [B, T, V]
    cache.update(xf=xf, z=z)
    if tgt is None:
        return None, cache
    lse = _logsumexp_rows(z)
    zt = np.take_along_axis(z, tgt[..., None], axis=-1)[..., 0]
    loss = float((lse - zt).mean())
    cache["lse"] = lse
    if not keep_cache:
        cache = {"z": z, "lse": lse}
    return loss, cache


# --------------------------------------------------------------------------
# backward
# --------------------------------------------------------------------------


def backward(cfg: Config, P: Dict[str, np.ndarray], cache, loss_scale: float = 1.0) -> Dict[str, np.ndarray]:
    """Gradients of loss_scale * loss, by the chain rule written out per op.

    microGPT "核心训练循环": backward walks the graph in reverse; here every
    op's derivative is written by hand.  Cross-entropy: dz = softmax(z) -
    onehot(target), divided by the number of positions.  Attention:
    dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dP * P)),
    dQ = dS K / sqrt(hd), dK = dS^T Q / sqrt(hd).
    """
    B, T = cache["B"], cache["T"]
    d, H, L = cfg.n_embd, cfg.n_head, cfg.n_layer
    hd = d // H
    gpt2 = cfg.variant == "gpt2"
    drop = cache["drop"]
    p_drop = cfg.dropout if drop is not None else 0.0
    inv_keep = 1.0 / (1.0 - p_drop) if p_drop > 0 else 1.0
    G = {t.name: np.zeros(t.shape) for t in tensor_specs(cfg)}
    z, tgt, idx = cache["z"], cache["tgt"], cache["idx"]
    M = B * T
    pz = np.exp(z - cache["lse"][..., None])
    dz = pz
    np.put_along_axis(dz, tgt[..., None], np.take_along_axis(dz, tgt[..., None], axis=-1) - 1.0, axis=-1)
    dz = dz * (loss_scale / M)
    w_head = P["wte"] if gpt2 else P["lm_head.weight"]
    dxf = dz @ w_head
    dw_head = dz.reshape(M, -1).T @ cache["xf"].reshape(M, d)
    if gpt2:
        G["wte"] += dw_head
    else:
        G["lm_head.weight"] += dw_head
    dx, dw, db = _norm_bwd(cfg, dxf, cache["nf"], P.get("ln_f.weight"))
    if gpt2:
        G["ln_f.weight"] += dw
        G["ln_f.bias"] += db
    for l in reversed(range(L)):
        pre = f"h.{l}."
        lc = cache["layers"][l]
        # MLP
        dy = dx if lc["m3"] is None else dx * lc["m3"] * inv_keep
        if gpt2:
            G[pre + "mlp.c_proj.bias"] += dy.reshape(M, d).sum(axis=0)
        G[pre + "mlp.c_proj.weight"] += dy.reshape(M, d).T @ lc["g"].reshape(M, 4 * d)
        dg = dy @ P[pre + "mlp.c_proj.weight"]
        dh = dg * _act_bwd(cfg, lc["h"])
        if gpt2:
            G[pre + "mlp.c_fc.bias"] += dh.reshape(M, 4 * d).sum(axis=0)
        G[pre + "mlp.c_fc.weight"] += dh.reshape(M, 4 * d).T @ lc["a2"].reshape(M, d)
        da2 = dh @ P[pre + "mlp.c_fc.weight"]
        dxn, dw, db = _norm_bwd(cfg, da2, lc["n2"], P.get(pre + "ln_2.weight"))
        if gpt2:
            G[pre + "ln_2.weight"] += dw
            G[pre + "ln_2.bias"] += db
        dx = dx + dxn
        # attention
        dy = dx if lc["m2"] is None else dx * lc["m2"] * inv_keep
        if gpt2:
            G[pre + "attn.c_proj.bias"] += dy.reshape(M, d).sum(axis=0)
        G[pre + "attn.c_proj.weight"] += dy.reshape(M, d).T @ lc["o"].reshape(M, d)
        do = (dy @ P[pre + "attn.c_proj.weight"]).reshape(B, T, H, hd).transpose(0, 2, 1, 3)
        q, k, v, pr, m1 = lc["q"], lc["k"], lc["v"], lc["p"], lc["m1"]
        dq, dk, dv = attention_bwd(q, k, v, pr, do, m1, p_drop)
        dqkv = np.concatenate([t.transpose(0, 2, 1, 3).reshape(B, T, d) for t in (dq, dk, dv)], axis=-1)
        if gpt2:
            G[pre + "attn.c_attn.bias"] += dqkv.reshape(M, 3 * d).sum(axis=0)
        G[pre + "attn.c_attn.weight"] += dqkv.reshape(M, 3 * d).T @ lc["a"].reshape(M, d)
        da = dqkv @ P[pre + "attn.c_attn.weight"]
        dxn, dw, db = _norm_bwd(cfg, da, lc["n1"], P.get(pre + "ln_1.weight"))
        if gpt2:
            G[pre + "ln_1.weight"] += dw
            G[pre + "ln_1.bias"] += db
        dx = dx + dxn
    if cache["m0"] is not None:
        dx = dx * cache["m0"] * inv_keep
    np.add.at(G["wte"], idx.reshape(-1), dx.reshape(M, d))
    G["wpe"][:T] += dx.sum(axis=0)
    return G


def loss_and_grads(cfg: Config, P, idx, tgt, drop: Optional[DropCtx] = None, loss_scale: float = 1.0):
    loss, cache = forward(cfg, P, idx, tgt, drop)
    return loss, backward(cfg, P, cache, loss_scale), cache


# --------------------------------------------------------------------------
# clip + AdamW, learning-rate schedules
# --------------------------------------------------------------------------


def global_grad_norm(G: Dict[str, np.ndarray]) -> float:
    """L2 norm over every gradient element (the norm clip_grad 1.0 acts on)."""
    return math.sqrt(sum(float((g * g).sum()) for g in G.values()))


@dataclass
class AdamState:
    m: Dict[str, np.ndarray] = field(default_factory=dict)
    v: Dict[str, np.ndarray] = field(default_factory=dict)


def clip_adamw(cfg: Config, P: Dict[str, np.ndarray], G: Dict[str, np.ndarray], S: AdamState,
               lr: float, step: int) -> float:
    """Clip by global norm, then one AdamW update in place; returns the norm.

    Run log section 2.1: AdamW with beta1 0.9, beta2 0.95, weight decay 0.1;
    microGPT "核心训练循环": Adam(0.85, 0.99, eps 1e-8), clip_grad 1.0.
    c = min(1, clip / (norm + 1e-6)); g <- c g; for decayed tensors
    w <- w (1 - lr wd); m <- b1 m + (1 - b1) g; v <- b2 v + (1 - b2) g^2;
    w <- w - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps).
    """
    norm = global_grad_norm(G)
    c = 1.0
    if cfg.grad_clip > 0:
        c = min(1.0, cfg.grad_clip / (norm + 1e-6))
    b1, b2 = cfg.beta1, cfg.beta2
    bc1 = 1.0 - b1 ** step
    bc2 = 1.0 - b2 ** step
    specs = {t.name: t for t in tensor_specs(cfg)}
    for name, w in P.items():
        g = G[name] * c
        if name not in S.m:
            S.m[name] = np.zeros_like(w)
            S.v[name] = np.zeros_like(w)
        if cfg.weight_decay != 0.0 and (cfg.decay_1d or specs[name].decayed_by_default):
            w *= (1.0 - lr * cfg.weight_decay)
        S.m[name] = b1 * S.m[name] + (1.0 - b1) * g
        S.v[name] = b2 * S.v[name] + (1.0 - b2) * g * g
        w -= lr * (S.m[name] / bc1) / (np.sqrt(S.v[name] / bc2) + cfg.eps)
    return norm


def lr_cosine(lr: float, it: int, warmup: int, max_iters: int) -> float:
    """get_lr of the practical guide, section 6: linear warmup from 0, then
    a half cosine from the peak down to 0 at max_iters (no floor)."""
    if it < warmup:
        return lr * it / warmup
    return lr * 0.5 * (1.0 + math.cos(math.pi * (it - warmup) / (max_iters - warmup)))


def lr_linear(lr: float, it: int, max_iters: int) -> float:
    """microGPT "核心训练循环": lr decays linearly to 0."""
    return lr * (1.0 - it / max_iters)


def train_step(cfg: Config, P, S: AdamState, stream: np.ndarray, data_seed: int, lr: float, step: int):
    """grad_accum micro-batches (run log section 3.1: gradients of the micro
    batches are summed, each loss divided by grad_accum), then clip + AdamW.
    Returns (mean loss over the micro-batches, grad norm before clipping)."""
    G = None
    losses = []
    for mu in range(cfg.grad_accum):
        idx, tgt = gather_batch(stream, cfg.block_size, data_seed, step, mu, cfg.batch_size)
        drop = DropCtx(cfg.dropout_seed, step * cfg.grad_accum + mu) if cfg.dropout > 0 else None
        loss, g, _ = loss_and_grads(cfg, P, idx, tgt, drop, 1.0 / cfg.grad_accum)
        losses.append(loss)
        if G is None:
            G = g
        else:
            for k in G:
                G[k] += g[k]
    norm = clip_adamw(cfg, P, G, S, lr, step)
    return float(np.mean(losses)), norm


def argmax_rows(z: np.ndarray) -> np.ndarray:
    """Index of the largest logit per row; ties go to the lowest index."""
    return np.argmax(z, axis=-1)
