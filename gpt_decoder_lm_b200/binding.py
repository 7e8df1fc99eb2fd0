"""ctypes binding of libgpt.so (include/gpt.h, include/gpt_testing.h).

Argument marshalling only: every step of the training step runs in the CUDA
library.  PyTorch provides device memory (the workspace) and the stream.
Loading fails loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes as C
import os
import re
from typing import Dict, List, Optional, Tuple

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgpt.so")
HEADERS = [os.path.join(os.path.dirname(_PKG), "include", h) for h in ("gpt.h", "gpt_testing.h")]

GPT_ABI_VERSION = 2
GPT_PREC_FP32, GPT_PREC_BF16 = 0, 1
GPT_VARIANT_GPT2, GPT_VARIANT_MICRO = 0, 1
GPT_TOK_I32, GPT_TOK_U16 = 0, 1
GPT_PARAM, GPT_GRAD, GPT_ADAM_M, GPT_ADAM_V = 0, 1, 2, 3
GPT_PATH_GEMM_TC, GPT_PATH_ATTN_TC = 1, 2
STATUS = ["GPT_OK", "GPT_ERR_INVALID_ARG", "GPT_ERR_CONFIG", "GPT_ERR_WORKSPACE_TOO_SMALL", "GPT_ERR_CUDA",
          "GPT_ERR_TOKEN_RANGE", "GPT_ERR_NONFINITE", "GPT_ERR_STATE", "GPT_ERR_UNSUPPORTED", "GPT_ERR_TIMEOUT"]
FLAG_TOKEN, FLAG_LOSS, FLAG_NORM, FLAG_TIMEOUT = 1, 2, 4, 8


class GptConfig(C.Structure):
    _fields_ = [
        ("abi_version", C.c_uint32), ("vocab_size", C.c_int32), ("padded_vocab", C.c_int32),
        ("n_layer", C.c_int32), ("n_head", C.c_int32), ("n_embd", C.c_int32), ("block_size", C.c_int32),
        ("batch_size", C.c_int32), ("grad_accum", C.c_int32), ("precision", C.c_int32), ("variant", C.c_int32),
        ("token_dtype", C.c_int32), ("dropout", C.c_float), ("beta1", C.c_float),
        ("beta2", C.c_float), ("eps", C.c_float), ("weight_decay", C.c_float), ("grad_clip", C.c_float),
        ("decay_1d", C.c_int32), ("recompute", C.c_int32), ("dropout_seed", C.c_uint64),
        ("init_std", C.c_double), ("zero_world", C.c_int32), ("zero_rank", C.c_int32),
    ]


class GptError(RuntimeError):
    def __init__(self, status: int, msg: str):
        self.status = status
        self.name = STATUS[status] if 0 <= status < len(STATUS) else str(status)
        super().__init__(f"{self.name}: {msg}")


_lib = None
P, I32, I64, U32, U64, F32, SZ = C.c_void_p, C.c_int32, C.c_int64, C.c_uint32, C.c_uint64, C.c_float, C.c_size_t
_PROTOS = {
    "gpt_param_count": (SZ, [P]),
    "gpt_config_kernel_paths": (I32, [P, P]),
    "gpt_workspace_bytes": (I32, [P, P]),
    "gpt_grad_buckets": (I32, [P, I32, P, P, P, P]),
    "gpt_grad_arena": (I32, [P, P, P]),
    "gpt_zero1_shard": (I32, [P, I32, I32, P, P, P]),
    "gpt_state_arenas": (I32, [P, P, P, P, P, P, P, P, P]),
    "gpt_grad_sumsq_shard": (I32, [P, I64, I64, P]),
    "gpt_clip_adamw_shard": (I32, [P, F32, I32, I64, I64, F32, P, I32, P]),
    "gpt_train_step_accumulate": (I32, [P, P, U64, U64, I32, P]),
    "gpt_stream_wait_bucket": (I32, [P, I32, P]),
    "gpt_step_loss": (I32, [P, P]),
    "gpt_train_step_host_accumulate": (I32, [P, P, P, I32, P]),
    "gpt_lr_cosine": (F32, [F32, I32, I32, I32]),
    "gpt_lr_linear": (F32, [F32, I32, I32]),
    "gpt_create": (I32, [P, U64, P, SZ, P, P]),
    "gpt_destroy": (None, [P]),
    "gpt_set_stream": (I32, [P, P]),
    "gpt_forward_loss": (I32, [P, P, P, P]),
    "gpt_backward": (I32, [P]),
    "gpt_clip_adamw_step": (I32, [P, F32, I32, P]),
    "gpt_train_step": (I32, [P, P, U64, U64, F32, I32, P, P]),
    "gpt_train_step_host": (I32, [P, P, P, F32, I32, P, P]),
    "gpt_gather_batch": (I32, [P, P, U64, U64, I32, I32, P, P]),
    "gpt_set_dropout_cursor": (I32, [P, I32, I32]),
    "gpt_set_graphs": (I32, [P, I32]),
    "gpt_eval_loss": (I32, [P, P, U64, U64, I32, P]),
    "gpt_sample": (I32, [P, I32, I32, I32, I64, F32, I32, F32, P, P, P]),
    "gpt_generate": (I32, [P, P, I32, I32, F32, I32, F32, P, P]),
    "gpt_lora_workspace_bytes": (I32, [P, I32, I32, P]),
    "gpt_lora_attach": (I32, [P, I32, F32, I32, P, P, SZ]),
    "gpt_lora_detach": (I32, [P]),
    "gpt_lora_read": (I32, [P, I32, P, SZ]),
    "gpt_lora_write": (I32, [P, P, SZ]),
    "gpt_num_tensors": (I32, [P, P]),
    "gpt_tensor_info": (I32, [P, I32, P, P]),
    "gpt_get_tensor": (I32, [P, I32, I32, P]),
    "gpt_set_tensor": (I32, [P, I32, I32, P]),
    "gpt_get_logits": (I32, [P, P]),
    "gpt_get_argmax": (I32, [P, P]),
    "gpt_argmax_rows": (I32, [P, P, I32, I32, P]),
    "gpt_get_lse": (I32, [P, P]),
    "gpt_get_embed_routing": (I32, [P, P, P, P]),
    "gpt_dropout_mask": (I32, [P, I64, I32, I32, I64, P]),
    "gpt_state_floats": (SZ, [P]),
    "gpt_get_state": (I32, [P, P, P, P]),
    "gpt_set_state": (I32, [P, P, P, P]),
    "gpt_read_flags": (I32, [P, P]),
    "gpt_clear_flags": (I32, [P]),
    "gpt_enable_timing": (I32, [P, I32]),
    "gpt_kernel_times": (I32, [P, I32, P, P, P, P]),
    "gpt_launch_count": (U64, [P]),
    "gpt_last_error": (C.c_char_p, [P]),
    "gpt_status_string": (C.c_char_p, [I32]),
    "gpt_test_gemm": (I32, [I32, I32, I32, I32, P, I64, I32, P, I64, I32, I32, I32, P, P, I32, P, P, P, P, I32, P,
                            P, P, P]),
    "gpt_test_attention": (I32, [I32, I32, I32, I32, I32, I32, I32, P, P, P, P, P, P, P, F32, U64, U64, I32, P, P]),
    "gpt_test_wait_timeout": (I32, [U64, P, P, P]),
    "gpt_gemm_dw_accumulate_noalloc": (I32, [I32, I32, I32, P, I64, P, I64, P, I32, P]),
}


def lib() -> C.CDLL:
    """The loaded CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m gpt_decoder_lm_b200.build`")
        l = C.CDLL(LIB_PATH)
        for name, (res, args) in _PROTOS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def declared_symbols() -> List[str]:
    """Function names declared in include/*.h."""
    out = []
    for h in HEADERS:
        txt = open(h).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        out += re.findall(r"\b(gpt_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(out))


def _check(st: int, model=None, what: str = ""):
    if st != 0:
        msg = lib().gpt_last_error(model).decode() if model else ""
        raise GptError(st, f"{what} {msg}".strip())


def _ptr(a) -> int:
    """Device or host address of a torch tensor / numpy array (None -> 0)."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if isinstance(a, np.ndarray):
        assert a.flags["C_CONTIGUOUS"]
        return a.ctypes.data
    return a.data_ptr()


def make_config(w, **over) -> GptConfig:
    """gpt_config from a workloads.Workload (keyword overrides allowed)."""
    d = dict(vocab_size=w.vocab_size, n_layer=w.n_layer, n_head=w.n_head, n_embd=w.n_embd,
             block_size=w.block_size, batch_size=w.batch_size, grad_accum=w.grad_accum,
             precision=GPT_PREC_BF16 if w.precision == "bf16" else GPT_PREC_FP32,
             variant=GPT_VARIANT_MICRO if w.variant == "micro" else GPT_VARIANT_GPT2,
             token_dtype=GPT_TOK_U16 if w.token_dtype == "uint16" else GPT_TOK_I32,
             init_std=w.init_std, dropout=w.dropout, beta1=w.beta1, beta2=w.beta2, eps=w.eps,
             weight_decay=w.weight_decay, grad_clip=w.grad_clip, decay_1d=0, dropout_seed=w.dropout_seed,
             padded_vocab=0)
    d.update(over)
    c = GptConfig()
    c.abi_version = GPT_ABI_VERSION
    for k, v in d.items():
        setattr(c, k, v)
    return c


def grad_buckets(cfg: GptConfig):
    """The gradient exchange plan: [(offset, count, bucket)] in the order the
    backward finalises the buckets."""
    n = C.c_int32(0)
    _check(lib().gpt_grad_buckets(C.byref(cfg), 0, None, None, None, C.byref(n)), None, "grad_buckets")
    off = (C.c_int64 * n.value)()
    cnt = (C.c_int64 * n.value)()
    bkt = (C.c_int32 * n.value)()
    _check(lib().gpt_grad_buckets(C.byref(cfg), n.value, off, cnt, bkt, C.byref(n)), None, "grad_buckets")
    return [(int(off[i]), int(cnt[i]), int(bkt[i])) for i in range(n.value)]


NORM_PARTIALS = 592  # GPT_NORM_PARTIALS


def zero1_shard(cfg: GptConfig, world: int, rank: int):
    """(offset, count, stride) of optimiser shard `rank` of `world`."""
    off, cnt, stride = C.c_int64(), C.c_int64(), C.c_int64()
    _check(lib().gpt_zero1_shard(C.byref(cfg), world, rank, C.byref(off), C.byref(cnt), C.byref(stride)), None,
           "zero1_shard")
    return int(off.value), int(cnt.value), int(stride.value)


def kernel_paths(cfg: GptConfig) -> int:
    """GPT_PATH_* bits: which kernels a model with this config runs."""
    n = C.c_uint32(0)
    _check(lib().gpt_config_kernel_paths(C.byref(cfg), C.byref(n)), None, "config_kernel_paths")
    return int(n.value)


def param_count(cfg: GptConfig) -> int:
    return int(lib().gpt_param_count(C.byref(cfg)))


def workspace_bytes(cfg: GptConfig) -> int:
    n = C.c_size_t(0)
    _check(lib().gpt_workspace_bytes(C.byref(cfg), C.byref(n)), None, "workspace_bytes")
    return int(n.value)


def lr_cosine(lr, it, warmup, max_iters) -> float:
    return float(lib().gpt_lr_cosine(lr, it, warmup, max_iters))


def lr_linear(lr, it, max_iters) -> float:
    return float(lib().gpt_lr_linear(lr, it, max_iters))


class Model:
    """One model in a torch-allocated device workspace, on torch's current stream."""

    def __init__(self, cfg: GptConfig, seed: int, device=None, stream=None, workspace=None):
        import torch
        self.cfg = cfg
        self.device = torch.device(device or "cuda")
        nbytes = workspace_bytes(cfg)
        self.ws = workspace if workspace is not None else torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.stream = stream or torch.cuda.current_stream(self.device)
        h = C.c_void_p()
        st = lib().gpt_create(C.byref(cfg), seed, self.ws.data_ptr(), self.ws.numel(), self.stream.cuda_stream,
                              C.byref(h))
        _check(st, None, "gpt_create")
        self.h = h
        self.M = cfg.batch_size * cfg.block_size

    def close(self):
        h = getattr(self, "h", None)
        if h:
            self.h = None
            f = globals().get("lib")  # None while the interpreter shuts down
            if f is not None:
                f().gpt_destroy(h)

    __del__ = close

    # -- step
    def forward_loss(self, idx, tgt, sync: bool = True) -> Optional[float]:
        out = C.c_float()
        _check(lib().gpt_forward_loss(self.h, _ptr(idx), _ptr(tgt), C.byref(out) if sync else None), self.h,
               "forward_loss")
        return float(out.value) if sync else None

    def backward(self):
        _check(lib().gpt_backward(self.h), self.h, "backward")

    def clip_adamw_step(self, lr: float, step: int, sync: bool = True) -> Optional[float]:
        out = C.c_float()
        _check(lib().gpt_clip_adamw_step(self.h, lr, step, C.byref(out) if sync else None), self.h, "clip_adamw")
        return float(out.value) if sync else None

    def train_step(self, stream_tokens, data_seed: int, lr: float, step: int, sync: bool = True):
        loss, norm = C.c_float(), C.c_float()
        _check(lib().gpt_train_step(self.h, _ptr(stream_tokens), stream_tokens.numel(), data_seed, lr, step,
                                    C.byref(loss) if sync else None, C.byref(norm) if sync else None), self.h,
               "train_step")
        return (float(loss.value), float(norm.value)) if sync else None

    def train_step_host(self, h_idx, h_tgt, lr: float, step: int):
        loss, norm = C.c_float(), C.c_float()
        _check(lib().gpt_train_step_host(self.h, _ptr(h_idx), _ptr(h_tgt), lr, step, C.byref(loss), C.byref(norm)),
               self.h, "train_step_host")
        return float(loss.value), float(norm.value)

    def train_step_accumulate(self, stream_tokens, data_seed: int, step: int, sync: bool = False):
        loss = C.c_float()
        _check(lib().gpt_train_step_accumulate(self.h, _ptr(stream_tokens), stream_tokens.numel(), data_seed, step,
                                               C.byref(loss) if sync else None), self.h, "train_step_accumulate")
        return float(loss.value) if sync else None

    def train_step_host_accumulate(self, h_idx, h_tgt, step: int, sync: bool = False):
        loss = C.c_float()
        _check(lib().gpt_train_step_host_accumulate(self.h, _ptr(h_idx), _ptr(h_tgt), step,
                                                    C.byref(loss) if sync else None), self.h,
               "train_step_host_accumulate")
        return float(loss.value) if sync else None

    def step_loss(self) -> float:
        out = C.c_float()
        _check(lib().gpt_step_loss(self.h, C.byref(out)), self.h, "step_loss")
        return float(out.value)

    def stream_wait_bucket(self, bucket: int, stream):
        _check(lib().gpt_stream_wait_bucket(self.h, bucket, stream.cuda_stream), self.h, "stream_wait_bucket")

    def grad_arena(self):
        """The fp32 gradient arena as a torch tensor view of the workspace."""
        import torch
        p, n = C.c_void_p(), C.c_int64()
        _check(lib().gpt_grad_arena(self.h, C.byref(p), C.byref(n)), self.h, "grad_arena")
        off = p.value - self.ws.data_ptr()
        assert off % 4 == 0 and off >= 0
        return self.ws[off:off + 4 * n.value].view(torch.float32)

    def state_arenas(self):
        """{"param", "grad", "adam_m", "adam_v": fp32, "param_bf16": bf16 or None}
        as torch views of the workspace, each of the allocated length (the
        used length is ["n"])."""
        import torch
        ptr = [C.c_void_p() for _ in range(5)]
        n, n_alloc, n_mom = C.c_int64(), C.c_int64(), C.c_int64()
        _check(lib().gpt_state_arenas(self.h, *[C.byref(x) for x in ptr], C.byref(n), C.byref(n_alloc),
                                      C.byref(n_mom)), self.h, "state_arenas")
        base = self.ws.data_ptr()

        def view(p, dtype, esize, length):
            if not p.value:
                return None
            off = p.value - base
            assert off >= 0 and off % esize == 0
            return self.ws[off:off + esize * length].view(dtype)
        out = {k: view(p, torch.float32, 4, n_alloc.value) for k, p in zip(("param", "grad"), ptr[:2])}
        out.update({k: view(p, torch.float32, 4, n_mom.value) for k, p in zip(("adam_m", "adam_v"), ptr[2:4])})
        out["param_bf16"] = view(ptr[4], torch.bfloat16, 2, n_alloc.value)
        out["n"] = int(n.value)
        out["moments_sharded"] = self.cfg.zero_world > 1
        return out

    def grad_sumsq_shard(self, offset: int, count: int, partials):
        """NORM_PARTIALS fp64 partial sums of squares of gradient elements
        [offset, offset + count) into the device tensor `partials`."""
        assert partials.numel() >= NORM_PARTIALS and partials.dtype.itemsize == 8
        _check(lib().gpt_grad_sumsq_shard(self.h, offset, count, _ptr(partials)), self.h, "grad_sumsq_shard")

    def clip_adamw_shard(self, lr: float, step: int, offset: int, count: int, grad_scale: float, partials,
                         sync: bool = True) -> Optional[float]:
        """Clip + AdamW on one shard; the global norm from the gathered partials."""
        out = C.c_float()
        _check(lib().gpt_clip_adamw_shard(self.h, lr, step, offset, count, grad_scale, _ptr(partials),
                                          partials.numel(), C.byref(out) if sync else None), self.h,
               "clip_adamw_shard")
        return float(out.value) if sync else None

    def gather_batch(self, stream_tokens, data_seed: int, step: int, micro: int, idx, tgt):
        _check(lib().gpt_gather_batch(self.h, _ptr(stream_tokens), stream_tokens.numel(), data_seed, step, micro,
                                      _ptr(idx), _ptr(tgt)), self.h, "gather_batch")

    def set_dropout_cursor(self, step: int, micro: int):
        _check(lib().gpt_set_dropout_cursor(self.h, step, micro), self.h, "set_dropout_cursor")

    def eval_loss(self, stream_tokens, data_seed: int, n_batches: int) -> float:
        """Mean loss of n_batches evaluation batches (forward only, no dropout)."""
        out = C.c_float()
        _check(lib().gpt_eval_loss(self.h, _ptr(stream_tokens), stream_tokens.numel(), data_seed, n_batches,
                                   C.byref(out)), self.h, "eval_loss")
        return float(out.value)

    def generate(self, prompt, n_new: int, temperature: float, top_k: int, top_p: float, uniform, out):
        """prompt: device int32 [batch_size, T0]; uniform: device fp32 [n_new, batch_size];
        out: device int32 [batch_size, T0 + n_new]."""
        _check(lib().gpt_generate(self.h, _ptr(prompt), prompt.shape[1], n_new, temperature, top_k, top_p,
                                  _ptr(uniform), _ptr(out)), self.h, "generate")

    # -- LoRA adapters on the fused QKV blocks (targets: 1 q, 2 k, 4 v)
    def lora_attach(self, r: int, alpha: float, targets: int, A):
        """A: host float32 [blocks, r, d] (the adapted blocks' A; B starts at 0).
        Allocates the adapter workspace as a torch tensor owned by the model."""
        import torch
        n = C.c_size_t(0)
        _check(lib().gpt_lora_workspace_bytes(C.byref(self.cfg), r, targets, C.byref(n)), self.h, "lora_workspace")
        self.lora_ws = torch.empty(int(n.value), dtype=torch.uint8, device=self.device)
        A = np.ascontiguousarray(A, np.float32)
        _check(lib().gpt_lora_attach(self.h, r, alpha, targets, A.ctypes.data_as(C.c_void_p), self.lora_ws.data_ptr(),
                                     self.lora_ws.numel()), self.h, "lora_attach")
        self.lora_n = int(np.prod(A.shape)) * 2

    def lora_detach(self):
        _check(lib().gpt_lora_detach(self.h), self.h, "lora_detach")
        self.lora_ws = None

    def lora_read(self, which: int = 0) -> np.ndarray:
        out = np.empty(self.lora_n, np.float32)
        _check(lib().gpt_lora_read(self.h, which, out.ctypes.data_as(C.c_void_p), out.size), self.h, "lora_read")
        return out

    def lora_write(self, params):
        params = np.ascontiguousarray(params, np.float32)
        _check(lib().gpt_lora_write(self.h, params.ctypes.data_as(C.c_void_p), params.size), self.h, "lora_write")

    def set_graphs(self, on: bool):
        """CUDA-graph replay of train_step / train_step_host / generate (default on)."""
        _check(lib().gpt_set_graphs(self.h, 1 if on else 0), self.h, "set_graphs")

    # -- introspection
    def tensors(self) -> List[Tuple[str, Tuple[int, int]]]:
        n = C.c_int32()
        _check(lib().gpt_num_tensors(self.h, C.byref(n)), self.h)
        out = []
        for i in range(n.value):
            name = C.c_char_p()
            shape = (C.c_int64 * 2)()
            _check(lib().gpt_tensor_info(self.h, i, C.byref(name), shape), self.h)
            out.append((name.value.decode(), (int(shape[0]), int(shape[1]))))
        return out

    def get(self, kind: int = GPT_PARAM) -> Dict[str, np.ndarray]:
        res = {}
        for i, (name, (r, c)) in enumerate(self.tensors()):
            a = np.empty(r * c, dtype=np.float32)
            _check(lib().gpt_get_tensor(self.h, i, kind, a.ctypes.data), self.h, "get_tensor")
            res[name] = a.reshape((r, c) if c > 1 else (r,))
        return res

    def set(self, values: Dict[str, np.ndarray], kind: int = GPT_PARAM):
        for i, (name, (r, c)) in enumerate(self.tensors()):
            if name in values:
                a = np.ascontiguousarray(values[name], dtype=np.float32).reshape(-1)
                assert a.size == r * c, name
                _check(lib().gpt_set_tensor(self.h, i, kind, a.ctypes.data), self.h, "set_tensor")

    def logits(self) -> np.ndarray:
        a = np.empty((self.M, self.cfg.vocab_size), dtype=np.float32)
        _check(lib().gpt_get_logits(self.h, a.ctypes.data), self.h, "get_logits")
        return a

    def argmax(self) -> np.ndarray:
        a = np.empty(self.M, dtype=np.int32)
        _check(lib().gpt_get_argmax(self.h, a.ctypes.data), self.h, "get_argmax")
        return a

    def argmax_rows(self, d_rows) -> np.ndarray:
        rows, cols = d_rows.shape
        a = np.empty(rows, dtype=np.int32)
        _check(lib().gpt_argmax_rows(self.h, _ptr(d_rows), rows, cols, a.ctypes.data), self.h, "argmax_rows")
        return a

    def lse(self) -> np.ndarray:
        a = np.empty(self.M, dtype=np.float32)
        _check(lib().gpt_get_lse(self.h, a.ctypes.data), self.h, "get_lse")
        return a

    def embed_routing(self):
        n = C.c_int32()
        tok = np.empty(self.M, dtype=np.int32)
        pos = np.empty(self.M, dtype=np.int32)
        _check(lib().gpt_get_embed_routing(self.h, C.byref(n), tok.ctypes.data, pos.ctypes.data), self.h)
        return int(n.value), tok, pos

    def dropout_mask(self, counter: int, layer: int, site: int, n: int) -> np.ndarray:
        a = np.empty(n, dtype=np.uint8)
        _check(lib().gpt_dropout_mask(self.h, counter, layer, site, n, a.ctypes.data), self.h, "dropout_mask")
        return a.astype(bool)

    def get_state(self):
        n = int(lib().gpt_state_floats(self.h))
        p, m, v = (np.empty(n, dtype=np.float32) for _ in range(3))
        _check(lib().gpt_get_state(self.h, p.ctypes.data, m.ctypes.data, v.ctypes.data), self.h, "get_state")
        return p, m, v

    def set_state(self, p, m, v):
        _check(lib().gpt_set_state(self.h, _ptr(np.ascontiguousarray(p, np.float32)),
                                   _ptr(np.ascontiguousarray(m, np.float32)),
                                   _ptr(np.ascontiguousarray(v, np.float32))), self.h, "set_state")

    def flags(self) -> int:
        f = C.c_uint32()
        _check(lib().gpt_read_flags(self.h, C.byref(f)), self.h)
        return int(f.value)

    def clear_flags(self):
        _check(lib().gpt_clear_flags(self.h), self.h)

    def enable_timing(self, on: bool):
        _check(lib().gpt_enable_timing(self.h, 1 if on else 0), self.h)

    def kernel_times(self) -> Dict[str, Tuple[float, int]]:
        cap = 256
        names = (C.c_char_p * cap)()
        ms = (C.c_float * cap)()
        ln = (C.c_int32 * cap)()
        n = C.c_int32()
        _check(lib().gpt_kernel_times(self.h, cap, names, ms, ln, C.byref(n)), self.h)
        return {names[i].decode(): (float(ms[i]), int(ln[i])) for i in range(n.value)}

    def launch_count(self) -> int:
        return int(lib().gpt_launch_count(self.h))


def sample(logits, temperature: float, top_k: int, top_p: float, uniform, out, V=None, stream=None):
    """One draw per row of a device logits tensor [rows, ld] (bf16 or fp32);
    uniform: device fp32 [rows]; out: device int32 [rows]."""
    import torch
    rows, ld = logits.shape
    st = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    _check(lib().gpt_sample(_ptr(logits), 1 if logits.dtype == torch.bfloat16 else 0, rows, V or ld, ld, temperature,
                            top_k, top_p, _ptr(uniform), _ptr(out), st), None, "sample")


def test_gemm(backend, M, N, K, A, lda, a_kmajor, B, ldb, b_kmajor, epi_kind, act=0, out=None, out2=None, ldo=0,
              aux=None, bias=None, res_in=None, res_out=None, split_k=1, partial=None, stream=None, flags=None,
              colsum=None):
    return int(lib().gpt_test_gemm(backend, M, N, K, _ptr(A), lda, a_kmajor, _ptr(B), ldb, b_kmajor, epi_kind, act,
                                   _ptr(out), _ptr(out2), ldo, _ptr(aux), _ptr(bias), _ptr(res_in), _ptr(res_out),
                                   split_k, _ptr(partial), _ptr(colsum), stream, _ptr(flags)))


def test_attention(backend, backward, dtype, B, T, H, hd, qkv, o, lse, dout=None, dqkv=None, dsum=None, p=0.0,
                   seed=0, counter=0, layer=0, stream=None, flags=None, colsum=None):
    return int(lib().gpt_test_attention(backend, backward, dtype, B, T, H, hd, _ptr(qkv), _ptr(o), _ptr(lse),
                                        _ptr(dout), _ptr(dqkv), _ptr(dsum), _ptr(colsum), p, seed, counter, layer,
                                        stream, _ptr(flags)))


def test_wait_timeout(limit_ns: int, flags, gave_up, stream=None) -> int:
    """The kernels' bounded mbarrier wait with a short limit, on a barrier
    nothing arrives at; returns the status code."""
    return int(lib().gpt_test_wait_timeout(limit_ns, stream, _ptr(flags), _ptr(gave_up)))
