"""Data-parallel training step over torch.distributed (argument marshalling
and collective plumbing only; every step of the training step runs in the
CUDA library).

The nanoGPT README's multi-GPU recipe ("复现 GPT-2": torchrun over 8 GPUs
with DDP) keeps one replica of the model per GPU, gives each replica its own
micro-batches and averages the gradients across replicas before the
optimiser step.  Here:

  1. gpt_train_step_accumulate runs the replica's grad_accum forward and
     backward passes (a replayed CUDA graph) and records one event per
     gradient bucket as the last micro-batch's backward finalises it
     (buckets in backward order: the last layer first, the embeddings last);
  2. for each bucket, a second stream waits for that event and all-reduces
     the bucket's ranges of the fp32 gradient arena (NCCL over NVLink on
     GPUs; gloo in the CPU tests), so the exchange of layer l overlaps the
     backward of layers < l;
  3. the model's stream waits for the exchange, and gpt_clip_adamw_step clips
     the averaged gradients by their global norm and applies AdamW, which is
     identical on every replica.

The all-reduce sums; the mean is that sum times 1 / world_size (skipped for
a single rank, where the exchange is the identity).

ZeroTrainer is the same step with the optimiser sharded (ZeRO stage 1, the
DeepSpeed scheme the fine-tuning pipelines page points to for larger
models): each replica owns one contiguous shard of the arenas
(gpt_zero1_shard); every bucket part is sum-reduced to the replica that owns
it, the owner clips by the global norm (its partial sums of squares are
all-gathered, so every replica computes the same norm) and runs AdamW on its
shard alone, with the 1 / world_size of the mean folded into the update, and
the updated fp32 weights and their bf16 copies are all-gathered in place.
"""

from __future__ import annotations

from typing import Dict, List, Tuple

from . import binding as gb


def bucket_plan(cfg) -> List[Tuple[int, List[Tuple[int, int]]]]:
    """[(bucket, [(offset, count), ...])] in the order the backward finalises them."""
    by: Dict[int, List[Tuple[int, int]]] = {}
    for off, cnt, b in gb.grad_buckets(cfg):
        by.setdefault(b, []).append((off, cnt))
    return sorted(by.items())


def exchange_bucket(grad, ranges, group=None, world: int = 1):
    """All-reduce (mean) of the given ranges of a flat gradient tensor."""
    import torch.distributed as dist
    for off, cnt in ranges:
        view = grad[off:off + cnt]
        dist.all_reduce(view, op=dist.ReduceOp.SUM, group=group)
        if world > 1:
            view.mul_(1.0 / world)


class DataParallelTrainer:
    """One replica of a data-parallel training run (one process per GPU)."""

    def __init__(self, model: "gb.Model", group=None):
        import torch
        import torch.distributed as dist
        self.model = model
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.plan = bucket_plan(model.cfg)
        self.side = torch.cuda.Stream(device=model.device)
        self.grad = model.grad_arena()

    def _exchange(self):
        import torch
        m, main = self.model, self.model.stream
        for bucket, ranges in self.plan:
            m.stream_wait_bucket(bucket, self.side)
            with torch.cuda.stream(self.side):
                exchange_bucket(self.grad, ranges, self.group, self.world)
        main.wait_stream(self.side)

    def step(self, stream_tokens, data_seed: int, lr: float, step: int, sync: bool = True):
        """One optimiser step: local micro-batches (from this replica's
        data_seed), the gradient exchange, clip + AdamW.  Returns the local
        mean loss and the global-norm of the averaged gradients when sync."""
        self.model.train_step_accumulate(stream_tokens, data_seed, step)  # asynchronous: the exchange overlaps it
        self._exchange()
        norm = self.model.clip_adamw_step(lr, step, sync=sync)
        return (self.model.step_loss(), norm) if sync else None

    def step_host(self, h_idx, h_tgt, lr: float, step: int, sync: bool = True):
        """The same with this replica's micro-batches from host memory."""
        self.model.train_step_host_accumulate(h_idx, h_tgt, step)
        self._exchange()
        norm = self.model.clip_adamw_step(lr, step, sync=sync)
        return (self.model.step_loss(), norm) if sync else None


def shard_parts(plan, stride: int, world: int) -> List[Tuple[int, List[Tuple[int, int, int]]]]:
    """The bucket plan cut at the shard bounds (multiples of `stride`):
    [(bucket, [(owner rank, offset, count), ...])] in the plan's order."""
    out = []
    for bucket, ranges in plan:
        parts = []
        for off, cnt in ranges:
            lo, hi = off, off + cnt
            while lo < hi:
                r = min(lo // stride, world - 1)
                e = hi if r == world - 1 else min(hi, (r + 1) * stride)
                parts.append((r, lo, e - lo))
                lo = e
        out.append((bucket, parts))
    return out


def reduce_parts(grad, parts, group=None):
    """Sum-reduce each part of a flat gradient tensor to its owner rank."""
    import torch.distributed as dist
    for r, off, cnt in parts:
        dst = dist.get_global_rank(group, r) if group is not None else r
        dist.reduce(grad[off:off + cnt], dst=dst, op=dist.ReduceOp.SUM, group=group)


def all_gather_shards(arena, stride: int, world: int, rank: int, group=None):
    """All-gather of `world` equal shards of `stride` elements of a flat
    tensor (at least world * stride long), in place: shard r comes from rank r."""
    import torch.distributed as dist
    full = arena[:world * stride]
    src = full[rank * stride:(rank + 1) * stride]
    if dist.get_backend(group) != "nccl":
        src = src.clone()  # NCCL takes the in-place form; the CPU backend gets its own source buffer
    dist.all_gather_into_tensor(full, src, group=group)


class ZeroTrainer:
    """One replica of a data-parallel run with the optimiser sharded (ZeRO-1)."""

    def __init__(self, model: "gb.Model", group=None):
        import torch
        import torch.distributed as dist
        self.model = model
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.offset, self.count, self.stride = gb.zero1_shard(model.cfg, self.world, self.rank)
        if model.cfg.zero_world > 1 and (model.cfg.zero_world, model.cfg.zero_rank) != (self.world, self.rank):
            raise ValueError("the model's zero_world / zero_rank differ from the process group's")
        self.arenas = model.state_arenas()
        self.parts = shard_parts(bucket_plan(model.cfg), self.stride, self.world)
        self.side = torch.cuda.Stream(device=model.device)
        self.partials = torch.zeros(gb.NORM_PARTIALS, dtype=torch.float64, device=model.device)
        self.gathered = torch.zeros(self.world * gb.NORM_PARTIALS, dtype=torch.float64, device=model.device)

    def _exchange(self):
        import torch
        m, main = self.model, self.model.stream
        for bucket, parts in self.parts:
            m.stream_wait_bucket(bucket, self.side)
            with torch.cuda.stream(self.side):
                reduce_parts(self.arenas["grad"], parts, self.group)
        main.wait_stream(self.side)

    def _update(self, lr: float, step: int, sync: bool):
        import torch
        import torch.distributed as dist
        m = self.model
        with torch.cuda.stream(m.stream):
            m.grad_sumsq_shard(self.offset, self.count, self.partials)
            dist.all_gather_into_tensor(self.gathered, self.partials, group=self.group)
            norm = m.clip_adamw_shard(lr, step, self.offset, self.count, 1.0 / self.world, self.gathered, sync=sync)
            for name in ("param", "param_bf16"):
                if self.arenas[name] is not None:
                    all_gather_shards(self.arenas[name], self.stride, self.world, self.rank, self.group)
            if sync:
                m.stream.synchronize()
        return norm

    def gather_optimizer_state(self):
        """All-gather the AdamW moments so that every replica holds all of
        them (before gpt_get_state on a sharded run).  Not with a model whose
        config shards the moments themselves (zero_world > 1): it holds its
        own shard only, which is what it checkpoints."""
        import torch
        if self.arenas["moments_sharded"]:
            raise RuntimeError("the model holds its own shard of the moments only (zero_world > 1)")
        with torch.cuda.stream(self.model.stream):
            for name in ("adam_m", "adam_v"):
                all_gather_shards(self.arenas[name], self.stride, self.world, self.rank, self.group)

    def step(self, stream_tokens, data_seed: int, lr: float, step: int, sync: bool = True):
        """As DataParallelTrainer.step, with the sharded optimiser."""
        self.model.train_step_accumulate(stream_tokens, data_seed, step)
        self._exchange()
        norm = self._update(lr, step, sync)
        return (self.model.step_loss(), norm) if sync else None

    def step_host(self, h_idx, h_tgt, lr: float, step: int, sync: bool = True):
        self.model.train_step_host_accumulate(h_idx, h_tgt, step)
        self._exchange()
        norm = self._update(lr, step, sync)
        return (self.model.step_loss(), norm) if sync else None
