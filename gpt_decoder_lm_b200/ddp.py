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
