"""Training-step benchmark: tokens/s and MFU of the GPT-2 training step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one full optimiser step of the GPT-2 124M workload (vocab 50257,
12 layers, 12 heads, d 768, block 1024, micro-batch 12, grad-accum 5 ->
61,440 tokens): batch gather from a device-resident synthetic token stream,
forward, cross-entropy, backward, clip and AdamW, all in libgpt.so.  For
N > 1 (torchrun) every rank gathers its own micro-batches and the replicas'
gradients are averaged before clip + AdamW (data-parallel training: a
bucketed NCCL all-reduce on a second stream, overlapping the backward;
gpt_decoder_lm_b200/ddp.py); --zero1 shards the optimiser step instead
(reduce to the shard owner, clip + AdamW on the own shard, all-gather of the
weights); --replicas runs independent replicas.
The barrier and the max-over-ranks timing use torch.distributed.

`--impl reference` times the CPU oracle (float64 numpy) on a bounded sample
of the same workload on the host cores (rank 0 only).

Prints one JSON line.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gpt_decoder_lm_b200 import workloads as W  # noqa: E402

METRIC = "train tokens/sec (GPT-2 124M bf16, T=1024, 1 B200 per replica)"
UNIT = "tokens/s"
NOMINAL_BF16_TFLOPS = 2250.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def flops_per_token(w) -> float:
    """6 N + 12 L d T with N = parameters excluding wpe (PaLM appendix convention)."""
    d, L, T, V = w.n_embd, w.n_layer, w.block_size, w.vocab_size
    if w.variant == "micro":  # untied lm_head, no biases, parameter-free norms
        n = 2 * V * d + 12 * L * d * d
    else:
        n = V * d + L * (12 * d * d + 13 * d) + 2 * d
    return 6.0 * n + 12.0 * L * d * T


def gemm_flops_per_step(w) -> float:
    """Algorithmic dense-contraction FLOPs of one step (forward x3 for dX and dW)."""
    d, L, V = w.n_embd, w.n_layer, w.vocab_size
    M = w.batch_size * w.block_size
    fwd = 2.0 * M * (L * (3 * d * d + d * d + 4 * d * d + 4 * d * d) + V * d)
    return 3.0 * fwd * w.grad_accum


def attn_flops_per_step(w) -> float:
    """Causal attention FLOPs (S = QK^T and PV, lower triangle): fwd 2 matmuls, bwd 5 (+1 recompute)."""
    T, d, L = w.block_size, w.n_embd, w.n_layer
    per_layer_fwd = 2 * 2.0 * w.batch_size * d * T * (T + 1) / 2
    return L * w.grad_accum * per_layer_fwd * (1 + 2.5)


# dram__bytes_read.sum + dram__bytes_write.sum of the tensor-core GEMMs per launch (ncu, one
# pass, on `bench.py --layer-case 2`: every GEMM shape of a layer and the lm_head at full size),
# weighted to the 12-layer step: (12 x one layer's 12 GEMMs + the lm_head's 3) / 147 launches.
# None once the kernels change after that capture: the GEMM epilogue changed after the last one,
# which gave 107,559,868 bytes per launch.
GEMM_DRAM_BYTES_PER_LAUNCH = None
GEMM_DRAM_BYTES_NOTE = ("null: the GEMM epilogue changed after the last per-launch DRAM capture "
                        "(107,559,868 bytes per launch on the layer case before the change)")


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        self.offset = 0

    def wait_ready(self, timeout_s: float = 10.0):
        """Block until nvidia-smi has written its first sample: its start-up (device
        enumeration) must not overlap the timed region."""
        t0 = time.time()
        while self.p is not None and time.time() - t0 < timeout_s:
            if os.path.getsize(self.f.name) > 0 or self.p.poll() is not None:
                break
            time.sleep(0.05)

    def mark(self):
        """Samples written before this call (warm-up) are left out of the summary."""
        self.offset = os.path.getsize(self.f.name)

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(5)
        except Exception:
            self.p.kill()
        self.f.flush()
        text = open(self.f.name).read()
        if self.offset:
            nl = text.find("\n", self.offset - 1)
            text = text[nl + 1:] if nl >= 0 else ""
        rows = [l.split(",") for l in text.splitlines() if l.strip()]
        os.unlink(self.f.name)
        sm = []
        smax = None
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.strip() == "Active":
                        reasons.add(n)
            except Exception:
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


def reduce_max(value: float, device) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_sample_step(w, T_sample: int, state=None):
    """One oracle training step (fwd + bwd + clip + AdamW) on a B=1 window of T_sample tokens
    at the workload's model dims.  Returns (seconds, tokens, state)."""
    import oracle
    cfg = oracle.Config(vocab_size=w.vocab_size, n_layer=w.n_layer, n_head=w.n_head, n_embd=w.n_embd,
                        block_size=T_sample, batch_size=1, grad_accum=1, variant=w.variant,
                        init_std=w.init_std, beta1=w.beta1, beta2=w.beta2, eps=w.eps,
                        weight_decay=w.weight_decay, grad_clip=w.grad_clip)
    if state is None:
        P = oracle.init_params(cfg, w.weight_seed)
        state = (cfg, P, oracle.AdamState(), W.token_stream(w, n=1 << 16), 0)
    cfg, P, S, stream, it = state
    it += 1
    t0 = time.perf_counter()
    oracle.train_step(cfg, P, S, stream.astype(np.int64), w.data_seed, w.lr, it)
    dt = time.perf_counter() - t0
    return dt, T_sample, (cfg, P, S, stream, it)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, w, rank):
    if rank != 0:
        return
    T_sample = 256
    state = None
    for _ in range(args.warmup):
        _, _, state = oracle_sample_step(w, T_sample, state)
    tot, toks = 0.0, 0
    for _ in range(args.steps):
        dt, n, state = oracle_sample_step(w, T_sample, state)
        tot += dt
        toks += n
    value = toks / tot
    cores = blas_threads()
    sample = (f"1 window x {T_sample} tokens per step at the full model dims (fp64 numpy oracle, "
              f"fwd+bwd+clip+AdamW over all 124M parameters)")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000 * tot / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": w.name, "sample": sample},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def decode_bytes_per_step(w, pos: float) -> float:
    """Algorithmic HBM bytes of one decoding step over the batch rows: every
    bf16 weight matrix once (the four per-layer matrices and the tied head)
    plus the bf16 keys and values of positions 0..pos of every row and layer."""
    d, L = w.n_embd, w.n_layer
    vp = ((w.vocab_size + 63) // 64) * 64
    weights = 2.0 * (L * 12 * d * d + vp * d)
    kv = 2.0 * 2 * d * (pos + 1) * w.batch_size * L
    return weights + kv


def measure_decode(model, w, stream_host, dev, rank):
    """Autoregressive sampling through gpt_generate at the workload's batch:
    a 64-token prompt and 64 new tokens (temperature 0.8, top-k 40, top-p
    0.95), replayed as a CUDA graph after two untimed calls.  The per-token
    step time is (t(64 new) - t(1 new)) / 63, which removes the prompt's
    forward pass."""
    import torch
    B, T0, n_new = w.batch_size, 64, 64
    rng = np.random.default_rng(17 + rank)
    starts = rng.integers(0, len(stream_host) - T0, B)
    prompt = torch.from_numpy(np.stack([stream_host[s:s + T0] for s in starts]).astype(np.int32)).to(dev)
    U = torch.from_numpy(rng.random((n_new, B)).astype(np.float32)).to(dev)
    out = torch.empty((B, T0 + n_new), dtype=torch.int32, device=dev)

    def timed(n):
        for _ in range(2):  # warm-up: the first call runs eagerly, the second captures its CUDA graph
            model.generate(prompt, n, 0.8, 40, 0.95, U, out)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        model.generate(prompt, n, 0.8, 40, 0.95, U, out)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    t_full, t_one = timed(n_new), timed(1)
    step_ms = (t_full - t_one) / (n_new - 1)
    pos = T0 + n_new / 2.0
    achieved = decode_bytes_per_step(w, pos) / (step_ms / 1000.0) / 1e9
    hbm = peaks()["hbm_gbs"]
    return {"tokens_per_s": B * n_new / (t_full / 1000.0), "ms_per_token_step": step_ms, "prefill_ms": t_one,
            "batch": B, "prompt": T0, "new_tokens": n_new, "sampling": "temperature 0.8, top-k 40, top-p 0.95",
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "per_step_bytes": decode_bytes_per_step(w, pos),
                         "note": "one decoding step (weights once + the rows' keys / values) at mean position"}}


def measure_recompute(w, d_stream, data_seed, dev, warmup):
    """The same training step with activation recompute (each layer's norms,
    QKV GEMM, attention forward and fc GEMM re-run in the backward): device
    time over 5 graph-replayed steps with the L2 flush between them, and the
    workspace with and without recompute."""
    import torch

    from gpt_decoder_lm_b200 import binding as gb

    cfg = gb.make_config(w, recompute=1)
    m = gb.Model(cfg, seed=w.weight_seed, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    st = 0
    for _ in range(max(warmup, 3)):
        st += 1
        m.train_step(d_stream, data_seed, 1e-4, st, sync=False)
        flush.zero_()
    torch.cuda.synchronize()
    n = 5
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        st += 1
        m.train_step(d_stream, data_seed, 1e-4, st, sync=False)
        flush.zero_()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    m.close()
    del m
    return {"ms_per_step": ms, "tokens_per_s": w.tokens_per_step / (ms / 1000.0), "steps": n,
            "workspace_gb": gb.workspace_bytes(cfg) / 1e9,
            "workspace_gb_stored": gb.workspace_bytes(gb.make_config(w)) / 1e9}


def measure_lora(w, d_stream, data_seed, dev, warmup):
    """The LoRA fine-tuning step (rank 8 on q and v, alpha 16) at the same
    workload: device time over 5 graph-replayed steps, L2 flushed between them."""
    import torch

    from gpt_decoder_lm_b200 import binding as gb

    cfg = gb.make_config(w)
    m = gb.Model(cfg, seed=w.weight_seed, device=dev)
    r, blocks = 8, 2 * w.n_layer
    A = np.random.default_rng(1).standard_normal((blocks, r, w.n_embd)).astype(np.float32) / np.sqrt(w.n_embd)
    m.lora_attach(r, 16.0, 1 | 4, A)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    st = 0
    for _ in range(max(warmup, 3)):
        st += 1
        m.train_step(d_stream, data_seed, 1e-4, st, sync=False)
        flush.zero_()
    torch.cuda.synchronize()
    n = 5
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        st += 1
        m.train_step(d_stream, data_seed, 1e-4, st, sync=False)
        flush.zero_()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    m.close()
    return {"ms_per_step": ms, "tokens_per_s": w.tokens_per_step / (ms / 1000.0), "steps": n, "rank": r,
            "targets": "q,v", "trainable_params": blocks * 2 * r * w.n_embd}


# bounded oracle samples for the other workloads: (batch, window) per step
ORACLE_SAMPLES = {W.MICRO.name: (8, 16), W.CHAR.name: (1, 256), W.DROPOUT_512.name: (1, 128),
                  W.GPT2_XL.name: (1, 16)}


def oracle_tokens_per_s(w, B: int, T: int, threads: int | None):
    """Oracle tokens/s on one step of a B x T sample at the workload's model
    dims (fwd + bwd + clip + AdamW), with the BLAS pool limited to `threads`
    (None: every core)."""
    import oracle
    from threadpoolctl import threadpool_limits
    cfg = oracle.Config(vocab_size=w.vocab_size, n_layer=w.n_layer, n_head=w.n_head, n_embd=w.n_embd,
                        block_size=T, batch_size=B, grad_accum=1, variant=w.variant, init_std=w.init_std,
                        beta1=w.beta1, beta2=w.beta2, eps=w.eps, weight_decay=w.weight_decay, grad_clip=w.grad_clip,
                        dropout=w.dropout, dropout_seed=w.dropout_seed)
    P = oracle.init_params(cfg, w.weight_seed)
    stream = W.token_stream(w, n=1 << 16).astype(np.int64)
    with threadpool_limits(limits=threads, user_api="blas"):
        n = blas_threads()
        t0 = time.perf_counter()
        oracle.train_step(cfg, P, oracle.AdamState(), stream, w.data_seed, w.lr, 1)
        dt = time.perf_counter() - t0
    return B * T / dt, n


def measure_configs(dev, warmup: int, with_oracle: bool):
    """Every other workload of the pages' configurations at its own size: the
    graph-replayed training step timed over 5 steps (L2 flushed between
    them), tokens/s and MFU, next to the oracle's tokens/s on a bounded
    sample at one core and at every core."""
    import torch

    from gpt_decoder_lm_b200 import binding as gb
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    pk = peaks()
    def timed(w, cfg):
        m = gb.Model(cfg, seed=w.weight_seed, device=dev)
        host = W.token_stream(w)
        d_stream = torch.from_numpy(host.view(np.int16) if host.dtype == np.uint16 else host).to(dev)
        st = 0
        for _ in range(max(warmup, 3)):
            st += 1
            m.train_step(d_stream, w.data_seed, w.lr, st, sync=False)
            flush.zero_()
        torch.cuda.synchronize()
        n = 5
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            st += 1
            m.train_step(d_stream, w.data_seed, w.lr, st, sync=False)
            flush.zero_()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / n
        loss, norm = m.train_step(d_stream, w.data_seed, w.lr, st + 1)
        m.close()
        del m, d_stream
        torch.cuda.empty_cache()
        return ms, loss, norm, n

    for w in (W.MICRO, W.CHAR, W.DROPOUT_512, W.GPT2_XL):
        cfg = gb.make_config(w)
        ms, loss, norm, n = timed(w, cfg)
        tps = w.tokens_per_step / (ms / 1000.0)
        fpt = flops_per_token(w)
        rec = {"ms_per_step": ms, "tokens_per_s": tps, "tokens_per_step": w.tokens_per_step,
               "dtype": "f32" if w.precision == "fp32" else "bf16", "flops_per_token": fpt,
               "mfu_nominal_2250": tps * fpt / (NOMINAL_BF16_TFLOPS * 1e12),
               "mfu_measured_peak": tps * fpt / (pk["bf16"] * 1e12), "steps": n,
               "final_loss": loss, "final_grad_norm": norm}
        if w is W.GPT2_XL:  # the configuration activation recompute exists for
            rcfg = gb.make_config(w, recompute=1)
            rms, _, _, _ = timed(w, rcfg)
            rec["recompute"] = {"ms_per_step": rms, "tokens_per_s": w.tokens_per_step / (rms / 1000.0),
                                "workspace_gb": gb.workspace_bytes(rcfg) / 1e9,
                                "workspace_gb_stored": gb.workspace_bytes(cfg) / 1e9}
        if with_oracle:
            B, T = ORACLE_SAMPLES[w.name]
            one, _ = oracle_tokens_per_s(w, B, T, 1)
            allc, nc = oracle_tokens_per_s(w, B, T, None)
            rec["oracle"] = {"tokens_per_s_1_core": one, "tokens_per_s_all_cores": allc, "cores": nc,
                             "sample": f"{B} x {T} tokens per step at the full model dims (fp64 numpy "
                                       f"fwd+bwd+clip+AdamW)"}
        out[w.name] = rec
    return out


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from gpt_decoder_lm_b200 import binding as gb

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    gb.lib()
    # --zero1: each rank's workspace holds the AdamW moments of its own shard only
    sharded = args.zero1 and world > 1 and not args.replicas
    cfg = gb.make_config(w, zero_world=world, zero_rank=rank) if sharded else gb.make_config(w)
    model = gb.Model(cfg, seed=w.weight_seed, device=dev)
    stream_host = W.token_stream(w)
    d_stream = torch.from_numpy(stream_host.view(np.int16)).to(dev)
    data_seed = w.data_seed + 1000003 * rank
    tok_step = w.tokens_per_step
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    st = 0

    def lr_at(i):
        return gb.lr_cosine(w.lr, i, 100, 5000)

    # N > 1: data-parallel training (the gradients of the replicas averaged by a
    # bucketed NCCL all-reduce that overlaps the backward) unless --replicas
    use_ddp = world > 1 and not args.replicas
    trainer = None
    if use_ddp:
        from gpt_decoder_lm_b200 import ddp
        trainer = ddp.ZeroTrainer(model) if args.zero1 else ddp.DataParallelTrainer(model)

    def step_fn(i, sync=False):
        if trainer is not None:
            return trainer.step(d_stream, data_seed, lr_at(i), i, sync=sync)
        return model.train_step(d_stream, data_seed, lr_at(i), i, sync=sync)

    # clock sampler first, so that its start-up falls before the timed region
    clocks = Clocks(local_rank) if rank == 0 else None
    if clocks:
        clocks.wait_ready()
    # warm-up (untimed): the same work as a timed step, L2 flush included (its first launch
    # also loads torch's fill kernel, which must not land in the timed region)
    for _ in range(args.warmup):
        st += 1
        step_fn(st)
        flush.zero_()
    torch.cuda.synchronize()
    if clocks:
        clocks.mark()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    l0 = model.launch_count()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    ev0, ev1 = evs[0], evs[-1]
    ev0.record()
    h0 = time.perf_counter()
    for k in range(args.steps):
        st += 1
        step_fn(st)
        flush.zero_()          # L2 flush between steps (256 MiB > 126 MB L2)
        evs[k + 1].record()
    host_enqueue_ms = (time.perf_counter() - h0) * 1000.0 / args.steps
    torch.cuda.synchronize()
    per_step_ms = [evs[k].elapsed_time(evs[k + 1]) for k in range(args.steps)]
    if world > 1:
        dist.barrier()
    launches = model.launch_count() - l0
    ms = ev0.elapsed_time(ev1)
    ms_max = reduce_max(ms, dev)
    clk = clocks.stop() if clocks else None
    loss, norm = step_fn(st + 1, sync=True)
    st += 1
    value = world * args.steps * tok_step / (ms_max / 1000.0)

    # per-kernel durations: instrumented pass of the same steps (events around every launch)
    model.enable_timing(True)
    for _ in range(args.steps):
        st += 1
        model.train_step(d_stream, data_seed, lr_at(st), st, sync=False)
        flush.zero_()
    torch.cuda.synchronize()
    kt = model.kernel_times()
    model.enable_timing(False)

    # end to end through the host-buffer entry point (H2D of the batch + D2H of loss/norm each step)
    B, T, ga = w.batch_size, w.block_size, w.grad_accum
    rng = np.random.default_rng(7 + rank)
    hb = []
    for k in range(args.steps):
        starts = rng.integers(0, len(stream_host) - T - 1, size=(ga, B))
        rows = starts[..., None] + np.arange(T)
        xi = torch.from_numpy(stream_host[rows].astype(np.int32)).pin_memory()
        yi = torch.from_numpy(stream_host[rows + 1].astype(np.int32)).pin_memory()
        hb.append((xi, yi))
    # untimed warm-up of the host-buffer entry point (its first calls run eagerly
    # and capture its CUDA graph)
    def host_step(xi, yi, i):
        if trainer is not None:
            return trainer.step_host(xi, yi, lr_at(i), i)
        return model.train_step_host(xi, yi, lr_at(i), i)

    for xi, yi in hb[:2]:
        st += 1
        host_step(xi, yi, st)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for xi, yi in hb:
        st += 1
        host_step(xi, yi, st)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1), dev)
    e2e_value = world * args.steps * tok_step / (e2e_ms / 1000.0)

    decode = measure_decode(model, w, stream_host, dev, rank)
    recompute = measure_recompute(w, d_stream, data_seed, dev, args.warmup)
    lora = measure_lora(w, d_stream, data_seed, dev, args.warmup)
    configs = None
    if not args.no_configs:
        configs = measure_configs(dev, args.warmup, rank == 0 and world == 1 and not args.no_cpu_baseline)

    pk = peaks()
    gemm_names = [k for k in kt if k.startswith("gemm")]
    gemm_ms = sum(kt[k][0] for k in gemm_names)
    gemm_n = sum(kt[k][1] for k in gemm_names)
    top = max(kt.items(), key=lambda kv: kv[1][0]) if kt else ("", (0.0, 0))
    gemm_flops = gemm_flops_per_step(w) * args.steps
    achieved = gemm_flops / (gemm_ms / 1000.0) / 1e12 if gemm_ms > 0 else 0.0
    roofline = {"bound": "tensor", "kernel": "tensor-core GEMMs k_gemm_tc2 + k_gemm_tc (all dense contractions)",
                "achieved": achieved,
                "peak": pk["bf16_sustained"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_sustained"],
                "traffic": GEMM_DRAM_BYTES_PER_LAUNCH, "traffic_unit": "bytes per launch (ncu)",
                "traffic_note": GEMM_DRAM_BYTES_NOTE,
                "peak_source": pk["source"] + " sustained bf16",
                "launches": gemm_n, "avg_launch_ms": gemm_ms / max(gemm_n, 1)}
    step_ms = ms_max / args.steps
    kern = {k: {"ms_per_step": v[0] / args.steps, "launches_per_step": v[1] / args.steps,
                "share": v[0] / max(sum(x[0] for x in kt.values()), 1e-9)} for k, v in kt.items()}
    fpt = flops_per_token(w)
    mfu_nom = (value / world) * fpt / (NOMINAL_BF16_TFLOPS * 1e12)
    mfu_meas = (value / world) * fpt / (pk["bf16"] * 1e12)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, n, _ = oracle_sample_step(w, 1024)
        cpu = {"value": n / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": "1 window x 1024 tokens (B=1) at the full GPT-2 124M dims, one oracle step "
                         "(fp64 numpy fwd+bwd+clip+AdamW)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "vocab": w.vocab_size, "n_layer": w.n_layer, "n_head": w.n_head,
                       "n_embd": w.n_embd, "seq_len": w.block_size, "micro_batch": w.batch_size,
                       "grad_accum": w.grad_accum, "tokens_per_step_per_gpu": tok_step,
                       "global_batch_tokens": tok_step * world,
                       "parallelism": (f"dp{world} zero1 (bucketed NCCL reduce to the shard owners overlapped "
                                       "with the backward, sharded clip + AdamW, weight all-gather)" if args.zero1 else
                                       f"dp{world} (bucketed NCCL all-reduce overlapped with the backward)")
                       if use_ddp else f"replicas x{world}",
                       "l2": "256 MiB buffer zeroed between timed steps; step working set ~8 GB"},
            "mfu": {"nominal_2250": mfu_nom, "measured_peak": mfu_meas, "flops_per_token": fpt},
            "roofline": roofline,
            "decode": decode,
            "recompute": recompute,
            "lora": lora,
            "configs": configs,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": 2 * ga * B * T * 4,
                    "d2h_bytes_per_step": 16},
            "gpu_launches": int(launches),
            "host_enqueue_ms_per_step": host_enqueue_ms,
            "step_ms_spread": {"min": min(per_step_ms), "median": statistics.median(per_step_ms),
                               "max": max(per_step_ms), "steps": [round(x, 3) for x in per_step_ms]},
            "clocks": clk,
            "final_loss": loss, "final_grad_norm": norm,
            "kernels": kern,
        }
        print(json.dumps(line), flush=True)
    model.close()


def run_kernels(w):
    """One launch of each hot kernel at the workload's micro-batch shapes through
    the kernel-level test entry points (the small case for ncu captures): the
    GEMMs with the kernel and split the step's cost model picks, the
    tensor-core attention forward and backward."""
    import torch

    from gpt_decoder_lm_b200 import binding as gb
    st = torch.cuda.current_stream().cuda_stream
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    M, d, Vp = w.batch_size * w.block_size, w.n_embd, ((w.vocab_size + 63) // 64) * 64
    PLANNED = 5

    def bf(*s):
        return torch.randn(*s, device="cuda").bfloat16()

    x, wqkv, wfc = bf(M, d), bf(3 * d, d), bf(4 * d, d)
    qkv_out = torch.empty(M, 3 * d, dtype=torch.bfloat16, device="cuda")
    h, g = (torch.empty(M, 4 * d, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    assert gb.test_gemm(PLANNED, M, 3 * d, d, x, d, 1, wqkv, d, 1, 1, 0, qkv_out, None, 3 * d, None, None, None, None,
                        1, None, st, flags) == 0
    assert gb.test_gemm(PLANNED, M, 4 * d, d, x, d, 1, wfc, d, 1, 2, 0, h, g, 4 * d, None,
                        torch.zeros(4 * d, device="cuda"), None, None, 1, None, st, flags) == 0
    wte = bf(Vp, d)
    logits = torch.empty(M, Vp, dtype=torch.bfloat16, device="cuda")
    assert gb.test_gemm(PLANNED, M, Vp, d, x, d, 1, wte, d, 1, 0, 0, logits, None, Vp, None, None, None, None, 1, None,
                        st, flags) == 0
    dwte = torch.zeros(Vp, d, device="cuda")
    assert gb.test_gemm(PLANNED, Vp, d, M, logits, Vp, 0, x, d, 0, 5, 0, dwte, None, d, None, None, None, None, 1, None,
                        st, flags) == 0
    B, T, H = w.batch_size, w.block_size, w.n_head
    q = bf(B, T, 3, H, 64)
    o = torch.empty(B, T, H, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, T, device="cuda")
    do, dq, ds = bf(B, T, H, 64), torch.empty_like(q), torch.empty_like(lse)
    assert gb.test_attention(1, 0, 1, B, T, H, 64, q, o, lse, stream=st, flags=flags) == 0
    assert gb.test_attention(1, 1, 1, B, T, H, 64, q, o, lse, do, dq, ds, stream=st, flags=flags) == 0
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    print(json.dumps({"kernels": "ok", "workload": w.name}))


def run_layer_case(w, layers: int):
    """Two optimiser steps of the workload's dimensions cut to `layers` layers and
    one micro-batch (the small case for per-kernel DRAM captures: every GEMM,
    attention and norm launch of a layer has the full model's shapes). The
    second step is the one to capture: 12 GEMM launches per layer (4 forward,
    4 dX, 4 dW) and 3 for the lm_head, in the engine's own order."""
    import dataclasses

    import torch

    from gpt_decoder_lm_b200 import binding as gb
    wl = dataclasses.replace(w, n_layer=layers, grad_accum=1)
    model = gb.Model(gb.make_config(wl), seed=wl.weight_seed, device=torch.device("cuda", 0))
    d_stream = torch.from_numpy(W.token_stream(wl).view(np.int16)).cuda()
    model.set_graphs(False)
    out = []
    for st in (1, 2):
        l0 = model.launch_count()
        loss, norm = model.train_step(d_stream, wl.data_seed, wl.lr, st, sync=True)
        out.append({"step": st, "loss": loss, "launches": model.launch_count() - l0})
    torch.cuda.synchronize()
    print(json.dumps({"layer_case": wl.name, "n_layer": layers, "grad_accum": 1, "steps": out}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.GPT2_124M.name, choices=list(W.ALL))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' step timings")
    ap.add_argument("--zero1", action="store_true",
                    help="N > 1: data-parallel training with the optimiser step sharded (ZeRO stage 1)")
    ap.add_argument("--replicas", action="store_true",
                    help="N > 1: independent replicas instead of data-parallel training")
    ap.add_argument("--kernels", action="store_true",
                    help="one launch of each hot kernel at the workload's shapes (for ncu), then exit")
    ap.add_argument("--layer-case", type=int, default=0, metavar="L",
                    help="two eager optimiser steps at the workload's dimensions with L layers and one "
                         "micro-batch (for per-kernel ncu captures), then exit")
    args = ap.parse_args()
    w = W.ALL[args.workload]
    if args.kernels:
        run_kernels(w)
        return
    if args.layer_case > 0:
        run_layer_case(w, args.layer_case)
        return
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
