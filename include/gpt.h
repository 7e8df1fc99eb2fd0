/*
 * gpt.h -- C ABI of the B200 (sm_100a) GPT-2 causal-LM training step.
 *
 * The library implements one training step of a nanoGPT-style GPT-2:
 * token + learned position embedding, n_layer pre-norm blocks (norm, fused
 * QKV projection, causal scaled-dot-product attention, output projection,
 * residual; norm, 4x MLP, residual), a final norm, an lm_head tied to the
 * token embedding, mean cross-entropy, the full backward pass, global-norm
 * gradient clipping and AdamW.
 *
 * Sources (web pages; section names are the pages' own):
 *   - "nanoGPT README" (translated): model.py / train.py, GPT-2 124M
 *     reproduction ("复现 GPT-2"), benchmarking ("效率说明").
 *   - "从零实现GPT训练与推理：基于nanoGPT的实战指南": section 3 (config
 *     n_layer/n_head/n_embd), section 6 ("性能优化技巧": get_lr warmup +
 *     cosine, bf16, gradient accumulation).
 *   - nanoGPT run log (wmrh.cn): section 1.3 (train.bin token stream,
 *     block_size windows), 2.1 (config table), 2.2 (head_dim), 2.3
 *     (parameter count), 3.1 (gradient accumulation), 4.5 (fixed seeds).
 *   - "微型 GPT 从零构建：核心训练循环、分词与单 GPU 高效推理": sections
 *     "模型核心" (microGPT architecture: RMSNorm, ReLU, 4192 params) and
 *     "核心训练循环" (forward, -log p loss, backward, Adam, clip 1.0).
 *
 * Conventions for every entry point:
 *   - Device pointers are plain CUDA device addresses on the device that
 *     was current when the model was created; host pointers are ordinary
 *     (preferably pinned) host memory.
 *   - All device work is enqueued on the model's stream (gpt_create /
 *     gpt_set_stream).  A call that takes a host output pointer (h_loss,
 *     h_grad_norm, h_out ...) synchronises that stream before it returns;
 *     passing NULL keeps the call asynchronous.
 *   - The caller owns the device workspace (see gpt_workspace_bytes); the
 *     library carves every device buffer it uses out of it and performs no
 *     device allocation.  The workspace must outlive the model.
 *   - Errors are returned as gpt_status; nothing aborts the process or
 *     traps the GPU.  Argument and sequencing errors are detected on the
 *     host before any launch.  Conditions only the device can see (a token
 *     id >= vocab_size, a non-finite loss or gradient norm, a bounded wait
 *     in a kernel that ran out) set bits in a device flag word that the
 *     next synchronising call reports (and gpt_read_flags returns).
 *   - gpt_last_error() gives a human-readable message for the last failing
 *     call on a model.
 */
#ifndef GPT_B200_H
#define GPT_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPT_ABI_VERSION 2u

typedef enum {
  GPT_OK = 0,
  GPT_ERR_INVALID_ARG = 1,       /* NULL pointer, bad size, bad enum value            */
  GPT_ERR_CONFIG = 2,            /* inconsistent config (n_embd % n_head != 0 ...)    */
  GPT_ERR_WORKSPACE_TOO_SMALL = 3,
  GPT_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed                 */
  GPT_ERR_TOKEN_RANGE = 5,       /* a token id was outside [0, vocab_size)            */
  GPT_ERR_NONFINITE = 6,         /* loss or gradient norm was NaN/Inf                 */
  GPT_ERR_STATE = 7,             /* call out of sequence (backward before forward)    */
  GPT_ERR_UNSUPPORTED = 8,       /* valid request the library does not implement      */
  GPT_ERR_TIMEOUT = 9            /* a bounded device-side wait ran out                */
} gpt_status;

enum { GPT_PREC_FP32 = 0, GPT_PREC_BF16 = 1 };
/* GPT2: LayerNorm with gain/bias, biases on every linear layer, GELU (erf
 * form), lm_head tied to wte.  MICRO (microGPT page, "模型核心"):
 * parameter-free RMSNorm, no biases, ReLU, untied lm_head. */
enum { GPT_VARIANT_GPT2 = 0, GPT_VARIANT_MICRO = 1 };
enum { GPT_TOK_I32 = 0, GPT_TOK_U16 = 1 };
/* kinds of per-parameter arrays for gpt_get_tensor / gpt_set_tensor */
enum { GPT_PARAM = 0, GPT_GRAD = 1, GPT_ADAM_M = 2, GPT_ADAM_V = 3 };
/* device flag bits (gpt_read_flags) */
enum {
  GPT_FLAG_TOKEN_RANGE = 1u << 0,
  GPT_FLAG_NONFINITE_LOSS = 1u << 1,
  GPT_FLAG_NONFINITE_NORM = 1u << 2,
  GPT_FLAG_TIMEOUT = 1u << 3
};

/* Plain-old-data model + optimiser configuration.  Field names follow the
 * nanoGPT config files (practical guide section 3; run log section 2.1). */
typedef struct gpt_config {
  uint32_t abi_version;   /* must be GPT_ABI_VERSION                                 */
  int32_t vocab_size;     /* V: token ids are in [0, V)                              */
  int32_t padded_vocab;   /* Vp >= V, multiple of 64; 0 = round V up to 64.  Rows
                             V..Vp-1 of wte are layout padding: zero, never updated,
                             excluded from the loss (their logits are masked).       */
  int32_t n_layer;        /* L >= 1                                                  */
  int32_t n_head;         /* H; head_dim = n_embd / n_head (run log section 2.2)     */
  int32_t n_embd;         /* d, multiple of 8, at most 2048                          */
  int32_t block_size;     /* T: sequence length of every window                      */
  int32_t batch_size;     /* B: windows per micro-batch                              */
  int32_t grad_accum;     /* micro-batches per optimiser step (>= 1)                 */
  int32_t precision;      /* GPT_PREC_FP32 (all fp32, SIMT) or GPT_PREC_BF16         */
  int32_t variant;        /* GPT_VARIANT_GPT2 or GPT_VARIANT_MICRO                   */
  int32_t token_dtype;    /* element type of the token stream in gpt_train_step      */
  float dropout;          /* p in [0, 1); 0 disables every dropout site              */
  float beta1, beta2, eps;
  float weight_decay;     /* decoupled (AdamW); applied to 2-D tensors only unless
                             decay_1d != 0                                           */
  float grad_clip;        /* global-norm clip threshold; <= 0 disables clipping      */
  int32_t decay_1d;
  int32_t recompute;      /* 0: keep every layer's activations for the backward.
                             1: activation recompute (checkpointing): per layer only
                             the residual stream, the norm statistics and the
                             attention LSE are kept; the backward re-runs each
                             layer's norms, QKV GEMM, attention forward and fc GEMM
                             from them before that layer's backward.  Results are
                             bit-identical to 0; the workspace holds one layer of
                             the other activations instead of L (14 M d elements
                             of the operand type per layer saved); gpt_generate is
                             GPT_ERR_UNSUPPORTED (its cache is those activations). */
  uint64_t dropout_seed;  /* key of the dropout counter hash                         */
  double init_std;        /* std of the Gaussian init of matrices and embeddings
                             (double: the init is computed in double precision and
                             rounded to fp32 once)                                   */
  int32_t zero_world;     /* ZeRO stage 1 (sharded optimiser state).  0 or 1: the
                             model holds every AdamW moment.  W in 2..64: the model
                             is rank zero_rank of W data-parallel replicas and its
                             workspace holds the moments of its own shard only
                             (gpt_zero1_shard); the optimiser step is then
                             gpt_clip_adamw_shard on that shard, and the calls that
                             need every moment (gpt_train_step*, without the
                             accumulate forms, gpt_clip_adamw_step, gpt_get_state,
                             gpt_set_state) return GPT_ERR_UNSUPPORTED.            */
  int32_t zero_rank;      /* 0 <= zero_rank < zero_world (0 when zero_world <= 1)    */
} gpt_config;

typedef struct gpt_model gpt_model;

/* ---------------------------------------------------------------- pure host */

/* Number of trainable parameters (padding excluded): for GPT2
 * V*d + T*d + L*(12 d^2 + 13 d) + 2 d (run log section 2.3 breakdown);
 * for MICRO 2*V*d + T*d + 12*L*d^2 (4192 at the microGPT size).
 * Returns 0 for an invalid config. */
size_t gpt_param_count(const gpt_config* cfg);

/* Bytes of device workspace a model with this config needs (out). */
gpt_status gpt_workspace_bytes(const gpt_config* cfg, size_t* out);

/* Which kernels a model with this config runs (pure host; out receives
 * GPT_PATH_* bits).  The choice is a fixed rule of the config, made once, and
 * never a fallback taken at run time (a kernel that cannot be launched is
 * GPT_ERR_CUDA):
 *   - GPT_PATH_GEMM_TC: bf16 mode.  Every dense contraction runs on the
 *     tcgen05 tensor-core GEMM, except products of at most 16 rows (the
 *     decoding step of gpt_generate), which run on the decoding GEMM (warp
 *     MMAs streaming the weights).  fp32 mode runs CUDA-core GEMMs.
 *   - GPT_PATH_ATTN_TC: bf16 mode with head_dim 64 and block_size a multiple
 *     of 128 (every bf16 workload of the pages' configurations).  The causal
 *     attention runs on the tcgen05 flash kernels; other shapes, and fp32
 *     mode, run the CUDA-core attention kernels. */
enum { GPT_PATH_GEMM_TC = 1u << 0, GPT_PATH_ATTN_TC = 1u << 1 };
gpt_status gpt_config_kernel_paths(const gpt_config* cfg, uint32_t* out);

/* get_lr of the practical guide, section 6: lr*it/warmup while it < warmup,
 * then lr*0.5*(1+cos(pi*(it-warmup)/(max_iters-warmup))).  Pure function. */
float gpt_lr_cosine(float lr, int32_t it, int32_t warmup, int32_t max_iters);
/* microGPT "核心训练循环": lr*(1 - it/max_iters).  Pure function. */
float gpt_lr_linear(float lr, int32_t it, int32_t max_iters);

/* ---------------------------------------------------------------- lifetime */

/* Creates a model in a caller-owned device workspace of `bytes` bytes
 * (>= gpt_workspace_bytes) and initialises its weights from `seed`
 * (matrices/embeddings ~ N(0, init_std^2) from a SplitMix64 counter hash
 * with Box-Muller, biases 0, norm gains 1; AdamW moments 0).  `cuda_stream`
 * is a cudaStream_t (NULL = legacy default stream).  Synchronises. */
gpt_status gpt_create(const gpt_config* cfg, uint64_t seed, void* d_workspace, size_t bytes,
                      void* cuda_stream, gpt_model** out);
void gpt_destroy(gpt_model* m);
gpt_status gpt_set_stream(gpt_model* m, void* cuda_stream);

/* ---------------------------------------------------------------- the step */

/* Forward pass and mean cross-entropy of one micro-batch.
 * d_idx, d_tgt: device int32 [batch_size, block_size] token ids and next-token
 * targets (owned by the caller, read during the call's device work).
 * h_loss (nullable): receives the loss (synchronises).
 * The dropout masks use the cursor set by gpt_set_dropout_cursor. */
gpt_status gpt_forward_loss(gpt_model* m, const int32_t* d_idx, const int32_t* d_tgt, float* h_loss);

/* Backward pass of the last gpt_forward_loss; gradients of loss/grad_accum
 * are ADDED into the fp32 gradient arena.  GPT_ERR_STATE without a
 * preceding forward. */
gpt_status gpt_backward(gpt_model* m);

/* Global-norm clip + one AdamW update of every parameter with learning rate
 * `lr` and bias-correction index `step` (>= 1); zeroes the gradients and
 * refreshes the bf16 weight copy.  h_grad_norm (nullable) receives the
 * pre-clip norm.  A non-finite norm skips the update on the device (weights
 * and moments unchanged, gradients still zeroed) and, when h_grad_norm is
 * given, returns GPT_ERR_NONFINITE. */
gpt_status gpt_clip_adamw_step(gpt_model* m, float lr, int32_t step, float* h_grad_norm);

/* One full optimiser step: for micro = 0..grad_accum-1, gather a batch of
 * random windows from the device-resident token stream (d_stream,
 * stream_len tokens of cfg.token_dtype), forward, backward; then clip +
 * AdamW with (lr, step).  Window starts: SplitMix64 hash of
 * (data_seed, step, micro, b) mod (stream_len - block_size).
 * Dropout counter = step*grad_accum + micro.  h_loss (mean over the
 * micro-batches) and h_grad_norm are nullable. */
gpt_status gpt_train_step(gpt_model* m, const void* d_stream, uint64_t stream_len, uint64_t data_seed,
                          float lr, int32_t step, float* h_loss, float* h_grad_norm);

/* Same step with the micro-batches supplied from HOST memory: h_idx and
 * h_tgt are int32 [grad_accum, batch_size, block_size] (pinned memory keeps
 * the copies asynchronous).  The host->device copies are part of the call. */
gpt_status gpt_train_step_host(gpt_model* m, const int32_t* h_idx, const int32_t* h_tgt, float lr,
                               int32_t step, float* h_loss, float* h_grad_norm);

/* CUDA-graph replay of gpt_train_step / gpt_train_step_host (default on;
 * gpt_generate is replayed under the same switch).
 * When on, and per-kernel timing is off, the first step of each kind runs
 * eagerly, the second is captured into a graph (on a stream the library
 * creates) and every later step replays it on the model's stream after a
 * one-thread kernel writes the step's index, lr and bias corrections to
 * device memory; the replayed kernels read them there, and derive their
 * dropout keys from that step index.  A new d_stream / stream_len /
 * data_seed triggers a new capture.  The replayed step runs the same kernels
 * on the same values as the eager one, so results are bit-identical.  A
 * capture that fails returns GPT_ERR_CUDA (that step did not run; graphs stay
 * on, and gpt_set_graphs(m, 0) runs every step eagerly). */
gpt_status gpt_set_graphs(gpt_model* m, int32_t on);

/* ---------------------------------------------------------------- data-parallel training
 * The nanoGPT README's multi-GPU training ("复现 GPT-2": torchrun over 8 GPUs
 * with DDP) averages the gradients of the replicas before the optimiser
 * step.  The library runs the step in two calls around that exchange; the
 * exchange itself is NCCL's all-reduce, issued by the caller (the Python
 * layer, gpt_decoder_lm_b200/ddp.py) on a second stream so that it overlaps
 * the rest of the backward:
 *   gpt_train_step_accumulate   gather + grad_accum forward/backward passes,
 *                               no optimiser; records one event per bucket of
 *                               the gradient arena as the last micro-batch's
 *                               backward makes the bucket final
 *   gpt_stream_wait_bucket      makes a stream wait for a bucket's event
 *   (caller)                    all-reduce (mean) of the bucket's ranges
 *   gpt_clip_adamw_step         clip + AdamW on the averaged gradients
 * gpt_grad_buckets gives the plan: the arena as ranges (element offset,
 * count) with their bucket, buckets in the order the backward finalises
 * them (bucket i < n_layer: layer n_layer-1-i; bucket n_layer: embeddings,
 * final norm, an untied head).  Pure host; with cap < the number of ranges
 * (or null arrays) only *n_ranges is written. */
gpt_status gpt_grad_buckets(const gpt_config* cfg, int32_t cap, int64_t* h_offset, int64_t* h_count,
                            int32_t* h_bucket, int32_t* n_ranges);
/* Mean loss of the last training step (gpt_train_step*, including the
 * accumulate forms).  Synchronising. */
gpt_status gpt_step_loss(gpt_model* m, float* h_loss);
/* Device address and length (floats) of the fp32 gradient arena. */
gpt_status gpt_grad_arena(gpt_model* m, float** d_grad, int64_t* n_floats);
/* The step of gpt_train_step without clip + AdamW; gradients are left in
 * the arena (added to what it holds).  Replayed as its own CUDA graph with
 * graphs on.  h_loss (nullable) as gpt_train_step.  GPT_ERR_UNSUPPORTED with
 * LoRA adapters attached. */
gpt_status gpt_train_step_accumulate(gpt_model* m, const void* d_stream, uint64_t stream_len, uint64_t data_seed,
                                     int32_t step, float* h_loss);
/* The same with the micro-batches from host memory (as gpt_train_step_host). */
gpt_status gpt_train_step_host_accumulate(gpt_model* m, const int32_t* h_idx, const int32_t* h_tgt, int32_t step,
                                          float* h_loss);
/* cudaStreamWaitEvent(cuda_stream, event of `bucket`) for the last
 * gpt_train_step_accumulate / gpt_train_step_host_accumulate. */
gpt_status gpt_stream_wait_bucket(gpt_model* m, int32_t bucket, void* cuda_stream);

/* ---------------------------------------------------------------- sharded optimiser (ZeRO stage 1)
 * The fine-tuning pipelines page's distributed-training paragraph points to
 * DeepSpeed ZeRO for models past DDP's reach; ZeRO's first stage shards the
 * optimiser step.  Each of `world` ranks owns one contiguous shard of the
 * arenas; the step becomes
 *   gpt_train_step_accumulate   as for DDP (bucket events included)
 *   (caller)                    per bucket, a sum-reduce of each part of the
 *                               bucket to the rank whose shard holds it
 *   gpt_grad_sumsq_shard        partial sums of squares of the own shard
 *   (caller)                    all-gather of every rank's partials
 *   gpt_clip_adamw_shard        clip by the global norm + AdamW on the own
 *                               shard only; the rest of the gradient arena
 *                               is cleared
 *   (caller)                    all-gather of the fp32 weights and their
 *                               bf16 copies (in place, shard by shard)
 * Every rank sums the same gathered partials in the same order, so the
 * norm and the clip factor are identical on every rank. */

/* Number of doubles gpt_grad_sumsq_shard writes. */
#define GPT_NORM_PARTIALS 592

/* Shard `rank` of `world` (1 <= world <= 64): elements [*offset, *offset +
 * *count) of the arenas, *stride = the shard length every rank but the last
 * has (a multiple of 64; world * *stride never exceeds the arenas'
 * allocated length, so an all-gather of `world` equal shards fits in
 * place).  *count is 0 for a rank past the end.  Pure host. */
gpt_status gpt_zero1_shard(const gpt_config* cfg, int32_t world, int32_t rank, int64_t* offset, int64_t* count,
                           int64_t* stride);
/* Device addresses of the model's flat arenas: fp32 weights, gradients, the
 * AdamW first and second moments, and the bf16 operand copy of the weights
 * (null in fp32 mode).  *n_floats elements are in use; the weight, gradient
 * and bf16 arenas are allocated for *n_alloc >= n_floats + 4096 elements (the
 * slack is never read by the step).  The moments use the same offsets and
 * length, except with zero_world > 1, where they hold the own shard only:
 * element offset + i of the arenas at index i, *n_moment_alloc = the shard
 * stride. */
gpt_status gpt_state_arenas(gpt_model* m, float** d_param, float** d_grad, float** d_adam_m, float** d_adam_v,
                            void** d_param_bf16, int64_t* n_floats, int64_t* n_alloc, int64_t* n_moment_alloc);
/* GPT_NORM_PARTIALS partial sums of squares (fp64, device) of gradient
 * elements [offset, offset + count) into d_partials; their sum is the
 * shard's squared norm.  offset and count multiples of 4 (the shard bounds
 * of gpt_zero1_shard are).  Asynchronous.  GPT_ERR_STATE with LoRA
 * adapters attached. */
gpt_status gpt_grad_sumsq_shard(gpt_model* m, int64_t offset, int64_t count, double* d_partials);
/* Clip + AdamW (as gpt_clip_adamw_step) on elements [offset, offset + count)
 * only, with the gradient taken as grad_scale times the arena's values (1 /
 * world for the mean of summed gradients) and its global norm as grad_scale
 * times the square root of the sum of the n_partials doubles at d_partials
 * (device; every rank's gpt_grad_sumsq_shard output, gathered in rank
 * order).  Clears the whole gradient arena.  h_grad_norm (nullable): the
 * global norm, read after a synchronise (GPT_ERR_NONFINITE as
 * gpt_clip_adamw_step).  With offset 0, count = the arena, grad_scale 1 and
 * the one rank's partials this is gpt_clip_adamw_step bit for bit.  With
 * zero_world > 1 in the config, offset and count must be the config's own
 * shard (the only moments the model holds), else GPT_ERR_INVALID_ARG. */
gpt_status gpt_clip_adamw_shard(gpt_model* m, float lr, int32_t step, int64_t offset, int64_t count,
                                float grad_scale, const double* d_partials, int32_t n_partials, float* h_grad_norm);

/* The batch gather of gpt_train_step on its own: writes int32
 * [batch_size, block_size] ids and targets to d_idx / d_tgt. */
gpt_status gpt_gather_batch(gpt_model* m, const void* d_stream, uint64_t stream_len, uint64_t data_seed,
                            int32_t step, int32_t micro, int32_t* d_idx, int32_t* d_tgt);

/* Dropout cursor used by gpt_forward_loss / gpt_backward: counter =
 * step*grad_accum + micro. */
gpt_status gpt_set_dropout_cursor(gpt_model* m, int32_t step, int32_t micro);

/* ---------------------------------------------------------------- evaluation and sampling */

/* Evaluation loss (nanoGPT README, train.py's estimate_loss: the mean loss of
 * eval_iters batches): the mean over n_batches >= 1 batches of the batch's
 * mean token loss, forward only, without dropout.  Batch i is the training
 * gather's window set for step i + 1, micro-batch 0, of d_stream /
 * data_seed (a validation stream and seed in practice).  Overwrites the
 * activations (a following gpt_backward is GPT_ERR_STATE); synchronising.
 * *h_loss receives the mean. */
gpt_status gpt_eval_loss(gpt_model* m, const void* d_stream, uint64_t stream_len, uint64_t data_seed,
                         int32_t n_batches, float* h_loss);

/* Autoregressive generation with a key / value cache (nanoGPT sample.py,
 * README section "采样 / 推理"; microGPT page, section "单 GPU 高效推理：
 * 采样 + KV Cache"): d_prompt int32 [batch_size, T0] (device), n_new >= 1
 * new tokens per row, T0 + n_new <= block_size.  The prompt runs through the
 * forward once (prefill); every further token costs one decoding step over
 * the batch rows, whose attention reads the keys / values of the earlier
 * positions from the forward's own qkv activations (the cache) and appends
 * its own.  Draws as gpt_sample with d_uniform fp32 [n_new, batch_size]
 * (device, row i for the i-th new token).  d_out int32 [batch_size,
 * T0 + n_new] (device) receives prompt and continuation.  No dropout.
 * Overwrites the activations (a following gpt_backward is GPT_ERR_STATE);
 * synchronising; GPT_ERR_TOKEN_RANGE for prompt ids outside the vocabulary.
 * With graphs on (gpt_set_graphs), a call repeating the previous call's
 * buffers, lengths and sampling parameters replays a CUDA graph of the whole
 * call (the first such call runs eagerly, the second is captured). */
gpt_status gpt_generate(gpt_model* m, const int32_t* d_prompt, int32_t T0, int32_t n_new, float temperature,
                        int32_t top_k, float top_p, const float* d_uniform, int32_t* d_out);

/* One draw from each of `rows` rows of logits (microGPT page, section
 * "单 GPU 高效推理：采样 + KV Cache"; nanoGPT sample.py): d_logits is
 * [rows, ld] (bf16 when logits_bf16, else fp32; device), V <= ld valid
 * columns.  temperature <= 0: greedy (arg-max, lowest index on ties).
 * Otherwise: top_k in (0, V) keeps the logits >= the k-th largest (ties
 * kept); p = exp((z - max) / temperature) over those; top_p < 1 keeps
 * p >= tau for the largest tau whose kept mass reaches top_p of the total
 * (top_p <= 0 keeps the maximum); the token is the first, in index order,
 * whose running kept mass exceeds d_uniform[row] (in [0, 1), device fp32)
 * times the kept mass.  d_out: int32 [rows] (device).  Asynchronous on
 * cuda_stream; GPT_ERR_INVALID_ARG on null pointers, rows < 1 or V < 1. */
gpt_status gpt_sample(const void* d_logits, int32_t logits_bf16, int32_t rows, int32_t V, int64_t ld,
                      float temperature, int32_t top_k, float top_p, const float* d_uniform, int32_t* d_out,
                      void* cuda_stream);

/* ---------------------------------------------------------------- introspection (tests, resume) */

gpt_status gpt_num_tensors(gpt_model* m, int32_t* n);
/* Name (static storage) and logical shape of tensor i in the canonical
 * order: wte, wpe, per layer ln_1.{weight,bias}, attn.c_attn.{weight,bias},
 * attn.c_proj.{weight,bias}, ln_2.{weight,bias}, mlp.c_fc.{weight,bias},
 * mlp.c_proj.{weight,bias} (MICRO: weights only), then ln_f.{weight,bias}
 * (GPT2) or lm_head.weight (MICRO).  shape[1] = 1 for vectors.  The logical
 * shape of wte / lm_head is [vocab_size, n_embd] (padding rows hidden). */
gpt_status gpt_tensor_info(gpt_model* m, int32_t i, const char** name, int64_t shape[2]);
/* Copies tensor i of the given kind (GPT_PARAM .. GPT_ADAM_V) as fp32
 * to / from host memory (shape as gpt_tensor_info).  Setting GPT_PARAM also
 * refreshes the bf16 copy.  Synchronising.  The moment kinds are
 * GPT_ERR_UNSUPPORTED with zero_world > 1 (the model holds one shard). */
gpt_status gpt_get_tensor(gpt_model* m, int32_t i, int32_t kind, float* h_out);
gpt_status gpt_set_tensor(gpt_model* m, int32_t i, int32_t kind, const float* h_in);
/* Logits of the last forward as fp32 [B*T, vocab_size] (pad columns
 * dropped), and their row argmax (ties -> lowest index) as int32 [B*T].
 * Valid between gpt_forward_loss and the next gpt_backward, which reuses the
 * logits buffer for the logits' gradient. */
gpt_status gpt_get_logits(gpt_model* m, float* h_out);
gpt_status gpt_get_argmax(gpt_model* m, int32_t* h_out);
/* Argmax of caller-supplied fp32 rows [rows, cols] held in device memory
 * (same kernel as gpt_get_argmax); h_out int32 [rows]. */
gpt_status gpt_argmax_rows(gpt_model* m, const float* d_rows, int32_t rows, int32_t cols, int32_t* h_out);
/* Per-row log-sum-exp of the last forward's logits, fp32 [B*T]. */
gpt_status gpt_get_lse(gpt_model* m, float* h_out);
/* The embedding-gradient routing of the last backward: number of distinct
 * token ids touched (h_n_unique), the sorted token of each position
 * (h_sorted_tok int32 [B*T]) and the position each sorted slot came from
 * (h_sorted_pos int32 [B*T]); positions of one token are ascending. */
gpt_status gpt_get_embed_routing(gpt_model* m, int32_t* h_n_unique, int32_t* h_sorted_tok, int32_t* h_sorted_pos);
/* Dropout keep mask of one site as uint8 [n] for elements [0, n) of
 * (counter, layer, site) -- the same device function the kernels use. */
gpt_status gpt_dropout_mask(gpt_model* m, int64_t counter, int32_t layer, int32_t site, int64_t n, uint8_t* h_out);

/* Optimiser state for checkpoint / resume: fp32 master weights, AdamW m and
 * v (each gpt_param_count()-sized in canonical tensor order) and the step
 * counter.  Buffers are host memory of state_floats() floats each. */
size_t gpt_state_floats(gpt_model* m);
gpt_status gpt_get_state(gpt_model* m, float* h_param, float* h_m, float* h_v);
gpt_status gpt_set_state(gpt_model* m, const float* h_param, const float* h_m, const float* h_v);

/* Device flag word (GPT_FLAG_*) since the last gpt_clear_flags; synchronising. */
gpt_status gpt_read_flags(gpt_model* m, uint32_t* h_flags);
gpt_status gpt_clear_flags(gpt_model* m);

/* Per-kernel timing of the last step (CUDA events on the model's stream):
 * enable with on != 0; gpt_kernel_times copies up to `cap` (name, total ms,
 * launches) records.  Used by the bench's roofline report. */
gpt_status gpt_enable_timing(gpt_model* m, int32_t on);
gpt_status gpt_kernel_times(gpt_model* m, int32_t cap, const char** names, float* total_ms, int32_t* launches,
                            int32_t* n_out);
/* Number of kernel launches the library made since the model was created. */
uint64_t gpt_launch_count(gpt_model* m);

const char* gpt_last_error(const gpt_model* m);
const char* gpt_status_string(gpt_status s);

/* ---------------------------------------------------------------- allocation-free entry point */

/* The pages have no counterpart of this entry point: it exists for callers
 * that cannot allocate device memory -- code inside a plugin or
 * custom-operator interface that only hands over its input and output
 * buffers, a process whose device memory belongs to another allocator or
 * pool, or work that must not call cudaMalloc (it synchronises the whole
 * device).
 *
 * Weight-gradient GEMM of the training step, dW[M, N] += sum_k A[k, m] *
 * B[k, n], on the tensor cores: A is bf16 [K, M] row-major with pitch lda,
 * B is bf16 [K, N] with pitch ldb (the layouts of a layer's output gradient
 * and input activations, tokens outermost), dW is fp32 [M, N] with pitch N.
 * The contraction is split into split_k ranges whose partial sums go to a
 * 16 MiB array inside the library (split_k * M * N <= 4,194,304 floats;
 * larger requests return GPT_ERR_WORKSPACE_TOO_SMALL) and are added to dW in
 * a fixed order, so the result matches the same GEMM run with caller-provided
 * scratch.  Nothing is allocated: no cudaMalloc, cudaFree or allocating
 * library call.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address.
 *   - Every GPU that loads the library holds the array until the process
 *     exits.  All calls share it and it keeps the last call's contents (every
 *     partial sum is written before it is read, so nothing needs clearing);
 *     calls whose GPU work overlaps -- on two streams at once, or from two
 *     threads -- race on it.
 *   - Work is enqueued on cuda_stream (a cudaStream_t) and the call
 *     synchronises that stream before returning.  A CUDA error left pending
 *     by the caller's own earlier work is neither reported nor cleared.
 * Returns GPT_ERR_INVALID_ARG for bad sizes or NULL pointers,
 * GPT_ERR_UNSUPPORTED when the shape or alignment does not suit the tensor
 * cores (pitches multiple of 8, M and N multiple of 8, 16-byte aligned
 * pointers), GPT_ERR_TIMEOUT if a bounded wait in the kernel ran out,
 * GPT_ERR_CUDA for a CUDA failure. */
gpt_status gpt_gemm_dw_accumulate_noalloc(int32_t M, int32_t N, int32_t K, const void* d_a, int64_t lda,
                                          const void* d_b, int64_t ldb, float* d_dw, int32_t split_k,
                                          void* cuda_stream);

/* ---------------------------------------------------------------- LoRA adapters
 * Low-rank adapters on row blocks of each layer's fused QKV weight ("使用
 * nanoGPT 构建中型 GPT 微调管道" page, LoRA integration paragraph): the base
 * weights stay frozen and a block computes h = W0 x + s B (A x), s = alpha / r,
 * A [r, d], B [d, r].  targets: bit 0 q (rows 0..d-1), bit 1 k (d..2d-1),
 * bit 2 v (2d..3d-1); the page adapts q and v (targets = 5).  Adapter layout
 * (params, grads, Adam moments alike): per adapted block, layers ascending and
 * q, k, v ascending within a layer, A row-major then B row-major.
 * While attached, gpt_train_step / gpt_train_step_host / gpt_clip_adamw_step
 * train the adapters only: the step's forward and backward run on the merged
 * operand W0 + s B A, the adapters' gradients follow from the merged blocks'
 * gradient G (dB = s G A^T, dA = s B^T G), clip + AdamW (the config's
 * hyper-parameters; every adapter tensor decayed) run over the adapters, and
 * the base weights and their Adam state are not touched.  The reported grad
 * norm is the adapters'.  bf16 models only (GPT_ERR_UNSUPPORTED otherwise). */

/* Bytes of device memory the adapters of (cfg, r, targets) need. */
gpt_status gpt_lora_workspace_bytes(const gpt_config* cfg, int32_t r, int32_t targets, size_t* out);

/* Attaches adapters of rank r (1..256) on `targets`: h_a (host) holds A of
 * every adapted block ([blocks][r][d] fp32; random numbers are inputs), B
 * starts at zero, so the model is unchanged until the first step.  d_ws:
 * device memory of gpt_lora_workspace_bytes, 256-byte aligned, owned by the
 * caller until detach.  Replaces adapters already attached.  Synchronising. */
gpt_status gpt_lora_attach(gpt_model* m, int32_t r, float alpha, int32_t targets, const float* h_a, void* d_ws,
                           size_t ws_bytes);

/* Detaches the adapters: the QKV operands return to the base weights (the
 * adapters are not merged into them).  Synchronising; no-op when none. */
gpt_status gpt_lora_detach(gpt_model* m);

/* Copies the adapter parameters (which 0), their gradients (1: formed by the
 * backward of the step's last micro-batch, zero again after the optimiser
 * step), or the Adam moments (2, 3) to host memory; count must be the adapter
 * size.  Synchronising. */
gpt_status gpt_lora_read(gpt_model* m, int32_t which, float* h_out, size_t count);

/* Replaces the adapter parameters (host, adapter layout) and rebuilds the
 * merged operands.  Synchronising. */
gpt_status gpt_lora_write(gpt_model* m, const float* h_params, size_t count);

#ifdef __cplusplus
}
#endif
#endif /* GPT_B200_H */
