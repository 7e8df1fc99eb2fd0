// Step engine behind the C ABI of include/gpt.h: validates the config, lays
// out every device buffer inside the caller's workspace, initialises the
// weights from the seed, and enqueues the kernels of one training step on the
// model's stream.  No device allocation happens here.
#include <math.h>
#include <stdlib.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <string>
#include <thread>
#include <vector>

#include "../../include/gpt.h"
#include "kernels.cuh"

using namespace gpt;

// ============================================================================
// timing by kernel name (CUDA events on the model's stream)
// ============================================================================
namespace gpt {
struct Timing {
  struct Rec {
    std::vector<cudaEvent_t> ev;  // begin/end pairs
    int launches = 0;
  };
  std::map<std::string, Rec> recs;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  cudaEvent_t get() {
    if (used == pool.size()) {
      cudaEvent_t e;
      cudaEventCreate(&e);
      pool.push_back(e);
    }
    return pool[used++];
  }
  void reset() {
    recs.clear();
    used = 0;
  }
  ~Timing() {
    for (auto e : pool) cudaEventDestroy(e);
  }
};
void timing_begin(Ctx& c, const char* name) {
  auto& r = c.timing->recs[name];
  cudaEvent_t e = c.timing->get();
  cudaEventRecord(e, c.stream);
  r.ev.push_back(e);
  r.launches++;
}
void timing_end(Ctx& c, const char* name) {
  auto& r = c.timing->recs[name];
  cudaEvent_t e = c.timing->get();
  cudaEventRecord(e, c.stream);
  r.ev.push_back(e);
}
}  // namespace gpt

// ============================================================================
// model
// ============================================================================
namespace {

struct TensorRec {
  std::string name;
  int64_t rows, cols;   // logical shape (cols = 1 for vectors)
  int64_t alloc_rows;   // rows in the arena (wte / lm_head: padded vocab)
  int64_t off;          // element offset in the arenas
  int init;             // 0 normal, 1 ones, 2 zeros
  bool decay;
};

struct LayerP {  // element offsets of one block's tensors (-1 when absent)
  int64_t ln1_w = -1, ln1_b = -1, qkv_w, qkv_b = -1, ap_w, ap_b = -1, ln2_w = -1, ln2_b = -1, fc_w, fc_b = -1, pr_w,
          pr_b = -1;
};

struct Layout {
  size_t off = 0;
  size_t take(size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  }
};

// Elements allocated past the last tensor of every arena: an all-gather of
// `world` equal shards of ceil(n / world / 64) * 64 elements (world <= 64)
// overruns the arena by less than 64 * 64.
constexpr int64_t kArenaSlack = 64 * 64;
constexpr int kZeroMaxWorld = 64;

// shard `rank` of `world` over an arena of n elements: equal strides that are
// multiples of 64, the last one ragged (or empty)
void zero_shard_of(int64_t n, int world, int rank, int64_t* off, int64_t* cnt, int64_t* stride) {
  const int64_t S = ((n + world - 1) / world + 63) / 64 * 64;
  *stride = S;
  *off = std::min<int64_t>((int64_t)rank * S, n);
  *cnt = std::max<int64_t>(0, std::min<int64_t>(S, n - *off));
}

// split-K count of a weight-gradient GEMM (sizes the partial-sum scratch; the
// plan of a 148-SM B200)
int choose_splits(long M, long N, long K) { return gemm_tc_plan(M, N, K, true, 148).splits; }

}  // namespace

struct gpt_model {
  gpt_config cfg;
  int V, Vp, L, H, d, T, B, ga, hd;
  long M;
  bool bf16m, micro;
  bool rc;     // activation recompute: one slot of per-layer activations
  size_t asz;  // bytes per activation element (2 bf16 / 4 fp32)
  std::vector<TensorRec> tensors;
  std::vector<LayerP> layers;
  int64_t wte, wpe, lnf_w = -1, lnf_b = -1, head;  // offsets
  int64_t n_total = 0, n_decay = 0;
  // ZeRO-1 (zero_world > 1): the moments hold this rank's shard only
  bool zero_sharded = false;
  int64_t zero_off = 0, zero_cnt = 0, zero_stride = 0;

  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  // arenas
  float *w = nullptr, *g = nullptr, *am = nullptr, *av = nullptr;
  bf16* wb = nullptr;
  // activations
  float* res;  // [(2L+1), M, d]
  uint8_t *ln1, *qkv, *atto, *ln2, *fch, *fcg, *lnf, *logits;
  float *ln1_mean, *ln1_rstd, *ln2_mean, *ln2_rstd, *lnf_mean, *lnf_rstd, *lse;
  float *row_loss, *row_lse;
  int32_t *idx, *tgt, *stage_idx, *stage_tgt;
  // backward scratch
  float *dres, *dln, *dsum, *splitk, *seg;
  uint8_t *dyb, *dqkv, *datt, *dh;
  int32_t *stok, *spos, *nuniq;
  double* norm_part;
  float* scal;  // [0] micro loss, [1] step loss, [2] grad norm, [3] flags (uint32)
  int32_t* argmax_out;
  size_t splitk_floats = 0;
  int part_blocks = 0;
  // Reductions deferred to the last micro-batch of a step: the column
  // partials of every norm backward and bias column sum, and the split-K
  // partials of every weight-gradient GEMM, accumulate across micro-batches
  // in per-instance buffers and are added to the gradients once per step.
  int cur_micro = 0, n_micro = 1;
  // a training step gathers every micro-batch's tokens first and sorts their
  // embedding-gradient routing in one launch (one CTA per micro-batch)
  int32_t *idx_all = nullptr, *tgt_all = nullptr, *stok_all = nullptr, *spos_all = nullptr, *nuniq_all = nullptr;
  int32_t *idx0 = nullptr, *tgt0 = nullptr;  // the stand-alone forward's buffers
  bool presorted = false;
  // decoding scratch, [B] rows of one position each
  int32_t* dec_tok = nullptr;
  float *dec_res = nullptr, *dec_mean = nullptr, *dec_rstd = nullptr;
  uint8_t *dec_a = nullptr, *dec_o = nullptr, *dec_dact = nullptr, *dec_g = nullptr, *dec_logits = nullptr;
  // CUDA-graph replay of gpt_generate for a repeated call shape
  cudaGraphExec_t gen_exec = nullptr;
  int gen_warm = 0;
  bool capturing = false;  // a graph of the step is being captured
  uint64_t gen_launches = 0;
  uint64_t gen_key[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int part_cap = 0;                 // partial rows per norm instance
  float* norm_parts = nullptr;      // [2L+1][part_cap][3][d]
  float* colsum_parts = nullptr;    // [L][2][colsum_rows][4d]
  long colsum_rows = 0;             // partial rows per instance: row chunks, or 32-row groups
  float* split_parts = nullptr;     // per (layer, dW kind): [splits, Mo, No]
  std::vector<size_t> split_off;    // offset of each (layer, kind) instance; kind: 0 mlp proj, 1 fc, 2 attn proj, 3 qkv
  std::vector<int> split_n;         // its split count (1: no split buffer)

  Ctx ctx;
  Timing* timing = nullptr;
  // CUDA-graph replay of the full step: [0] device token stream, [1] host batches
  bool graphs_on = true;
  cudaStream_t cap_stream = nullptr;
  struct {
    bool on = false;
    int targets = 0;
    float alpha = 0.f;
    LoraBlocks lb;
    float *m = nullptr, *v = nullptr;  // Adam moments of the adapters
    long n = 0;                        // adapter parameters (2 r d per block)
  } lora;
  // graph kinds: [0] device token stream, [1] host batches, [2] / [3] the
  // same without the optimiser (the data-parallel step's accumulate part)
  cudaGraphExec_t gexec[4] = {nullptr, nullptr, nullptr, nullptr};
  uint64_t graph_launches[4] = {0, 0, 0, 0};
  int warm[4] = {0, 0, 0, 0};
  const void* g_dstream[4] = {nullptr, nullptr, nullptr, nullptr};
  uint64_t g_len[4] = {0, 0, 0, 0}, g_seed[4] = {0, 0, 0, 0};
  // data-parallel gradient exchange: one event per bucket of the gradient
  // arena, recorded in the last micro-batch's backward as the bucket's
  // gradients become final (gpt_train_step_accumulate)
  bool bucket_record = false;
  std::vector<cudaEvent_t> bucket_ev;
  int* step_dev = nullptr;     // per-step scalars read by replayed graphs
  float* hyper_dev = nullptr;  // {lr, 1 - b1^t, 1 - b2^t}
  bool dev_keys = false;  // dropout keys from the device step index (a graph being captured)
  bool attn_tc = false;   // attention on the tensor-core kernels (gpt_config_kernel_paths)
  bool have_forward = false;
  bool ce_grad_done = false;
  int64_t drop_counter = 0;
  uint32_t reported = 0;
  std::string err;

  float* P(int64_t off) const { return w + off; }
  float* G(int64_t off) const { return g + off; }
  const void* Wop(int64_t off) const {  // GEMM operand copy of a weight
    return bf16m ? (const void*)(wb + off) : (const void*)(w + off);
  }
};

namespace {

gpt_status fail(gpt_model* m, gpt_status s, const char* fmt, ...) {
  if (m) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    m->err = buf;
  }
  return s;
}

gpt_status check_cuda(gpt_model* m, const char* where) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(m, GPT_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
  return GPT_OK;
}

// Validation of a config; fills derived fields when m != nullptr.
gpt_status validate(const gpt_config* c, std::string* why) {
  auto bad = [&](const char* s) {
    if (why) *why = s;
    return GPT_ERR_CONFIG;
  };
  if (!c) {
    if (why) *why = "null config";
    return GPT_ERR_INVALID_ARG;
  }
  if (c->abi_version != GPT_ABI_VERSION) return bad("abi_version mismatch");
  if (c->vocab_size < 2 || c->vocab_size > 65535) return bad("vocab_size must be in [2, 65535]");
  int Vp = c->padded_vocab ? c->padded_vocab : ((c->vocab_size + 63) / 64) * 64;
  if (Vp < c->vocab_size || Vp % 64) return bad("padded_vocab must be >= vocab_size and a multiple of 64");
  if (c->n_layer < 1 || c->n_head < 1 || c->n_embd < 8) return bad("n_layer, n_head >= 1 and n_embd >= 8 required");
  if (c->n_embd % c->n_head) return bad("n_embd must be divisible by n_head");
  int hd = c->n_embd / c->n_head;
  if (hd != 4 && hd != 8 && hd != 16 && hd != 32 && hd != 64 && hd != 128) return bad("head_dim must be 4..128, power of 2");
  if (c->n_embd % 8) return bad("n_embd must be a multiple of 8");
  if (c->n_embd > 2048) return bad("n_embd must be <= 2048");
  if (c->block_size < 1 || c->batch_size < 1 || c->grad_accum < 1) return bad("block_size, batch_size, grad_accum >= 1");
  long M = (long)c->block_size * c->batch_size;
  if (M > 32768) return bad("batch_size * block_size must be <= 32768");
  if (c->precision != GPT_PREC_FP32 && c->precision != GPT_PREC_BF16) return bad("precision");
  if (c->variant != GPT_VARIANT_GPT2 && c->variant != GPT_VARIANT_MICRO) return bad("variant");
  if (c->token_dtype != GPT_TOK_I32 && c->token_dtype != GPT_TOK_U16) return bad("token_dtype");
  if (!(c->dropout >= 0.f && c->dropout < 1.f)) return bad("dropout must be in [0, 1)");
  if (!(c->beta1 >= 0.f && c->beta1 < 1.f && c->beta2 >= 0.f && c->beta2 < 1.f)) return bad("betas in [0, 1)");
  if (!(c->eps > 0.f) || !(c->init_std >= 0.0)) return bad("eps > 0 and init_std >= 0 required");
  if (c->recompute != 0 && c->recompute != 1) return bad("recompute must be 0 or 1");
  if (c->zero_world < 0 || c->zero_world > kZeroMaxWorld) return bad("zero_world must be in [0, 64]");
  if (c->zero_rank < 0 || c->zero_rank >= std::max(1, c->zero_world)) return bad("zero_rank must be in [0, zero_world)");
  return GPT_OK;
}

// tensor table in canonical order; returns arena sizes
void build_tensors(gpt_model& m) {
  int V = m.V, Vp = m.Vp, d = m.d, T = m.T, L = m.L;
  bool gpt2 = !m.micro;
  std::vector<TensorRec> t;
  auto add = [&](const std::string& n, int64_t r, int64_t c, int64_t ar, int init) {
    TensorRec x;
    x.name = n;
    x.rows = r;
    x.cols = c;
    x.alloc_rows = ar;
    x.off = -1;
    x.init = init;
    x.decay = (c > 1) || m.cfg.decay_1d;
    t.push_back(x);
  };
  add("wte", V, d, Vp, 0);
  add("wpe", T, d, T, 0);
  for (int l = 0; l < L; l++) {
    std::string p = "h." + std::to_string(l) + ".";
    if (gpt2) {
      add(p + "ln_1.weight", d, 1, d, 1);
      add(p + "ln_1.bias", d, 1, d, 2);
    }
    add(p + "attn.c_attn.weight", 3 * d, d, 3 * d, 0);
    if (gpt2) add(p + "attn.c_attn.bias", 3 * d, 1, 3 * d, 2);
    add(p + "attn.c_proj.weight", d, d, d, 0);
    if (gpt2) {
      add(p + "attn.c_proj.bias", d, 1, d, 2);
      add(p + "ln_2.weight", d, 1, d, 1);
      add(p + "ln_2.bias", d, 1, d, 2);
    }
    add(p + "mlp.c_fc.weight", 4 * d, d, 4 * d, 0);
    if (gpt2) add(p + "mlp.c_fc.bias", 4 * d, 1, 4 * d, 2);
    add(p + "mlp.c_proj.weight", d, 4 * d, d, 0);
    if (gpt2) add(p + "mlp.c_proj.bias", d, 1, d, 2);
  }
  if (gpt2) {
    add("ln_f.weight", d, 1, d, 1);
    add("ln_f.bias", d, 1, d, 2);
  } else {
    add("lm_head.weight", V, d, Vp, 0);
  }
  // arena: decayed tensors first, each aligned to 64 elements
  int64_t off = 0;
  for (int pass = 0; pass < 2; pass++) {
    for (auto& x : t) {
      if (x.decay != (pass == 0)) continue;
      x.off = off;
      off += ((x.alloc_rows * x.cols + 63) / 64) * 64;
    }
    if (pass == 0) m.n_decay = off;
  }
  m.n_total = off;
  m.tensors = t;
  // named offsets
  auto find = [&](const std::string& n) -> int64_t {
    for (auto& x : m.tensors)
      if (x.name == n) return x.off;
    return -1;
  };
  m.wte = find("wte");
  m.wpe = find("wpe");
  m.layers.assign(L, LayerP());
  for (int l = 0; l < L; l++) {
    std::string p = "h." + std::to_string(l) + ".";
    LayerP& y = m.layers[l];
    y.ln1_w = find(p + "ln_1.weight");
    y.ln1_b = find(p + "ln_1.bias");
    y.qkv_w = find(p + "attn.c_attn.weight");
    y.qkv_b = find(p + "attn.c_attn.bias");
    y.ap_w = find(p + "attn.c_proj.weight");
    y.ap_b = find(p + "attn.c_proj.bias");
    y.ln2_w = find(p + "ln_2.weight");
    y.ln2_b = find(p + "ln_2.bias");
    y.fc_w = find(p + "mlp.c_fc.weight");
    y.fc_b = find(p + "mlp.c_fc.bias");
    y.pr_w = find(p + "mlp.c_proj.weight");
    y.pr_b = find(p + "mlp.c_proj.bias");
  }
  m.lnf_w = find("ln_f.weight");
  m.lnf_b = find("ln_f.bias");
  m.head = gpt2 ? m.wte : find("lm_head.weight");
}

void derive(gpt_model& m, const gpt_config* c) {
  m.cfg = *c;
  m.V = c->vocab_size;
  m.Vp = c->padded_vocab ? c->padded_vocab : ((c->vocab_size + 63) / 64) * 64;
  m.L = c->n_layer;
  m.H = c->n_head;
  m.d = c->n_embd;
  m.T = c->block_size;
  m.B = c->batch_size;
  m.ga = c->grad_accum;
  m.hd = m.d / m.H;
  m.M = (long)m.B * m.T;
  m.bf16m = c->precision == GPT_PREC_BF16;
  m.micro = c->variant == GPT_VARIANT_MICRO;
  m.rc = c->recompute != 0;
  m.asz = m.bf16m ? 2 : 4;
  build_tensors(m);
  m.zero_sharded = c->zero_world > 1;
  if (m.zero_sharded) zero_shard_of(m.n_total, c->zero_world, c->zero_rank, &m.zero_off, &m.zero_cnt, &m.zero_stride);
}

// Carves the workspace (base may be null to size it).  Returns total bytes.
size_t carve(gpt_model& m, uint8_t* base) {
  Layout lay;
  auto F = [&](size_t n) { return (float*)(base + lay.take(n * 4)); };
  auto Bt = [&](size_t n) { return base + lay.take(n * m.asz); };
  auto I = [&](size_t n) { return (int32_t*)(base + lay.take(n * 4)); };
  long M = m.M;
  int d = m.d, L = m.L;
  // the arenas carry kArenaSlack elements past the last tensor: room for an
  // in-place all-gather of equal optimiser shards (gpt_zero1_shard)
  size_t P = (size_t)(m.n_total + kArenaSlack);
  m.scal = F(64);
  m.w = F(P);
  m.g = F(P);
  const size_t Pm = m.zero_sharded ? (size_t)m.zero_stride : P;  // moments: the own shard under ZeRO-1
  m.am = F(Pm);
  m.av = F(Pm);
  m.wb = m.bf16m ? (bf16*)(base + lay.take(P * 2)) : nullptr;
  const int La = m.rc ? 1 : L;  // slots of the recomputable activations
  m.res = F((size_t)(2 * L + 1) * M * d);
  m.ln1 = Bt((size_t)La * M * d);
  m.ln1_mean = F((size_t)L * M);
  m.ln1_rstd = F((size_t)L * M);
  m.qkv = Bt((size_t)La * M * 3 * d);
  m.atto = Bt((size_t)La * M * d);
  m.lse = F((size_t)L * M * m.H);
  m.ln2 = Bt((size_t)La * M * d);
  m.ln2_mean = F((size_t)L * M);
  m.ln2_rstd = F((size_t)L * M);
  m.fch = Bt((size_t)La * M * 4 * d);
  m.fcg = Bt((size_t)La * M * 4 * d);
  m.lnf = Bt((size_t)M * d);
  m.lnf_mean = F(M);
  m.lnf_rstd = F(M);
  m.logits = Bt((size_t)M * m.Vp);
  m.row_loss = F(M);
  m.row_lse = F(M);
  m.idx = I(M);
  m.tgt = I(M);
  m.stage_idx = I((size_t)m.ga * M);
  m.stage_tgt = I((size_t)m.ga * M);
  m.dres = F((size_t)M * d);
  m.dln = F((size_t)M * d);
  m.dsum = F((size_t)M * m.H);
  m.part_blocks = (int)std::min<long>(M, 148 * 8);  // capacity; the launch count is set at create
  m.part_cap = m.part_blocks;
  m.norm_parts = F((size_t)(2 * L + 1) * m.part_cap * 3 * d);
  m.colsum_rows = std::max<long>(colsum_chunks(M), (M + 31) / 32);
  m.colsum_parts = F((size_t)L * 2 * m.colsum_rows * 4 * d);
  {
    // weight-gradient shapes [Mo, No] of the four per-layer GEMMs
    const long dw[4][2] = {{d, 4L * d}, {4L * d, d}, {d, d}, {3L * d, d}};
    m.split_off.assign((size_t)L * 4, 0);
    m.split_n.assign((size_t)L * 4, 1);
    size_t tot = 0;
    for (int l = 0; l < L; l++)
      for (int k = 0; k < 4; k++) {
        const int sp = m.bf16m ? choose_splits(dw[k][0], dw[k][1], M) : 1;
        m.split_off[(size_t)l * 4 + k] = tot;
        m.split_n[(size_t)l * 4 + k] = sp;
        if (sp > 1) tot += (size_t)sp * dw[k][0] * dw[k][1];
      }
    m.split_parts = F(std::max<size_t>(tot, 64));
  }
  // split-K scratch: the largest dW partial set
  size_t sk = 0;
  long shapes[4][2] = {{3L * d, d}, {d, d}, {4L * d, d}, {d, 4L * d}};
  for (auto& s : shapes) {
    int sp = choose_splits(s[0], s[1], M);
    if (sp > 1) sk = std::max(sk, (size_t)sp * s[0] * s[1]);
  }
  {
    int sp = choose_splits(m.Vp, d, M);
    if (sp > 1) sk = std::max(sk, (size_t)sp * m.Vp * d);
  }
  m.splitk_floats = sk;
  m.splitk = F(std::max<size_t>(sk, 64));
  m.dyb = Bt((size_t)M * d);
  m.dqkv = Bt((size_t)M * 3 * d);
  m.datt = Bt((size_t)M * d);
  m.dh = Bt((size_t)M * 4 * d);
  m.seg = F((size_t)2 * ((M + 31) / 32) * d);
  m.stok = I(M);
  m.spos = I(M);
  m.nuniq = I(64);
  m.idx_all = I((size_t)m.ga * M);
  m.tgt_all = I((size_t)m.ga * M);
  m.stok_all = I((size_t)m.ga * M);
  m.spos_all = I((size_t)m.ga * M);
  m.nuniq_all = I((size_t)m.ga + 64);
  m.idx0 = m.idx;
  m.tgt0 = m.tgt;
  m.dec_tok = I((size_t)m.B + 64);
  m.dec_res = F((size_t)m.B * d);
  m.dec_mean = F((size_t)m.B + 64);
  m.dec_rstd = F((size_t)m.B + 64);
  m.dec_a = Bt((size_t)m.B * d);
  m.dec_o = Bt((size_t)m.B * d);
  m.dec_dact = Bt((size_t)m.B * 4 * d);
  m.dec_g = Bt((size_t)m.B * 4 * d);
  m.dec_logits = Bt((size_t)m.B * m.Vp);
  m.norm_part = (double*)(base + lay.take(148 * 4 * 8 + 64));
  m.argmax_out = I(M + 64);
  return lay.off + 1024;
}

// ---------------------------------------------------------------- host init
uint64_t sm64(uint64_t x) { return splitmix64(x); }

void init_tensor_host(const TensorRec& t, double std_, uint64_t seed, int index, float* out /* rows*cols */) {
  int64_t n = t.rows * t.cols;
  if (t.init == 1) {
    std::fill(out, out + n, 1.0f);
    return;
  }
  if (t.init == 2) {
    std::fill(out, out + n, 0.0f);
    return;
  }
  uint64_t k = sm64(seed ^ sm64((uint64_t)index));
  unsigned nt = std::max(1u, std::min(64u, std::thread::hardware_concurrency()));
  if (n < (1 << 16)) nt = 1;
  std::vector<std::thread> th;
  for (unsigned w = 0; w < nt; w++) {
    th.emplace_back([=] {
      int64_t a = n * w / nt, b = n * (w + 1) / nt;
      for (int64_t e = a; e < b; e++) {
        uint64_t b1 = sm64(k ^ (uint64_t)(2 * e));
        uint64_t b2 = sm64(k ^ (uint64_t)(2 * e + 1));
        double u1 = ((double)(b1 >> 11) + 1.0) * (1.0 / 9007199254740992.0);
        double u2 = (double)(b2 >> 11) * (1.0 / 9007199254740992.0);
        double z = sqrt(-2.0 * log(u1)) * cos(2.0 * 3.14159265358979323846 * u2);
        out[e] = (float)(std_ * z);
      }
    });
  }
  for (auto& x : th) x.join();
}

gpt_status sync_and_flags(gpt_model* m, const char* where, float* h_scal /* 4 floats or null */) {
  float tmp[4];
  cudaMemcpyAsync(tmp, m->scal, 16, cudaMemcpyDeviceToHost, m->ctx.stream);
  cudaError_t e = cudaStreamSynchronize(m->ctx.stream);
  if (e != cudaSuccess) return fail(m, GPT_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
  if (h_scal) memcpy(h_scal, tmp, 16);
  uint32_t fl;
  memcpy(&fl, &tmp[3], 4);
  uint32_t fresh = fl & ~m->reported;
  m->reported |= fl;
  if (fresh & FLAG_TIMEOUT) return fail(m, GPT_ERR_TIMEOUT, "%s: a bounded device wait ran out", where);
  if (fresh & FLAG_TOKEN) return fail(m, GPT_ERR_TOKEN_RANGE, "%s: token id outside [0, vocab_size)", where);
  if (fresh & (FLAG_LOSS | FLAG_NORM)) return fail(m, GPT_ERR_NONFINITE, "%s: non-finite loss or gradient norm", where);
  return GPT_OK;
}

// ---------------------------------------------------------------- step pieces
// fp32 mode: CUDA-core GEMM.  bf16 mode: the tensor-core GEMM, or the
// decoding GEMM for at most 16 rows; every bf16 shape of a valid config suits
// one of them, so false means the launch failed (a tensor map that could not
// be encoded), never a switch to another kernel.
bool gemm(gpt_model* m, GemmDesc& g) {
  if (!m->bf16m) {
    gemm_simt_f32(m->ctx, g);
    return true;
  }
  if (gemm_skinny_supported(g)) {
    gemm_skinny_bf16(m->ctx, g);
    return true;
  }
  if (!gemm_tc_supported(g)) return false;
  return gemm_tc_bf16(m->ctx, g);
}

// causal attention: the tensor-core kernels where the config's shape rule
// allows them (bf16, head_dim 64, T a multiple of 128), else the CUDA-core
// kernels; decided once per model, a failed launch is an error
template <typename T>
gpt_status attention(gpt_model* m, const AttnDesc& ad, bool backward) {
  if (m->attn_tc) {
    const bool ok = attn_tc_supported(ad) && (backward ? attn_bwd_tc(m->ctx, ad) : attn_fwd_tc(m->ctx, ad));
    if (!ok) return fail(m, GPT_ERR_CUDA, "tensor-core attention could not be launched (tensor map encode failed)");
    return GPT_OK;
  }
  if (backward) attn_bwd_simt<T>(m->ctx, ad);
  else attn_fwd_simt<T>(m->ctx, ad);
  return GPT_OK;
}

GemmDesc gd(int M, int N, int K, const void* A, long lda, bool ak, const void* B, long ldb, bool bk) {
  GemmDesc g;
  g.M = M;
  g.N = N;
  g.K = K;
  g.A = A;
  g.lda = lda;
  g.a_kmajor = ak;
  g.B = B;
  g.ldb = ldb;
  g.b_kmajor = bk;
  return g;
}

DropKey dkey(gpt_model* m, int layer, int site) {
  if (m->dev_keys)
    return make_drop_key_dev(m->cfg.dropout_seed, m->step_dev, m->ga, m->cur_micro, layer, site, m->cfg.dropout);
  return make_drop_key(m->cfg.dropout_seed, (uint64_t)m->drop_counter, layer, site, m->cfg.dropout);
}

template <typename T> T* at(uint8_t* base, size_t elems) { return reinterpret_cast<T*>(base) + elems; }

// Bucket i of the data-parallel gradient exchange is final: record its event
// on the model's stream (an external event node when a graph is captured).
void record_bucket(gpt_model* m, int i) {
  if (!m->bucket_record || i >= (int)m->bucket_ev.size()) return;
  if (m->capturing) cudaEventRecordWithFlags(m->bucket_ev[i], m->ctx.stream, cudaEventRecordExternal);
  else cudaEventRecord(m->bucket_ev[i], m->ctx.stream);
}

struct GradRange {
  int64_t off, count;
  int bucket;
};
// The gradient arena as ranges in the order the backward finalises them:
// bucket i < L holds layer L-1-i (its four matrices, contiguous in the decayed
// part of the arena, and its vectors, contiguous in the rest); bucket L the
// token and position embeddings, the final norm and an untied head.
std::vector<GradRange> grad_ranges(const gpt_model& m) {
  std::vector<GradRange> t;  // every tensor with its bucket, then merged runs
  for (auto& x : m.tensors) {
    int bucket = m.L;
    if (x.name.compare(0, 2, "h.") == 0) bucket = m.L - 1 - atoi(x.name.c_str() + 2);
    t.push_back({x.off, ((x.alloc_rows * x.cols + 63) / 64) * 64, bucket});
  }
  std::sort(t.begin(), t.end(), [](const GradRange& a, const GradRange& b) {
    return a.bucket != b.bucket ? a.bucket < b.bucket : a.off < b.off;
  });
  std::vector<GradRange> r;
  for (auto& x : t) {
    if (!r.empty() && r.back().bucket == x.bucket && r.back().off + r.back().count == x.off) r.back().count += x.count;
    else r.push_back(x);
  }
  return r;
}

template <typename T>
gpt_status forward_t(gpt_model* m, bool fuse_ce_grad, float* loss_acc, float loss_scale, int accumulate) {
  Ctx& c = m->ctx;
  long M = m->M;
  int d = m->d, L = m->L;
  bool rms = m->micro;
  float eps = 1e-5f;
  int act = m->micro ? ACT_RELU : ACT_GELU;
  size_t Md = (size_t)M * d;
  embed_fwd<T>(c, m->idx, m->P(m->wte), m->P(m->wpe), m->res, m->B, m->T, d, dkey(m, L, 0));
  for (int l = 0; l < L; l++) {
    const LayerP& y = m->layers[l];
    const size_t sl = m->rc ? 0 : l;  // activation slot
    float* x = m->res + (size_t)(2 * l) * Md;
    float* xm = m->res + (size_t)(2 * l + 1) * Md;
    float* xo = m->res + (size_t)(2 * l + 2) * Md;
    T* a1 = at<T>(m->ln1, sl * Md);
    T* qkv = at<T>(m->qkv, sl * 3 * Md);
    T* o = at<T>(m->atto, sl * Md);
    T* a2 = at<T>(m->ln2, sl * Md);
    T* h = at<T>(m->fch, sl * 4 * Md);  // act'(fc pre-activation), for the backward
    T* gg = at<T>(m->fcg, sl * 4 * Md);
    norm_fwd<T>(c, x, rms ? nullptr : m->P(y.ln1_w), rms ? nullptr : m->P(y.ln1_b), a1, m->ln1_mean + l * M,
                m->ln1_rstd + l * M, M, d, rms, eps);
    GemmDesc g = gd((int)M, 3 * d, d, a1, d, true, m->Wop(y.qkv_w), d, true);
    g.epi.kind = EPI_BIAS;
    g.name = "gemm_qkv_fwd";
    g.epi.bias = y.qkv_b >= 0 ? m->P(y.qkv_b) : nullptr;
    g.epi.out = qkv;
    g.epi.ldo = 3 * d;
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "qkv gemm: tensor map encode failed");
    AttnDesc ad{m->B, m->T, m->H, m->hd, qkv, o, m->lse + (size_t)l * M * m->H, nullptr, nullptr, nullptr,
                dkey(m, l, 1)};
    const gpt_status as = attention<T>(m, ad, false);
    if (as != GPT_OK) return as;
    g = gd((int)M, d, d, o, d, true, m->Wop(y.ap_w), d, true);
    g.epi.kind = EPI_RESADD;
    g.name = "gemm_attnproj_fwd";
    g.epi.bias = y.ap_b >= 0 ? m->P(y.ap_b) : nullptr;
    g.epi.res_in = x;
    g.epi.res_out = xm;
    g.epi.ld_res = d;
    g.epi.ldo = d;
    g.epi.drop = dkey(m, l, 2);
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "attn proj gemm failed");
    norm_fwd<T>(c, xm, rms ? nullptr : m->P(y.ln2_w), rms ? nullptr : m->P(y.ln2_b), a2, m->ln2_mean + l * M,
                m->ln2_rstd + l * M, M, d, rms, eps);
    g = gd((int)M, 4 * d, d, a2, d, true, m->Wop(y.fc_w), d, true);
    g.epi.kind = EPI_BIAS_ACT;
    g.name = "gemm_fc_fwd";
    g.epi.act = act;
    g.epi.bias = y.fc_b >= 0 ? m->P(y.fc_b) : nullptr;
    g.epi.out = h;
    g.epi.out2 = gg;
    g.epi.ldo = 4 * d;
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "fc gemm failed");
    g = gd((int)M, d, 4 * d, gg, 4 * d, true, m->Wop(y.pr_w), 4 * d, true);
    g.epi.kind = EPI_RESADD;
    g.name = "gemm_mlpproj_fwd";
    g.epi.bias = y.pr_b >= 0 ? m->P(y.pr_b) : nullptr;
    g.epi.res_in = xm;
    g.epi.res_out = xo;
    g.epi.ld_res = d;
    g.epi.ldo = d;
    g.epi.drop = dkey(m, l, 3);
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "mlp proj gemm failed");
  }
  T* xf = reinterpret_cast<T*>(m->lnf);
  norm_fwd<T>(c, m->res + (size_t)(2 * L) * Md, rms ? nullptr : m->P(m->lnf_w), rms ? nullptr : m->P(m->lnf_b), xf,
              m->lnf_mean, m->lnf_rstd, M, d, rms, eps);
  GemmDesc g = gd((int)M, m->Vp, d, xf, d, true, m->Wop(m->head), d, true);
  g.epi.kind = EPI_STORE;
  g.name = "gemm_lmhead_fwd";
  g.epi.out = m->logits;
  g.epi.ldo = m->Vp;
  if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "lm_head gemm failed");
  ce_fwd_bwd<T>(c, reinterpret_cast<T*>(m->logits), m->tgt, M, m->V, m->Vp, m->row_lse, m->row_loss, fuse_ce_grad,
                1.0f / (float)(M * m->ga));
  loss_reduce(c, m->row_loss, M, loss_scale, loss_acc, accumulate);
  m->have_forward = true;
  m->ce_grad_done = fuse_ce_grad;
  return check_cuda(m, "forward");
}

void add_bias_grads_from_norm(gpt_model* m, const float* part, int64_t gain, int64_t beta, int64_t next_bias) {
  partial_reduce3(m->ctx, part, m->part_blocks, m->d, gain >= 0 ? m->G(gain) : nullptr,
                  beta >= 0 ? m->G(beta) : nullptr, next_bias >= 0 ? m->G(next_bias) : nullptr);
}

// Activation recompute of layer l into the single activation slot: the
// layer's forward from its stored residual inputs, minus the two projection
// GEMMs whose outputs are those residuals.  The same kernels on the same
// inputs (dropout keys included) as the forward, so the activations are
// bit-identical to the ones the forward wrote.
template <typename T>
gpt_status recompute_layer(gpt_model* m, int l) {
  Ctx& c = m->ctx;
  const long M = m->M;
  const int d = m->d;
  const bool rms = m->micro;
  const float eps = 1e-5f;
  const int act = m->micro ? ACT_RELU : ACT_GELU;
  const size_t Md = (size_t)M * d;
  const LayerP& y = m->layers[l];
  T* a1 = at<T>(m->ln1, 0);
  T* qkv = at<T>(m->qkv, 0);
  T* o = at<T>(m->atto, 0);
  T* a2 = at<T>(m->ln2, 0);
  norm_fwd<T>(c, m->res + (size_t)(2 * l) * Md, rms ? nullptr : m->P(y.ln1_w), rms ? nullptr : m->P(y.ln1_b), a1,
              m->ln1_mean + l * M, m->ln1_rstd + l * M, M, d, rms, eps);
  GemmDesc g = gd((int)M, 3 * d, d, a1, d, true, m->Wop(y.qkv_w), d, true);
  g.epi.kind = EPI_BIAS;
  g.name = "gemm_qkv_recompute";
  g.epi.bias = y.qkv_b >= 0 ? m->P(y.qkv_b) : nullptr;
  g.epi.out = qkv;
  g.epi.ldo = 3 * d;
  if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "qkv recompute gemm failed");
  AttnDesc ad{m->B, m->T, m->H, m->hd, qkv, o, m->lse + (size_t)l * M * m->H, nullptr, nullptr, nullptr,
              dkey(m, l, 1)};
  const gpt_status as = attention<T>(m, ad, false);
  if (as != GPT_OK) return as;
  norm_fwd<T>(c, m->res + (size_t)(2 * l + 1) * Md, rms ? nullptr : m->P(y.ln2_w), rms ? nullptr : m->P(y.ln2_b),
              a2, m->ln2_mean + l * M, m->ln2_rstd + l * M, M, d, rms, eps);
  g = gd((int)M, 4 * d, d, a2, d, true, m->Wop(y.fc_w), d, true);
  g.epi.kind = EPI_BIAS_ACT;
  g.name = "gemm_fc_recompute";
  g.epi.act = act;
  g.epi.bias = y.fc_b >= 0 ? m->P(y.fc_b) : nullptr;
  g.epi.out = at<T>(m->fch, 0);
  g.epi.out2 = at<T>(m->fcg, 0);
  g.epi.ldo = 4 * d;
  if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "fc recompute gemm failed");
  return GPT_OK;
}

template <typename T>
gpt_status backward_t(gpt_model* m) {
  Ctx& c = m->ctx;
  long M = m->M;
  int d = m->d, L = m->L, Vp = m->Vp;
  bool rms = m->micro;
  int act = m->micro ? ACT_RELU : ACT_GELU;
  size_t Md = (size_t)M * d;
  T* dl = reinterpret_cast<T*>(m->logits);
  if (!m->ce_grad_done)
    ce_fwd_bwd<T>(c, dl, m->tgt, M, m->V, Vp, m->row_lse, m->row_loss, true, 1.0f / (float)(M * m->ga));
  m->ce_grad_done = true;
  T* dyb = reinterpret_cast<T*>(m->dyb);
  T* dh = reinterpret_cast<T*>(m->dh);
  T* dqkv = reinterpret_cast<T*>(m->dqkv);
  T* datt = reinterpret_cast<T*>(m->datt);
  const bool first = m->cur_micro == 0, last = m->cur_micro == m->n_micro - 1;
  // inst: (layer, kind) of a per-layer weight gradient, -1 for the lm_head
  // with adapters attached the base weights are frozen: their gradients are
  // not formed, except the adapted QKV blocks' (the adapters' chain rule)
  const bool frozen = m->lora.on;
  auto dW = [&](int Mo, int No, const void* A, const void* Bm, float* out, const char* name, int inst) -> bool {
    if (frozen) return true;
    // out[Mo, No] += A^T B with A [M, Mo], B [M, No] (tokens outermost)
    GemmDesc g = gd(Mo, No, (int)M, A, Mo, false, Bm, No, false);
    g.epi.kind = EPI_ACC_F32;
    g.name = name;
    g.epi.out = out;
    g.epi.ldo = No;
    if (m->bf16m) {
      g.split_k = choose_splits(Mo, No, M);
      g.partial = m->splitk;
      if (inst >= 0 && m->split_n[inst] > 1 && gemm_tc_supported(g) &&
          gemm_tc_splits(g, c.num_sms) == m->split_n[inst]) {
        // split partials accumulate over the step's micro-batches in this
        // instance's buffer; the last micro-batch adds them to the gradient
        g.partial = m->split_parts + m->split_off[inst];
        g.partial_accumulate = !first;
        g.reduce_partials = last;
      }
    }
    return gemm(m, g);
  };
  auto norm_part = [&](int k) { return m->norm_parts + (size_t)k * m->part_cap * 3 * d; };
  auto colsum_part = [&](int l, int which) {
    return m->colsum_parts + ((size_t)l * 2 + which) * m->colsum_rows * 4 * d;
  };
  // bias gradient = column sums of the operand-typed gradient x [M, N]
  auto bias_grad = [&](const T* x, int N, int l, int which, float* grad) {
    if (frozen) return;
    colsum_partial<T>(c, x, M, N, colsum_part(l, which), !first);
    if (last) colsum_reduce(c, colsum_part(l, which), colsum_chunks(M), N, grad);
  };
  // lm_head: dx_f = dlogits W_head; dW_head += dlogits^T x_f
  GemmDesc g = gd((int)M, d, Vp, dl, Vp, true, m->Wop(m->head), d, false);
  g.epi.kind = EPI_STORE_F32;
  g.name = "gemm_lmhead_dx";
  g.epi.out = m->dln;
  g.epi.ldo = d;
  if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "lm_head dX gemm failed");
  if (!dW(Vp, d, dl, m->lnf, m->G(m->head), "gemm_lmhead_dw", -1))
    return fail(m, GPT_ERR_CUDA, "lm_head dW gemm failed");
  // final norm
  NormBwd nb;
  nb.dy = m->dln;
  nb.x = m->res + (size_t)(2 * L) * Md;
  nb.mean = m->lnf_mean;
  nb.rstd = m->lnf_rstd;
  nb.w = rms ? nullptr : m->P(m->lnf_w);
  nb.dres = m->dres;
  nb.accumulate = false;
  nb.dyb = dyb;
  nb.drop = dkey(m, L - 1, 3);
  nb.want_dyb = true;
  nb.part = norm_part(2 * L);
  nb.part_accumulate = !first;
  nb.blocks = m->part_blocks;
  nb.rows = M;
  nb.d = d;
  nb.rms = rms;
  norm_bwd<T>(c, nb);
  if (last && !frozen) add_bias_grads_from_norm(m, nb.part, m->lnf_w, m->lnf_b, m->layers[L - 1].pr_b);
  for (int l = L - 1; l >= 0; l--) {
    const LayerP& y = m->layers[l];
    // with recompute the slot still holds the last layer's forward activations
    if (m->rc && l != L - 1) {
      const gpt_status rs = recompute_layer<T>(m, l);
      if (rs != GPT_OK) return rs;
    }
    const size_t sl = m->rc ? 0 : l;
    T* a1 = at<T>(m->ln1, sl * Md);
    T* qkv = at<T>(m->qkv, sl * 3 * Md);
    T* o = at<T>(m->atto, sl * Md);
    T* a2 = at<T>(m->ln2, sl * Md);
    T* h = at<T>(m->fch, sl * 4 * Md);
    T* gg = at<T>(m->fcg, sl * 4 * Md);
    // MLP projection
    if (!dW(d, 4 * d, dyb, gg, m->G(y.pr_w), "gemm_mlpproj_dw", l * 4 + 0))
      return fail(m, GPT_ERR_CUDA, "proj dW failed");
    g = gd((int)M, 4 * d, d, dyb, d, true, m->Wop(y.pr_w), 4 * d, false);
    g.epi.kind = EPI_ACT_BWD;
    g.name = "gemm_mlpproj_dx";
    g.epi.act = act;
    g.epi.aux = h;
    g.epi.out = dh;
    g.epi.ldo = 4 * d;
    // bf16: the fc bias gradient's column sums of dh come from this GEMM's
    // epilogue (one partial row per 32-row group), not from a second pass
    const bool fused_colsum = m->bf16m && y.fc_b >= 0 && !frozen;
    if (fused_colsum) {
      g.epi.colsum = colsum_part(l, 0);
      g.epi.colsum_acc = !first;
    }
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "proj dX failed");
    if (fused_colsum) {
      if (last) colsum_reduce(c, colsum_part(l, 0), (int)((M + 31) / 32), 4 * d, m->G(y.fc_b));
    } else if (y.fc_b >= 0) {
      bias_grad(dh, 4 * d, l, 0, m->G(y.fc_b));
    }
    if (!dW(4 * d, d, dh, a2, m->G(y.fc_w), "gemm_fc_dw", l * 4 + 1)) return fail(m, GPT_ERR_CUDA, "fc dW failed");
    g = gd((int)M, d, 4 * d, dh, 4 * d, true, m->Wop(y.fc_w), d, false);
    g.epi.kind = EPI_STORE_F32;
    g.name = "gemm_fc_dx";
    g.epi.out = m->dln;
    g.epi.ldo = d;
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "fc dX failed");
    nb.dy = m->dln;
    nb.x = m->res + (size_t)(2 * l + 1) * Md;
    nb.mean = m->ln2_mean + l * M;
    nb.rstd = m->ln2_rstd + l * M;
    nb.w = rms ? nullptr : m->P(y.ln2_w);
    nb.accumulate = true;
    nb.drop = dkey(m, l, 2);
    nb.want_dyb = true;
    nb.part = norm_part(2 * l + 1);
    norm_bwd<T>(c, nb);
    if (last && !frozen) add_bias_grads_from_norm(m, nb.part, y.ln2_w, y.ln2_b, y.ap_b);
    // attention projection
    if (!dW(d, d, dyb, o, m->G(y.ap_w), "gemm_attnproj_dw", l * 4 + 2))
      return fail(m, GPT_ERR_CUDA, "attn proj dW failed");
    g = gd((int)M, d, d, dyb, d, true, m->Wop(y.ap_w), d, false);
    g.epi.kind = EPI_STORE;
    g.name = "gemm_attnproj_dx";
    g.epi.out = datt;
    g.epi.ldo = d;
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "attn proj dX failed");
    AttnDesc ad{m->B, m->T, m->H, m->hd, qkv, o, m->lse + (size_t)l * M * m->H, datt, dqkv, m->dsum, dkey(m, l, 1)};
    // tensor-core attention: the qkv bias gradient's column sums of dqkv come
    // from the backward kernels' epilogues (one partial row per 128-row block)
    const bool fused_qkv_colsum = m->attn_tc && y.qkv_b >= 0 && !frozen;
    if (fused_qkv_colsum) {
      ad.colsum = colsum_part(l, 1);
      ad.colsum_acc = first ? 0 : 1;
    }
    const gpt_status as = attention<T>(m, ad, true);
    if (as != GPT_OK) return as;
    if (fused_qkv_colsum) {
      if (last) colsum_reduce(c, colsum_part(l, 1), (int)(M / 128), 3 * d, m->G(y.qkv_b));
    } else if (y.qkv_b >= 0) {
      bias_grad(dqkv, 3 * d, l, 1, m->G(y.qkv_b));
    }
    if (!dW(3 * d, d, dqkv, a1, m->G(y.qkv_w), "gemm_qkv_dw", l * 4 + 3))
      return fail(m, GPT_ERR_CUDA, "qkv dW failed");
    if (frozen) {
      // the adapted blocks only: G[t d .. t d + d) += dqkv[:, t d .. t d + d)^T a1
      for (int t = 0; t < 3; t++) {
        if (!(m->lora.targets & (1 << t))) continue;
        GemmDesc gq = gd(d, d, (int)M, dqkv + (size_t)t * d, 3 * d, false, a1, d, false);
        gq.epi.kind = EPI_ACC_F32;
        gq.name = "gemm_qkv_dw_adapted";
        gq.epi.out = m->G(y.qkv_w) + (size_t)t * d * d;
        gq.epi.ldo = d;
        if (m->bf16m) {
          gq.split_k = choose_splits(d, d, M);
          gq.partial = m->splitk;
        }
        if (!gemm(m, gq)) return fail(m, GPT_ERR_CUDA, "adapted qkv dW failed");
      }
    }
    g = gd((int)M, d, 3 * d, dqkv, 3 * d, true, m->Wop(y.qkv_w), d, false);
    g.epi.kind = EPI_STORE_F32;
    g.name = "gemm_qkv_dx";
    g.epi.out = m->dln;
    g.epi.ldo = d;
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "qkv dX failed");
    nb.dy = m->dln;
    nb.x = m->res + (size_t)(2 * l) * Md;
    nb.mean = m->ln1_mean + l * M;
    nb.rstd = m->ln1_rstd + l * M;
    nb.w = rms ? nullptr : m->P(y.ln1_w);
    nb.accumulate = true;
    nb.drop = l > 0 ? dkey(m, l - 1, 3) : DropKey{};
    nb.want_dyb = l > 0;
    nb.part = norm_part(2 * l);
    norm_bwd<T>(c, nb);
    if (last && !frozen)
      add_bias_grads_from_norm(m, nb.part, y.ln1_w, y.ln1_b, l > 0 ? m->layers[l - 1].pr_b : -1);
    if (last) record_bucket(m, L - 1 - l);  // layer l's gradients are final
  }
  if (frozen) {  // no embedding gradients; the adapters' from the merged blocks
    if (last) lora_grads(c, m->lora.lb, m->g);
    return check_cuda(m, "backward");
  }
  const int32_t *stok = m->stok, *spos = m->spos;
  if (m->presorted) {
    stok = m->stok_all + (size_t)m->cur_micro * M;
    spos = m->spos_all + (size_t)m->cur_micro * M;
  } else {
    embed_sort(c, m->idx, M, m->stok, m->spos, m->nuniq);
  }
  embed_bwd(c, m->dres, stok, spos, M, m->T, m->B, d, dkey(m, L, 0), m->G(m->wte), m->G(m->wpe), m->seg);
  if (last) record_bucket(m, L);  // the embeddings, the final norm (and an untied head)
  return check_cuda(m, "backward");
}

gpt_status forward_any(gpt_model* m, bool fuse, float* acc, float scale, int accumulate) {
  return m->bf16m ? forward_t<bf16>(m, fuse, acc, scale, accumulate)
                  : forward_t<float>(m, fuse, acc, scale, accumulate);
}
gpt_status backward_any(gpt_model* m) { return m->bf16m ? backward_t<bf16>(m) : backward_t<float>(m); }

gpt_status lora_step(gpt_model* m, float lr, int step, bool dev_params);

gpt_status adamw_step(gpt_model* m, float lr, int step, bool dev_params = false) {
  if (m->lora.on) return lora_step(m, lr, step, dev_params);
  Ctx& c = m->ctx;
  int blocks = sumsq_blocks(c);
  sumsq_partials(c, m->g, m->n_total, m->norm_part, blocks);
  AdamArgs a;
  a.w = m->w;
  a.g = m->g;
  a.m = m->am;
  a.v = m->av;
  a.wb = m->wb;
  a.n = m->n_total;
  a.n_decay = m->n_decay;
  a.norm_partials = m->norm_part;
  a.norm_blocks = blocks;
  a.norm_out = m->scal + 2;
  a.lr = lr;
  a.beta1 = m->cfg.beta1;
  a.beta2 = m->cfg.beta2;
  a.eps = m->cfg.eps;
  a.wd = m->cfg.weight_decay;
  a.clip = m->cfg.grad_clip;
  a.bc1 = (float)(1.0 - pow((double)m->cfg.beta1, (double)step));
  a.bc2 = (float)(1.0 - pow((double)m->cfg.beta2, (double)step));
  if (dev_params) a.hyper = m->hyper_dev;
  adamw(c, a);
  return check_cuda(m, "adamw");
}

// The optimiser step with adapters attached: the base weights are frozen.
// The adapters' gradients (formed at the end of the step's last backward from
// the merged QKV blocks' gradient) go through clip + AdamW (every adapter
// tensor is 2-D, hence decayed) alone; the base gradient arena is cleared (the base
// AdamW is what clears it otherwise); the merged operands are rebuilt.
gpt_status lora_step(gpt_model* m, float lr, int step, bool dev_params) {
  Ctx& c = m->ctx;
  auto& L = m->lora;
  const int blocks = sumsq_blocks(c);
  sumsq_partials(c, L.lb.grads, L.n, m->norm_part, blocks);
  AdamArgs a;
  a.w = L.lb.params;
  a.g = L.lb.grads;
  a.m = L.m;
  a.v = L.v;
  a.wb = nullptr;
  a.n = L.n;
  a.n_decay = L.n;
  a.norm_partials = m->norm_part;
  a.norm_blocks = blocks;
  a.norm_out = m->scal + 2;
  a.lr = lr;
  a.beta1 = m->cfg.beta1;
  a.beta2 = m->cfg.beta2;
  a.eps = m->cfg.eps;
  a.wd = m->cfg.weight_decay;
  a.clip = m->cfg.grad_clip;
  a.bc1 = (float)(1.0 - pow((double)m->cfg.beta1, (double)step));
  a.bc2 = (float)(1.0 - pow((double)m->cfg.beta2, (double)step));
  if (dev_params) a.hyper = m->hyper_dev;
  adamw(c, a);
  cudaMemsetAsync(m->g, 0, (size_t)m->n_total * 4, c.stream);
  lora_merge(c, L.lb, m->w, m->wb);
  return check_cuda(m, "lora step");
}

void bias_corrections(const gpt_model* m, int step, float* bc1, float* bc2) {
  *bc1 = (float)(1.0 - pow((double)m->cfg.beta1, (double)step));
  *bc2 = (float)(1.0 - pow((double)m->cfg.beta2, (double)step));
}

}  // namespace

// ============================================================================
// C ABI
// ============================================================================
// One decoding step for every batch row: the token dec_tok[b] at position t
// goes through the model with the per-layer qkv activations as the key /
// value cache (this step's K and V are written at position t), leaving the
// logits of the next token in dec_logits [B, Vp].
template <typename T>
gpt_status decode_step_t(gpt_model* m, int t) {
  Ctx& c = m->ctx;
  const int B = m->B, d = m->d, L = m->L, Tn = m->T;
  const bool rms = m->micro;
  const float eps = 1e-5f;
  const int act = m->micro ? ACT_RELU : ACT_GELU;
  const size_t Md = (size_t)m->M * d;
  T* a = reinterpret_cast<T*>(m->dec_a);
  T* o = reinterpret_cast<T*>(m->dec_o);
  // norm of the residual rows, then a GEMM on it: one skinny GEMM that
  // computes the norm itself where it applies, else the two kernels
  auto norm_gemm = [&](int64_t wi, int64_t bi, GemmDesc& g) -> bool {
    const float* nw = rms ? nullptr : m->P(wi);
    const float* nb = rms ? nullptr : m->P(bi);
    if (m->bf16m && gemm_skinny_supported(g)) {
      SkinnyNorm n;
      n.x = m->dec_res;
      n.w = nw;
      n.b = nb;
      n.ldx = d;
      n.rms = rms ? 1 : 0;
      n.eps = eps;
      if (skinny_norm_supported(g, n)) {
        gemm_skinny_bf16(c, g, &n);
        return true;
      }
    }
    norm_fwd<T>(c, m->dec_res, nw, nb, a, m->dec_mean, m->dec_rstd, B, d, rms, eps);
    return gemm(m, g);
  };
  embed_fwd<T>(c, m->dec_tok, m->P(m->wte), m->P(m->wpe) + (size_t)t * d, m->dec_res, B, 1, d, DropKey{});
  for (int l = 0; l < L; l++) {
    const LayerP& y = m->layers[l];
    T* qkv = at<T>(m->qkv, l * 3 * Md);
    GemmDesc g = gd(B, 3 * d, d, a, d, true, m->Wop(y.qkv_w), d, true);
    g.epi.kind = EPI_BIAS;
    g.name = "gemm_qkv_decode";
    g.epi.bias = y.qkv_b >= 0 ? m->P(y.qkv_b) : nullptr;
    g.epi.out = qkv + (size_t)t * 3 * d;  // row b at position t of the cache
    g.epi.ldo = Tn * 3 * d;
    if (!norm_gemm(y.ln1_w, y.ln1_b, g)) return fail(m, GPT_ERR_CUDA, "decode qkv gemm failed");
    attn_decode<T>(c, qkv, B, Tn, m->H, m->hd, t, o);
    g = gd(B, d, d, o, d, true, m->Wop(y.ap_w), d, true);
    g.epi.kind = EPI_RESADD;
    g.name = "gemm_attnproj_decode";
    g.epi.bias = y.ap_b >= 0 ? m->P(y.ap_b) : nullptr;
    g.epi.res_in = m->dec_res;
    g.epi.res_out = m->dec_res;
    g.epi.ld_res = d;
    g.epi.ldo = d;
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "decode attn proj gemm failed");
    g = gd(B, 4 * d, d, a, d, true, m->Wop(y.fc_w), d, true);
    g.epi.kind = EPI_BIAS_ACT;
    g.name = "gemm_fc_decode";
    g.epi.act = act;
    g.epi.bias = y.fc_b >= 0 ? m->P(y.fc_b) : nullptr;
    g.epi.out = m->dec_dact;
    g.epi.out2 = m->dec_g;
    g.epi.ldo = 4 * d;
    if (!norm_gemm(y.ln2_w, y.ln2_b, g)) return fail(m, GPT_ERR_CUDA, "decode fc gemm failed");
    g = gd(B, d, 4 * d, m->dec_g, 4 * d, true, m->Wop(y.pr_w), 4 * d, true);
    g.epi.kind = EPI_RESADD;
    g.name = "gemm_mlpproj_decode";
    g.epi.bias = y.pr_b >= 0 ? m->P(y.pr_b) : nullptr;
    g.epi.res_in = m->dec_res;
    g.epi.res_out = m->dec_res;
    g.epi.ld_res = d;
    g.epi.ldo = d;
    if (!gemm(m, g)) return fail(m, GPT_ERR_CUDA, "decode mlp proj gemm failed");
  }
  GemmDesc g = gd(B, m->Vp, d, a, d, true, m->Wop(m->head), d, true);
  g.epi.kind = EPI_STORE;
  g.name = "gemm_lmhead_decode";
  g.epi.out = m->dec_logits;
  g.epi.ldo = m->Vp;
  if (!norm_gemm(m->lnf_w, m->lnf_b, g)) return fail(m, GPT_ERR_CUDA, "decode lm_head gemm failed");
  return check_cuda(m, "decode step");
}

extern "C" {

const char* gpt_status_string(gpt_status s) {
  switch (s) {
    case GPT_OK: return "ok";
    case GPT_ERR_INVALID_ARG: return "invalid argument";
    case GPT_ERR_CONFIG: return "invalid config";
    case GPT_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case GPT_ERR_CUDA: return "CUDA error";
    case GPT_ERR_TOKEN_RANGE: return "token id out of range";
    case GPT_ERR_NONFINITE: return "non-finite value";
    case GPT_ERR_STATE: return "call out of sequence";
    case GPT_ERR_UNSUPPORTED: return "unsupported";
    case GPT_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* gpt_last_error(const gpt_model* m) { return m ? m->err.c_str() : "null model"; }

size_t gpt_param_count(const gpt_config* c) {
  if (validate(c, nullptr) != GPT_OK) return 0;
  size_t V = c->vocab_size, d = c->n_embd, T = c->block_size, L = c->n_layer;
  if (c->variant == GPT_VARIANT_GPT2) return V * d + T * d + L * (12 * d * d + 13 * d) + 2 * d;
  return 2 * V * d + T * d + 12 * L * d * d;
}

gpt_status gpt_workspace_bytes(const gpt_config* c, size_t* out) {
  if (!out) return GPT_ERR_INVALID_ARG;
  gpt_status s = validate(c, nullptr);
  if (s != GPT_OK) return s;
  gpt_model m;
  derive(m, c);
  *out = carve(m, nullptr);
  return GPT_OK;
}

gpt_status gpt_config_kernel_paths(const gpt_config* c, uint32_t* out) {
  if (!out) return GPT_ERR_INVALID_ARG;
  gpt_status s = validate(c, nullptr);
  if (s != GPT_OK) return s;
  uint32_t p = 0;
  if (c->precision == GPT_PREC_BF16) {
    p |= GPT_PATH_GEMM_TC;
    if (attn_tc_shape_ok(c->block_size, c->n_embd / c->n_head)) p |= GPT_PATH_ATTN_TC;
  }
  *out = p;
  return GPT_OK;
}

float gpt_lr_cosine(float lr, int32_t it, int32_t warmup, int32_t max_iters) {
  if (it < warmup) return (float)((double)lr * it / warmup);
  double r = (double)(it - warmup) / (double)(max_iters - warmup);
  return (float)((double)lr * 0.5 * (1.0 + cos(3.14159265358979323846 * r)));
}

float gpt_lr_linear(float lr, int32_t it, int32_t max_iters) {
  return (float)((double)lr * (1.0 - (double)it / (double)max_iters));
}

gpt_status gpt_create(const gpt_config* cfg, uint64_t seed, void* d_workspace, size_t bytes, void* cuda_stream,
                      gpt_model** out) {
  if (!out || !d_workspace) return GPT_ERR_INVALID_ARG;
  *out = nullptr;
  std::string why;
  gpt_status s = validate(cfg, &why);
  if (s != GPT_OK) return s;
  gpt_model* m = new gpt_model();
  derive(*m, cfg);
  size_t need = carve(*m, nullptr);
  if (bytes < need) {
    delete m;
    return GPT_ERR_WORKSPACE_TOO_SMALL;
  }
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(d_workspace) + 1023) & ~uintptr_t(1023));
  carve(*m, base);
  m->ws = (uint8_t*)d_workspace;
  m->ws_bytes = bytes;
  m->ctx.stream = (cudaStream_t)cuda_stream;
  m->ctx.flags = reinterpret_cast<uint32_t*>(m->scal + 3);
  m->step_dev = reinterpret_cast<int*>(m->scal + 8);
  m->hyper_dev = m->scal + 9;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) m->ctx.num_sms = sms;
  m->part_blocks = std::min(m->part_blocks, norm_bwd_blocks(m->ctx, m->M, m->d, m->bf16m));
  m->attn_tc = m->bf16m && attn_tc_shape_ok(m->T, m->hd);
  cudaStream_t st = m->ctx.stream;
  // zero the arenas (weights, grads, moments) and the scalars
  cudaMemsetAsync(m->scal, 0, 64 * 4, st);
  const size_t arena_bytes = (size_t)(m->n_total + kArenaSlack) * 4;
  cudaMemsetAsync(m->w, 0, arena_bytes, st);
  cudaMemsetAsync(m->g, 0, arena_bytes, st);
  const size_t moment_bytes = m->zero_sharded ? (size_t)m->zero_stride * 4 : arena_bytes;
  cudaMemsetAsync(m->am, 0, moment_bytes, st);
  cudaMemsetAsync(m->av, 0, moment_bytes, st);
  if (m->wb) cudaMemsetAsync(m->wb, 0, arena_bytes / 2, st);
  // weights from the seed, uploaded one tensor at a time
  std::vector<float> host;
  for (size_t i = 0; i < m->tensors.size(); i++) {
    const TensorRec& t = m->tensors[i];
    host.resize((size_t)t.rows * t.cols);
    init_tensor_host(t, cfg->init_std, seed, (int)i, host.data());
    cudaMemcpyAsync(m->w + t.off, host.data(), host.size() * 4, cudaMemcpyHostToDevice, st);
    cudaStreamSynchronize(st);
  }
  if (m->bf16m) to_bf16(m->ctx, m->w, m->wb, m->n_total);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    delete m;
    return GPT_ERR_CUDA;
  }
  *out = m;
  return GPT_OK;
}

void gpt_destroy(gpt_model* m) {
  if (!m) return;
  for (auto& e : m->gexec)
    if (e) cudaGraphExecDestroy(e);
  for (auto e : m->bucket_ev) cudaEventDestroy(e);
  if (m->gen_exec) cudaGraphExecDestroy(m->gen_exec);
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  delete m->timing;
  delete m;
}

gpt_status gpt_set_graphs(gpt_model* m, int32_t on) {
  if (!m) return GPT_ERR_INVALID_ARG;
  m->graphs_on = on != 0;
  return GPT_OK;
}

gpt_status gpt_set_stream(gpt_model* m, void* st) {
  if (!m) return GPT_ERR_INVALID_ARG;
  m->ctx.stream = (cudaStream_t)st;
  return GPT_OK;
}

gpt_status gpt_set_dropout_cursor(gpt_model* m, int32_t step, int32_t micro) {
  if (!m || step < 0 || micro < 0) return GPT_ERR_INVALID_ARG;
  m->drop_counter = (int64_t)step * m->ga + micro;
  return GPT_OK;
}

gpt_status gpt_forward_loss(gpt_model* m, const int32_t* d_idx, const int32_t* d_tgt, float* h_loss) {
  if (!m || !d_idx || !d_tgt) return fail(m, GPT_ERR_INVALID_ARG, "forward_loss: null argument");
  check_tokens(m->ctx, d_idx, d_tgt, m->M, m->V, m->idx, m->tgt);
  gpt_status s = forward_any(m, false, m->scal + 0, 1.0f / (float)m->M, 0);
  if (s != GPT_OK) return s;
  if (h_loss) {
    float sc[4];
    s = sync_and_flags(m, "forward_loss", sc);
    *h_loss = sc[0];
  }
  return s;
}

gpt_status gpt_backward(gpt_model* m) {
  if (!m) return GPT_ERR_INVALID_ARG;
  if (!m->have_forward) return fail(m, GPT_ERR_STATE, "backward called without a preceding forward_loss");
  m->cur_micro = 0;  // a stand-alone backward completes its gradients
  m->n_micro = 1;
  gpt_status s = backward_any(m);
  m->have_forward = false;
  return s;
}

gpt_status gpt_clip_adamw_step(gpt_model* m, float lr, int32_t step, float* h_grad_norm) {
  if (!m) return GPT_ERR_INVALID_ARG;
  if (m->zero_sharded && !m->lora.on)
    return fail(m, GPT_ERR_UNSUPPORTED, "clip_adamw_step: the moments are sharded; use gpt_clip_adamw_shard");
  if (step < 1) return fail(m, GPT_ERR_INVALID_ARG, "step must be >= 1");
  gpt_status s = adamw_step(m, lr, step);
  if (s != GPT_OK) return s;
  if (h_grad_norm) {
    float sc[4];
    s = sync_and_flags(m, "clip_adamw_step", sc);
    *h_grad_norm = sc[2];
  }
  return s;
}

// The kernels of one optimiser step (grad_accum micro-batches, clip + AdamW;
// without the optimiser for the data-parallel accumulate step, kind 2).
// dev_params: the step index, lr and bias corrections are read from device
// memory (the form captured into a graph and replayed every step).
static gpt_status train_body(gpt_model* m, int kind, const void* d_stream, uint64_t len, uint64_t seed, float lr,
                             int32_t step, bool dev_params) {
  Ctx& c = m->ctx;
  const size_t Mz = (size_t)m->M;
  for (int mu = 0; mu < m->ga; mu++) {
    if (d_stream) {
      gather_batch(c, d_stream, m->cfg.token_dtype == GPT_TOK_U16, len, seed, step, mu, m->B, m->T, m->V,
                   m->idx_all + mu * Mz, m->tgt_all + mu * Mz, dev_params ? m->step_dev : nullptr);
    } else {
      check_tokens(c, m->stage_idx + mu * Mz, m->stage_tgt + mu * Mz, m->M, m->V, m->idx_all + mu * Mz,
                   m->tgt_all + mu * Mz);
    }
  }
  embed_sort(c, m->idx_all, m->M, m->stok_all, m->spos_all, m->nuniq_all, m->ga);
  gpt_status s = GPT_OK;
  m->presorted = true;
  for (int mu = 0; mu < m->ga && s == GPT_OK; mu++) {
    m->drop_counter = (int64_t)step * m->ga + mu;
    m->cur_micro = mu;
    m->n_micro = m->ga;
    m->idx = m->idx_all + mu * Mz;
    m->tgt = m->tgt_all + mu * Mz;
    s = forward_any(m, true, m->scal + 1, 1.0f / (float)(m->M * m->ga), mu > 0);
    if (s == GPT_OK) s = backward_any(m);
  }
  m->presorted = false;
  m->idx = m->idx0;
  m->tgt = m->tgt0;
  if (s != GPT_OK) return s;
  m->have_forward = false;
  if (kind >= 2) return GPT_OK;  // the caller exchanges the gradients, then runs clip + AdamW
  return adamw_step(m, lr, step, dev_params);
}

// Captures train_body into a CUDA graph on an internal stream (the caller's
// stream may be the legacy default stream, which cannot be captured).
static bool capture_step(gpt_model* m, int kind, const void* d_stream, uint64_t len, uint64_t seed, float lr,
                         int32_t step) {
  if (!m->cap_stream && cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  cudaStream_t user = m->ctx.stream;
  const uint64_t l0 = m->ctx.launches;
  m->ctx.stream = m->cap_stream;
  cudaGraph_t g = nullptr;
  bool ok = cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
  m->dev_keys = true;  // dropout keys follow the step index the replay writes
  m->capturing = true;
  gpt_status s = ok ? train_body(m, kind, d_stream, len, seed, lr, step, true) : GPT_ERR_CUDA;
  m->capturing = false;
  m->dev_keys = false;
  if (ok) ok = cudaStreamEndCapture(m->cap_stream, &g) == cudaSuccess && s == GPT_OK;
  m->ctx.stream = user;
  if (ok) ok = cudaGraphInstantiate(&m->gexec[kind], g, 0) == cudaSuccess;
  if (g) cudaGraphDestroy(g);
  m->graph_launches[kind] = m->ctx.launches - l0;
  m->ctx.launches = l0;
  if (!ok) {
    cudaGetLastError();
    m->gexec[kind] = nullptr;
  }
  return ok;
}

static gpt_status train_common(gpt_model* m, int kind, const void* d_stream, uint64_t len, uint64_t seed, float lr,
                               int32_t step, float* h_loss, float* h_norm) {
  if (step < 1) return fail(m, GPT_ERR_INVALID_ARG, "step must be >= 1");
  if (kind < 2 && m->zero_sharded && !m->lora.on)
    return fail(m, GPT_ERR_UNSUPPORTED, "train_step: the moments are sharded; use the accumulate form");
  Ctx& c = m->ctx;
  m->bucket_record = kind >= 2;
  // Replay a captured graph of the whole step: everything that changes from
  // step to step (the step index, the learning rate, the bias corrections and
  // through the step index the dropout keys) is read from device memory.  Not
  // with per-kernel timing.  The first call of each kind runs eagerly, the
  // second captures, later calls only replay.
  bool replay = m->graphs_on && !c.timing;
  if (replay && (kind == 0 || kind == 2) && m->gexec[kind] &&
      (m->g_dstream[kind] != d_stream || m->g_len[kind] != len || m->g_seed[kind] != seed)) {
    cudaGraphExecDestroy(m->gexec[kind]);
    m->gexec[kind] = nullptr;
    m->warm[kind] = 0;
  }
  if (replay && !m->gexec[kind]) {
    if (m->warm[kind] < 1) {
      m->warm[kind]++;
      replay = false;
    } else if (capture_step(m, kind, d_stream, len, seed, lr, step)) {
      m->g_dstream[kind] = d_stream;
      m->g_len[kind] = len;
      m->g_seed[kind] = seed;
    } else {
      // reported, not hidden: the step did not run; the next call tries the
      // capture again, and gpt_set_graphs(m, 0) runs every step eagerly
      return fail(m, GPT_ERR_CUDA,
                  "train_step: capturing the step into a CUDA graph failed (graphs stay on; "
                  "gpt_set_graphs(m, 0) runs steps eagerly)");
    }
  }
  gpt_status s = GPT_OK;
  if (replay) {
    float bc1, bc2;
    bias_corrections(m, step, &bc1, &bc2);
    set_step_params(c, m->step_dev, m->hyper_dev, step, lr, bc1, bc2);
    if (cudaGraphLaunch(m->gexec[kind], c.stream) != cudaSuccess) return check_cuda(m, "graph launch");
    c.launches += m->graph_launches[kind];
    m->have_forward = false;
  } else {
    s = train_body(m, kind, d_stream, len, seed, lr, step, false);
  }
  m->bucket_record = false;
  if (s != GPT_OK) return s;
  if (h_loss || h_norm) {
    float sc[4];
    s = sync_and_flags(m, "train_step", sc);
    if (h_loss) *h_loss = sc[1];
    if (h_norm) *h_norm = sc[2];
  }
  return s;
}

gpt_status gpt_train_step(gpt_model* m, const void* d_stream, uint64_t stream_len, uint64_t data_seed, float lr,
                          int32_t step, float* h_loss, float* h_grad_norm) {
  if (!m || !d_stream) return fail(m, GPT_ERR_INVALID_ARG, "train_step: null argument");
  if (stream_len <= (uint64_t)m->T) return fail(m, GPT_ERR_INVALID_ARG, "stream shorter than block_size + 1");
  return train_common(m, 0, d_stream, stream_len, data_seed, lr, step, h_loss, h_grad_norm);
}

static gpt_status make_bucket_events(gpt_model* m) {
  if (!m->bucket_ev.empty()) return GPT_OK;
  for (int i = 0; i < m->L + 1; i++) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess)
      return check_cuda(m, "train_step_accumulate: event creation");
    m->bucket_ev.push_back(e);
  }
  return GPT_OK;
}

gpt_status gpt_train_step_accumulate(gpt_model* m, const void* d_stream, uint64_t stream_len, uint64_t data_seed,
                                     int32_t step, float* h_loss) {
  if (!m || !d_stream) return fail(m, GPT_ERR_INVALID_ARG, "train_step_accumulate: null argument");
  if (stream_len <= (uint64_t)m->T) return fail(m, GPT_ERR_INVALID_ARG, "stream shorter than block_size + 1");
  if (m->lora.on) return fail(m, GPT_ERR_UNSUPPORTED, "train_step_accumulate: not with adapters attached");
  gpt_status s = make_bucket_events(m);
  if (s != GPT_OK) return s;
  return train_common(m, 2, d_stream, stream_len, data_seed, 0.f, step, h_loss, nullptr);
}

gpt_status gpt_train_step_host_accumulate(gpt_model* m, const int32_t* h_idx, const int32_t* h_tgt, int32_t step,
                                          float* h_loss) {
  if (!m || !h_idx || !h_tgt) return fail(m, GPT_ERR_INVALID_ARG, "train_step_host_accumulate: null argument");
  if (m->lora.on) return fail(m, GPT_ERR_UNSUPPORTED, "train_step_host_accumulate: not with adapters attached");
  gpt_status s = make_bucket_events(m);
  if (s != GPT_OK) return s;
  size_t bytes = (size_t)m->ga * m->M * 4;
  cudaMemcpyAsync(m->stage_idx, h_idx, bytes, cudaMemcpyHostToDevice, m->ctx.stream);
  cudaMemcpyAsync(m->stage_tgt, h_tgt, bytes, cudaMemcpyHostToDevice, m->ctx.stream);
  return train_common(m, 3, nullptr, 0, 0, 0.f, step, h_loss, nullptr);
}

gpt_status gpt_stream_wait_bucket(gpt_model* m, int32_t bucket, void* cuda_stream) {
  if (!m) return GPT_ERR_INVALID_ARG;
  if (bucket < 0 || bucket >= (int)m->bucket_ev.size())
    return fail(m, GPT_ERR_INVALID_ARG, "stream_wait_bucket: no such bucket (run gpt_train_step_accumulate first)");
  if (cudaStreamWaitEvent((cudaStream_t)cuda_stream, m->bucket_ev[bucket], 0) != cudaSuccess)
    return check_cuda(m, "stream_wait_bucket");
  return GPT_OK;
}

gpt_status gpt_step_loss(gpt_model* m, float* h_loss) {
  if (!m || !h_loss) return GPT_ERR_INVALID_ARG;
  float sc[4];
  gpt_status s = sync_and_flags(m, "step_loss", sc);
  *h_loss = sc[1];
  return s;
}

gpt_status gpt_grad_arena(gpt_model* m, float** d_grad, int64_t* n_floats) {
  if (!m || !d_grad || !n_floats) return GPT_ERR_INVALID_ARG;
  *d_grad = m->g;
  *n_floats = m->n_total;
  return GPT_OK;
}

gpt_status gpt_zero1_shard(const gpt_config* cfg, int32_t world, int32_t rank, int64_t* offset, int64_t* count,
                           int64_t* stride) {
  if (!offset || !count || !stride || world < 1 || world > kZeroMaxWorld || rank < 0 || rank >= world)
    return GPT_ERR_INVALID_ARG;
  gpt_status s = validate(cfg, nullptr);
  if (s != GPT_OK) return s;
  gpt_model m;
  derive(m, cfg);
  zero_shard_of(m.n_total, world, rank, offset, count, stride);
  return GPT_OK;
}

gpt_status gpt_state_arenas(gpt_model* m, float** d_param, float** d_grad, float** d_adam_m, float** d_adam_v,
                            void** d_param_bf16, int64_t* n_floats, int64_t* n_alloc, int64_t* n_moment_alloc) {
  if (!m || !d_param || !d_grad || !d_adam_m || !d_adam_v || !d_param_bf16 || !n_floats || !n_alloc ||
      !n_moment_alloc)
    return GPT_ERR_INVALID_ARG;
  *n_moment_alloc = m->zero_sharded ? m->zero_stride : m->n_total + kArenaSlack;
  *d_param = m->w;
  *d_grad = m->g;
  *d_adam_m = m->am;
  *d_adam_v = m->av;
  *d_param_bf16 = m->wb;
  *n_floats = m->n_total;
  *n_alloc = m->n_total + kArenaSlack;
  return GPT_OK;
}

// shard bounds as gpt_zero1_shard gives them: float4-aligned, inside the arena
static gpt_status check_shard(gpt_model* m, int64_t offset, int64_t count, const char* what) {
  if (m->lora.on) return fail(m, GPT_ERR_STATE, "%s: LoRA adapters are attached", what);
  if (offset < 0 || count < 0 || offset % 4 || count % 4 || offset + count > m->n_total)
    return fail(m, GPT_ERR_INVALID_ARG, "%s: shard outside the arena or not a multiple of 4", what);
  return GPT_OK;
}

gpt_status gpt_grad_sumsq_shard(gpt_model* m, int64_t offset, int64_t count, double* d_partials) {
  if (!m || !d_partials) return GPT_ERR_INVALID_ARG;
  gpt_status s = check_shard(m, offset, count, "grad_sumsq_shard");
  if (s != GPT_OK) return s;
  Ctx& c = m->ctx;
  const int blocks = sumsq_blocks(c);
  cudaMemsetAsync(d_partials, 0, GPT_NORM_PARTIALS * sizeof(double), c.stream);
  if (count > 0) sumsq_partials(c, m->g + offset, count, d_partials, blocks);
  return check_cuda(m, "grad_sumsq_shard");
}

gpt_status gpt_clip_adamw_shard(gpt_model* m, float lr, int32_t step, int64_t offset, int64_t count,
                                float grad_scale, const double* d_partials, int32_t n_partials, float* h_grad_norm) {
  if (!m || !d_partials || n_partials < 1) return GPT_ERR_INVALID_ARG;
  if (step < 1) return fail(m, GPT_ERR_INVALID_ARG, "step must be >= 1");
  if (!(grad_scale > 0.f) || !isfinite(grad_scale)) return fail(m, GPT_ERR_INVALID_ARG, "grad_scale must be > 0");
  gpt_status s = check_shard(m, offset, count, "clip_adamw_shard");
  if (s != GPT_OK) return s;
  if (m->zero_sharded && (offset != m->zero_off || count != m->zero_cnt))
    return fail(m, GPT_ERR_INVALID_ARG, "clip_adamw_shard: the model holds the moments of shard [%lld, +%lld) only",
                (long long)m->zero_off, (long long)m->zero_cnt);
  Ctx& c = m->ctx;
  AdamArgs a;
  a.w = m->w + offset;
  a.g = m->g + offset;
  a.m = m->zero_sharded ? m->am : m->am + offset;  // sharded: the compact moments of the own shard
  a.v = m->zero_sharded ? m->av : m->av + offset;
  a.wb = m->wb ? m->wb + offset : nullptr;
  a.n = count;
  a.n_decay = std::max<int64_t>(0, std::min<int64_t>(count, m->n_decay - offset));
  a.norm_partials = d_partials;
  a.norm_blocks = n_partials;
  a.norm_out = m->scal + 2;
  a.lr = lr;
  a.beta1 = m->cfg.beta1;
  a.beta2 = m->cfg.beta2;
  a.eps = m->cfg.eps;
  a.wd = m->cfg.weight_decay;
  a.clip = m->cfg.grad_clip;
  a.gscale = grad_scale;
  bias_corrections(m, step, &a.bc1, &a.bc2);
  // k_adamw clears the shard's gradients; the rest of the arena (this
  // replica's own sums of the other shards) is cleared here
  if (offset > 0) cudaMemsetAsync(m->g, 0, (size_t)offset * 4, c.stream);
  if (offset + count < m->n_total)
    cudaMemsetAsync(m->g + offset + count, 0, (size_t)(m->n_total - offset - count) * 4, c.stream);
  adamw(c, a);
  s = check_cuda(m, "clip_adamw_shard");
  if (s != GPT_OK) return s;
  if (h_grad_norm) {
    float sc[4];
    s = sync_and_flags(m, "clip_adamw_shard", sc);
    *h_grad_norm = sc[2];
  }
  return s;
}

gpt_status gpt_grad_buckets(const gpt_config* cfg, int32_t cap, int64_t* h_offset, int64_t* h_count,
                            int32_t* h_bucket, int32_t* n_ranges) {
  if (!n_ranges) return GPT_ERR_INVALID_ARG;
  gpt_status s = validate(cfg, nullptr);
  if (s != GPT_OK) return s;
  gpt_model m;
  derive(m, cfg);
  const std::vector<GradRange> r = grad_ranges(m);
  *n_ranges = (int32_t)r.size();
  if (cap < (int32_t)r.size()) return h_offset ? GPT_ERR_INVALID_ARG : GPT_OK;
  if (!h_offset || !h_count || !h_bucket) return GPT_ERR_INVALID_ARG;
  for (size_t i = 0; i < r.size(); i++) {
    h_offset[i] = r[i].off;
    h_count[i] = r[i].count;
    h_bucket[i] = r[i].bucket;
  }
  return GPT_OK;
}

gpt_status gpt_train_step_host(gpt_model* m, const int32_t* h_idx, const int32_t* h_tgt, float lr, int32_t step,
                               float* h_loss, float* h_grad_norm) {
  if (!m || !h_idx || !h_tgt) return fail(m, GPT_ERR_INVALID_ARG, "train_step_host: null argument");
  size_t bytes = (size_t)m->ga * m->M * 4;
  cudaMemcpyAsync(m->stage_idx, h_idx, bytes, cudaMemcpyHostToDevice, m->ctx.stream);
  cudaMemcpyAsync(m->stage_tgt, h_tgt, bytes, cudaMemcpyHostToDevice, m->ctx.stream);
  return train_common(m, 1, nullptr, 0, 0, lr, step, h_loss, h_grad_norm);
}

// The kernels and copies of one gpt_generate call (prefill, draws, decoding
// steps), enqueued on the model's stream.
static gpt_status generate_body(gpt_model* m, const int32_t* d_prompt, int32_t T0, int32_t n_new, float temperature,
                                int32_t top_k, float top_p, const float* d_uniform, int32_t* d_out) {
  Ctx& c = m->ctx;
  const int B = m->B, Tn = m->T, Tout = T0 + n_new;
  const size_t es = m->asz;
  const float saved_drop = m->cfg.dropout;
  m->cfg.dropout = 0.f;  // inference runs without dropout
  const float tp = top_p > 0.f ? top_p : 1e-30f;
  // prefill: the prompt (zero-padded to block_size; causal attention keeps the
  // padding out of the prompt's positions) through the full forward, which
  // fills the qkv caches of positions < T0 and the logits of position T0 - 1
  cudaMemsetAsync(m->stage_idx, 0, (size_t)m->M * 4, c.stream);
  cudaMemsetAsync(m->stage_tgt, 0, (size_t)m->M * 4, c.stream);
  cudaMemcpy2DAsync(m->stage_idx, (size_t)Tn * 4, d_prompt, (size_t)T0 * 4, (size_t)T0 * 4, B,
                    cudaMemcpyDeviceToDevice, c.stream);
  cudaMemcpy2DAsync(d_out, (size_t)Tout * 4, d_prompt, (size_t)T0 * 4, (size_t)T0 * 4, B, cudaMemcpyDeviceToDevice,
                    c.stream);
  check_tokens(c, m->stage_idx, m->stage_tgt, m->M, m->V, m->idx, m->tgt);
  gpt_status s = forward_any(m, false, m->scal + 6, 1.0f / (float)m->M, 0);
  if (s == GPT_OK) {
    sample_rows(c, m->logits + (size_t)(T0 - 1) * m->Vp * es, m->bf16m, B, m->V, (long)Tn * m->Vp, temperature,
                top_k, tp, d_uniform, m->dec_tok);
    cudaMemcpy2DAsync(d_out + T0, (size_t)Tout * 4, m->dec_tok, 4, 4, B, cudaMemcpyDeviceToDevice, c.stream);
  }
  for (int i = 1; i < n_new && s == GPT_OK; i++) {
    const int t = T0 + i - 1;  // position of the token just drawn
    s = m->bf16m ? decode_step_t<bf16>(m, t) : decode_step_t<float>(m, t);
    if (s != GPT_OK) break;
    sample_rows(c, m->dec_logits, m->bf16m, B, m->V, m->Vp, temperature, top_k, tp, d_uniform + (size_t)i * B,
                m->dec_tok);
    cudaMemcpy2DAsync(d_out + t + 1, (size_t)Tout * 4, m->dec_tok, 4, 4, B, cudaMemcpyDeviceToDevice, c.stream);
  }
  m->cfg.dropout = saved_drop;
  if (s != GPT_OK) return s;
  return check_cuda(m, "generate");
}

gpt_status gpt_generate(gpt_model* m, const int32_t* d_prompt, int32_t T0, int32_t n_new, float temperature,
                        int32_t top_k, float top_p, const float* d_uniform, int32_t* d_out) {
  if (!m || !d_prompt || !d_uniform || !d_out) return fail(m, GPT_ERR_INVALID_ARG, "generate: null argument");
  if (T0 < 1 || n_new < 1 || (long)T0 + n_new > m->T)
    return fail(m, GPT_ERR_INVALID_ARG, "generate: need 1 <= prompt length and prompt + new tokens <= block_size");
  if (m->rc) return fail(m, GPT_ERR_UNSUPPORTED, "generate: the key / value cache needs recompute = 0");
  Ctx& c = m->ctx;
  // A repeated call shape (same buffers, lengths and sampling parameters)
  // replays a CUDA graph of the whole call: the first call runs eagerly, the
  // second is captured, later ones replay.
  uint64_t key[8] = {(uint64_t)(uintptr_t)d_prompt, (uint64_t)(uintptr_t)d_uniform, (uint64_t)(uintptr_t)d_out,
                     (uint64_t)T0, (uint64_t)n_new, 0, (uint64_t)(uint32_t)top_k, 0};
  memcpy(&key[5], &temperature, 4);
  memcpy(&key[7], &top_p, 4);
  bool replay = m->graphs_on && !c.timing;
  if (memcmp(key, m->gen_key, sizeof key) != 0) {  // a new call shape starts over
    if (m->gen_exec) cudaGraphExecDestroy(m->gen_exec);
    m->gen_exec = nullptr;
    m->gen_warm = 0;
    memcpy(m->gen_key, key, sizeof key);
  }
  gpt_status s = GPT_OK;
  if (replay && !m->gen_exec) {
    if (m->gen_warm < 1) {
      m->gen_warm++;
      replay = false;
    } else {
      bool ok = m->cap_stream || cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking) == cudaSuccess;
      cudaStream_t user = c.stream;
      const uint64_t l0 = c.launches;
      cudaGraph_t g = nullptr;
      if (ok) ok = cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
      if (ok) {
        c.stream = m->cap_stream;
        s = generate_body(m, d_prompt, T0, n_new, temperature, top_k, top_p, d_uniform, d_out);
        c.stream = user;
        m->gen_launches = c.launches - l0;
        ok = cudaStreamEndCapture(m->cap_stream, &g) == cudaSuccess && s == GPT_OK;
      }
      if (ok) ok = cudaGraphInstantiate(&m->gen_exec, g, 0) == cudaSuccess;
      if (g) cudaGraphDestroy(g);
      c.launches = l0;
      if (!ok) {
        cudaGetLastError();
        m->gen_exec = nullptr;
        m->gen_warm = 0;
        m->have_forward = false;
        if (s != GPT_OK) return s;
        return fail(m, GPT_ERR_CUDA,
                    "generate: capturing the call into a CUDA graph failed (nothing ran; "
                    "gpt_set_graphs(m, 0) runs calls eagerly)");
      }
    }
  }
  if (replay && m->gen_exec) {
    if (cudaGraphLaunch(m->gen_exec, c.stream) != cudaSuccess) return check_cuda(m, "generate graph launch");
    c.launches += m->gen_launches;
  } else {
    s = generate_body(m, d_prompt, T0, n_new, temperature, top_k, top_p, d_uniform, d_out);
  }
  m->have_forward = false;
  if (s != GPT_OK) return s;
  return sync_and_flags(m, "generate", nullptr);
}

gpt_status gpt_eval_loss(gpt_model* m, const void* d_stream, uint64_t stream_len, uint64_t data_seed,
                         int32_t n_batches, float* h_loss) {
  if (!m || !d_stream || !h_loss || n_batches < 1) return fail(m, GPT_ERR_INVALID_ARG, "eval_loss: bad argument");
  if (stream_len <= (uint64_t)m->T) return fail(m, GPT_ERR_INVALID_ARG, "stream shorter than block_size + 1");
  Ctx& c = m->ctx;
  const float saved_drop = m->cfg.dropout;
  m->cfg.dropout = 0.f;  // evaluation runs without dropout
  gpt_status s = GPT_OK;
  for (int i = 0; i < n_batches && s == GPT_OK; i++) {
    gather_batch(c, d_stream, m->cfg.token_dtype == GPT_TOK_U16, stream_len, data_seed, i + 1, 0, m->B, m->T, m->V,
                 m->idx, m->tgt);
    s = forward_any(m, false, m->scal + 5, 1.0f / (float)(m->M * (long)n_batches), i > 0);
  }
  m->cfg.dropout = saved_drop;
  m->have_forward = false;
  if (s != GPT_OK) return s;
  float v = 0.f;
  cudaMemcpyAsync(&v, m->scal + 5, 4, cudaMemcpyDeviceToHost, c.stream);
  s = sync_and_flags(m, "eval_loss", nullptr);
  *h_loss = v;
  return s;
}

gpt_status gpt_sample(const void* d_logits, int32_t logits_bf16, int32_t rows, int32_t V, int64_t ld,
                      float temperature, int32_t top_k, float top_p, const float* d_uniform, int32_t* d_out,
                      void* cuda_stream) {
  if (!d_logits || !d_uniform || !d_out || rows < 1 || V < 1 || ld < V) return GPT_ERR_INVALID_ARG;
  Ctx c;
  c.stream = (cudaStream_t)cuda_stream;
  // top_p <= 0: the nucleus is the most probable token(s)
  sample_rows(c, d_logits, logits_bf16 != 0, rows, V, ld, temperature, top_k, top_p > 0.f ? top_p : 1e-30f,
              d_uniform, d_out);
  return cudaGetLastError() == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

gpt_status gpt_gather_batch(gpt_model* m, const void* d_stream, uint64_t stream_len, uint64_t data_seed, int32_t step,
                            int32_t micro, int32_t* d_idx, int32_t* d_tgt) {
  if (!m || !d_stream || !d_idx || !d_tgt) return fail(m, GPT_ERR_INVALID_ARG, "gather_batch: null argument");
  if (stream_len <= (uint64_t)m->T) return fail(m, GPT_ERR_INVALID_ARG, "stream shorter than block_size + 1");
  gather_batch(m->ctx, d_stream, m->cfg.token_dtype == GPT_TOK_U16, stream_len, data_seed, step, micro, m->B, m->T,
               m->V, d_idx, d_tgt);
  return check_cuda(m, "gather_batch");
}

gpt_status gpt_num_tensors(gpt_model* m, int32_t* n) {
  if (!m || !n) return GPT_ERR_INVALID_ARG;
  *n = (int32_t)m->tensors.size();
  return GPT_OK;
}

gpt_status gpt_tensor_info(gpt_model* m, int32_t i, const char** name, int64_t shape[2]) {
  if (!m || i < 0 || i >= (int32_t)m->tensors.size()) return GPT_ERR_INVALID_ARG;
  if (name) *name = m->tensors[i].name.c_str();
  if (shape) {
    shape[0] = m->tensors[i].rows;
    shape[1] = m->tensors[i].cols;
  }
  return GPT_OK;
}

static float* kind_arena(gpt_model* m, int kind) {
  switch (kind) {
    case GPT_PARAM: return m->w;
    case GPT_GRAD: return m->g;
    case GPT_ADAM_M: return m->am;
    case GPT_ADAM_V: return m->av;
  }
  return nullptr;
}

gpt_status gpt_get_tensor(gpt_model* m, int32_t i, int32_t kind, float* h_out) {
  if (!m || !h_out || i < 0 || i >= (int32_t)m->tensors.size()) return GPT_ERR_INVALID_ARG;
  if (m->zero_sharded && (kind == GPT_ADAM_M || kind == GPT_ADAM_V))
    return fail(m, GPT_ERR_UNSUPPORTED, "the moments are sharded (zero_world > 1)");
  float* a = kind_arena(m, kind);
  if (!a) return GPT_ERR_INVALID_ARG;
  const TensorRec& t = m->tensors[i];
  cudaMemcpyAsync(h_out, a + t.off, (size_t)t.rows * t.cols * 4, cudaMemcpyDeviceToHost, m->ctx.stream);
  return sync_and_flags(m, "get_tensor", nullptr);
}

gpt_status gpt_set_tensor(gpt_model* m, int32_t i, int32_t kind, const float* h_in) {
  if (!m || !h_in || i < 0 || i >= (int32_t)m->tensors.size()) return GPT_ERR_INVALID_ARG;
  if (m->zero_sharded && (kind == GPT_ADAM_M || kind == GPT_ADAM_V))
    return fail(m, GPT_ERR_UNSUPPORTED, "the moments are sharded (zero_world > 1)");
  float* a = kind_arena(m, kind);
  if (!a) return GPT_ERR_INVALID_ARG;
  const TensorRec& t = m->tensors[i];
  size_t n = (size_t)t.rows * t.cols;
  cudaMemcpyAsync(a + t.off, h_in, n * 4, cudaMemcpyHostToDevice, m->ctx.stream);
  if (kind == GPT_PARAM && m->bf16m) to_bf16(m->ctx, m->w + t.off, m->wb + t.off, (long)n);
  return sync_and_flags(m, "set_tensor", nullptr);
}

gpt_status gpt_get_logits(gpt_model* m, float* h_out) {
  if (!m || !h_out) return GPT_ERR_INVALID_ARG;
  gpt_status s = sync_and_flags(m, "get_logits", nullptr);
  if (s != GPT_OK) return s;
  size_t rows = m->M;
  if (m->bf16m) {
    std::vector<uint16_t> tmp((size_t)rows * m->Vp);
    cudaMemcpy(tmp.data(), m->logits, tmp.size() * 2, cudaMemcpyDeviceToHost);
    for (size_t r = 0; r < rows; r++)
      for (int j = 0; j < m->V; j++) {
        uint32_t u = (uint32_t)tmp[r * m->Vp + j] << 16;
        memcpy(&h_out[r * m->V + j], &u, 4);
      }
  } else {
    cudaMemcpy2D(h_out, (size_t)m->V * 4, m->logits, (size_t)m->Vp * 4, (size_t)m->V * 4, rows,
                 cudaMemcpyDeviceToHost);
  }
  return check_cuda(m, "get_logits");
}

gpt_status gpt_get_argmax(gpt_model* m, int32_t* h_out) {
  if (!m || !h_out) return GPT_ERR_INVALID_ARG;
  argmax_rows(m->ctx, m->logits, m->bf16m ? 1 : 0, m->M, m->V, m->Vp, m->argmax_out);
  cudaMemcpyAsync(h_out, m->argmax_out, (size_t)m->M * 4, cudaMemcpyDeviceToHost, m->ctx.stream);
  return sync_and_flags(m, "get_argmax", nullptr);
}

gpt_status gpt_argmax_rows(gpt_model* m, const float* d_rows, int32_t rows, int32_t cols, int32_t* h_out) {
  if (!m || !d_rows || !h_out || rows <= 0 || cols <= 0 || rows > m->M + 64) return GPT_ERR_INVALID_ARG;
  argmax_rows(m->ctx, d_rows, 0, rows, cols, cols, m->argmax_out);
  cudaMemcpyAsync(h_out, m->argmax_out, (size_t)rows * 4, cudaMemcpyDeviceToHost, m->ctx.stream);
  return sync_and_flags(m, "argmax_rows", nullptr);
}

gpt_status gpt_get_lse(gpt_model* m, float* h_out) {
  if (!m || !h_out) return GPT_ERR_INVALID_ARG;
  cudaMemcpyAsync(h_out, m->row_lse, (size_t)m->M * 4, cudaMemcpyDeviceToHost, m->ctx.stream);
  return sync_and_flags(m, "get_lse", nullptr);
}

gpt_status gpt_get_embed_routing(gpt_model* m, int32_t* h_n_unique, int32_t* h_sorted_tok, int32_t* h_sorted_pos) {
  if (!m || !h_n_unique || !h_sorted_tok || !h_sorted_pos) return GPT_ERR_INVALID_ARG;
  cudaMemcpyAsync(h_n_unique, m->nuniq, 4, cudaMemcpyDeviceToHost, m->ctx.stream);
  cudaMemcpyAsync(h_sorted_tok, m->stok, (size_t)m->M * 4, cudaMemcpyDeviceToHost, m->ctx.stream);
  cudaMemcpyAsync(h_sorted_pos, m->spos, (size_t)m->M * 4, cudaMemcpyDeviceToHost, m->ctx.stream);
  return sync_and_flags(m, "get_embed_routing", nullptr);
}

gpt_status gpt_dropout_mask(gpt_model* m, int64_t counter, int32_t layer, int32_t site, int64_t n, uint8_t* h_out) {
  if (!m || !h_out || n <= 0 || counter < 0) return GPT_ERR_INVALID_ARG;
  size_t cap = (size_t)m->M * 4 * m->d * m->asz;  // the MLP-gradient buffer serves as scratch
  if ((size_t)n > cap) return fail(m, GPT_ERR_INVALID_ARG, "dropout_mask: n larger than the scratch buffer");
  DropKey k = make_drop_key(m->cfg.dropout_seed, (uint64_t)counter, layer, site, m->cfg.dropout);
  dropout_mask(m->ctx, k, n, m->dh);
  cudaMemcpyAsync(h_out, m->dh, (size_t)n, cudaMemcpyDeviceToHost, m->ctx.stream);
  return sync_and_flags(m, "dropout_mask", nullptr);
}

size_t gpt_state_floats(gpt_model* m) {
  if (!m) return 0;
  size_t n = 0;
  for (auto& t : m->tensors) n += (size_t)t.rows * t.cols;
  return n;
}

gpt_status gpt_get_state(gpt_model* m, float* hp, float* hm, float* hv) {
  if (!m || !hp || !hm || !hv) return GPT_ERR_INVALID_ARG;
  if (m->zero_sharded) return fail(m, GPT_ERR_UNSUPPORTED, "get_state: the moments are sharded (zero_world > 1)");
  size_t o = 0;
  for (auto& t : m->tensors) {
    size_t n = (size_t)t.rows * t.cols;
    cudaMemcpyAsync(hp + o, m->w + t.off, n * 4, cudaMemcpyDeviceToHost, m->ctx.stream);
    cudaMemcpyAsync(hm + o, m->am + t.off, n * 4, cudaMemcpyDeviceToHost, m->ctx.stream);
    cudaMemcpyAsync(hv + o, m->av + t.off, n * 4, cudaMemcpyDeviceToHost, m->ctx.stream);
    o += n;
  }
  return sync_and_flags(m, "get_state", nullptr);
}

gpt_status gpt_set_state(gpt_model* m, const float* hp, const float* hm, const float* hv) {
  if (!m || !hp || !hm || !hv) return GPT_ERR_INVALID_ARG;
  if (m->zero_sharded) return fail(m, GPT_ERR_UNSUPPORTED, "set_state: the moments are sharded (zero_world > 1)");
  size_t o = 0;
  for (auto& t : m->tensors) {
    size_t n = (size_t)t.rows * t.cols;
    cudaMemcpyAsync(m->w + t.off, hp + o, n * 4, cudaMemcpyHostToDevice, m->ctx.stream);
    cudaMemcpyAsync(m->am + t.off, hm + o, n * 4, cudaMemcpyHostToDevice, m->ctx.stream);
    cudaMemcpyAsync(m->av + t.off, hv + o, n * 4, cudaMemcpyHostToDevice, m->ctx.stream);
    o += n;
  }
  if (m->bf16m) to_bf16(m->ctx, m->w, m->wb, m->n_total);
  return sync_and_flags(m, "set_state", nullptr);
}

gpt_status gpt_read_flags(gpt_model* m, uint32_t* h_flags) {
  if (!m || !h_flags) return GPT_ERR_INVALID_ARG;
  float sc[4];
  cudaMemcpyAsync(sc, m->scal, 16, cudaMemcpyDeviceToHost, m->ctx.stream);
  if (cudaStreamSynchronize(m->ctx.stream) != cudaSuccess) return check_cuda(m, "read_flags");
  memcpy(h_flags, &sc[3], 4);
  return GPT_OK;
}

gpt_status gpt_clear_flags(gpt_model* m) {
  if (!m) return GPT_ERR_INVALID_ARG;
  cudaMemsetAsync(m->scal + 3, 0, 4, m->ctx.stream);
  m->reported = 0;
  return check_cuda(m, "clear_flags");
}

gpt_status gpt_enable_timing(gpt_model* m, int32_t on) {
  if (!m) return GPT_ERR_INVALID_ARG;
  if (on) {
    if (!m->timing) m->timing = new Timing();
    m->timing->reset();
    m->ctx.timing = m->timing;
  } else {
    m->ctx.timing = nullptr;
  }
  return GPT_OK;
}

gpt_status gpt_kernel_times(gpt_model* m, int32_t cap, const char** names, float* total_ms, int32_t* launches,
                            int32_t* n_out) {
  if (!m || !n_out) return GPT_ERR_INVALID_ARG;
  if (!m->timing) {
    *n_out = 0;
    return GPT_OK;
  }
  cudaStreamSynchronize(m->ctx.stream);
  int k = 0;
  for (auto& kv : m->timing->recs) {
    if (k >= cap) break;
    float tot = 0.f;
    for (size_t j = 0; j + 1 < kv.second.ev.size(); j += 2) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, kv.second.ev[j], kv.second.ev[j + 1]);
      tot += ms;
    }
    if (names) names[k] = kv.first.c_str();
    if (total_ms) total_ms[k] = tot;
    if (launches) launches[k] = kv.second.launches;
    k++;
  }
  *n_out = k;
  return check_cuda(m, "kernel_times");
}

uint64_t gpt_launch_count(gpt_model* m) { return m ? m->ctx.launches : 0; }


// ---------------------------------------------------------------- LoRA adapters
static int lora_blocks(int L, int targets) { return L * __builtin_popcount((unsigned)targets & 7u); }

static size_t lora_bytes(long n) { return 4 * (((size_t)n * 4 + 255) / 256 * 256) + 1024; }

static void drop_train_graphs(gpt_model* m) {
  for (int k = 0; k < 4; k++) {
    if (m->gexec[k]) cudaGraphExecDestroy(m->gexec[k]);
    m->gexec[k] = nullptr;
    m->warm[k] = 0;
  }
}

gpt_status gpt_lora_workspace_bytes(const gpt_config* cfg, int32_t r, int32_t targets, size_t* out) {
  if (!cfg || !out) return GPT_ERR_INVALID_ARG;
  if (validate(cfg, nullptr) != GPT_OK) return GPT_ERR_CONFIG;
  if (r < 1 || r > 256 || targets < 1 || targets > 7) return GPT_ERR_INVALID_ARG;
  const long n = (long)lora_blocks(cfg->n_layer, targets) * 2 * r * cfg->n_embd;
  *out = lora_bytes(n);
  return GPT_OK;
}

gpt_status gpt_lora_attach(gpt_model* m, int32_t r, float alpha, int32_t targets, const float* h_a, void* d_ws,
                           size_t ws_bytes) {
  if (!m || !h_a || !d_ws) return fail(m, GPT_ERR_INVALID_ARG, "lora_attach: null argument");
  if (!m->bf16m) return fail(m, GPT_ERR_UNSUPPORTED, "lora_attach: adapters need the bf16 operand copies");
  if (r < 1 || r > 256 || targets < 1 || targets > 7 || !(alpha > 0.f))
    return fail(m, GPT_ERR_INVALID_ARG, "lora_attach: need 1 <= r <= 256, targets in 1..7, alpha > 0");
  const int d = m->d, nblk = lora_blocks(m->L, targets);
  if (nblk > LORA_MAX_BLOCKS) return fail(m, GPT_ERR_UNSUPPORTED, "lora_attach: too many adapted blocks");
  if (((long)r * d) % 4) return fail(m, GPT_ERR_INVALID_ARG, "lora_attach: r * n_embd must be a multiple of 4");
  const long n = (long)nblk * 2 * r * d;
  if (ws_bytes < lora_bytes(n) || (reinterpret_cast<uintptr_t>(d_ws) & 255))
    return fail(m, GPT_ERR_WORKSPACE_TOO_SMALL, "lora_attach: workspace too small or not 256-byte aligned");
  if (m->lora.on) {
    gpt_status s = gpt_lora_detach(m);
    if (s != GPT_OK) return s;
  }
  auto& L = m->lora;
  uint8_t* base = reinterpret_cast<uint8_t*>(d_ws);
  const size_t part = ((size_t)n * 4 + 255) / 256 * 256;
  L.lb.params = reinterpret_cast<float*>(base);
  L.lb.grads = reinterpret_cast<float*>(base + part);
  L.m = reinterpret_cast<float*>(base + 2 * part);
  L.v = reinterpret_cast<float*>(base + 3 * part);
  L.lb.d = d;
  L.lb.r = r;
  L.lb.nblk = nblk;
  L.lb.scale = alpha / (float)r;
  L.alpha = alpha;
  L.targets = targets;
  L.n = n;
  int b = 0;
  for (int l = 0; l < m->L; l++)
    for (int t = 0; t < 3; t++)
      if (targets & (1 << t)) L.lb.w_off[b++] = (long)m->layers[l].qkv_w + (long)t * d * d;
  // A from the caller, B = 0: the adapted model starts as the base model
  std::vector<float> host((size_t)n, 0.f);
  for (int k = 0; k < nblk; k++)
    memcpy(host.data() + (size_t)k * 2 * r * d, h_a + (size_t)k * r * d, (size_t)r * d * 4);
  Ctx& c = m->ctx;
  cudaMemcpyAsync(L.lb.params, host.data(), (size_t)n * 4, cudaMemcpyHostToDevice, c.stream);
  cudaMemsetAsync(L.lb.grads, 0, (size_t)n * 4, c.stream);
  cudaMemsetAsync(L.m, 0, (size_t)n * 4, c.stream);
  cudaMemsetAsync(L.v, 0, (size_t)n * 4, c.stream);
  lora_merge(c, L.lb, m->w, m->wb);
  drop_train_graphs(m);
  L.on = true;
  return sync_and_flags(m, "lora_attach", nullptr);
}

gpt_status gpt_lora_detach(gpt_model* m) {
  if (!m) return GPT_ERR_INVALID_ARG;
  auto& L = m->lora;
  if (!L.on) return GPT_OK;
  const long dd = (long)m->d * m->d;
  for (int k = 0; k < L.lb.nblk; k++) to_bf16(m->ctx, m->w + L.lb.w_off[k], m->wb + L.lb.w_off[k], dd);
  L.on = false;
  drop_train_graphs(m);
  return sync_and_flags(m, "lora_detach", nullptr);
}

gpt_status gpt_lora_read(gpt_model* m, int32_t which, float* h_out, size_t count) {
  if (!m || !h_out) return GPT_ERR_INVALID_ARG;
  auto& L = m->lora;
  if (!L.on) return fail(m, GPT_ERR_STATE, "lora_read: no adapters attached");
  if (count != (size_t)L.n || which < 0 || which > 3) return fail(m, GPT_ERR_INVALID_ARG, "lora_read: bad which/count");
  const float* src = which == 0 ? L.lb.params : which == 1 ? L.lb.grads : which == 2 ? L.m : L.v;
  cudaStreamSynchronize(m->ctx.stream);
  if (cudaMemcpy(h_out, src, count * 4, cudaMemcpyDeviceToHost) != cudaSuccess) return check_cuda(m, "lora_read");
  return GPT_OK;
}

gpt_status gpt_lora_write(gpt_model* m, const float* h_params, size_t count) {
  if (!m || !h_params) return GPT_ERR_INVALID_ARG;
  auto& L = m->lora;
  if (!L.on) return fail(m, GPT_ERR_STATE, "lora_write: no adapters attached");
  if (count != (size_t)L.n) return fail(m, GPT_ERR_INVALID_ARG, "lora_write: count must be the adapter size");
  cudaMemcpyAsync(L.lb.params, h_params, count * 4, cudaMemcpyHostToDevice, m->ctx.stream);
  lora_merge(m->ctx, L.lb, m->w, m->wb);
  return sync_and_flags(m, "lora_write", nullptr);
}

}  // extern "C"
