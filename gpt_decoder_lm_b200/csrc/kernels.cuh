// Internal launch interface between the step engine and the kernels.
#pragma once

#include "common.cuh"

namespace gpt {

// Per-launch bookkeeping: launch counter and optional CUDA-event timing by
// kernel name (used by the bench's per-kernel roofline report).
struct Timing;
struct Ctx {
  cudaStream_t stream = nullptr;
  uint32_t* flags = nullptr;  // device flag word
  int num_sms = 148;
  uint64_t launches = 0;
  Timing* timing = nullptr;   // null when timing is off
};

void timing_begin(Ctx& c, const char* name);
void timing_end(Ctx& c, const char* name);

// Launches kernel k as a programmatic dependent of the stream's previous
// kernel (cudaLaunchAttributeProgrammaticStreamSerialization): its blocks may
// be scheduled while that kernel's last wave drains, and wait in pdl_wait()
// for its completion.  Every kernel launched this way calls pdl_wait() in
// every block before any global-memory access that a kernel before it may
// write or read.
template <typename... KP, typename... A>
inline cudaError_t launch_pdl(void (*k)(KP...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, A... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

struct LaunchScope {
  Ctx& c;
  const char* name;
  LaunchScope(Ctx& c_, const char* n) : c(c_), name(n) {
    c.launches++;
    if (c.timing) timing_begin(c, name);
  }
  ~LaunchScope() {
    if (c.timing) timing_end(c, name);
  }
};

// ---------------------------------------------------------------- GEMM
// D[m, n] = sum_k A[m, k] * B[n, k], fp32 accumulation, then an epilogue.
enum EpiKind {
  EPI_STORE = 0,      // out = acc                                   (operand type)
  EPI_BIAS = 1,       // out = acc + bias                            (operand type)
  EPI_BIAS_ACT = 2,   // h = acc + bias: out = act'(h) (kept for backward), out2 = act(h)
  EPI_RESADD = 3,     // res_out = res_in + drop(acc + bias)         (fp32)
  EPI_ACT_BWD = 4,    // out = acc * aux (aux = the saved act'(h))   (operand type)
  EPI_ACC_F32 = 5,    // outf += acc                                 (fp32, grad accumulation)
  EPI_STORE_F32 = 6   // outf = acc                                  (fp32)
};
enum ActKind { ACT_GELU = 0, ACT_RELU = 1 };

struct GemmEpi {
  int kind = EPI_STORE;
  int act = ACT_GELU;
  void* out = nullptr;        // operand-typed output (kinds 0,1,2,4) or fp32 (5,6)
  void* out2 = nullptr;       // activation output of EPI_BIAS_ACT (same ld as out)
  int ldo = 0;
  const void* aux = nullptr;  // act'(h) of EPI_ACT_BWD (operand type, ld = ldo)
  const float* bias = nullptr;
  const float* res_in = nullptr;
  float* res_out = nullptr;
  int ld_res = 0;
  DropKey drop{};             // EPI_RESADD; element index = m * N + n
  // EPI_ACT_BWD on the tensor cores: column sums of the stored (operand-typed)
  // output, one fp32 row per 32-row group: colsum[m / 32][n] (= or += with
  // colsum_acc).  Null: none.
  float* colsum = nullptr;
  bool colsum_acc = false;
};

struct GemmDesc {
  int M = 0, N = 0, K = 0;
  const void* A = nullptr;
  long lda = 0;
  bool a_kmajor = true;       // true: A[m,k] at A[m*lda + k]; false: at A[k*lda + m]
  const void* B = nullptr;
  long ldb = 0;
  bool b_kmajor = true;       // true: B[n,k] at B[n*ldb + k]; false: at B[k*ldb + n]
  GemmEpi epi;
  int split_k = 1;            // > 1 only with EPI_ACC_F32: most splits `partial` holds
  float* partial = nullptr;   // [split_k, M, N] fp32 scratch
  bool partial_accumulate = false;  // split partials are added into `partial` (else stored)
  bool reduce_partials = true;      // out += sum of the partials after the GEMM
  const char* name = nullptr; // timing label
};

// Kernel, tile width and split-K count the tensor-core GEMM uses for an
// M x N x K problem on `num_sms` SMs (split_ok: fp32-accumulating dW): the
// single-CTA kernel (128 x bn tiles, bn 256 or 128) or the pair-CTA kernel
// (256 x 256 tiles over two SMs).  mode: TC_ANY (the cost model picks),
// TC_SINGLE or TC_PAIR (forced; kernel tests).
enum { TC_ANY = 0, TC_SINGLE = 1, TC_PAIR = 2 };
struct TcPlan {
  int bn;
  int splits;
  int pair;
};
TcPlan gemm_tc_plan(long M, long N, long K, bool split_ok, int num_sms, int mode = TC_ANY);

// fp32 operands on CUDA cores (fp32 mode); bf16 operands on CUDA cores
// (reference path used by tests); bf16 operands on tcgen05 tensor cores.
void gemm_simt_f32(Ctx& c, const GemmDesc& g);
void gemm_simt_bf16(Ctx& c, const GemmDesc& g);
bool gemm_tc_supported(const GemmDesc& g);
// the pair-CTA kernel (256-row tiles over two SMs, cta_group::2) with a
// given split count; gemm_tc_bf16 calls it when the plan says so
bool gemm_tc2_launch(Ctx& c, const GemmDesc& g, int splits);
// GEMMs of at most 16 rows (decoding): bf16, both operands K-major, no split-K.
// With a SkinnyNorm, A is not read: the kernel computes it as the norm of the
// fp32 rows x [M, ldx] over K columns (LayerNorm with w, b; RMSNorm without).
struct SkinnyNorm {
  const float* x = nullptr;
  const float* w = nullptr;
  const float* b = nullptr;
  long ldx = 0;
  int rms = 0;
  float eps = 1e-5f;
};
bool gemm_skinny_supported(const GemmDesc& g);
bool skinny_norm_supported(const GemmDesc& g, const SkinnyNorm& n);
void gemm_skinny_bf16(Ctx& c, const GemmDesc& g, const SkinnyNorm* nrm = nullptr);
bool gemm_tc_bf16(Ctx& c, const GemmDesc& g, int mode = TC_ANY);  // false: tensor-map encode failed
// the split-K count gemm_tc_bf16 uses for g (1: none)
int gemm_tc_splits(const GemmDesc& g, int num_sms, int mode = TC_ANY);
// split-K reduction: out[m,n] += sum_s partial[s,m,n] (fixed order)
void splitk_reduce(Ctx& c, const float* partial, int splits, long MN, float* out);

// ---------------------------------------------------------------- attention
// qkv: [B, T, 3, H, hd] (row m = b*T + t holds q | k | v, heads contiguous)
// o: [B, T, H, hd]; lse: [B, H, T] natural-log log-sum-exp of the scaled scores.
struct AttnDesc {
  int B, T, H, hd;
  const void* qkv;
  void* o;
  float* lse;
  const void* dout;   // bwd: dO [B, T, H, hd]
  void* dqkv;         // bwd: [B, T, 3, H, hd]
  float* dsum;        // bwd scratch: rowsum(dO * O) [B, H, T]
  DropKey drop;       // site 1; elem = ((b*H + h)*T + i)*T + j
  // bwd (tensor-core kernels): column sums of the stored dqkv per 128-row
  // block, colsum[m / 128][3 H hd] (= or += with colsum_acc); null: none
  float* colsum = nullptr;
  int colsum_acc = 0;
};
template <typename T> void attn_fwd_simt(Ctx& c, const AttnDesc& a);
template <typename T> void attn_bwd_simt(Ctx& c, const AttnDesc& a);
// the tensor-core kernels' shape rule: head_dim 64 and T a multiple of 128
bool attn_tc_shape_ok(int T, int hd);
bool attn_tc_supported(const AttnDesc& a);  // shape rule plus 16-byte aligned pointers
// false: a tensor map could not be encoded (nothing launched)
bool attn_fwd_tc(Ctx& c, const AttnDesc& a);
bool attn_bwd_tc(Ctx& c, const AttnDesc& a);
// decoding: o [B, H*hd] = attention of position t against positions 0..t of
// the cache qkv [B, T, 3, H, hd]
template <typename T> void attn_decode(Ctx& c, const T* qkv, int B, int Tn, int H, int hd, int t, T* o);

// ---------------------------------------------------------------- memory-bound kernels
// step_dev (nullable): read the step index from device memory instead of `step`
void gather_batch(Ctx& c, const void* stream, int tok_u16, uint64_t len, uint64_t seed, int step, int micro,
                  int B, int T, int V, int32_t* idx, int32_t* tgt, const int* step_dev = nullptr);
// one-thread kernel: *step_dev = step; hyper = {lr, bc1, bc2}
void set_step_params(Ctx& c, int* step_dev, float* hyper, int step, float lr, float bc1, float bc2);
void check_tokens(Ctx& c, const int32_t* idx, const int32_t* tgt, long n, int V, int32_t* idx_out,
                  int32_t* tgt_out);

template <typename T>
void embed_fwd(Ctx& c, const int32_t* idx, const float* wte, const float* wpe, float* res, int B, int Tn, int d,
               DropKey drop);

// LayerNorm / RMSNorm forward: y (T), mean, rstd fp32 [rows]
template <typename T>
void norm_fwd(Ctx& c, const float* x, const float* w, const float* b, T* y, float* mean, float* rstd, long rows,
              int d, bool rms, float eps);

// Norm backward.  dx = norm'(dy) is added to dres (or stored when !accumulate);
// then dyb = drop(dres) is written (operand type) and its column sums, together
// with dgain = sum dy*xhat and dbias = sum dy, go to per-block partials
// part[blocks, 3, d] (order: dgain, dbeta, dbias_next).
struct NormBwd {
  const float* dy; const float* x; const float* mean; const float* rstd; const float* w;
  float* dres; bool accumulate;
  void* dyb; DropKey drop; bool want_dyb;
  float* part; int blocks;
  bool part_accumulate = false;  // add into part (else store)
  long rows; int d; bool rms;
};
template <typename T> void norm_bwd(Ctx& c, const NormBwd& p);
// partial rows k_norm_bwd writes (one resident wave of blocks)
int norm_bwd_blocks(Ctx& c, long rows, int d, bool bf16_out);
// the three slots of part[blocks, 3, d] into g0, g1, g2 (each nullable), one launch
void partial_reduce3(Ctx& c, const float* part, int blocks, int d, float* g0, float* g1, float* g2);

// column sums of an operand-typed [rows, N] matrix, deterministic: chunk
// partials part[colsum_chunks(rows), N] (= or += with accumulate), which
// colsum_reduce adds to grad
int colsum_chunks(long rows);
template <typename T> void colsum_partial(Ctx& c, const T* x, long rows, int N, float* part, bool accumulate);

// Cross-entropy over [M, Vp] logits (operand type).  Writes per-row lse and
// loss terms; with want_grad, overwrites logits with (softmax - onehot)*scale
// (pad columns 0).
template <typename T>
void ce_fwd_bwd(Ctx& c, T* logits, const int32_t* tgt, long M, int V, int Vp, float* lse, float* row_loss,
                bool want_grad, float scale);
void loss_reduce(Ctx& c, const float* row_loss, long M, float scale, float* loss_acc, int accumulate);

// embedding backward: routing (stable sort of positions by token) + sums
// `batches` independent sorts of M tokens each, stored back to back (one CTA each)
void embed_sort(Ctx& c, const int32_t* idx, long M, int32_t* sorted_tok, int32_t* sorted_pos, int32_t* n_unique,
                int batches = 1);
// seg_scratch: 2 * ceil(M / 32) * d floats (partial sums of segments that cross 32-slot chunks)
void embed_bwd(Ctx& c, const float* dres, const int32_t* sorted_tok, const int32_t* sorted_pos, long M, int Tn,
               int Bn, int d, DropKey drop, float* dwte, float* dwpe, float* seg_scratch);
// column partials [chunks, N] -> grad (+=), fixed order
void colsum_reduce(Ctx& c, const float* part, int chunks, int N, float* grad);

// grad norm partials, clip + AdamW
void sumsq_partials(Ctx& c, const float* g, long n, double* partials, int blocks);
int sumsq_blocks(Ctx& c);
struct AdamArgs {
  float* w; float* g; float* m; float* v; bf16* wb;  // wb may be null (fp32 mode)
  long n; long n_decay;
  const double* norm_partials; int norm_blocks; float* norm_out;
  float lr, beta1, beta2, eps, wd, clip, bc1, bc2;
  const float* hyper = nullptr;  // when set: {lr, bc1, bc2} read from device memory
  float gscale = 1.f;            // the gradient is gscale times the arena's values
};
void adamw(Ctx& c, const AdamArgs& a);

// LoRA adapters on row blocks (d x d) of the fused QKV weight
constexpr int LORA_MAX_BLOCKS = 144;
struct LoraBlocks {
  int d = 0, r = 0, nblk = 0;
  float scale = 0.f;            // alpha / r
  float* params = nullptr;      // per block: A [r, d], then B [d, r]
  float* grads = nullptr;       // the same layout
  long w_off[LORA_MAX_BLOCKS];  // element offset of each block's first row in the weight arena
};
// wb (bf16 operand copy) of every adapted block <- W0 + scale B A
void lora_merge(Ctx& c, const LoraBlocks& lb, const float* w, bf16* wb);
// adapter gradients from the gradient g of the merged weights (weight arena layout)
void lora_grads(Ctx& c, const LoraBlocks& lb, const float* g);
void to_bf16(Ctx& c, const float* src, bf16* dst, long n);
void argmax_rows(Ctx& c, const void* x, int is_bf16, long rows, int cols, int ld, int32_t* out);
void dropout_mask(Ctx& c, DropKey k, long n, uint8_t* out);
// one draw per row of logits [rows, ld] (temperature, top-k, top-p, uniform[row])
void sample_rows(Ctx& c, const void* logits, bool bf16_logits, int rows, int V, long ld, float temperature, int top_k,
                 float top_p, const float* uniform, int32_t* out);

}  // namespace gpt
