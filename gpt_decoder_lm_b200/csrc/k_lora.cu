// LoRA adapters on row blocks of the fused QKV projection ("使用 nanoGPT 构建
// 中型 GPT 微调管道" page, LoRA integration paragraph): a frozen W0 plus a
// trainable low-rank update, h = W0 x + s B (A x) with s = alpha / r,
// A [r, d], B [d, r].  Since h = (W0 + s B A) x, the GEMMs of the step run on
// the merged bf16 operand W0 + s B A of each adapted block, and the gradient
// of a block's merged weight, G = dL/dW (what the weight-gradient GEMM of the
// projection produces), gives the adapters' gradients by the chain rule:
//   dL/dB = s G A^T     dL/dA = s B^T G
// Every sum runs in a fixed order (deterministic).
#include "kernels.cuh"

namespace gpt {
namespace {

// wb[row0 + i][j] = bf16(w0[row0 + i][j] + s sum_k B[i][k] A[k][j]) for one
// block per blockIdx.y; threads over j (A reads coalesced, B broadcast)
__global__ void k_lora_merge(LoraBlocks lb, const float* __restrict__ w, bf16* __restrict__ wb) {
  pdl_trigger();
  const int blk = blockIdx.y, d = lb.d, r = lb.r;
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)d * d) return;
  const int i = (int)(idx / d), j = (int)(idx - (long)i * d);
  const float* A = lb.params + (size_t)blk * 2 * r * d;  // [r, d]
  const float* B = A + (size_t)r * d;                     // [d, r]
  float acc = 0.f;
  for (int k = 0; k < r; k++) acc = fmaf(B[(size_t)i * r + k], A[(size_t)k * d + j], acc);
  const long off = lb.w_off[blk] + (long)i * d + j;
  wb[off] = __float2bfloat16_rn(w[off] + lb.scale * acc);
}

// dB[i][k] = s sum_j G[i][j] A[k][j]: one thread per (i, k), j ascending
__global__ void k_lora_grad_b(LoraBlocks lb, const float* __restrict__ g) {
  pdl_trigger();
  const int blk = blockIdx.y, d = lb.d, r = lb.r;
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)d * r) return;
  const int i = (int)(idx / r), k = (int)(idx - (long)i * r);
  const float* A = lb.params + (size_t)blk * 2 * r * d;
  const float* G = g + lb.w_off[blk] + (size_t)i * d;
  float acc = 0.f;
  for (int j = 0; j < d; j++) acc = fmaf(G[j], A[(size_t)k * d + j], acc);
  lb.grads[(size_t)blk * 2 * r * d + (size_t)r * d + (size_t)i * r + k] = lb.scale * acc;
}

// dA[k][j] = s sum_i B[i][k] G[i][j]: one thread per (k, j), i ascending (G
// reads coalesced over j, B broadcast)
__global__ void k_lora_grad_a(LoraBlocks lb, const float* __restrict__ g) {
  pdl_trigger();
  const int blk = blockIdx.y, d = lb.d, r = lb.r;
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)r * d) return;
  const int k = (int)(idx / d), j = (int)(idx - (long)k * d);
  const float* B = lb.params + (size_t)blk * 2 * r * d + (size_t)r * d;
  const float* G = g + lb.w_off[blk] + j;
  float acc = 0.f;
  for (int i = 0; i < d; i++) acc = fmaf(B[(size_t)i * r + k], G[(size_t)i * d], acc);
  lb.grads[(size_t)blk * 2 * r * d + (size_t)k * d + j] = lb.scale * acc;
}

}  // namespace

void lora_merge(Ctx& c, const LoraBlocks& lb, const float* w, bf16* wb) {
  LaunchScope s(c, "lora_merge");
  dim3 grid((unsigned)(((long)lb.d * lb.d + 255) / 256), (unsigned)lb.nblk);
  k_lora_merge<<<grid, 256, 0, c.stream>>>(lb, w, wb);
}

void lora_grads(Ctx& c, const LoraBlocks& lb, const float* g) {
  const dim3 grid((unsigned)(((long)lb.d * lb.r + 255) / 256), (unsigned)lb.nblk);
  {
    LaunchScope s(c, "lora_grad_b");
    k_lora_grad_b<<<grid, 256, 0, c.stream>>>(lb, g);
  }
  LaunchScope s(c, "lora_grad_a");
  k_lora_grad_a<<<grid, 256, 0, c.stream>>>(lb, g);
}

}  // namespace gpt
