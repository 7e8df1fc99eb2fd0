// Attention of one new position against the key / value cache, for
// autoregressive decoding (microGPT page, section "单 GPU 高效推理：采样 +
// KV Cache": the keys and values of every earlier position are kept and the
// new token's are appended, instead of recomputing the past).
//
// The cache is the forward pass's own qkv activation [B, T, 3, H, hd] of each
// layer: the decode step's QKV GEMM writes position t there, and this kernel
// reads q_t and the keys / values of positions 0..t:
//   o[b, h] = softmax(q_t k_j^T / sqrt(hd), j <= t) V
#include "kernels.cuh"

namespace gpt {
namespace {

constexpr int DT = 128;  // threads per (b, h)

template <typename T>
__global__ void __launch_bounds__(DT) k_attn_decode(const T* __restrict__ qkv, int Tn, int H, int hd, int t,
                                                    float scale, T* __restrict__ o) {
  pdl_trigger();
  extern __shared__ float sc[];  // [t + 1] scores, then probabilities
  __shared__ float red[DT / 32];
  __shared__ float part[DT];
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const size_t row = (size_t)3 * H * hd;  // elements per position
  const T* base = qkv + (size_t)b * Tn * row;
  const T* q = base + (size_t)t * row + (size_t)h * hd;
  // scores: one warp per key, lanes across the head dimension
  for (int j = w; j <= t; j += DT / 32) {
    const T* k = base + (size_t)j * row + (size_t)(H + h) * hd;
    float s = 0.f;
    for (int e = lane; e < hd; e += 32) s = fmaf(to_f<T>(q[e]), to_f<T>(k[e]), s);
    s = warp_sum(s);
    if (lane == 0) sc[j] = s * scale;
  }
  __syncthreads();
  // maximum, then exp and the sum, in a fixed order
  float m = -INFINITY;
  for (int j = tid; j <= t; j += DT) m = fmaxf(m, sc[j]);
  m = warp_max(m);
  if (lane == 0) red[w] = m;
  __syncthreads();
  m = red[0];
  for (int k = 1; k < DT / 32; k++) m = fmaxf(m, red[k]);
  __syncthreads();
  float s = 0.f;
  for (int j = tid; j <= t; j += DT) {
    const float p = __expf(sc[j] - m);
    sc[j] = p;
    s += p;
  }
  s = warp_sum(s);
  if (lane == 0) red[w] = s;
  __syncthreads();
  float tot = 0.f;
  for (int k = 0; k < DT / 32; k++) tot += red[k];
  // o: thread (half, e) sums keys j = half, half + 2, ... of dimension e
  const int half = tid / 64, e0 = tid % 64;
  for (int eb = 0; eb < hd; eb += 64) {  // the same trip count in every thread
    const int e = eb + e0;
    float acc = 0.f;
    if (e < hd)
      for (int j = half; j <= t; j += 2)
        acc = fmaf(sc[j], to_f<T>(base[(size_t)j * row + (size_t)(2 * H + h) * hd + e]), acc);
    part[tid] = acc;
    __syncthreads();
    if (half == 0 && e < hd) o[(size_t)b * H * hd + (size_t)h * hd + e] = from_f<T>((part[tid] + part[tid + 64]) / tot);
    __syncthreads();
  }
}

}  // namespace

template <typename T>
void attn_decode(Ctx& c, const T* qkv, int B, int Tn, int H, int hd, int t, T* o) {
  LaunchScope s(c, "attn_decode");
  k_attn_decode<T><<<B * H, DT, (size_t)(t + 1) * sizeof(float), c.stream>>>(qkv, Tn, H, hd, t,
                                                                          1.0f / sqrtf((float)hd), o);
}
template void attn_decode<float>(Ctx&, const float*, int, int, int, int, int, float*);
template void attn_decode<bf16>(Ctx&, const bf16*, int, int, int, int, int, bf16*);

}  // namespace gpt
