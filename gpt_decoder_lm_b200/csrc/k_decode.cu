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

// The same attention with 16-byte accesses and the loads of several keys in
// flight per thread: thread (g, c) handles chunk c (16 bytes of the head
// dimension) of the keys g, g + KP, g + 2 KP, ... (KP = threads / chunks per
// row).  Scores are reduced over the chunk lanes of a key by shuffles; the
// output sums each key group's p-weighted values, then adds the groups in
// order.  Needs hd * sizeof(T) a multiple of 16 and hd / (16 / sizeof(T)) a
// power of two of at most 32.
constexpr int DU = 8;  // keys per thread in flight

template <typename T>
__global__ void __launch_bounds__(DT) k_attn_decode_v(const T* __restrict__ qkv, int Tn, int H, int hd, int t,
                                                      float scale, T* __restrict__ o) {
  pdl_trigger();
  constexpr int VEC = 16 / sizeof(T);
  extern __shared__ float sc[];  // [t + 1] scores, then probabilities
  __shared__ float red[DT / 32];
  __shared__ float part[DT * 8];  // [key group][hd]
  const int CH = hd / VEC, KP = DT / CH;
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int c = tid % CH, g = tid / CH;
  const size_t row = (size_t)3 * H * hd;
  const T* base = qkv + (size_t)b * Tn * row;
  float qv[VEC];
  {
    const uint4 r = *reinterpret_cast<const uint4*>(base + (size_t)t * row + (size_t)h * hd + c * VEC);
    const T* e = reinterpret_cast<const T*>(&r);
#pragma unroll
    for (int v = 0; v < VEC; v++) qv[v] = to_f<T>(e[v]);
  }
  const T* kbase = base + (size_t)(H + h) * hd + c * VEC;
  const T* vbase = base + (size_t)(2 * H + h) * hd + c * VEC;
  for (int j0 = 0; j0 <= t; j0 += KP * DU) {
    uint4 kv[DU];
#pragma unroll
    for (int u = 0; u < DU; u++) {
      const int j = j0 + u * KP + g;
      kv[u] = j <= t ? *reinterpret_cast<const uint4*>(kbase + (size_t)j * row) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < DU; u++) {
      const T* e = reinterpret_cast<const T*>(&kv[u]);
      float s = 0.f;
#pragma unroll
      for (int v = 0; v < VEC; v++) s = fmaf(qv[v], to_f<T>(e[v]), s);
      for (int x = CH / 2; x > 0; x >>= 1) s += __shfl_xor_sync(0xffffffffu, s, x);
      const int j = j0 + u * KP + g;
      if (c == 0 && j <= t) sc[j] = s * scale;
    }
  }
  __syncthreads();
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
  float acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; v++) acc[v] = 0.f;
  for (int j0 = 0; j0 <= t; j0 += KP * DU) {
    uint4 vv[DU];
#pragma unroll
    for (int u = 0; u < DU; u++) {
      const int j = j0 + u * KP + g;
      vv[u] = j <= t ? *reinterpret_cast<const uint4*>(vbase + (size_t)j * row) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < DU; u++) {
      const int j = j0 + u * KP + g;
      const float p = j <= t ? sc[j] : 0.f;
      const T* e = reinterpret_cast<const T*>(&vv[u]);
#pragma unroll
      for (int v = 0; v < VEC; v++) acc[v] = fmaf(p, to_f<T>(e[v]), acc[v]);
    }
  }
#pragma unroll
  for (int v = 0; v < VEC; v++) part[g * hd + c * VEC + v] = acc[v];
  __syncthreads();
  for (int e = tid; e < hd; e += DT) {
    float r = 0.f;
    for (int k = 0; k < KP; k++) r += part[k * hd + e];
    o[(size_t)b * H * hd + (size_t)h * hd + e] = from_f<T>(r / tot);
  }
}

}  // namespace

template <typename T>
void attn_decode(Ctx& c, const T* qkv, int B, int Tn, int H, int hd, int t, T* o) {
  LaunchScope s(c, "attn_decode");
  const int vec = 16 / (int)sizeof(T), ch = hd / vec;
  const bool vec_ok = hd % vec == 0 && ch >= 1 && ch <= 32 && (ch & (ch - 1)) == 0 &&
                      (reinterpret_cast<uintptr_t>(qkv) & 15) == 0;
  const size_t smem = (size_t)(t + 1) * sizeof(float);
  const float scale = 1.0f / sqrtf((float)hd);
  if (vec_ok)
    k_attn_decode_v<T><<<B * H, DT, smem, c.stream>>>(qkv, Tn, H, hd, t, scale, o);
  else
    k_attn_decode<T><<<B * H, DT, smem, c.stream>>>(qkv, Tn, H, hd, t, scale, o);
}
template void attn_decode<float>(Ctx&, const float*, int, int, int, int, int, float*);
template void attn_decode<bf16>(Ctx&, const bf16*, int, int, int, int, int, bf16*);

}  // namespace gpt
