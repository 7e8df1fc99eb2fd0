// Shared device/host helpers of the sm_100a GPT-2 training-step library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#define GPT_HD __host__ __device__ __forceinline__

namespace gpt {

typedef __nv_bfloat16 bf16;

// ----------------------------------------------------------------------------
// SplitMix64 (Steele, Lea & Flood 2014) used as a counter-based hash: the
// output of a generator whose state is x before its golden-gamma increment.
// ----------------------------------------------------------------------------
GPT_HD uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Dropout sites (GPT-2 placement): 0 embedding output (layer = n_layer),
// 1 attention probabilities, 2 attention projection output, 3 MLP output.
// The key of a site is splitmix64(seed ^ splitmix64(counter<<32 ^ layer<<8 ^
// site)) with counter = step * grad_accum + micro.  Eagerly launched kernels
// get it computed on the host; kernels of a replayed CUDA graph get step_dev
// (the step index the replay writes to device memory) and derive the key
// from it with drop_live(), so one captured step serves every step.
struct DropKey {
  uint64_t key;      // the site's key (valid when step_dev is null)
  uint32_t thresh;   // floor(p * 2^32); keep iff hash >> 32 >= thresh
  float scale;       // 1 / (1 - p)
  int active;
  int micro, ga;     // counter = (*step_dev) * ga + micro
  uint64_t seed, tag;  // tag = layer<<8 ^ site
  const int* step_dev;
};

GPT_HD uint64_t drop_site_key(uint64_t seed, uint64_t counter, uint64_t tag) {
  return splitmix64(seed ^ splitmix64((counter << 32) ^ tag));
}

GPT_HD DropKey make_drop_key(uint64_t seed, uint64_t counter, int layer, int site, float p) {
  DropKey k;
  k.tag = ((uint64_t)layer << 8) ^ (uint64_t)site;
  k.seed = seed;
  k.key = drop_site_key(seed, counter, k.tag);
  double t = (double)p * 4294967296.0;
  k.thresh = (uint32_t)(t >= 4294967295.0 ? 4294967295.0 : t);
  k.scale = p > 0.f ? 1.0f / (1.0f - p) : 1.0f;
  k.active = p > 0.f;
  k.micro = 0;
  k.ga = 1;
  k.step_dev = nullptr;
  return k;
}

// the key of a replayed graph's kernel: counter from the device step index
inline DropKey make_drop_key_dev(uint64_t seed, const int* step_dev, int ga, int micro, int layer, int site,
                                 float p) {
  DropKey k = make_drop_key(seed, 0, layer, site, p);
  k.step_dev = step_dev;
  k.ga = ga;
  k.micro = micro;
  return k;
}

#ifdef __CUDACC__
__device__ __forceinline__ DropKey drop_live(DropKey k) {
  if (k.active && k.step_dev) {
    const uint64_t counter = (uint64_t)((int64_t)(*k.step_dev) * k.ga + k.micro);
    k.key = drop_site_key(k.seed, counter, k.tag);
    k.step_dev = nullptr;
  }
  return k;
}
#endif

GPT_HD bool drop_keep(const DropKey& k, uint64_t elem) {
  return (uint32_t)(splitmix64(k.key ^ elem) >> 32) >= k.thresh;
}

// multiplier applied to an element: 0 or 1/(1-p); 1 when dropout is off
GPT_HD float drop_mul(const DropKey& k, uint64_t elem) {
  if (!k.active) return 1.0f;
  return drop_keep(k, elem) ? k.scale : 0.0f;
}

// ----------------------------------------------------------------------------
// type helpers
// ----------------------------------------------------------------------------
template <typename T> GPT_HD float to_f(T v);
template <> GPT_HD float to_f<float>(float v) { return v; }
template <> GPT_HD float to_f<bf16>(bf16 v) { return __bfloat162float(v); }
template <typename T> GPT_HD T from_f(float v);
template <> GPT_HD float from_f<float>(float v) { return v; }
template <> GPT_HD bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// Programmatic dependent launch: a kernel lets the next kernel of the stream
// begin launching once all of its own blocks have started (the next kernel's
// blocks then fill SMs as this kernel's last wave drains); a kernel launched
// with the programmatic-serialization attribute waits in pdl_wait() until its
// predecessor has completed and its writes are visible, and before that reads
// only memory that no kernel of the stream writes while it may run (the
// decoding GEMM prefetches weights) and writes none.  Both are no-ops without
// such a launch.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// flags (device word in the workspace)
enum : uint32_t { FLAG_TOKEN = 1u, FLAG_LOSS = 2u, FLAG_NORM = 4u, FLAG_TIMEOUT = 8u };

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// erf by Abramowitz & Stegun (1964), formula 7.1.26, |error| <= 1.5e-7:
// for z >= 0, erf(z) = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) e^{-z^2},
// t = 1 / (1 + p z); odd extension for z < 0.  Also returns e^{-z^2}.
__device__ __forceinline__ float erf_as(float z, float& e) {
  const float az = fabsf(z);
  const float t = __fdividef(1.0f, fmaf(0.3275911f, az, 1.0f));
  const float poly =
      t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, 1.061405429f, -1.453152027f), 1.421413741f), -0.284496736f), 0.254829592f);
  e = __expf(-az * az);
  return copysignf(fmaf(-poly, e, 1.0f), z);
}
// GELU, exact erf form x * Phi(x) with Phi(x) = (1 + erf(x / sqrt 2)) / 2, and
// its derivative Phi(x) + x phi(x), phi(x) = e^{-x^2/2} / sqrt(2 pi).
__device__ __forceinline__ float gelu_f(float x) {
  float e;
  return 0.5f * x * (1.0f + erf_as(x * 0.70710678118654752f, e));
}
__device__ __forceinline__ float gelu_grad_f(float x) {
  float e;  // e^{-(x / sqrt 2)^2} = e^{-x^2 / 2}
  const float cdf = 0.5f * (1.0f + erf_as(x * 0.70710678118654752f, e));
  return fmaf(x * 0.3989422804014327f, e, cdf);
}

// Two fp32 lanes in one 64-bit register: the sm_100 f32x2 FMA-pipe forms
// (each lane rounds exactly like the scalar instruction).
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 f2split(uint64_t r) {
  float2 v;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
  return v;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2c(float c) { return f2(c, c); }

// The SFU's approximate reciprocal and base-2 exponential (PTX rcp.approx and
// ex2.approx, denormals flushed; relative error about 2^-22).
__device__ __forceinline__ float sfu_rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sfu_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// gelu_f and gelu_grad_f of a pair (a, b) at once: the activations replace
// (a, b), the derivatives go to (ga, gb).  The same erf (Abramowitz & Stegun
// 7.1.26 at z = |x| / sqrt 2) with its constants folded so that most steps are
// f32x2 operations on the pair:
//   t = 1 / (1 + (p / sqrt 2) |x|),   e = e^{-x^2/2} = 2^{-(log2 e / 2) x^2},
//   q = -(a1 t + a2 t^2 + ... + a5 t^5) / 2, so that q e = (erf(|z|) - 1) / 2,
//   Phi(x) = 1/2 + sign(x) (1/2 + q e),
//   GELU(x) = x Phi(x),   GELU'(x) = Phi(x) + x e / sqrt(2 pi).
__device__ __forceinline__ void gelu_and_grad2(float& a, float& b, float& ga, float& gb) {
  constexpr float kP = 0.3275911f * 0.70710678118654752f;  // p / sqrt 2
  constexpr float kE = -0.72134752044448170f;              // -(log2 e) / 2
  const uint64_t x = f2(a, b);
  const float2 den = f2split(f2fma(f2(fabsf(a), fabsf(b)), f2c(kP), f2c(1.0f)));
  const uint64_t t = f2(sfu_rcp(den.x), sfu_rcp(den.y));
  uint64_t q = f2fma(t, f2c(-0.5f * 1.061405429f), f2c(0.5f * 1.453152027f));
  q = f2fma(t, q, f2c(-0.5f * 1.421413741f));
  q = f2fma(t, q, f2c(0.5f * 0.284496736f));
  q = f2fma(t, q, f2c(-0.5f * 0.254829592f));
  q = f2mul(t, q);
  const float2 y = f2split(f2mul(f2mul(x, f2c(kE)), x));
  const uint64_t e = f2(sfu_exp2(y.x), sfu_exp2(y.y));
  const float2 u = f2split(f2fma(q, e, f2c(0.5f)));  // erf(|x| / sqrt 2) / 2
  const uint64_t cdf = f2add(f2(copysignf(u.x, a), copysignf(u.y, b)), f2c(0.5f));
  const float2 g = f2split(f2mul(x, cdf));
  const float2 d = f2split(f2fma(f2mul(x, f2c(0.3989422804014327f)), e, cdf));
  a = g.x;
  b = g.y;
  ga = d.x;
  gb = d.y;
}
}  // namespace gpt
