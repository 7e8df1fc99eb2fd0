// Causal multi-head attention on CUDA cores, flash-style (no T x T matrix in
// memory): forward with online softmax and saved log-sum-exp, backward that
// recomputes the probabilities from the log-sum-exp.  Used by the fp32 mode
// and for head sizes the tensor-core kernel does not take.
//
// Per (b, h): S = Q K^T / sqrt(hd) with key j > query i masked, P = softmax(S),
// O = drop(P) V (dropout site 1 on the probabilities).  Backward:
// D_i = sum_d dO_id O_id; dP = drop(dO V^T); dS = P * (dP - D);
// dQ = dS K / sqrt(hd); dK = dS^T Q / sqrt(hd); dV = drop(P)^T dO.
// Each query (or key) is owned by 4 adjacent threads holding hd/4 dims.
#include "kernels.cuh"

#include <math.h>

namespace gpt {

namespace {

constexpr int QB = 64;  // queries (or keys) per block

__device__ __forceinline__ float grp4_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

template <typename T, int HD>
__device__ __forceinline__ void load_tile(float (*dst)[HD + 1], const T* qkv, int which, int b, int h, int H, int T_,
                                          int t0, int ld) {
  for (int l = threadIdx.x; l < QB * HD; l += blockDim.x) {
    int r = l / HD, c = l % HD;
    int t = t0 + r;
    float v = 0.f;
    if (t < T_) v = to_f<T>(qkv[((long)b * T_ + t) * ld + which * H * HD + h * HD + c]);
    dst[r][c] = v;
  }
}

template <typename T, int HD>
__global__ void __launch_bounds__(256) k_attn_fwd(AttnDesc a) {
  pdl_trigger();
  const DropKey dropk = drop_live(a.drop);
  constexpr int DPT = HD / 4;
  extern __shared__ float smem_f[];
  float(*Ks)[HD + 1] = reinterpret_cast<float(*)[HD + 1]>(smem_f);
  float(*Vs)[HD + 1] = reinterpret_cast<float(*)[HD + 1]>(smem_f + QB * (HD + 1));
  const T* qkv = reinterpret_cast<const T*>(a.qkv);
  int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  int qi = blockIdx.x * QB + (threadIdx.x >> 2);
  int part = threadIdx.x & 3;
  int ld = 3 * a.H * HD;
  float scale = 1.0f / sqrtf((float)HD);
  bool valid = qi < a.T;
  float q[DPT], o[DPT];
#pragma unroll
  for (int k = 0; k < DPT; k++) {
    q[k] = valid ? to_f<T>(qkv[((long)b * a.T + qi) * ld + h * HD + part * DPT + k]) * scale : 0.f;
    o[k] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  int last_q = min(a.T - 1, blockIdx.x * QB + QB - 1);
  for (int k0 = 0; k0 <= last_q; k0 += QB) {
    __syncthreads();
    load_tile<T, HD>(Ks, qkv, 1, b, h, a.H, a.T, k0, ld);
    load_tile<T, HD>(Vs, qkv, 2, b, h, a.H, a.T, k0, ld);
    __syncthreads();
    float s[QB];
    float tmax = -INFINITY;
#pragma unroll 4
    for (int j = 0; j < QB; j++) {
      float p = 0.f;
#pragma unroll
      for (int k = 0; k < DPT; k++) p = fmaf(q[k], Ks[j][part * DPT + k], p);
      p = grp4_sum(p);
      int kj = k0 + j;
      s[j] = (kj <= qi && kj < a.T) ? p : -INFINITY;
      tmax = fmaxf(tmax, s[j]);
    }
    float mn = fmaxf(m, tmax);
    if (mn == -INFINITY) continue;
    float alpha = expf(m - mn);
    l *= alpha;
#pragma unroll
    for (int k = 0; k < DPT; k++) o[k] *= alpha;
    uint64_t ebase = (((uint64_t)bh) * a.T + qi) * a.T;
#pragma unroll 4
    for (int j = 0; j < QB; j++) {
      float p = s[j] == -INFINITY ? 0.f : expf(s[j] - mn);
      l += p;
      float pd = p * drop_mul(dropk, ebase + k0 + j);
#pragma unroll
      for (int k = 0; k < DPT; k++) o[k] = fmaf(pd, Vs[j][part * DPT + k], o[k]);
    }
    m = mn;
  }
  if (!valid) return;
  float inv = 1.0f / l;
  T* out = reinterpret_cast<T*>(a.o) + ((long)b * a.T + qi) * (a.H * HD) + h * HD + part * DPT;
#pragma unroll
  for (int k = 0; k < DPT; k++) out[k] = from_f<T>(o[k] * inv);
  if (part == 0) a.lse[(long)bh * a.T + qi] = m + logf(l);
}

// D[b,h,i] = sum_d dO[b,i,h,d] * O[b,i,h,d]
template <typename T, int HD>
__global__ void k_attn_dsum(AttnDesc a) {
  pdl_trigger();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  long n = (long)a.B * a.H * a.T;
  if (i >= n) return;
  int t = (int)(i % a.T);
  int bh = (int)(i / a.T);
  int b = bh / a.H, h = bh % a.H;
  long off = ((long)b * a.T + t) * (a.H * HD) + h * HD;
  const T* o = reinterpret_cast<const T*>(a.o) + off;
  const T* d = reinterpret_cast<const T*>(a.dout) + off;
  float s = 0.f;
  for (int k = 0; k < HD; k++) s += to_f<T>(o[k]) * to_f<T>(d[k]);
  a.dsum[i] = s;
}

template <typename T, int HD>
__device__ __forceinline__ void load_do_tile(float (*dst)[HD + 1], const T* dout, int b, int h, int H, int T_, int t0) {
  for (int l = threadIdx.x; l < QB * HD; l += blockDim.x) {
    int r = l / HD, c = l % HD;
    int t = t0 + r;
    dst[r][c] = t < T_ ? to_f<T>(dout[((long)b * T_ + t) * (H * HD) + h * HD + c]) : 0.f;
  }
}

// dK, dV: each 4-thread group owns one key j and walks the queries i >= j.
template <typename T, int HD>
__global__ void __launch_bounds__(256) k_attn_bwd_kv(AttnDesc a) {
  pdl_trigger();
  const DropKey dropk = drop_live(a.drop);
  constexpr int DPT = HD / 4;
  extern __shared__ float smem_f[];
  float(*Qs)[HD + 1] = reinterpret_cast<float(*)[HD + 1]>(smem_f);
  float(*Ds)[HD + 1] = reinterpret_cast<float(*)[HD + 1]>(smem_f + QB * (HD + 1));
  float* Ls = smem_f + 2 * QB * (HD + 1);
  float* Dsum = Ls + QB;
  const T* qkv = reinterpret_cast<const T*>(a.qkv);
  const T* dout = reinterpret_cast<const T*>(a.dout);
  int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  int kj = blockIdx.x * QB + (threadIdx.x >> 2);
  int part = threadIdx.x & 3;
  int ld = 3 * a.H * HD;
  float scale = 1.0f / sqrtf((float)HD);
  bool valid = kj < a.T;
  float kv[DPT], vv[DPT], dk[DPT], dv[DPT];
#pragma unroll
  for (int k = 0; k < DPT; k++) {
    long base = ((long)b * a.T + kj) * ld + h * HD + part * DPT + k;
    kv[k] = valid ? to_f<T>(qkv[base + a.H * HD]) : 0.f;
    vv[k] = valid ? to_f<T>(qkv[base + 2 * a.H * HD]) : 0.f;
    dk[k] = 0.f;
    dv[k] = 0.f;
  }
  for (int q0 = blockIdx.x * QB; q0 < a.T; q0 += QB) {
    __syncthreads();
    load_tile<T, HD>(Qs, qkv, 0, b, h, a.H, a.T, q0, ld);
    load_do_tile<T, HD>(Ds, dout, b, h, a.H, a.T, q0);
    for (int l = threadIdx.x; l < QB; l += blockDim.x) {
      int t = q0 + l;
      Ls[l] = t < a.T ? a.lse[(long)bh * a.T + t] : 0.f;
      Dsum[l] = t < a.T ? a.dsum[(long)bh * a.T + t] : 0.f;
    }
    __syncthreads();
    for (int i = 0; i < QB; i++) {
      int qi = q0 + i;
      float s = 0.f, dpt = 0.f;
#pragma unroll
      for (int k = 0; k < DPT; k++) {
        s = fmaf(Qs[i][part * DPT + k], kv[k], s);
        dpt = fmaf(Ds[i][part * DPT + k], vv[k], dpt);
      }
      s = grp4_sum(s);
      dpt = grp4_sum(dpt);
      if (!(valid && qi < a.T && kj <= qi)) continue;
      float p = expf(s * scale - Ls[i]);
      float mk = drop_mul(dropk, (((uint64_t)bh) * a.T + qi) * a.T + kj);
      float ds = p * (dpt * mk - Dsum[i]);
#pragma unroll
      for (int k = 0; k < DPT; k++) {
        dv[k] = fmaf(p * mk, Ds[i][part * DPT + k], dv[k]);
        dk[k] = fmaf(ds * scale, Qs[i][part * DPT + k], dk[k]);
      }
    }
  }
  if (!valid) return;
  T* out = reinterpret_cast<T*>(a.dqkv) + ((long)b * a.T + kj) * ld + h * HD + part * DPT;
#pragma unroll
  for (int k = 0; k < DPT; k++) {
    out[a.H * HD + k] = from_f<T>(dk[k]);
    out[2 * a.H * HD + k] = from_f<T>(dv[k]);
  }
}

// dQ: each 4-thread group owns one query i and walks the keys j <= i.
template <typename T, int HD>
__global__ void __launch_bounds__(256) k_attn_bwd_q(AttnDesc a) {
  pdl_trigger();
  const DropKey dropk = drop_live(a.drop);
  constexpr int DPT = HD / 4;
  extern __shared__ float smem_f[];
  float(*Ks)[HD + 1] = reinterpret_cast<float(*)[HD + 1]>(smem_f);
  float(*Vs)[HD + 1] = reinterpret_cast<float(*)[HD + 1]>(smem_f + QB * (HD + 1));
  const T* qkv = reinterpret_cast<const T*>(a.qkv);
  const T* dout = reinterpret_cast<const T*>(a.dout);
  int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  int qi = blockIdx.x * QB + (threadIdx.x >> 2);
  int part = threadIdx.x & 3;
  int ld = 3 * a.H * HD;
  float scale = 1.0f / sqrtf((float)HD);
  bool valid = qi < a.T;
  float q[DPT], dov[DPT], dq[DPT];
#pragma unroll
  for (int k = 0; k < DPT; k++) {
    q[k] = valid ? to_f<T>(qkv[((long)b * a.T + qi) * ld + h * HD + part * DPT + k]) : 0.f;
    dov[k] = valid ? to_f<T>(dout[((long)b * a.T + qi) * (a.H * HD) + h * HD + part * DPT + k]) : 0.f;
    dq[k] = 0.f;
  }
  float lse = valid ? a.lse[(long)bh * a.T + qi] : 0.f;
  float Di = valid ? a.dsum[(long)bh * a.T + qi] : 0.f;
  int last_q = min(a.T - 1, blockIdx.x * QB + QB - 1);
  for (int k0 = 0; k0 <= last_q; k0 += QB) {
    __syncthreads();
    load_tile<T, HD>(Ks, qkv, 1, b, h, a.H, a.T, k0, ld);
    load_tile<T, HD>(Vs, qkv, 2, b, h, a.H, a.T, k0, ld);
    __syncthreads();
    for (int j = 0; j < QB; j++) {
      int kj = k0 + j;
      float s = 0.f, dpt = 0.f;
#pragma unroll
      for (int k = 0; k < DPT; k++) {
        s = fmaf(q[k], Ks[j][part * DPT + k], s);
        dpt = fmaf(dov[k], Vs[j][part * DPT + k], dpt);
      }
      s = grp4_sum(s);
      dpt = grp4_sum(dpt);
      if (!(valid && kj <= qi)) continue;
      float p = expf(s * scale - lse);
      float mk = drop_mul(dropk, (((uint64_t)bh) * a.T + qi) * a.T + kj);
      float ds = p * (dpt * mk - Di);
#pragma unroll
      for (int k = 0; k < DPT; k++) dq[k] = fmaf(ds * scale, Ks[j][part * DPT + k], dq[k]);
    }
  }
  if (!valid) return;
  T* out = reinterpret_cast<T*>(a.dqkv) + ((long)b * a.T + qi) * ld + h * HD + part * DPT;
#pragma unroll
  for (int k = 0; k < DPT; k++) out[k] = from_f<T>(dq[k]);
}

template <typename T, int HD>
void run_fwd(Ctx& c, const AttnDesc& a) {
  size_t smem = 2 * QB * (HD + 1) * sizeof(float);
  // per-device function attribute: set before every launch
  cudaFuncSetAttribute(k_attn_fwd<T, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid((a.T + QB - 1) / QB, a.B * a.H);
  LaunchScope s(c, "attn_fwd_simt");
  k_attn_fwd<T, HD><<<grid, 256, smem, c.stream>>>(a);
}

template <typename T, int HD>
void run_bwd(Ctx& c, const AttnDesc& a) {
  {
    long n = (long)a.B * a.H * a.T;
    LaunchScope s(c, "attn_bwd_dsum");
    k_attn_dsum<T, HD><<<(unsigned)((n + 255) / 256), 256, 0, c.stream>>>(a);
  }
  dim3 grid((a.T + QB - 1) / QB, a.B * a.H);
  size_t smem_kv = (2 * QB * (HD + 1) + 2 * QB) * sizeof(float);
  size_t smem_q = 2 * QB * (HD + 1) * sizeof(float);
  // per-device function attribute: set before every launch
  cudaFuncSetAttribute(k_attn_bwd_kv<T, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kv);
  cudaFuncSetAttribute(k_attn_bwd_q<T, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_q);
  {
    LaunchScope s(c, "attn_bwd_kv_simt");
    k_attn_bwd_kv<T, HD><<<grid, 256, smem_kv, c.stream>>>(a);
  }
  {
    LaunchScope s(c, "attn_bwd_q_simt");
    k_attn_bwd_q<T, HD><<<grid, 256, smem_q, c.stream>>>(a);
  }
}

}  // namespace

#define ATTN_DISPATCH(FN)            \
  switch (a.hd) {                    \
    case 4: FN<T, 4>(c, a); break;   \
    case 8: FN<T, 8>(c, a); break;   \
    case 16: FN<T, 16>(c, a); break; \
    case 32: FN<T, 32>(c, a); break; \
    case 64: FN<T, 64>(c, a); break; \
    case 128: FN<T, 128>(c, a); break; \
    default: break;                  \
  }

template <typename T> void attn_fwd_simt(Ctx& c, const AttnDesc& a) { ATTN_DISPATCH(run_fwd) }
template <typename T> void attn_bwd_simt(Ctx& c, const AttnDesc& a) { ATTN_DISPATCH(run_bwd) }
template void attn_fwd_simt<float>(Ctx&, const AttnDesc&);
template void attn_fwd_simt<bf16>(Ctx&, const AttnDesc&);
template void attn_bwd_simt<float>(Ctx&, const AttnDesc&);
template void attn_bwd_simt<bf16>(Ctx&, const AttnDesc&);

}  // namespace gpt
