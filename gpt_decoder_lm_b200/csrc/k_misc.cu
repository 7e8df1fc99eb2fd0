// Memory-bound kernels of the training step: batch gather, embedding,
// LayerNorm/RMSNorm, cross-entropy, column sums, embedding backward,
// gradient norm and the fused clip + AdamW update.
#include "kernels.cuh"
#include "sm100.cuh"

#include <math.h>

namespace gpt {

// ============================================================================
// get_batch: random windows of the token stream (run log section 1.3; the
// target is the window shifted by one).  One thread per (b, t).
// ============================================================================
__global__ void k_gather(const void* __restrict__ stream, int tok_u16, uint64_t len, uint64_t seed, int step,
                         const int* step_dev, int micro, int B, int T, int V, int32_t* __restrict__ idx,
                         int32_t* __restrict__ tgt, uint32_t* flags) {
  pdl_trigger();
  pdl_wait();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)B * T) return;
  if (step_dev) step = *step_dev;  // step index held in device memory (replayed graphs)
  int b = (int)(i / T), t = (int)(i % T);
  uint64_t key = ((uint64_t)(uint32_t)step << 40) ^ ((uint64_t)(uint32_t)micro << 20) ^ (uint64_t)b;
  uint64_t ix = splitmix64(seed ^ splitmix64(key)) % (len - (uint64_t)T);
  int x, y;
  if (tok_u16) {
    const uint16_t* s = (const uint16_t*)stream;
    x = s[ix + t];
    y = s[ix + t + 1];
  } else {
    const int32_t* s = (const int32_t*)stream;
    x = s[ix + t];
    y = s[ix + t + 1];
  }
  if (x < 0 || x >= V || y < 0 || y >= V) {
    atomicOr(flags, FLAG_TOKEN);
    x = (x < 0 || x >= V) ? 0 : x;
    y = (y < 0 || y >= V) ? 0 : y;
  }
  idx[i] = x;
  tgt[i] = y;
}

void gather_batch(Ctx& c, const void* stream, int tok_u16, uint64_t len, uint64_t seed, int step, int micro, int B,
                  int T, int V, int32_t* idx, int32_t* tgt, const int* step_dev) {
  long n = (long)B * T;
  LaunchScope s(c, "gather_batch");
  k_gather<<<(unsigned)((n + 255) / 256), 256, 0, c.stream>>>(stream, tok_u16, len, seed, step, step_dev, micro, B, T,
                                                              V, idx, tgt, c.flags);
}

// writes the per-step scalars read by replayed graphs: step, lr, 1 - b1^t, 1 - b2^t
__global__ void k_set_step(int* step_dev, float* hyper, int step, float lr, float bc1, float bc2) {
  pdl_trigger();
  pdl_wait();
  *step_dev = step;
  hyper[0] = lr;
  hyper[1] = bc1;
  hyper[2] = bc2;
}

void set_step_params(Ctx& c, int* step_dev, float* hyper, int step, float lr, float bc1, float bc2) {
  LaunchScope s(c, "set_step");
  k_set_step<<<1, 1, 0, c.stream>>>(step_dev, hyper, step, lr, bc1, bc2);
}

__global__ void k_check_tokens(const int32_t* __restrict__ idx, const int32_t* __restrict__ tgt, long n, int V,
                               int32_t* __restrict__ io, int32_t* __restrict__ to, uint32_t* flags) {
  pdl_trigger();
  pdl_wait();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int x = idx[i], y = tgt[i];
  if (x < 0 || x >= V || y < 0 || y >= V) {
    atomicOr(flags, FLAG_TOKEN);
    x = (x < 0 || x >= V) ? 0 : x;
    y = (y < 0 || y >= V) ? 0 : y;
  }
  io[i] = x;
  to[i] = y;
}

void check_tokens(Ctx& c, const int32_t* idx, const int32_t* tgt, long n, int V, int32_t* io, int32_t* to) {
  LaunchScope s(c, "check_tokens");
  k_check_tokens<<<(unsigned)((n + 255) / 256), 256, 0, c.stream>>>(idx, tgt, n, V, io, to, c.flags);
}

// ============================================================================
// embedding: res = drop0(wte[idx] + wpe[t]) in fp32 (microGPT "模型核心":
// token embedding plus learned position embedding).
// ============================================================================
__global__ void k_embed_fwd(const int32_t* __restrict__ idx, const float* __restrict__ wte,
                            const float* __restrict__ wpe, float* __restrict__ res, int T, int d, long n4,
                            DropKey drop) {
  pdl_trigger();
  pdl_wait();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  int d4 = d >> 2;
  long m = i / d4;
  int c4 = (int)(i % d4);
  int t = (int)(m % T);
  int tok = idx[m];
  float4 a = reinterpret_cast<const float4*>(wte + (long)tok * d)[c4];
  float4 p = reinterpret_cast<const float4*>(wpe + (long)t * d)[c4];
  float4 r = make_float4(a.x + p.x, a.y + p.y, a.z + p.z, a.w + p.w);
  if (drop.active) {
    drop = drop_live(drop);
    uint64_t e = (uint64_t)m * d + c4 * 4;
    r.x *= drop_mul(drop, e);
    r.y *= drop_mul(drop, e + 1);
    r.z *= drop_mul(drop, e + 2);
    r.w *= drop_mul(drop, e + 3);
  }
  reinterpret_cast<float4*>(res)[i] = r;
}

template <typename T>
void embed_fwd(Ctx& c, const int32_t* idx, const float* wte, const float* wpe, float* res, int B, int Tn, int d,
               DropKey drop) {
  long n4 = (long)B * Tn * d / 4;
  LaunchScope s(c, "embed_fwd");
  k_embed_fwd<<<(unsigned)((n4 + 255) / 256), 256, 0, c.stream>>>(idx, wte, wpe, res, Tn, d, n4, drop);
}
template void embed_fwd<float>(Ctx&, const int32_t*, const float*, const float*, float*, int, int, int, DropKey);
template void embed_fwd<bf16>(Ctx&, const int32_t*, const float*, const float*, float*, int, int, int, DropKey);

// ============================================================================
// norm forward: one warp per row, the row held in registers (VPL float4 per
// lane).  LayerNorm: biased variance, y = (x - mean) * rstd * w + b.
// RMSNorm (micro variant): y = x * rstd with rstd = 1/sqrt(mean(x^2) + eps).
// ============================================================================
template <typename T> __device__ __forceinline__ void store4(T* p, float4 v);
template <> __device__ __forceinline__ void store4<float>(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
template <> __device__ __forceinline__ void store4<bf16>(bf16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// One warp per row at a time, rows strided over a single resident wave of
// warps; the next row's loads are issued before the current row's
// reductions, so every warp keeps a row of loads in flight while it computes.
template <typename T, int VPL>
__global__ void __launch_bounds__(256) k_norm_fwd(const float* __restrict__ x, const float* __restrict__ w,
                                                  const float* __restrict__ b, T* __restrict__ y,
                                                  float* __restrict__ mean_out, float* __restrict__ rstd_out,
                                                  long rows, int d, int rms, float eps) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long nwarps = (long)gridDim.x * (blockDim.x >> 5);
  long row = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int d4 = d >> 2;
  float4 cur[VPL], nxt[VPL];
  auto load = [&](long r, float4 (&v)[VPL]) {
    const float4* xr = reinterpret_cast<const float4*>(x + r * d);
#pragma unroll
    for (int k = 0; k < VPL; k++) {
      const int c = lane + 32 * k;
      v[k] = (r < rows && c < d4) ? xr[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  if (row >= rows) return;
  load(row, cur);
  for (; row < rows; row += nwarps) {
    load(row + nwarps, nxt);  // in flight while this row is reduced and written
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; k++)
      s += rms ? (cur[k].x * cur[k].x + cur[k].y * cur[k].y + cur[k].z * cur[k].z + cur[k].w * cur[k].w)
               : (cur[k].x + cur[k].y + cur[k].z + cur[k].w);
    s = warp_sum(s);
    float mean = 0.f, rstd;
    if (rms) {
      rstd = 1.0f / sqrtf(s / d + eps);
    } else {
      mean = s / d;
      float q = 0.f;
#pragma unroll
      for (int k = 0; k < VPL; k++) {
        if (lane + 32 * k < d4) {
          const float a = cur[k].x - mean, bb = cur[k].y - mean, cc = cur[k].z - mean, dd = cur[k].w - mean;
          q += a * a + bb * bb + cc * cc + dd * dd;
        }
      }
      q = warp_sum(q);
      rstd = 1.0f / sqrtf(q / d + eps);
    }
    T* yr = y + row * d;
#pragma unroll
    for (int k = 0; k < VPL; k++) {
      const int c = lane + 32 * k;
      if (c < d4) {
        float4 o;
        o.x = (cur[k].x - mean) * rstd;
        o.y = (cur[k].y - mean) * rstd;
        o.z = (cur[k].z - mean) * rstd;
        o.w = (cur[k].w - mean) * rstd;
        if (!rms) {
          const float4 ww = reinterpret_cast<const float4*>(w)[c];
          const float4 bb = reinterpret_cast<const float4*>(b)[c];
          o.x = o.x * ww.x + bb.x;
          o.y = o.y * ww.y + bb.y;
          o.z = o.z * ww.z + bb.z;
          o.w = o.w * ww.w + bb.w;
        }
        store4<T>(yr + 4 * c, o);
      }
    }
    if (lane == 0) {
      mean_out[row] = mean;
      rstd_out[row] = rstd;
    }
#pragma unroll
    for (int k = 0; k < VPL; k++) cur[k] = nxt[k];
  }
}

// at most a single resident wave (the SM count times the blocks of this
// instantiation that fit on an SM), trimmed so that every warp walks the same
// number of rows: with R rounds of rows per warp, ceil(rows / R) warps
template <typename T, int VPL>
void launch_norm_fwd(Ctx& c, const float* x, const float* w, const float* b, T* y, float* mean, float* rstd,
                     long rows, int d, bool rms, float eps) {
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_norm_fwd<T, VPL>, 256, 0) != cudaSuccess || occ < 1) {
    cudaGetLastError();
    occ = 1;
  }
  const long resident = (long)c.num_sms * occ * 8;  // warps
  const long rounds = (rows + resident - 1) / resident;
  const long warps = (rows + rounds - 1) / rounds;
  const long grid = (warps + 7) / 8;
  k_norm_fwd<T, VPL><<<(unsigned)grid, 256, 0, c.stream>>>(x, w, b, y, mean, rstd, rows, d, rms, eps);
}

template <typename T>
void norm_fwd(Ctx& c, const float* x, const float* w, const float* b, T* y, float* mean, float* rstd, long rows,
              int d, bool rms, float eps) {
  int d4 = d / 4;
  int vpl = (d4 + 31) / 32;
  LaunchScope s(c, "norm_fwd");
#define NF(V) launch_norm_fwd<T, V>(c, x, w, b, y, mean, rstd, rows, d, rms, eps)
  if (vpl <= 1) NF(1);
  else if (vpl <= 2) NF(2);
  else if (vpl <= 4) NF(4);
  else if (vpl <= 6) NF(6);
  else if (vpl <= 8) NF(8);
  else NF(16);
#undef NF
}
template void norm_fwd<float>(Ctx&, const float*, const float*, const float*, float*, float*, float*, long, int,
                              bool, float);
template void norm_fwd<bf16>(Ctx&, const float*, const float*, const float*, bf16*, float*, float*, long, int, bool,
                             float);

// ============================================================================
// norm backward.  A block of ceil(d/4) threads (rounded to warps) walks a
// contiguous range of rows; thread j owns columns 4j..4j+3, so the column
// partial sums stay in registers and the result is deterministic.
//   LayerNorm: g = dy * w; dx = rstd * (g - mean(g) - xhat * mean(g * xhat))
//   RMSNorm:   g = dy;     dx = rstd * (g - xhat * mean(g * xhat))
// ============================================================================
template <typename T>
__global__ void k_norm_bwd(NormBwd p) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float red[];  // [2 buffers][warps][4]
  int tid = threadIdx.x;
  int d4 = p.d >> 2;
  int nw = blockDim.x >> 5;
  bool own = tid < d4;
  long per = (p.rows + gridDim.x - 1) / gridDim.x;
  long r0 = blockIdx.x * per, r1 = min(p.rows, r0 + per);
  float4 gw = make_float4(1.f, 1.f, 1.f, 1.f);
  if (own && !p.rms) gw = reinterpret_cast<const float4*>(p.w)[tid];
  const DropKey dk = drop_live(p.drop);
  float pg[4] = {0, 0, 0, 0}, pb[4] = {0, 0, 0, 0}, pn[4] = {0, 0, 0, 0};
  int buf = 0;
  const float wv[4] = {gw.x, gw.y, gw.z, gw.w};
  // Two rows per round (one barrier for both rows' reductions); the inputs of
  // the next round (dy, x, the residual gradient they add to, mean, rstd) are
  // loaded before this round's work, so loads stay in flight throughout.
  struct Rows {
    float4 dy[2], x[2], old[2];
    float mean[2], rstd[2];
  };
  auto load = [&](long r, Rows& q) {
#pragma unroll
    for (int u = 0; u < 2; u++) {
      const long rr = r + u;
      const bool live = rr < r1;
      q.mean[u] = (p.rms || !live) ? 0.f : p.mean[rr];
      q.rstd[u] = live ? p.rstd[rr] : 0.f;
      q.dy[u] = q.x[u] = q.old[u] = make_float4(0, 0, 0, 0);
      if (own && live) {
        q.dy[u] = reinterpret_cast<const float4*>(p.dy + rr * p.d)[tid];
        q.x[u] = reinterpret_cast<const float4*>(p.x + rr * p.d)[tid];
        if (p.accumulate) q.old[u] = reinterpret_cast<const float4*>(p.dres + rr * p.d)[tid];
      }
    }
  };
  Rows cur;
  if (r0 < r1) load(r0, cur);
  for (long r = r0; r < r1; r += 2) {
    Rows nxt;
    if (r + 2 < r1) load(r + 2, nxt);
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 2; u++) {
      const float dya[4] = {cur.dy[u].x, cur.dy[u].y, cur.dy[u].z, cur.dy[u].w};
      const float xa[4] = {cur.x[u].x, cur.x[u].y, cur.x[u].z, cur.x[u].w};
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const float xh = (xa[k] - cur.mean[u]) * cur.rstd[u];
        const float g = dya[k] * wv[k];
        s[2 * u] += g;
        s[2 * u + 1] += g * xh;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; k++) s[k] = warp_sum(s[k]);
    if ((tid & 31) == 0) {
#pragma unroll
      for (int k = 0; k < 4; k++) red[(buf * nw + (tid >> 5)) * 4 + k] = s[k];
    }
    __syncthreads();
    float t[4] = {0.f, 0.f, 0.f, 0.f};
    for (int w = 0; w < nw; w++) {
#pragma unroll
      for (int k = 0; k < 4; k++) t[k] += red[(buf * nw + w) * 4 + k];
    }
    buf ^= 1;
#pragma unroll
    for (int u = 0; u < 2; u++) {
      const long rr = r + u;
      if (!own || rr >= r1) continue;
      const float mg = p.rms ? 0.f : t[2 * u] / p.d;
      const float mgx = t[2 * u + 1] / p.d;
      const float dya[4] = {cur.dy[u].x, cur.dy[u].y, cur.dy[u].z, cur.dy[u].w};
      const float xa[4] = {cur.x[u].x, cur.x[u].y, cur.x[u].z, cur.x[u].w};
      const float ov[4] = {cur.old[u].x, cur.old[u].y, cur.old[u].z, cur.old[u].w};
      float nv[4];
#pragma unroll
      for (int k = 0; k < 4; k++) {
        const float xh = (xa[k] - cur.mean[u]) * cur.rstd[u];
        const float g = dya[k] * wv[k];
        nv[k] = ov[k] + cur.rstd[u] * (g - mg - xh * mgx);
        pg[k] += dya[k] * xh;
        pb[k] += dya[k];
      }
      reinterpret_cast<float4*>(p.dres + rr * p.d)[tid] = make_float4(nv[0], nv[1], nv[2], nv[3]);
      if (p.want_dyb) {
        float q[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
          q[k] = nv[k] * drop_mul(dk, (uint64_t)rr * p.d + 4 * tid + k);
          pn[k] += q[k];
        }
        store4<T>(reinterpret_cast<T*>(p.dyb) + rr * p.d + 4 * tid, make_float4(q[0], q[1], q[2], q[3]));
      }
    }
    cur = nxt;
  }
  if (own) {
    float4* out = reinterpret_cast<float4*>(p.part + (long)blockIdx.x * 3 * p.d) + tid;
    float4 s0 = make_float4(pg[0], pg[1], pg[2], pg[3]), s1 = make_float4(pb[0], pb[1], pb[2], pb[3]),
           s2 = make_float4(pn[0], pn[1], pn[2], pn[3]);
    if (p.part_accumulate) {  // earlier micro-batches' partials of the same rows range
      const float4 o0 = out[0], o1 = out[d4], o2 = out[2 * d4];
      s0 = make_float4(o0.x + s0.x, o0.y + s0.y, o0.z + s0.z, o0.w + s0.w);
      s1 = make_float4(o1.x + s1.x, o1.y + s1.y, o1.z + s1.z, o1.w + s1.w);
      s2 = make_float4(o2.x + s2.x, o2.y + s2.y, o2.z + s2.z, o2.w + s2.w);
    }
    out[0] = s0;
    out[d4] = s1;
    out[2 * d4] = s2;
  }
}

// one resident wave: the SM count times the blocks of k_norm_bwd<T> that fit
// on an SM at this row length (each block walks a contiguous row range)
int norm_bwd_blocks(Ctx& c, long rows, int d, bool bf16_out) {
  const int threads = ((d / 4 + 31) / 32) * 32;
  const size_t smem = (size_t)2 * (threads / 32) * 4 * sizeof(float);
  int occ = 0;
  cudaError_t e = bf16_out ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_norm_bwd<bf16>, threads, smem)
                           : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_norm_bwd<float>, threads, smem);
  if (e != cudaSuccess || occ < 1) {
    cudaGetLastError();
    occ = 1;
  }
  const long b = (long)c.num_sms * occ;
  return (int)(rows < b ? rows : b);
}

template <typename T>
void norm_bwd(Ctx& c, const NormBwd& p) {
  int d4 = p.d / 4;
  LaunchScope s(c, "norm_bwd");
  int threads = ((d4 + 31) / 32) * 32;
  int nw = threads / 32;
  k_norm_bwd<T><<<p.blocks, threads, 2 * nw * 4 * sizeof(float), c.stream>>>(p);
}
template void norm_bwd<float>(Ctx&, const NormBwd&);
template void norm_bwd<bf16>(Ctx&, const NormBwd&);

// dst_y[j] += sum_{k < rows} src[y * slot_off + k * stride + j] for j < n and
// each destination y = blockIdx.y (null: skipped), in a fixed order: block =
// 32 columns x 32 row groups; row group g sums rows g, g + 32, ... in
// increasing order, then the 32 group sums are added in group order.
struct Dst3 {
  float* p[3];
};
__global__ void __launch_bounds__(1024) k_rows_reduce(const float* __restrict__ src, long stride, long slot_off,
                                                      int rows, int n, Dst3 dsts) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sh[32][33];
  float* dst = dsts.p[blockIdx.y];
  if (!dst) return;  // uniform per block
  src += (long)blockIdx.y * slot_off;
  const int x = threadIdx.x, y = threadIdx.y;
  const int j = blockIdx.x * 32 + x;
  float s = 0.f;
  if (j < n) {
#pragma unroll 4
    for (int k = y; k < rows; k += 32) s += src[(long)k * stride + j];
  }
  sh[y][x] = s;
  __syncthreads();
  if (y == 0 && j < n) {
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 32; k++) t += sh[k][x];
    dst[j] += t;
  }
}

// grad_s[j] += sum_b part[b, s, j] for the three slots of the norm-backward
// partials (each nullable), one launch
void partial_reduce3(Ctx& c, const float* part, int blocks, int d, float* g0, float* g1, float* g2) {
  if (!g0 && !g1 && !g2) return;
  LaunchScope s(c, "partial_reduce");
  Dst3 g{{g0, g1, g2}};
  k_rows_reduce<<<dim3((d + 31) / 32, 3), dim3(32, 32), 0, c.stream>>>(part, 3L * d, d, blocks, d, g);
}

// ============================================================================
// column sums (bias gradients): chunk partials then a fixed-order reduce
// ============================================================================
template <typename T>
__global__ void k_colsum(const T* __restrict__ x, long rows, int N, int chunks, float* __restrict__ part,
                         int accumulate) {
  pdl_trigger();
  pdl_wait();
  int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= N) return;
  long per = (rows + chunks - 1) / chunks;
  long r0 = blockIdx.y * per, r1 = min(rows, r0 + per);
  float s = 0.f;
  for (long r = r0; r < r1; r++) s += to_f<T>(x[r * N + j]);
  float* dst = part + (long)blockIdx.y * N + j;
  *dst = accumulate ? *dst + s : s;
}

// grad[j] += sum_c part[c, j]: row group y of 8 sums chunks y, y+8, ...; the
// group sums are added in a fixed order
void colsum_reduce(Ctx& c, const float* part, int chunks, int N, float* grad) {
  LaunchScope s(c, "colsum");
  Dst3 g{{grad, nullptr, nullptr}};
  k_rows_reduce<<<dim3((N + 31) / 32, 1), dim3(32, 32), 0, c.stream>>>(part, N, 0, chunks, N, g);
}

// bf16 rows with N % 8 == 0: each thread sums 8 adjacent columns over its
// row chunk with 16-byte loads
__global__ void k_colsum_bf16x8(const bf16* __restrict__ x, long rows, int N, int chunks, float* __restrict__ part,
                                int accumulate) {
  pdl_trigger();
  pdl_wait();
  const int j8 = blockIdx.x * blockDim.x + threadIdx.x;
  if (j8 * 8 >= N) return;
  const long per = (rows + chunks - 1) / chunks;
  const long r0 = blockIdx.y * per, r1 = min(rows, r0 + per);
  float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  auto add = [&](const uint4& u) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int k = 0; k < 4; k++) {
      float2 f = __bfloat1622float2(h[k]);
      s[2 * k] += f.x;
      s[2 * k + 1] += f.y;
    }
  };
  long r = r0;
  for (; r + 4 <= r1; r += 4) {  // four rows of loads in flight, added in row order
    const uint4 u0 = reinterpret_cast<const uint4*>(x + r * N)[j8];
    const uint4 u1 = reinterpret_cast<const uint4*>(x + (r + 1) * N)[j8];
    const uint4 u2 = reinterpret_cast<const uint4*>(x + (r + 2) * N)[j8];
    const uint4 u3 = reinterpret_cast<const uint4*>(x + (r + 3) * N)[j8];
    add(u0);
    add(u1);
    add(u2);
    add(u3);
  }
  for (; r < r1; r++) add(reinterpret_cast<const uint4*>(x + r * N)[j8]);
  float4* dst = reinterpret_cast<float4*>(part + (long)blockIdx.y * N + j8 * 8);
  if (accumulate) {  // earlier micro-batches' sums of the same chunk
    const float4 o0 = dst[0], o1 = dst[1];
    s[0] += o0.x, s[1] += o0.y, s[2] += o0.z, s[3] += o0.w;
    s[4] += o1.x, s[5] += o1.y, s[6] += o1.z, s[7] += o1.w;
  }
  dst[0] = make_float4(s[0], s[1], s[2], s[3]);
  dst[1] = make_float4(s[4], s[5], s[6], s[7]);
}

int colsum_chunks(long rows) { return (int)min(512L, rows); }

template <typename T>
void colsum_partial(Ctx& c, const T* x, long rows, int N, float* part, bool accumulate) {
  const bool vec = sizeof(T) == 2 && N % 8 == 0;
  const int chunks = colsum_chunks(rows);  // few threads per row, many row chunks
  LaunchScope s(c, "colsum");
  if (vec) {
    dim3 grid((N / 8 + 127) / 128, chunks);
    k_colsum_bf16x8<<<grid, 128, 0, c.stream>>>(reinterpret_cast<const bf16*>(x), rows, N, chunks, part,
                                                accumulate ? 1 : 0);
  } else {
    dim3 grid((N + 127) / 128, chunks);
    k_colsum<T><<<grid, 128, 0, c.stream>>>(x, rows, N, chunks, part, accumulate ? 1 : 0);
  }
}
template void colsum_partial<float>(Ctx&, const float*, long, int, float*, bool);
template void colsum_partial<bf16>(Ctx&, const bf16*, long, int, float*, bool);


// ============================================================================
// cross-entropy (microGPT "核心训练循环": loss = -log softmax(z)[target],
// mean over positions).  One block per row: pass 1 keeps an online
// (max, sum exp) per thread and merges them; pass 2 writes
// (softmax - onehot) * scale over the logits in place (pad columns 0).
// ============================================================================
template <typename T>
__global__ void k_ce(T* __restrict__ logits, const int32_t* __restrict__ tgt, int V, int Vp,
                     float* __restrict__ lse_out, float* __restrict__ row_loss, int want_grad, float scale) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sm[32], ss[32];
  long row = blockIdx.x;
  T* z = logits + row * Vp;
  float m = -INFINITY, s = 0.f;
  for (int j = threadIdx.x; j < V; j += blockDim.x) {
    float v = to_f<T>(z[j]);
    if (v > m) {
      s = s * expf(m - v) + 1.f;
      m = v;
    } else {
      s += expf(v - m);
    }
  }
  // merge (m, s) pairs: warp then block
  for (int o = 16; o > 0; o >>= 1) {
    float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    float mm = fmaxf(m, m2);
    s = (m == -INFINITY ? 0.f : s * expf(m - mm)) + (m2 == -INFINITY ? 0.f : s2 * expf(m2 - mm));
    m = mm;
  }
  int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    sm[w] = m;
    ss[w] = s;
  }
  __syncthreads();
  float M = -INFINITY;
  for (int k = 0; k < nw; k++) M = fmaxf(M, sm[k]);
  float S = 0.f;
  for (int k = 0; k < nw; k++) S += (sm[k] == -INFINITY ? 0.f : ss[k] * expf(sm[k] - M));
  float lse = M + logf(S);
  int t = tgt[row];
  if (threadIdx.x == 0) {
    lse_out[row] = lse;
    row_loss[row] = lse - to_f<T>(z[t]);
  }
  __syncthreads();  // the target logit is read before pass 2 overwrites it
  if (!want_grad) return;
  for (int j = threadIdx.x; j < Vp; j += blockDim.x) {
    float g = 0.f;
    if (j < V) g = (expf(to_f<T>(z[j]) - lse) - (j == t ? 1.f : 0.f)) * scale;
    z[j] = from_f<T>(g);
  }
}

__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  float M = fmaxf(m, m2);
  if (M == -INFINITY) return;
  s = (m == -INFINITY ? 0.f : s * sfu_exp2(m - M)) + (m2 == -INFINITY ? 0.f : s2 * sfu_exp2(m2 - M));
  m = M;
}

// Streaming variant, 256 threads per row and several rows per SM.  Pass 1
// keeps an online (max, sum) of 2^(z log2 e) per thread over 16-byte vectors
// (one rescale per vector); the block merges them into the row's
// log-sum-exp.  Pass 2 re-reads the row (it is still in L2) and writes
// (softmax - onehot) * scale.
template <typename T>
__global__ void __launch_bounds__(256, 4) k_ce_stream(T* __restrict__ logits, const int32_t* __restrict__ tgt, int V,
                                                      int Vp, float* __restrict__ lse_out,
                                                      float* __restrict__ row_loss, int want_grad, float scale) {
  pdl_trigger();
  pdl_wait();
  constexpr int EPV = 16 / sizeof(T);
  constexpr float LOG2E = 1.4426950408889634f;
  __shared__ float sm[8], ss[8];
  const long row = blockIdx.x;
  T* z = logits + row * Vp;
  const int nvec = Vp / EPV;
  const int t = tgt[row];
  float zt = 0.f;
  if (threadIdx.x == 0) zt = to_f<T>(z[t]);
  float m = -INFINITY, s = 0.f;
  for (int vi = threadIdx.x; vi < nvec; vi += 256) {
    uint4 u = reinterpret_cast<const uint4*>(z)[vi];
    const T* e = reinterpret_cast<const T*>(&u);
    float x[EPV];
    float mv = -INFINITY;
#pragma unroll
    for (int k = 0; k < EPV; k++) {
      x[k] = (vi * EPV + k < V) ? to_f<T>(e[k]) * LOG2E : -INFINITY;
      mv = fmaxf(mv, x[k]);
    }
    if (mv > m) {
      s = (m == -INFINITY) ? 0.f : s * sfu_exp2(m - mv);
      m = mv;
    }
#pragma unroll
    for (int k = 0; k < EPV; k++) s += sfu_exp2(x[k] - m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse_merge(m, s, m2, s2);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    sm[w] = m;
    ss[w] = s;
  }
  __syncthreads();
  float M = sm[0], S = ss[0];
#pragma unroll
  for (int k = 1; k < 8; k++) lse_merge(M, S, sm[k], ss[k]);
  const float lse2 = M + log2f(S);  // log2-domain log-sum-exp
  const float lse = lse2 * 0.6931471805599453f;
  if (threadIdx.x == 0) {
    lse_out[row] = lse;
    row_loss[row] = lse - zt;
  }
  if (!want_grad) return;
  __syncthreads();  // the target logit is read before any gradient is written
  for (int vi = threadIdx.x; vi < nvec; vi += 256) {
    uint4 u = reinterpret_cast<const uint4*>(z)[vi];
    const T* e = reinterpret_cast<const T*>(&u);
    uint4 outv;
    T* o = reinterpret_cast<T*>(&outv);
#pragma unroll
    for (int k = 0; k < EPV; k++) {
      const int j = vi * EPV + k;
      float g = 0.f;
      if (j < V) g = (sfu_exp2(fmaf(to_f<T>(e[k]), LOG2E, -lse2)) - (j == t ? 1.f : 0.f)) * scale;
      o[k] = from_f<T>(g);
    }
    reinterpret_cast<uint4*>(z)[vi] = outv;
  }
}

// Rows staged in shared memory: two blocks per SM, each with one row buffer,
// walk their rows; a row arrives by bulk copies (TMA, cp.async.bulk) and both
// passes read the staged copy, so each logit is read from HBM once: pass 1
// (the row's log-sum-exp) and pass 2 (softmax - onehot, written in place).
// While one block waits for its next row, the other computes.  The arithmetic
// is k_ce_stream's (16-byte vectors strided over the block's threads, an
// online (max, sum) per thread, then warp and block merges in a fixed order)
// with fewer instructions per logit: bf16 widened by bit shifts, the
// vocabulary mask and the one-hot term only where they can apply, exponents
// and scaling as paired (f32x2) operations, two running sums per thread.
// Every wait is bounded; a block that gives up raises FLAG_TIMEOUT, waits for
// its own copies in flight (again bounded) and returns.
constexpr int CE_THREADS = 512;

// a 16-byte vector of logits as floats (bf16 widened exactly by bit shifts),
// and back (round to nearest)
template <typename T>
__device__ __forceinline__ void ce_unpack(const uint4& u, float (&x)[16 / sizeof(T)]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int k = 0; k < 4; k++) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; k++) x[k] = __uint_as_float(w[k]);
  }
}
template <typename T>
__device__ __forceinline__ uint4 ce_pack(const float (&g)[16 / sizeof(T)]) {
  uint32_t w[4];
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const __nv_bfloat162 v = __floats2bfloat162_rn(g[2 * k], g[2 * k + 1]);
      w[k] = *reinterpret_cast<const uint32_t*>(&v);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; k++) w[k] = __float_as_uint(g[k]);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
constexpr uint32_t CE_CHUNK = 32768;  // bytes per bulk copy

template <typename T>
__global__ void __launch_bounds__(CE_THREADS, 2) k_ce_smem(T* __restrict__ logits, const int32_t* __restrict__ tgt,
                                                          long M, int V, int Vp, float* __restrict__ lse_out,
                                                          float* __restrict__ row_loss, int want_grad, float scale,
                                                          uint32_t* flags) {
  pdl_trigger();
  constexpr int EPV = 16 / sizeof(T);
  constexpr float LOG2E = 1.4426950408889634f;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float sm[CE_THREADS / 32], ss[CE_THREADS / 32];
  __shared__ __align__(8) uint64_t full[2];
  __shared__ int abort_flag;
  const uint32_t RB = (uint32_t)Vp * sizeof(T);  // row bytes (a multiple of 16)
  const uint32_t RBA = (RB + 127) & ~127u;       // buffer stride
  const int nvec = Vp / EPV;
  int issued[2] = {0, 0}, waited[2] = {0, 0};    // copies per buffer (kept by thread 0)
  auto issue = [&](long row, int b) {            // thread 0: the bulk copies of one row into buffer b
    issued[b]++;
    const uint32_t bar = sm100::smem_u32(&full[b]);
    const uint32_t dst = sm100::smem_u32(smem + b * RBA);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(logits + row * Vp);
    sm100::fence_proxy_async_smem();  // the buffer's earlier generic reads come first
    sm100::mbar_expect_tx(bar, RB);
    for (uint32_t o = 0; o < RB; o += CE_CHUNK) sm100::bulk_load(dst + o, src + o, min(CE_CHUNK, RB - o), bar);
  };
  if (threadIdx.x == 0) {
    sm100::mbar_init(sm100::smem_u32(&full[0]), 1);
    sm100::mbar_init(sm100::smem_u32(&full[1]), 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
    if (blockIdx.x < M) issue(blockIdx.x, 0);
  }
  __syncthreads();
  int it = 0;
  for (long row = blockIdx.x; row < M; row += gridDim.x, it++) {
    const int b = 0;  // one row buffer: the other block on the SM covers this one's load
    const bool ok = sm100::mbar_wait(sm100::smem_u32(&full[b]), it & 1, &abort_flag, flags);
    if (__syncthreads_or(!ok)) break;  // every thread takes the same branch
    waited[b]++;
    const T* z = reinterpret_cast<const T*>(smem + b * RBA);
    const uint4* z4 = reinterpret_cast<const uint4*>(z);
    const int t = tgt[row];
    const int vfull = V / EPV;  // vectors below it lie inside the vocabulary
    const uint64_t l2 = f2(LOG2E, LOG2E);
    // pass 1: online (max, sum) of 2^(z log2 e), masks only in the last vectors,
    // the exponents as paired FMAs, two running sums
    float m = -INFINITY, s0 = 0.f, s1 = 0.f;
    for (int vi = threadIdx.x; vi < nvec; vi += CE_THREADS) {
      if (vi * EPV >= V) continue;
      float x[EPV];
      ce_unpack<T>(z4[vi], x);
      if (vi >= vfull) {
#pragma unroll
        for (int k = 0; k < EPV; k++)
          if (vi * EPV + k >= V) x[k] = -INFINITY;
      }
      float mv = x[0];
#pragma unroll
      for (int k = 1; k < EPV; k++) mv = fmaxf(mv, x[k]);
      mv *= LOG2E;
      if (mv > m) {
        if (m != -INFINITY) {
          const float r = sfu_exp2(m - mv);
          s0 *= r;
          s1 *= r;
        }
        m = mv;
      }
      const uint64_t nm = f2(-m, -m);
#pragma unroll
      for (int k = 0; k < EPV; k += 2) {
        const float2 y = f2split(f2fma(f2(x[k], x[k + 1]), l2, nm));
        s0 += sfu_exp2(y.x);
        s1 += sfu_exp2(y.y);
      }
    }
    float s = s0 + s1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      float s2 = __shfl_xor_sync(0xffffffffu, s, o);
      lse_merge(m, s, m2, s2);
    }
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
      sm[w] = m;
      ss[w] = s;
    }
    __syncthreads();
    float Mx = sm[0], S = ss[0];
#pragma unroll
    for (int k = 1; k < CE_THREADS / 32; k++) lse_merge(Mx, S, sm[k], ss[k]);
    const float lse2 = Mx + log2f(S);  // log2-domain log-sum-exp
    const float lse = lse2 * 0.6931471805599453f;
    if (threadIdx.x == 0) {
      lse_out[row] = lse;
      row_loss[row] = lse - to_f<T>(z[t]);
    }
    if (want_grad) {
      // pass 2: (2^(z log2 e - lse2) - [j == t]) * scale, zero past the vocabulary
      uint4* dst = reinterpret_cast<uint4*>(logits + row * Vp);
      const uint64_t nl = f2(-lse2, -lse2), sc2 = f2(scale, scale);
      const int tv = t / EPV;
      for (int vi = threadIdx.x; vi < nvec; vi += CE_THREADS) {
        float x[EPV], g[EPV];
        ce_unpack<T>(z4[vi], x);
#pragma unroll
        for (int k = 0; k < EPV; k += 2) {
          const float2 y = f2split(f2fma(f2(x[k], x[k + 1]), l2, nl));
          g[k] = sfu_exp2(y.x);
          g[k + 1] = sfu_exp2(y.y);
        }
        if (vi == tv) {
#pragma unroll
          for (int k = 0; k < EPV; k++)
            if (vi * EPV + k == t) g[k] -= 1.f;
        }
#pragma unroll
        for (int k = 0; k < EPV; k += 2) {
          const float2 q = f2split(f2mul(f2(g[k], g[k + 1]), sc2));
          g[k] = q.x;
          g[k + 1] = q.y;
        }
        if (vi >= vfull) {
#pragma unroll
          for (int k = 0; k < EPV; k++)
            if (vi * EPV + k >= V) g[k] = 0.f;
        }
        dst[vi] = ce_pack<T>(g);
      }
    }
    __syncthreads();  // the buffer and sm / ss are free again
    if (threadIdx.x == 0 && row + gridDim.x < M) issue(row + gridDim.x, 0);
  }
  if (threadIdx.x == 0) {
    // after a failed wait: no copy of this block may still be writing its
    // shared memory when it exits (bounded waits, which ignore the abort flag)
    volatile int no_abort = 0;
    for (int k = 0; k < 2; k++)
      for (; waited[k] < issued[k]; waited[k]++)
        if (!sm100::mbar_wait(sm100::smem_u32(&full[k]), waited[k] & 1, &no_abort, flags, 100000000ull)) break;
  }
}

// shared memory of k_ce_smem for rows of `row_bytes` (0: the row does not fit)
size_t ce_smem_bytes(size_t row_bytes) {
  if (row_bytes % 16) return 0;
  const size_t b = (row_bytes + 127) & ~size_t(127);
  return b <= 110 * 1024 ? b : 0;
}

template <typename T>
void ce_fwd_bwd(Ctx& c, T* logits, const int32_t* tgt, long M, int V, int Vp, float* lse, float* row_loss,
                bool want_grad, float scale) {
  LaunchScope s(c, want_grad ? "ce_fwd_bwd" : "ce_fwd");
  constexpr int EPV = 16 / sizeof(T);
  const size_t sh = ce_smem_bytes((size_t)Vp * sizeof(T));
  if (Vp % EPV == 0 && sh > 0) {
    // per-device function attribute: set before every launch
    cudaFuncSetAttribute(k_ce_smem<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh);
    const unsigned grid = (unsigned)std::min<long>(M, 2L * c.num_sms);
    k_ce_smem<T><<<grid, CE_THREADS, sh, c.stream>>>(logits, tgt, M, V, Vp, lse, row_loss, want_grad ? 1 : 0, scale,
                                                     c.flags);
  } else if (Vp % EPV == 0)
    k_ce_stream<T><<<(unsigned)M, 256, 0, c.stream>>>(logits, tgt, V, Vp, lse, row_loss, want_grad ? 1 : 0, scale);
  else
    k_ce<T><<<(unsigned)M, 512, 0, c.stream>>>(logits, tgt, V, Vp, lse, row_loss, want_grad ? 1 : 0, scale);
}
template void ce_fwd_bwd<float>(Ctx&, float*, const int32_t*, long, int, int, float*, float*, bool, float);
template void ce_fwd_bwd<bf16>(Ctx&, bf16*, const int32_t*, long, int, int, float*, float*, bool, float);

// loss_acc[0] (+)= scale * sum(row_loss); fixed-order double reduction.
__global__ void k_loss_reduce(const float* __restrict__ rl, long M, float scale, float* acc, int accumulate,
                              uint32_t* flags) {
  pdl_trigger();
  pdl_wait();
  __shared__ double sh[32];
  double s = 0.0;
  for (long i = threadIdx.x; i < M; i += blockDim.x) s += (double)rl[i];
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int k = 0; k < (int)(blockDim.x >> 5); k++) t += sh[k];
    float v = (float)(t * (double)scale);
    if (!isfinite(v)) atomicOr(flags, FLAG_LOSS);
    acc[0] = accumulate ? acc[0] + v : v;
  }
}

void loss_reduce(Ctx& c, const float* row_loss, long M, float scale, float* loss_acc, int accumulate) {
  LaunchScope s(c, "loss_reduce");
  k_loss_reduce<<<1, 1024, 0, c.stream>>>(row_loss, M, scale, loss_acc, accumulate, c.flags);
}

// ============================================================================
// embedding backward.  Routing: the keys token << 16 | position sorted by
// token, stably (positions ascending within a token): an LSD radix sort, four
// passes of 4 bits of the token, one CTA of 1024 threads per batch.  A pass
// walks the keys in their current order in rounds of 1024 (one per thread); a
// warp ranks each lane among the lanes with the same digit by four ballots,
// the per-(round, warp) digit counts are scanned in that order for every
// digit, and each key moves to its digit's base + the keys of that digit
// before it.  The keys alternate between two shared-memory arrays, or, when
// 2 M keys do not fit, between one and the stok array.
// ============================================================================
constexpr int RS_T = 1024, RS_W = RS_T / 32, RS_MAXR = 32;  // rounds of 1024 keys: M <= 32768

__global__ void __launch_bounds__(RS_T) k_embed_sort(const int32_t* __restrict__ idx, int M, int smem2,
                                                     int32_t* __restrict__ stok, int32_t* __restrict__ spos,
                                                     int32_t* __restrict__ n_unique) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint32_t key[];                 // [M] (and the second array [M] when smem2)
  __shared__ uint16_t cnt[RS_MAXR * RS_W][16];     // digit counts per (round, warp), then their prefixes
  __shared__ uint32_t base[16];
  __shared__ int ucnt[RS_W];
  // block b sorts the b-th batch of M tokens (batches stored back to back)
  idx += (long)blockIdx.x * M;
  stok += (long)blockIdx.x * M;
  spos += (long)blockIdx.x * M;
  n_unique += blockIdx.x;
  uint32_t* gkey = smem2 ? key + M : reinterpret_cast<uint32_t*>(stok);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int R = (M + RS_T - 1) / RS_T;
  const uint32_t lt = (1u << lane) - 1u;
  for (int i = tid; i < M; i += RS_T) key[i] = ((uint32_t)idx[i] << 16) | (uint32_t)i;
  // lanes of this warp whose digit equals this lane's (valid lanes only)
  auto peers = [&](bool valid, uint32_t d) {
    uint32_t m = __ballot_sync(0xffffffffu, valid);
#pragma unroll
    for (int b = 0; b < 4; b++) {
      const uint32_t bb = __ballot_sync(0xffffffffu, valid && ((d >> b) & 1u));
      m &= ((d >> b) & 1u) ? bb : ~bb;
    }
    return m;
  };
  for (int pass = 0; pass < 4; pass++) {
    const int sh = 16 + 4 * pass;
    const uint32_t* src = (pass & 1) ? gkey : key;
    uint32_t* dst = (pass & 1) ? key : gkey;
    __syncthreads();  // the previous pass's keys are in place and its counts read
    for (int i = tid; i < R * RS_W * 16; i += RS_T) (&cnt[0][0])[i] = 0;
    __syncthreads();
    for (int r = 0; r < R; r++) {
      const int e = r * RS_T + tid;
      const bool valid = e < M;
      const uint32_t d = valid ? (src[e] >> sh) & 15u : 0u;
      const uint32_t m = peers(valid, d);
      if (valid && (m & lt) == 0) cnt[r * RS_W + w][d] = (uint16_t)__popc(m);
    }
    __syncthreads();
    if (w < 16) {  // warp w: exclusive prefix of digit w's counts over the slots in order
      const int slots = R * RS_W, per = (slots + 31) / 32;
      const int s0 = min(slots, lane * per), s1 = min(slots, s0 + per);
      uint32_t loc = 0;
      for (int q = s0; q < s1; q++) loc += cnt[q][w];
      uint32_t inc = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
      }
      uint32_t run = inc - loc;
      for (int q = s0; q < s1; q++) {
        const uint32_t c = cnt[q][w];
        cnt[q][w] = (uint16_t)run;
        run += c;
      }
      if (lane == 31) base[w] = inc;  // the digit's total, for now
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t run = 0;
      for (int d = 0; d < 16; d++) {
        const uint32_t t = base[d];
        base[d] = run;
        run += t;
      }
    }
    __syncthreads();
    for (int r = 0; r < R; r++) {
      const int e = r * RS_T + tid;
      const bool valid = e < M;
      const uint32_t k = valid ? src[e] : 0u;
      const uint32_t d = (k >> sh) & 15u;
      const uint32_t m = peers(valid, d);
      if (valid) dst[base[d] + cnt[r * RS_W + w][d] + __popc(m & lt)] = k;
    }
  }
  __syncthreads();  // the sorted keys are in shared memory
  int u = 0;
  for (int i = tid; i < M; i += RS_T) {
    const uint32_t kk = key[i];
    stok[i] = (int32_t)(kk >> 16);
    spos[i] = (int32_t)(kk & 0xFFFFu);
    if (i == 0 || (key[i - 1] >> 16) != (kk >> 16)) u++;
  }
  for (int o = 16; o > 0; o >>= 1) u += __shfl_xor_sync(0xffffffffu, u, o);
  if (lane == 0) ucnt[w] = u;
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int k = 0; k < RS_W; k++) t += ucnt[k];
    *n_unique = t;
  }
}

void embed_sort(Ctx& c, const int32_t* idx, long M, int32_t* sorted_tok, int32_t* sorted_pos, int32_t* n_unique,
                int batches) {
  constexpr size_t kMaxDyn = 190 * 1024;  // with the kernel's 33 KB of static shared memory
  const int smem2 = (size_t)M * 8 <= kMaxDyn ? 1 : 0;
  const size_t smem = (size_t)M * 4 * (smem2 ? 2 : 1);
  // per-device function attribute: set before every launch
  cudaFuncSetAttribute(k_embed_sort, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDyn);
  LaunchScope s(c, "embed_sort");
  k_embed_sort<<<batches, RS_T, smem, c.stream>>>(idx, (int)M, smem2, sorted_tok, sorted_pos, n_unique);
}

// dwte[v] += sum over the sorted positions of token v (in position order) of
// drop0(dres[pos]): the segmented sums of k_embed_seg_a / k_embed_seg_b below.

// dwpe[t] += sum_b drop0(dres[b, t]) (b ascending)
__global__ void k_embed_bwd_wpe(const float* __restrict__ dres, int Bn, int Tn, int d, DropKey drop,
                                float* __restrict__ dwpe) {
  pdl_trigger();
  pdl_wait();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)Tn * d) return;
  int t = (int)(i / d), c = (int)(i % d);
  drop = drop_live(drop);
  float acc = 0.f;
  for (int b = 0; b < Bn; b++) {
    long m = (long)b * Tn + t;
    acc += dres[m * d + c] * drop_mul(drop, (uint64_t)m * d + c);
  }
  dwpe[i] += acc;
}

// Segment sums in fixed chunks of EC sorted slots.  Kernel A: one block per
// chunk, threads across columns, rows in sorted order; a segment that lies
// inside the chunk is added to dwte directly, the chunk's first segment when
// it began in an earlier chunk goes to head[chunk], its last segment when it
// continues into the next chunk goes to tail[chunk].  Kernel B: for every
// segment that starts in chunk c and continues, dwte[tok] += tail[c] + the
// heads of the following chunks it covers, in chunk order.
// Every load a thread needs is issued before the additions that use it: the
// chunk's rows, then the dwte rows of all its inner segments (distinct tokens,
// so the read-modify-writes are independent), then the sums and the stores.
constexpr int EC = 32;
enum : int8_t { SEG_NONE = 0, SEG_INNER = 1, SEG_HEAD = 2, SEG_TAIL = 3 };

// Grid: chunks x column groups of SEG_T columns, one column per thread, so a
// block does one pass over its chunk; the per-slot row offsets, destination
// rows and segment ends are prepared once per block in shared memory.
constexpr int SEG_T = 256;

template <bool DROP>
__global__ void __launch_bounds__(SEG_T, 2) k_embed_seg_a(const float* __restrict__ dres,
                                                          const int32_t* __restrict__ stok,
                                                          const int32_t* __restrict__ spos, int M, int d, DropKey drop,
                                                          float* __restrict__ dwte, float* __restrict__ head,
                                                          float* __restrict__ tail) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_tok[EC + 2];
  __shared__ long long s_src[EC], s_dst[EC];  // element offsets of the slot's dres row and dwte row
  __shared__ int8_t s_kind[EC];                // what ends at slot k: nothing, an inner segment, the head, the tail
  if (DROP) drop = drop_live(drop);
  const int c = blockIdx.x;
  const int j0 = c * EC, j1 = min(M, j0 + EC);
  const int n = j1 - j0;
  if (threadIdx.x < n) {
    s_tok[threadIdx.x + 1] = stok[j0 + threadIdx.x];
    s_src[threadIdx.x] = (long long)spos[j0 + threadIdx.x] * d;
  }
  if (threadIdx.x == 0) {
    s_tok[0] = j0 > 0 ? stok[j0 - 1] : -1;
    s_tok[n + 1] = j1 < M ? stok[j1] : -1;
  }
  __syncthreads();
  if (threadIdx.x < EC) {
    const int k = threadIdx.x;
    int8_t kind = SEG_NONE;
    if (k < n) {
      const int tok = s_tok[k + 1];
      if (k == n - 1 || s_tok[k + 2] != tok) {  // a segment ends at slot k (or at the chunk edge)
        // sorted slots: the segment reaches slot 0 iff slot 0 holds its token
        const bool began_before = s_tok[1] == tok && s_tok[0] == tok;
        const bool continues = k == n - 1 && s_tok[n + 1] == tok;
        kind = began_before ? SEG_HEAD : continues ? SEG_TAIL : SEG_INNER;
      }
      s_dst[k] = (long long)tok * d;
    }
    s_kind[k] = kind;
  }
  __syncthreads();
  const int col = blockIdx.y * SEG_T + threadIdx.x;
  if (col >= d) return;
  float vals[EC];
#pragma unroll
  for (int k = 0; k < EC; k++) vals[k] = k < n ? dres[s_src[k] + col] : 0.f;
  // segment sums in slot order, left in vals[k] at the slot where each ends
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < EC; k++) {
    float v = vals[k];
    if (DROP && k < n) v *= drop_mul(drop, (uint64_t)(s_src[k] + col));
    acc += v;
    if (s_kind[k] != SEG_NONE) {
      vals[k] = acc;
      acc = 0.f;
    }
  }
  float old[EC];
#pragma unroll
  for (int k = 0; k < EC; k++) old[k] = s_kind[k] == SEG_INNER ? dwte[s_dst[k] + col] : 0.f;
#pragma unroll
  for (int k = 0; k < EC; k++) {
    const int kind = s_kind[k];
    if (kind == SEG_INNER) dwte[s_dst[k] + col] = old[k] + vals[k];
    else if (kind == SEG_HEAD) head[(long)c * d + col] = vals[k];
    else if (kind == SEG_TAIL) tail[(long)c * d + col] = vals[k];
  }
}

// threads across groups of four columns (d a multiple of 4); the heads are
// loaded eight chunks at a time and added in chunk order
__global__ void k_embed_seg_b(const int32_t* __restrict__ stok, int M, int d, const float* __restrict__ head,
                              const float* __restrict__ tail, float* __restrict__ dwte) {
  pdl_trigger();
  pdl_wait();
  const int c = blockIdx.x;
  const int j0 = c * EC, j1 = min(M, j0 + EC);
  const int tok = stok[j1 - 1];
  if (j1 >= M || stok[j1] != tok) return;  // the chunk's last segment ends inside it
  // began earlier (its start chunk sums it): slot j0 holds the token and so does slot j0 - 1
  if (j0 > 0 && stok[j0] == tok && stok[j0 - 1] == tok) return;
  // the last chunk cend whose head belongs to the segment: the first chunk
  // after c at whose end the token changes (or the stream ends), found by all
  // threads at once rather than one chunk after another
  __shared__ int s_end;
  const int nch = (M + EC - 1) / EC;
  if (threadIdx.x == 0) s_end = nch;
  __syncthreads();
  for (int cc = c + 1 + threadIdx.x; cc < nch; cc += blockDim.x) {
    const int e = min(M, (cc + 1) * EC);
    if (e >= M || stok[e] != tok) atomicMin(&s_end, cc);
  }
  __syncthreads();
  const int cend = s_end < nch ? s_end : c;  // (the segment continues past c, so a later chunk ends it)
  const int d4 = d >> 2;
  const float4* __restrict__ h4 = reinterpret_cast<const float4*>(head);
  for (int q = threadIdx.x; q < d4; q += blockDim.x) {
    float4 s = reinterpret_cast<const float4*>(tail)[(long)c * d4 + q];
    int cc = c + 1;
    for (; cc + 8 <= cend + 1; cc += 8) {
      float4 h[8];
#pragma unroll
      for (int u = 0; u < 8; u++) h[u] = h4[(long)(cc + u) * d4 + q];
#pragma unroll
      for (int u = 0; u < 8; u++) {
        s.x += h[u].x;
        s.y += h[u].y;
        s.z += h[u].z;
        s.w += h[u].w;
      }
    }
    for (; cc <= cend; cc++) {
      const float4 h = h4[(long)cc * d4 + q];
      s.x += h.x;
      s.y += h.y;
      s.z += h.z;
      s.w += h.w;
    }
    float4* dst = reinterpret_cast<float4*>(dwte + (long)tok * d) + q;
    float4 o = *dst;
    o.x += s.x;
    o.y += s.y;
    o.z += s.z;
    o.w += s.w;
    *dst = o;
  }
}

void embed_bwd(Ctx& c, const float* dres, const int32_t* sorted_tok, const int32_t* sorted_pos, long M, int Tn,
               int Bn, int d, DropKey drop, float* dwte, float* dwpe, float* seg_scratch) {
  {
    LaunchScope s(c, "embed_bwd_wte");
    const int chunks = (int)((M + EC - 1) / EC);
    float* head = seg_scratch;
    float* tail = seg_scratch + (size_t)chunks * d;
    const dim3 ga(chunks, (d + SEG_T - 1) / SEG_T);
    if (drop.active)
      k_embed_seg_a<true><<<ga, SEG_T, 0, c.stream>>>(dres, sorted_tok, sorted_pos, (int)M, d, drop, dwte, head, tail);
    else
      k_embed_seg_a<false><<<ga, SEG_T, 0, c.stream>>>(dres, sorted_tok, sorted_pos, (int)M, d, drop, dwte, head, tail);
    k_embed_seg_b<<<chunks, 256, 0, c.stream>>>(sorted_tok, (int)M, d, head, tail, dwte);
  }
  {
    LaunchScope s(c, "embed_bwd_wpe");
    long n = (long)Tn * d;
    k_embed_bwd_wpe<<<(unsigned)((n + 255) / 256), 256, 0, c.stream>>>(dres, Bn, Tn, d, drop, dwpe);
  }
}

// ============================================================================
// global gradient norm: per-block partial sums of squares (double)
// ============================================================================
int sumsq_blocks(Ctx& c) { return c.num_sms * 4 < 592 ? c.num_sms * 4 : 592; }  // partial buffer holds 592

__global__ void k_sumsq(const float* __restrict__ g, long n4, double* __restrict__ part) {
  pdl_trigger();
  pdl_wait();
  __shared__ double sh[32];
  double s = 0.0;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long)gridDim.x * blockDim.x) {
    float4 v = reinterpret_cast<const float4*>(g)[i];
    s += (double)(v.x * v.x + v.y * v.y) + (double)(v.z * v.z + v.w * v.w);
  }
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int k = 0; k < (int)(blockDim.x >> 5); k++) t += sh[k];
    part[blockIdx.x] = t;
  }
}

void sumsq_partials(Ctx& c, const float* g, long n, double* partials, int blocks) {
  LaunchScope s(c, "grad_norm");
  k_sumsq<<<blocks, 512, 0, c.stream>>>(g, n / 4, partials);
}

// ============================================================================
// clip + AdamW (one pass over the fp32 arenas; decayed tensors first).  The
// gradient is gscale times the arena's values (1 for a whole-model step; 1 /
// world for a shard of summed replica gradients), its norm gscale times the
// square root of the sum of the partials.
//   c = min(1, clip / (norm + 1e-6)); g <- c g
//   w <- w (1 - lr wd)                      (decayed tensors only)
//   m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2
//   w <- w - lr (m / bc1) / (sqrt(v / bc2) + eps);  wb <- bf16(w);  g <- 0
// A non-finite norm skips the update (gradients are still zeroed).
// ============================================================================
__global__ void k_adamw(AdamArgs a, uint32_t* flags) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_coef;
  __shared__ int s_ok;
  if (threadIdx.x < 32) {
    double t = 0.0;
    for (int k = threadIdx.x; k < a.norm_blocks; k += 32) t += a.norm_partials[k];
    t = warp_sum_d(t);
    if (threadIdx.x == 0) {
      double norm = sqrt(t) * (double)a.gscale;
      int ok = isfinite(norm) ? 1 : 0;
      float coef = 1.f;
      if (a.clip > 0.f && ok) coef = (float)fmin(1.0, (double)a.clip / (norm + 1e-6));
      s_coef = coef;
      s_ok = ok;
      if (blockIdx.x == 0) {
        a.norm_out[0] = (float)norm;
        if (!ok) atomicOr(flags, FLAG_NORM);
      }
    }
  }
  __syncthreads();
  if (a.hyper) {  // learning rate and bias corrections of this step from device memory
    a.lr = a.hyper[0];
    a.bc1 = a.hyper[1];
    a.bc2 = a.hyper[2];
  }
  const float coef = s_coef * a.gscale;
  const int ok = s_ok;
  const float om1 = 1.f - a.beta1, om2 = 1.f - a.beta2;
  const float decay = 1.f - a.lr * a.wd;
  const long n4 = a.n / 4;
  float4* __restrict__ W4 = reinterpret_cast<float4*>(a.w);
  float4* __restrict__ G4 = reinterpret_cast<float4*>(a.g);
  float4* __restrict__ M4 = reinterpret_cast<float4*>(a.m);
  float4* __restrict__ V4 = reinterpret_cast<float4*>(a.v);
  bf16* __restrict__ WB = a.wb;
  const long stride = (long)gridDim.x * blockDim.x;
  for (long i0 = (long)blockIdx.x * blockDim.x + threadIdx.x; i0 < n4; i0 += 2 * stride) {
    // two independent float4 per iteration: more loads in flight
    float4 g4[2], w4[2], m4[2], v4[2];
    bool in[2] = {true, i0 + stride < n4};
#pragma unroll
    for (int u = 0; u < 2; u++) {
      long i = i0 + u * stride;
      if (!in[u]) continue;
      g4[u] = G4[i];
      if (ok) {
        w4[u] = W4[i];
        m4[u] = M4[i];
        v4[u] = V4[i];
      }
    }
#pragma unroll
    for (int u = 0; u < 2; u++) {
      long i = i0 + u * stride;
      if (!in[u]) continue;
      G4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (!ok) continue;
      float* w = &w4[u].x;
      float* m = &m4[u].x;
      float* v = &v4[u].x;
      const float* g = &g4[u].x;
      const bool dec = (i * 4) < a.n_decay;
#pragma unroll
      for (int k = 0; k < 4; k++) {
        float gg = g[k] * coef;
        float ww = dec ? w[k] * decay : w[k];
        m[k] = a.beta1 * m[k] + om1 * gg;
        v[k] = a.beta2 * v[k] + om2 * gg * gg;
        ww -= a.lr * (m[k] / a.bc1) / (sqrtf(v[k] / a.bc2) + a.eps);
        w[k] = ww;
      }
      W4[i] = w4[u];
      M4[i] = m4[u];
      V4[i] = v4[u];
      if (WB) store4<bf16>(WB + 4 * i, w4[u]);
    }
  }
}

void adamw(Ctx& c, const AdamArgs& a) {
  LaunchScope s(c, "adamw");
  k_adamw<<<c.num_sms * 8, 256, 0, c.stream>>>(a, c.flags);
}

__global__ void k_to_bf16(const float* __restrict__ s, bf16* __restrict__ d, long n) {
  pdl_trigger();
  pdl_wait();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) d[i] = __float2bfloat16_rn(s[i]);
}

void to_bf16(Ctx& c, const float* src, bf16* dst, long n) {
  LaunchScope s(c, "to_bf16");
  k_to_bf16<<<(unsigned)((n + 255) / 256), 256, 0, c.stream>>>(src, dst, n);
}

// row argmax, ties to the lowest index
__global__ void k_argmax(const void* __restrict__ x, int is_bf16, int cols, int ld, int32_t* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  __shared__ float bv[32];
  __shared__ int bi[32];
  long row = blockIdx.x;
  float best = -INFINITY;
  int bidx = 0x7fffffff;
  for (int j = threadIdx.x; j < cols; j += blockDim.x) {
    float v = is_bf16 ? __bfloat162float(((const bf16*)x)[row * ld + j]) : ((const float*)x)[row * ld + j];
    if (v > best || (v == best && j < bidx)) {
      best = v;
      bidx = j;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    float v2 = __shfl_xor_sync(0xffffffffu, best, o);
    int i2 = __shfl_xor_sync(0xffffffffu, bidx, o);
    if (v2 > best || (v2 == best && i2 < bidx)) {
      best = v2;
      bidx = i2;
    }
  }
  if ((threadIdx.x & 31) == 0) {
    bv[threadIdx.x >> 5] = best;
    bi[threadIdx.x >> 5] = bidx;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < (int)(blockDim.x >> 5); k++)
      if (bv[k] > best || (bv[k] == best && bi[k] < bidx)) {
        best = bv[k];
        bidx = bi[k];
      }
    out[row] = bidx == 0x7fffffff ? 0 : bidx;
  }
}

void argmax_rows(Ctx& c, const void* x, int is_bf16, long rows, int cols, int ld, int32_t* out) {
  LaunchScope s(c, "argmax");
  k_argmax<<<(unsigned)rows, 256, 0, c.stream>>>(x, is_bf16, cols, ld, out);
}

__global__ void k_dropmask(DropKey k, long n, uint8_t* out) {
  pdl_trigger();
  pdl_wait();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = drop_keep(k, (uint64_t)i) ? 1 : 0;
}

void dropout_mask(Ctx& c, DropKey k, long n, uint8_t* out) {
  LaunchScope s(c, "dropout_mask");
  k_dropmask<<<(unsigned)((n + 255) / 256), 256, 0, c.stream>>>(k, n, out);
}

}  // namespace gpt
