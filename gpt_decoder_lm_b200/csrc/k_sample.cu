// Fused softmax-sample of rows of logits: temperature, top-k, top-p
// (nucleus) and an inverse-CDF draw at a caller-given uniform, one CTA per
// row, every reduction in a fixed order (deterministic).
//
// Pipeline of the microGPT page, section "单 GPU 高效推理：采样 + KV Cache"
// (logits / temperature -> top-k -> softmax -> top-p -> draw) and nanoGPT's
// sample.py (README section "采样 / 推理"):
//   temperature <= 0       greedy: arg-max, lowest index on ties
//   0 < top_k < V          keep logits >= the k-th largest logit (ties kept)
//   p_i = exp((z_i - max) / temperature) over the kept tokens
//   top_p < 1              keep p_i >= tau, tau the largest value with
//                          sum_{p_j >= tau} p_j >= top_p * sum_j p_j
//   draw                   the first token (index order) whose running sum
//                          of kept p exceeds u * (kept mass)
// The k-th largest logit is found by an MSB-first radix select over an
// order-preserving integer image of the floats (warp-aggregated histogram
// updates), tau by bisection over the bit pattern of positive floats.  When
// the kept set is small (top-k), it is first compacted in index order into
// shared memory with its probabilities, and one warp runs the bisection and
// the draw over that list instead of the whole row.
#include "kernels.cuh"

namespace gpt {
namespace {

constexpr int ST = 1024;   // threads per row
constexpr int CAP = 4096;  // kept tokens handled by the compacted path

// order-preserving image of a float as an unsigned integer
__device__ __forceinline__ uint32_t fkey(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// block sum in a fixed order: warp trees in lane order, then the warp sums
__device__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (w == 0) {
    t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
    t = warp_sum(t);
    if (lane == 0) red[32] = t;
  }
  __syncthreads();
  return red[32];
}

template <typename T>
__global__ void __launch_bounds__(ST) k_sample(const T* __restrict__ logits, long ld, int V, float temperature,
                                               int top_k, float top_p, const float* __restrict__ uniform,
                                               int32_t* __restrict__ out) {
  __shared__ float red[33];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sel[2];
  __shared__ int pick;
  const T* z = logits + (long)blockIdx.x * ld;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

  // maximum (and its lowest index, for greedy decoding)
  float best = -INFINITY;
  int bi = 0x7fffffff;
#pragma unroll 4
  for (int i = tid; i < V; i += ST) {
    const float v = to_f<T>(z[i]);
    if (v > best) {  // strided order: the first hit of a thread is its lowest index
      best = v;
      bi = i;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ob > best || (ob == best && oi < bi)) {
      best = ob;
      bi = oi;
    }
  }
  __shared__ float wb[32];
  __shared__ int wi[32];
  if (lane == 0) {
    wb[w] = best;
    wi[w] = bi;
  }
  __syncthreads();
  if (tid == 0) {
    float b = wb[0];
    int ix = wi[0];
    for (int k = 1; k < ST / 32; k++)
      if (wb[k] > b || (wb[k] == b && wi[k] < ix)) {
        b = wb[k];
        ix = wi[k];
      }
    red[0] = b;
    pick = ix;
  }
  __syncthreads();
  const float zmax = red[0];
  if (temperature <= 0.f) {
    if (tid == 0) out[blockIdx.x] = pick;
    return;
  }
  __syncthreads();

  // top-k: the integer image of the k-th largest logit, by an MSB-first
  // radix select.  The first byte is taken from the four byte values at and
  // just below the maximum's, counted in registers (no histogram atomics);
  // only when those hold fewer than k logits does the full first-byte
  // histogram run.  bf16 logits widen to floats whose low 16 bits (of the
  // integer image) are the same for every logit of one sign, so two byte
  // passes decide them and the low half follows from the sign.
  uint32_t thr = 0;
  if (top_k > 0 && top_k < V) {
    constexpr int kLow = sizeof(T) == 2 ? 16 : 0;  // the last byte pass starts at this bit
    uint32_t prefix = 0, mask = 0;
    int need = top_k;
    int shift = 24;
    {
      const int mb = (int)(fkey(zmax) >> 24);
      int cnt[4] = {0, 0, 0, 0};
#pragma unroll 4
      for (int i = tid; i < V; i += ST) {
        const int d = mb - (int)(fkey(to_f<T>(z[i])) >> 24);
#pragma unroll
        for (int j = 0; j < 4; j++) cnt[j] += d == j ? 1 : 0;
      }
#pragma unroll
      for (int j = 0; j < 4; j++) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt[j] += __shfl_xor_sync(0xffffffffu, cnt[j], o);
      }
      __shared__ int wcnt[ST / 32][4];
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 4; j++) wcnt[w][j] = cnt[j];
      }
      __syncthreads();
      if (tid == 0) {
        int cum = 0, found = -1;
        for (int j = 0; j < 4 && mb - j >= 0; j++) {
          int c = 0;
          for (int k = 0; k < ST / 32; k++) c += wcnt[k][j];
          if (cum + c >= need) {
            found = j;
            break;
          }
          cum += c;
        }
        sel[0] = found >= 0 ? (uint32_t)(mb - found) << 24 : 0xFFFFFFFFu;
        sel[1] = (uint32_t)(need - cum);
      }
      __syncthreads();
      if (sel[0] != 0xFFFFFFFFu) {  // the first byte is decided
        prefix = sel[0];
        need = (int)sel[1];
        mask = 255u << 24;
        shift = 16;
      }
      __syncthreads();
    }
    for (; shift >= kLow; shift -= 8) {
      for (int b = tid; b < 256; b += ST) hist[b] = 0;
      __syncthreads();
      for (int i0 = 0; i0 < V; i0 += 4 * ST) {  // whole warps iterate together, 4 loads in flight
        uint32_t key[4];
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const int i = i0 + u * ST + tid;
          key[u] = i < V ? fkey(to_f<T>(z[i])) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const bool hit = i0 + u * ST + tid < V && (key[u] & mask) == prefix;
          const uint32_t want = __ballot_sync(0xffffffffu, hit);
          if (hit) {  // one shared-memory atomic per distinct bin of the warp
            const uint32_t bin = (key[u] >> shift) & 255u;
            const uint32_t peers = __match_any_sync(want, bin);
            if (lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
          }
        }
      }
      __syncthreads();
      if (tid == 0) {
        int cum = 0, b = 255;
        for (; b > 0; b--) {
          if (cum + (int)hist[b] >= need) break;
          cum += (int)hist[b];
        }
        sel[0] = prefix | ((uint32_t)b << shift);
        sel[1] = (uint32_t)(need - cum);
      }
      __syncthreads();
      prefix = sel[0];
      need = (int)sel[1];
      mask |= 255u << shift;
      __syncthreads();
    }
    // bf16: the low 16 bits of the image are 0 for positive logits, all ones for negative ones
    if (kLow == 16) prefix |= (prefix & 0x80000000u) ? 0u : 0xFFFFu;
    thr = prefix;
  }
  const float inv_t = 1.0f / temperature;
  auto prob = [&](int i) -> float {  // unnormalised, 0 outside the top-k set
    const float v = to_f<T>(z[i]);
    return fkey(v) >= thr ? __expf((v - zmax) * inv_t) : 0.f;
  };

  // compacted path: the kept tokens (logit key >= thr) of each warp's
  // contiguous index range, counted, then written in index order with their
  // probabilities; one warp finishes when they fit in shared memory
  __shared__ int c_idx[CAP];
  __shared__ float c_p[CAP];
  __shared__ int wbase[33];
  if (thr != 0u) {
    const int segw = (V + 31) / 32 / 128 * 128 + 128;  // per-warp range, a multiple of 128
    const int w0 = min(V, w * segw), w1 = min(V, w0 + segw);
    int cnt = 0;
    for (int i0 = w0 + lane; i0 - lane < w1; i0 += 128) {  // 4 loads in flight
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; u++) v[u] = i0 + 32 * u < w1 ? to_f<T>(z[i0 + 32 * u]) : 0.f;
#pragma unroll
      for (int u = 0; u < 4; u++) cnt += __popc(__ballot_sync(0xffffffffu, i0 + 32 * u < w1 && fkey(v[u]) >= thr));
    }
    if (lane == 0) wbase[w] = cnt;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int k = 0; k < ST / 32; k++) {
        const int t = wbase[k];
        wbase[k] = run;
        run += t;
      }
      wbase[32] = run;
    }
    __syncthreads();
    const int n = wbase[32];
    if (n <= CAP) {
      int off = wbase[w];
      for (int i0 = w0 + lane; i0 - lane < w1; i0 += 128) {
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; u++) v[u] = i0 + 32 * u < w1 ? to_f<T>(z[i0 + 32 * u]) : 0.f;
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const int i = i0 + 32 * u;
          const bool k = i < w1 && fkey(v[u]) >= thr;
          const uint32_t b = __ballot_sync(0xffffffffu, k);
          if (k) {
            const int o = off + __popc(b & ((1u << lane) - 1u));
            c_idx[o] = i;
            c_p[o] = __expf((v[u] - zmax) * inv_t);
          }
          off += __popc(b);
        }
      }
      __syncthreads();
      if (w != 0) return;
      // top-p over the list: lane-strided sums, butterfly totals (identical in every lane)
      float tau_c = 0.f;
      if (top_p < 1.f) {
        float s0 = 0.f;
        for (int j = lane; j < n; j += 32) s0 += c_p[j];
        const float target = top_p * warp_sum(s0);
        uint32_t cur = 0;
        for (int bit = 30; bit >= 0; bit--) {
          const uint32_t cand = cur | (1u << bit);
          const float t = __uint_as_float(cand);
          float m = 0.f;
          for (int j = lane; j < n; j += 32) {
            const float p = c_p[j];
            if (p >= t) m += p;
          }
          if (warp_sum(m) >= target) cur = cand;
        }
        tau_c = __uint_as_float(cur);
      }
      // draw: contiguous runs of the list per lane, a lane-order scan of their sums
      const int cs = (n + 31) / 32;
      const int j0 = min(n, lane * cs), j1 = min(n, j0 + cs);
      float local = 0.f;
      int last = -1;
      for (int j = j0; j < j1; j++) {
        const float p = c_p[j];
        if (p >= tau_c && p > 0.f) {
          local += p;
          last = c_idx[j];
        }
      }
      float incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      const float total = __shfl_sync(0xffffffffu, incl, 31);
      const float excl = incl - local;
      const float target = uniform[blockIdx.x] * total;
      int hit = 0x7fffffff;
      if (excl + local > target && excl <= target) {
        float run = excl;
        for (int j = j0; j < j1; j++) {
          const float p = c_p[j];
          if (p >= tau_c && p > 0.f) {
            run += p;
            if (run > target) {
              hit = c_idx[j];
              break;
            }
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        hit = min(hit, __shfl_xor_sync(0xffffffffu, hit, o));
        last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
      }
      if (lane == 0) out[blockIdx.x] = hit != 0x7fffffff ? hit : last;
      return;
    }
    __syncthreads();
  }

  // top-p: tau by bisection over the bits of a positive float
  float tau = 0.f;
  if (top_p < 1.f) {
    float s = 0.f;
    for (int i = tid; i < V; i += ST) s += prob(i);
    const float target = top_p * block_sum(s, red);
    uint32_t cur = 0;
    for (int bit = 30; bit >= 0; bit--) {
      const uint32_t cand = cur | (1u << bit);
      const float t = __uint_as_float(cand);
      float m = 0.f;
      for (int i = tid; i < V; i += ST) {
        const float p = prob(i);
        if (p >= t) m += p;
      }
      if (block_sum(m, red) >= target) cur = cand;
    }
    tau = __uint_as_float(cur);
  }

  // draw: contiguous segments per thread, a fixed-order scan of the segment sums
  const int seg = (V + ST - 1) / ST;
  const int i0 = min(V, tid * seg), i1 = min(V, i0 + seg);
  float local = 0.f;
  int last = -1;
  for (int i = i0; i < i1; i++) {
    const float p = prob(i);
    if (p >= tau && p > 0.f) {
      local += p;
      last = i;
    }
  }
  // inclusive scan over threads: lanes in order, then warps in order
  float incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  __shared__ float wsum[32];
  if (lane == 31) wsum[w] = incl;
  if (tid == 0) pick = 0x7fffffff;
  __syncthreads();
  if (tid == 0) {
    float run = 0.f;
    for (int k = 0; k < ST / 32; k++) {
      const float t = wsum[k];
      wsum[k] = run;  // exclusive prefix of warp k
      run += t;
    }
    red[1] = run;  // kept mass
  }
  __syncthreads();
  const float excl = wsum[w] + (incl - local);
  const float target = uniform[blockIdx.x] * red[1];
  if (excl + local > target && excl <= target) {  // the crossing lies in this segment
    float run = excl;
    for (int i = i0; i < i1; i++) {
      const float p = prob(i);
      if (p >= tau && p > 0.f) {
        run += p;
        if (run > target) {
          atomicMin(&pick, i);
          break;
        }
      }
    }
  }
  __syncthreads();
  // rounding can leave the target at or past the total: the last kept token
  __shared__ int last_kept;
  if (tid == 0) last_kept = -1;
  __syncthreads();
  if (last >= 0) atomicMax(&last_kept, last);
  __syncthreads();
  if (tid == 0) out[blockIdx.x] = pick != 0x7fffffff ? pick : last_kept;
}

}  // namespace

void sample_rows(Ctx& c, const void* logits, bool bf16_logits, int rows, int V, long ld, float temperature, int top_k,
                 float top_p, const float* uniform, int32_t* out) {
  LaunchScope s(c, "sample");
  if (bf16_logits)
    k_sample<bf16><<<rows, ST, 0, c.stream>>>(reinterpret_cast<const bf16*>(logits), ld, V, temperature, top_k,
                                             top_p, uniform, out);
  else
    k_sample<float><<<rows, ST, 0, c.stream>>>(reinterpret_cast<const float*>(logits), ld, V, temperature, top_k,
                                              top_p, uniform, out);
}

}  // namespace gpt
