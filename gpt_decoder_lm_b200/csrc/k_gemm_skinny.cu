// Skinny GEMM for the decoding step: D[M, N] = A[M, K] . W[N, K]^T with at
// most 16 rows (one token per batch row), bf16 operands, fp32 accumulation,
// then the shared element-wise epilogue.
//
// With M <= 16 every weight element is used M times, so the op is bound by
// streaming W from HBM once (2 N K bytes), not by arithmetic.  The kernel is
// built around that stream: each warp owns 16 rows of W (16 output columns)
// and one slice of K, and pulls its W rows straight from global memory into
// registers in the register layout of a 16x8x16 warp-level MMA, where W takes
// the MMA's 16-row side and the activation rows the 8-column side (one or two
// 8-row tiles).  No shared-memory staging of W, no tile padding of M to 128
// rows: the tensor-core 128-row tiles of the training GEMM would read the
// same weights with 8-16 CTAs for an N of 768-3072 and leave most SMs idle.
//
// Because a dot product does not depend on the order of its terms, lane
// (g, q) of the MMA layout loads the 16 contiguous bytes at k = 8q .. 8q+7 of
// a 32-wide k block, and both operands agree to feed k = 8q .. 8q+3 to the
// first k16 step and 8q+4 .. 8q+7 to the second.  Every W row is thereby read
// as fully used 64-byte segments.  The activations (M x K, a few KB) are
// staged once per CTA in shared memory with a row pitch of 64 mod 128 bytes,
// which keeps the fragment reads free of bank conflicts.
//
// Warps of a CTA split K so that each warp's whole slice of W is requested in
// one round of loads (the op is latency-bound at these sizes); their partial
// sums are added in shared memory in a fixed order (deterministic).  The
// first round of weight loads is issued before the programmatic-launch wait:
// the decoding step writes no weights.
#include "common.cuh"
#include "epilogue.cuh"
#include "kernels.cuh"

namespace gpt {
namespace {

constexpr int SK_WARPS = 16;  // warps per CTA
constexpr int SK_U = 6;       // 32-wide k blocks in flight per warp

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// NT = number of 8-row activation tiles (1: M <= 8, 2: M <= 16).
// ks = warps splitting K (a power of two up to SK_WARPS); pitch =
// shared-memory row pitch of the staged activations in bytes.
template <int NT>
__global__ void __launch_bounds__(SK_WARPS * 32) k_gemm_skinny(GemmDesc g, SkinnyNorm nrm, int ks, int pitch) {
  extern __shared__ __align__(16) uint8_t smem[];
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, q = lane & 3;
  const int cw = SK_WARPS / ks;  // column groups per CTA
  const int wc = warp % cw, wk = warp / cw;
  const int n0 = (blockIdx.x * cw + wc) * 16;
  const int nkb = g.K >> 5;
  const int per = (nkb + ks - 1) / ks;
  const int kb0 = min(nkb, wk * per), kb1 = min(nkb, kb0 + per);

  // this lane's two W rows (output columns n0 + gr and n0 + gr + 8); rows past
  // N are clamped to the last row, read and discarded
  const bf16* W = reinterpret_cast<const bf16*>(g.B);
  const long r0 = min(n0 + gr, g.N - 1), r1 = min(n0 + gr + 8, g.N - 1);
  const uint4* w0 = reinterpret_cast<const uint4*>(W + r0 * g.ldb + 8 * q);
  const uint4* w1 = reinterpret_cast<const uint4*>(W + r1 * g.ldb + 8 * q);
  uint4 wa[SK_U], wb[SK_U];
  auto load = [&](int kb) {
#pragma unroll
    for (int u = 0; u < SK_U; u++)
      if (kb + u < kb1) {
        wa[u] = ld_stream(w0 + 4 * (kb + u));
        wb[u] = ld_stream(w1 + 4 * (kb + u));
      }
  };
  load(kb0);
  pdl_wait();

  if (nrm.x) {
    // A = norm(x) computed here (one warp per row, the norm kernel's formulas
    // and summation order): LayerNorm (x - mean) rstd w + b, or RMSNorm x rstd
    const int d4 = g.K >> 2;
    for (int r = warp; r < 8 * NT; r += SK_WARPS) {
      uint8_t* srow = smem + (size_t)r * pitch;
      if (r >= g.M) {
        for (int c8 = lane; c8 < (g.K >> 3); c8 += 32)
          *reinterpret_cast<uint4*>(srow + 16 * c8) = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      const float4* xr = reinterpret_cast<const float4*>(nrm.x + (long)r * nrm.ldx);
      float sum = 0.f;
#pragma unroll 4
      for (int c = lane; c < d4; c += 32) {
        const float4 v = xr[c];
        sum += nrm.rms ? (v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w) : (v.x + v.y + v.z + v.w);
      }
      sum = warp_sum(sum);
      float mean = 0.f, rstd;
      if (nrm.rms) {
        rstd = 1.0f / sqrtf(sum / g.K + nrm.eps);
      } else {
        mean = sum / g.K;
        float qs = 0.f;
#pragma unroll 4
        for (int c = lane; c < d4; c += 32) {
          const float4 v = xr[c];
          const float a = v.x - mean, b = v.y - mean, cc = v.z - mean, dd = v.w - mean;
          qs += a * a + b * b + cc * cc + dd * dd;
        }
        qs = warp_sum(qs);
        rstd = 1.0f / sqrtf(qs / g.K + nrm.eps);
      }
#pragma unroll 2
      for (int c8 = lane; c8 < (g.K >> 3); c8 += 32) {
        float y[8];
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const float4 v = xr[2 * c8 + h];
          y[4 * h + 0] = (v.x - mean) * rstd;
          y[4 * h + 1] = (v.y - mean) * rstd;
          y[4 * h + 2] = (v.z - mean) * rstd;
          y[4 * h + 3] = (v.w - mean) * rstd;
          if (!nrm.rms) {
            const float4 ww = reinterpret_cast<const float4*>(nrm.w)[2 * c8 + h];
            const float4 bb = reinterpret_cast<const float4*>(nrm.b)[2 * c8 + h];
            y[4 * h + 0] = y[4 * h + 0] * ww.x + bb.x;
            y[4 * h + 1] = y[4 * h + 1] * ww.y + bb.y;
            y[4 * h + 2] = y[4 * h + 2] * ww.z + bb.z;
            y[4 * h + 3] = y[4 * h + 3] * ww.w + bb.w;
          }
        }
        uint4 o;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int k = 0; k < 4; k++) {
          __nv_bfloat162 p2;
          p2.x = __float2bfloat16_rn(y[2 * k]);
          p2.y = __float2bfloat16_rn(y[2 * k + 1]);
          ow[k] = *reinterpret_cast<uint32_t*>(&p2);
        }
        *reinterpret_cast<uint4*>(srow + 16 * c8) = o;
      }
    }
  } else {
    // activations -> shared memory, rows M .. 8 NT - 1 zero; eight 16-byte
    // loads per thread in flight before their stores
    const bf16* A = reinterpret_cast<const bf16*>(g.A);
    const int cpr = g.K >> 3;  // 16-byte chunks per row
    const int total = 8 * NT * cpr;
    for (int i0 = threadIdx.x; i0 < total; i0 += 8 * SK_WARPS * 32) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const int i = i0 + u * SK_WARPS * 32, r = i / cpr, cidx = i - r * cpr;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (i < total && r < g.M) v[u] = *reinterpret_cast<const uint4*>(A + (long)r * g.lda + 8 * cidx);
      }
#pragma unroll
      for (int u = 0; u < 8; u++) {
        const int i = i0 + u * SK_WARPS * 32, r = i / cpr, cidx = i - r * cpr;
        if (i < total) *reinterpret_cast<uint4*>(smem + (size_t)r * pitch + 16 * cidx) = v[u];
      }
    }
  }
  __syncthreads();

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; t++) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  const uint8_t* a_lane = smem + (size_t)gr * pitch + 16 * q;
  for (int kb = kb0; kb < kb1; kb += SK_U) {
    if (kb != kb0) load(kb);
#pragma unroll
    for (int u = 0; u < SK_U; u++) {
      if (kb + u < kb1) {
#pragma unroll
        for (int t = 0; t < NT; t++) {
          const uint4 b = *reinterpret_cast<const uint4*>(a_lane + (size_t)t * 8 * pitch + 64 * (kb + u));
          mma_16816(acc[t], wa[u].x, wb[u].x, wa[u].y, wb[u].y, b.x, b.y);
          mma_16816(acc[t], wa[u].z, wb[u].z, wa[u].w, wb[u].w, b.z, b.w);
        }
      }
    }
  }

  if (ks > 1) {  // add the K slices in warp order
    float* red = reinterpret_cast<float*>(smem + (size_t)8 * NT * pitch);  // [warp][NT*4][32]
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
      for (int j = 0; j < 4; j++) red[(warp * NT * 4 + t * 4 + j) * 32 + lane] = acc[t][j];
    __syncthreads();
    if (wk != 0) return;
    for (int s = 1; s < ks; s++) {
      const int w2 = s * cw + wc;
#pragma unroll
      for (int t = 0; t < NT; t++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[t][j] += red[(w2 * NT * 4 + t * 4 + j) * 32 + lane];
    }
  }

  // accumulator (row = output column n, column = activation row m)
#pragma unroll
  for (int t = 0; t < NT; t++)
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const int n = n0 + gr + (j >= 2 ? 8 : 0);
      const int m = 8 * t + 2 * q + (j & 1);
      if (m < g.M && n < g.N) epi_apply<bf16>(g.epi, g.N, m, n, acc[t][j]);
    }
}

constexpr int SK_MAX_SMEM = 200 * 1024;

int skinny_pitch(int K) { return ((2 * K + 127) / 128) * 128 + 64; }

// K split: the fewest warps that leave each at most SK_U k blocks (one round
// of loads), then more while the grid has fewer CTAs than the GPU has SMs and
// every warp keeps at least two k blocks (the weight stream spread over more
// SMs), up to the CTA's warps
int skinny_ks(const GemmDesc& g, int num_sms) {
  const int nkb = g.K / 32, groups = (g.N + 15) / 16;
  int ks = 1;
  while (ks < SK_WARPS && (nkb + ks - 1) / ks > SK_U) ks *= 2;
  while (ks < SK_WARPS && (groups + SK_WARPS / ks - 1) / (SK_WARPS / ks) < num_sms && nkb / (2 * ks) >= 2) ks *= 2;
  return ks;
}

size_t skinny_smem(const GemmDesc& g, int ks) {
  const int nt = g.M > 8 ? 2 : 1;
  return (size_t)8 * nt * skinny_pitch(g.K) + (ks > 1 ? (size_t)SK_WARPS * nt * 4 * 32 * 4 : 0);
}

template <int NT>
void launch_skinny(Ctx& c, const GemmDesc& g, const SkinnyNorm& nrm) {
  const int ks = skinny_ks(g, c.num_sms);
  const int cw = SK_WARPS / ks, groups = (g.N + 15) / 16;
  const int pitch = skinny_pitch(g.K);
  const size_t smem = skinny_smem(g, ks);
  // per-device function attribute: set before every launch
  cudaFuncSetAttribute(k_gemm_skinny<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, SK_MAX_SMEM);
  LaunchScope s(c, g.name ? g.name : "gemm_skinny");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((groups + cw - 1) / cw);
  cfg.blockDim = dim3(SK_WARPS * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_gemm_skinny<NT>, g, nrm, ks, pitch) != cudaSuccess) {
    cudaGetLastError();  // programmatic serialization refused: an ordinary launch
    k_gemm_skinny<NT><<<cfg.gridDim, cfg.blockDim, smem, c.stream>>>(g, nrm, ks, pitch);
  }
}

}  // namespace

bool gemm_skinny_supported(const GemmDesc& g) {
  if (g.M < 1 || g.M > 16 || g.N < 1 || g.K < 32 || (g.K % 32)) return false;
  if (!g.a_kmajor || !g.b_kmajor || g.partial) return false;
  if ((g.lda % 8) || (g.ldb % 8)) return false;  // 16-byte rows
  if ((reinterpret_cast<uintptr_t>(g.A) & 15) || (reinterpret_cast<uintptr_t>(g.B) & 15)) return false;
  return skinny_smem(g, SK_WARPS) <= (size_t)SK_MAX_SMEM;
}

bool skinny_norm_supported(const GemmDesc& g, const SkinnyNorm& n) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  return n.x && al(n.x) && (n.ldx % 4) == 0 && n.ldx >= g.K && (n.rms || (n.w && n.b && al(n.w) && al(n.b)));
}

void gemm_skinny_bf16(Ctx& c, const GemmDesc& g, const SkinnyNorm* nrm) {
  const SkinnyNorm none{};
  const SkinnyNorm& n = nrm ? *nrm : none;
  if (g.M > 8) launch_skinny<2>(c, g, n);
  else launch_skinny<1>(c, g, n);
}

}  // namespace gpt
