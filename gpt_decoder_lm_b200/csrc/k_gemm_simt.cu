// CUDA-core GEMM with arbitrary operand strides: the fp32-mode contraction
// (fp32 mode keeps fp32 rounding everywhere, which the tensor cores' TF32
// would not) and a bf16-operand reference used to cross-check the tensor-core
// kernel.  D[m, n] = sum_k A[m, k] B[n, k], 64x64 tiles, 4x4 per thread.
#include "epilogue.cuh"

namespace gpt {

template <typename T>
__global__ void __launch_bounds__(256) k_gemm_simt(GemmDesc g) {
  pdl_trigger();
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const T* A = reinterpret_cast<const T*>(g.A);
  const T* B = reinterpret_cast<const T*>(g.B);
  int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  long m0 = (long)blockIdx.y * 64;
  int n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += 16) {
    // 64 x 16 elements of A and of B, 4 per thread
    for (int l = threadIdx.x; l < 64 * 16; l += 256) {
      int r, kk;
      if (g.a_kmajor) { r = l >> 4; kk = l & 15; } else { kk = l >> 6; r = l & 63; }
      long m = m0 + r;
      int k = k0 + kk;
      float v = 0.f;
      if (m < g.M && k < g.K) v = to_f<T>(g.a_kmajor ? A[m * g.lda + k] : A[(long)k * g.lda + m]);
      As[kk][r] = v;
    }
    for (int l = threadIdx.x; l < 64 * 16; l += 256) {
      int r, kk;
      if (g.b_kmajor) { r = l >> 4; kk = l & 15; } else { kk = l >> 6; r = l & 63; }
      int n = n0 + r;
      int k = k0 + kk;
      float v = 0.f;
      if (n < g.N && k < g.K) v = to_f<T>(g.b_kmajor ? B[(long)n * g.ldb + k] : B[(long)k * g.ldb + n]);
      Bs[kk][r] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; kk++) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; i++) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; j++) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++) {
    long m = m0 + ty * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; j++) {
      int n = n0 + tx * 4 + j;
      if (n < g.N) epi_apply<T>(g.epi, g.N, m, n, acc[i][j]);
    }
  }
}

static void launch_simt_f32(Ctx& c, const GemmDesc& g) {
  dim3 grid((g.N + 63) / 64, (unsigned)((g.M + 63) / 64));
  LaunchScope s(c, "gemm_simt_f32");
  k_gemm_simt<float><<<grid, 256, 0, c.stream>>>(g);
}

void gemm_simt_f32(Ctx& c, const GemmDesc& g) {
  GemmDesc d = g;
  d.split_k = 1;
  launch_simt_f32(c, d);
}

void gemm_simt_bf16(Ctx& c, const GemmDesc& g) {
  GemmDesc d = g;
  d.split_k = 1;
  dim3 grid((d.N + 63) / 64, (unsigned)((d.M + 63) / 64));
  LaunchScope s(c, "gemm_simt_bf16");
  k_gemm_simt<bf16><<<grid, 256, 0, c.stream>>>(d);
}

__global__ void k_splitk_reduce(const float* __restrict__ part, int splits, long MN, float* __restrict__ out) {
  pdl_trigger();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= MN) return;
  float s = 0.f;
  for (int k = 0; k < splits; k++) s += part[(long)k * MN + i];
  out[i] += s;
}

// the same sums, four adjacent elements per thread with 16-byte accesses; the
// partial loads of up to 8 splits are issued before any add (same add order)
__global__ void k_splitk_reduce4(const float4* __restrict__ part, int splits, long MN4, float4* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= MN4) return;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k0 = 0; k0 < splits; k0 += 8) {
    float4 v[8];
#pragma unroll
    for (int k = 0; k < 8; k++)
      if (k0 + k < splits) v[k] = part[(long)(k0 + k) * MN4 + i];
#pragma unroll
    for (int k = 0; k < 8; k++)
      if (k0 + k < splits) {
        s.x += v[k].x;
        s.y += v[k].y;
        s.z += v[k].z;
        s.w += v[k].w;
      }
  }
  float4 o = out[i];
  o.x += s.x;
  o.y += s.y;
  o.z += s.z;
  o.w += s.w;
  out[i] = o;
}

void splitk_reduce(Ctx& c, const float* partial, int splits, long MN, float* out) {
  LaunchScope s(c, "splitk_reduce");
  if (MN % 4 == 0 && !(reinterpret_cast<uintptr_t>(partial) & 15) && !(reinterpret_cast<uintptr_t>(out) & 15)) {
    const long MN4 = MN / 4;
    launch_pdl(k_splitk_reduce4, (unsigned)((MN4 + 255) / 256), 256, 0, c.stream,
               reinterpret_cast<const float4*>(partial), splits, MN4, reinterpret_cast<float4*>(out));
  } else {
    k_splitk_reduce<<<(unsigned)((MN + 255) / 256), 256, 0, c.stream>>>(partial, splits, MN, out);
  }
}

}  // namespace gpt
