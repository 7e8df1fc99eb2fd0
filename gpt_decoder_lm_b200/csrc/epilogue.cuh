// Element-wise GEMM epilogue shared by the CUDA-core and tensor-core GEMMs.
#pragma once
#include "kernels.cuh"

namespace gpt {

__device__ __forceinline__ float act_fwd(int act, float h) { return act == ACT_RELU ? fmaxf(h, 0.f) : gelu_f(h); }
__device__ __forceinline__ float act_grad(int act, float h) {
  return act == ACT_RELU ? (h > 0.f ? 1.f : 0.f) : gelu_grad_f(h);
}

// Applies the epilogue to one accumulator element D[m, n] (0 <= m < M, 0 <= n < N).
template <typename T>
__device__ __forceinline__ void epi_apply(const GemmEpi& e, int N, long m, int n, float acc) {
  switch (e.kind) {
    case EPI_STORE:
      reinterpret_cast<T*>(e.out)[m * e.ldo + n] = from_f<T>(acc);
      break;
    case EPI_BIAS:
      reinterpret_cast<T*>(e.out)[m * e.ldo + n] = from_f<T>(acc + (e.bias ? e.bias[n] : 0.f));
      break;
    case EPI_BIAS_ACT: {
      float h = acc + (e.bias ? e.bias[n] : 0.f);
      reinterpret_cast<T*>(e.out)[m * e.ldo + n] = from_f<T>(act_grad(e.act, h));
      reinterpret_cast<T*>(e.out2)[m * e.ldo + n] = from_f<T>(act_fwd(e.act, h));
      break;
    }
    case EPI_RESADD: {
      float y = acc + (e.bias ? e.bias[n] : 0.f);
      if (e.drop.active) y *= drop_mul(drop_live(e.drop), (uint64_t)m * N + n);
      e.res_out[m * e.ld_res + n] = e.res_in[m * e.ld_res + n] + y;
      break;
    }
    case EPI_ACT_BWD: {
      float dact = to_f<T>(reinterpret_cast<const T*>(e.aux)[m * e.ldo + n]);
      reinterpret_cast<T*>(e.out)[m * e.ldo + n] = from_f<T>(acc * dact);
      break;
    }
    case EPI_ACC_F32:
      reinterpret_cast<float*>(e.out)[m * e.ldo + n] += acc;
      break;
    case EPI_STORE_F32:
      reinterpret_cast<float*>(e.out)[m * e.ldo + n] = acc;
      break;
  }
}

}  // namespace gpt
