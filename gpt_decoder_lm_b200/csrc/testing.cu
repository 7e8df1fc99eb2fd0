// Kernel-level entry points for the parity tests (include/gpt_testing.h).
#include "../../include/gpt_testing.h"
#include "kernels.cuh"
#include "sm100.cuh"

using namespace gpt;

extern "C" gpt_status gpt_test_gemm(int32_t backend, int32_t M, int32_t N, int32_t K, const void* A, int64_t lda,
                                    int32_t a_kmajor, const void* B, int64_t ldb, int32_t b_kmajor, int32_t epi_kind,
                                    int32_t act, void* out, void* out2, int32_t ldo, const void* aux,
                                    const float* bias, const float* res_in, float* res_out, int32_t split_k,
                                    float* partial, float* colsum, void* stream, uint32_t* d_flags) {
  if (M <= 0 || N <= 0 || K <= 0 || !A || !B || epi_kind < 0 || epi_kind > 6) return GPT_ERR_INVALID_ARG;
  if (colsum && epi_kind != EPI_ACT_BWD) return GPT_ERR_INVALID_ARG;
  Ctx c;
  c.stream = (cudaStream_t)stream;
  c.flags = d_flags;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) c.num_sms = sms;
  GemmDesc g;
  g.M = M;
  g.N = N;
  g.K = K;
  g.A = A;
  g.lda = lda;
  g.a_kmajor = a_kmajor != 0;
  g.B = B;
  g.ldb = ldb;
  g.b_kmajor = b_kmajor != 0;
  g.epi.kind = epi_kind;
  g.epi.act = act;
  g.epi.out = out;
  g.epi.out2 = out2;
  g.epi.ldo = ldo;
  g.epi.aux = aux;
  g.epi.bias = bias;
  g.epi.res_in = res_in;
  g.epi.res_out = res_out;
  g.epi.ld_res = ldo;
  g.split_k = split_k;
  g.partial = partial;
  g.epi.colsum = colsum;
  switch (backend) {
    case GPT_GEMM_SIMT_F32: gemm_simt_f32(c, g); break;
    case GPT_GEMM_SIMT_BF16: gemm_simt_bf16(c, g); break;
    case GPT_GEMM_TC_BF16:
    case GPT_GEMM_TC2_BF16:
    case GPT_GEMM_TC_PLANNED:
      if (!gemm_tc_supported(g)) return GPT_ERR_UNSUPPORTED;
      if (!gemm_tc_bf16(c, g, backend == GPT_GEMM_TC_BF16 ? TC_SINGLE : backend == GPT_GEMM_TC2_BF16 ? TC_PAIR : TC_ANY))
        return GPT_ERR_CUDA;
      break;
    case GPT_GEMM_SKINNY_BF16:
      if (!gemm_skinny_supported(g)) return GPT_ERR_UNSUPPORTED;
      gemm_skinny_bf16(c, g);
      break;
    default: return GPT_ERR_INVALID_ARG;
  }
  if (cudaStreamSynchronize(c.stream) != cudaSuccess || cudaGetLastError() != cudaSuccess) return GPT_ERR_CUDA;
  return GPT_OK;
}

extern "C" gpt_status gpt_test_attention(int32_t backend, int32_t backward, int32_t dtype, int32_t B, int32_t T,
                                         int32_t H, int32_t hd, const void* qkv, void* o, float* lse,
                                         const void* dout, void* dqkv, float* dsum, float* colsum, float p,
                                         uint64_t seed, uint64_t counter, int32_t layer, void* stream,
                                         uint32_t* d_flags) {
  if (B <= 0 || T <= 0 || H <= 0 || !qkv || !o || !lse) return GPT_ERR_INVALID_ARG;
  if (backward && (!dout || !dqkv || !dsum)) return GPT_ERR_INVALID_ARG;
  Ctx c;
  c.stream = (cudaStream_t)stream;
  c.flags = d_flags;
  AttnDesc a{B, T, H, hd, qkv, o, lse, dout, dqkv, dsum, make_drop_key(seed, counter, layer, 1, p)};
  if (colsum && !(backward && backend == 1)) return GPT_ERR_INVALID_ARG;
  a.colsum = colsum;
  if (backend == 1) {
    if (dtype != 1 || !attn_tc_supported(a)) return GPT_ERR_UNSUPPORTED;
    if (!(backward ? attn_bwd_tc(c, a) : attn_fwd_tc(c, a))) return GPT_ERR_CUDA;
  } else if (backend == 0) {
    if (hd != 4 && hd != 8 && hd != 16 && hd != 32 && hd != 64 && hd != 128) return GPT_ERR_UNSUPPORTED;
    if (dtype == 1) {
      if (backward) attn_bwd_simt<bf16>(c, a);
      else attn_fwd_simt<bf16>(c, a);
    } else {
      if (backward) attn_bwd_simt<float>(c, a);
      else attn_fwd_simt<float>(c, a);
    }
  } else {
    return GPT_ERR_INVALID_ARG;
  }
  if (cudaStreamSynchronize(c.stream) != cudaSuccess || cudaGetLastError() != cudaSuccess) return GPT_ERR_CUDA;
  return GPT_OK;
}

// One warp waits on an mbarrier that nothing ever arrives at, through the
// same bounded wait the tensor-core kernels use, with the given limit.
__global__ void k_test_wait_timeout(uint64_t limit_ns, uint32_t* flags, int* gave_up) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = sm100::smem_u32(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = sm100::mbar_wait(b, 0, &abort_flag, flags, limit_ns);
  if (!ok && threadIdx.x == 0) *gave_up = 1;
}

extern "C" gpt_status gpt_test_wait_timeout(uint64_t limit_ns, void* stream, uint32_t* d_flags, int32_t* d_gave_up) {
  if (!d_flags || !d_gave_up || limit_ns < 1000 || limit_ns > 10000000000ull) return GPT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  k_test_wait_timeout<<<1, 32, 0, st>>>(limit_ns, d_flags, d_gave_up);
  if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess) return GPT_ERR_CUDA;
  uint32_t f = 0;
  if (cudaMemcpy(&f, d_flags, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return GPT_ERR_CUDA;
  return (f & FLAG_TIMEOUT) ? GPT_ERR_TIMEOUT : GPT_OK;
}

