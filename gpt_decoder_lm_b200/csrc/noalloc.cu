// Allocation-free entry point: the split-K weight-gradient GEMM with its
// partial sums in a file-scope device array instead of caller-provided scratch.
//
// Some callers cannot allocate device memory: code running inside a plugin or
// custom-operator interface that only hands over its input and output buffers,
// a process whose device memory is owned by another allocator or pool, or work
// that must not call cudaMalloc (which synchronises the whole device).  They
// call gpt_gemm_dw_accumulate_noalloc with inputs and outputs only.
//
// The scratch array is part of this library's device image: every GPU that
// loads the library holds its 16 MiB until the process exits.  Host code gets
// the array's device address per device with cudaGetSymbolAddress (the array's
// name in host code is only a host-side stand-in).
#include <mutex>

#include "../../include/gpt.h"
#include "kernels.cuh"

namespace {

constexpr size_t kScratchFloats = size_t(4) << 20;  // 16 MiB of fp32 partial sums (the stated maximum)
constexpr size_t kHead = 64;                        // first 256 bytes: the kernels' flag word

static __device__ __align__(256) float g_scratch[kHead + kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_dev[kMaxDevices] = {};

// Device address of the array on the current device, looked up (and checked)
// once per device by the first call made while that device is current.
gpt_status device_arrays(float** scratch, uint32_t** flags) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_dev[dev]) {
    void* s = nullptr;
    if (cudaGetSymbolAddress(&s, g_scratch) != cudaSuccess || !s) return GPT_ERR_CUDA;
    g_scratch_dev[dev] = static_cast<float*>(s);
  }
  *flags = reinterpret_cast<uint32_t*>(g_scratch_dev[dev]);
  *scratch = g_scratch_dev[dev] + kHead;
  return GPT_OK;
}

}  // namespace

extern "C" gpt_status gpt_gemm_dw_accumulate_noalloc(int32_t M, int32_t N, int32_t K, const void* d_a, int64_t lda,
                                                     const void* d_b, int64_t ldb, float* d_dw, int32_t split_k,
                                                     void* cuda_stream) {
  using namespace gpt;
  if (M <= 0 || N <= 0 || K <= 0 || !d_a || !d_b || !d_dw || split_k < 1) return GPT_ERR_INVALID_ARG;
  if ((size_t)split_k * (size_t)M * (size_t)N > kScratchFloats) return GPT_ERR_WORKSPACE_TOO_SMALL;
  float* scratch = nullptr;
  uint32_t* flags = nullptr;
  gpt_status st = device_arrays(&scratch, &flags);
  if (st != GPT_OK) return st;
  Ctx c;
  c.stream = static_cast<cudaStream_t>(cuda_stream);
  c.flags = flags;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) c.num_sms = sms;
  GemmDesc g;
  g.M = M;
  g.N = N;
  g.K = K;
  g.A = d_a;
  g.lda = lda;
  g.a_kmajor = false;
  g.B = d_b;
  g.ldb = ldb;
  g.b_kmajor = false;
  g.epi.kind = EPI_ACC_F32;
  g.epi.out = d_dw;
  g.epi.ldo = N;
  g.split_k = split_k;
  g.partial = scratch;  // every partial element is written before it is read: nothing needs clearing
  g.name = "gemm_dw_noalloc";
  if (!gemm_tc_supported(g)) return GPT_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(flags, 0, sizeof(uint32_t), c.stream) != cudaSuccess) return GPT_ERR_CUDA;
  // A launch error of our own kernels shows as a new last error; one the
  // caller's earlier work left behind is not ours to report or to clear.
  const bool clean_before = cudaPeekAtLastError() == cudaSuccess;
  if (!gemm_tc_bf16(c, g)) return GPT_ERR_CUDA;
  if (clean_before && cudaPeekAtLastError() != cudaSuccess) {
    cudaGetLastError();
    return GPT_ERR_CUDA;
  }
  uint32_t h_flags = 0;
  if (cudaMemcpyAsync(&h_flags, flags, sizeof(uint32_t), cudaMemcpyDeviceToHost, c.stream) != cudaSuccess)
    return GPT_ERR_CUDA;
  if (cudaStreamSynchronize(c.stream) != cudaSuccess) return GPT_ERR_CUDA;
  return (h_flags & FLAG_TIMEOUT) ? GPT_ERR_TIMEOUT : GPT_OK;
}
