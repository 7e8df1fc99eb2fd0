/*
 * gpt_testing.h -- kernel-level entry points of libgpt.so used by the parity
 * tests to check one kernel at a time (the GEMM with its epilogues, the
 * attention forward/backward) against the CPU oracle.  Not part of the
 * training step's hot path.  All pointers are device pointers on the current
 * device; work is enqueued on `stream` (a cudaStream_t) and the call
 * synchronises it before returning.  `d_flags` is a device uint32 that
 * receives the GPT_FLAG_* bits the kernels raise.
 */
#ifndef GPT_B200_TESTING_H
#define GPT_B200_TESTING_H

#include <stdint.h>

#include "gpt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Backends of gpt_test_gemm (GPT_GEMM_TC_BF16 forces the single-CTA
 * tensor-core kernel). */
enum {
  GPT_GEMM_SIMT_F32 = 0,
  GPT_GEMM_SIMT_BF16 = 1,
  GPT_GEMM_TC_BF16 = 2,
  GPT_GEMM_SKINNY_BF16 = 3,
  GPT_GEMM_TC2_BF16 = 4,  /* pair-CTA tensor-core GEMM (256-row tiles over two SMs) */
  GPT_GEMM_TC_PLANNED = 5 /* the tensor-core kernel and split the training step's cost model picks */
};

/* D[m, n] = sum_k A[m, k] * B[n, k] followed by epilogue `epi_kind`:
 *   0 out = D; 1 out = D + bias; 2 with h = D + bias: out = act'(h), out2 = act(h);
 *   3 res_out = res_in + D + bias; 4 out = D * aux (aux: a saved act'(h));
 *   5 out += D (fp32); 6 out = D (fp32).
 * A is [M, K] row-major with pitch lda when a_kmajor, else [K, M] (pitch lda);
 * B is [N, K] when b_kmajor, else [K, N].  Operands are fp32 for
 * GPT_GEMM_SIMT_F32 and bf16 otherwise; outputs of kinds 0-2 and 4 have the
 * operand type, kinds 3, 5 and 6 are fp32.  act: 0 GELU (erf), 1 ReLU.
 * split_k > 1 (kind 5 only, tensor-core backend) needs `partial`
 * [split_k, M, N] fp32 scratch.  GPT_GEMM_SKINNY_BF16 (the decoding-step
 * GEMM) takes M <= 16, K a multiple of 32, both operands K-major, no split-K.
 * GPT_ERR_UNSUPPORTED when the tensor-core or skinny backend cannot take the
 * shape.  colsum (nullable; kind 4 on the tensor-core backends): fp32
 * [ceil(M / 32), N] receives the column sums of the stored output over each
 * 32-row group. */
gpt_status gpt_test_gemm(int32_t backend, int32_t M, int32_t N, int32_t K, const void* A, int64_t lda,
                         int32_t a_kmajor, const void* B, int64_t ldb, int32_t b_kmajor, int32_t epi_kind,
                         int32_t act, void* out, void* out2, int32_t ldo, const void* aux, const float* bias,
                         const float* res_in, float* res_out, int32_t split_k, float* partial, float* colsum,
                         void* stream, uint32_t* d_flags);

/* Causal attention of one layer.  qkv [B, T, 3, H, hd], o [B, T, H, hd],
 * lse fp32 [B, H, T]; backward also takes dout [B, T, H, hd] and writes
 * dqkv [B, T, 3, H, hd] using dsum fp32 [B, H, T] as scratch.  dtype: 0 fp32,
 * 1 bf16.  backend: 0 CUDA cores, 1 tensor cores (GPT_ERR_UNSUPPORTED when
 * the shape is not supported).  colsum (nullable; backward of backend 1):
 * fp32 [B T / 128, 3 H hd] receives the column sums of the stored dqkv over
 * each 128-row block.  Dropout on the probabilities with
 * (p, seed, counter, layer) as in the model (site 1); p = 0 disables it. */
gpt_status gpt_test_attention(int32_t backend, int32_t backward, int32_t dtype, int32_t B, int32_t T, int32_t H,
                              int32_t hd, const void* qkv, void* o, float* lse, const void* dout, void* dqkv,
                              float* dsum, float* colsum, float p, uint64_t seed, uint64_t counter, int32_t layer,
                              void* stream, uint32_t* d_flags);

/* The bounded device-side wait of the tensor-core kernels, made to run out:
 * one warp waits on an mbarrier that nothing arrives at, with a limit of
 * limit_ns nanoseconds (1e3 .. 1e10) instead of the kernels' 2 s.  The wait
 * gives up, sets GPT_FLAG_TIMEOUT in *d_flags and 1 in *d_gave_up (device
 * uint32 / int32, zeroed by the caller), and the kernel returns: the GPU
 * context stays usable.  Synchronising.  Returns GPT_ERR_TIMEOUT when the
 * flag was raised (the expected outcome), GPT_OK otherwise. */
gpt_status gpt_test_wait_timeout(uint64_t limit_ns, void* stream, uint32_t* d_flags, int32_t* d_gave_up);

#ifdef __cplusplus
}
#endif
#endif /* GPT_B200_TESTING_H */
