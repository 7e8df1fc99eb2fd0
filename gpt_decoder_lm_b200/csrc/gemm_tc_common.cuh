// Pieces the single-CTA (k_gemm_tc.cu) and pair-CTA (k_gemm_tc2.cu)
// tensor-core GEMMs share: tile constants, kernel arguments, the epilogue's
// swizzled staging-tile accessors and bias helpers, and the host-side tensor
// map encoders.  Internal linkage: each including file gets its own copy.
#pragma once

#include <cudaTypedefs.h>

#include <mutex>

#include "epilogue.cuh"
#include "sm100.cuh"

namespace gpt {
namespace {

using namespace sm100;

constexpr int BM = 128, BK = 64;
constexpr int EPI_WARPS = 16;                // 4 per TMEM lane quadrant
constexpr int EPI_PARTS = EPI_WARPS / 4;     // column ranges per quadrant
constexpr int kThreads = 64 + 32 * EPI_WARPS;  // producer, MMA, epilogue warps
constexpr int EPI_BUF = 4096;                // one 32x32 fp32 (or two bf16) staging tiles

struct TcArgs {
  int M, N, K;
  int num_m, num_n, splits, kb_per_split, nkb;
  int n_fast;  // tile order: 1 = N-fastest (concurrent CTAs share A tiles in L2), 0 = M-fastest
  int kind, act;
  int acc_partial;  // split partials: 1 = TMA reduce-add into the partial buffer, 0 = store
  const float* bias;
  DropKey drop;
  uint32_t* flags;
  float* colsum;    // EPI_ACT_BWD: column sums per 32-row group (null: none)
  int colsum_acc;
};

// Column sums of a warp's staged 32 x 32 bf16 chunk (64-byte rows, 64-byte
// swizzle: 16-byte chunk q of row r at q ^ ((r >> 1) & 3)): lane c adds
// column c over the 32 rows in order and writes (or adds) the group's partial.
__device__ __forceinline__ void chunk_colsum(const TcArgs& p, uint32_t buf, int lane, int row0, int col0) {
  if (row0 >= p.M) return;
  float s = 0.f;
#pragma unroll 8
  for (int r = 0; r < 32; r++) {
    const uint32_t addr = buf + r * 64 + ((((lane >> 3) ^ ((r >> 1) & 3))) << 4) + (lane & 7) * 2;
    unsigned short u;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(u) : "r"(addr));
    s += __bfloat162float(__ushort_as_bfloat16(u));
  }
  const int col = col0 + lane;
  if (col < p.N) {
    float* dst = p.colsum + (size_t)(row0 >> 5) * p.N + col;
    *dst = p.colsum_acc ? *dst + s : s;
  }
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

// Staging tiles hold 32 rows x 32 columns; row r belongs to lane r.
// fp32 rows are 128 bytes (TMA 128-byte swizzle: 16-byte chunk q of row r at
// q ^ (r & 7)); bf16 rows are 64 bytes (64-byte swizzle: chunk q at
// q ^ ((r >> 1) & 3)).  Both keep a warp's 16-byte accesses conflict-free.
// The epilogue works on half-rows of 16 columns (h = 0, 1) to keep its
// register footprint small.
__device__ __forceinline__ void stage_f32(uint32_t buf, int r, int h, const float (&x)[16]) {
#pragma unroll
  for (int qq = 0; qq < 4; qq++)
    st_shared_v4(buf + r * 128 + (((4 * h + qq) ^ (r & 7)) << 4), __float_as_uint(x[4 * qq]),
                 __float_as_uint(x[4 * qq + 1]), __float_as_uint(x[4 * qq + 2]), __float_as_uint(x[4 * qq + 3]));
}
__device__ __forceinline__ void unstage_f32(uint32_t buf, int r, int h, float (&x)[16]) {
#pragma unroll
  for (int qq = 0; qq < 4; qq++) {
    uint4 u = ld_shared_v4(buf + r * 128 + (((4 * h + qq) ^ (r & 7)) << 4));
    x[4 * qq] = __uint_as_float(u.x);
    x[4 * qq + 1] = __uint_as_float(u.y);
    x[4 * qq + 2] = __uint_as_float(u.z);
    x[4 * qq + 3] = __uint_as_float(u.w);
  }
}
__device__ __forceinline__ void stage_bf16(uint32_t buf, int r, int h, const float (&x)[16]) {
#pragma unroll
  for (int qq = 0; qq < 2; qq++)
    st_shared_v4(buf + r * 64 + (((2 * h + qq) ^ ((r >> 1) & 3)) << 4), pack_bf16(x[8 * qq], x[8 * qq + 1]),
                 pack_bf16(x[8 * qq + 2], x[8 * qq + 3]), pack_bf16(x[8 * qq + 4], x[8 * qq + 5]),
                 pack_bf16(x[8 * qq + 6], x[8 * qq + 7]));
}
__device__ __forceinline__ void unstage_bf16(uint32_t buf, int r, int h, float (&x)[16]) {
#pragma unroll
  for (int qq = 0; qq < 2; qq++) {
    uint4 u = ld_shared_v4(buf + r * 64 + (((2 * h + qq) ^ ((r >> 1) & 3)) << 4));
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
      float2 f = unpack_bf16(w[k]);
      x[8 * qq + 2 * k] = f.x;
      x[8 * qq + 2 * k + 1] = f.y;
    }
  }
}

// Row r of a bf16 staging tile as 16 packed pairs: word k holds columns 2k
// and 2k + 1.
__device__ __forceinline__ void load_row_bf16(uint32_t buf, int r, uint32_t (&w)[16]) {
#pragma unroll
  for (int q = 0; q < 4; q++) {
    const uint4 u = ld_shared_v4(buf + r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
    w[4 * q] = u.x;
    w[4 * q + 1] = u.y;
    w[4 * q + 2] = u.z;
    w[4 * q + 3] = u.w;
  }
}

// The 16 bias values of a half-row, loaded before the TMEM wait so that their
// latency overlaps it (zeros past N).
__device__ __forceinline__ void load_bias(const TcArgs& p, int col0, float4 (&b)[4]) {
  if (col0 + 16 <= p.N) {
    const float4* b4 = reinterpret_cast<const float4*>(p.bias + col0);
#pragma unroll
    for (int i = 0; i < 4; i++) b[i] = b4[i];
  } else {
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int c = col0 + 4 * i;
      b[i] = make_float4(c < p.N ? p.bias[c] : 0.f, c + 1 < p.N ? p.bias[c + 1] : 0.f,
                         c + 2 < p.N ? p.bias[c + 2] : 0.f, c + 3 < p.N ? p.bias[c + 3] : 0.f);
    }
  }
}
__device__ __forceinline__ void add_bias(const float4 (&b)[4], float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; i++) {
    v[4 * i] += b[i].x;
    v[4 * i + 1] += b[i].y;
    v[4 * i + 2] += b[i].z;
    v[4 * i + 3] += b[i].w;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D tensor map: `inner` contiguous elements per row, `outer` rows, row
// pitch `ld` elements; box = box_inner x box_outer.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner, uint64_t outer,
              uint64_t ld, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * esize};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_out_map(CUtensorMap* m, bool f32, const void* base, int M, int N, long ld) {
  return f32 ? make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, N, M, ld, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B)
             : make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, N, M, ld, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

// split-K partials [splits, M, N] fp32 as a 3-D map so boxes clip per split
bool make_partial_map(CUtensorMap* m, const void* base, int M, int N, int splits) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)M, (cuuint64_t)splits};
  cuuint64_t strides[2] = {(cuuint64_t)N * 4, (cuuint64_t)M * N * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace gpt
