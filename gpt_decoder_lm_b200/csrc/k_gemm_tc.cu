// bf16 GEMM on the sm_100a tensor cores: D[m, n] = sum_k A[m, k] B[n, k]
// with fp32 accumulation in TMEM and the fused epilogues of the training
// step (bias, bias + GELU/ReLU, bias + dropout + residual add, activation
// backward, fp32 gradient accumulation, split-K partials).
//
// Persistent, warp-specialised kernel, one CTA per SM:
//   warp 0      TMA producer: 128x64 A tile + BNx64 B tile per pipeline stage
//               (128-byte swizzle; K-major or MN-major operands, so dX and dW
//               need no transposed copies)
//   warp 1      TMEM allocator + MMA issuer (tcgen05.mma, M=128, N=BN, K=16)
//   warps 2..9  epilogue: tcgen05.ld of the 128 x BN fp32 tile, one row and
//               half of the columns per thread, fused element-wise work
// TMEM holds two BN-column accumulators so the epilogue of tile i overlaps
// the MMAs of tile i+1.  Every mbarrier wait is bounded.
#include <cudaTypedefs.h>

#include <mutex>

#include "epilogue.cuh"
#include "sm100.cuh"

namespace gpt {
namespace {

using namespace sm100;

constexpr int BM = 128, BK = 64;
constexpr int kThreads = 320;   // producer, MMA, 8 epilogue warps (2 per TMEM lane quadrant)

struct TcArgs {
  int M, N, K;
  int num_m, num_n, splits, kb_per_split, nkb;
  GemmEpi epi;
  float* partial;
  uint32_t* flags;
};

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;  // + barriers + alignment slack
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

// Epilogue of one 32-column chunk of one row.
__device__ __forceinline__ void epi_chunk(const TcArgs& p, long row, int col0, int split, const uint32_t (&r)[32]) {
  if (row >= p.M || col0 >= p.N) return;
  const GemmEpi& e = p.epi;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
  if (p.splits > 1) {  // split-K partial of an fp32 accumulation
    float* dst = p.partial + ((long)split * p.M + row) * p.N + col0;
    if (col0 + 32 <= p.N) {
#pragma unroll
      for (int i = 0; i < 8; i++) reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
      const int n = p.N - col0;
#pragma unroll
      for (int i = 0; i < 32; i++)  // static indices keep v[] in registers
        if (i < n) dst[i] = v[i];
    }
    return;
  }
  if (col0 + 32 > p.N) {  // ragged right edge: scalar path
    const int n = p.N - col0;
#pragma unroll
    for (int i = 0; i < 32; i++)
      if (i < n) epi_apply<bf16>(e, p.N, row, col0 + i, v[i]);
    return;
  }
  switch (e.kind) {
    case EPI_STORE:
    case EPI_BIAS:
    case EPI_BIAS_ACT: {
      if (e.bias) {
        const float4* b4 = reinterpret_cast<const float4*>(e.bias + col0);
#pragma unroll
        for (int i = 0; i < 8; i++) {
          float4 b = b4[i];
          v[4 * i] += b.x;
          v[4 * i + 1] += b.y;
          v[4 * i + 2] += b.z;
          v[4 * i + 3] += b.w;
        }
      }
      uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(e.out) + row * e.ldo + col0);
#pragma unroll
      for (int i = 0; i < 4; i++)
        o[i] = make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                          pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
      if (e.kind == EPI_BIAS_ACT) {
#pragma unroll
        for (int i = 0; i < 32; i++) v[i] = act_fwd(e.act, v[i]);
        uint4* o2 = reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(e.out2) + row * e.ldo + col0);
#pragma unroll
        for (int i = 0; i < 4; i++)
          o2[i] = make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                             pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
      }
      break;
    }
    case EPI_RESADD: {
      const float4* ri = reinterpret_cast<const float4*>(e.res_in + row * e.ld_res + col0);
      float4* ro = reinterpret_cast<float4*>(e.res_out + row * e.ld_res + col0);
      const float4* b4 = e.bias ? reinterpret_cast<const float4*>(e.bias + col0) : nullptr;
#pragma unroll
      for (int i = 0; i < 8; i++) {
        float4 x = ri[i];
        float4 b = b4 ? b4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        float y0 = v[4 * i] + b.x, y1 = v[4 * i + 1] + b.y, y2 = v[4 * i + 2] + b.z, y3 = v[4 * i + 3] + b.w;
        if (e.drop.active) {
          uint64_t el = (uint64_t)row * p.N + col0 + 4 * i;
          y0 *= drop_mul(e.drop, el);
          y1 *= drop_mul(e.drop, el + 1);
          y2 *= drop_mul(e.drop, el + 2);
          y3 *= drop_mul(e.drop, el + 3);
        }
        ro[i] = make_float4(x.x + y0, x.y + y1, x.z + y2, x.w + y3);
      }
      break;
    }
    case EPI_ACT_BWD: {
      const uint4* h4 = reinterpret_cast<const uint4*>(reinterpret_cast<const bf16*>(e.aux) + row * e.ldo + col0);
      uint4* o = reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(e.out) + row * e.ldo + col0);
#pragma unroll
      for (int i = 0; i < 4; i++) {
        uint4 hv = h4[i];
        uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
        uint32_t ow[4];
#pragma unroll
        for (int q = 0; q < 4; q++) {
          float2 h = unpack_bf16(hw[q]);
          ow[q] = pack_bf16(v[8 * i + 2 * q] * act_grad(e.act, h.x), v[8 * i + 2 * q + 1] * act_grad(e.act, h.y));
        }
        o[i] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      }
      break;
    }
    case EPI_ACC_F32:
    case EPI_STORE_F32: {
      float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(e.out) + row * e.ldo + col0);
#pragma unroll
      for (int i = 0; i < 8; i++) {
        float4 a = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        if (e.kind == EPI_ACC_F32) {
          float4 old = o[i];
          a.x += old.x;
          a.y += old.y;
          a.z += old.z;
          a.w += old.w;
        }
        o[i] = a;
      }
      break;
    }
  }
}

template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b, TcArgs p) {
  using C = TcCfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = p.num_m * p.num_n * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; s++) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 8);  // one arrival per epilogue warp
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tma_a);
    prefetch_tmap(&tma_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        int split = t / (p.num_m * p.num_n);
        int r = t % (p.num_m * p.num_n);
        int mb = r % p.num_m, nb = r / p.num_m;
        int kb0 = split * p.kb_per_split, kb1 = min(p.nkb, kb0 + p.kb_per_split);
        for (int kb = kb0; kb < kb1; kb++) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, p.flags)) {
            ok = false;
            break;
          }
          uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, C::STAGE_BYTES);
          uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          uint32_t sb = sa + C::A_BYTES;
          int k = kb * BK;
          if (!A_MN) {
            tma_load_2d(sa, &tma_a, fb, k, mb * BM);
          } else {
            tma_load_2d(sa, &tma_a, fb, mb * BM, k);
            tma_load_2d(sa + 8192, &tma_a, fb, mb * BM + 64, k);
          }
          if (!B_MN) {
            tma_load_2d(sb, &tma_b, fb, k, nb * BN);
          } else {
#pragma unroll
            for (int q = 0; q < BN / 64; q++) tma_load_2d(sb + q * 8192, &tma_b, fb, nb * BN + q * 64, k);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // drain: wait (bounded) for the loads already issued to land
        for (int s = 0; s < C::STAGES; s++) mbar_wait(smem_u32(&full[s]), phase, abort_flag, p.flags);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        int split = t / (p.num_m * p.num_n);
        int kb0 = split * p.kb_per_split, kb1 = min(p.nkb, kb0 + p.kb_per_split);
        if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1, abort_flag, p.flags)) break;
        tc_fence_after();
        uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; kb++) {
          if (!mbar_wait(smem_u32(&full[stage]), phase, abort_flag, p.flags)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          uint32_t sb = sa + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; kk++) {
            uint64_t ad = A_MN ? desc_sw128(sa + kk * 2048, 8192, 1024) : desc_sw128(sa + kk * 32, 16, 1024);
            uint64_t bd = B_MN ? desc_sw128(sb + kk * 2048, 8192, 1024) : desc_sw128(sb + kk * 32, 16, 1024);
            mma_bf16_ss(d_tmem, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(&empty[stage]));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&tfull[acc]));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok || *abort_flag) {
        // let every issued MMA finish before TMEM is released
        mma_commit(smem_u32(&tfull[acc]));
        mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.flags);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;         // TMEM lanes quad*32 .. quad*32+31
    const int half = (warp - 2) >> 2;  // which half of the BN columns
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      int split = t / (p.num_m * p.num_n);
      int r = t % (p.num_m * p.num_n);
      int mb = r % p.num_m, nb = r / p.num_m;
      if (!mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.flags)) break;
      tc_fence_after();
      long row = (long)mb * BM + quad * 32 + lane;
      uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int c = half * (BN / 64); c < (half + 1) * (BN / 64); c++) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + c * 32, v);
        tmem_ld_wait();
        epi_chunk(p, row, nb * BN + c * 32, split, v);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ---------------------------------------------------------------- host side
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

// 2-D bf16 tensor map: `inner` contiguous elements per row, `outer` rows,
// row pitch `ld` elements; box = box_inner x box_outer, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld, uint32_t box_inner,
              uint32_t box_outer) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, bool A_MN, bool B_MN>
bool launch(Ctx& c, const GemmDesc& g, int splits) {
  using Cf = TcCfg<BN>;
  CUtensorMap ma, mb;
  bool ok = true;
  if (!A_MN) ok &= make_map(&ma, g.A, g.K, g.M, g.lda, BK, BM);
  else ok &= make_map(&ma, g.A, g.M, g.K, g.lda, 64, BK);
  if (!B_MN) ok &= make_map(&mb, g.B, g.K, g.N, g.ldb, BK, BN);
  else ok &= make_map(&mb, g.B, g.N, g.K, g.ldb, 64, BK);
  if (!ok) return false;
  TcArgs a;
  a.M = g.M;
  a.N = g.N;
  a.K = g.K;
  a.num_m = (g.M + BM - 1) / BM;
  a.num_n = (g.N + BN - 1) / BN;
  a.nkb = (g.K + BK - 1) / BK;
  a.splits = splits;
  a.kb_per_split = (a.nkb + splits - 1) / splits;
  a.epi = g.epi;
  a.partial = g.partial;
  a.flags = c.flags;
  int tiles = a.num_m * a.num_n * splits;
  int grid = tiles < c.num_sms ? tiles : c.num_sms;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(k_gemm_tc<BN, A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM_BYTES);
    attr = true;
  }
  LaunchScope s(c, "gemm_tc");
  k_gemm_tc<BN, A_MN, B_MN><<<grid, kThreads, Cf::SMEM_BYTES, c.stream>>>(ma, mb, a);
  return true;
}

}  // namespace

bool gemm_tc_supported(const GemmDesc& g) {
  if (!get_encode()) return false;
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return false;
  if ((g.lda % 8) || (g.ldb % 8)) return false;  // 16-byte row pitch for TMA
  if ((reinterpret_cast<uintptr_t>(g.A) & 15) || (reinterpret_cast<uintptr_t>(g.B) & 15)) return false;
  if (!g.a_kmajor && (g.M % 8)) return false;  // MN-major inner extent: 16-byte multiple
  if (!g.b_kmajor && (g.N % 8)) return false;
  if (g.a_kmajor && (g.K % 8)) return false;
  if (g.b_kmajor && (g.K % 8)) return false;
  // vector epilogue alignment
  if (g.epi.ldo % 8 || (g.epi.kind == EPI_RESADD && g.epi.ld_res % 4)) return false;
  if (!(g.a_kmajor && g.b_kmajor) && !(g.a_kmajor && !g.b_kmajor) && !(!g.a_kmajor && !g.b_kmajor)) return false;
  return true;
}

bool gemm_tc_bf16(Ctx& c, const GemmDesc& g) {
  int num_m = (g.M + BM - 1) / BM;
  int nkb = (g.K + BK - 1) / BK;
  bool wide = (long)num_m * ((g.N + 255) / 256) >= c.num_sms && g.N >= 256;
  int BNsel = wide ? 256 : 128;
  int splits = 1;
  if (g.epi.kind == EPI_ACC_F32 && g.partial && g.split_k > 1) {
    splits = g.split_k;
    if (splits > nkb) splits = nkb;
    // keep every split non-empty
    int kbps = (nkb + splits - 1) / splits;
    splits = (nkb + kbps - 1) / kbps;
  }
  bool amn = !g.a_kmajor, bmn = !g.b_kmajor;
  bool ok;
  if (BNsel == 256) {
    if (!amn && !bmn) ok = launch<256, false, false>(c, g, splits);
    else if (!amn && bmn) ok = launch<256, false, true>(c, g, splits);
    else ok = launch<256, true, true>(c, g, splits);
  } else {
    if (!amn && !bmn) ok = launch<128, false, false>(c, g, splits);
    else if (!amn && bmn) ok = launch<128, false, true>(c, g, splits);
    else ok = launch<128, true, true>(c, g, splits);
  }
  if (!ok) return false;
  if (splits > 1) splitk_reduce(c, g.partial, splits, (long)g.M * g.N, reinterpret_cast<float*>(g.epi.out));
  return true;
}

}  // namespace gpt
