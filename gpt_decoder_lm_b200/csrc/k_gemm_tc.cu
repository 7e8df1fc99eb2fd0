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
//   warps 2..17 epilogue: four warps per TMEM lane quadrant, each taking a
//               quarter of the BN columns in 32x32 chunks (processed as two
//               16-column halves): tcgen05.ld -> fused element-wise work ->
//               swizzled shared-memory staging tile -> TMA tensor store (or
//               TMA reduce-add for gradient accumulation).  Inputs the
//               epilogue needs (the residual stream, the saved
//               pre-activation) arrive by TMA into the same staging tiles,
//               the first one while the tile's MMAs still run, so every
//               global access of the epilogue is a coalesced bulk transfer.
// TMEM holds two BN-column accumulators so the epilogue of tile i overlaps
// the MMAs of tile i+1.  Every mbarrier wait is bounded.
#include "gemm_tc_common.cuh"

namespace gpt {
namespace {

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 3 : 5;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES;
  static constexpr int BAR_OFF = EPI_OFF + EPI_WARPS * EPI_BUF;
  static constexpr int SMEM_BYTES = BAR_OFF + 512 + 1024;  // + barriers + alignment slack
};


template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
              const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_out2,
              const __grid_constant__ CUtensorMap tm_in, TcArgs p) {
  using C = TcCfg<BN>;
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* ebar = tempty + 2;  // [EPI_WARPS] staging-tile loads
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ebar + EPI_WARPS);
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
      mbar_init(smem_u32(&tempty[b]), EPI_WARPS);  // one arrival per epilogue warp
    }
    for (int w = 0; w < EPI_WARPS; w++) mbar_init(smem_u32(&ebar[w]), 1);
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
  // the set-up above overlaps the previous kernel's tail; its outputs (our
  // operands, epilogue inputs, the buffers we write) are ready from here on
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        int split = t / (p.num_m * p.num_n);
        int r = t % (p.num_m * p.num_n);
        int mb = p.n_fast ? r / p.num_n : r % p.num_m, nb = p.n_fast ? r % p.num_n : r / p.num_m;
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
    const int ew = warp - 2;          // 0 .. EPI_WARPS-1
    const int quad = warp & 3;        // TMEM lanes quad*32 .. quad*32+31
    const int part = ew >> 2;         // which of the EPI_PARTS column ranges
    constexpr int CPW = BN / 32 / EPI_PARTS;  // 32-column chunks per warp and tile
    // one 4 KB staging set per warp: one fp32 tile, or two bf16 tiles (A at
    // +0, B at +2 KB)
    const uint32_t stg = smem_u32(smem + C::EPI_OFF + ew * EPI_BUF);
    const uint32_t lbar = smem_u32(&ebar[ew]);
    uint32_t lphase = 0;
    const int kind = p.kind;
    const bool f32_in = kind == EPI_RESADD, bf16_in = kind == EPI_ACT_BWD;
    const bool has_bias = p.bias && p.splits == 1 && kind != EPI_ACT_BWD && kind < EPI_ACC_F32;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      int split = t / (p.num_m * p.num_n);
      int r = t % (p.num_m * p.num_n);
      int mb = p.n_fast ? r / p.num_n : r % p.num_m, nb = p.n_fast ? r % p.num_n : r / p.num_m;
      const int row0 = mb * BM + quad * 32;
      const long row = row0 + lane;
      const int c_first = part * CPW;
      // the epilogue input of a warp's first chunk (residual stream or saved
      // pre-activation) is fetched while the tile's MMAs still run
      auto fetch_input = [&](int c) {
        if (lane == 0) {
          bulk_wait_read0();  // the previous chunk's stores have read the staging set
          mbar_expect_tx(lbar, f32_in ? 4096 : 2048);
          tma_load_2d(f32_in ? stg : stg + 2048, &tm_in, lbar, nb * BN + c * 32, row0);
        }
        __syncwarp();
      };
      if (f32_in || bf16_in) fetch_input(c_first);
      if (!(ok = mbar_wait(smem_u32(&tfull[acc]), acc_phase, abort_flag, p.flags))) {
        if (f32_in || bf16_in) mbar_wait(lbar, lphase, abort_flag, p.flags);  // no load left in flight
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int c = c_first; c < c_first + CPW; c++) {
        const int col0 = nb * BN + c * 32;
        const uint32_t bufA = stg, bufB = stg + 2048;
        if (f32_in || bf16_in) {
          if (c > c_first) fetch_input(c);
          if (!mbar_wait(lbar, lphase, abort_flag, p.flags)) {
            ok = false;
            break;
          }
          lphase ^= 1;
        } else {
          if (lane == 0) bulk_wait_read0();  // the previous chunk's stores have read the staging set
          __syncwarp();
        }
#pragma unroll
        for (int hh = 0; hh < 2; hh++) {
          float4 bias[4];
          if (has_bias) load_bias(p, col0 + 16 * hh, bias);
          uint32_t raw[16];
          tmem_ld_32x32b_x16(tbase + c * 32 + 16 * hh, raw);
          tmem_ld_wait();
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; i++) v[i] = __uint_as_float(raw[i]);
          if (p.splits > 1) {
            stage_f32(bufA, lane, hh, v);
          } else {
            switch (kind) {
              case EPI_STORE:
              case EPI_BIAS:
                if (has_bias) add_bias(bias, v);
                stage_bf16(bufA, lane, hh, v);
                break;
              case EPI_BIAS_ACT: {
                if (has_bias) add_bias(bias, v);
                float dv[16];  // act'(h), kept for the backward pass
                if (p.act == ACT_GELU) {
#pragma unroll
                  for (int i = 0; i < 16; i += 2) gelu_and_grad2(v[i], v[i + 1], dv[i], dv[i + 1]);
                } else {
#pragma unroll
                  for (int i = 0; i < 16; i++) {
                    dv[i] = act_grad(p.act, v[i]);
                    v[i] = act_fwd(p.act, v[i]);
                  }
                }
                stage_bf16(bufA, lane, hh, dv);
                stage_bf16(bufB, lane, hh, v);
                break;
              }
              case EPI_ACT_BWD: {
                float dv[16];  // the saved act'(h)
                unstage_bf16(bufB, lane, hh, dv);
#pragma unroll
                for (int i = 0; i < 16; i++) v[i] *= dv[i];
                stage_bf16(bufA, lane, hh, v);
                break;
              }
              case EPI_RESADD: {
                float x[16];
                unstage_f32(bufA, lane, hh, x);
                if (has_bias) add_bias(bias, v);
                if (p.drop.active) {
                  const uint64_t el = (uint64_t)row * p.N + col0 + 16 * hh;
                  const DropKey dk = drop_live(p.drop);
#pragma unroll
                  for (int i = 0; i < 16; i++) v[i] *= drop_mul(dk, el + i);
                }
#pragma unroll
                for (int i = 0; i < 16; i++) v[i] += x[i];
                stage_f32(bufA, lane, hh, v);
                break;
              }
              default:  // EPI_ACC_F32, EPI_STORE_F32
                stage_f32(bufA, lane, hh, v);
                break;
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (kind == EPI_ACT_BWD && p.colsum && p.splits == 1) chunk_colsum(p, bufA, lane, row0, col0);
        if (lane == 0) {
          if (p.splits > 1) {
            if (p.acc_partial) tma_reduce_add_3d(&tm_out, bufA, col0, row0, split);
            else tma_store_3d(&tm_out, bufA, col0, row0, split);
          }
          else if (kind == EPI_ACC_F32) tma_reduce_add_2d(&tm_out, bufA, col0, row0);
          else tma_store_2d(&tm_out, bufA, col0, row0);
          if (kind == EPI_BIAS_ACT && p.splits == 1) tma_store_2d(&tm_out2, bufB, col0, row0);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) bulk_wait0();  // every store of this warp has landed
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ---------------------------------------------------------------- host side

template <int BN, bool A_MN, bool B_MN>
bool launch(Ctx& c, const GemmDesc& g, int splits) {
  using Cf = TcCfg<BN>;
  const GemmEpi& e = g.epi;
  CUtensorMap ma, mb, mo, mo2, mi;
  bool ok = true;
  constexpr auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  constexpr auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!A_MN) ok &= make_map(&ma, BF, 2, g.A, g.K, g.M, g.lda, BK, BM, SW);
  else ok &= make_map(&ma, BF, 2, g.A, g.M, g.K, g.lda, 64, BK, SW);
  if (!B_MN) ok &= make_map(&mb, BF, 2, g.B, g.K, g.N, g.ldb, BK, BN, SW);
  else ok &= make_map(&mb, BF, 2, g.B, g.N, g.K, g.ldb, 64, BK, SW);
  mo2 = mb;  // unused unless EPI_BIAS_ACT
  mi = mb;   // unused unless the epilogue reads an input tile
  if (splits > 1) {
    ok &= make_partial_map(&mo, g.partial, g.M, g.N, splits);
  } else {
    switch (e.kind) {
      case EPI_STORE:
      case EPI_BIAS:
        ok &= make_out_map(&mo, false, e.out, g.M, g.N, e.ldo);
        break;
      case EPI_BIAS_ACT:
        ok &= make_out_map(&mo, false, e.out, g.M, g.N, e.ldo);
        ok &= make_out_map(&mo2, false, e.out2, g.M, g.N, e.ldo);
        break;
      case EPI_ACT_BWD:
        ok &= make_out_map(&mo, false, e.out, g.M, g.N, e.ldo);
        ok &= make_out_map(&mi, false, e.aux, g.M, g.N, e.ldo);
        break;
      case EPI_RESADD:
        ok &= make_out_map(&mo, true, e.res_out, g.M, g.N, e.ld_res);
        ok &= make_out_map(&mi, true, e.res_in, g.M, g.N, e.ld_res);
        break;
      default:
        ok &= make_out_map(&mo, true, e.out, g.M, g.N, e.ldo);
        break;
    }
  }
  if (!ok) return false;
  TcArgs a;
  a.M = g.M;
  a.N = g.N;
  a.K = g.K;
  a.num_m = (g.M + BM - 1) / BM;
  a.num_n = (g.N + BN - 1) / BN;
  a.n_fast = g.M > g.N ? 1 : 0;  // reuse the larger operand across neighbouring tiles
  a.nkb = (g.K + BK - 1) / BK;
  a.splits = splits;
  a.kb_per_split = (a.nkb + splits - 1) / splits;
  a.kind = e.kind;
  a.act = e.act;
  a.acc_partial = g.partial_accumulate ? 1 : 0;
  a.bias = e.bias;
  a.drop = e.drop;
  a.flags = c.flags;
  a.colsum = (e.kind == EPI_ACT_BWD && splits == 1) ? e.colsum : nullptr;
  a.colsum_acc = e.colsum_acc ? 1 : 0;
  int tiles = a.num_m * a.num_n * splits;
  int grid = tiles < c.num_sms ? tiles : c.num_sms;
  // per-device function attribute: set before every launch
  cudaFuncSetAttribute(k_gemm_tc<BN, A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM_BYTES);
  LaunchScope s(c, g.name ? g.name : "gemm_tc");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cf::SMEM_BYTES;
  cfg.stream = c.stream;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k_gemm_tc<BN, A_MN, B_MN>, ma, mb, mo, mo2, mi, a) != cudaSuccess) {
    cudaGetLastError();  // programmatic serialization refused: an ordinary launch
    k_gemm_tc<BN, A_MN, B_MN><<<grid, kThreads, Cf::SMEM_BYTES, c.stream>>>(ma, mb, mo, mo2, mi, a);
  }
  return true;
}

}  // namespace

// Kernel, tile width and split-K count from a simple cost model: MMA cycles
// per work unit (k-blocks x cycles per k-block; 128-wide tiles pay for their
// lower operand reuse, pair tiles gain from each SM loading half of B), whole
// waves over the SMs (pairs of SMs for the pair kernel), and the traffic of
// split-K partials (written and read back once).
constexpr double KB_CYCLES_256 = 512.0, KB_CYCLES_128 = 330.0, KB_CYCLES_PAIR = 470.0;
TcPlan gemm_tc_plan(long M, long N, long K, bool split_ok, int num_sms, int mode) {
  TcPlan best{256, 1, 0};
  double best_t = 1e30;
  long nkb = (K + BK - 1) / BK;
  for (int pair = 0; pair < 2; pair++) {
    if ((mode == TC_SINGLE && pair) || (mode == TC_PAIR && !pair)) continue;
    if (mode == TC_ANY && pair && M < 256) continue;
    const int slots = pair ? num_sms / 2 : num_sms;
    for (int bn : {256, 128}) {
      if (pair && bn != 256) continue;
      if (!pair && bn == 256 && N <= 128) continue;
      long tiles = ((M + (pair ? 2 * BM : BM) - 1) / (pair ? 2 * BM : BM)) * ((N + bn - 1) / bn);
      for (int s = 1; s <= 16; s++) {
        if (s > 1 && (!split_ok || s > nkb / 8)) break;
        long units = tiles * s;
        long waves = (units + slots - 1) / slots;
        const double kbc = pair ? KB_CYCLES_PAIR : (bn == 256 ? KB_CYCLES_256 : KB_CYCLES_128);
        double per_unit = (double)((nkb + s - 1) / s) * kbc + bn * 12.0;
        double t = waves * per_unit;
        if (s > 1) t += 2.0 * s * M * N * 4 / (num_sms * 96.0);
        if (t < best_t * 0.98) {
          best_t = t;
          best = TcPlan{bn, s, pair};
        }
      }
    }
  }
  return best;
}

bool gemm_tc_supported(const GemmDesc& g) {
  if (!get_encode()) return false;
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return false;
  if ((g.lda % 8) || (g.ldb % 8)) return false;  // 16-byte row pitch for TMA
  if ((reinterpret_cast<uintptr_t>(g.A) & 15) || (reinterpret_cast<uintptr_t>(g.B) & 15)) return false;
  if (!g.a_kmajor && (g.M % 8)) return false;  // MN-major inner extent: 16-byte multiple
  if (!g.b_kmajor && (g.N % 8)) return false;
  if (g.a_kmajor && (g.K % 8)) return false;
  if (g.b_kmajor && (g.K % 8)) return false;
  if (g.N % 4) return false;  // fp32 output rows: 16-byte multiple
  const GemmEpi& e = g.epi;
  if (e.kind == EPI_RESADD) {
    if (e.ld_res % 4 || (reinterpret_cast<uintptr_t>(e.res_in) & 15) || (reinterpret_cast<uintptr_t>(e.res_out) & 15))
      return false;
  } else {
    if (e.ldo % 8 || (reinterpret_cast<uintptr_t>(e.out) & 15)) return false;
  }
  if (e.kind == EPI_BIAS_ACT && (reinterpret_cast<uintptr_t>(e.out2) & 15)) return false;
  if (e.kind == EPI_ACT_BWD && (reinterpret_cast<uintptr_t>(e.aux) & 15)) return false;
  if (e.bias && (reinterpret_cast<uintptr_t>(e.bias) & 15)) return false;
  if (!(g.a_kmajor && g.b_kmajor) && !(g.a_kmajor && !g.b_kmajor) && !(!g.a_kmajor && !g.b_kmajor)) return false;
  return true;
}

int gemm_tc_splits(const GemmDesc& g, int num_sms, int mode) {
  bool split_ok = g.epi.kind == EPI_ACC_F32 && g.partial && g.split_k > 1;
  TcPlan plan = gemm_tc_plan(g.M, g.N, g.K, split_ok, num_sms, mode);
  int splits = plan.splits;
  if (splits > g.split_k) splits = g.split_k < 1 ? 1 : g.split_k;  // never beyond the caller's scratch
  if (splits > 1) {  // keep every split non-empty
    int nkb = (g.K + BK - 1) / BK;
    int kbps = (nkb + splits - 1) / splits;
    splits = (nkb + kbps - 1) / kbps;
  }
  return splits;
}

bool gemm_tc_bf16(Ctx& c, const GemmDesc& g, int mode) {
  bool split_ok = g.epi.kind == EPI_ACC_F32 && g.partial && g.split_k > 1;
  TcPlan plan = gemm_tc_plan(g.M, g.N, g.K, split_ok, c.num_sms, mode);
  const int splits = gemm_tc_splits(g, c.num_sms, mode);
  bool amn = !g.a_kmajor, bmn = !g.b_kmajor;
  bool ok;
  if (plan.pair) {
    ok = gemm_tc2_launch(c, g, splits);
  } else if (plan.bn == 256) {
    if (!amn && !bmn) ok = launch<256, false, false>(c, g, splits);
    else if (!amn && bmn) ok = launch<256, false, true>(c, g, splits);
    else ok = launch<256, true, true>(c, g, splits);
  } else {
    if (!amn && !bmn) ok = launch<128, false, false>(c, g, splits);
    else if (!amn && bmn) ok = launch<128, false, true>(c, g, splits);
    else ok = launch<128, true, true>(c, g, splits);
  }
  if (!ok) return false;
  if (splits > 1 && g.reduce_partials)
    splitk_reduce(c, g.partial, splits, (long)g.M * g.N, reinterpret_cast<float*>(g.epi.out));
  return true;
}

}  // namespace gpt
