// Pair-CTA (cta_group::2) variant of the tcgen05 GEMM.  A 256 x BN tile per CTA pair: each CTA loads its own 128 rows
// of A and BN/2 rows of B, the even CTA issues M=256 MMAs that read both CTAs'
// shared memory, and each CTA's TMEM holds its 128 rows of the accumulator.
// No TMA multicast: every load writes the issuing CTA's own shared memory;
// the odd CTA's loads signal the even CTA's full barrier.
#include "gemm_tc_common.cuh"

namespace gpt {
namespace {

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma2_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the mbarrier at `bar` (a CTA-local offset) in every CTA of `mask`
// once the issuing thread's tcgen05 operations complete
__device__ __forceinline__ void mma2_commit(uint32_t bar, uint16_t mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::
                   "r"(bar), "h"(mask)
               : "memory");
}
// TMA load into this CTA's shared memory, completion counted on `bar`, which
// may be the peer CTA's barrier (a shared::cluster address)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}


template <int BN>
struct TcCfg {  // per CTA of the pair: 128 rows of A, BN/2 rows of B per stage
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = (BN / 2) * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 5;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int EPI_OFF = STAGES * STAGE_BYTES;
  static constexpr int BAR_OFF = EPI_OFF + EPI_WARPS * EPI_BUF;
  static constexpr int SMEM_BYTES = BAR_OFF + 512 + 1024;  // + barriers + alignment slack
};


template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_tc2(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
               const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_out2,
               const __grid_constant__ CUtensorMap tm_in, TcArgs p) {
  using C = TcCfg<BN>;
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the pair's shared-memory layouts must coincide: the MMA descriptors are
  // CTA-relative offsets used in both CTAs
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
  const uint32_t rank = cluster_rank();  // 0: issues the MMAs; 1: its peer
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int tiles = p.num_m * p.num_n * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; s++) {
      mbar_init(smem_u32(&full[s]), 1);   // even CTA: its producer's arrive + both CTAs' bytes
      mbar_init(smem_u32(&empty[s]), 1);  // the MMA commit, multicast to both CTAs
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 2 * EPI_WARPS);  // every epilogue warp of both CTAs
    }
    for (int w = 0; w < EPI_WARPS; w++) mbar_init(smem_u32(&ebar[w]), 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tma_a);
    prefetch_tmap(&tma_b);
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), C::TMEM_COLS);  // one warp of each CTA, collectively
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += npairs) {
        int split = t / (p.num_m * p.num_n);
        int r = t % (p.num_m * p.num_n);
        int mb = p.n_fast ? r / p.num_n : r % p.num_m, nb = p.n_fast ? r % p.num_n : r / p.num_m;
        int kb0 = split * p.kb_per_split, kb1 = min(p.nkb, kb0 + p.kb_per_split);
        const int arow = mb * (2 * BM) + (int)rank * BM;      // this CTA's 128 rows of A
        const int brow = nb * BN + (int)rank * (BN / 2);      // this CTA's BN/2 rows of B
        for (int kb = kb0; kb < kb1; kb++) {
          if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1, abort_flag, p.flags)) {
            ok = false;
            break;
          }
          // both CTAs' loads complete on the even CTA's full barrier: the
          // cta_group::2 form takes the local barrier address with the peer
          // bit (bit 24) cleared, as CUTLASS's 2-SM TMA copy does
          const uint32_t fb = smem_u32(&full[stage]) & 0xFEFFFFFFu;
          if (rank == 0) mbar_expect_tx(smem_u32(&full[stage]), 2 * C::STAGE_BYTES);
          uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
          uint32_t sb = sa + C::A_BYTES;
          int k = kb * BK;
          if (!A_MN) {
            tma_load_2d_pair(sa, &tma_a, fb, k, arow);
          } else {
            tma_load_2d_pair(sa, &tma_a, fb, arow, k);
            tma_load_2d_pair(sa + 8192, &tma_a, fb, arow + 64, k);
          }
          if (!B_MN) {
            tma_load_2d_pair(sb, &tma_b, fb, k, brow);
          } else {
#pragma unroll
            for (int q = 0; q < BN / 128; q++) tma_load_2d_pair(sb + q * 8192, &tma_b, fb, brow + q * 64, k);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && rank == 0) {
        for (int s = 0; s < C::STAGES; s++) mbar_wait(smem_u32(&full[s]), phase, abort_flag, p.flags);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA only)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += npairs) {
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
            mma2_bf16_ss(d_tmem, ad, bd, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          mma2_commit(smem_u32(&empty[stage]), 0x3);  // frees the stage in both CTAs
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma2_commit(smem_u32(&tfull[acc]), 0x3);  // both CTAs' epilogues
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok || *abort_flag) {
        mma2_commit(smem_u32(&tfull[acc]), 0x1);
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
    // (the split-K planner splits only EPI_ACC_F32 products)
    const bool f32_in = kind == EPI_RESADD && p.splits == 1, bf16_in = kind == EPI_ACT_BWD && p.splits == 1;
    const bool has_bias = p.bias && p.splits == 1 && kind != EPI_ACT_BWD && kind < EPI_ACC_F32;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = pair; t < tiles && ok; t += npairs) {
      int split = t / (p.num_m * p.num_n);
      int r = t % (p.num_m * p.num_n);
      int mb = p.n_fast ? r / p.num_n : r % p.num_m, nb = p.n_fast ? r % p.num_n : r / p.num_m;
      const int row0 = mb * (2 * BM) + (int)rank * BM + quad * 32;
      const long row = row0 + lane;
      const int c_first = part * CPW;
      // the epilogue input of a warp's first chunk (residual stream or saved
      // act'(h)) is fetched while the tile's MMAs still run
      auto fetch_input = [&](int c) {
        if (lane == 0) {
          // the fp32 input shares its buffer with the output: the previous
          // chunk's stores must have read it (the bf16 input has its own half)
          if (f32_in) bulk_wait_read0();
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
          if (f32_in && c > c_first) fetch_input(c);
          if (!mbar_wait(lbar, lphase, abort_flag, p.flags)) {
            ok = false;
            break;
          }
          lphase ^= 1;
        }
        if (bf16_in) {
          // EPI_ACT_BWD: the chunk's act'(h) into registers, so that the next
          // chunk's can be fetched into the buffer while this one is computed
          // and stored
          uint32_t aux[16];
          load_row_bf16(bufB, lane, aux);
          if (c + 1 < c_first + CPW) {
            fence_proxy_async_smem();
            __syncwarp();
            fetch_input(c + 1);
          }
#pragma unroll
          for (int q = 0; q < 4; q++) {  // 8 columns at a time: aux holds 16 registers
            uint32_t raw[8];
            tmem_ld_32x32b_x8(tbase + c * 32 + 8 * q, raw);
            tmem_ld_wait();
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
              const float2 d = unpack_bf16(aux[4 * q + k]);
              w[k] = pack_bf16(__uint_as_float(raw[2 * k]) * d.x, __uint_as_float(raw[2 * k + 1]) * d.y);
            }
            if (q == 0) {  // the previous chunk's stores have read the output half
              if (lane == 0) bulk_wait_read0();
              __syncwarp();
            }
            st_shared_v4(bufA + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4), w[0], w[1], w[2], w[3]);
          }
        } else {
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
            // before the first write of a chunk's outputs: the previous
            // chunk's stores have read the staging set (the fp32-input kind
            // waited before its fetch)
            auto staging_free = [&]() {
              if (hh == 0 && !f32_in) {
                if (lane == 0) bulk_wait_read0();
                __syncwarp();
              }
            };
            if (p.splits > 1) {
              staging_free();
              stage_f32(bufA, lane, hh, v);
            } else {
              switch (kind) {
                case EPI_STORE:
                case EPI_BIAS:
                  if (has_bias) add_bias(bias, v);
                  staging_free();
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
                  staging_free();
                  stage_bf16(bufA, lane, hh, dv);
                  stage_bf16(bufB, lane, hh, v);
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
                  staging_free();
                  stage_f32(bufA, lane, hh, v);
                  break;
              }
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
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));  // the even CTA's barrier
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) bulk_wait0();  // every store of this warp has landed
  }
  tc_fence_before();
  cluster_sync();  // both CTAs are done with TMEM and with each other's barriers
  tc_fence_after();
  if (warp == 1) tmem_dealloc2(tmem_base, C::TMEM_COLS);
}

// ---------------------------------------------------------------- host side

template <int BN, bool A_MN, bool B_MN>
bool launch2(Ctx& c, const GemmDesc& g, int splits) {
  using Cf = TcCfg<BN>;
  const GemmEpi& e = g.epi;
  CUtensorMap ma, mb, mo, mo2, mi;
  bool ok = true;
  constexpr auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  constexpr auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!A_MN) ok &= make_map(&ma, BF, 2, g.A, g.K, g.M, g.lda, BK, BM, SW);
  else ok &= make_map(&ma, BF, 2, g.A, g.M, g.K, g.lda, 64, BK, SW);
  if (!B_MN) ok &= make_map(&mb, BF, 2, g.B, g.K, g.N, g.ldb, BK, BN / 2, SW);  // half of B per CTA
  else ok &= make_map(&mb, BF, 2, g.B, g.N, g.K, g.ldb, 64, BK, SW);
  mo2 = mb;
  mi = mb;
  if (splits > 1) {
    ok &= make_partial_map(&mo, g.partial, g.M, g.N, splits);
  } else {
    switch (e.kind) {
      case EPI_STORE:
      case EPI_BIAS: ok &= make_out_map(&mo, false, e.out, g.M, g.N, e.ldo); break;
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
      default: ok &= make_out_map(&mo, true, e.out, g.M, g.N, e.ldo); break;
    }
  }
  if (!ok) return false;
  TcArgs a;
  a.M = g.M;
  a.N = g.N;
  a.K = g.K;
  a.num_m = (g.M + 2 * BM - 1) / (2 * BM);  // 256-row pair tiles
  a.num_n = (g.N + BN - 1) / BN;
  a.n_fast = g.M > g.N ? 1 : 0;
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
  const int tiles = a.num_m * a.num_n * splits;
  // per-device function attribute: set before every launch
  cudaFuncSetAttribute(k_gemm_tc2<BN, A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM_BYTES);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cf::SMEM_BYTES;
  cfg.stream = c.stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  // persistent: as many pairs as can be resident at once, at most one per tile
  int pairs = 0;
  cfg.gridDim = dim3(2 * tiles);
  if (cudaOccupancyMaxActiveClusters(&pairs, k_gemm_tc2<BN, A_MN, B_MN>, &cfg) != cudaSuccess || pairs < 1) {
    cudaGetLastError();
    pairs = c.num_sms / 2;
  }
  if (pairs > tiles) pairs = tiles;
  cfg.gridDim = dim3(2 * pairs);
  cfg.numAttrs = 2;
  LaunchScope s(c, g.name ? g.name : "gemm_tc2");
  if (cudaLaunchKernelEx(&cfg, k_gemm_tc2<BN, A_MN, B_MN>, ma, mb, mo, mo2, mi, a) != cudaSuccess) {
    cudaGetLastError();
    cfg.numAttrs = 1;  // without programmatic serialization
    if (cudaLaunchKernelEx(&cfg, k_gemm_tc2<BN, A_MN, B_MN>, ma, mb, mo, mo2, mi, a) != cudaSuccess) return false;
  }
  return true;
}

}  // namespace

// launch only: the caller (gemm_tc_bf16) reduces split partials
bool gemm_tc2_launch(Ctx& c, const GemmDesc& g, int splits) {
  const bool amn = !g.a_kmajor, bmn = !g.b_kmajor;
  if (!amn && !bmn) return launch2<256, false, false>(c, g, splits);
  if (!amn && bmn) return launch2<256, false, true>(c, g, splits);
  return launch2<256, true, true>(c, g, splits);
}

}  // namespace gpt
