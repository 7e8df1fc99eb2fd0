// Causal flash attention on the sm_100a tensor cores (tcgen05), head_dim 64,
// bf16 operands, fp32 softmax statistics, T a multiple of 128.
//
// Per (b, h): S = Q K^T / sqrt(64), key j > query i masked, P = softmax(S),
// O = drop(P) V, LSE = log-sum-exp of each row of S (kept for backward).
// Backward recomputes P from LSE:
//   D_i = sum_d dO_id O_id;  dP = drop(dO V^T);  dS = P * (dP - D)
//   dV = drop(P)^T dO;  dK = dS^T Q / sqrt(64);  dQ = dS K / sqrt(64)
// dK/dV and dQ come from two kernels (each output tile owned by one CTA, no
// atomics), so the result is deterministic.
//
// Every kernel: warp 0 issues TMA loads of 128-row bf16 tiles (128-byte
// swizzle) from the [B*T, 3, H, 64] qkv activations, warp 1 owns TMEM and
// issues tcgen05.mma, warps 2..5 (one TMEM lane / tile row per thread) do the
// softmax arithmetic, write bf16 probability tiles to shared memory as the
// A operand of the next MMA, and run the epilogue.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.cuh"
#include "sm100.cuh"

namespace gpt {
namespace {

using namespace sm100;

constexpr int TILE = 16384;                 // 128 rows x 64 bf16, 128-byte swizzle
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct AttnTcArgs {
  int B, T, H;
  const bf16* o;      // fwd output / bwd input O
  bf16* o_out;
  float* lse;         // [B, H, T] natural log
  const float* dsum;  // [B, H, T]
  bf16* dqkv;
  float scale_log2;   // log2(e) / sqrt(64)
  float scale;        // 1 / sqrt(64)
  DropKey drop;
  uint32_t* flags;
};

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Row r, 32-column chunk c (0..3) of a 128 x 128 K-major bf16 operand tile
// stored as two 64-wide K-blocks of 128 rows x 128 bytes (128-byte swizzle).
__device__ __forceinline__ void store_chunk32(uint32_t tile, int r, int c, const uint32_t (&pk)[16]) {
  uint32_t rowbase = tile + (c >> 1) * TILE + r * 128;
#pragma unroll
  for (int q = 0; q < 4; q++) {
    int chunk = (c & 1) * 4 + q;
    st_shared_v4(rowbase + ((chunk ^ (r & 7)) << 4), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  }
}

// A operand descriptor of K-step kk (16 elements) of such a 128-wide tile
__device__ __forceinline__ uint64_t desc_k128(uint32_t tile, int kk) {
  return desc_sw128(tile + (kk >> 2) * TILE + (kk & 3) * 32, 16, 1024);
}
// K-major 64-wide tile (Q, K, V, dO as [rows, hd]), K-step kk (0..3)
__device__ __forceinline__ uint64_t desc_k64(uint32_t tile, int kk) { return desc_sw128(tile + kk * 32, 16, 1024); }
// the same [rows, 64] tile read MN-major (N = the 64 columns, K = rows), K-step kk (0..7)
__device__ __forceinline__ uint64_t desc_mn64(uint32_t tile, int kk) { return desc_sw128(tile + kk * 2048, TILE, 1024); }

// ============================================================================
// forward
// smem: Q | K[2] | V[2] | P (2 K-blocks) | barriers   (112 KB + 128 B)
// TMEM: S cols [0,128), PV cols [128,192)  (256 allocated)
// ============================================================================
constexpr int F_Q = 0, F_K = TILE, F_V = 3 * TILE, F_P = 5 * TILE, F_BAR = 7 * TILE;
constexpr int F_SMEM = F_BAR + 128;

__global__ void __launch_bounds__(192, 2) k_attn_fwd_tc(const __grid_constant__ CUtensorMap tm, AttnTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {  // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(a.flags, FLAG_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + F_BAR);
  uint32_t q_full = smem_u32(bars + 0), kv_full0 = smem_u32(bars + 1), kv_empty0 = smem_u32(bars + 3);
  uint32_t s_full = smem_u32(bars + 5), p_full = smem_u32(bars + 6), pv_full = smem_u32(bars + 7);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const uint32_t sb = smem_u32(smem);

  const int nqb = a.T / 128;
  const int qb = nqb - 1 - (int)blockIdx.x;  // longest rows first
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int nkb = qb + 1;
  const int row0 = b * a.T;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(kv_full0, 1);
    mbar_init(kv_full0 + 8, 1);
    mbar_init(kv_empty0, 1);
    mbar_init(kv_empty0 + 8, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(pv_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(q_full, TILE);
      tma_load_3d(sb + F_Q, &tm, q_full, 0, h, row0 + qb * 128);
      for (int j = 0; j < nkb; j++) {
        int s = j & 1;
        if (!mbar_wait(kv_empty0 + 8 * s, ((j >> 1) & 1) ^ 1, abort_flag, a.flags)) break;
        mbar_expect_tx(kv_full0 + 8 * s, 2 * TILE);
        tma_load_3d(sb + F_K + s * TILE, &tm, kv_full0 + 8 * s, 0, a.H + h, row0 + j * 128);
        tma_load_3d(sb + F_V + s * TILE, &tm, kv_full0 + 8 * s, 0, 2 * a.H + h, row0 + j * 128);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_pv = idesc_bf16_f32(128, 64, false, true);
      bool ok = mbar_wait(q_full, 0, abort_flag, a.flags);
      for (int j = 0; j < nkb && ok; j++) {
        int s = j & 1;
        if (!(ok = mbar_wait(kv_full0 + 8 * s, (j >> 1) & 1, abort_flag, a.flags))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ss(tmem, desc_k64(sb + F_Q, kk), desc_k64(sb + F_K + s * TILE, kk), id_s, kk > 0);
        mma_commit(s_full);
        if (!(ok = mbar_wait(p_full, j & 1, abort_flag, a.flags))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; kk++)
          mma_bf16_ss(tmem + 128, desc_k128(sb + F_P, kk), desc_mn64(sb + F_V + s * TILE, kk), id_pv, kk > 0);
        mma_commit(pv_full);
        mma_commit(kv_empty0 + 8 * s);
      }
    }
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qi = qb * 128 + r;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    float m = -INFINITY, l = 0.f;
    float o[64];
#pragma unroll
    for (int i = 0; i < 64; i++) o[i] = 0.f;
    const uint64_t ebase = ((uint64_t)bh * a.T + qi) * a.T;
    bool ok = true;
    for (int j = 0; j < nkb; j++) {
      if (!(ok = mbar_wait(s_full, j & 1, abort_flag, a.flags))) break;
      tc_fence_after();
      const bool diag = (j == qb);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; c++) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(trow + c * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; i++) {
          int key = j * 128 + c * 32 + i;
          float s = __uint_as_float(v[i]) * a.scale_log2;
          if (!(diag && key > qi)) mx = fmaxf(mx, s);
        }
      }
      const float mn = fmaxf(m, mx);
      const float alpha = exp2f(m - mn);
      float ls = 0.f;
#pragma unroll
      for (int c = 0; c < 4; c++) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(trow + c * 32, v);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          int key = j * 128 + c * 32 + i;
          float p0 = (diag && key > qi) ? 0.f : exp2f(__uint_as_float(v[i]) * a.scale_log2 - mn);
          float p1 = (diag && key + 1 > qi) ? 0.f : exp2f(__uint_as_float(v[i + 1]) * a.scale_log2 - mn);
          ls += p0 + p1;
          if (a.drop.active) {
            p0 *= drop_mul(a.drop, ebase + key);
            p1 *= drop_mul(a.drop, ebase + key + 1);
          }
          pk[i >> 1] = pack2(p0, p1);
        }
        store_chunk32(sb + F_P, r, c, pk);
      }
      l = l * alpha + ls;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
      if (!(ok = mbar_wait(pv_full, j & 1, abort_flag, a.flags))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; c++) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(trow + 128 + c * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; i++) o[c * 32 + i] = o[c * 32 + i] * alpha + __uint_as_float(v[i]);
      }
      m = mn;
    }
    if (ok) {
      const float inv = 1.0f / l;
      uint4* dst = reinterpret_cast<uint4*>(a.o_out + ((size_t)(row0 + qi) * a.H + h) * 64);
#pragma unroll
      for (int q = 0; q < 8; q++)
        dst[q] = make_uint4(pack2(o[8 * q] * inv, o[8 * q + 1] * inv), pack2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                            pack2(o[8 * q + 4] * inv, o[8 * q + 5] * inv), pack2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
      a.lse[(size_t)bh * a.T + qi] = (m + log2f(l)) * LN2;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

// ============================================================================
// backward, dK and dV: one CTA per (128-key block, b, h), walking the query
// blocks i >= key block.  Keys are the MMA rows:
//   S^T = K Q^T, dP^T = V dO^T  ->  P^T, dS^T (bf16, smem)
//   dV += P~^T dO,  dK += dS^T Q
// smem: K | V | Q[2] | dO[2] | P^T (2 blk) | dS^T (2 blk) | lse,D [2][128] | barriers
// TMEM: S^T [0,128), dP^T [128,256), dV [256,320), dK [320,384)  (512 allocated)
// ============================================================================
constexpr int K_K = 0, K_V = TILE, K_Q = 2 * TILE, K_DO = 4 * TILE, K_P = 6 * TILE, K_DS = 8 * TILE,
              K_LD = 10 * TILE, K_BAR = K_LD + 2 * 2 * 128 * 4;
constexpr int K_SMEM = K_BAR + 128;

__global__ void __launch_bounds__(192, 1) k_attn_bwd_kv_tc(const __grid_constant__ CUtensorMap tq,
                                                           const __grid_constant__ CUtensorMap tdo, AttnTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.flags, FLAG_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K_BAR);
  uint32_t kv_full = smem_u32(bars + 0), st_full0 = smem_u32(bars + 1), st_empty0 = smem_u32(bars + 3);
  uint32_t sdp_full = smem_u32(bars + 5), pds_full = smem_u32(bars + 6), acc_full = smem_u32(bars + 7);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  float* sld = reinterpret_cast<float*>(smem + K_LD);  // [2][lse2 128 | D 128]
  const uint32_t sb = smem_u32(smem);

  const int nqb = a.T / 128;
  const int kb = (int)blockIdx.x;  // key block 0 has the most query blocks: first
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int row0 = b * a.T;
  const int nit = nqb - kb;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(st_full0, 1);
    mbar_init(st_full0 + 8, 1);
    mbar_init(st_empty0, 1);
    mbar_init(st_empty0 + 8, 1);
    mbar_init(sdp_full, 1);
    mbar_init(pds_full, 128);
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tq);
    prefetch_tmap(&tdo);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(kv_full, 2 * TILE);
      tma_load_3d(sb + K_K, &tq, kv_full, 0, a.H + h, row0 + kb * 128);
      tma_load_3d(sb + K_V, &tq, kv_full, 0, 2 * a.H + h, row0 + kb * 128);
      for (int it = 0; it < nit; it++) {
        int i = kb + it, s = it & 1;
        if (!mbar_wait(st_empty0 + 8 * s, ((it >> 1) & 1) ^ 1, abort_flag, a.flags)) break;
        mbar_expect_tx(st_full0 + 8 * s, 2 * TILE + 1024);
        tma_load_3d(sb + K_Q + s * TILE, &tq, st_full0 + 8 * s, 0, h, row0 + i * 128);
        tma_load_3d(sb + K_DO + s * TILE, &tdo, st_full0 + 8 * s, 0, h, row0 + i * 128);
        bulk_load(sb + K_LD + s * 1024, a.lse + (size_t)bh * a.T + i * 128, 512, st_full0 + 8 * s);
        bulk_load(sb + K_LD + s * 1024 + 512, a.dsum + (size_t)bh * a.T + i * 128, 512, st_full0 + 8 * s);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_acc = idesc_bf16_f32(128, 64, false, true);
      bool ok = mbar_wait(kv_full, 0, abort_flag, a.flags);
      for (int it = 0; it < nit && ok; it++) {
        int s = it & 1;
        if (!(ok = mbar_wait(st_full0 + 8 * s, (it >> 1) & 1, abort_flag, a.flags))) break;
        tc_fence_after();
        uint32_t q = sb + K_Q + s * TILE, dO = sb + K_DO + s * TILE;
#pragma unroll
        for (int kk = 0; kk < 4; kk++) mma_bf16_ss(tmem, desc_k64(sb + K_K, kk), desc_k64(q, kk), id_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ss(tmem + 128, desc_k64(sb + K_V, kk), desc_k64(dO, kk), id_s, kk > 0);
        mma_commit(sdp_full);
        if (!(ok = mbar_wait(pds_full, it & 1, abort_flag, a.flags))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; kk++)
          mma_bf16_ss(tmem + 256, desc_k128(sb + K_P, kk), desc_mn64(dO, kk), id_acc, (it > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < 8; kk++)
          mma_bf16_ss(tmem + 320, desc_k128(sb + K_DS, kk), desc_mn64(q, kk), id_acc, (it > 0 || kk > 0));
        mma_commit(st_empty0 + 8 * s);
      }
      mma_commit(acc_full);
    }
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int kj = kb * 128 + r;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    bool ok = true;
    for (int it = 0; it < nit; it++) {
      const int i = kb + it;
      const float* ld = sld + (it & 1) * 256;  // [lse 128 | D 128] of query block i (bulk-copied)
      if (!(ok = mbar_wait(st_full0 + 8 * (it & 1), (it >> 1) & 1, abort_flag, a.flags))) break;
      if (!(ok = mbar_wait(sdp_full, it & 1, abort_flag, a.flags))) break;
      tc_fence_after();
      const bool diag = (it == 0);
#pragma unroll
      for (int c = 0; c < 4; c++) {
        uint32_t sv[32], dv[32];
        tmem_ld_32x32b_x32(trow + c * 32, sv);
        tmem_ld_32x32b_x32(trow + 128 + c * 32, dv);
        tmem_ld_wait();
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float pv[2], dsv[2];
#pragma unroll
          for (int u = 0; u < 2; u++) {
            int col = c * 32 + e + u;
            int qi = i * 128 + col;
            float p = (diag && kj > qi) ? 0.f : exp2f(__uint_as_float(sv[e + u]) * a.scale_log2 - ld[col] * LOG2E);
            float mk = drop_mul(a.drop, ((uint64_t)bh * a.T + qi) * a.T + kj);
            pv[u] = p * mk;
            dsv[u] = p * (__uint_as_float(dv[e + u]) * mk - ld[128 + col]);
          }
          pp[e >> 1] = pack2(pv[0], pv[1]);
          pd[e >> 1] = pack2(dsv[0], dsv[1]);
        }
        store_chunk32(sb + K_P, r, c, pp);
        store_chunk32(sb + K_DS, r, c, pd);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(pds_full);
    }
    if (ok && mbar_wait(acc_full, 0, abort_flag, a.flags)) {
      tc_fence_after();
      bf16* rowp = a.dqkv + (size_t)(row0 + kj) * (3 * a.H * 64);
      // dV at slot 2H+h, dK (times 1/sqrt(hd)) at slot H+h
#pragma unroll
      for (int w2 = 0; w2 < 2; w2++) {
        const float f = w2 == 0 ? 1.0f : a.scale;
        uint4* dst = reinterpret_cast<uint4*>(rowp + (size_t)((w2 == 0 ? 2 : 1) * a.H + h) * 64);
#pragma unroll
        for (int c = 0; c < 2; c++) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(trow + 256 + w2 * 64 + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 4; q++) {
            const float* x = reinterpret_cast<const float*>(v) + 8 * q;
            dst[c * 4 + q] = make_uint4(pack2(x[0] * f, x[1] * f), pack2(x[2] * f, x[3] * f),
                                        pack2(x[4] * f, x[5] * f), pack2(x[6] * f, x[7] * f));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ============================================================================
// backward, dQ: one CTA per (128-query block, b, h), walking key blocks <= it.
//   S = Q K^T, dP = dO V^T  ->  dS (bf16, smem);  dQ += dS K
// smem: Q | dO | K[2] | V[2] | dS (2 blk) | barriers
// TMEM: S [0,128), dP [128,256), dQ [256,320)  (512 allocated)
// ============================================================================
constexpr int Q_Q = 0, Q_DO = TILE, Q_K = 2 * TILE, Q_V = 4 * TILE, Q_DS = 6 * TILE, Q_BAR = 8 * TILE;
constexpr int Q_SMEM = Q_BAR + 128;

__global__ void __launch_bounds__(192, 1) k_attn_bwd_q_tc(const __grid_constant__ CUtensorMap tq,
                                                          const __grid_constant__ CUtensorMap tdo, AttnTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.flags, FLAG_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Q_BAR);
  uint32_t qd_full = smem_u32(bars + 0), kv_full0 = smem_u32(bars + 1), kv_empty0 = smem_u32(bars + 3);
  uint32_t sdp_full = smem_u32(bars + 5), ds_full = smem_u32(bars + 6), acc_full = smem_u32(bars + 7);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const uint32_t sb = smem_u32(smem);

  const int nqb = a.T / 128;
  const int qb = nqb - 1 - (int)blockIdx.x;
  const int bh = blockIdx.y, b = bh / a.H, h = bh % a.H;
  const int row0 = b * a.T;
  const int nkb = qb + 1;

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    mbar_init(kv_full0, 1);
    mbar_init(kv_full0 + 8, 1);
    mbar_init(kv_empty0, 1);
    mbar_init(kv_empty0 + 8, 1);
    mbar_init(sdp_full, 1);
    mbar_init(ds_full, 128);
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tq);
    prefetch_tmap(&tdo);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(qd_full, 2 * TILE);
      tma_load_3d(sb + Q_Q, &tq, qd_full, 0, h, row0 + qb * 128);
      tma_load_3d(sb + Q_DO, &tdo, qd_full, 0, h, row0 + qb * 128);
      for (int j = 0; j < nkb; j++) {
        int s = j & 1;
        if (!mbar_wait(kv_empty0 + 8 * s, ((j >> 1) & 1) ^ 1, abort_flag, a.flags)) break;
        mbar_expect_tx(kv_full0 + 8 * s, 2 * TILE);
        tma_load_3d(sb + Q_K + s * TILE, &tq, kv_full0 + 8 * s, 0, a.H + h, row0 + j * 128);
        tma_load_3d(sb + Q_V + s * TILE, &tq, kv_full0 + 8 * s, 0, 2 * a.H + h, row0 + j * 128);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_acc = idesc_bf16_f32(128, 64, false, true);
      bool ok = mbar_wait(qd_full, 0, abort_flag, a.flags);
      for (int j = 0; j < nkb && ok; j++) {
        int s = j & 1;
        if (!(ok = mbar_wait(kv_full0 + 8 * s, (j >> 1) & 1, abort_flag, a.flags))) break;
        tc_fence_after();
        uint32_t k = sb + Q_K + s * TILE, v = sb + Q_V + s * TILE;
#pragma unroll
        for (int kk = 0; kk < 4; kk++) mma_bf16_ss(tmem, desc_k64(sb + Q_Q, kk), desc_k64(k, kk), id_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ss(tmem + 128, desc_k64(sb + Q_DO, kk), desc_k64(v, kk), id_s, kk > 0);
        mma_commit(sdp_full);
        if (!(ok = mbar_wait(ds_full, j & 1, abort_flag, a.flags))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; kk++)
          mma_bf16_ss(tmem + 256, desc_k128(sb + Q_DS, kk), desc_mn64(k, kk), id_acc, (j > 0 || kk > 0));
        mma_commit(kv_empty0 + 8 * s);
      }
      mma_commit(acc_full);
    }
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qi = qb * 128 + r;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const float lse2 = a.lse[(size_t)bh * a.T + qi] * LOG2E;
    const float Di = a.dsum[(size_t)bh * a.T + qi];
    const uint64_t ebase = ((uint64_t)bh * a.T + qi) * a.T;
    bool ok = true;
    for (int j = 0; j < nkb; j++) {
      if (!(ok = mbar_wait(sdp_full, j & 1, abort_flag, a.flags))) break;
      tc_fence_after();
      const bool diag = (j == qb);
#pragma unroll
      for (int c = 0; c < 4; c++) {
        uint32_t sv[32], dv[32];
        tmem_ld_32x32b_x32(trow + c * 32, sv);
        tmem_ld_32x32b_x32(trow + 128 + c * 32, dv);
        tmem_ld_wait();
        uint32_t pd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float dsv[2];
#pragma unroll
          for (int u = 0; u < 2; u++) {
            int key = j * 128 + c * 32 + e + u;
            float p = (diag && key > qi) ? 0.f : exp2f(__uint_as_float(sv[e + u]) * a.scale_log2 - lse2);
            float mk = drop_mul(a.drop, ebase + key);
            dsv[u] = p * (__uint_as_float(dv[e + u]) * mk - Di);
          }
          pd[e >> 1] = pack2(dsv[0], dsv[1]);
        }
        store_chunk32(sb + Q_DS, r, c, pd);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok && mbar_wait(acc_full, 0, abort_flag, a.flags)) {
      tc_fence_after();
      uint4* dst = reinterpret_cast<uint4*>(a.dqkv + (size_t)(row0 + qi) * (3 * a.H * 64) + (size_t)h * 64);
#pragma unroll
      for (int c = 0; c < 2; c++) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(trow + 256 + c * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; q++) {
          const float* x = reinterpret_cast<const float*>(v) + 8 * q;
          const float f = a.scale;
          dst[c * 4 + q] = make_uint4(pack2(x[0] * f, x[1] * f), pack2(x[2] * f, x[3] * f),
                                      pack2(x[4] * f, x[5] * f), pack2(x[6] * f, x[7] * f));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// D[b,h,i] = sum_d dO[b,i,h,d] * O[b,i,h,d]: one warp per (row, head), 2 elements per lane
__global__ void k_attn_dsum64(const bf16* __restrict__ o, const bf16* __restrict__ dout, int B, int T, int H,
                              float* __restrict__ dsum) {
  long w = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (w >= (long)B * T * H) return;
  long row = w / H;  // b*T + t
  int h = (int)(w % H);
  const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(o + (row * H + h) * 64);
  const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(dout + (row * H + h) * 64);
  float2 x = __bfloat1622float2(a2[lane]);
  float2 y = __bfloat1622float2(b2[lane]);
  float s = warp_sum(x.x * y.x + x.y * y.y);
  if (lane == 0) {
    long b = row / T, t = row % T;
    dsum[(b * H + h) * T + t] = s;
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// [rows, slots, 64] bf16 viewed as 3-D {64, slots, rows}; box = one slot x 128 rows
bool map_rows(CUtensorMap* m, const void* base, int slots, long rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)slots, (cuuint64_t)rows};
  cuuint64_t strides[2] = {128, (cuuint64_t)slots * 128};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

AttnTcArgs make_args(const AttnDesc& d, uint32_t* flags) {
  AttnTcArgs a;
  a.B = d.B;
  a.T = d.T;
  a.H = d.H;
  a.o = reinterpret_cast<const bf16*>(d.o);
  a.o_out = reinterpret_cast<bf16*>(d.o);
  a.lse = d.lse;
  a.dsum = d.dsum;
  a.dqkv = reinterpret_cast<bf16*>(d.dqkv);
  a.scale = 0.125f;
  a.scale_log2 = 0.125f * LOG2E;
  a.drop = d.drop;
  a.flags = flags;
  return a;
}

}  // namespace

bool attn_tc_supported(const AttnDesc& a) {
  if (a.hd != 64 || a.T % 128 != 0 || a.T <= 0 || !encode_fn()) return false;
  if ((reinterpret_cast<uintptr_t>(a.qkv) & 15) || (reinterpret_cast<uintptr_t>(a.o) & 15)) return false;
  if (a.dout && (reinterpret_cast<uintptr_t>(a.dout) & 15)) return false;
  return true;
}

void attn_fwd_tc(Ctx& c, const AttnDesc& d) {
  CUtensorMap tm;
  if (!map_rows(&tm, d.qkv, 3 * d.H, (long)d.B * d.T)) {
    attn_fwd_simt<bf16>(c, d);
    return;
  }
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(k_attn_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, F_SMEM);
    attr = true;
  }
  dim3 grid(d.T / 128, d.B * d.H);
  LaunchScope s(c, "attn_fwd_tc");
  k_attn_fwd_tc<<<grid, 192, F_SMEM, c.stream>>>(tm, make_args(d, c.flags));
}

void attn_bwd_tc(Ctx& c, const AttnDesc& d) {
  CUtensorMap tq, tdo;
  if (!map_rows(&tq, d.qkv, 3 * d.H, (long)d.B * d.T) || !map_rows(&tdo, d.dout, d.H, (long)d.B * d.T)) {
    attn_bwd_simt<bf16>(c, d);
    return;
  }
  {
    long warps = (long)d.B * d.T * d.H;
    LaunchScope s(c, "attn_bwd_dsum");
    k_attn_dsum64<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, c.stream>>>(
        reinterpret_cast<const bf16*>(d.o), reinterpret_cast<const bf16*>(d.dout), d.B, d.T, d.H, d.dsum);
  }
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(k_attn_bwd_kv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, K_SMEM);
    cudaFuncSetAttribute(k_attn_bwd_q_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, Q_SMEM);
    attr = true;
  }
  AttnTcArgs a = make_args(d, c.flags);
  dim3 grid(d.T / 128, d.B * d.H);
  {
    LaunchScope s(c, "attn_bwd_kv_tc");
    k_attn_bwd_kv_tc<<<grid, 192, K_SMEM, c.stream>>>(tq, tdo, a);
  }
  {
    LaunchScope s(c, "attn_bwd_q_tc");
    k_attn_bwd_q_tc<<<grid, 192, Q_SMEM, c.stream>>>(tq, tdo, a);
  }
}

}  // namespace gpt
