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
// Every kernel: warp 0 issues TMA loads of bf16 tiles (128-byte swizzle) from
// the [B*T, 3, H, 64] qkv activations, warp 1 owns TMEM and issues
// tcgen05.mma, and the math warps (forward: warps 2..5, one TMEM lane / tile
// row per thread; backward: warps 2..9, two per lane quadrant) do the softmax
// arithmetic, write the bf16 probability (or dS) tile back into TMEM, where the
// next MMA reads it as its A operand, and run the epilogue.  Each kernel keeps
// its TMEM at 256 columns and its shared memory under 113 KB so that two CTAs
// share an SM: one CTA's softmax overlaps the other's MMAs.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.cuh"
#include "sm100.cuh"

namespace gpt {
namespace {

using namespace sm100;

constexpr int TILE = 16384;  // 128 rows x 64 bf16 (128 bytes), 128-byte swizzle
constexpr int HTILE = 8192;  // 64 rows x 64 bf16
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct AttnTcArgs {
  int B, T, H;
  bf16* o_out;
  float* lse;         // [B, H, T] natural log
  float* dsum;        // [B, H, T] D = rowsum(dO * O): written by the dQ kernel, read by dK/dV
  bf16* dqkv;
  float scale_log2;   // log2(e) / sqrt(64)
  float scale;        // 1 / sqrt(64)
  DropKey drop;
  uint32_t* flags;
  float* colsum;      // backward: column sums of dqkv per 128-row block (null: none)
  int colsum_acc;
};

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
// 2^x with the SFU instruction (relative error ~2^-22; 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// K-major operand: K-step kk (16 elements) of a tile with 64-wide K-blocks
__device__ __forceinline__ uint64_t desc_k(uint32_t tile, int kb_bytes, int kk) {
  return desc_sw128(tile + (kk >> 2) * kb_bytes + (kk & 3) * 32, 16, 1024);
}
// a [rows, 64] tile read MN-major (N = the 64 columns, K = rows), K-step kk
__device__ __forceinline__ uint64_t desc_mn64(uint32_t tile, int kk) { return desc_sw128(tile + kk * 2048, TILE, 1024); }

__device__ __forceinline__ void ld64(uint32_t taddr, uint32_t (&a)[32], uint32_t (&b)[32]) {
  tmem_ld_32x32b_x32(taddr, a);
  tmem_ld_32x32b_x32(taddr + 32, b);
  tmem_ld_wait();
}

// ============================================================================
// forward, pipelined: one CTA per (128-query block, b, h), 64-key blocks.
// S is double-buffered in TMEM, so the MMA warp computes S of block j+1
// while the softmax warps work on block j.  O accumulates in TMEM (the P V
// MMAs add into it) against a per-row reference maximum m that is raised only
// when a block's maximum exceeds it by more than 2^RESCALE_LOG2 (then the
// softmax warps rescale that row of O and l once); otherwise probabilities are
// taken against the stale m, which leaves O / l and m + log2 l unchanged.
// smem: Q | (K, V)[3 stages] | barriers   (64 KB + 256 B)
// TMEM: S[2] cols [0,64), [64,128); O cols [128,192)  (256 allocated).  The
// softmax warps overwrite the first 32 columns of S[u] with bf16 P, which the
// P V MMA reads as its TMEM A operand (tcgen05 MMAs of one thread execute in
// issue order, so S of block j+2 lands in S[u] only after P V of block j).
// ============================================================================
constexpr int D_Q = 0, D_KV = TILE, D_BAR = 4 * TILE;
constexpr int D_SMEM = D_BAR + 256;
constexpr int D_STAGES = 3;
constexpr float RESCALE_LOG2 = 8.0f;

template <bool DROP>
__global__ void __launch_bounds__(192, 2) k_attn_fwd_o(const __grid_constant__ CUtensorMap tq,
                                                       const __grid_constant__ CUtensorMap tkv64, AttnTcArgs a) {
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {  // swizzled tiles need 1024-byte alignment
    pdl_wait();
    if (threadIdx.x == 0) atomicOr(a.flags, FLAG_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + D_BAR);
  const uint32_t q_full = smem_u32(bars + 0);
  const uint32_t kv_full0 = smem_u32(bars + 1), kv_empty0 = smem_u32(bars + 1 + D_STAGES);
  // pv_done[i & 1] completes when the P V product of block i has landed in O
  const uint32_t s_full0 = smem_u32(bars + 1 + 2 * D_STAGES), p_full0 = s_full0 + 16, pv_done0 = s_full0 + 32;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 7 + 2 * D_STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const uint32_t sb = smem_u32(smem);

  const int nqb = a.T / 128;
  // blocks are dispatched x-fastest: every (b, h) of the longest query block
  // first, so the launch ends on short blocks (longest-first scheduling)
  const int qb = nqb - 1 - (int)blockIdx.y;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int nkb = 2 * (qb + 1);  // 64-key blocks up to and including the diagonal (>= 2)
  const int row0 = b * a.T;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < D_STAGES; s++) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 1);
    }
    for (int u = 0; u < 2; u++) {
      mbar_init(s_full0 + 8 * u, 1);
      mbar_init(p_full0 + 8 * u, 4);
      mbar_init(pv_done0 + 8 * u, 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tq);
    prefetch_tmap(&tkv64);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // predecessor kernels complete from here on (programmatic dependent launch);
  // the dropout key of this launch (derived from the device step index in a replayed graph)
  pdl_wait();
  const DropKey dk = DROP ? drop_live(a.drop) : a.drop;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(q_full, TILE);
      tma_load_3d(sb + D_Q, &tq, q_full, 0, h, row0 + qb * 128);
      for (int j = 0; j < nkb; j++) {
        const int s = j % D_STAGES;
        const uint32_t fb = kv_full0 + 8 * s;
        if (!mbar_wait(kv_empty0 + 8 * s, ((j / D_STAGES) & 1) ^ 1, abort_flag, a.flags)) break;
        mbar_expect_tx(fb, 2 * HTILE);
        tma_load_3d(sb + D_KV + s * TILE, &tkv64, fb, 0, a.H + h, row0 + j * 64);
        tma_load_3d(sb + D_KV + s * TILE + HTILE, &tkv64, fb, 0, 2 * a.H + h, row0 + j * 64);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_n64 = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t id_pv = idesc_bf16_f32(128, 64, false, true);
      bool ok = mbar_wait(q_full, 0, abort_flag, a.flags);
      // O += P V of block i: P over the first 32 columns of S[i&1] (K = 64
      // keys), V of block i MN-major (N = 64)
      auto issue_pv = [&](int i) -> bool {
        const int u = i & 1;
        if (!mbar_wait(p_full0 + 8 * u, (i >> 1) & 1, abort_flag, a.flags)) return false;
        tc_fence_after();
        const uint32_t v = sb + D_KV + (i % D_STAGES) * TILE + HTILE;
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ts(tmem + 128, tmem + 64 * u + 8 * kk, desc_mn64(v, kk), id_pv, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(pv_done0 + 8 * u);
        mma_commit(kv_empty0 + 8 * (i % D_STAGES));
        return true;
      };
      for (int j = 0; j < nkb && ok; j++) {
        const int s = j % D_STAGES;
        if (!(ok = mbar_wait(kv_full0 + 8 * s, (j / D_STAGES) & 1, abort_flag, a.flags))) break;
        tc_fence_after();
        // S[j&1] is free: its previous block's P (j-2) was waited for below
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ss(tmem + 64 * (j & 1), desc_k(sb + D_Q, TILE, kk), desc_k(sb + D_KV + s * TILE, HTILE, kk), id_n64,
                      kk > 0);
        mma_commit(s_full0 + 8 * (j & 1));
        if (j >= 1 && !(ok = issue_pv(j - 1))) break;
      }
      if (ok) issue_pv(nkb - 1);
    }
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qi = qb * 128 + r;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const float sl2 = a.scale_log2;
    float m = -INFINITY, l = 0.f;  // reference maximum (log2 units) and row sum against it
    const uint64_t ebase = ((uint64_t)bh * a.T + qi) * a.T;
    bool ok = true;
    for (int j = 0; j < nkb; j++) {
      const int u = j & 1;
      if (!(ok = mbar_wait(s_full0 + 8 * u, (j >> 1) & 1, abort_flag, a.flags))) break;
      tc_fence_after();
      uint32_t v0[32], v1[32];
      ld64(trow + 64 * u, v0, v1);
      const int key0 = j * 64;
      const int lim = qi - key0;  // key key0 + i is visible iff i <= lim
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
      if (lim >= 63) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          mx0 = fmaxf(mx0, __uint_as_float(v0[i]));
          mx1 = fmaxf(mx1, __uint_as_float(v0[i + 1]));
          mx2 = fmaxf(mx2, __uint_as_float(v1[i]));
          mx3 = fmaxf(mx3, __uint_as_float(v1[i + 1]));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; i++) {
          if (i <= lim) mx0 = fmaxf(mx0, __uint_as_float(v0[i]));
          if (i + 32 <= lim) mx1 = fmaxf(mx1, __uint_as_float(v1[i]));
        }
      }
      const float bm = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      if (j == 0) {
        m = bm;  // key 0 is visible to every row, so m is finite from here on
      } else {
        const bool need = bm > m + RESCALE_LOG2;
        if (__any_sync(0xffffffffu, need)) {
          // O holds the P V products of blocks < j.  S of block j was issued
          // after P V of block j-2, so P V of block j-1 is the only one that
          // may be in flight.
          if (!(ok = mbar_wait(pv_done0 + 8 * ((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, a.flags))) break;
          tc_fence_after();
          const float sc = need ? ex2(m - bm) : 1.f;
          uint32_t o0[32], o1[32];
          ld64(trow + 128, o0, o1);
          uint32_t w[16];
#pragma unroll
          for (int h2 = 0; h2 < 4; h2++) {
            const uint32_t* src = h2 < 2 ? o0 + 16 * h2 : o1 + 16 * (h2 - 2);
#pragma unroll
            for (int i = 0; i < 16; i++) w[i] = __float_as_uint(__uint_as_float(src[i]) * sc);
            tmem_st_32x32b_x16(trow + 128 + 16 * h2, w);
          }
          l *= sc;
          if (need) m = bm;
        }
      }
      float ls0 = 0.f, ls1 = 0.f;
      uint32_t pk0[16], pk1[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float p0 = ex2(fmaf(__uint_as_float(v0[i]), sl2, -m));
        float p1 = ex2(fmaf(__uint_as_float(v0[i + 1]), sl2, -m));
        float p2 = ex2(fmaf(__uint_as_float(v1[i]), sl2, -m));
        float p3 = ex2(fmaf(__uint_as_float(v1[i + 1]), sl2, -m));
        if (lim < 63) {
          if (i > lim) p0 = 0.f;
          if (i + 1 > lim) p1 = 0.f;
          if (i + 32 > lim) p2 = 0.f;
          if (i + 33 > lim) p3 = 0.f;
        }
        ls0 += p0 + p1;
        ls1 += p2 + p3;
        if (DROP) {
          const uint64_t e = ebase + key0 + i;
          p0 *= drop_mul(dk, e);
          p1 *= drop_mul(dk, e + 1);
          p2 *= drop_mul(dk, e + 32);
          p3 *= drop_mul(dk, e + 33);
        }
        pk0[i >> 1] = pack2(p0, p1);
        pk1[i >> 1] = pack2(p2, p3);
      }
      // P (bf16 pairs) over the first 32 columns of S[u]: the A operand of P V
      tmem_st_32x32b_x16(trow + 64 * u, pk0);
      tmem_st_32x32b_x16(trow + 64 * u + 16, pk1);
      l += ls0 + ls1;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full0 + 8 * u);  // one arrival per math warp
    }
    // the last two P V products may both be in flight
    if (ok) ok = mbar_wait(pv_done0 + 8 * (nkb & 1), ((nkb - 2) >> 1) & 1, abort_flag, a.flags);
    if (ok) ok = mbar_wait(pv_done0 + 8 * ((nkb - 1) & 1), ((nkb - 1) >> 1) & 1, abort_flag, a.flags);
    if (ok) {
      tc_fence_after();
      uint32_t o0[32], o1[32];
      ld64(trow + 128, o0, o1);
      const float inv = 1.0f / l;
      uint4* dst = reinterpret_cast<uint4*>(a.o_out + ((size_t)(row0 + qi) * a.H + h) * 64);
#pragma unroll
      for (int q = 0; q < 8; q++) {
        const uint32_t* x = q < 4 ? o0 + 8 * q : o1 + 8 * (q - 4);
        dst[q] = make_uint4(pack2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv),
                            pack2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv),
                            pack2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv),
                            pack2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv));
      }
      a.lse[(size_t)bh * a.T + qi] = (m + log2f(l)) * LN2;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

// packed bf16 pair column of element column c (0..63) of a 64-column block:
// the half that owns c writes inside its own fp32 columns
__device__ __forceinline__ int pcol(int c) { return (c & 32) + ((c & 31) >> 1); }
// TMEM A-operand column of K-step kk (16 elements) under that layout
__device__ __forceinline__ uint32_t acol(int kk) { return (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8); }

__device__ __forceinline__ uint32_t pack2v(uint64_t v) {
  const float2 f = f2split(v);
  return pack2(f.x, f.y);
}

// Column sums of a warp's 32 rows (one per lane) x 32 columns (v[c] in lane
// order): a butterfly in which each step hands half of a lane's columns to its
// partner, so lane c ends with the sum of column c (31 shuffles, fixed order).
__device__ __forceinline__ float warp_colsum32(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; i++) {
      const float send = upper ? v[i] : v[i + o];
      const float keep = upper ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

// The 128-row block's column sums of 32 columns held by the four lane-quadrant
// warps of one half (sum_q: this warp's column sums, lane c for column c):
// combined in quadrant order through shared memory by the quadrant-0 warp,
// which writes (or adds to) colsum[blk][col0 + c].  All eight math warps
// must call it (named barrier 1).
__device__ __forceinline__ void block_colsum(float* s_red, int half, int quad, int lane, float sum_q, float* colsum,
                                             size_t blk, long ld, long col0, int acc) {
  s_red[(half * 4 + quad) * 32 + lane] = sum_q;
  asm volatile("bar.sync 1, 256;" ::: "memory");
  if (quad == 0) {
    const float t = ((s_red[(half * 4 + 0) * 32 + lane] + s_red[(half * 4 + 1) * 32 + lane]) +
                     s_red[(half * 4 + 2) * 32 + lane]) + s_red[(half * 4 + 3) * 32 + lane];
    float* dst = colsum + blk * ld + col0 + lane;
    *dst = acc ? *dst + t : t;
  }
  asm volatile("bar.sync 1, 256;" ::: "memory");
}

constexpr int BWD_STAGES = 3;  // Q/dO (or K/V) tiles in flight

// ============================================================================
// backward, dK and dV: one CTA per (128-key block, b, h), walking 64-query
// blocks from the key block on.  Keys are the MMA rows:
//   S^T = K Q^T, dP^T = V dO^T  ->  P~^T, dS^T (bf16, written into TMEM)
//   dV += P~^T dO,  dK += dS^T Q
// Eight math warps, two per TMEM lane quadrant, each take 32 of the 64 query
// columns of a block (the backward has no row reductions).  The math runs in
// two phases per block (P~^T from S^T, then dS^T from dP^T) with an mbarrier
// each way, and the MMA warp issues in the order
//   S(i) dP(i) | P~(i) ready: dV(i) S(i+1) | dS(i) ready: dK(i) dP(i+1) | ...
// so S^T of the next block is computed while the math warps work on dS^T, and
// dP^T of the next block while they work on P~^T.  (P~^T lives in the S^T
// columns and dS^T in the dP^T columns; tcgen05 MMAs of one thread execute in
// issue order, so each is read before it is overwritten.)
// smem: K | V | (Q, dO)[3 stages] | (lse, D)[3] | barriers (~82 KB)
// TMEM: S^T [0,64), dP^T [64,128), dV [128,192), dK [192,256)
// ============================================================================
constexpr int K_K = 0, K_V = TILE, K_ST = 2 * TILE, K_LD = (2 + BWD_STAGES) * TILE, K_BAR = K_LD + 2048;
constexpr int K_RED = K_BAR + 128;  // [2 halves][4 quadrants][32] column partials
constexpr int K_SMEM = K_RED + 1024;

template <bool DROP>
__global__ void __launch_bounds__(320, 2) k_attn_bwd_kv8(const __grid_constant__ CUtensorMap tkv,
                                                         const __grid_constant__ CUtensorMap tq64,
                                                         const __grid_constant__ CUtensorMap tdo64, AttnTcArgs a) {
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    pdl_wait();
    if (threadIdx.x == 0) atomicOr(a.flags, FLAG_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K_BAR);
  const uint32_t kv_full = smem_u32(bars + 0), st_full0 = smem_u32(bars + 1),
                 st_empty0 = smem_u32(bars + 1 + BWD_STAGES);
  const uint32_t s_full = smem_u32(bars + 1 + 2 * BWD_STAGES), dp_full = s_full + 8, p_ready = s_full + 16,
                 ds_ready = s_full + 24, acc_full = s_full + 32;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 6 + 2 * BWD_STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const float* sld = reinterpret_cast<const float*>(smem + K_LD);  // [stage][lse 64 | D 64]
  const uint32_t sb = smem_u32(smem);

  const int nq64 = a.T / 64;
  const int kb = (int)blockIdx.y;  // key block 0 (most query blocks) of every (b, h) first
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int row0 = b * a.T;
  const int i0 = 2 * kb;
  const int nit = nq64 - i0;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < BWD_STAGES; s++) {
      mbar_init(st_full0 + 8 * s, 1);
      mbar_init(st_empty0 + 8 * s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 8);
    mbar_init(ds_ready, 8);
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tkv);
    prefetch_tmap(&tq64);
    prefetch_tmap(&tdo64);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // predecessor kernels complete from here on (programmatic dependent launch);
  // the dropout key of this launch (derived from the device step index in a replayed graph)
  pdl_wait();
  const DropKey dk = DROP ? drop_live(a.drop) : a.drop;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(kv_full, 2 * TILE);
      tma_load_3d(sb + K_K, &tkv, kv_full, 0, a.H + h, row0 + kb * 128);
      tma_load_3d(sb + K_V, &tkv, kv_full, 0, 2 * a.H + h, row0 + kb * 128);
      for (int it = 0; it < nit; it++) {
        const int i = i0 + it, s = it % BWD_STAGES;
        const uint32_t fb = st_full0 + 8 * s;
        if (!mbar_wait(st_empty0 + 8 * s, ((it / BWD_STAGES) & 1) ^ 1, abort_flag, a.flags)) break;
        mbar_expect_tx(fb, 2 * HTILE + 512);
        tma_load_3d(sb + K_ST + s * TILE, &tq64, fb, 0, h, row0 + i * 64);
        tma_load_3d(sb + K_ST + s * TILE + HTILE, &tdo64, fb, 0, h, row0 + i * 64);
        bulk_load(sb + K_LD + s * 512, a.lse + (size_t)bh * a.T + i * 64, 256, fb);
        bulk_load(sb + K_LD + s * 512 + 256, a.dsum + (size_t)bh * a.T + i * 64, 256, fb);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t id_acc = idesc_bf16_f32(128, 64, false, true);
      auto q_of = [&](int it) { return sb + K_ST + (it % BWD_STAGES) * TILE; };
      auto issue_s = [&](int it) -> bool {  // S^T = K Q^T of block it
        if (!mbar_wait(st_full0 + 8 * (it % BWD_STAGES), (it / BWD_STAGES) & 1, abort_flag, a.flags)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ss(tmem, desc_k(sb + K_K, TILE, kk), desc_k(q_of(it), HTILE, kk), id_s, kk > 0);
        mma_commit(s_full);
        return true;
      };
      auto issue_dp = [&](int it) {  // dP^T = V dO^T of block it (its stage is loaded)
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ss(tmem + 64, desc_k(sb + K_V, TILE, kk), desc_k(q_of(it) + HTILE, HTILE, kk), id_s, kk > 0);
        mma_commit(dp_full);
      };
      bool ok = mbar_wait(kv_full, 0, abort_flag, a.flags) && issue_s(0);
      if (ok) issue_dp(0);
      for (int it = 0; it < nit && ok; it++) {
        const uint32_t q = q_of(it), dO = q + HTILE;
        if (!(ok = mbar_wait(p_ready, it & 1, abort_flag, a.flags))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ts(tmem + 128, tmem + acol(kk), desc_mn64(dO, kk), id_acc, (it > 0 || kk > 0));
        if (it + 1 < nit && !(ok = issue_s(it + 1))) break;
        if (!(ok = mbar_wait(ds_ready, it & 1, abort_flag, a.flags))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ts(tmem + 192, tmem + 64 + acol(kk), desc_mn64(q, kk), id_acc, (it > 0 || kk > 0));
        mma_commit(st_empty0 + 8 * (it % BWD_STAGES));
        if (it + 1 < nit) issue_dp(it + 1);
      }
      mma_commit(acc_full);
    }
  } else {
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    const int kj = kb * 128 + r;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const uint64_t sl2x2 = f2(a.scale_log2, a.scale_log2), nlog2e = f2(-LOG2E, -LOG2E);
    bool ok = true;
    for (int it = 0; it < nit; it++) {
      const int i = i0 + it;
      const int q0 = i * 64;
      const float* ld = sld + (it % BWD_STAGES) * 128;  // lse[64] | D[64] of this query block
      // lse / D of the stage (TMA-written: observed through the stage's own
      // barrier), then S^T of the block
      if (!(ok = mbar_wait(st_full0 + 8 * (it % BWD_STAGES), (it / BWD_STAGES) & 1, abort_flag, a.flags))) break;
      if (!(ok = mbar_wait(s_full, it & 1, abort_flag, a.flags))) break;
      tc_fence_after();
      const int lim = kj - q0;                  // query column c is masked iff c < lim
      const bool masked = q0 < kb * 128 + 128;  // only blocks that reach this CTA's keys
      float pk[2][16];                          // P^T of this thread's 32 columns
      // phase 1: P^T = 2^(S^T sl2 - lse log2 e) (masked), P~^T = drop(P^T)
#pragma unroll
      for (int sub = 0; sub < 2; sub++) {
        const int c0 = half * 32 + sub * 16;
        uint32_t sv[16];
        tmem_ld_32x32b_x16(trow + c0, sv);
        tmem_ld_wait();
        uint32_t pp[8];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(ld + c0 + e);
          const float2 y01 = f2split(f2fma(f2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sl2x2,
                                           f2mul(f2(l4.x, l4.y), nlog2e)));
          const float2 y23 = f2split(f2fma(f2(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3])), sl2x2,
                                           f2mul(f2(l4.z, l4.w), nlog2e)));
          float p4[4] = {ex2(y01.x), ex2(y01.y), ex2(y23.x), ex2(y23.y)};
#pragma unroll
          for (int u = 0; u < 4; u++) {
            if (masked && c0 + e + u < lim) p4[u] = 0.f;
            pk[sub][e + u] = p4[u];
          }
          if (DROP) {
#pragma unroll
            for (int u = 0; u < 4; u++)
              p4[u] *= drop_mul(dk, ((uint64_t)bh * a.T + q0 + c0 + e + u) * a.T + kj);
          }
          pp[e >> 1] = pack2(p4[0], p4[1]);
          pp[(e >> 1) + 1] = pack2(p4[2], p4[3]);
        }
        tmem_st_32x32b_x8(trow + pcol(c0), pp);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready);
      // phase 2: dS^T = P^T (drop(dP^T) - D)
      if (!(ok = mbar_wait(dp_full, it & 1, abort_flag, a.flags))) break;
      tc_fence_after();
#pragma unroll
      for (int sub = 0; sub < 2; sub++) {
        const int c0 = half * 32 + sub * 16;
        uint32_t dv[16];
        tmem_ld_32x32b_x16(trow + 64 + c0, dv);
        tmem_ld_wait();
        uint32_t pd[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float2 d2 = *reinterpret_cast<const float2*>(ld + 64 + c0 + e);
          float dp0 = __uint_as_float(dv[e]), dp1 = __uint_as_float(dv[e + 1]);
          if (DROP) {
            dp0 *= drop_mul(dk, ((uint64_t)bh * a.T + q0 + c0 + e) * a.T + kj);
            dp1 *= drop_mul(dk, ((uint64_t)bh * a.T + q0 + c0 + e + 1) * a.T + kj);
          }
          pd[e >> 1] = pack2v(f2mul(f2(pk[sub][e], pk[sub][e + 1]), f2sub(f2(dp0, dp1), f2(d2.x, d2.y))));
        }
        tmem_st_32x32b_x8(trow + 64 + pcol(c0), pd);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_ready);
    }
    const bool done = ok && mbar_wait(acc_full, 0, abort_flag, a.flags);
    if (done) {
      tc_fence_after();
      bf16* rowp = a.dqkv + (size_t)(row0 + kj) * (3 * a.H * 64);
      // half 0: dV at slot 2H+h; half 1: dK (times 1/sqrt(hd)) at slot H+h
      const float f = half == 0 ? 1.0f : a.scale;
      const int slot = (half == 0 ? 2 : 1) * a.H + h;
      uint4* dst = reinterpret_cast<uint4*>(rowp + (size_t)slot * 64);
#pragma unroll
      for (int c2 = 0; c2 < 2; c2++) {  // 32 columns at a time: stored, then their block column sums
        float cs[32];
#pragma unroll
        for (int c1 = 0; c1 < 2; c1++) {
          const int c = 2 * c2 + c1;
          uint32_t v[16];
          tmem_ld_32x32b_x16(trow + 128 + half * 64 + c * 16, v);
          tmem_ld_wait();
          const float* x = reinterpret_cast<const float*>(v);
          uint32_t w[8];
#pragma unroll
          for (int k = 0; k < 8; k++) {
            w[k] = pack2(x[2 * k] * f, x[2 * k + 1] * f);
            const float2 bk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
            cs[16 * c1 + 2 * k] = bk.x;  // the stored (bf16) values
            cs[16 * c1 + 2 * k + 1] = bk.y;
          }
          dst[2 * c] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[2 * c + 1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
        if (a.colsum) {
          const float sq = warp_colsum32(cs, lane);
          block_colsum(reinterpret_cast<float*>(smem + K_RED), half, quad, lane, sq, a.colsum,
                       (size_t)(row0 + kb * 128) / 128, 3L * a.H * 64, (long)slot * 64 + 32 * c2, a.colsum_acc);
        }
      }
    } else if (a.colsum) {
      // every math warp takes part in the column-sum barriers, even on a failed wait
      for (int c2 = 0; c2 < 4; c2++) asm volatile("bar.sync 1, 256;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

// ============================================================================
// backward, dQ: one CTA per (128-query block, b, h), walking 64-key blocks
// up to the diagonal.  S = Q K^T, dP = dO V^T -> dS (bf16, written into the
// dP columns of TMEM); dQ += dS K.  Eight math warps as in the dK/dV kernel,
// in two phases per block (P from S, then dS from dP); the MMA warp issues
//   S(j) dP(j) | S read: S(j+1) | dS(j) ready: dQ(j) dP(j+1) | ...
// so S of the next block is computed while the math warps work on dS.
// The kernel also computes D_i = sum_d dO_id O_id of its rows from the dO and
// O tiles in shared memory and stores it for the dK/dV kernel, which runs
// after it.
// smem: Q | dO | O | (K, V)[3 stages] | barriers   (~96 KB)
// TMEM: S [0,64), dP [64,128), dQ [128,192)  (256 allocated)
// ============================================================================
constexpr int Q_Q = 0, Q_DO = TILE, Q_OT = 2 * TILE, Q_ST = 3 * TILE, Q_BAR = (3 + BWD_STAGES) * TILE;
constexpr int Q_RED = Q_BAR + 128;
constexpr int Q_SMEM = Q_RED + 1024;

template <bool DROP>
__global__ void __launch_bounds__(320, 2) k_attn_bwd_q8(const __grid_constant__ CUtensorMap tq,
                                                        const __grid_constant__ CUtensorMap tdo,
                                                        const __grid_constant__ CUtensorMap tkv64,
                                                        const __grid_constant__ CUtensorMap tout, AttnTcArgs a) {
  pdl_trigger();
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023) {
    pdl_wait();
    if (threadIdx.x == 0) atomicOr(a.flags, FLAG_TIMEOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Q_BAR);
  const uint32_t qd_full = smem_u32(bars + 0), kv_full0 = smem_u32(bars + 1),
                 kv_empty0 = smem_u32(bars + 1 + BWD_STAGES);
  const uint32_t s_full = smem_u32(bars + 1 + 2 * BWD_STAGES), dp_full = s_full + 8, s_read = s_full + 16,
                 ds_ready = s_full + 24, acc_full = s_full + 32;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 6 + 2 * BWD_STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const uint32_t sb = smem_u32(smem);

  const int nqb = a.T / 128;
  const int qb = nqb - 1 - (int)blockIdx.y;  // longest rows of every (b, h) first
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int row0 = b * a.T;
  const int nkb = 2 * (qb + 1);  // 64-key blocks up to and including the diagonal

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    for (int s = 0; s < BWD_STAGES; s++) {
      mbar_init(kv_full0 + 8 * s, 1);
      mbar_init(kv_empty0 + 8 * s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(s_read, 8);
    mbar_init(ds_ready, 8);
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tq);
    prefetch_tmap(&tdo);
    prefetch_tmap(&tkv64);
    prefetch_tmap(&tout);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tslot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // predecessor kernels complete from here on (programmatic dependent launch);
  // the dropout key of this launch (derived from the device step index in a replayed graph)
  pdl_wait();
  const DropKey dk = DROP ? drop_live(a.drop) : a.drop;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(qd_full, 3 * TILE);
      tma_load_3d(sb + Q_Q, &tq, qd_full, 0, h, row0 + qb * 128);
      tma_load_3d(sb + Q_DO, &tdo, qd_full, 0, h, row0 + qb * 128);
      tma_load_3d(sb + Q_OT, &tout, qd_full, 0, h, row0 + qb * 128);
      for (int j = 0; j < nkb; j++) {
        const int s = j % BWD_STAGES;
        const uint32_t fb = kv_full0 + 8 * s;
        if (!mbar_wait(kv_empty0 + 8 * s, ((j / BWD_STAGES) & 1) ^ 1, abort_flag, a.flags)) break;
        mbar_expect_tx(fb, 2 * HTILE);
        tma_load_3d(sb + Q_ST + s * TILE, &tkv64, fb, 0, a.H + h, row0 + j * 64);
        tma_load_3d(sb + Q_ST + s * TILE + HTILE, &tkv64, fb, 0, 2 * a.H + h, row0 + j * 64);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t id_acc = idesc_bf16_f32(128, 64, false, true);
      auto k_of = [&](int j) { return sb + Q_ST + (j % BWD_STAGES) * TILE; };
      auto issue_s = [&](int j) -> bool {  // S = Q K^T of block j
        if (!mbar_wait(kv_full0 + 8 * (j % BWD_STAGES), (j / BWD_STAGES) & 1, abort_flag, a.flags)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ss(tmem, desc_k(sb + Q_Q, TILE, kk), desc_k(k_of(j), HTILE, kk), id_s, kk > 0);
        mma_commit(s_full);
        return true;
      };
      auto issue_dp = [&](int j) {  // dP = dO V^T of block j (its stage is loaded)
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ss(tmem + 64, desc_k(sb + Q_DO, TILE, kk), desc_k(k_of(j) + HTILE, HTILE, kk), id_s, kk > 0);
        mma_commit(dp_full);
      };
      bool ok = mbar_wait(qd_full, 0, abort_flag, a.flags) && issue_s(0);
      if (ok) issue_dp(0);
      for (int j = 0; j < nkb && ok; j++) {
        if (!(ok = mbar_wait(s_read, j & 1, abort_flag, a.flags))) break;
        if (j + 1 < nkb && !(ok = issue_s(j + 1))) break;
        if (!(ok = mbar_wait(ds_ready, j & 1, abort_flag, a.flags))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_bf16_ts(tmem + 128, tmem + 64 + acol(kk), desc_mn64(k_of(j), kk), id_acc, (j > 0 || kk > 0));
        mma_commit(kv_empty0 + 8 * (j % BWD_STAGES));
        if (j + 1 < nkb) issue_dp(j + 1);
      }
      mma_commit(acc_full);
    }
  } else {
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    const int qi = qb * 128 + r;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    const float lse2 = a.lse[(size_t)bh * a.T + qi] * LOG2E;
    // D of this row from the dO and O tiles (128-byte rows, 128-byte swizzle:
    // 16-byte chunk q of row r at q ^ (r & 7)); both halves compute it
    bool ok = mbar_wait(qd_full, 0, abort_flag, a.flags);
    float Di = 0.f;
    if (ok) {
#pragma unroll
      for (int q = 0; q < 8; q++) {
        const uint32_t off = r * 128 + ((q ^ (r & 7)) << 4);
        const uint4 x = ld_shared_v4(sb + Q_DO + off), y = ld_shared_v4(sb + Q_OT + off);
        const uint32_t xw[4] = {x.x, x.y, x.z, x.w}, yw[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int k = 0; k < 4; k++) {
          const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[k]));
          const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&yw[k]));
          Di = fmaf(xf.x, yf.x, fmaf(xf.y, yf.y, Di));
        }
      }
      if (half == 0) a.dsum[(size_t)bh * a.T + qi] = Di;
    }
    const uint64_t sl2x2 = f2(a.scale_log2, a.scale_log2), nlse2 = f2(-lse2, -lse2), Dx2 = f2(Di, Di);
    const uint64_t ebase = ((uint64_t)bh * a.T + qi) * a.T;
    for (int j = 0; j < nkb && ok; j++) {
      if (!(ok = mbar_wait(s_full, j & 1, abort_flag, a.flags))) break;
      tc_fence_after();
      const int key0 = j * 64;
      const int lim = qi - key0;                 // key column c is visible iff c <= lim
      const bool masked = key0 + 64 > qb * 128;  // only the blocks that reach the diagonal
      // phase 1: P = 2^(S sl2 - lse log2 e) (masked) into registers
      float pk[2][16];
#pragma unroll
      for (int sub = 0; sub < 2; sub++) {
        const int c0 = half * 32 + sub * 16;
        uint32_t sv[16];
        tmem_ld_32x32b_x16(trow + c0, sv);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float2 y = f2split(f2fma(f2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sl2x2, nlse2));
          pk[sub][e] = (masked && c0 + e > lim) ? 0.f : ex2(y.x);
          pk[sub][e + 1] = (masked && c0 + e + 1 > lim) ? 0.f : ex2(y.y);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_read);  // S may be overwritten by the next block
      // phase 2: dS = P (drop(dP) - D) over the dP columns
      if (!(ok = mbar_wait(dp_full, j & 1, abort_flag, a.flags))) break;
      tc_fence_after();
#pragma unroll
      for (int sub = 0; sub < 2; sub++) {
        const int c0 = half * 32 + sub * 16;
        uint32_t dv[16];
        tmem_ld_32x32b_x16(trow + 64 + c0, dv);
        tmem_ld_wait();
        uint32_t pd[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float dp0 = __uint_as_float(dv[e]), dp1 = __uint_as_float(dv[e + 1]);
          if (DROP) {
            dp0 *= drop_mul(dk, ebase + key0 + c0 + e);
            dp1 *= drop_mul(dk, ebase + key0 + c0 + e + 1);
          }
          pd[e >> 1] = pack2v(f2mul(f2(pk[sub][e], pk[sub][e + 1]), f2sub(f2(dp0, dp1), Dx2)));
        }
        tmem_st_32x32b_x8(trow + 64 + pcol(c0), pd);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_ready);
    }
    const bool done = ok && mbar_wait(acc_full, 0, abort_flag, a.flags);
    if (done) {
      tc_fence_after();
      uint4* dst = reinterpret_cast<uint4*>(a.dqkv + (size_t)(row0 + qi) * (3 * a.H * 64) + (size_t)h * 64 + half * 32);
      const float f = a.scale;
      float cs[32];
#pragma unroll
      for (int c = 0; c < 2; c++) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(trow + 128 + half * 32 + c * 16, v);
        tmem_ld_wait();
        const float* x = reinterpret_cast<const float*>(v);
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; k++) {
          w[k] = pack2(x[2 * k] * f, x[2 * k + 1] * f);
          const float2 bk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
          cs[16 * c + 2 * k] = bk.x;  // the stored (bf16) values
          cs[16 * c + 2 * k + 1] = bk.y;
        }
        dst[2 * c] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[2 * c + 1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      if (a.colsum) {
        const float sq = warp_colsum32(cs, lane);
        block_colsum(reinterpret_cast<float*>(smem + Q_RED), half, quad, lane, sq, a.colsum,
                     (size_t)(row0 + qb * 128) / 128, 3L * a.H * 64, (long)h * 64 + 32 * half, a.colsum_acc);
      }
    } else if (a.colsum) {
      // every math warp takes part in the column-sum barriers, even on a failed wait
      for (int c2 = 0; c2 < 2; c2++) asm volatile("bar.sync 1, 256;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 256);
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

// [rows, slots, 64] bf16 viewed as 3-D {64, slots, rows}; box = one slot x box_rows rows
bool map_rows(CUtensorMap* m, const void* base, int slots, long rows, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)slots, (cuuint64_t)rows};
  cuuint64_t strides[2] = {128, (cuuint64_t)slots * 128};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
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
  a.o_out = reinterpret_cast<bf16*>(d.o);
  a.lse = d.lse;
  a.dsum = d.dsum;
  a.dqkv = reinterpret_cast<bf16*>(d.dqkv);
  a.scale = 0.125f;
  a.scale_log2 = 0.125f * LOG2E;
  a.drop = d.drop;
  a.flags = flags;
  a.colsum = d.colsum;
  a.colsum_acc = d.colsum_acc;
  return a;
}

}  // namespace

bool attn_tc_shape_ok(int T, int hd) { return hd == 64 && T > 0 && T % 128 == 0; }

bool attn_tc_supported(const AttnDesc& a) {
  if (!attn_tc_shape_ok(a.T, a.hd) || !encode_fn()) return false;
  if ((reinterpret_cast<uintptr_t>(a.qkv) & 15) || (reinterpret_cast<uintptr_t>(a.o) & 15)) return false;
  if (a.dout && (reinterpret_cast<uintptr_t>(a.dout) & 15)) return false;
  if (a.lse && (reinterpret_cast<uintptr_t>(a.lse) & 15)) return false;
  if (a.dsum && (reinterpret_cast<uintptr_t>(a.dsum) & 15)) return false;
  return true;
}

// The dynamic shared-memory limit is a per-device function attribute: it is
// set before every launch (a host-side call, not captured into graphs), so a
// model on any device of the process gets it.
bool attn_fwd_tc(Ctx& c, const AttnDesc& d) {
  CUtensorMap tq, tkv64;
  long rows = (long)d.B * d.T;
  if (!map_rows(&tq, d.qkv, 3 * d.H, rows, 128) || !map_rows(&tkv64, d.qkv, 3 * d.H, rows, 64)) return false;
  const bool drop = d.drop.active;
  cudaFuncSetAttribute(drop ? k_attn_fwd_o<true> : k_attn_fwd_o<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       D_SMEM);
  dim3 grid(d.B * d.H, d.T / 128);
  LaunchScope s(c, "attn_fwd_tc");
  if (drop) launch_pdl(k_attn_fwd_o<true>, grid, 192, D_SMEM, c.stream, tq, tkv64, make_args(d, c.flags));
  else launch_pdl(k_attn_fwd_o<false>, grid, 192, D_SMEM, c.stream, tq, tkv64, make_args(d, c.flags));
  return true;
}

bool attn_bwd_tc(Ctx& c, const AttnDesc& d) {
  CUtensorMap tkv, tkv64, tq64, tdo, tdo64, tout;
  long rows = (long)d.B * d.T;
  if (!map_rows(&tkv, d.qkv, 3 * d.H, rows, 128) || !map_rows(&tkv64, d.qkv, 3 * d.H, rows, 64) ||
      !map_rows(&tdo, d.dout, d.H, rows, 128) || !map_rows(&tdo64, d.dout, d.H, rows, 64) ||
      !map_rows(&tout, d.o, d.H, rows, 128))
    return false;
  tq64 = tkv64;
  const bool drop = d.drop.active;
  cudaFuncSetAttribute(drop ? k_attn_bwd_kv8<true> : k_attn_bwd_kv8<false>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize, K_SMEM);
  cudaFuncSetAttribute(drop ? k_attn_bwd_q8<true> : k_attn_bwd_q8<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       Q_SMEM);
  AttnTcArgs a = make_args(d, c.flags);
  dim3 grid(d.B * d.H, d.T / 128);
  {  // dQ first: it also stores D = rowsum(dO * O), which the dK/dV kernel reads
    LaunchScope s(c, "attn_bwd_q_tc");
    if (drop) launch_pdl(k_attn_bwd_q8<true>, grid, 320, Q_SMEM, c.stream, tkv, tdo, tkv64, tout, a);
    else launch_pdl(k_attn_bwd_q8<false>, grid, 320, Q_SMEM, c.stream, tkv, tdo, tkv64, tout, a);
  }
  {
    LaunchScope s(c, "attn_bwd_kv_tc");
    if (drop) launch_pdl(k_attn_bwd_kv8<true>, grid, 320, K_SMEM, c.stream, tkv, tq64, tdo64, a);
    else launch_pdl(k_attn_bwd_kv8<false>, grid, 320, K_SMEM, c.stream, tkv, tq64, tdo64, a);
  }
  return true;
}

}  // namespace gpt
