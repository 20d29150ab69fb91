// Backward pass of the causal latent attention on the 5th-generation tensor cores.
// (gist.science explainer, 4. Experimental Results: the backward pass of CCA is measured
// against MHA's; the gradients follow from Softmax(QK^T)V in the compressed space, 2. Methodik
// of the German edition.)
//
// With s the scale 1/sqrt(d~), P the causal softmax of s Q K^T per head (recomputed from the
// forward's per-row log-sum-exp), dP = dO V^T and D = rowsum(dO * O):
//   dS = P * (dP - D),   dQ = s dS K,   dK = s dS^T Q (summed over the group's heads),
//   dV = P^T dO (summed over the group's heads).
// Two kernels, so that no gradient needs atomics:
//   attn_bwd_dq_kernel    one CTA per (query head, sequence, 128-query tile): S = Q K_j^T and
//                         dP = dO V_j^T per key tile j into tensor memory, dS written back as
//                         float16 pairs, dQ += dS K_j with dS as the MMA's A operand from
//                         tensor memory and the staged K tile read as the (MN-major) B operand.
//   attn_bwd_dkdv_kernel  one CTA per (key/value head, sequence, 128-key tile), walking every
//                         (query tile, query head of the group) pair at or after the diagonal:
//                         S^T = K Q^T and dP^T = V dO^T with the keys on the tensor-memory
//                         lanes, P^T and dS^T written back as float16 pairs, then
//                         dV += P^T dO and dK += dS^T Q straight from tensor memory.
// Warps 0-15 compute the elementwise part, four per tensor-memory lane quadrant (one query or
// key row per thread, each warp on a quarter of the tile's 128 columns); warp 16 is the TMA
// producer, warp 17 issues the MMAs.  P / dS go to their own tensor-memory columns, so as soon as every
// elementwise warp has loaded its scores the next item's S / dP MMAs start, overlapping this
// item's exponentials; a commit after the gradient MMAs guards the P / dS columns.  Every wait
// is bounded; on a timeout the CTA records it in the status word, stops, and frees its TMEM.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int BT = 128;              // rows of every tile (queries or keys)
constexpr int B_EW = 16;             // elementwise warps: four per TMEM lane quadrant
constexpr int NPART = B_EW / 4;      // column parts of a tile per lane quadrant
constexpr int CW = BT / NPART;       // score columns (keys or queries) per elementwise warp
constexpr int BW_TMA = B_EW, BW_MMA = B_EW + 1;
constexpr int B_THREADS = (B_EW + 2) * 32;
constexpr int BSLOTS = 3;            // ring depth of the streamed tiles
// TMEM columns: S (or S^T) 0..127, dP (dP^T) 128..255, gradient accumulators from 256,
// the float16 pairs of P / dS (P^T / dS^T) the gradient MMAs read at 384..447 / 448..511
constexpr uint32_t C_S = 0, C_DP = 128, C_ACC = 256, C_P = 384, C_DS = 448;

template <int DL>
struct BwdCfg {
  static constexpr int ROWB = DL * 2;
  static constexpr int TILE = BT * ROWB;
  static constexpr uint32_t SW = ROWB == 128 ? 2u : ROWB == 64 ? 4u : 6u;
  static constexpr int SBO = 8 * ROWB;
  static_assert(C_ACC + 2 * DL <= C_P, "accumulators below the P / dS columns");
};

struct BwdBars {
  uint64_t first_full;               // dq: Q and dO; dkdv: K and V
  uint64_t a_full[BSLOTS], a_empty[BSLOTS];   // dq: K ring; dkdv: Q + dO ring
  uint64_t b_full[BSLOTS], b_empty[BSLOTS];   // dq: V ring
  uint64_t s_full, s_free, p_full, pds_free, done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}


// The elementwise warp's CW columns of S and dP (its part of the tile's 128) for its TMEM lane.
__device__ __forceinline__ void load_part(uint32_t base, uint32_t (&rs)[CW], uint32_t (&rp)[CW]) {
  static_assert(CW == 32, "one 32-column load each");
  tmem_ld32(base + C_S, rs);
  tmem_ld32(base + C_DP, rp);
  tmem_ld_wait();
}

// This warp's PW = DL / NPART accumulator columns [col, col + PW) of its lane, as floats.
template <int PW>
__device__ __forceinline__ void load_acc(uint32_t taddr, float (&o)[PW]) {
  if constexpr (PW == 4) {
    uint32_t r[4];
    tmem_ld4(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = __uint_as_float(r[e]);
  } else {
#pragma unroll
    for (int c = 0; c < PW / 8; ++c) {
      uint32_t r[8];
      tmem_ld8(taddr + c * 8, r);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 8; ++e) o[c * 8 + e] = __uint_as_float(r[e]);
    }
  }
}

// ------------------------------------------------------------------------------------ dQ
template <int DL>
__global__ void __launch_bounds__(B_THREADS, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap mapQ,
                       const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV,
                       const __grid_constant__ CUtensorMap mapDO, const float *__restrict__ lse,
                       const float *__restrict__ Dd, float *__restrict__ dq, int S, int H,
                       int Hkv, int G, float scale_log2, float scale, int *status) {
  using C = BwdCfg<DL>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *sQ = smem, *sDO = smem + C::TILE, *sK = smem + 2 * C::TILE;
  uint8_t *sV = sK + BSLOTS * C::TILE;
  BwdBars *bars = reinterpret_cast<BwdBars *>(sV + BSLOTS * C::TILE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, b = blockIdx.y;
  const int qt = static_cast<int>(gridDim.z) - 1 - static_cast<int>(blockIdx.z);  // long first
  const int g = h / G;
  const int nk = qt + 1;                               // key tiles 0..qt
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report(status, DEV_LAYOUT);
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(&bars->first_full, 1);
    for (int s = 0; s < BSLOTS; ++s) {
      mbar_init(&bars->a_full[s], 1);
      mbar_init(&bars->a_empty[s], 1);
      mbar_init(&bars->b_full[s], 1);
      mbar_init(&bars->b_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, B_EW);
    mbar_init(&bars->p_full, B_EW);
    mbar_init(&bars->pds_free, 1);
    mbar_init(&bars->done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == BW_MMA) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int *abort = &bars->abort;

  if (warp == BW_TMA) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars->first_full, 2 * C::TILE);
      tma_load_3d(sQ, &mapQ, &bars->first_full, 0, qt * BT, b * H + h);
      tma_load_3d(sDO, &mapDO, &bars->first_full, 0, h, b * S + qt * BT);
      for (int j = 0; j < nk; ++j) {
        const int s = j % BSLOTS;
        if (!mbar_wait(&bars->a_empty[s], ((j / BSLOTS) & 1) ^ 1u, abort, status)) break;
        mbar_arrive_expect_tx(&bars->a_full[s], C::TILE);
        tma_load_3d(sK + s * C::TILE, &mapK, &bars->a_full[s], 0, j * BT, b * Hkv + g);
        if (!mbar_wait(&bars->b_empty[s], ((j / BSLOTS) & 1) ^ 1u, abort, status)) break;
        mbar_arrive_expect_tx(&bars->b_full[s], C::TILE);
        tma_load_3d(sV + s * C::TILE, &mapV, &bars->b_full[s], 0, j * BT, b * Hkv + g);
      }
    }
  } else if (warp == BW_MMA) {
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_f16_f32(BT, BT, 0, 0, 1);
    constexpr uint32_t idesc_q = idesc_f16_f32(BT, DL, 0, 1, 1);
    auto issue_s = [&](int j) {                      // S = Q K_j^T, dP = dO V_j^T
      const int s = j % BSLOTS;
      const uint64_t qd = smem_desc(smem_u32(sQ), 16, C::SBO, C::SW);
      const uint64_t dod = smem_desc(smem_u32(sDO), 16, C::SBO, C::SW);
      const uint64_t kd = smem_desc(smem_u32(sK + s * C::TILE), 16, C::SBO, C::SW);
      const uint64_t vd = smem_desc(smem_u32(sV + s * C::TILE), 16, C::SBO, C::SW);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < DL / 16; ++kk) {
          umma_f16_ss(tmem + C_S, qd + 2 * kk, kd + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
          umma_f16_ss(tmem + C_DP, dod + 2 * kk, vd + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full);
        umma_commit(&bars->b_empty[s]);              // V_j is read only by dP
      }
      __syncwarp();
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->first_full, 0, abort, status) &&
                                          mbar_wait(&bars->a_full[0], 0, abort, status) &&
                                          mbar_wait(&bars->b_full[0], 0, abort, status));
    if (ok) {
      tc_fence_after();
      issue_s(0);
    }
    for (int j = 0; ok && j < nk; ++j) {
      const int s = j % BSLOTS;
      if (j + 1 < nk) {                              // next tile's S / dP once this one is read
        const int s1 = (j + 1) % BSLOTS;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_free, j & 1, abort, status) &&
                                         mbar_wait(&bars->a_full[s1], ((j + 1) / BSLOTS) & 1, abort, status) &&
                                         mbar_wait(&bars->b_full[s1], ((j + 1) / BSLOTS) & 1, abort, status));
        if (!ok) break;
        tc_fence_after();
        issue_s(j + 1);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->p_full, j & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      // dQ += dS K_j: dS (float16 pairs) as A from TMEM, K_j as the MN-major B
      const uint64_t kb = smem_desc(smem_u32(sK + s * C::TILE), C::TILE, C::SBO, C::SW);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk)
          umma_f16_ts(tmem + C_ACC, tmem + C_DS + kk * 8, kb + kk * (2 * C::SBO / 16), idesc_q,
                      (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&bars->pds_free);
        umma_commit(&bars->a_empty[s]);
        if (j + 1 == nk) umma_commit(&bars->done);
      }
      __syncwarp();
    }
  } else {
    const int quad = warp & 3, hf = warp >> 2;       // lanes of quadrant, key columns of part
    const int row = quad * 32 + lane;
    const int qpos = qt * BT + row;
    const bool valid = qpos < S;
    const size_t ridx = (static_cast<size_t>(b) * H + h) * S + (valid ? qpos : 0);
    const float lrow = valid ? lse[ridx] : INFINITY;   // invalid rows: every p is 0
    const float drow = valid ? Dd[ridx] : 0.f;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t base = tmem + lane_off + hf * CW;
    bool ok = true;
    for (int j = 0; ok && j < nk; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, j & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      uint32_t rs[CW], rp[CW];
      load_part(base, rs, rp);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free);    // the next tile's S / dP may overwrite
      // dS = P * (dP - D) on pairs of keys: one packed FMA for the exponents, two MUFU ex2,
      // packed subtract and multiply; keys past this row's query masked on the diagonal tile
      const bool diag = j == qt;
      const uint64_t sc2 = f2(scale_log2, scale_log2), nl2 = f2(-lrow, -lrow), nd2 = f2(-drow, -drow);
      uint32_t pk[CW / 2];
#pragma unroll
      for (int e = 0; e < CW / 2; ++e) {
        float x0, x1;
        unf2(fma2(f2(__uint_as_float(rs[2 * e]), __uint_as_float(rs[2 * e + 1])), sc2, nl2), x0, x1);
        float p0 = ex2(x0), p1 = ex2(x1);
        if (diag) {
          const int kcol = hf * CW + 2 * e;
          if (kcol > row) p0 = 0.f;
          if (kcol + 1 > row) p1 = 0.f;
        }
        const uint64_t t2 = add2(f2(__uint_as_float(rp[2 * e]), __uint_as_float(rp[2 * e + 1])), nd2);
        float d0, d1;
        unf2(mul2(f2(p0, p1), t2), d0, d1);
        pk[e] = pack_f16x2(d0, d1);
      }
      // the previous tile's dQ MMA must have read its dS before this one is written
      if (j > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->pds_free, (j - 1) & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      tmem_st16(tmem + lane_off + C_DS + hf * (CW / 2), pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->done, 0, abort, status));
    if (ok) {
      tc_fence_after();
      constexpr int PW = DL / NPART;                 // this part's dQ columns
      float o[PW];
      load_acc<PW>(tmem + lane_off + C_ACC + hf * PW, o);
      if (valid) {
        float *dst = dq + ridx * DL + hf * PW;
#pragma unroll
        for (int c = 0; c < PW / 4; ++c)
          reinterpret_cast<float4 *>(dst)[c] = make_float4(o[4 * c] * scale, o[4 * c + 1] * scale,
                                                           o[4 * c + 2] * scale, o[4 * c + 3] * scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == BW_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------- dK dV
template <int DL>
__global__ void __launch_bounds__(B_THREADS, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap mapQ,
                         const __grid_constant__ CUtensorMap mapK,
                         const __grid_constant__ CUtensorMap mapV,
                         const __grid_constant__ CUtensorMap mapDO, const float *__restrict__ lse,
                         const float *__restrict__ Dd, float *__restrict__ dk,
                         float *__restrict__ dv, int S, int H, int Hkv, int G, int nqt,
                         float scale_log2, float scale, int *status) {
  using C = BwdCfg<DL>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t *sK = smem, *sV = smem + C::TILE, *sQ = smem + 2 * C::TILE;
  uint8_t *sDO = sQ + BSLOTS * C::TILE;
  // per elementwise warp: [2 items][-lse 32 | -D 32] of its 32 query columns
  float *sL = reinterpret_cast<float *>(sDO + BSLOTS * C::TILE);
  BwdBars *bars = reinterpret_cast<BwdBars *>(sL + B_EW * 2 * 2 * CW);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x, b = blockIdx.y, kt = blockIdx.z;       // small kt: most work first
  const int nitems = G * (nqt - kt);                // (query tile kt + n / G, head g*G + n % G)
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report(status, DEV_LAYOUT);
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(&bars->first_full, 1);
    for (int s = 0; s < BSLOTS; ++s) {
      mbar_init(&bars->a_full[s], 1);
      mbar_init(&bars->a_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, B_EW);
    mbar_init(&bars->p_full, B_EW);
    mbar_init(&bars->pds_free, 1);
    mbar_init(&bars->done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == BW_MMA) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int *abort = &bars->abort;

  if (warp == BW_TMA) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars->first_full, 2 * C::TILE);
      tma_load_3d(sK, &mapK, &bars->first_full, 0, kt * BT, b * Hkv + g);
      tma_load_3d(sV, &mapV, &bars->first_full, 0, kt * BT, b * Hkv + g);
      for (int n = 0; n < nitems; ++n) {
        const int s = n % BSLOTS;
        const int qt = kt + n / G, h = g * G + n % G;
        if (!mbar_wait(&bars->a_empty[s], ((n / BSLOTS) & 1) ^ 1u, abort, status)) break;
        mbar_arrive_expect_tx(&bars->a_full[s], 2 * C::TILE);
        tma_load_3d(sQ + s * C::TILE, &mapQ, &bars->a_full[s], 0, qt * BT, b * H + h);
        tma_load_3d(sDO + s * C::TILE, &mapDO, &bars->a_full[s], 0, h, b * S + qt * BT);
      }
    }
  } else if (warp == BW_MMA) {
    const bool leader = elect_one();
    constexpr uint32_t idesc_s = idesc_f16_f32(BT, BT, 0, 0, 1);
    constexpr uint32_t idesc_o = idesc_f16_f32(BT, DL, 0, 1, 1);
    auto issue_s = [&](int n) {                      // S^T = K Q^T, dP^T = V dO^T
      const int s = n % BSLOTS;
      const uint64_t kd = smem_desc(smem_u32(sK), 16, C::SBO, C::SW);
      const uint64_t vd = smem_desc(smem_u32(sV), 16, C::SBO, C::SW);
      const uint64_t qd = smem_desc(smem_u32(sQ + s * C::TILE), 16, C::SBO, C::SW);
      const uint64_t dod = smem_desc(smem_u32(sDO + s * C::TILE), 16, C::SBO, C::SW);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < DL / 16; ++kk) {
          umma_f16_ss(tmem + C_S, kd + 2 * kk, qd + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
          umma_f16_ss(tmem + C_DP, vd + 2 * kk, dod + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full);
      }
      __syncwarp();
    };
    bool ok = nitems > 0 &&
              __all_sync(0xffffffffu, mbar_wait(&bars->first_full, 0, abort, status) &&
                                          mbar_wait(&bars->a_full[0], 0, abort, status));
    if (ok) {
      tc_fence_after();
      issue_s(0);
    }
    for (int n = 0; ok && n < nitems; ++n) {
      const int s = n % BSLOTS;
      if (n + 1 < nitems) {                          // the next item's S^T / dP^T once read
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_free, n & 1, abort, status) &&
                                         mbar_wait(&bars->a_full[(n + 1) % BSLOTS], ((n + 1) / BSLOTS) & 1, abort, status));
        if (!ok) break;
        tc_fence_after();
        issue_s(n + 1);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->p_full, n & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      // dV += P^T dO and dK += dS^T Q, A operands from tensor memory, the item's dO and Q tiles
      // as MN-major B operands
      const uint64_t dob = smem_desc(smem_u32(sDO + s * C::TILE), C::TILE, C::SBO, C::SW);
      const uint64_t qb = smem_desc(smem_u32(sQ + s * C::TILE), C::TILE, C::SBO, C::SW);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < BT / 16; ++kk) {
          umma_f16_ts(tmem + C_ACC, tmem + C_P + kk * 8, dob + kk * (2 * C::SBO / 16), idesc_o,
                      (n > 0 || kk > 0) ? 1u : 0u);
          umma_f16_ts(tmem + C_ACC + DL, tmem + C_DS + kk * 8, qb + kk * (2 * C::SBO / 16),
                      idesc_o, (n > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->pds_free);
        umma_commit(&bars->a_empty[s]);
        if (n + 1 == nitems) umma_commit(&bars->done);
      }
      __syncwarp();
    }
  } else {
    const int quad = warp & 3, hf = warp >> 2;       // lanes of quadrant, query columns of part
    const int row = quad * 32 + lane;
    const int kpos = kt * BT + row;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t base = tmem + lane_off + hf * CW;
    // each warp stages the negated lse and D of its own 32 query columns one item ahead in its
    // own shared-memory slice (lane i the i-th column), so only __syncwarp orders them
    float *wsl = sL + warp * 2 * 2 * CW;
    auto stage_stats = [&](int n) {
      if (n >= nitems) return;
      const int qt = kt + n / G, h = g * G + n % G;
      const int q = qt * BT + hf * CW + lane;
      const size_t ridx = (static_cast<size_t>(b) * H + h) * S + q;
      float *buf = wsl + (n & 1) * 2 * CW;
      buf[lane] = q < S ? -lse[ridx] : -INFINITY;
      buf[CW + lane] = q < S ? -Dd[ridx] : 0.f;
    };
    static_assert(CW == 32, "a lane per query column");
    stage_stats(0);
    bool ok = true;
    for (int n = 0; n < nitems; ++n) {
      __syncwarp();                                  // stats of item n visible, n-1's read
      stage_stats(n + 1);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, n & 1, abort, status)) && ok;
      tc_fence_after();
      uint32_t rs[CW], rp[CW];
      load_part(base, rs, rp);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free);
      const int qt = kt + n / G;
      const bool diag = qt == kt;
      // per query column: -lse and -D (broadcast 8-byte shared-memory reads), then P^T and
      // dS^T on pairs of queries with packed FMA / subtract / multiply
      const float *bl = wsl + (n & 1) * 2 * CW, *bd = bl + CW;
      const uint64_t sc2 = f2(scale_log2, scale_log2);
      uint32_t pkp[CW / 2], pks[CW / 2];
#pragma unroll
      for (int e = 0; e < CW / 2; ++e) {
        const float2 nl = *reinterpret_cast<const float2 *>(bl + 2 * e);
        const float2 nd = *reinterpret_cast<const float2 *>(bd + 2 * e);
        float x0, x1;
        unf2(fma2(f2(__uint_as_float(rs[2 * e]), __uint_as_float(rs[2 * e + 1])), sc2, f2(nl.x, nl.y)), x0, x1);
        float p0 = ex2(x0), p1 = ex2(x1);
        if (diag) {                                  // a query before this key
          const int qcol = hf * CW + 2 * e;
          if (qcol < row) p0 = 0.f;
          if (qcol + 1 < row) p1 = 0.f;
        }
        const uint64_t t2 = add2(f2(__uint_as_float(rp[2 * e]), __uint_as_float(rp[2 * e + 1])), f2(nd.x, nd.y));
        float d0, d1;
        unf2(mul2(f2(p0, p1), t2), d0, d1);
        pkp[e] = pack_f16x2(p0, p1);
        pks[e] = pack_f16x2(d0, d1);
      }
      // the previous item's dV / dK MMAs must have read P^T / dS^T before they are rewritten
      if (n > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->pds_free, (n - 1) & 1, abort, status)) && ok;
      tc_fence_after();
      tmem_st16(tmem + lane_off + C_P + hf * (CW / 2), pkp);
      tmem_st16(tmem + lane_off + C_DS + hf * (CW / 2), pks);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (nitems > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bars->done, 0, abort, status)) && ok;
    if (ok) {
      tc_fence_after();
      const bool valid = kpos < S;
      const size_t ridx = (static_cast<size_t>(b) * Hkv + g) * S + (valid ? kpos : 0);
      constexpr int PW = DL / NPART;                 // this part's dV / dK columns
      float ov[PW], ok2[PW];
      load_acc<PW>(tmem + lane_off + C_ACC + hf * PW, ov);
      load_acc<PW>(tmem + lane_off + C_ACC + DL + hf * PW, ok2);
      if (valid && nitems > 0) {
        float *pv = dv + ridx * DL + hf * PW, *pk = dk + ridx * DL + hf * PW;
#pragma unroll
        for (int c = 0; c < PW / 4; ++c) {
          reinterpret_cast<float4 *>(pv)[c] = make_float4(ov[4 * c], ov[4 * c + 1], ov[4 * c + 2], ov[4 * c + 3]);
          reinterpret_cast<float4 *>(pk)[c] = make_float4(ok2[4 * c] * scale, ok2[4 * c + 1] * scale,
                                                          ok2[4 * c + 2] * scale, ok2[4 * c + 3] * scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == BW_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D[b, h, t] = sum_i dO[b*S + t, h*DL + i] * O[b*S + t, h*DL + i]  (one warp per (token, head))
__global__ void __launch_bounds__(256) rowdot_kernel(const __half *__restrict__ dO,
                                                     const __half *__restrict__ O,
                                                     float *__restrict__ D, int B, int S, int H,
                                                     int DL) {
  const long long item = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (item >= static_cast<long long>(B) * S * H) return;
  const long long bt = item / H;
  const int h = static_cast<int>(item % H);
  const size_t base = static_cast<size_t>(bt) * H * DL + static_cast<size_t>(h) * DL;
  float acc = 0.f;
  for (int i = lane; i < DL; i += 32) acc += __half2float(dO[base + i]) * __half2float(O[base + i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const int b = static_cast<int>(bt / S), t = static_cast<int>(bt % S);
    D[(static_cast<size_t>(b) * H + h) * S + t] = acc;
  }
}

template <int DL>
cudaError_t launch_bwd(const Dims &d, const AttnBwdArgs &a, cudaStream_t st) {
  using C = BwdCfg<DL>;
  const uint64_t row = static_cast<uint64_t>(DL) * 2;
  CUtensorMap mq, mk, mv, mdo;
  const uint32_t box[3] = {static_cast<uint32_t>(DL), static_cast<uint32_t>(BT), 1u};
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(DL), static_cast<uint64_t>(d.S),
                              static_cast<uint64_t>(d.B) * d.H};
    const uint64_t strides[2] = {row, row * d.S};
    if (!make_tma_16bit(&mq, a.q, 3, dims, strides, box, C::ROWB, 1)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(DL), static_cast<uint64_t>(d.S),
                              static_cast<uint64_t>(d.B) * d.Hkv};
    const uint64_t strides[2] = {row, row * static_cast<uint64_t>(a.kv_stride)};
    if (!make_tma_16bit(&mk, a.k, 3, dims, strides, box, C::ROWB, 1) ||
        !make_tma_16bit(&mv, a.v, 3, dims, strides, box, C::ROWB, 1))
      return cudaErrorInvalidValue;
  }
  {
    // dO [B*S, H*DL] token-major: dims {DL, H, B*S}, a box is one head's DL columns of 128 tokens
    const uint64_t dims[3] = {static_cast<uint64_t>(DL), static_cast<uint64_t>(d.H),
                              static_cast<uint64_t>(d.B) * d.S};
    const uint64_t strides[2] = {row, row * d.H};
    const uint32_t boxo[3] = {static_cast<uint32_t>(DL), 1u, static_cast<uint32_t>(BT)};
    if (!make_tma_16bit(&mdo, a.dO, 3, dims, strides, boxo, C::ROWB, 1)) return cudaErrorInvalidValue;
  }
  const float scale = static_cast<float>(1.0 / sqrt(static_cast<double>(DL)));
  const float scale_log2 = static_cast<float>(1.4426950408889634) * scale;
  const int nt = (d.S + BT - 1) / BT;
  const size_t smem_dq = (2 + 2 * BSLOTS) * C::TILE + sizeof(BwdBars);
  const size_t smem_kv = (2 + 2 * BSLOTS) * C::TILE + B_EW * 2 * 2 * CW * 4 + sizeof(BwdBars);
  cudaError_t e;
  if ((e = ensure_dyn_smem<attn_bwd_dq_kernel<DL>>(smem_dq)) != cudaSuccess) return e;
  if ((e = ensure_dyn_smem<attn_bwd_dkdv_kernel<DL>>(smem_kv)) != cudaSuccess) return e;
  attn_bwd_dkdv_kernel<DL><<<dim3(d.Hkv, d.B, nt), B_THREADS, smem_kv, st>>>(
      mq, mk, mv, mdo, a.lse, a.D, a.dk, a.dv, d.S, d.H, d.Hkv, d.G, nt, scale_log2, scale, a.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  attn_bwd_dq_kernel<DL><<<dim3(d.H, d.B, nt), B_THREADS, smem_dq, st>>>(
      mq, mk, mv, mdo, a.lse, a.D, a.dq, d.S, d.H, d.Hkv, d.G, scale_log2, scale, a.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t attention_rowdot(const Dims &d, const void *dO, const void *O, float *D,
                             cudaStream_t st) {
  const long long items = static_cast<long long>(d.B) * d.S * d.H;
  if (items == 0) return cudaSuccess;
  rowdot_kernel<<<static_cast<unsigned>((items + 7) / 8), 256, 0, st>>>(
      static_cast<const __half *>(dO), static_cast<const __half *>(O), D, d.B, d.S, d.H, d.DL);
  return cudaGetLastError();
}

cudaError_t latent_attention_backward(const Dims &d, const AttnBwdArgs &a, cudaStream_t st) {
  if (d.B == 0 || d.S == 0) return cudaSuccess;
  if (d.DL == 16) return launch_bwd<16>(d, a, st);
  if (d.DL == 32) return launch_bwd<32>(d, a, st);
  if (d.DL == 64) return launch_bwd<64>(d, a, st);
  return cudaErrorInvalidValue;
}

}  // namespace cca
