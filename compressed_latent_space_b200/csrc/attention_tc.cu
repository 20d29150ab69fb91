// Causal latent attention for 16-bit layers on the 5th-generation tensor cores.
//
//   O[b, t, h*d~ + :] = sum_{s <= t} softmax_s(q[b,h,t] . k[b,g,s] / sqrt(d~)) v[b,g,s],
//   g = h / (H/Hkv)
// (gist.science/de explainer, 2. Methodik: Softmax(QK^T)V evaluated entirely in the
// compressed space; gist.science explainer, Extension: CCGQA.)
//
// One CTA per SM owns NTILE (3; 2 at d~ = 128) query tiles of 128 rows and streams the TN-key
// (96) tiles of their key/value head once for all of them (causal: a tile reads the key tiles
// through its last row).  A query tile packs GP query heads of one key/value group (GP = the
// largest power of two dividing G, at most 8) over 128/GP consecutive tokens: row r of the tile
// is head h0 + r / (128/GP) at token qbase + r % (128/GP).  So every K/V tile staged in shared
// memory serves GP heads of the group in each of the NTILE tiles (GQA head reuse), and the
// tiles of a CTA cover only NTILE * 128/GP tokens, so their causal ranges differ by at most one
// key tile.  The tiles take turns on the tensor cores, so each tile's softmax runs while the
// others' MMAs execute, and three softmax warps per scheduler keep the exponential unit busier
// than two (the softmax, not the tensor pipe, bounds this kernel at d~ <= 64):
//   warps 4t..4t+3 : softmax of tile t.  One query row per thread (warp w reads TMEM lanes
//               32*(w%4)..), all TN keys of a tile in registers.  Online softmax in fp32 with
//               lazy rescaling (the reference max only moves when a row max grows by more than
//               2^8, and then the warp rescales its rows of O); the probabilities are packed to
//               float16 pairs and written over the tile's own scores in TMEM, where the P*V
//               MMA reads them as its A operand.  Key tiles that straddle the diagonal are
//               masked per row, with each row's own token index.
//   warp W_TMA : TMA producer: the Q tiles once, then K and V tiles into two rings.
//   warp W_MMA : allocates TMEM (S_t: TN fp32 columns each; O_t: d~ each, from a 64-aligned
//               column) and issues the MMAs (whole warp runs the loop, one elected lane
//               issues).  Per key tile j and tile t: O_t += P_t V_j, S_t = Q_t K_{j+1}^T.  The
//               tensor pipe executes in issue order, so a tile's next S overwrites its P only
//               after P*V has read it, and a tile's O is final for the softmax whenever its
//               next S is ready.
// Rows of q, k and v wider than 128 bytes (d~ = 128) are staged as 64-column chunks, each a
// [rows x 128 B] block in the 128-byte swizzled layout; QK^T walks the chunks along K, and the
// P*V MMA reads V's two chunks as the N halves of its B operand.
// Every wait is bounded; on a timeout the CTA records it in the status word, stops, and
// releases its tensor memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int TM = 128;          // query rows per tile (M of all MMAs)
constexpr int TN = 96;           // keys per tile
constexpr int MAXTILE = 3;
constexpr float kTau = 8.0f;     // lazy-rescale threshold, log2 units

template <int DL>
struct AttnCfg {
  static constexpr int NTILE = DL == 128 ? 2 : 3;      // query tiles per CTA
  static constexpr int NSOFT = 4 * NTILE;              // softmax warps: 4 per query tile
  static constexpr int W_TMA = NSOFT, W_MMA = NSOFT + 1;
  static constexpr int THREADS = (NSOFT + 2) * 32;
  static constexpr int SK = DL == 128 ? 3 : 4;         // K ring depth
  static constexpr int SV = SK;                        // V ring depth
  static constexpr int NCH = DL == 128 ? 2 : 1;        // 64-column chunks per row
  static constexpr int CW = DL / NCH;                  // columns per chunk
  static constexpr int ROWB = CW * 2;                  // bytes of one chunk row (<= 128)
  static constexpr int Q_CHUNK = TM * ROWB;
  static constexpr int Q_BYTES = NCH * Q_CHUNK;
  static constexpr int KV_CHUNK = TN * ROWB;
  static constexpr int KV_BYTES = NCH * KV_CHUNK;      // one K or one V tile
  static constexpr uint32_t SW_MODE = ROWB == 128 ? 2u : ROWB == 64 ? 4u : 6u;
  static constexpr int SBO = 8 * ROWB;                 // stride of 8-row core groups
  static constexpr int OFF_Q = 0;                      // the NTILE query tiles
  static constexpr int OFF_K = OFF_Q + NTILE * Q_BYTES;
  static constexpr int OFF_V = OFF_K + SK * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + SV * KV_BYTES;
  static constexpr int SMEM = OFF_BAR + 512;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_O = (NTILE * TN + 63) / 64 * 64;  // S_t at t * TN; O_t 64-aligned
  static_assert(COL_O + NTILE * DL <= TMEM_COLS, "S and O of all tiles must fit the TMEM allocation");
  static_assert(NTILE <= MAXTILE && SK <= 4, "barrier arrays");
  static_assert(Q_CHUNK % 1024 == 0 && KV_CHUNK % 1024 == 0, "swizzled chunks stay 1024-aligned");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

struct AttnBars {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4];
  uint64_t v_full[4], v_empty[4];
  uint64_t s_full[MAXTILE], p_full[MAXTILE], o_done[MAXTILE];
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// true in exactly one lane of the (converged) warp
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

template <int DL>
__global__ void __launch_bounds__(AttnCfg<DL>::THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap mapQ,
                   const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, __half *__restrict__ O, int S,
                   int H, int Hkv, int G, int gp_log2, int nqt, float scale_log2, int *status,
                   float *__restrict__ lse) {
  using C = AttnCfg<DL>;
  constexpr int NTILE = C::NTILE;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tok_log2 = 7 - gp_log2;                 // a tile holds 2^tok_log2 tokens per head
  const int TT = 1 << tok_log2;
  const int h0 = blockIdx.x << gp_log2, b = blockIdx.y;   // heads h0 .. h0 + GP - 1
  const int grp = static_cast<int>(gridDim.z) - 1 - static_cast<int>(blockIdx.z);  // long first
  const int qt0 = NTILE * grp;                       // token blocks qt0 .. qt0 + ntile - 1
  const int ntile = min(NTILE, nqt - qt0);
  // key tiles of query tile t: through its last token (the diagonal band is masked)
  auto nkv = [&](int t) { return ((qt0 + t + 1) * TT + TN - 1) / TN; };
  const int nsteps = nkv(ntile - 1);
  const int g = h0 / G;
  AttnBars *bars = reinterpret_cast<AttnBars *>(smem + C::OFF_BAR);

  // The swizzled tiles need 1024-byte alignment; refuse to run otherwise.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report(status, DEV_LAYOUT);
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < 4; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int t = 0; t < MAXTILE; ++t) {
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 4);
      mbar_init(&bars->o_done[t], 1);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == C::W_MMA) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int *abort = &bars->abort;

  if (warp == C::W_TMA) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      mbar_arrive_expect_tx(&bars->q_full, ntile * C::Q_BYTES);
      // a Q box is {chunk columns, TT tokens, GP heads}: GP x TT = 128 rows, head-major
      for (int t = 0; t < ntile; ++t)
        for (int c = 0; c < C::NCH; ++c)
          tma_load_3d(smem + C::OFF_Q + t * C::Q_BYTES + c * C::Q_CHUNK, &mapQ, &bars->q_full,
                      c * C::CW, (qt0 + t) * TT, b * H + h0);
      for (int j = 0; j < nsteps; ++j) {
        const int sk = j % C::SK, sv = j % C::SV;
        if (!mbar_wait(&bars->k_empty[sk], ((j / C::SK) & 1) ^ 1u, abort, status)) break;
        mbar_arrive_expect_tx(&bars->k_full[sk], C::KV_BYTES);
        for (int c = 0; c < C::NCH; ++c)
          tma_load_3d(smem + C::OFF_K + sk * C::KV_BYTES + c * C::KV_CHUNK, &mapK,
                      &bars->k_full[sk], c * C::CW, j * TN, b * Hkv + g);
        if (!mbar_wait(&bars->v_empty[sv], ((j / C::SV) & 1) ^ 1u, abort, status)) break;
        mbar_arrive_expect_tx(&bars->v_full[sv], C::KV_BYTES);
        for (int c = 0; c < C::NCH; ++c)
          tma_load_3d(smem + C::OFF_V + sv * C::KV_BYTES + c * C::KV_CHUNK, &mapV,
                      &bars->v_full[sv], c * C::CW, j * TN, b * Hkv + g);
      }
    }
  } else if (warp == C::W_MMA) {
    // ---------------------------------------------------------------- MMA issuer
    // Descriptors advance by adding to their start-address field (16-byte units): 32 bytes
    // per 16-wide K step of Q / K inside a chunk, a whole chunk after every 128 bytes of row;
    // 16 keys of V are 2*SBO bytes.  V's chunks are the N halves of P*V's B operand (leading
    // byte offset = one chunk).
    const bool leader = elect_one();
    constexpr uint32_t idesc_qk = idesc_f16_f32(TM, TN, 0, 0, 1);
    constexpr uint32_t idesc_pv = idesc_f16_f32(TM, DL, 0, 1, 1);
    constexpr int KSTEPS = DL / 16, KPC = C::CW / 16;  // K steps in all, per chunk
    auto issue_qk = [&](int t, int j) {              // S_t = Q_t K_j^T
      const uint64_t qd = smem_desc(smem_u32(smem + C::OFF_Q + t * C::Q_BYTES), 16, C::SBO, C::SW_MODE);
      const uint64_t kd = smem_desc(smem_u32(smem + C::OFF_K + (j % C::SK) * C::KV_BYTES), 16,
                                    C::SBO, C::SW_MODE);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const uint32_t qo = ((kk / KPC) * C::Q_CHUNK + (kk % KPC) * 32) >> 4;
          const uint32_t ko = ((kk / KPC) * C::KV_CHUNK + (kk % KPC) * 32) >> 4;
          umma_f16_ss(tmem + t * TN, qd + qo, kd + ko, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[t]);
      }
      __syncwarp();
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->q_full, 0, abort, status) &&
                                          mbar_wait(&bars->k_full[0], 0, abort, status));
    if (ok) {
      tc_fence_after();
      for (int t = 0; t < ntile; ++t) issue_qk(t, 0);
      if (leader) umma_commit(&bars->k_empty[0]);
      __syncwarp();
    }
    for (int j = 0; ok && j < nsteps; ++j) {
      const int sv = j % C::SV;
      const bool nextK = j + 1 < nsteps;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->v_full[sv], (j / C::SV) & 1, abort, status));
      if (ok && nextK)
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->k_full[(j + 1) % C::SK],
                                               ((j + 1) / C::SK) & 1, abort, status));
      if (!ok) break;
      const uint64_t vd = smem_desc(smem_u32(smem + C::OFF_V + sv * C::KV_BYTES), C::KV_CHUNK,
                                    C::SBO, C::SW_MODE);
      for (int t = 0; t < ntile; ++t) {
        const int nk = nkv(t);
        if (j >= nk) continue;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->p_full[t], j & 1, abort, status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + t * TN, tO = tmem + C::COL_O + t * DL;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < TN / 16; ++kk)    // 16 keys of P = 8 TMEM columns of f16 pairs
            umma_f16_ts(tO, tS + kk * 8, vd + kk * (2 * C::SBO / 16), idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
          if (j + 1 >= nk) umma_commit(&bars->o_done[t]);
        }
        __syncwarp();
        if (j + 1 < nk) issue_qk(t, j + 1);       // runs after this P*V: it overwrites P_t
      }
      if (!ok) break;
      if (leader) {
        umma_commit(&bars->v_empty[sv]);
        if (nextK) umma_commit(&bars->k_empty[(j + 1) % C::SK]);
      }
      __syncwarp();
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int t = warp >> 2, quad = warp & 3;
    const int row = quad * 32 + lane;                 // TMEM lane of this thread
    const int nk = nkv(t);
    const int qbase = (qt0 + t) * TT;                 // first token of this tile
    const int qpos = qbase + (row & (TT - 1));        // this row's token
    const int hrow = h0 + (row >> tok_log2);          // and its query head
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + t * TN + lane_off, tO = tmem + C::COL_O + t * DL + lane_off;
    const uint64_t sc2 = f2(scale_log2, scale_log2);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = t < ntile;
    for (int j = 0; ok && j < nk; ++j) {
      // S_t of tile j is ready, and every earlier MMA (this tile's P*V of j-1) is done
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[t], j & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      uint32_t r[TN];
#pragma unroll
      for (int c = 0; c < TN / 32; ++c)
        tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
      tmem_ld_wait();
      // Row max of the raw scores (the 1/sqrt(d~) * log2(e) scale is positive, so it is
      // applied afterwards), in four independent three-input chains.  Keys past this row's
      // position are masked on the tiles of the diagonal band only.
      if ((j + 1) * TN > qbase) {                     // a tile of the diagonal band
        const int last = qpos - j * TN;               // keys 0..last of this tile are visible
#pragma unroll
        for (int i = 0; i < TN; ++i)
          if (i > last) r[i] = __float_as_uint(-INFINITY);
      }
      static_assert(TN % 8 == 0, "four chains of pairs cover the tile");
      float mx4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        mx4[e] = fmaxf(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
#pragma unroll
      for (int i = 8; i < TN; i += 8)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          mx4[e] = max3(mx4[e], __uint_as_float(r[i + 2 * e]), __uint_as_float(r[i + 2 * e + 1]));
      // mx is -inf when a diagonal-band tile starts past this row's token (every score masked);
      // then resc is false and every p below is exp2(-inf) = 0, which is safe because key tile
      // 0 always holds a visible key (key 0), so m_ref is finite from j = 0 on.
      const float mx = max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * scale_log2;
      const bool resc = mx > m_ref + kTau;
      const float scale = resc ? ex2(m_ref - mx) : 1.f;
      if (resc) m_ref = mx;
      l *= scale;
      // O is final up to tile j-1 here; the tcgen05 loads and stores are warp-wide, so the
      // warp rescales together, with factor 1 in rows that keep their max
      if (j > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll
        for (int c = 0; c < DL / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tO + c * 16, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * scale);
          tmem_st16(tO + c * 16, o);
        }
      }
      // p = 2^(s * scale - m_ref): pairs scaled with one packed FMA, one MUFU ex2 each (at
      // d~ <= 64, where the exponential unit is the kernel's busiest pipe, three pairs in
      // sixteen by a cubic on the FMA pipes instead), rounded to float16 pairs (written over
      // this tile's scores), four paired partial sums.
      const uint64_t nm2 = f2(-m_ref, -m_ref);
      uint64_t l2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) l2[e] = 0;
#pragma unroll
      for (int c = 0; c < TN / 32; ++c) {             // 32 keys -> 16 TMEM columns
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = c * 32 + 2 * e;
          const uint64_t x2 = fma2(f2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), sc2, nm2);
          float p0, p1;
          if (DL < 128 && e % 5 == 4) {               // pairs 4, 9, 14 of 16: FMA pipes
            ex2_poly2(x2, p0, p1);
          } else {
            float x0, x1;
            unf2(x2, x0, x1);
            p0 = ex2(x0);
            p1 = ex2(x1);
          }
          l2[e & 3] = add2(l2[e & 3], f2(p0, p1));
          pk[e] = pack_f16x2(p0, p1);
        }
        tmem_st16(tS + c * 16, pk);
      }
      {
        const uint64_t s01 = add2(add2(l2[0], l2[1]), add2(l2[2], l2[3]));
        float a0, a1;
        unf2(s01, a0, a1);
        l += a0 + a1;
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[t]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_done[t], 0, abort, status));
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __half *dst = O + (static_cast<size_t>(b) * S + qpos) * (static_cast<size_t>(H) * DL) + hrow * DL;
#pragma unroll
      for (int c = 0; c < DL / 8; ++c) {
        uint32_t o[8];
        tmem_ld8(tO + c * 8, o);
        tmem_ld_wait();
        uint4 u;
        u.x = pack_f16x2(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
        u.y = pack_f16x2(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
        u.z = pack_f16x2(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
        u.w = pack_f16x2(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
        if (qpos < S) reinterpret_cast<uint4 *>(dst)[c] = u;
      }
      // log2-domain log-sum-exp of the row's scaled scores, for the backward pass:
      // p = 2^(s * scale * log2(e) - lse) are the row's probabilities
      if (lse && qpos < S)
        lse[(static_cast<size_t>(b) * H + hrow) * S + qpos] = m_ref + log2f(l);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::W_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Heads packed into one 128-row query tile: the largest power of two dividing the group
// size, at most 8 (so a tile holds at least 16 tokens of each head).
inline int pack_log2(int G) {
  int l = 0;
  while (l < 3 && G % (2 << l) == 0) ++l;
  return l;
}

template <int DL>
cudaError_t launch_tc(const Dims &d, const void *q, const void *k, const void *v, int kv_stride,
                      void *o, float scale_log2, int *status, cudaStream_t st, float *lse) {
  using C = AttnCfg<DL>;
  const int gpl = pack_log2(d.G);
  const int GP = 1 << gpl, TT = TM >> gpl;
  CUtensorMap mq, mk, mv;
  const uint64_t row = static_cast<uint64_t>(DL) * 2;
  const uint32_t box[3] = {static_cast<uint32_t>(C::CW), static_cast<uint32_t>(TT),
                           static_cast<uint32_t>(GP)};
  const uint32_t box_kv[3] = {static_cast<uint32_t>(C::CW), static_cast<uint32_t>(TN), 1u};
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(DL), static_cast<uint64_t>(d.S),
                              static_cast<uint64_t>(d.B) * d.H};
    const uint64_t strides[2] = {row, row * d.S};
    if (!make_tma_16bit(&mq, q, 3, dims, strides, box, C::ROWB, 1)) return cudaErrorInvalidValue;
  }
  {
    // keys / values past S read as zero (the cache may be longer than this sequence)
    const uint64_t dims[3] = {static_cast<uint64_t>(DL), static_cast<uint64_t>(d.S),
                              static_cast<uint64_t>(d.B) * d.Hkv};
    const uint64_t strides[2] = {row, row * static_cast<uint64_t>(kv_stride)};
    if (!make_tma_16bit(&mk, k, 3, dims, strides, box_kv, C::ROWB, 1) ||
        !make_tma_16bit(&mv, v, 3, dims, strides, box_kv, C::ROWB, 1))
      return cudaErrorInvalidValue;
  }
  if (cudaError_t e = ensure_dyn_smem<attn_tc_kernel<DL>>(C::SMEM); e != cudaSuccess) return e;
  const int nqt = (d.S + TT - 1) / TT;
  dim3 grid(d.H / GP, d.B, (nqt + C::NTILE - 1) / C::NTILE);
  attn_tc_kernel<DL><<<grid, C::THREADS, C::SMEM, st>>>(mq, mk, mv, static_cast<__half *>(o), d.S,
                                                        d.H, d.Hkv, d.G, gpl, nqt, scale_log2,
                                                        status, lse);
  return cudaGetLastError();
}

}  // namespace

cudaError_t latent_attention_tc(const Dims &d, const void *q, const void *k, const void *v,
                                int kv_stride, void *o, int *status, cudaStream_t st, float *lse) {
  const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(d.DL)));
  if (d.DL == 16) return launch_tc<16>(d, q, k, v, kv_stride, o, scale_log2, status, st, lse);
  if (d.DL == 32) return launch_tc<32>(d, q, k, v, kv_stride, o, scale_log2, status, st, lse);
  if (d.DL == 64) return launch_tc<64>(d, q, k, v, kv_stride, o, scale_log2, status, st, lse);
  if (d.DL == 128) return launch_tc<128>(d, q, k, v, kv_stride, o, scale_log2, status, st, lse);
  return cudaErrorInvalidValue;
}

}  // namespace cca
