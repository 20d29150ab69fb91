// Causal latent attention for 16-bit layers on the 5th-generation tensor cores.
//
//   O[b, t, h*d~ + :] = sum_{s <= t} softmax_s(q[b,h,t] . k[b,g,s] / sqrt(d~)) v[b,g,s],
//   g = h / (H/Hkv)
// (gist.science/de explainer, 2. Methodik: Softmax(QK^T)V evaluated entirely in the
// compressed space; gist.science explainer, Extension: CCGQA.)
//
// One CTA owns a 128-row query tile of one head and streams the 128-key tiles 0..qt of its
// key/value head (causal: tiles past the diagonal are never touched).  Two CTAs share an SM,
// so one CTA's softmax overlaps the other's tensor-core work.  Per CTA:
//   warps 0-7 : softmax.  Warp w reads TMEM lanes 32*(w%4).. (one query row per thread) and
//               key half w/4 of every tile (keys 0-63 or 64-127).  The two warps of a lane
//               quadrant swap their partial row maxima through shared memory each tile, so
//               both hold the same reference max.  Online softmax in fp32 with lazy
//               rescaling (the reference max only moves when a row max grows by more than
//               2^8); probabilities are packed to float16 pairs and stored into tensor memory,
//               where the P*V MMA reads them as its A operand.  Each half keeps a partial
//               row sum and rescales / normalises its half of the output columns.
//   warp 8    : TMA producer: the Q tile once, then K and V tiles into two rings (K deeper
//               than V: a K tile is released as soon as its QK^T is done, so the next scores
//               never wait on the P*V two tiles back).
//   warp 9    : allocates TMEM and issues tcgen05.mma from one thread: S = Q K^T (M=128,
//               N=128, K=d~, both from shared memory) and O += P V (M=128, N=d~, K=128, P
//               from TMEM, V MN-major from shared memory); QK^T of tile j+1 is issued as soon
//               as every softmax warp has read S of tile j, so it runs under tile j's softmax.
// TMEM columns: S [0, 128), O [128, 128 + d~), P [128 + d~, 192 + d~) (float16 pairs).
// Every wait is bounded; on a timeout the CTA records it in the status word, stops, and
// releases its tensor memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int TM = 128;          // query rows per tile (M of all MMAs)
constexpr int TN = 128;          // keys per tile
constexpr int KH = TN / 2;       // keys per softmax half
constexpr int NSOFT = 8;         // softmax warps
constexpr int W_TMA = 8, W_MMA = 9;
constexpr int THREADS = (NSOFT + 2) * 32;
constexpr float kTau = 8.0f;     // lazy-rescale threshold, log2 units

template <int DL>
struct AttnCfg {
  static constexpr int SK = DL >= 64 ? 3 : 4;          // K ring depth
  static constexpr int SV = DL >= 64 ? 2 : 3;          // V ring depth
  static constexpr int ROWB = DL * 2;                  // bytes of one q / k / v row
  static constexpr int Q_BYTES = TM * ROWB;
  static constexpr int KV_BYTES = TN * ROWB;           // one K or one V tile
  static constexpr uint32_t SW_MODE = ROWB == 128 ? 2u : ROWB == 64 ? 4u : 6u;
  static constexpr int SBO = 8 * ROWB;                 // stride of 8-row core groups
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + SK * KV_BYTES;
  static constexpr int OFF_X = OFF_V + SV * KV_BYTES;   // row-max swap [2][2][TM] fp32
  static constexpr int OFF_L = OFF_X + 2 * 2 * TM * 4;      // row-sum swap [2][TM] fp32
  static constexpr int OFF_BAR = OFF_L + 2 * TM * 4;
  static constexpr int SMEM = OFF_BAR + 256;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t COL_O = TN;
  static constexpr uint32_t COL_P = TN + DL;
  static_assert(COL_P + TN / 2 <= TMEM_COLS, "S, O and P must fit the TMEM allocation");
};

struct AttnBars {
  uint64_t q_full;
  uint64_t k_full[4];
  uint64_t k_empty[4];
  uint64_t v_full[4];
  uint64_t v_empty[4];
  uint64_t s_full;
  uint64_t s_free;
  uint64_t p_full;
  uint64_t pv_done;
  uint64_t swap[4];              // per lane quadrant: both halves posted their row values
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

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed pairs of fp32 (one register pair): sm_100 issues the fma on both halves at once.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unf2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

template <int DL>
__global__ void __launch_bounds__(THREADS, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap mapQ,
                   const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, __half *__restrict__ O, int S,
                   int H, int Hkv, int G, float scale_log2, int *status) {
  using C = AttnCfg<DL>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, b = blockIdx.y;
  const int qt = static_cast<int>(gridDim.z) - 1 - static_cast<int>(blockIdx.z);  // long first
  const int g = h / G;
  const int q0 = qt * TM;
  const int nkv = qt + 1;
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
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, NSOFT);
    mbar_init(&bars->p_full, NSOFT);
    mbar_init(&bars->pv_done, 1);
    for (int e = 0; e < 4; ++e) mbar_init(&bars->swap[e], 2);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t tS = tmem, tO = tmem + C::COL_O, tP = tmem + C::COL_P;
  volatile int *abort = &bars->abort;

  if (warp == W_TMA) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
      tma_load_3d(smem + C::OFF_Q, &mapQ, &bars->q_full, 0, q0, b * H + h);
      for (int j = 0; j < nkv; ++j) {
        const int sk = j % C::SK, sv = j % C::SV;
        if (!mbar_wait(&bars->k_empty[sk], ((j / C::SK) & 1) ^ 1u, abort, status)) break;
        mbar_arrive_expect_tx(&bars->k_full[sk], C::KV_BYTES);
        tma_load_3d(smem + C::OFF_K + sk * C::KV_BYTES, &mapK, &bars->k_full[sk], 0, j * TN,
                    b * Hkv + g);
        if (!mbar_wait(&bars->v_empty[sv], ((j / C::SV) & 1) ^ 1u, abort, status)) break;
        mbar_arrive_expect_tx(&bars->v_full[sv], C::KV_BYTES);
        tma_load_3d(smem + C::OFF_V + sv * C::KV_BYTES, &mapV, &bars->v_full[sv], 0, j * TN,
                    b * Hkv + g);
      }
    }
  } else if (warp == W_MMA) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop (waits and descriptor arithmetic stay warp-uniform) and
    // one elected lane issues.  Descriptors advance by adding to their start-address field:
    // +2 (32 bytes) per 16-wide K step of Q / K, +2*SBO/16 per 16 keys of V.
    const bool leader = elect_one();
    constexpr uint32_t idesc_qk = idesc_f16_f32(TM, TN, 0, 0, 1);
    constexpr uint32_t idesc_pv = idesc_f16_f32(TM, DL, 0, 1, 1);
    const uint64_t qd = smem_desc(smem_u32(smem + C::OFF_Q), 16, C::SBO, C::SW_MODE);
    auto issue_qk = [&](int j) {
      const int sk = j % C::SK;
      const uint64_t kd = smem_desc(smem_u32(smem + C::OFF_K + sk * C::KV_BYTES), 16, C::SBO,
                                    C::SW_MODE);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < DL / 16; ++kk)
          umma_f16_ss(tS, qd + 2 * kk, kd + 2 * kk, idesc_qk, kk > 0 ? 1u : 0u);
        umma_commit(&bars->s_full);
        umma_commit(&bars->k_empty[sk]);
      }
      __syncwarp();
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->q_full, 0, abort, status) &&
                                          mbar_wait(&bars->k_full[0], 0, abort, status));
    if (ok) {
      tc_fence_after();
      issue_qk(0);
    }
    for (int j = 0; ok && j < nkv; ++j) {
      if (j + 1 < nkv) {
        const int s1 = (j + 1) % C::SK;
        const uint32_t ph1 = ((j + 1) / C::SK) & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->k_full[s1], ph1, abort, status) &&
                                         mbar_wait(&bars->s_free, j & 1, abort, status));
        if (!ok) break;
        tc_fence_after();
        issue_qk(j + 1);
      }
      const int s = j % C::SV;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->v_full[s], (j / C::SV) & 1, abort, status) &&
                                       mbar_wait(&bars->p_full, j & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      const uint64_t vd = smem_desc(smem_u32(smem + C::OFF_V + s * C::KV_BYTES), C::KV_BYTES,
                                    C::SBO, C::SW_MODE);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < TN / 16; ++kk)      // 16 keys of P = 8 TMEM columns of f16 pairs
          umma_f16_ts(tO, tP + kk * 8, vd + kk * (2 * C::SBO / 16), idesc_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&bars->pv_done);
        umma_commit(&bars->v_empty[s]);
      }
      __syncwarp();
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-7
    const int quad = warp & 3, hf = warp >> 2;
    const int row = quad * 32 + lane;                 // TMEM lane of this thread
    const int qpos = q0 + row;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    float *xmax = reinterpret_cast<float *>(smem + C::OFF_X);    // [parity][half][row]
    float *xsum = reinterpret_cast<float *>(smem + C::OFF_L);    // [half][row]
    constexpr int OC = DL / 2;                                   // O columns per half
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, j & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      uint32_t r[KH];
      tmem_ld32(tS + lane_off + hf * KH, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(tS + lane_off + hf * KH + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free);

      // Row max of the raw scores (the 1/sqrt(d~) * log2(e) scale is positive, so it is
      // applied afterwards), in four independent three-input chains.  Keys past this row's
      // position are masked on the diagonal tile only.
      if (j == nkv - 1) {
        const int last = qpos - j * TN - hf * KH;     // keys 0..last of this half are visible
#pragma unroll
        for (int i = 0; i < KH; ++i)
          if (i > last) r[i] = __float_as_uint(-INFINITY);
      }
      float mx4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) mx4[e] = __uint_as_float(r[e]);
#pragma unroll
      for (int i = 4; i < KH; i += 8)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          mx4[e] = max3(mx4[e], __uint_as_float(r[i + 2 * e]), __uint_as_float(r[i + 2 * e + 1]));
      float mx = max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * scale_log2;
      // swap with the other half of the row (double-buffered by tile parity)
      xmax[((j & 1) * 2 + hf) * TM + row] = mx;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->swap[quad]);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->swap[quad], j & 1, abort, status));
      if (!ok) break;
      mx = fmaxf(mx, xmax[((j & 1) * 2 + (hf ^ 1)) * TM + row]);   // finite: key 0 is visible

      const bool resc = mx > m_ref + kTau;
      const float scale = resc ? ex2(m_ref - mx) : 1.f;
      if (resc) m_ref = mx;
      l *= scale;
      if (j > 0) {
        // the P columns and O are free once the previous P*V is done
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (j - 1) & 1, abort, status));
        if (!ok) break;
        tc_fence_after();
        // the tcgen05 loads and stores are warp-wide: the warp rescales together, with
        // factor 1 in rows that keep their max
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c = 0; c < OC / 8; ++c) {
            uint32_t o[8];
            tmem_ld8(tO + lane_off + hf * OC + c * 8, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * scale);
            tmem_st8(tO + lane_off + hf * OC + c * 8, o);
          }
        }
      }
      // p = 2^(s * scale - m_ref): pairs scaled with one packed FMA, one MUFU ex2 each,
      // rounded to float16 pairs; four paired partial sums.
      const uint64_t sc2 = f2(scale_log2, scale_log2), nm2 = f2(-m_ref, -m_ref);
      uint64_t l2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) l2[e] = 0;
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {                 // 32 keys -> 16 TMEM columns
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int i = hc * 32 + 2 * e;
          const uint64_t x2 = fma2(f2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), sc2, nm2);
          float x0, x1;
          unf2(x2, x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          l2[e & 3] = add2(l2[e & 3], f2(p0, p1));
          pk[e] = pack_f16x2(p0, p1);
        }
        tmem_st16(tP + lane_off + hf * (KH / 2) + hc * 16, pk);
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
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (nkv - 1) & 1, abort, status));
    if (ok) {
      // row sum = both halves' partial sums (same reference max)
      xsum[hf * TM + row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->swap[quad]);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->swap[quad], nkv & 1, abort, status));
    }
    if (ok) {
      tc_fence_after();
      const float lt = l + xsum[(hf ^ 1) * TM + row];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      __half *dst = O + (static_cast<size_t>(b) * S + qpos) * (static_cast<size_t>(H) * DL) +
                    h * DL + hf * OC;
#pragma unroll
      for (int c = 0; c < OC / 8; ++c) {
        uint32_t o[8];
        tmem_ld8(tO + lane_off + hf * OC + c * 8, o);
        tmem_ld_wait();
        uint4 u;
        u.x = pack_f16x2(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
        u.y = pack_f16x2(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
        u.z = pack_f16x2(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
        u.w = pack_f16x2(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
        if (qpos < S) reinterpret_cast<uint4 *>(dst)[c] = u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int DL>
cudaError_t launch_tc(const Dims &d, const void *q, const void *k, const void *v, int kv_stride,
                      void *o, float scale_log2, int *status, cudaStream_t st) {
  using C = AttnCfg<DL>;
  CUtensorMap mq, mk, mv;
  const uint64_t row = static_cast<uint64_t>(DL) * 2;
  const uint32_t box[3] = {static_cast<uint32_t>(DL), static_cast<uint32_t>(TM), 1u};
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
    if (!make_tma_16bit(&mk, k, 3, dims, strides, box, C::ROWB, 1) ||
        !make_tma_16bit(&mv, v, 3, dims, strides, box, C::ROWB, 1))
      return cudaErrorInvalidValue;
  }
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dim3 grid(d.H, d.B, (d.S + TM - 1) / TM);
  attn_tc_kernel<DL><<<grid, THREADS, C::SMEM, st>>>(mq, mk, mv, static_cast<__half *>(o), d.S, d.H,
                                                  d.Hkv, d.G, scale_log2, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t latent_attention_tc(const Dims &d, const void *q, const void *k, const void *v,
                                int kv_stride, void *o, int *status, cudaStream_t st) {
  const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(d.DL)));
  if (d.DL == 16) return launch_tc<16>(d, q, k, v, kv_stride, o, scale_log2, status, st);
  if (d.DL == 32) return launch_tc<32>(d, q, k, v, kv_stride, o, scale_log2, status, st);
  if (d.DL == 64) return launch_tc<64>(d, q, k, v, kv_stride, o, scale_log2, status, st);
  return cudaErrorInvalidValue;
}

}  // namespace cca
