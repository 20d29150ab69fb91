// Causal latent attention for 16-bit layers on the 5th-generation tensor cores.
//
//   O[b, t, h*d~ + :] = sum_{s <= t} softmax_s(q[b,h,t] . k[b,g,s] / sqrt(d~)) v[b,g,s],
//   g = h / (H/Hkv)
// (gist.science/de explainer, 2. Methodik: Softmax(QK^T)V evaluated entirely in the
// compressed space; gist.science explainer, Extension: CCGQA.)
//
// One CTA owns a 128-row query tile of one head and streams the 128-key tiles 0..qt of its
// key/value head (causal: tiles past the diagonal are never touched).  Two CTAs fit on an
// SM, so one CTA's softmax overlaps the other's tensor-core work.
//   warps 0-3 : softmax, one thread per query row = TMEM lane; online softmax in fp32 with
//               lazy rescaling (the reference max only moves when a row max grows by more
//               than 2^8), probabilities written to shared memory as float16 in the
//               128B-swizzled K-major layout the MMA reads; final O / l and store.
//   warp 4    : TMA producer: the Q tile once, then K and V tiles into a STAGES-deep ring.
//   warp 5    : allocates TMEM (S: 128 fp32 columns, O: d~ columns) and issues
//               tcgen05.mma from one thread: S = Q K^T (M=128, N=128, K=d~) and
//               O += P V (M=128, N=d~, K=128, V read MN-major); QK^T of tile j+1 is issued
//               as soon as the softmax warps have read S of tile j.
// Every wait is bounded; on a timeout the CTA records it in the status word, stops, and
// releases its tensor memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int TM = 128;          // query rows per tile (M of both MMAs)
constexpr int TN = 128;          // keys per tile
constexpr float kTau = 8.0f;     // lazy-rescale threshold, log2 units

template <int DL>
struct AttnCfg {
  static constexpr int STAGES = DL >= 64 ? 2 : 3;
  static constexpr int ROWB = DL * 2;                  // bytes of one q / k / v row
  static constexpr int Q_BYTES = TM * ROWB;
  static constexpr int KV_BYTES = TN * ROWB;           // one K or one V tile
  static constexpr int P_BYTES = TM * TN * 2;          // float16 probabilities
  static constexpr uint32_t SW_MODE = ROWB == 128 ? 2u : ROWB == 64 ? 4u : 6u;
  static constexpr int SBO = 8 * ROWB;                 // stride of 8-row core groups
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_P = OFF_V + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int SMEM = OFF_BAR + 256;
  static constexpr uint32_t TMEM_COLS = 256;           // S [0,128), O [128, 128+d~)
};

struct AttnBars {
  uint64_t q_full;
  uint64_t kv_full[3];
  uint64_t kv_empty[3];
  uint64_t s_full;
  uint64_t s_free;
  uint64_t p_full;
  uint64_t pv_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int DL>
__global__ void __launch_bounds__(192, 2)
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
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 4);
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->pv_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t tS = tmem, tO = tmem + 128;
  volatile int *abort = &bars->abort;

  if (warp == 4) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
      tma_load_3d(smem + C::OFF_Q, &mapQ, &bars->q_full, 0, q0, b * H + h);
      for (int j = 0; j < nkv; ++j) {
        const int s = j % C::STAGES;
        const uint32_t ph = (j / C::STAGES) & 1;
        if (!mbar_wait(&bars->kv_empty[s], ph ^ 1u, abort, status)) break;
        mbar_arrive_expect_tx(&bars->kv_full[s], 2 * C::KV_BYTES);
        tma_load_3d(smem + C::OFF_K + s * C::KV_BYTES, &mapK, &bars->kv_full[s], 0, j * TN,
                    b * Hkv + g);
        tma_load_3d(smem + C::OFF_V + s * C::KV_BYTES, &mapV, &bars->kv_full[s], 0, j * TN,
                    b * Hkv + g);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16_f32(TM, TN, 0, 0, 1);
      constexpr uint32_t idesc_pv = idesc_f16_f32(TM, DL, 0, 1, 1);
      const uint32_t qa = smem_u32(smem + C::OFF_Q);
      const uint32_t pa = smem_u32(smem + C::OFF_P);
      auto issue_qk = [&](int j) {
        const uint32_t ka = smem_u32(smem + C::OFF_K + (j % C::STAGES) * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < DL / 16; ++kk)
          umma_f16_ss(tS, smem_desc(qa + kk * 32, 16, C::SBO, C::SW_MODE),
                      smem_desc(ka + kk * 32, 16, C::SBO, C::SW_MODE), idesc_qk, kk > 0 ? 1u : 0u);
        umma_commit(&bars->s_full);
      };
      bool ok = mbar_wait(&bars->q_full, 0, abort, status) &&
                mbar_wait(&bars->kv_full[0], 0, abort, status);
      if (ok) {
        tc_fence_after();
        issue_qk(0);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv) {
          const int s1 = (j + 1) % C::STAGES;
          const uint32_t ph1 = ((j + 1) / C::STAGES) & 1;
          ok = mbar_wait(&bars->kv_full[s1], ph1, abort, status) &&
               mbar_wait(&bars->s_free, j & 1, abort, status);
          if (!ok) break;
          tc_fence_after();
          issue_qk(j + 1);
        }
        if (!mbar_wait(&bars->p_full, j & 1, abort, status)) break;
        tc_fence_after();
        const int s = j % C::STAGES;
        const uint32_t va = smem_u32(smem + C::OFF_V + s * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < TN / 16; ++kk) {
          const uint64_t pd = smem_desc(pa + (kk / 4) * (TM * 128) + (kk % 4) * 32, 16, 1024, 2);
          const uint64_t vd = smem_desc(va + kk * 2 * C::SBO, C::KV_BYTES, C::SBO, C::SW_MODE);
          umma_f16_ss(tO, pd, vd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->pv_done);
        umma_commit(&bars->kv_empty[s]);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-3
    const int row = warp * 32 + lane;                 // TMEM lane of this thread
    const int qpos = q0 + row;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    uint8_t *p_row = smem + C::OFF_P + row * 128;     // + atom * (TM * 128)
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, j & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      uint32_t r[TN];
      tmem_ld32(tS + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(tS + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_ld32(tS + lane_off + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
      tmem_ld32(tS + lane_off + 96, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free);

      // Row max of the raw scores (the 1/sqrt(d~) * log2(e) scale is positive, so it is
      // applied afterwards): eight independent partial maxima keep the dependency chains
      // short.  Keys past this row's position are masked on the diagonal tile only.
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
      if (j == nkv - 1) {
        const int last = qpos - j * TN;               // keys 0..last of this tile are visible
#pragma unroll
        for (int i = 0; i < TN; ++i) {
          if (i > last) r[i] = __float_as_uint(-INFINITY);
          mx8[i & 7] = fmaxf(mx8[i & 7], __uint_as_float(r[i]));
        }
      } else {
#pragma unroll
        for (int i = 0; i < TN; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], __uint_as_float(r[i]));
      }
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * scale_log2;
      bool resc = false;
      float m_new = m_ref;
      if (mx > m_ref + kTau) {
        m_new = mx;
        resc = true;
      }
      const float scale = resc ? ex2(m_ref - m_new) : 1.f;
      l *= scale;
      if (j > 0) {
        // P buffer and O accumulator are free once the previous P*V is done
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (j - 1) & 1, abort, status));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c = 0; c < DL / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(tO + lane_off + c * 16, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * scale);
            tmem_st16(tO + lane_off + c * 16, o);
          }
          tmem_st_wait();
        }
      }
      m_ref = m_new;
      // p = 2^(s * scale - m_ref): one FFMA and one MUFU ex2 per score; eight partial sums.
      const float neg_m = -m_ref;
      float l8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) l8[e] = 0.f;
#pragma unroll
      for (int c = 0; c < TN / 8; ++c) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = ex2(fmaf(__uint_as_float(r[c * 8 + e]), scale_log2, neg_m));
          l8[e] += p[e];
        }
        uint4 u;
        u.x = pack_f16x2(p[0], p[1]);
        u.y = pack_f16x2(p[2], p[3]);
        u.z = pack_f16x2(p[4], p[5]);
        u.w = pack_f16x2(p[6], p[7]);
        const int atom = c >> 3, chunk = (c & 7) ^ (row & 7);
        *reinterpret_cast<uint4 *>(p_row + atom * (TM * 128) + chunk * 16) = u;
      }
      l += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->pv_done, (nkv - 1) & 1, abort, status));
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __half *dst = O + (static_cast<size_t>(b) * S + qpos) * (static_cast<size_t>(H) * DL) + h * DL;
#pragma unroll
      for (int c = 0; c < DL / 16; ++c) {
        uint32_t o[16];
        tmem_ld16(tO + lane_off + c * 16, o);
        tmem_ld_wait();
        uint4 u0, u1;
        u0.x = pack_f16x2(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
        u0.y = pack_f16x2(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
        u0.z = pack_f16x2(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
        u0.w = pack_f16x2(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
        u1.x = pack_f16x2(__uint_as_float(o[8]) * inv, __uint_as_float(o[9]) * inv);
        u1.y = pack_f16x2(__uint_as_float(o[10]) * inv, __uint_as_float(o[11]) * inv);
        u1.z = pack_f16x2(__uint_as_float(o[12]) * inv, __uint_as_float(o[13]) * inv);
        u1.w = pack_f16x2(__uint_as_float(o[14]) * inv, __uint_as_float(o[15]) * inv);
        if (qpos < S) {
          reinterpret_cast<uint4 *>(dst + c * 16)[0] = u0;
          reinterpret_cast<uint4 *>(dst + c * 16)[1] = u1;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
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
  attn_tc_kernel<DL><<<grid, 192, C::SMEM, st>>>(mq, mk, mv, static_cast<__half *>(o), d.S, d.H,
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
