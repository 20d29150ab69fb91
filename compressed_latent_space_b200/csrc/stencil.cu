// Latent stencil of the prefill: everything between the down-projection and the attention,
// fused into one pass over the projected latents P = x W_qkv^T (float32).
//
// For every token t and key/value group g (gist.science explainer, 2. Methodology, Core
// Mechanism; edgentiq, "How Compressed Convolutional Attention Works"):
//   a  = causal depthwise conv of [pq | pk] along the sequence (KC taps, tap KC-1 = t)
//   b  = per-head channel conv of a (d~ x d~ matrix per head, pointwise in time)
//   q_h = b_h + (pq_h + pk_g)/2 ;  k_g = b_g + (mean_{h in g} pq_h + pk_g)/2   (Q-K-Mean)
//   v  = pv[t] on the lower half of the value channels, pv[t-1] on the upper half (Value-Shift)
//   q, k <- RMS-normalised per head, then rotated by RoPE at position t (RoPE Integration)
//
// One CTA owns a tile of TT tokens of one sequence and walks its key/value groups in turn
// (the RoPE table of the tile is built once for all of them): per group it stages the
// group's P rows (plus a halo of KC-1 earlier tokens) in shared memory, and writes q in
// head-major layout [B, H, S, d~] and k, v in [B, Hkv, kv_stride, d~] (the decode cache when
// one is given), as float16 for 16-bit layers.
//
// Channel conv: for 16-bit layers on the tensor cores (mma.sync m16n8k16), one warp per
// (head, 16 tokens), with both operands split into bfloat16 leading terms and remainders
// (a w ~ a_hi w_hi + a_hi w_lo + a_lo w_hi, about 16 significand bits); the norm and RoPE
// then run in the accumulator layout (a quad of lanes holds one token's head vector, and
// channels i and i + d~/2 sit in the same lane).  Float32 layers use exact fp32 FMAs.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

template <typename T>
struct StencilParams {
  using TL = typename LatentType<T>::type;
  const float *P;
  const float *conv_seq;
  const float *conv_chan;
  const uint2 *conv_chan_split;   // 16-bit layers: conv_chan as bf16 hi/lo pairs
  TL *q, *k, *v;
  float *conv_state, *vshift_state;
  int *lengths;
  int *status;
  int write_state;
  int B, S, H, Hkv, G, NQ, NKV, NQKV, KC, VS0, halo, TT, kv_stride;
  unsigned flags;
  float eps;
  double theta[32];        // RoPE frequencies base^(-2i/d~), i < d~/2, computed on the host
};

// Padded row strides (floats) of the staged P rows and of the sequence-conv output: +4 keeps
// the 8-row fragment loads of the tensor-core path free of bank conflicts.
__host__ __device__ inline int ch_pad(int G, int DL) { return (G + 2) * DL + 4; }
__host__ __device__ inline int qkc_pad(int G, int DL) { return (G + 1) * DL + 4; }

__host__ __device__ inline size_t stencil_smem_floats(int G, int DL, int TT, int halo, bool simt) {
  return static_cast<size_t>(TT + halo) * ch_pad(G, DL)        // Ps
         + static_cast<size_t>(TT) * qkc_pad(G, DL)            // As
         + static_cast<size_t>(TT) * DL                        // cos/sin table
         + (simt ? static_cast<size_t>(DL) * (DL + 1) : 0);   // Ws (float32 path)
}

template <int DL>
__device__ __forceinline__ float qk_mean_term(const float *prow, int G, int hh, int i) {
  const float pk = prow[G * DL + i];
  if (hh < G) return 0.5f * (prow[hh * DL + i] + pk);
  float mq = 0.f;
  for (int h2 = 0; h2 < G; ++h2) mq += prow[h2 * DL + i];
  return 0.5f * (mq / static_cast<float>(G) + pk);
}

// The tensor-core paths' epilogue for one warp's (head hh, 16 tokens from row tr0) channel-conv
// tile, in the m16n8k16 accumulator layout (a quad of lanes holds one token's head vector,
// channels i and i + d~/2 in the same lane): Q-K-Mean skip, RMS norm, RoPE, float16 store.
// Ps: the group's staged P rows (row tt + halo = token t0 + tt, pitch CHP); Rt: the tile's
// rotations [tt][d~/2][2]; MQ: Mq holds the mean of the group's q heads' P rows per token
// [tt][d~] for the k head's skip term (else it is summed here).
template <int DL, bool MQ>
__device__ __forceinline__ void store_head_tile(const StencilParams<__nv_bfloat16> &p,
                                                const float (&acc)[DL / 8][4], const float *Ps,
                                                int CHP, int halo, const float *Rt,
                                                const float *Mq, int b, int g, int hh, int t0,
                                                int tr0, int qc) {
  constexpr int NT = DL / 8, HALF = DL / 2;
  const int G = p.G;
  const bool is_q = hh < G;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int tt = tr0 + half * 8;
    const float *prow = Ps + (tt + halo) * CHP;
    float u[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = n * 8 + 2 * qc + e;
        float v = acc[n][half * 2 + e];
        if (p.flags & F_QK_MEAN) {
          if constexpr (MQ)
            v += 0.5f * ((is_q ? prow[hh * DL + i] : Mq[tt * DL + i]) + prow[G * DL + i]);
          else
            v += qk_mean_term<DL>(prow, G, hh, i);
        }
        u[n][e] = v;
      }
    if (p.flags & F_QK_NORM) {
      float ss = 0.f;
#pragma unroll
      for (int n = 0; n < NT; ++n) ss += u[n][0] * u[n][0] + u[n][1] * u[n][1];
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      const float inv = 1.0f / sqrtf(ss / static_cast<float>(DL) + p.eps);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        u[n][0] *= inv;
        u[n][1] *= inv;
      }
    }
    if (p.flags & F_ROPE) {
#pragma unroll
      for (int n = 0; n < NT / 2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = n * 8 + 2 * qc + e;          // < d~/2; partner i + d~/2 is n-tile n+NT/2
          const float c = Rt[(tt * HALF + i) * 2], s = Rt[(tt * HALF + i) * 2 + 1];
          const float x1 = u[n][e], x2 = u[n + NT / 2][e];
          u[n][e] = x1 * c - x2 * s;
          u[n + NT / 2][e] = x1 * s + x2 * c;
        }
    }
    const int t = t0 + tt;
    if (t < p.S) {
      __half *dst = is_q ? p.q + ((static_cast<size_t>(b) * p.H + g * G + hh) * p.S + t) * DL
                         : p.k + ((static_cast<size_t>(b) * p.Hkv + g) * p.kv_stride + t) * DL;
      bool fits = true;                                // every value within the float16 range
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        fits &= fabsf(u[n][0]) <= kF16Max && fabsf(u[n][1]) <= kF16Max;
        *reinterpret_cast<uint32_t *>(dst + n * 8 + 2 * qc) = pack_f16x2(u[n][0], u[n][1]);
      }
      if (!fits) report(p.status, DEV_RANGE);
    }
  }
}

// KCT: the sequence-conv width when it is the common 4 (taps unrolled exactly), 0 = any.
template <typename T, int DL, int KCT>
__global__ void __launch_bounds__(512) stencil_kernel(const StencilParams<T> p) {
  using TL = typename StencilParams<T>::TL;
  constexpr bool kTensor = sizeof(T) == 2;
  constexpr int HALF = DL / 2;
  extern __shared__ float sm[];
  const int G = p.G, QKC = (G + 1) * DL;
  const int CHP = ch_pad(G, DL), QKCP = qkc_pad(G, DL);
  const int TT = p.TT, halo = p.halo;
  float *Ps = sm;                                   // [TT+halo][CHP]
  float *As = Ps + (TT + halo) * CHP;               // [TT][QKCP]
  float *Rt = As + TT * QKCP;                       // [TT][HALF][2]
  float *Ws = Rt + TT * DL;                         // [DL][DL+1] (float32 path)

  const int b = blockIdx.z;
  const int t0 = blockIdx.x * TT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nwarps = blockDim.x >> 5;
  const int CH = (G + 2) * DL;

  // RoPE table for this tile, shared by every group: angle = t * base^(-2i/d~).
  if (p.flags & F_ROPE) {
    for (int i = tid; i < TT * HALF; i += blockDim.x) {
      const int tt = i / HALF, ip = i % HALF;
      rope_cos_sin(static_cast<double>(t0 + tt) * p.theta[ip], Rt[2 * i], Rt[2 * i + 1]);
    }
  }

  for (int g = 0; g < p.Hkv; ++g) {
  const int qcol0 = g * G * DL;                     // group's q channels in P
  const int kcol0 = p.NQ + g * DL;
  const int vcol0 = p.NQ + p.NKV + g * DL;
  if (g > 0) __syncthreads();                       // the previous group is done with Ps / As

  // 1. stage P rows t0-halo .. t0+TT-1 of the group's channels (zero outside [0, S)) with
  //    16-byte asynchronous copies, so every thread has all of its loads in flight at once.
  const int vec_per_row = CH / 4;
  for (int i = tid; i < (TT + halo) * vec_per_row; i += blockDim.x) {
    const int r = i / vec_per_row, c = (i % vec_per_row) * 4;
    const int t = t0 - halo + r;
    const bool in = t >= 0 && t < p.S;
    const int gc = c < G * DL ? qcol0 + c : (c < QKC ? kcol0 + (c - G * DL) : vcol0 + (c - QKC));
    const float *src = in ? p.P + (static_cast<size_t>(b) * p.S + t) * p.NQKV + gc : p.P;
    cp_async16_zfill(Ps + r * CHP + c, src, in);
  }
  cp_async_wait_all();
  __syncthreads();

  // 2. causal depthwise sequence conv of the q|k channels: one thread per channel, its
  //    filter in registers, sliding along the tile's tokens (KC <= 8).
  for (int c = tid; c < QKC; c += blockDim.x) {
    const int gc = c < G * DL ? qcol0 + c : p.NQ + g * DL + (c - G * DL);
    constexpr int NP = KCT ? KCT - 1 : 7;           // previous-token taps held in registers
    const int KC1 = KCT ? KCT - 1 : p.KC - 1;
    float wprev[NP], prev[NP], wcur = 0.f;
    const int r0 = halo - KC1;                      // Ps row of token t0 - (KC-1)
#pragma unroll
    for (int j = 0; j <= NP; ++j) {
      const float wj = j <= KC1 ? __ldg(p.conv_seq + static_cast<size_t>(gc) * (KC1 + 1) + j) : 0.f;
      if (j < NP) wprev[j] = j < KC1 ? wj : 0.f;
      if (j == KC1) wcur = wj;
    }
#pragma unroll
    for (int j = 0; j < NP; ++j) prev[j] = j < KC1 ? Ps[(r0 + j) * CHP + c] : 0.f;
    for (int tt = 0; tt < TT; ++tt) {
      const float cur = Ps[(halo + tt) * CHP + c];  // token t0 + tt
      float a = wcur * cur;
#pragma unroll
      for (int j = 0; j < NP; ++j) a = fmaf(wprev[j], prev[j], a);
      As[tt * QKCP + c] = a;
      if constexpr (KCT != 0) {
#pragma unroll
        for (int j = 0; j + 1 < NP; ++j) prev[j] = prev[j + 1];
        if (NP > 0) prev[NP - 1] = cur;
      } else {
#pragma unroll
        for (int j = 0; j < NP; ++j) prev[j] = j + 1 < KC1 ? prev[j + 1] : (j + 1 == KC1 ? cur : prev[j]);
      }
    }
  }
  __syncthreads();

  // 3. per head: channel conv, q-k-mean, RMS norm, RoPE, store.
  if constexpr (kTensor) {
    constexpr int NT = DL / 8;                      // n-tiles of 8 output channels
    const int MT = TT / 16;
    const int gr = lane >> 2, qc = lane & 3;
    for (int task = warp; task < (G + 1) * MT; task += nwarps) {
      const int hh = task / MT, mt = task % MT;
      const bool is_q = hh < G;
      // pre-split weights: for (head, n, k-pair) one uint2 {bf16x2 hi, bf16x2 lo}
      const uint2 *wb = p.conv_chan_split +
                        static_cast<size_t>(is_q ? g * G + hh : p.H + g) * DL * (DL / 2);
      float acc[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
      const float *a0p = As + (mt * 16 + gr) * QKCP + hh * DL;
      const float *a1p = a0p + 8 * QKCP;
#pragma unroll
      for (int ks = 0; ks < DL / 16; ++ks) {
        const int k0 = ks * 16 + 2 * qc;
        uint32_t ah[4], al[4];
        split_bf16x2(*reinterpret_cast<const float2 *>(a0p + k0), ah[0], al[0]);
        split_bf16x2(*reinterpret_cast<const float2 *>(a1p + k0), ah[1], al[1]);
        split_bf16x2(*reinterpret_cast<const float2 *>(a0p + k0 + 8), ah[2], al[2]);
        split_bf16x2(*reinterpret_cast<const float2 *>(a1p + k0 + 8), ah[3], al[3]);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint2 *wr = wb + (n * 8 + gr) * (DL / 2) + k0 / 2;
          const uint2 w0 = __ldg(wr), w1 = __ldg(wr + 4);
          const uint32_t bh[2] = {w0.x, w1.x}, bl[2] = {w0.y, w1.y};
          mma_bf16_16816(acc[n], ah, bh);
          mma_bf16_16816(acc[n], ah, bl);
          mma_bf16_16816(acc[n], al, bh);
        }
      }
      store_head_tile<DL, false>(p, acc, Ps, CHP, halo, Rt, nullptr, b, g, hh, t0, mt * 16 + gr, qc);
    }
  } else {
    constexpr int LPI = DL < 32 ? DL : 32;   // lanes per (token, head) item
    constexpr int EPL = DL / LPI;            // elements per lane
    constexpr int IPW = 32 / LPI;            // items per warp pass
    for (int hh = 0; hh <= G; ++hh) {
      const bool is_q = hh < G;
      const int head_w = is_q ? g * G + hh : p.H + g;
      __syncthreads();                                  // previous Ws consumed
      for (int i = tid; i < DL * DL; i += blockDim.x)
        Ws[(i / DL) * (DL + 1) + (i % DL)] = p.conv_chan[static_cast<size_t>(head_w) * DL * DL + i];
      __syncthreads();
      const int sub = lane / LPI, li = lane % LPI;
      for (int tt0 = warp * IPW; tt0 < TT; tt0 += nwarps * IPW) {
        const int tt = tt0 + sub;
        float u[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const int i = e * LPI + li;
          const float *arow = As + tt * QKCP + hh * DL;
          const float *wrow = Ws + i * (DL + 1);
          float acc = 0.f;
#pragma unroll 8
          for (int j = 0; j < DL; ++j) acc = fmaf(wrow[j], arow[j], acc);
          if (p.flags & F_QK_MEAN) acc += qk_mean_term<DL>(Ps + (tt + halo) * CHP, G, hh, i);
          u[e] = acc;
        }
        if (p.flags & F_QK_NORM) {
          float ss = 0.f;
#pragma unroll
          for (int e = 0; e < EPL; ++e) ss += u[e] * u[e];
#pragma unroll
          for (int off = LPI / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
          const float inv = 1.0f / sqrtf(ss / static_cast<float>(DL) + p.eps);
#pragma unroll
          for (int e = 0; e < EPL; ++e) u[e] *= inv;
        }
        if (p.flags & F_ROPE) {
          if constexpr (EPL == 2) {
            const float c = Rt[(tt * HALF + li) * 2], s = Rt[(tt * HALF + li) * 2 + 1];
            const float x1 = u[0], x2 = u[1];
            u[0] = x1 * c - x2 * s;
            u[1] = x1 * s + x2 * c;
          } else {
            const float other = __shfl_xor_sync(0xffffffffu, u[0], HALF);
            const int ip = li % HALF;
            const float c = Rt[(tt * HALF + ip) * 2], s = Rt[(tt * HALF + ip) * 2 + 1];
            u[0] = li < HALF ? u[0] * c - other * s : other * s + u[0] * c;
          }
        }
        const int t = t0 + tt;
        if (t < p.S) {
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            const int i = e * LPI + li;
            if (is_q)
              p.q[((static_cast<size_t>(b) * p.H + g * G + hh) * p.S + t) * DL + i] = from_f32<TL>(u[e]);
            else
              p.k[((static_cast<size_t>(b) * p.Hkv + g) * p.kv_stride + t) * DL + i] = from_f32<TL>(u[e]);
          }
        }
      }
    }
  }

  // 4. values with the value-shift: upper half of the value channels from token t-1.
  const int vhalf = p.VS0;
  for (int i = tid; i < TT * (DL / 2); i += blockDim.x) {
    const int tt = i / (DL / 2), c = (i % (DL / 2)) * 2;
    const int t = t0 + tt;
    if (t >= p.S) continue;
    float val[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const bool shifted = (p.flags & F_VALUE_SHIFT) && (g * DL + c + e >= vhalf);
      val[e] = Ps[(tt + halo - (shifted ? 1 : 0)) * CHP + QKC + c + e];
    }
    TL *dst = p.v + ((static_cast<size_t>(b) * p.Hkv + g) * p.kv_stride + t) * DL + c;
    if constexpr (sizeof(TL) == 2) {
      if (!(fabsf(val[0]) <= kF16Max && fabsf(val[1]) <= kF16Max)) report(p.status, DEV_RANGE);
      *reinterpret_cast<uint32_t *>(dst) = pack_f16x2(val[0], val[1]);
    } else {
      *reinterpret_cast<float2 *>(dst) = make_float2(val[0], val[1]);
    }
  }

  // 5. decode state after the last token, written by the tile that holds it.
  if (p.write_state && t0 <= p.S - 1 && p.S - 1 < t0 + TT) {
    const int KC1 = p.KC - 1;
    const int W = p.NQ + p.NKV;
    for (int i = tid; i < KC1 * QKC; i += blockDim.x) {
      const int j = i / QKC, c = i % QKC;
      const int ts = p.S - KC1 + j;
      const int r = ts - t0 + halo;
      const int gc = c < G * DL ? qcol0 + c : p.NQ + g * DL + (c - G * DL);
      p.conv_state[(static_cast<size_t>(b) * KC1 + j) * W + gc] = Ps[r * CHP + c];
    }
    const int rl = p.S - 1 - t0 + halo;
    for (int c = tid; c < DL; c += blockDim.x) {
      const int gch = g * DL + c;
      if (gch >= vhalf)
        p.vshift_state[static_cast<size_t>(b) * (p.NKV - vhalf) + (gch - vhalf)] =
            Ps[rl * CHP + QKC + c];
    }
    if (g == 0 && tid == 0) p.lengths[b] = p.S;
  }
  }  // groups
}

// ------------------------------------------------------------------ persistent 16-bit path
// One CTA per SM, each bound to one key/value group for its whole life: the group's channel
// filters (split into bf16 hi / lo pairs) and sequence taps are staged in shared memory once,
// and the CTA then walks a contiguous run of (sequence, TT-token tile) units, the P rows of the
// next unit copied in (cp.async, second buffer) while the current one is computed.  Against
// one CTA per tile walking the groups, the filters cross from L2 once per CTA instead of once
// per (tile, group, 16-token task), and no unit waits for its own P rows.  The sequence conv is
// evaluated straight into the MMA's A fragments (each fragment element belongs to one task),
// so there is no intermediate buffer.  Same arithmetic as the per-tile kernel above.
constexpr int GT = 32;                  // tokens per unit
constexpr int kGroupSmemLimit = 220 * 1024;

__host__ __device__ inline int wsp_ld(int DL) { return DL / 2 + 4; }   // uint2 per filter row
// P row pitch (floats): = 8 mod 16 banks' worth, so the 8 rows x 4 column pairs of an A
// fragment's float2 reads fall on distinct banks
__host__ __device__ inline int gps_pitch(int G, int DL) { return (G + 2) * DL + 8; }

struct GroupSmem {                      // byte offsets of the persistent kernel's buffers
  size_t w, wseq, ps, rt, mq, total;
};
__host__ __device__ inline GroupSmem group_smem(int G, int DL, int KC, int halo) {
  GroupSmem m;
  m.w = 0;                                                             // [G+1][DL][wsp_ld] uint2
  m.wseq = m.w + static_cast<size_t>(G + 1) * DL * wsp_ld(DL) * 8;     // [QKC][KC] float
  m.ps = m.wseq + ((static_cast<size_t>(G + 1) * DL * KC * 4 + 15) / 16) * 16;  // [2][GT+halo][CHP]
  m.rt = m.ps + static_cast<size_t>(2) * (GT + halo) * gps_pitch(G, DL) * 4;    // [GT][HALF][2]
  m.mq = m.rt + static_cast<size_t>(GT) * DL * 4;                     // [GT][DL]
  m.total = m.mq + static_cast<size_t>(GT) * DL * 4;
  return m;
}

// MAXW: the most warps a launch uses ((G + 1) * GT / 16); a smaller bound leaves each thread
// more registers.
template <int DL, int KCT, int MAXW>
__global__ void __launch_bounds__(32 * MAXW, 1) stencil_group_kernel(
    const StencilParams<__nv_bfloat16> p, int ctas_per_group, int tiles) {
  using TL = __half;
  constexpr int HALF = DL / 2;
  constexpr int NT = DL / 8;
  constexpr int MT = GT / 16;
  extern __shared__ __align__(16) uint8_t gsm[];
  const int G = p.G, QKC = (G + 1) * DL, CH = (G + 2) * DL;
  const int CHP = gps_pitch(G, DL), WLD = wsp_ld(DL);
  const int halo = p.halo, KC = p.KC;
  const int KC1 = KCT ? KCT - 1 : KC - 1;
  const GroupSmem L = group_smem(G, DL, KC, halo);
  uint2 *Wsp = reinterpret_cast<uint2 *>(gsm + L.w);
  float *wseq = reinterpret_cast<float *>(gsm + L.wseq);
  float *PsBuf = reinterpret_cast<float *>(gsm + L.ps);
  float *Rt = reinterpret_cast<float *>(gsm + L.rt);   // rotations of the unit's tokens
  float *Mq = reinterpret_cast<float *>(gsm + L.mq);   // mean of the group's q heads' P rows
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
  const int g = blockIdx.x / ctas_per_group, r = blockIdx.x % ctas_per_group;
  const int units = p.B * tiles;
  const int u_beg = static_cast<int>(static_cast<long>(units) * r / ctas_per_group);
  const int u_end = static_cast<int>(static_cast<long>(units) * (r + 1) / ctas_per_group);
  const int qcol0 = g * G * DL, kcol0 = p.NQ + g * DL, vcol0 = p.NQ + p.NKV + g * DL;

  // the group's filters: heads g*G .. g*G+G-1, then k head H+g; rows padded to WLD uint2
  for (int i = tid; i < (G + 1) * DL * (HALF / 2); i += blockDim.x) {   // 16-byte pieces
    const int hh = i / (DL * (HALF / 2)), rem = i % (DL * (HALF / 2));
    const int row = rem / (HALF / 2), piece = rem % (HALF / 2);
    const int head = hh < G ? g * G + hh : p.H + g;
    cp_async16_zfill(Wsp + (hh * DL + row) * WLD + piece * 2,
                     p.conv_chan_split + (static_cast<size_t>(head) * DL + row) * HALF + piece * 2,
                     true);
  }
  for (int e = tid; e < QKC * KC; e += blockDim.x) {
    const int c = e / KC, t = e % KC;
    const int gc = c < G * DL ? qcol0 + c : kcol0 + (c - G * DL);
    wseq[e] = p.conv_seq[static_cast<size_t>(gc) * KC + t];
  }
  auto issue = [&](int u, int buf) {              // P rows of unit u into buffer buf
    if (u < u_end) {
      const int b = u / tiles, t0 = (u % tiles) * GT;
      float *Ps = PsBuf + static_cast<size_t>(buf) * (GT + halo) * CHP;
      for (int rr = warp; rr < GT + halo; rr += nwarps) {     // a warp per row
        const int t = t0 - halo + rr;
        const bool in = t >= 0 && t < p.S;
        const float *row = p.P + (static_cast<size_t>(b) * p.S + (in ? t : 0)) * p.NQKV;
        for (int c = lane * 4; c < CH; c += 128) {
          const int gc = c < G * DL ? qcol0 + c : (c < QKC ? kcol0 + (c - G * DL) : vcol0 + (c - QKC));
          cp_async16_zfill(Ps + rr * CHP + c, row + gc, in);
        }
      }
    }
    cp_async_commit();
  };
  issue(u_beg, 0);                                  // (the filter copies join this group)

  const int gr = lane >> 2, qc = lane & 3;
  const int vhalf = p.VS0;
  for (int u = u_beg, k = 0; u < u_end; ++u, ++k) {
    const int buf = k & 1;
    issue(u + 1, buf ^ 1);
    const int b = u / tiles, t0 = (u % tiles) * GT;
    if (p.flags & F_ROPE)                           // this unit's rotations
      for (int i = tid; i < GT * HALF; i += blockDim.x)
        rope_cos_sin(static_cast<double>(t0 + i / HALF) * p.theta[i % HALF], Rt[2 * i], Rt[2 * i + 1]);
    asm volatile("cp.async.wait_group 1;" ::: "memory");   // unit u's rows have landed
    __syncthreads();
    const float *Ps = PsBuf + static_cast<size_t>(buf) * (GT + halo) * CHP;
    if (p.flags & F_QK_MEAN) {                      // the k head's share of Q-K-Mean, once
      for (int i = tid; i < GT * DL; i += blockDim.x) {
        const float *prow = Ps + (i / DL + halo) * CHP + (i % DL);
        float m = 0.f;
        for (int h2 = 0; h2 < G; ++h2) m += prow[h2 * DL];
        Mq[i] = m / static_cast<float>(G);
      }
      __syncthreads();
    }

    // channel conv tasks: (head, 16 tokens) per warp
    for (int task = warp; task < (G + 1) * MT; task += nwarps) {
      const int hh = task / MT, mt = task % MT;
      const uint2 *wb = Wsp + static_cast<size_t>(hh) * DL * WLD;
      float acc[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
      const int tr0 = mt * 16 + gr;                 // fragment rows tr0, tr0 + 8
#pragma unroll
      for (int ks = 0; ks < DL / 16; ++ks) {
        // A = the sequence conv of channels hh*DL + ks*16 + {2qc, 2qc+1, 2qc+8, 2qc+9}
        float2 av[4];
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) {            // column pair 2qc (+0 / +8)
          const int c = hh * DL + ks * 16 + 2 * qc + hp * 8;
          const float *w0 = wseq + c * KC, *w1 = w0 + KC;
#pragma unroll
          for (int rh = 0; rh < 2; ++rh) {          // row tr0 (+0 / +8)
            const int rbase = tr0 + rh * 8 + halo - KC1;   // Ps row of the first tap
            float x = 0.f, y = 0.f;
            if constexpr (KCT != 0) {
#pragma unroll
              for (int j = 0; j < KCT; ++j) {
                const float2 pv = *reinterpret_cast<const float2 *>(Ps + (rbase + j) * CHP + c);
                x = fmaf(w0[j], pv.x, x);
                y = fmaf(w1[j], pv.y, y);
              }
            } else {
              for (int j = 0; j <= KC1; ++j) {
                const float2 pv = *reinterpret_cast<const float2 *>(Ps + (rbase + j) * CHP + c);
                x = fmaf(w0[j], pv.x, x);
                y = fmaf(w1[j], pv.y, y);
              }
            }
            av[hp * 2 + rh] = make_float2(x, y);
          }
        }
        uint32_t ah[4], al[4];                      // a0: (r, k), a1: (r+8, k), a2: (r, k+8), a3
        split_bf16x2(av[0], ah[0], al[0]);
        split_bf16x2(av[1], ah[1], al[1]);
        split_bf16x2(av[2], ah[2], al[2]);
        split_bf16x2(av[3], ah[3], al[3]);
        const int k0 = ks * 16 + 2 * qc;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint2 *wr = wb + (n * 8 + gr) * WLD + k0 / 2;
          const uint2 w0 = wr[0], w1 = wr[4];
          const uint32_t bh[2] = {w0.x, w1.x}, bl[2] = {w0.y, w1.y};
          mma_bf16_16816(acc[n], ah, bh);
          mma_bf16_16816(acc[n], ah, bl);
          mma_bf16_16816(acc[n], al, bh);
        }
      }
      store_head_tile<DL, true>(p, acc, Ps, CHP, halo, Rt, Mq, b, g, hh, t0, tr0, qc);
    }

    // values with the value-shift: upper half of the value channels from token t-1
    for (int i = tid; i < GT * HALF; i += blockDim.x) {
      const int tt = i / HALF, c = (i % HALF) * 2;
      const int t = t0 + tt;
      if (t >= p.S) continue;
      float val[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool shifted = (p.flags & F_VALUE_SHIFT) && (g * DL + c + e >= vhalf);
        val[e] = Ps[(tt + halo - (shifted ? 1 : 0)) * CHP + QKC + c + e];
      }
      if (!(fabsf(val[0]) <= kF16Max && fabsf(val[1]) <= kF16Max)) report(p.status, DEV_RANGE);
      *reinterpret_cast<uint32_t *>(
          p.v + ((static_cast<size_t>(b) * p.Hkv + g) * p.kv_stride + t) * DL + c) =
          pack_f16x2(val[0], val[1]);
    }

    // decode state after the sequence's last token, by the unit that holds it
    if (p.write_state && t0 <= p.S - 1 && p.S - 1 < t0 + GT) {
      const int W = p.NQ + p.NKV;
      for (int i = tid; i < KC1 * QKC; i += blockDim.x) {
        const int j = i / QKC, c = i % QKC;
        const int rr = p.S - KC1 + j - t0 + halo;
        const int gc = c < G * DL ? qcol0 + c : kcol0 + (c - G * DL);
        p.conv_state[(static_cast<size_t>(b) * KC1 + j) * W + gc] = Ps[rr * CHP + c];
      }
      const int rl = p.S - 1 - t0 + halo;
      for (int c = tid; c < DL; c += blockDim.x) {
        const int gch = g * DL + c;
        if (gch >= vhalf)
          p.vshift_state[static_cast<size_t>(b) * (p.NKV - vhalf) + (gch - vhalf)] =
              Ps[rl * CHP + QKC + c];
      }
      if (g == 0 && tid == 0) p.lengths[b] = p.S;
    }
    __syncthreads();                                // buffer buf and Rt are rewritten next
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

constexpr int kTensorSmemKB = 110;   // staging budget per CTA of the 16-bit path

template <typename T, int DL>
cudaError_t launch(const Dims &d, const StencilArgs &a, cudaStream_t st) {
  using TL = typename LatentType<T>::type;
  constexpr bool simt = sizeof(T) == 4;
  StencilParams<T> p;
  p.P = a.P;
  p.conv_seq = a.conv_seq;
  p.conv_chan = a.conv_chan;
  p.conv_chan_split = static_cast<const uint2 *>(a.conv_chan_split);
  p.q = static_cast<TL *>(a.q);
  p.k = static_cast<TL *>(a.k);
  p.v = static_cast<TL *>(a.v);
  p.status = a.status;
  p.conv_state = a.conv_state;
  p.vshift_state = a.vshift_state;
  p.lengths = a.lengths;
  p.write_state = a.write_state ? 1 : 0;
  p.B = d.B; p.S = d.S; p.H = d.H; p.Hkv = d.Hkv; p.G = d.G;
  p.NQ = d.NQ; p.NKV = d.NKV; p.NQKV = d.NQKV; p.KC = d.KC; p.VS0 = d.VS0;
  p.halo = d.KC - 1 > 1 ? d.KC - 1 : 1;
  p.kv_stride = a.kv_stride;
  p.flags = d.flags;
  p.eps = d.eps;
  for (int i = 0; i < DL / 2; ++i)
    p.theta[i] = pow(static_cast<double>(d.rope_base), -2.0 * i / DL);
  if constexpr (!simt) {
    const GroupSmem gs = group_smem(d.G, DL, d.KC, p.halo);
    const int warps = (d.G + 1) * (GT / 16);
    if (gs.total <= static_cast<size_t>(kGroupSmemLimit) && warps <= 18) {
      const int tiles = (d.S + GT - 1) / GT;
      const int units = d.B * tiles;
      int cpg = num_sms() / d.Hkv;                   // CTAs per group: one per SM in all
      if (cpg < 1) cpg = 1;
      if (cpg > units) cpg = units;
      p.TT = GT;
      const dim3 grid(d.Hkv * cpg), block(32 * (warps < 4 ? 4 : warps));
      auto go = [&](auto kernel) -> cudaError_t {
        kernel<<<grid, block, gs.total, st>>>(p, cpg, tiles);
        return cudaGetLastError();
      };
      cudaError_t e;
      if (warps <= 12) {
        e = d.KC == 4 ? ensure_dyn_smem<stencil_group_kernel<DL, 4, 12>>(gs.total)
                      : ensure_dyn_smem<stencil_group_kernel<DL, 0, 12>>(gs.total);
        if (e != cudaSuccess) return e;
        return d.KC == 4 ? go(stencil_group_kernel<DL, 4, 12>) : go(stencil_group_kernel<DL, 0, 12>);
      }
      e = d.KC == 4 ? ensure_dyn_smem<stencil_group_kernel<DL, 4, 18>>(gs.total)
                    : ensure_dyn_smem<stencil_group_kernel<DL, 0, 18>>(gs.total);
      if (e != cudaSuccess) return e;
      return d.KC == 4 ? go(stencil_group_kernel<DL, 4, 18>) : go(stencil_group_kernel<DL, 0, 18>);
    }
  }
  // Largest token tile (a multiple of 16) whose staging fits two CTAs per SM.
  const size_t budget = (simt ? 72 : kTensorSmemKB) * 1024;
  int TT = 64;
  while (TT > 16 && stencil_smem_floats(d.G, DL, TT, p.halo, simt) * 4 > budget) TT /= 2;
  p.TT = TT;
  const size_t smem = stencil_smem_floats(d.G, DL, TT, p.halo, simt) * 4;
  if (smem > 220 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e = d.KC == 4 ? ensure_dyn_smem<stencil_kernel<T, DL, 4>>(smem)
                            : ensure_dyn_smem<stencil_kernel<T, DL, 0>>(smem);
  if (e != cudaSuccess) return e;
  int threads = 256;
  if (!simt) {
    const int tasks = (d.G + 1) * (TT / 16);      // (head, 16-token) channel-conv tasks
    threads = 32 * (tasks < 4 ? 4 : tasks > 16 ? 16 : tasks);
  }
  dim3 grid((d.S + TT - 1) / TT, 1, d.B);
  if (d.KC == 4) stencil_kernel<T, DL, 4><<<grid, threads, smem, st>>>(p);
  else stencil_kernel<T, DL, 0><<<grid, threads, smem, st>>>(p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ identity convolutions
// The latent step with both convolutions the identity (CCA_NO_CONV): q = pq, k = pk before
// Q-K-Mean (whose pre- and post-conv terms then coincide), value-shift, RMS norm and RoPE as
// selected.  With C = 1 and only RoPE on, this is the projection-to-attention step of plain
// multi-head (or grouped-query) attention with rotary embeddings, for any latent width up to
// 128.  A memory-bound pass: one (token, head row) unit per d~/8 consecutive threads, each
// thread holding four RoPE pairs (channels i..i+3 and i+d~/2..i+d~/2+3) as two float4 loads of
// the P row (the q heads, k groups and v groups of a token lie at row offset unit * d~ in
// that order), the row's sum of squares reduced over the unit's lanes by shuffles.
template <typename T>
struct PointParams {
  using TL = typename LatentType<T>::type;
  const float *P;
  TL *q, *k, *v;
  int *status;
  int B, S, H, Hkv, G, DL, NQ, NKV, NQKV, VS0, kv_stride;
  unsigned flags;
  float eps;
  // RoPE frequency base^(-2i/d~) / (2 pi) in turns, i < d~/2, as a float pair hi + lo
  // (computed on the host in double)
  float turns_hi[64], turns_lo[64];
};

template <typename TL>
__device__ __forceinline__ void store4(TL *dst, const float (&x)[4]) {
  if constexpr (sizeof(TL) == 2) {
    uint2 u;
    u.x = pack_f16x2(x[0], x[1]);
    u.y = pack_f16x2(x[2], x[3]);
    *reinterpret_cast<uint2 *>(dst) = u;
  } else {
    *reinterpret_cast<float4 *>(dst) = make_float4(x[0], x[1], x[2], x[3]);
  }
}

__device__ __forceinline__ void load4(const float *src, float (&x)[4]) {
  const float4 f = __ldg(reinterpret_cast<const float4 *>(src));
  x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
}

// Loads one unit's eight channels (Q-K-Mean applied for query / key heads, the value-shift
// for value groups).
template <typename T, int DL, bool QKM>
__device__ __forceinline__ void pointwise_load(const PointParams<T> &p, int bt, int hh, int i0,
                                               float (&u0)[4], float (&u1)[4]) {
  constexpr int HALF = DL / 2;
  const float *row = p.P + static_cast<size_t>(bt) * p.NQKV;
  if (hh < p.H + p.Hkv) {                           // a query or key head
    const bool is_q = hh < p.H;
    const int g = is_q ? hh / p.G : hh - p.H;
    load4(row + hh * DL + i0, u0);
    load4(row + hh * DL + HALF + i0, u1);
    if (QKM) {                                      // post-conv == pre-conv here
      float k0[4], k1[4], m0[4], m1[4];
      load4(row + p.NQ + g * DL + i0, k0);
      load4(row + p.NQ + g * DL + HALF + i0, k1);
      if (is_q) {
#pragma unroll
        for (int e = 0; e < 4; ++e) { m0[e] = u0[e]; m1[e] = u1[e]; }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) { m0[e] = 0.f; m1[e] = 0.f; }
        for (int h2 = 0; h2 < p.G; ++h2) {
          float a0[4], a1[4];
          load4(row + (g * p.G + h2) * DL + i0, a0);
          load4(row + (g * p.G + h2) * DL + HALF + i0, a1);
#pragma unroll
          for (int e = 0; e < 4; ++e) { m0[e] += a0[e]; m1[e] += a1[e]; }
        }
        const float inv_g = 1.f / static_cast<float>(p.G);
#pragma unroll
        for (int e = 0; e < 4; ++e) { m0[e] *= inv_g; m1[e] *= inv_g; }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        u0[e] += 0.5f * (m0[e] + k0[e]);
        u1[e] += 0.5f * (m1[e] + k1[e]);
      }
    }
  } else {                                          // a value group, with the value-shift
    const int g = hh - p.H - p.Hkv;
    const int t = bt % p.S;
    // the channel boundary of the shift is a multiple of 4 (checked on the host), so each
    // 4-channel run is shifted or not as a whole
    const int c0 = g * DL + i0, c1 = c0 + HALF;
    const bool sh0 = (p.flags & F_VALUE_SHIFT) && c0 >= p.VS0;
    const bool sh1 = (p.flags & F_VALUE_SHIFT) && c1 >= p.VS0;
    const float *vrow = row + p.NQ + p.NKV;
    const float *prev = vrow - p.NQKV;              // the previous token's row (t > 0 only)
#pragma unroll
    for (int e = 0; e < 4; ++e) { u0[e] = 0.f; u1[e] = 0.f; }
    if (!sh0) load4(vrow + c0, u0);
    else if (t > 0) load4(prev + c0, u0);
    if (!sh1) load4(vrow + c1, u1);
    else if (t > 0) load4(prev + c1, u1);
  }
}

// Norm (its sum of squares reduced over the unit's lanes; every lane of the warp takes part),
// RoPE, range check and store of one unit.
template <typename T, int DL>
__device__ __forceinline__ void pointwise_finish(const PointParams<T> &p, const float2 *turns,
                                                 int bt, int hh, int i0, bool live,
                                                 float (&u0)[4], float (&u1)[4]) {
  using TL = typename LatentType<T>::type;
  constexpr int TPU = DL / 8, HALF = DL / 2;
  const bool is_qk = hh < p.H + p.Hkv;
  if (p.flags & F_QK_NORM) {                        // uniform over the grid
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) ss += u0[e] * u0[e] + u1[e] * u1[e];
#pragma unroll
    for (int o = TPU / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (is_qk) {
      const float inv = 1.0f / sqrtf(ss / static_cast<float>(DL) + p.eps);
#pragma unroll
      for (int e = 0; e < 4; ++e) { u0[e] *= inv; u1[e] *= inv; }
    }
  }
  if (!live) return;
  const int b = bt / p.S, t = bt - b * p.S;
  TL *dst;
  if (is_qk) {
    if (p.flags & F_ROPE) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float cs, sn;
        const float2 tr = turns[i0 + e];
        rope_cos_sin_turns(t, tr.x, tr.y, cs, sn);
        const float x1 = u0[e], x2 = u1[e];
        u0[e] = x1 * cs - x2 * sn;
        u1[e] = x1 * sn + x2 * cs;
      }
    }
    const bool is_q = hh < p.H;
    dst = is_q ? p.q + ((static_cast<size_t>(b) * p.H + hh) * p.S + t) * DL
               : p.k + ((static_cast<size_t>(b) * p.Hkv + (hh - p.H)) * p.kv_stride + t) * DL;
  } else {
    const int g = hh - p.H - p.Hkv;
    dst = p.v + ((static_cast<size_t>(b) * p.Hkv + g) * p.kv_stride + t) * DL;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) { check_latent<TL>(u0[e], p.status); check_latent<TL>(u1[e], p.status); }
  store4(dst + i0, u0);
  store4(dst + HALF + i0, u1);
}

// Grid-stride over units, two units per thread per pass with both units' loads issued first.
// Lanes of a warp walk together: the warp's pass continues while its first unit exists, and
// lanes whose unit lies past the end redo the last unit without storing.
template <typename T, int DL, bool QKM>
__global__ void __launch_bounds__(256, QKM ? 3 : 6) pointwise_kernel(const PointParams<T> p) {
  constexpr int TPU = DL / 8;                       // threads per unit (divides 32)
  const unsigned per_tok = p.H + 2 * p.Hkv;
  const unsigned units = static_cast<unsigned>(p.B) * p.S * per_tok;   // < 2^31 (host check)
  const unsigned total = gridDim.x * blockDim.x;
  const unsigned lane = threadIdx.x & 31;
  const int i0 = static_cast<int>(lane % TPU) * 4;  // pairs i0..i0+3 with i0+HALF..
  // the RoPE frequencies in shared memory: lanes of a warp read different ones, which a
  // constant-bank access would serialise
  __shared__ float2 turns[64];
  if (threadIdx.x < 64) turns[threadIdx.x] = make_float2(p.turns_hi[threadIdx.x], p.turns_lo[threadIdx.x]);
  __syncthreads();
  for (unsigned wb = blockIdx.x * blockDim.x + (threadIdx.x & ~31u); wb / TPU < units;
       wb += 2 * total) {
    float u0[2][4], u1[2][4];
    int bt[2], hh[2];
    bool live[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const unsigned g = (wb + r * total + lane) / TPU;
      live[r] = g < units;
      const unsigned unit = live[r] ? g : units - 1;
      bt[r] = static_cast<int>(unit / per_tok);
      hh[r] = static_cast<int>(unit % per_tok);
      pointwise_load<T, DL, QKM>(p, bt[r], hh[r], i0, u0[r], u1[r]);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) pointwise_finish<T, DL>(p, turns, bt[r], hh[r], i0, live[r], u0[r], u1[r]);
  }
}

template <typename T>
cudaError_t launch_pointwise(const Dims &d, const StencilArgs &a, cudaStream_t st) {
  using TL = typename LatentType<T>::type;
  if (d.DL != 16 && d.DL != 32 && d.DL != 64 && d.DL != 128) return cudaErrorInvalidValue;
  if (d.VS0 % 4 != 0 || d.NQKV % 4 != 0) return cudaErrorInvalidValue;
  PointParams<T> p;
  p.P = a.P;
  p.q = static_cast<TL *>(a.q);
  p.k = static_cast<TL *>(a.k);
  p.v = static_cast<TL *>(a.v);
  p.status = a.status;
  p.B = d.B; p.S = d.S; p.H = d.H; p.Hkv = d.Hkv; p.G = d.G; p.DL = d.DL;
  p.NQ = d.NQ; p.NKV = d.NKV; p.NQKV = d.NQKV; p.VS0 = d.VS0;
  p.kv_stride = a.kv_stride;
  p.flags = d.flags;
  p.eps = d.eps;
  rope_turns_host(d.DL, d.rope_base, p.turns_hi, p.turns_lo, 64);
  const long long units = static_cast<long long>(d.B) * d.S * (d.H + 2 * d.Hkv);
  const long long threads = units * (d.DL / 8);
  if (threads >= (1LL << 30) || d.S >= (1 << 24)) return cudaErrorInvalidValue;
  const long long want = (threads + 511) / 512;      // two units per thread
  const long long cap = static_cast<long long>(num_sms()) * ((d.flags & F_QK_MEAN) ? 3 : 6);
  const unsigned blocks = static_cast<unsigned>(want < cap ? want : cap);
  const bool qkm = (d.flags & F_QK_MEAN) != 0;
  switch (d.DL) {
    case 16:
      if (qkm) pointwise_kernel<T, 16, true><<<blocks, 256, 0, st>>>(p);
      else pointwise_kernel<T, 16, false><<<blocks, 256, 0, st>>>(p);
      break;
    case 32:
      if (qkm) pointwise_kernel<T, 32, true><<<blocks, 256, 0, st>>>(p);
      else pointwise_kernel<T, 32, false><<<blocks, 256, 0, st>>>(p);
      break;
    case 64:
      if (qkm) pointwise_kernel<T, 64, true><<<blocks, 256, 0, st>>>(p);
      else pointwise_kernel<T, 64, false><<<blocks, 256, 0, st>>>(p);
      break;
    default:
      if (qkm) pointwise_kernel<T, 128, true><<<blocks, 256, 0, st>>>(p);
      else pointwise_kernel<T, 128, false><<<blocks, 256, 0, st>>>(p);
      break;
  }
  return cudaGetLastError();
}

__global__ void split_conv_chan_kernel(const float *__restrict__ w, uint2 *__restrict__ out,
                                       size_t npairs) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < npairs;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    uint2 r;
    split_bf16x2(*reinterpret_cast<const float2 *>(w + 2 * i), r.x, r.y);
    out[i] = r;
  }
}

}  // namespace

size_t conv_chan_split_bytes(const Dims &d) {
  return d.bf16 ? static_cast<size_t>(d.H + d.Hkv) * d.DL * d.DL * 4 : 0;
}

cudaError_t split_conv_chan(const Dims &d, const float *conv_chan, void *out, cudaStream_t st) {
  const size_t npairs = static_cast<size_t>(d.H + d.Hkv) * d.DL * d.DL / 2;
  const unsigned blocks = static_cast<unsigned>((npairs + 255) / 256 < 1024 ? (npairs + 255) / 256 : 1024);
  split_conv_chan_kernel<<<blocks, 256, 0, st>>>(conv_chan, static_cast<uint2 *>(out), npairs);
  return cudaGetLastError();
}

cudaError_t latent_stencil(const Dims &d, const StencilArgs &a, cudaStream_t st) {
  if (d.B == 0 || d.S == 0) return cudaSuccess;
  if (d.flags & F_NO_CONV) {
    if (a.write_state) return cudaErrorInvalidValue;   // no decode state without the convs
    return d.bf16 ? launch_pointwise<__nv_bfloat16>(d, a, st) : launch_pointwise<float>(d, a, st);
  }
  if (d.bf16) {
    if (d.DL == 16) return launch<__nv_bfloat16, 16>(d, a, st);
    if (d.DL == 32) return launch<__nv_bfloat16, 32>(d, a, st);
    if (d.DL == 64) return launch<__nv_bfloat16, 64>(d, a, st);
  } else {
    if (d.DL == 16) return launch<float, 16>(d, a, st);
    if (d.DL == 32) return launch<float, 32>(d, a, st);
    if (d.DL == 64) return launch<float, 64>(d, a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace cca
