// Latent stencil of the prefill: everything between the down-projection and the attention,
// fused into one pass over the projected latents P = x W_qkv^T.
//
// For every token t and key/value group g (gist.science explainer, 2. Methodology, Core
// Mechanism; edgentiq, "How Compressed Convolutional Attention Works"):
//   a  = causal depthwise conv of [pq | pk] along the sequence (KC taps, tap KC-1 = t)
//   b  = per-head channel conv of a (d~ x d~ matrix per head, pointwise in time)
//   q_h = b_h + (pq_h + pk_g)/2 ;  k_g = b_g + (mean_{h in g} pq_h + pk_g)/2   (Q-K-Mean)
//   v  = pv[t] on the lower half of the value channels, pv[t-1] on the upper half (Value-Shift)
//   q, k <- RMS-normalised per head, then rotated by RoPE at position t (RoPE Integration)
//
// One CTA owns a tile of TT tokens of one group of one sequence: it stages the group's
// P rows (plus a halo of KC-1 earlier tokens) in shared memory once, and writes q in
// head-major layout [B, H, S, d~] and k, v in [B, Hkv, kv_stride, d~] (the decode cache when
// one is given), as float16 for 16-bit layers.  Float32 arithmetic throughout.
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
  TL *q, *k, *v;
  float *conv_state, *vshift_state;
  int *lengths;
  int *status;
  int write_state;
  int B, S, H, Hkv, G, NQ, NKV, NQKV, KC, halo, TT, kv_stride;
  unsigned flags;
  float eps;
  float rope_base;
};

__host__ __device__ inline int stencil_ch(int G, int DL) { return (G + 2) * DL; }

template <int DL>
__host__ __device__ inline size_t stencil_smem_floats(int G, int TT, int halo) {
  return static_cast<size_t>(TT + halo) * stencil_ch(G, DL)      // Ps
         + static_cast<size_t>(TT) * (G + 1) * DL                // As
         + static_cast<size_t>(DL) * (DL + 1)                    // Ws
         + static_cast<size_t>(TT) * DL;                         // cos/sin table
}

template <typename T, int DL>
__global__ void __launch_bounds__(256) stencil_kernel(const StencilParams<T> p) {
  using TL = typename StencilParams<T>::TL;
  constexpr int LPI = DL < 32 ? DL : 32;   // lanes per (token, head) item
  constexpr int EPL = DL / LPI;            // elements per lane
  constexpr int IPW = 32 / LPI;            // items per warp pass
  constexpr int HALF = DL / 2;
  extern __shared__ float sm[];
  const int G = p.G, CH = stencil_ch(G, DL), QKC = (G + 1) * DL;
  const int TT = p.TT, halo = p.halo;
  float *Ps = sm;                                   // [TT+halo][CH]
  float *As = Ps + (TT + halo) * CH;                // [TT][QKC]
  float *Ws = As + TT * QKC;                        // [DL][DL+1]
  float *Rt = Ws + DL * (DL + 1);                   // [TT][HALF][2]

  const int g = blockIdx.y, b = blockIdx.z;
  const int t0 = blockIdx.x * TT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qcol0 = g * G * DL;                     // group's q channels in P
  const int kcol0 = p.NQ + g * DL;
  const int vcol0 = p.NQ + p.NKV + g * DL;

  // 1. stage P rows t0-halo .. t0+TT-1 of the group's channels (zero outside [0, S)).
  const int vec_per_row = CH / 8;
  for (int i = tid; i < (TT + halo) * vec_per_row; i += blockDim.x) {
    const int r = i / vec_per_row, c = (i % vec_per_row) * 8;
    const int t = t0 - halo + r;
    float v8[8];
    if (t >= 0 && t < p.S) {
      const int gc = c < G * DL ? qcol0 + c : (c < QKC ? kcol0 + (c - G * DL) : vcol0 + (c - QKC));
      load8(p.P + (static_cast<size_t>(b) * p.S + t) * p.NQKV + gc, v8);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v8[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) Ps[r * CH + c + e] = v8[e];
  }
  // RoPE table for this tile: angle = t * base^(-2i/d~), evaluated in double.
  if (p.flags & F_ROPE) {
    for (int i = tid; i < TT * HALF; i += blockDim.x) {
      const int tt = i / HALF, ip = i % HALF;
      const double theta = pow(static_cast<double>(p.rope_base), -2.0 * ip / DL);
      double s, c;
      sincos(static_cast<double>(t0 + tt) * theta, &s, &c);
      Rt[2 * i] = static_cast<float>(c);
      Rt[2 * i + 1] = static_cast<float>(s);
    }
  }
  __syncthreads();

  // 2. causal depthwise sequence conv of the q|k channels.
  for (int i = tid; i < TT * QKC; i += blockDim.x) {
    const int tt = i / QKC, c = i % QKC;
    const int gc = c < G * DL ? qcol0 + c : p.NQ + g * DL + (c - G * DL);
    const float *w = p.conv_seq + static_cast<size_t>(gc) * p.KC;
    float a = 0.f;
    const int r0 = tt + halo - (p.KC - 1);
    for (int j = 0; j < p.KC; ++j) a = fmaf(w[j], Ps[(r0 + j) * CH + c], a);
    As[tt * QKC + c] = a;
  }

  // 3. per head: channel conv, q-k-mean, RMS norm, RoPE, store.
  for (int hh = 0; hh <= G; ++hh) {
    const bool is_q = hh < G;
    const int head_w = is_q ? g * G + hh : p.H + g;     // row block of conv_chan
    __syncthreads();                                    // As ready / previous Ws consumed
    for (int i = tid; i < DL * DL; i += blockDim.x)
      Ws[(i / DL) * (DL + 1) + (i % DL)] = p.conv_chan[static_cast<size_t>(head_w) * DL * DL + i];
    __syncthreads();
    const int sub = lane / LPI, li = lane % LPI;
    for (int tt0 = warp * IPW; tt0 < TT; tt0 += (blockDim.x / 32) * IPW) {
      const int tt = tt0 + sub;
      const bool valid_tt = tt < TT;
      const int ttc = valid_tt ? tt : TT - 1;
      float u[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int i = e * LPI + li;
        const float *arow = As + ttc * QKC + hh * DL;
        const float *wrow = Ws + i * (DL + 1);
        float acc = 0.f;
#pragma unroll 8
        for (int j = 0; j < DL; ++j) acc = fmaf(wrow[j], arow[j], acc);
        if (p.flags & F_QK_MEAN) {
          const float *prow = Ps + (ttc + halo) * CH;
          const float pk = prow[G * DL + i];
          if (is_q) {
            acc += 0.5f * (prow[hh * DL + i] + pk);
          } else {
            float mq = 0.f;
            for (int h2 = 0; h2 < G; ++h2) mq += prow[h2 * DL + i];
            acc += 0.5f * (mq / static_cast<float>(G) + pk);
          }
        }
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
          const float c = Rt[(ttc * HALF + li) * 2], s = Rt[(ttc * HALF + li) * 2 + 1];
          const float x1 = u[0], x2 = u[1];
          u[0] = x1 * c - x2 * s;
          u[1] = x1 * s + x2 * c;
        } else {
          const float other = __shfl_xor_sync(0xffffffffu, u[0], HALF);
          const int ip = li % HALF;
          const float c = Rt[(ttc * HALF + ip) * 2], s = Rt[(ttc * HALF + ip) * 2 + 1];
          u[0] = li < HALF ? u[0] * c - other * s : other * s + u[0] * c;
        }
      }
      const int t = t0 + tt;
      if (valid_tt && t < p.S) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const int i = e * LPI + li;
          check_latent<TL>(u[e], p.status);
          if (is_q) {
            const int h = g * G + hh;
            p.q[((static_cast<size_t>(b) * p.H + h) * p.S + t) * DL + i] = from_f32<TL>(u[e]);
          } else {
            p.k[((static_cast<size_t>(b) * p.Hkv + g) * p.kv_stride + t) * DL + i] =
                from_f32<TL>(u[e]);
          }
        }
      }
    }
  }

  // 4. values with the value-shift: upper half of the value channels from token t-1.
  const int vhalf = p.NKV / 2;
  for (int i = tid; i < TT * DL; i += blockDim.x) {
    const int tt = i / DL, c = i % DL;
    const int t = t0 + tt;
    if (t >= p.S) continue;
    const bool shifted = (p.flags & F_VALUE_SHIFT) && (g * DL + c >= vhalf);
    const float val = Ps[(tt + halo - (shifted ? 1 : 0)) * CH + QKC + c];
    check_latent<TL>(val, p.status);
    p.v[((static_cast<size_t>(b) * p.Hkv + g) * p.kv_stride + t) * DL + c] = from_f32<TL>(val);
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
      p.conv_state[(static_cast<size_t>(b) * KC1 + j) * W + gc] = Ps[r * CH + c];
    }
    const int rl = p.S - 1 - t0 + halo;
    for (int c = tid; c < DL; c += blockDim.x) {
      const int gch = g * DL + c;
      if (gch >= vhalf)
        p.vshift_state[static_cast<size_t>(b) * (p.NKV - vhalf) + (gch - vhalf)] =
            Ps[rl * CH + QKC + c];
    }
    if (g == 0 && tid == 0) p.lengths[b] = p.S;
  }
}

template <typename T, int DL>
cudaError_t launch(const Dims &d, const StencilArgs &a, cudaStream_t st) {
  using TL = typename LatentType<T>::type;
  StencilParams<T> p;
  p.P = a.P;
  p.conv_seq = a.conv_seq;
  p.conv_chan = a.conv_chan;
  p.q = static_cast<TL *>(a.q);
  p.k = static_cast<TL *>(a.k);
  p.v = static_cast<TL *>(a.v);
  p.status = a.status;
  p.conv_state = a.conv_state;
  p.vshift_state = a.vshift_state;
  p.lengths = a.lengths;
  p.write_state = a.write_state ? 1 : 0;
  p.B = d.B; p.S = d.S; p.H = d.H; p.Hkv = d.Hkv; p.G = d.G;
  p.NQ = d.NQ; p.NKV = d.NKV; p.NQKV = d.NQKV; p.KC = d.KC;
  p.halo = d.KC - 1 > 1 ? d.KC - 1 : 1;
  p.kv_stride = a.kv_stride;
  p.flags = d.flags;
  p.eps = d.eps;
  p.rope_base = d.rope_base;
  int TT = 64;
  while (TT > 4 && stencil_smem_floats<DL>(d.G, TT, p.halo) * 4 > 72 * 1024) TT /= 2;
  p.TT = TT;
  const size_t smem = stencil_smem_floats<DL>(d.G, TT, p.halo) * 4;
  if (smem > 200 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(stencil_kernel<T, DL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((d.S + TT - 1) / TT, d.Hkv, d.B);
  stencil_kernel<T, DL><<<grid, 256, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t latent_stencil(const Dims &d, const StencilArgs &a, cudaStream_t st) {
  if (d.B == 0 || d.S == 0) return cudaSuccess;
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
