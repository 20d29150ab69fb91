// Causal softmax attention on latent-width heads (gist.science/de explainer, 2. Methodik:
// Softmax(QK^T)V is evaluated entirely in the compressed space; gist.science explainer,
// Extension: CCGQA: query head h reads key/value head h / (H/Hkv)).
//
//   O[b, t, h*d~ + :] = sum_{s <= t} softmax_s(q[b,h,t] . k[b,g,s] / sqrt(d~)) v[b,g,s]
//
// Two kernels:
//  * attn_mma_kernel (16-bit layers): flash-style online softmax over 64-key tiles, mma.sync
//    m16n8k16 f16 x f16 -> f32 for QK^T and PV (float16 latents and probabilities), fp32
//    softmax, float16 output; causal tiles above the diagonal are skipped.
//  * attn_simt_kernel (float32): one warp per query row, exact fp32 arithmetic.
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int BM = 64, BN = 64;

template <int DL>
__global__ void __launch_bounds__(128) attn_mma_kernel(
    const __half *__restrict__ Q, const __half *__restrict__ K,
    const __half *__restrict__ V, __half *__restrict__ O, int S, int H, int Hkv,
    int G, int kv_stride, float scale_log2) {
  constexpr int KP = DL + 8;      // padded K row (bf16)
  constexpr int VP = BN + 8;      // padded V^T row (bf16)
  __shared__ __align__(16) __half Ks[BN * KP];
  __shared__ __align__(16) __half Vt[DL * VP];
  const int nqt = (S + BM - 1) / BM;
  const int qt = nqt - 1 - blockIdx.x;            // longest rows first
  const int h = blockIdx.y, b = blockIdx.z, g = h / G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, qc = lane & 3;
  const int q0 = qt * BM;
  const int qa = q0 + warp * 16 + gr, qb = qa + 8;

  const __half *Qh = Q + (static_cast<size_t>(b) * H + h) * S * DL;
  const __half *Kg = K + (static_cast<size_t>(b) * Hkv + g) * kv_stride * DL;
  const __half *Vg = V + (static_cast<size_t>(b) * Hkv + g) * kv_stride * DL;

  // Q fragments (A operand), zero for rows past the sequence end.
  uint32_t qf[DL / 16][4];
#pragma unroll
  for (int kk = 0; kk < DL / 16; ++kk) {
    const int c0 = kk * 16 + 2 * qc;
    auto ld = [&](int row, int col) -> uint32_t {
      if (row >= S) return 0u;
      return *reinterpret_cast<const uint32_t *>(Qh + static_cast<size_t>(row) * DL + col);
    };
    qf[kk][0] = ld(qa, c0);
    qf[kk][1] = ld(qb, c0);
    qf[kk][2] = ld(qa, c0 + 8);
    qf[kk][3] = ld(qb, c0 + 8);
  }

  float o[DL / 8][4];
#pragma unroll
  for (int i = 0; i < DL / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  for (int kt = 0; kt <= qt; ++kt) {
    const int kv0 = kt * BN;
    __syncthreads();
    // stage K (row-major) and V (transposed) tiles; zero past the sequence end
    for (int i = threadIdx.x; i < BN * DL / 8; i += blockDim.x) {
      const int r = i / (DL / 8), c = (i % (DL / 8)) * 8;
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (kv0 + r < S) {
        kv = *reinterpret_cast<const uint4 *>(Kg + static_cast<size_t>(kv0 + r) * DL + c);
        vv = *reinterpret_cast<const uint4 *>(Vg + static_cast<size_t>(kv0 + r) * DL + c);
      }
      *reinterpret_cast<uint4 *>(Ks + r * KP + c) = kv;
      const __half *ve = reinterpret_cast<const __half *>(&vv);
#pragma unroll
      for (int e = 0; e < 8; ++e) Vt[(c + e) * VP + r] = ve[e];
    }
    __syncthreads();

    float s[BN / 8][4];
#pragma unroll
    for (int j = 0; j < BN / 8; ++j) {
      s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < DL / 16; ++kk) {
        const __half *kr = Ks + (j * 8 + gr) * KP + kk * 16 + 2 * qc;
        uint32_t bf[2] = {*reinterpret_cast<const uint32_t *>(kr),
                          *reinterpret_cast<const uint32_t *>(kr + 8)};
        mma_f16_16816(s[j], qf[kk], bf);
      }
    }
    // scale, causal mask, running max
    const bool diag = (kt == qt);
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int j = 0; j < BN / 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float x = s[j][e] * scale_log2;
        const int key = kv0 + j * 8 + 2 * qc + (e & 1);
        const int qrow = (e < 2) ? qa : qb;
        if (diag && key > qrow) x = -INFINITY;
        s[j][e] = x;
      }
      mx_a = fmaxf(mx_a, fmaxf(s[j][0], s[j][1]));
      mx_b = fmaxf(mx_b, fmaxf(s[j][2], s[j][3]));
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    // rows past the sequence end see only masked keys on the diagonal tile; keep them finite
    const float base_a = mn_a == -INFINITY ? 0.f : mn_a;
    const float base_b = mn_b == -INFINITY ? 0.f : mn_b;
    const float corr_a = exp2f(m_a - base_a), corr_b = exp2f(m_b - base_b);
    m_a = mn_a;
    m_b = mn_b;
    float sum_a = 0.f, sum_b = 0.f;
    uint32_t pf[BN / 16][4];
#pragma unroll
    for (int j = 0; j < BN / 8; ++j) {
      const float p0 = exp2f(s[j][0] - base_a), p1 = exp2f(s[j][1] - base_a);
      const float p2 = exp2f(s[j][2] - base_b), p3 = exp2f(s[j][3] - base_b);
      sum_a += p0 + p1;
      sum_b += p2 + p3;
      const int kk = j >> 1;
      if ((j & 1) == 0) {
        pf[kk][0] = pack_f16x2(p0, p1);
        pf[kk][1] = pack_f16x2(p2, p3);
      } else {
        pf[kk][2] = pack_f16x2(p0, p1);
        pf[kk][3] = pack_f16x2(p2, p3);
      }
    }
    l_a = l_a * corr_a + sum_a;
    l_b = l_b * corr_b + sum_b;
#pragma unroll
    for (int dt = 0; dt < DL / 8; ++dt) {
      o[dt][0] *= corr_a;
      o[dt][1] *= corr_a;
      o[dt][2] *= corr_b;
      o[dt][3] *= corr_b;
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        const __half *vr = Vt + (dt * 8 + gr) * VP + kk * 16 + 2 * qc;
        uint32_t bf[2] = {*reinterpret_cast<const uint32_t *>(vr),
                          *reinterpret_cast<const uint32_t *>(vr + 8)};
        mma_f16_16816(o[dt], pf[kk], bf);
      }
    }
  }
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float ia = l_a > 0.f ? 1.f / l_a : 0.f, ib = l_b > 0.f ? 1.f / l_b : 0.f;
  const int NQ = H * DL;
#pragma unroll
  for (int dt = 0; dt < DL / 8; ++dt) {
    const int col = h * DL + dt * 8 + 2 * qc;
    if (qa < S)
      *reinterpret_cast<uint32_t *>(O + (static_cast<size_t>(b) * S + qa) * NQ + col) =
          pack_f16x2(o[dt][0] * ia, o[dt][1] * ia);
    if (qb < S)
      *reinterpret_cast<uint32_t *>(O + (static_cast<size_t>(b) * S + qb) * NQ + col) =
          pack_f16x2(o[dt][2] * ib, o[dt][3] * ib);
  }
}

// float32: one warp per (b, h, t); lanes hold dims lane and lane+32.
template <int DL>
__global__ void __launch_bounds__(256) attn_simt_kernel(const float *__restrict__ Q,
                                                        const float *__restrict__ K,
                                                        const float *__restrict__ V,
                                                        float *__restrict__ O, int B, int S, int H,
                                                        int Hkv, int G, int kv_stride,
                                                        float scale_log2) {
  constexpr int EPL = (DL + 31) / 32;
  const int gw = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= B * H * S) return;
  const int t = gw % S, h = (gw / S) % H, b = gw / (S * H), g = h / G;
  const float *q = Q + ((static_cast<size_t>(b) * H + h) * S + t) * DL;
  const float *Kg = K + (static_cast<size_t>(b) * Hkv + g) * kv_stride * DL;
  const float *Vg = V + (static_cast<size_t>(b) * Hkv + g) * kv_stride * DL;
  float qv[EPL], acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int d = lane + 32 * e;
    qv[e] = d < DL ? q[d] * scale_log2 : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int s = 0; s <= t; ++s) {
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int d = lane + 32 * e;
      if (d < DL) part = fmaf(qv[e], Kg[static_cast<size_t>(s) * DL + d], part);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    const float mn = fmaxf(m, part);
    const float corr = exp2f(m - mn), p = exp2f(part - mn);
    l = l * corr + p;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int d = lane + 32 * e;
      const float vv = d < DL ? Vg[static_cast<size_t>(s) * DL + d] : 0.f;
      acc[e] = acc[e] * corr + p * vv;
    }
    m = mn;
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int d = lane + 32 * e;
    if (d < DL) O[(static_cast<size_t>(b) * S + t) * (H * DL) + h * DL + d] = acc[e] / l;
  }
}

}  // namespace

static cudaError_t launch_mma(const Dims &d, const void *q, const void *k, const void *v,
                              int kv_stride, void *o, float scale_log2, cudaStream_t st) {
  dim3 grid((d.S + BM - 1) / BM, d.H, d.B);
  auto Q = static_cast<const __half *>(q);
  auto Kp = static_cast<const __half *>(k);
  auto Vp = static_cast<const __half *>(v);
  auto Op = static_cast<__half *>(o);
  if (d.DL == 16)
    attn_mma_kernel<16><<<grid, 128, 0, st>>>(Q, Kp, Vp, Op, d.S, d.H, d.Hkv, d.G, kv_stride, scale_log2);
  else if (d.DL == 32)
    attn_mma_kernel<32><<<grid, 128, 0, st>>>(Q, Kp, Vp, Op, d.S, d.H, d.Hkv, d.G, kv_stride, scale_log2);
  else if (d.DL == 64)
    attn_mma_kernel<64><<<grid, 128, 0, st>>>(Q, Kp, Vp, Op, d.S, d.H, d.Hkv, d.G, kv_stride, scale_log2);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t latent_attention(const Dims &d, const void *q, const void *k, const void *v,
                             int kv_stride, void *o, int *status, cudaStream_t st) {
  (void)status;
  if (d.B == 0 || d.S == 0) return cudaSuccess;
  const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(d.DL)));
  if (d.bf16) {
    return launch_mma(d, q, k, v, kv_stride, o, scale_log2, st);
  } else {
    const long long rows = static_cast<long long>(d.B) * d.H * d.S;
    const int grid = static_cast<int>((rows + 7) / 8);
    auto Q = static_cast<const float *>(q);
    auto Kp = static_cast<const float *>(k);
    auto Vp = static_cast<const float *>(v);
    auto Op = static_cast<float *>(o);
    if (d.DL == 16)
      attn_simt_kernel<16><<<grid, 256, 0, st>>>(Q, Kp, Vp, Op, d.B, d.S, d.H, d.Hkv, d.G, kv_stride, scale_log2);
    else if (d.DL == 32)
      attn_simt_kernel<32><<<grid, 256, 0, st>>>(Q, Kp, Vp, Op, d.B, d.S, d.H, d.Hkv, d.G, kv_stride, scale_log2);
    else if (d.DL == 64)
      attn_simt_kernel<64><<<grid, 256, 0, st>>>(Q, Kp, Vp, Op, d.B, d.S, d.H, d.Hkv, d.G, kv_stride, scale_log2);
    else
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace cca
