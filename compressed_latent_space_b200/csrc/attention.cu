// Causal softmax attention on latent-width heads (gist.science/de explainer, 2. Methodik:
// Softmax(QK^T)V is evaluated entirely in the compressed space; gist.science explainer,
// Extension: CCGQA: query head h reads key/value head h / (H/Hkv)).
//
//   O[b, t, h*d~ + :] = sum_{s <= t} softmax_s(q[b,h,t] . k[b,g,s] / sqrt(d~)) v[b,g,s]
//
// 16-bit layers run the tcgen05 kernel of attention_tc.cu; float32 layers run
// attn_simt_kernel below: one warp per query row, exact fp32 arithmetic.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

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

cudaError_t latent_attention(const Dims &d, const void *q, const void *k, const void *v,
                             int kv_stride, void *o, int *status, cudaStream_t st) {
  if (d.B == 0 || d.S == 0) return cudaSuccess;
  const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(d.DL)));
  if (d.bf16) {
    return latent_attention_tc(d, q, k, v, kv_stride, o, status, st);
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
