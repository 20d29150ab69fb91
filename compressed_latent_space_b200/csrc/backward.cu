// Backward pass of the latent stencil, and the layout helpers of the backward pass's GEMMs.
// (gist.science explainer, 2. Methodology, Core Mechanism: the steps between the projections
// and the attention; 4. Experimental Results: the backward pass is measured.)
//
// The forward stencil maps the projections P to q, k, v (sequence conv, channel conv,
// Q-K-Mean, value-shift, RMS norm, RoPE).  Given dq, dk, dv from the attention's backward pass,
// pass 1 recomputes the forward's intermediates of each token from P and takes the chain rule
// back through RoPE (a rotation by the negative angle), the norm (du = (dn - n mean(dn n)) / r),
// Q-K-Mean (its skip terms go straight to dP; the post-conv term to the channel conv) and the
// channel conv (dA = W_c^T dB per head; dW_c = sum over tokens of dB A^T), and writes the
// value gradient with the value-shift undone.  Pass 2 takes the sequence conv back
// (dP[s, c] += sum_j w[c, j] dA[s + k-1-j, c]; dw[c, j] = sum_t dA[t, c] P[t-(k-1)+j, c]) and
// writes dP in bfloat16 for the gradient GEMMs.  Weight gradients are reduced per CTA in
// registers and added to the float32 outputs once per CTA.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int S1_TT = 16;          // tokens per pass-1 tile
constexpr int S1_THREADS = 256;
constexpr int S1_MAX_BLOCKS = 5;        // 4 x 4 blocks of filter-gradient entries per thread
constexpr int S1_MAX_PER_THREAD = 16 * S1_MAX_BLOCKS;

struct S1Params {
  const float *P;                  // [B*S, NQKV] forward projections
  const float *dq, *dk, *dv;       // [B, H, S, DL], [B, Hkv, S, DL] float32
  const float *conv_seq;           // [NQ + NKV, KC]
  const float *conv_chan;          // [H + Hkv, DL, DL]
  float *dA;                       // [B*S, NQ + NKV] gradient of the sequence-conv output
  float *dPpart;                   // [B*S, NQKV] Q-K-Mean skip and value gradients
  float *dconv_chan;               // [H + Hkv, DL, DL] (accumulated)
  int B, S, H, Hkv, G, DL, NQ, NKV, NQKV, KC, VS0;
  unsigned flags;
  float eps;
  double theta[32];
};

// smem (floats): Wc [(G+1) DL x (DL+4)] (rows padded by four floats: 16-byte aligned rows whose
// 128-bit reads across a quarter warp's rows hit distinct banks, and column reads across a
// warp's columns stay contiguous) | Ps [(TT + KC-1) x (G+2)DL] | A [TT x (G+1)DL] | U [same] |
// dU [same] | N [same]
__host__ __device__ inline size_t s1_smem_floats(int G, int DL, int KC) {
  const size_t QK = static_cast<size_t>(G + 1) * DL;
  return QK * (DL + 4) + static_cast<size_t>(S1_TT + KC - 1) * (G + 2) * DL + 4 * S1_TT * QK;
}

__global__ void __launch_bounds__(S1_THREADS, 1) stencil_bwd1_kernel(const S1Params p, int cpg,
                                                                     int tiles_per_seq) {
  extern __shared__ __align__(16) float sm[];
  const int G = p.G, DL = p.DL, KC = p.KC, KC1 = KC - 1;
  const int QK = (G + 1) * DL, CH = (G + 2) * DL;
  const int WL = DL + 4;                             // padded filter row
  float *Wc = sm;
  float *Ps = Wc + QK * WL;
  float *A = Ps + (S1_TT + KC1) * CH;
  float *U = A + S1_TT * QK;
  float *dU = U + S1_TT * QK;
  float *Nn = dU + S1_TT * QK;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
  const int g = blockIdx.y, ci = blockIdx.x;
  const int units = p.B * tiles_per_seq;
  const int u_beg = static_cast<int>(static_cast<long long>(units) * ci / cpg);
  const int u_end = static_cast<int>(static_cast<long long>(units) * (ci + 1) / cpg);
  const int qcol0 = g * G * DL, kcol0 = p.NQ + g * DL, vcol0 = p.NQ + p.NKV + g * DL;
  auto head_glob = [&](int hh) { return hh < G ? g * G + hh : p.H + g; };
  // the group's channel filters, [head][out i][in c]
  for (int e = tid; e < QK * DL; e += nt) {
    const int hh = e / (DL * DL), r = e % (DL * DL);
    Wc[(hh * DL + r / DL) * WL + r % DL] = p.conv_chan[static_cast<size_t>(head_glob(hh)) * DL * DL + r];
  }
  const int BPH = (DL / 4) * (DL / 4);               // 4 x 4 filter-gradient blocks per head
  const int NB = (G + 1) * BPH;
  float acc[S1_MAX_PER_THREAD];
#pragma unroll
  for (int m = 0; m < S1_MAX_PER_THREAD; ++m) acc[m] = 0.f;
  __syncthreads();

  for (int u = u_beg; u < u_end; ++u) {
    const int b = u / tiles_per_seq, t0 = (u % tiles_per_seq) * S1_TT;
    // P rows t0-KC1 .. t0+TT-1 of the group's q | k | v channels (zero outside the sequence)
    for (int e = tid; e < (S1_TT + KC1) * CH; e += nt) {
      const int r = e / CH, c = e % CH;
      const int t = t0 - KC1 + r;
      const int gc = c < G * DL ? qcol0 + c : (c < QK ? kcol0 + (c - G * DL) : vcol0 + (c - QK));
      Ps[e] = (t >= 0 && t < p.S) ? p.P[(static_cast<size_t>(b) * p.S + t) * p.NQKV + gc] : 0.f;
    }
    __syncthreads();
    // sequence conv of the q | k channels
    for (int e = tid; e < S1_TT * QK; e += nt) {
      const int tt = e / QK, c = e % QK;
      const int gc = c < G * DL ? qcol0 + c : kcol0 + (c - G * DL);
      float a = 0.f;
      for (int j = 0; j < KC; ++j) a = fmaf(p.conv_seq[static_cast<size_t>(gc) * KC + j], Ps[(tt + j) * CH + c], a);
      A[e] = a;
    }
    __syncthreads();
    // channel conv and Q-K-Mean: U = W_c A + skip; a thread per output channel, all TT tokens,
    // the filter row and the tokens' inputs read four floats at a time
    for (int hc = tid; hc < QK; hc += nt) {
      const int hh = hc / DL, i = hc % DL;
      const float4 *w4 = reinterpret_cast<const float4 *>(Wc + (hh * DL + i) * WL);
      float v[S1_TT];
#pragma unroll
      for (int tt = 0; tt < S1_TT; ++tt) v[tt] = 0.f;
      for (int c4 = 0; c4 < DL / 4; ++c4) {
        const float4 w = w4[c4];
#pragma unroll
        for (int tt = 0; tt < S1_TT; ++tt) {
          const float4 a = reinterpret_cast<const float4 *>(A + tt * QK + hh * DL)[c4];
          v[tt] = fmaf(w.x, a.x, fmaf(w.y, a.y, fmaf(w.z, a.z, fmaf(w.w, a.w, v[tt]))));
        }
      }
#pragma unroll
      for (int tt = 0; tt < S1_TT; ++tt) {
        float x = v[tt];
        if (p.flags & F_QK_MEAN) {
          const float *pr = Ps + (tt + KC1) * CH;
          const float pk = pr[G * DL + i];
          float pq;
          if (hh < G) {
            pq = pr[hh * DL + i];
          } else {
            pq = 0.f;
            for (int h2 = 0; h2 < G; ++h2) pq += pr[h2 * DL + i];
            pq /= static_cast<float>(G);
          }
          x += 0.5f * (pq + pk);
        }
        U[tt * QK + hc] = x;
      }
    }
    __syncthreads();
    // per (token, head): norm statistics, dn = RoPE^-1(dq or dk), du; one warp per pair
    for (int it = warp; it < S1_TT * (G + 1); it += nwarps) {
      const int tt = it / (G + 1), hh = it % (G + 1);
      const int t = t0 + tt;
      float *uu = U + tt * QK + hh * DL, *nn = Nn + tt * QK + hh * DL, *du = dU + tt * QK + hh * DL;
      if (t >= p.S) {                                // past the sequence: no gradient
        for (int c = lane; c < DL; c += 32) { du[c] = 0.f; nn[c] = 0.f; }
        continue;
      }
      float ss = 0.f;
      for (int c = lane; c < DL; c += 32) ss += uu[c] * uu[c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const bool norm = (p.flags & F_QK_NORM) != 0;
      const float r = norm ? sqrtf(ss / static_cast<float>(DL) + p.eps) : 1.f;
      const float *src = hh < G ? p.dq + ((static_cast<size_t>(b) * p.H + g * G + hh) * p.S + t) * DL
                                : p.dk + ((static_cast<size_t>(b) * p.Hkv + g) * p.S + t) * DL;
      const int HALF = DL / 2;
      float dot = 0.f;
      for (int i = lane; i < HALF; i += 32) {
        float d1 = src[i], d2 = src[i + HALF];
        if (p.flags & F_ROPE) {                      // rotate back by -t theta_i
          float cs, sn;
          rope_cos_sin(static_cast<double>(t) * p.theta[i], cs, sn);
          const float a1 = d1 * cs + d2 * sn, a2 = -d1 * sn + d2 * cs;
          d1 = a1;
          d2 = a2;
        }
        const float n1 = uu[i] / r, n2 = uu[i + HALF] / r;
        nn[i] = n1;
        nn[i + HALF] = n2;
        du[i] = d1;                                  // dn for now
        du[i + HALF] = d2;
        dot += d1 * n1 + d2 * n2;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      __syncwarp();
      if (norm) {
        const float mdn = dot / static_cast<float>(DL);
        for (int c = lane; c < DL; c += 32) du[c] = (du[c] - nn[c] * mdn) / r;
      }
    }
    __syncthreads();
    // dA = W_c^T dU per head, and the Q-K-Mean skip gradients of the q | k projections; a
    // thread per input channel, all TT tokens, the tokens' dU read four floats at a time
    for (int hc = tid; hc < QK; hc += nt) {
      const int hh = hc / DL, c = hc % DL;
      float v[S1_TT];
#pragma unroll
      for (int tt = 0; tt < S1_TT; ++tt) v[tt] = 0.f;
      for (int i4 = 0; i4 < DL / 4; ++i4) {
        const float *wc = Wc + (hh * DL + 4 * i4) * WL + c;
        const float w0 = wc[0], w1 = wc[WL], w2 = wc[2 * WL], w3 = wc[3 * WL];
#pragma unroll
        for (int tt = 0; tt < S1_TT; ++tt) {
          const float4 d = reinterpret_cast<const float4 *>(dU + tt * QK + hh * DL)[i4];
          v[tt] = fmaf(w0, d.x, fmaf(w1, d.y, fmaf(w2, d.z, fmaf(w3, d.w, v[tt]))));
        }
      }
      const int gc = hh < G ? qcol0 + hh * DL + c : kcol0 + c;
#pragma unroll
      for (int tt = 0; tt < S1_TT; ++tt) {
        const int t = t0 + tt;
        if (t >= p.S) continue;
        const size_t row = static_cast<size_t>(b) * p.S + t;
        p.dA[row * (p.NQ + p.NKV) + gc] = v[tt];
        float skip = 0.f;
        if (p.flags & F_QK_MEAN) {
          const float duk = dU[tt * QK + G * DL + c];
          if (hh < G) {
            skip = 0.5f * dU[tt * QK + hh * DL + c] + duk / (2.0f * static_cast<float>(G));
          } else {
            float sq = 0.f;
            for (int h2 = 0; h2 < G; ++h2) sq += dU[tt * QK + h2 * DL + c];
            skip = 0.5f * sq + 0.5f * duk;
          }
        }
        p.dPpart[row * p.NQKV + gc] = skip;
      }
    }
    // values: dPv[t, c] = dv[t, c] unshifted, dv[t+1, c] shifted
    for (int e = tid; e < S1_TT * DL; e += nt) {
      const int tt = e / DL, c = e % DL;
      const int t = t0 + tt;
      if (t >= p.S) continue;
      const int gvc = g * DL + c;
      const bool shifted = (p.flags & F_VALUE_SHIFT) && gvc >= p.VS0;
      const int ts = shifted ? t + 1 : t;
      const float val = ts < p.S ? p.dv[((static_cast<size_t>(b) * p.Hkv + g) * p.S + ts) * DL + c] : 0.f;
      p.dPpart[(static_cast<size_t>(b) * p.S + t) * p.NQKV + vcol0 + c] = val;
    }
    // channel-filter gradient: dW_c[h][i][c] += sum_tt dU[tt][h][i] A[tt][h][c], a 4 x 4 block
    // of (i, c) per thread and block slot
#pragma unroll
    for (int m = 0; m < S1_MAX_BLOCKS; ++m) {
      const int blk = tid + m * S1_THREADS;
      if (blk < NB) {
        const int hh = blk / BPH, r = blk % BPH;
        const int i0 = (r / (DL / 4)) * 4, c0 = (r % (DL / 4)) * 4;
#pragma unroll
        for (int tt = 0; tt < S1_TT; ++tt) {
          const float4 d = *reinterpret_cast<const float4 *>(dU + tt * QK + hh * DL + i0);
          const float4 a = *reinterpret_cast<const float4 *>(A + tt * QK + hh * DL + c0);
          const float dv4[4] = {d.x, d.y, d.z, d.w}, av4[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
          for (int ii = 0; ii < 4; ++ii)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              acc[m * 16 + ii * 4 + cc] = fmaf(dv4[ii], av4[cc], acc[m * 16 + ii * 4 + cc]);
        }
      }
    }
    __syncthreads();                                 // Ps, A, U, dU rewritten by the next tile
  }
#pragma unroll
  for (int m = 0; m < S1_MAX_BLOCKS; ++m) {
    const int blk = tid + m * S1_THREADS;
    if (blk < NB && u_end > u_beg) {
      const int hh = blk / BPH, r = blk % BPH;
      const int i0 = (r / (DL / 4)) * 4, c0 = (r % (DL / 4)) * 4;
      float *dst = p.dconv_chan + static_cast<size_t>(head_glob(hh)) * DL * DL;
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          atomicAdd(dst + (i0 + ii) * DL + c0 + cc, acc[m * 16 + ii * 4 + cc]);
    }
  }
}

// Pass 2: one thread per (q|k channel, token range); the sequence conv's transpose and its
// filter gradient, then dP in bfloat16 (the value columns are converted as they are).
constexpr int S2_TOK = 256;                          // tokens per thread's range

__global__ void __launch_bounds__(256) stencil_bwd2_kernel(
    const float *__restrict__ P, const float *__restrict__ dA, const float *__restrict__ dPpart,
    const float *__restrict__ conv_seq, __nv_bfloat16 *__restrict__ dP, float *__restrict__ dconv_seq,
    int B, int S, int NQ, int NKV, int NQKV, int KC) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;   // column of dP (all NQKV)
  const int seg = blockIdx.y;                            // token range of (B*S)
  if (c >= NQKV) return;
  const long long M = static_cast<long long>(B) * S;
  const long long t_beg = static_cast<long long>(seg) * S2_TOK;
  const long long t_end = t_beg + S2_TOK < M ? t_beg + S2_TOK : M;
  const bool qk = c < NQ + NKV;
  float w[8], dw[8];
  for (int j = 0; j < 8; ++j) {
    w[j] = (qk && j < KC) ? conv_seq[static_cast<size_t>(c) * KC + j] : 0.f;
    dw[j] = 0.f;
  }
  const int W = NQ + NKV;
  for (long long row = t_beg; row < t_end; ++row) {
    const int t = static_cast<int>(row % S);
    float v = dPpart[row * NQKV + c];
    if (qk) {
      for (int j = 0; j < KC; ++j) {
        const int lag = KC - 1 - j;                      // output t + lag read input t by tap j
        if (t + lag < S) v = fmaf(w[j], dA[(row + lag) * W + c], v);
        if (t - lag >= 0) dw[j] = fmaf(dA[row * W + c], P[(row - lag) * NQKV + c], dw[j]);
      }
    }
    dP[row * NQKV + c] = __float2bfloat16_rn(v);
  }
  if (qk)
    for (int j = 0; j < KC; ++j) atomicAdd(dconv_seq + static_cast<size_t>(c) * KC + j, dw[j]);
}

// out[c][r] = in[r][c] for r < R, zero for R <= r < R8 (R8 = R rounded up to 8, so every output
// row is a whole number of 16-byte pieces for TMA); 16-bit elements, float16 converted to
// bfloat16 when to_bf16.
__global__ void __launch_bounds__(256) transpose16_kernel(const uint16_t *__restrict__ in,
                                                          uint16_t *__restrict__ out, int R, int C,
                                                          int R8, int from_f16) {
  __shared__ uint16_t tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;     // 8 rows of 32 per pass
  for (int k = ty; k < 32; k += 8) {
    const int r = r0 + k, c = c0 + tx;
    uint16_t v = 0;
    if (r < R && c < C) {
      v = in[static_cast<size_t>(r) * C + c];
      if (from_f16) {
        const __half hv = *reinterpret_cast<const __half *>(&v);
        const __nv_bfloat16 bv = __float2bfloat16_rn(__half2float(hv));
        v = *reinterpret_cast<const uint16_t *>(&bv);
      }
    }
    tile[k][tx] = v;
  }
  __syncthreads();
  for (int k = ty; k < 32; k += 8) {
    const int c = c0 + k, r = r0 + tx;
    if (c < C && r < R8) out[static_cast<size_t>(c) * R8 + r] = tile[tx][k];
  }
}

}  // namespace

bool stencil_backward_supported(const Dims &d) {
  return d.bf16 && !(d.flags & F_NO_CONV) && d.DL <= 64 && d.KC <= 8 &&
         (d.G + 1) * (d.DL / 4) * (d.DL / 4) <= S1_MAX_BLOCKS * S1_THREADS &&
         s1_smem_floats(d.G, d.DL, d.KC) * 4 <= 200 * 1024;
}

cudaError_t stencil_backward(const Dims &d, const StencilBwdArgs &a, cudaStream_t st) {
  if (d.B == 0 || d.S == 0) return cudaSuccess;
  S1Params p;
  p.P = a.P;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.conv_seq = a.conv_seq;
  p.conv_chan = a.conv_chan;
  p.dA = a.dA;
  p.dPpart = a.dPpart;
  p.dconv_chan = a.dconv_chan;
  p.B = d.B; p.S = d.S; p.H = d.H; p.Hkv = d.Hkv; p.G = d.G; p.DL = d.DL;
  p.NQ = d.NQ; p.NKV = d.NKV; p.NQKV = d.NQKV; p.KC = d.KC; p.VS0 = d.VS0;
  p.flags = d.flags;
  p.eps = d.eps;
  for (int i = 0; i < 32; ++i)
    p.theta[i] = i < d.DL / 2 ? pow(static_cast<double>(d.rope_base), -2.0 * i / d.DL) : 0.0;
  const int tiles = (d.S + S1_TT - 1) / S1_TT;
  const int units = d.B * tiles;
  int cpg = num_sms() / d.Hkv;
  if (cpg < 1) cpg = 1;
  if (cpg > units) cpg = units;
  const size_t smem = s1_smem_floats(d.G, d.DL, d.KC) * 4;
  cudaError_t e;
  if ((e = ensure_dyn_smem<stencil_bwd1_kernel>(smem)) != cudaSuccess) return e;
  stencil_bwd1_kernel<<<dim3(cpg, d.Hkv), S1_THREADS, smem, st>>>(p, cpg, tiles);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long M = static_cast<long long>(d.B) * d.S;
  const dim3 g2((d.NQKV + 255) / 256, static_cast<unsigned>((M + S2_TOK - 1) / S2_TOK));
  stencil_bwd2_kernel<<<g2, 256, 0, st>>>(a.P, a.dA, a.dPpart, a.conv_seq,
                                         static_cast<__nv_bfloat16 *>(a.dP), a.dconv_seq, d.B, d.S,
                                         d.NQ, d.NKV, d.NQKV, d.KC);
  return cudaGetLastError();
}

cudaError_t transpose16(const void *in, void *out, int R, int C, int R8, bool from_f16,
                        cudaStream_t st) {
  if (R8 <= 0 || C <= 0) return cudaSuccess;
  const dim3 grid((C + 31) / 32, (R8 + 31) / 32);
  transpose16_kernel<<<grid, 256, 0, st>>>(static_cast<const uint16_t *>(in),
                                          static_cast<uint16_t *>(out), R, C, R8, from_f16 ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace cca
