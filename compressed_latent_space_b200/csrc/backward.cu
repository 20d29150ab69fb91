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

constexpr int S1_TT = 16;          // tokens per pass-1 tile (the M of its mma.sync tiles)
constexpr int S1_THREADS = 256;
constexpr int S1_WARPS = S1_THREADS / 32;
constexpr int S1_MAXB = 20;        // filter-gradient 16 x 8 blocks per warp
constexpr int S1_KCMAX = 8;

struct S1Params {
  const float *P;                  // [B*S, NQKV] forward projections
  const float *dq, *dk, *dv;       // [B, H, S, DL], [B, Hkv, S, DL] float32
  const float *conv_seq;           // [NQ + NKV, KC]
  const uint2 *wsplit;             // channel filters as bf16 hi/lo pairs, [head][out i][in pair]
  const uint2 *wsplitT;            // the same transposed, [head][in c][out pair]
  float *dA;                       // [B*S, NQ + NKV] gradient of the sequence-conv output
  float *dPpart;                   // [B*S, NQKV] Q-K-Mean skip and value gradients
  float *dconv_chan;               // [H + Hkv, DL, DL] (accumulated)
  int B, S, H, Hkv, G, NQ, NKV, NQKV, KC, VS0;
  unsigned flags;
  float eps;
  float turns_hi[32], turns_lo[32];  // RoPE frequencies in turns, as float pairs
};

// Row strides of the shared-memory tiles: a multiple of 32 floats plus 4, so that the mma
// fragment reads (eight rows x four column pairs, or four row pairs x eight columns) fall on
// distinct banks.
__host__ __device__ constexpr int s1_pad(int w) { return (w + 31) / 32 * 32 + 4; }

// smem (floats): Ps [2][(TT + KC-1) x CHP] (P rows with the conv halo, double-buffered) |
// Dq [2][TT x QKP] (dq of the G heads and dk) | Dv [2][(TT + 1) x DL] | A [TT x QKP] (sequence-
// conv output) | U [TT x QKP] (channel-conv output, then its gradient in place) |
// Rt [TT x DL] (cos, sin of the tile's RoPE angles) | turns [2 x 32]
__host__ __device__ inline size_t s1_smem_floats(int G, int DL, int KC) {
  const size_t QKP = s1_pad((G + 1) * DL), CHP = s1_pad((G + 2) * DL);
  return 2 * static_cast<size_t>(S1_TT + KC - 1) * CHP + 2 * S1_TT * QKP +
         2 * static_cast<size_t>(S1_TT + 1) * DL + 2 * S1_TT * QKP + S1_TT * DL + 64;
}

// Pass 1, persistent: CTA (ci, g) walks the 16-token tiles u_beg .. u_end-1 of key/value group
// g, the next tile's P rows, dq / dk and dv copied in (16-byte asynchronous copies) while the
// current one is computed.  The three channel-conv products are warp mma.sync tiles on bf16
// hi / lo splits (three products each: hi*hi + hi*lo + lo*hi, about fp32 accuracy):
//   U  = A W^T per head (tokens x out channels), then Q-K-Mean's skip terms
//   dA = dU W  per head (tokens x in channels)
//   dW += dU^T A per head (out x in channels, the tile's tokens as K), accumulated in
//         registers over the CTA's tiles and added to the output once.
template <int DL>
__global__ void __launch_bounds__(S1_THREADS, 1) stencil_bwd1_kernel(const S1Params p, int cpg,
                                                                     int tiles_per_seq) {
  extern __shared__ __align__(16) float sm[];
  constexpr int TT = S1_TT, HALF = DL / 2, NTI = DL / 8, KST = DL / 16, MT = DL / 16;
  const int G = p.G, KC = p.KC, KC1 = KC - 1, S = p.S;
  const int QK = (G + 1) * DL, CH = (G + 2) * DL;
  const int QKP = s1_pad(QK), CHP = s1_pad(CH), PR = TT + KC1;
  float *Ps = sm;
  float *Dq = Ps + 2 * PR * CHP;
  float *Dv = Dq + 2 * TT * QKP;
  float *A = Dv + 2 * (TT + 1) * DL;
  float *U = A + TT * QKP;
  float *Rt = U + TT * QKP;
  float2 *turns = reinterpret_cast<float2 *>(Rt + TT * DL);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, qc = lane & 3;
  const int g = blockIdx.y, ci = blockIdx.x;
  const int units = p.B * tiles_per_seq;
  const int u_beg = static_cast<int>(static_cast<long long>(units) * ci / cpg);
  const int u_end = static_cast<int>(static_cast<long long>(units) * (ci + 1) / cpg);
  const int qcol0 = g * G * DL, kcol0 = p.NQ + g * DL, vcol0 = p.NQ + p.NKV + g * DL;
  const bool qkm = (p.flags & F_QK_MEAN) != 0, norm = (p.flags & F_QK_NORM) != 0;
  const bool rope = (p.flags & F_ROPE) != 0;
  auto head_glob = [&](int hh) { return hh < G ? g * G + hh : p.H + g; };
  if (tid < 32) turns[tid] = make_float2(p.turns_hi[tid], p.turns_lo[tid]);

  auto issue = [&](int u, int k) {                  // tile u's inputs into buffer k
    const int b = u / tiles_per_seq, t0 = (u % tiles_per_seq) * TT;
    float *ps = Ps + k * PR * CHP, *dqs = Dq + k * TT * QKP, *dvs = Dv + k * (TT + 1) * DL;
    const int C4 = CH / 4;
    for (int e = tid; e < PR * C4; e += S1_THREADS) {
      const int r = e / C4, c = (e % C4) * 4;
      const int t = t0 - KC1 + r;
      const int gc = c < G * DL ? qcol0 + c : (c < QK ? kcol0 + (c - G * DL) : vcol0 + (c - QK));
      const bool ok = t >= 0 && t < S;
      cp_async16_zfill(ps + r * CHP + c, p.P + (static_cast<size_t>(b) * S + (ok ? t : 0)) * p.NQKV + gc, ok);
    }
    constexpr int D4 = DL / 4;
    for (int e = tid; e < TT * (G + 1) * D4; e += S1_THREADS) {
      const int tt = e / ((G + 1) * D4), rem = e % ((G + 1) * D4), hh = rem / D4, i = (rem % D4) * 4;
      const int t = t0 + tt;
      const bool ok = t < S;
      const size_t tr = ok ? t : 0;
      const float *src = hh < G ? p.dq + ((static_cast<size_t>(b) * p.H + g * G + hh) * S + tr) * DL + i
                                : p.dk + ((static_cast<size_t>(b) * p.Hkv + g) * S + tr) * DL + i;
      cp_async16_zfill(dqs + tt * QKP + hh * DL + i, src, ok);
    }
    for (int e = tid; e < (TT + 1) * D4; e += S1_THREADS) {
      const int tt = e / D4, i = (e % D4) * 4;
      const int t = t0 + tt;
      const bool ok = t < S;
      cp_async16_zfill(dvs + tt * DL + i,
                       p.dv + ((static_cast<size_t>(b) * p.Hkv + g) * S + (ok ? t : 0)) * DL + i, ok);
    }
  };

  // filter-gradient blocks of this warp: (head, 16 out channels, 8 in channels)
  const int NB = (G + 1) * MT * NTI;
  const int BPW = (NB + S1_WARPS - 1) / S1_WARPS;
  float accW[S1_MAXB][4];
#pragma unroll
  for (int m = 0; m < S1_MAXB; ++m) accW[m][0] = accW[m][1] = accW[m][2] = accW[m][3] = 0.f;

  if (u_beg < u_end) issue(u_beg, 0);
  cp_async_commit();
  int k = 0;
  for (int u = u_beg; u < u_end; ++u, k ^= 1) {
    if (u + 1 < u_end) issue(u + 1, k ^ 1);
    cp_async_commit();
    cp_async_wait_one();                             // tile u's copies have landed
    __syncthreads();
    const int b = u / tiles_per_seq, t0 = (u % tiles_per_seq) * TT;
    const float *ps = Ps + k * PR * CHP, *dqs = Dq + k * TT * QKP, *dvs = Dv + k * (TT + 1) * DL;

    // 1. sequence conv of the q | k channels (tap j of token t reads token t - (KC-1) + j),
    //    and the tile's RoPE angles
    for (int c = tid; c < QK; c += S1_THREADS) {
      const int gc = c < G * DL ? qcol0 + c : kcol0 + (c - G * DL);
      float w[S1_KCMAX];
#pragma unroll
      for (int j = 0; j < S1_KCMAX; ++j) w[j] = j < KC ? __ldg(p.conv_seq + static_cast<size_t>(gc) * KC + j) : 0.f;
#pragma unroll 4
      for (int tt = 0; tt < TT; ++tt) {
        float a = 0.f;
#pragma unroll
        for (int j = 0; j < S1_KCMAX; ++j)
          if (j < KC) a = fmaf(w[j], ps[(tt + j) * CHP + c], a);
        A[tt * QKP + c] = a;
      }
    }
    if (rope)
      for (int e = tid; e < TT * HALF; e += S1_THREADS) {
        const int tt = e / HALF, i = e % HALF;
        float cs, sn;
        const float2 tr = turns[i];
        rope_cos_sin_turns(t0 + tt, tr.x, tr.y, cs, sn);
        Rt[2 * e] = cs;
        Rt[2 * e + 1] = sn;
      }
    __syncthreads();

    // 2. U = A W^T per head (+ Q-K-Mean's skip terms); a warp per (head, 8 out channels)
    for (int task = warp; task < (G + 1) * NTI; task += S1_WARPS) {
      const int hh = task / NTI, nt = task % NTI;
      const uint2 *wb = p.wsplit + static_cast<size_t>(head_glob(hh)) * DL * (DL / 2);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const float *a0p = A + gr * QKP + hh * DL, *a1p = a0p + 8 * QKP;
#pragma unroll
      for (int ks = 0; ks < KST; ++ks) {
        const int k0 = ks * 16 + 2 * qc;
        uint32_t ah[4], al[4];
        split_bf16x2(*reinterpret_cast<const float2 *>(a0p + k0), ah[0], al[0]);
        split_bf16x2(*reinterpret_cast<const float2 *>(a1p + k0), ah[1], al[1]);
        split_bf16x2(*reinterpret_cast<const float2 *>(a0p + k0 + 8), ah[2], al[2]);
        split_bf16x2(*reinterpret_cast<const float2 *>(a1p + k0 + 8), ah[3], al[3]);
        const uint2 *wr = wb + (nt * 8 + gr) * (DL / 2) + k0 / 2;
        const uint2 w0 = __ldg(wr), w1 = __ldg(wr + 4);
        const uint32_t bh[2] = {w0.x, w1.x}, bl[2] = {w0.y, w1.y};
        mma_bf16_16816(acc, ah, bh);
        mma_bf16_16816(acc, ah, bl);
        mma_bf16_16816(acc, al, bh);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tt = gr + 8 * (e >> 1), i = nt * 8 + 2 * qc + (e & 1);
        float x = acc[e];
        if (qkm) {                                   // post-conv + (pre-conv q + k) / 2
          const float *pr = ps + (tt + KC1) * CHP;
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
        U[tt * QKP + hh * DL + i] = x;
      }
    }
    __syncthreads();

    // 3. per (token, head): norm statistics, dn = RoPE^-1(dq or dk), du (over U in place); a
    //    warp per pair, lane i holding the RoPE pair (i, i + d~/2)
    for (int it = warp; it < TT * (G + 1); it += S1_WARPS) {
      const int tt = it / (G + 1), hh = it % (G + 1);
      float *uu = U + tt * QKP + hh * DL;
      const bool act = lane < HALF;
      if (t0 + tt >= S) {                            // past the sequence: no gradient
        if (act) { uu[lane] = 0.f; uu[lane + HALF] = 0.f; }
        continue;
      }
      const float *ds = dqs + tt * QKP + hh * DL;
      float u1 = 0.f, u2 = 0.f, d1 = 0.f, d2 = 0.f;
      if (act) {
        u1 = uu[lane];
        u2 = uu[lane + HALF];
        d1 = ds[lane];
        d2 = ds[lane + HALF];
        if (rope) {                                  // rotate back by -t theta_i
          const float cs = Rt[2 * (tt * HALF + lane)], sn = Rt[2 * (tt * HALF + lane) + 1];
          const float a1 = d1 * cs + d2 * sn, a2 = -d1 * sn + d2 * cs;
          d1 = a1;
          d2 = a2;
        }
      }
      float ss = u1 * u1 + u2 * u2;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv_r = norm ? rsqrtf(ss / static_cast<float>(DL) + p.eps) : 1.f;
      const float n1 = u1 * inv_r, n2 = u2 * inv_r;
      float dot = d1 * n1 + d2 * n2;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (norm) {
        const float mdn = dot / static_cast<float>(DL);
        d1 = (d1 - n1 * mdn) * inv_r;
        d2 = (d2 - n2 * mdn) * inv_r;
      }
      if (act) {
        uu[lane] = d1;
        uu[lane + HALF] = d2;
      }
    }
    __syncthreads();

    // 4. dA = dU W per head (the channel conv's transpose); a warp per (head, 8 in channels)
    for (int task = warp; task < (G + 1) * NTI; task += S1_WARPS) {
      const int hh = task / NTI, nt = task % NTI;
      const uint2 *wt = p.wsplitT + static_cast<size_t>(head_glob(hh)) * DL * (DL / 2);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const float *a0p = U + gr * QKP + hh * DL, *a1p = a0p + 8 * QKP;
#pragma unroll
      for (int ks = 0; ks < KST; ++ks) {
        const int k0 = ks * 16 + 2 * qc;
        uint32_t ah[4], al[4];
        split_bf16x2(*reinterpret_cast<const float2 *>(a0p + k0), ah[0], al[0]);
        split_bf16x2(*reinterpret_cast<const float2 *>(a1p + k0), ah[1], al[1]);
        split_bf16x2(*reinterpret_cast<const float2 *>(a0p + k0 + 8), ah[2], al[2]);
        split_bf16x2(*reinterpret_cast<const float2 *>(a1p + k0 + 8), ah[3], al[3]);
        const uint2 *wr = wt + (nt * 8 + gr) * (DL / 2) + k0 / 2;
        const uint2 w0 = __ldg(wr), w1 = __ldg(wr + 4);
        const uint32_t bh[2] = {w0.x, w1.x}, bl[2] = {w0.y, w1.y};
        mma_bf16_16816(acc, ah, bh);
        mma_bf16_16816(acc, ah, bl);
        mma_bf16_16816(acc, al, bh);
      }
      const int c = nt * 8 + 2 * qc;
      const int gc = hh < G ? qcol0 + hh * DL + c : kcol0 + c;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int t = t0 + gr + 8 * h2;
        if (t < S)
          *reinterpret_cast<float2 *>(p.dA + (static_cast<size_t>(b) * S + t) * (p.NQ + p.NKV) + gc) =
              make_float2(acc[2 * h2], acc[2 * h2 + 1]);
      }
    }
    // Q-K-Mean's skip gradients of the q | k projections, and the value gradients (the
    // value-shift undone: a shifted channel of token t received dv of token t + 1)
    for (int e = tid; e < TT * CH; e += S1_THREADS) {
      const int tt = e / CH, c = e % CH;
      const int t = t0 + tt;
      if (t >= S) continue;
      const size_t row = static_cast<size_t>(b) * S + t;
      if (c < QK) {
        float skip = 0.f;
        if (qkm) {
          const int i = c % DL;
          const float duk = U[tt * QKP + G * DL + i];
          if (c < G * DL) {
            skip = 0.5f * U[tt * QKP + c] + duk / (2.0f * static_cast<float>(G));
          } else {
            float sq = 0.f;
            for (int h2 = 0; h2 < G; ++h2) sq += U[tt * QKP + h2 * DL + i];
            skip = 0.5f * sq + 0.5f * duk;
          }
        }
        const int gc = c < G * DL ? qcol0 + c : kcol0 + (c - G * DL);
        p.dPpart[row * p.NQKV + gc] = skip;
      } else {
        const int i = c - QK;
        const bool shifted = (p.flags & F_VALUE_SHIFT) && g * DL + i >= p.VS0;
        p.dPpart[row * p.NQKV + vcol0 + i] = dvs[(tt + (shifted ? 1 : 0)) * DL + i];
      }
    }
    // 5. dW[h][i][c] += sum over the tile's tokens of dU[t][h][i] A[t][h][c]
#pragma unroll
    for (int m = 0; m < S1_MAXB; ++m) {
      const int blk = warp * BPW + m;
      if (m < BPW && blk < NB) {
        const int hh = blk / (MT * NTI), rem = blk % (MT * NTI);
        const int cu = hh * DL + (rem / NTI) * 16 + gr;   // dU column (out channel i)
        const int ca = hh * DL + (rem % NTI) * 8 + gr;    // A column (in channel c)
        uint32_t ah[4], al[4], bh[2], bl[2];
        split_bf16x2(make_float2(U[(2 * qc) * QKP + cu], U[(2 * qc + 1) * QKP + cu]), ah[0], al[0]);
        split_bf16x2(make_float2(U[(2 * qc) * QKP + cu + 8], U[(2 * qc + 1) * QKP + cu + 8]), ah[1], al[1]);
        split_bf16x2(make_float2(U[(2 * qc + 8) * QKP + cu], U[(2 * qc + 9) * QKP + cu]), ah[2], al[2]);
        split_bf16x2(make_float2(U[(2 * qc + 8) * QKP + cu + 8], U[(2 * qc + 9) * QKP + cu + 8]), ah[3], al[3]);
        split_bf16x2(make_float2(A[(2 * qc) * QKP + ca], A[(2 * qc + 1) * QKP + ca]), bh[0], bl[0]);
        split_bf16x2(make_float2(A[(2 * qc + 8) * QKP + ca], A[(2 * qc + 9) * QKP + ca]), bh[1], bl[1]);
        mma_bf16_16816(accW[m], ah, bh);
        mma_bf16_16816(accW[m], ah, bl);
        mma_bf16_16816(accW[m], al, bh);
      }
    }
    __syncthreads();                                 // A, U and this buffer reused next
  }
  cp_async_wait_none();
#pragma unroll
  for (int m = 0; m < S1_MAXB; ++m) {
    const int blk = warp * BPW + m;
    if (m < BPW && blk < NB && u_end > u_beg) {
      const int hh = blk / (MT * NTI), rem = blk % (MT * NTI);
      const int i = (rem / NTI) * 16 + gr, c = (rem % NTI) * 8 + 2 * qc;
      float *dst = p.dconv_chan + static_cast<size_t>(head_glob(hh)) * DL * DL;
      atomicAdd(dst + i * DL + c, accW[m][0]);
      atomicAdd(dst + i * DL + c + 1, accW[m][1]);
      atomicAdd(dst + (i + 8) * DL + c, accW[m][2]);
      atomicAdd(dst + (i + 8) * DL + c + 1, accW[m][3]);
    }
  }
}

// The channel filters transposed and split: out[(head * DL + c) * DL/2 + i/2] = the bf16 hi / lo
// pairs of (W[head][i][c], W[head][i+1][c]).
__global__ void split_conv_chan_t_kernel(const float *__restrict__ w, uint2 *__restrict__ out,
                                         int heads, int DL) {
  const int half = DL / 2;
  const size_t n = static_cast<size_t>(heads) * DL * half;
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int ip = static_cast<int>(e % half);
    const int c = static_cast<int>((e / half) % DL);
    const size_t h = e / (static_cast<size_t>(half) * DL);
    const float *wh = w + h * DL * DL;
    uint2 r;
    split_bf16x2(make_float2(wh[(2 * ip) * DL + c], wh[(2 * ip + 1) * DL + c]), r.x, r.y);
    out[e] = r;
  }
}

// Pass 2: a CTA per (32 columns of dP, 256 rows), a warp per 32-row slice of them (so every
// load and store of a warp covers 32 consecutive columns of one row); the sequence conv's
// transpose and its filter gradient from sliding windows of dA (rows t .. t+KC-1) and P (rows
// t-KC+1 .. t) held in registers, then dP in bfloat16 (the value columns converted as they
// are).  The filter gradient is summed over the CTA's warps in shared memory and added once
// per CTA.
constexpr int S2_COLS = 32;
constexpr int S2_SUB = 32;                           // rows per warp
constexpr int S2_WARPS = 8;
constexpr int S2_KCMAX = 8;

__global__ void __launch_bounds__(256) stencil_bwd2_kernel(
    const float *__restrict__ P, const float *__restrict__ dA, const float *__restrict__ dPpart,
    const float *__restrict__ conv_seq, __nv_bfloat16 *__restrict__ dP, float *__restrict__ dconv_seq,
    int B, int S, int NQ, int NKV, int NQKV, int KC) {
  __shared__ float red[S2_WARPS][S2_KCMAX][S2_COLS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = blockIdx.x * S2_COLS + lane;             // column of dP (all NQKV)
  const long long M = static_cast<long long>(B) * S;
  const long long r_beg = (static_cast<long long>(blockIdx.y) * S2_WARPS + warp) * S2_SUB;
  const long long r_end = r_beg + S2_SUB < M ? r_beg + S2_SUB : M;
  const int W = NQ + NKV;
  const bool live = c < NQKV;
  const bool qk = live && c < W;
  float w[S2_KCMAX], dw[S2_KCMAX];
#pragma unroll
  for (int j = 0; j < S2_KCMAX; ++j) {
    w[j] = (qk && j < KC) ? conv_seq[static_cast<size_t>(c) * KC + j] : 0.f;
    dw[j] = 0.f;
  }
  if (qk) {
    // windows: da[l] = dA[row + l] (l < KC, zero past the sequence), pp[l] = P[row - l]
    // (zero before the sequence start), for the current row
    float da[S2_KCMAX], pp[S2_KCMAX];
    if (r_beg < r_end) {
      const int t0 = static_cast<int>(r_beg % S);
#pragma unroll
      for (int l = 0; l < S2_KCMAX; ++l) {
        da[l] = (l < KC && t0 + l < S) ? dA[(r_beg + l) * W + c] : 0.f;
        pp[l] = (l < KC && t0 - l >= 0) ? P[(r_beg - l) * NQKV + c] : 0.f;
      }
    }
    for (long long row = r_beg; row < r_end; ++row) {
      const int t = static_cast<int>(row % S);
      float v = dPpart[row * NQKV + c];
#pragma unroll
      for (int j = 0; j < S2_KCMAX; ++j) {
        if (j < KC) {
          const int lag = KC - 1 - j;                    // output t + lag read input t by tap j
          v = fmaf(w[j], da[lag], v);                    // da[lag] is zero past the sequence
          dw[j] = fmaf(da[0], pp[lag], dw[j]);           // pp[lag] is zero before its start
        }
      }
      dP[row * NQKV + c] = __float2bfloat16_rn(v);
      // slide both windows by one row
#pragma unroll
      for (int l = S2_KCMAX - 1; l > 0; --l) pp[l] = pp[l - 1];
#pragma unroll
      for (int l = 0; l + 1 < S2_KCMAX; ++l) da[l] = da[l + 1];
      const long long nrow = row + 1;
      if (nrow < r_end) {
        const int nt = t + 1 == S ? 0 : t + 1;           // a new sequence starts at nt == 0
        pp[0] = P[nrow * NQKV + c];
        if (nt == 0) {
#pragma unroll
          for (int l = 1; l < S2_KCMAX; ++l) pp[l] = 0.f;
#pragma unroll
          for (int l = 0; l < S2_KCMAX; ++l)
            da[l] = (l < KC && l < S) ? dA[(nrow + l) * W + c] : 0.f;
        } else {
          const int l = KC - 1;                          // the window's new last row
          if (l < S2_KCMAX) da[l] = nt + l < S ? dA[(nrow + l) * W + c] : 0.f;
        }
      }
    }
  } else if (live) {
    for (long long row = r_beg; row < r_end; ++row)
      dP[row * NQKV + c] = __float2bfloat16_rn(dPpart[row * NQKV + c]);
  }
#pragma unroll
  for (int j = 0; j < S2_KCMAX; ++j) red[warp][j][lane] = dw[j];
  __syncthreads();
  if (warp == 0 && qk) {
    for (int j = 0; j < KC; ++j) {
      float sum = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < S2_WARPS; ++w2) sum += red[w2][j][lane];
      atomicAdd(dconv_seq + static_cast<size_t>(c) * KC + j, sum);
    }
  }
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
  return d.bf16 && !(d.flags & F_NO_CONV) && (d.DL == 16 || d.DL == 32 || d.DL == 64) &&
         d.KC <= S1_KCMAX && (d.G + 1) * (d.DL / 16) * (d.DL / 8) <= S1_WARPS * S1_MAXB &&
         s1_smem_floats(d.G, d.DL, d.KC) * 4 <= 200 * 1024;
}

template <int DL>
cudaError_t launch_bwd1(const Dims &d, const S1Params &p, int cpg, int tiles, cudaStream_t st) {
  const size_t smem = s1_smem_floats(d.G, DL, d.KC) * 4;
  cudaError_t e;
  if ((e = ensure_dyn_smem<stencil_bwd1_kernel<DL>>(smem)) != cudaSuccess) return e;
  stencil_bwd1_kernel<DL><<<dim3(cpg, d.Hkv), S1_THREADS, smem, st>>>(p, cpg, tiles);
  return cudaGetLastError();
}

cudaError_t stencil_backward(const Dims &d, const StencilBwdArgs &a, cudaStream_t st) {
  if (d.B == 0 || d.S == 0) return cudaSuccess;
  if (!stencil_backward_supported(d)) return cudaErrorInvalidValue;
  cudaError_t e;
  {
    const int heads = d.H + d.Hkv;
    const size_t n = static_cast<size_t>(heads) * d.DL * (d.DL / 2);
    const int blocks = static_cast<int>((n + 255) / 256);
    split_conv_chan_t_kernel<<<blocks, 256, 0, st>>>(a.conv_chan, static_cast<uint2 *>(a.conv_chan_split_t),
                                                     heads, d.DL);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  S1Params p;
  p.P = a.P;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.conv_seq = a.conv_seq;
  p.wsplit = static_cast<const uint2 *>(a.conv_chan_split);
  p.wsplitT = static_cast<const uint2 *>(a.conv_chan_split_t);
  p.dA = a.dA;
  p.dPpart = a.dPpart;
  p.dconv_chan = a.dconv_chan;
  p.B = d.B; p.S = d.S; p.H = d.H; p.Hkv = d.Hkv; p.G = d.G;
  p.NQ = d.NQ; p.NKV = d.NKV; p.NQKV = d.NQKV; p.KC = d.KC; p.VS0 = d.VS0;
  p.flags = d.flags;
  p.eps = d.eps;
  rope_turns_host(d.DL, d.rope_base, p.turns_hi, p.turns_lo, 32);
  const int tiles = (d.S + S1_TT - 1) / S1_TT;
  const int units = d.B * tiles;
  int cpg = num_sms() / d.Hkv;
  if (cpg < 1) cpg = 1;
  if (cpg > units) cpg = units;
  e = d.DL == 16 ? launch_bwd1<16>(d, p, cpg, tiles, st)
    : d.DL == 32 ? launch_bwd1<32>(d, p, cpg, tiles, st) : launch_bwd1<64>(d, p, cpg, tiles, st);
  if (e != cudaSuccess) return e;
  const long long M = static_cast<long long>(d.B) * d.S;
  const long long rows_per_cta = static_cast<long long>(S2_WARPS) * S2_SUB;
  const dim3 g2((d.NQKV + S2_COLS - 1) / S2_COLS, static_cast<unsigned>((M + rows_per_cta - 1) / rows_per_cta));
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
