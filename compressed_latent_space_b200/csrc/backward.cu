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
constexpr int S1_THREADS = 512;    // sixteen warps: more of each phase in flight (8 warps: +25 %)
constexpr int S1_WARPS = S1_THREADS / 32;
constexpr int S1_MAXB = 10;        // filter-gradient 16 x 8 blocks per warp (160 per CTA)
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

// Row strides of the float32 shared-memory tiles: a multiple of 32 floats plus 4, so that
// fragment-pattern reads (eight rows x four column pairs) fall on distinct banks.
__host__ __device__ constexpr int s1_pad(int w) { return (w + 31) / 32 * 32 + 4; }
// Row stride (bf16 elements) of the bf16 planes: a multiple of 128 bytes plus 16, so that the
// eight 16-byte rows of an ldmatrix phase hit distinct bank groups.
__host__ __device__ constexpr int s1_plane_ld(int w) { return ((w * 2 + 127) / 128 * 128 + 16) / 2; }

// smem: Ps [2][(TT + KC-1) x CHP] f32 (P rows with the conv halo, double-buffered) | Dq [2][TT x
// QKP] f32 (dq of the G heads and dk) | Dv [2][(TT + 1) x DL] f32 | U [TT x QKP] f32 (channel-
// conv output, then its gradient in place) | Rt [TT x DL] f32 (cos, sin of the tile's RoPE
// angles) | turns [64] f32 | planes [4][TT x PLD] bf16: the sequence-conv output A and the
// gradient dU, each as a bf16 leading term and remainder (about 16 significand bits in all)
__host__ __device__ inline size_t s1_smem_bytes(int G, int DL, int KC) {
  const size_t QKP = s1_pad((G + 1) * DL), CHP = s1_pad((G + 2) * DL);
  const size_t floats = 2 * static_cast<size_t>(S1_TT + KC - 1) * CHP + 2 * S1_TT * QKP +
                        2 * static_cast<size_t>(S1_TT + 1) * DL + S1_TT * QKP + S1_TT * DL + 64;
  return floats * 4 + 4 * static_cast<size_t>(S1_TT) * s1_plane_ld((G + 1) * DL) * 2;
}

__device__ __forceinline__ void split_store(__nv_bfloat16 *hi, __nv_bfloat16 *lo, float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  *hi = h;
  *lo = __float2bfloat16_rn(v - __bfloat162float(h));
}

// Pass 1, persistent: CTA (ci, g) walks the 16-token tiles u_beg .. u_end-1 of key/value group
// g, the next tile's P rows, dq / dk and dv copied in (16-byte asynchronous copies) while the
// current one is computed.  The three channel-conv products are warp mma.sync tiles on bf16
// hi / lo splits (three products each: hi*hi + hi*lo + lo*hi, about fp32 accuracy), their
// activation fragments read from the split planes by ldmatrix:
//   U  = A W^T per head (tokens x out channels), then Q-K-Mean's skip terms
//   dA = dU W  per head (tokens x in channels)
//   dW += dU^T A per head (out x in channels, the tile's tokens as K, both operands through
//         ldmatrix.trans), accumulated in registers over the CTA's tiles, added once.
template <int DL>
__global__ void __launch_bounds__(S1_THREADS, 1) stencil_bwd1_kernel(const S1Params p, int cpg,
                                                                     int tiles_per_seq) {
  extern __shared__ __align__(16) float sm[];
  constexpr int TT = S1_TT, HALF = DL / 2, NTI = DL / 8, KST = DL / 16, MT = DL / 16;
  constexpr int D4 = DL / 4;
  const int G = p.G, KC = p.KC, KC1 = KC - 1, S = p.S;
  const int QK = (G + 1) * DL, CH = (G + 2) * DL;
  const int QKP = s1_pad(QK), CHP = s1_pad(CH), PR = TT + KC1, PLD = s1_plane_ld(QK);
  float *Ps = sm;
  float *Dq = Ps + 2 * PR * CHP;
  float *Dv = Dq + 2 * TT * QKP;
  float *U = Dv + 2 * (TT + 1) * DL;
  float *Rt = U + TT * QKP;
  float2 *turns = reinterpret_cast<float2 *>(Rt + TT * DL);
  __nv_bfloat16 *Ahi = reinterpret_cast<__nv_bfloat16 *>(Rt + TT * DL + 64);
  __nv_bfloat16 *Alo = Ahi + TT * PLD, *Dhi = Alo + TT * PLD, *Dlo = Dhi + TT * PLD;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, qc = lane & 3;
  const int lr = lane & 7, lm = lane >> 3;          // ldmatrix: row of matrix lm
  const int g = blockIdx.y, ci = blockIdx.x;
  const int units = p.B * tiles_per_seq;
  const int u_beg = static_cast<int>(static_cast<long long>(units) * ci / cpg);
  const int u_end = static_cast<int>(static_cast<long long>(units) * (ci + 1) / cpg);
  const int qcol0 = g * G * DL, kcol0 = p.NQ + g * DL, vcol0 = p.NQ + p.NKV + g * DL;
  const bool qkm = (p.flags & F_QK_MEAN) != 0, norm = (p.flags & F_QK_NORM) != 0;
  const bool rope = (p.flags & F_ROPE) != 0;
  auto head_glob = [&](int hh) { return hh < G ? g * G + hh : p.H + g; };
  if (tid < 32) turns[tid] = make_float2(p.turns_hi[tid], p.turns_lo[tid]);

  // copy assignments fixed per thread: P rows by C4 16-byte pieces, dq / dk rows by D4
  const int C4 = CH / 4;                            // <= 256 (host check)
  const int p_rows_pass = S1_THREADS / C4, p_r0 = tid / C4, p_c = (tid % C4) * 4;
  const int p_gc = p_c < G * DL ? qcol0 + p_c : (p_c < QK ? kcol0 + (p_c - G * DL) : vcol0 + (p_c - QK));
  constexpr int q_rows_pass = S1_THREADS / D4;
  const int q_r0 = tid / D4, q_i = (tid % D4) * 4;
  auto issue = [&](int u, int k) {                  // tile u's inputs into buffer k
    const int b = u / tiles_per_seq, t0 = (u % tiles_per_seq) * TT;
    float *ps = Ps + k * PR * CHP, *dqs = Dq + k * TT * QKP, *dvs = Dv + k * (TT + 1) * DL;
    if (p_r0 < p_rows_pass)
      for (int r = p_r0; r < PR; r += p_rows_pass) {
        const int t = t0 - KC1 + r;
        const bool ok = t >= 0 && t < S;
        cp_async16_zfill(ps + r * CHP + p_c, p.P + (static_cast<size_t>(b) * S + (ok ? t : 0)) * p.NQKV + p_gc, ok);
      }
    for (int r = q_r0; r < TT * (G + 1); r += q_rows_pass) {   // (token, head) rows
      const int tt = r / (G + 1), hh = r % (G + 1);
      const int t = t0 + tt;
      const bool ok = t < S;
      const size_t tr = ok ? t : 0;
      const float *src = hh < G ? p.dq + ((static_cast<size_t>(b) * p.H + g * G + hh) * S + tr) * DL + q_i
                                : p.dk + ((static_cast<size_t>(b) * p.Hkv + g) * S + tr) * DL + q_i;
      cp_async16_zfill(dqs + tt * QKP + hh * DL + q_i, src, ok);
    }
    for (int r = q_r0; r < TT + 1; r += q_rows_pass) {
      const int t = t0 + r;
      const bool ok = t < S;
      cp_async16_zfill(dvs + r * DL + q_i,
                       p.dv + ((static_cast<size_t>(b) * p.Hkv + g) * S + (ok ? t : 0)) * DL + q_i, ok);
    }
  };

  // filter-gradient blocks of this warp: (head, 16 out channels, 8 in channels)
  const int NB = (G + 1) * MT * NTI;
  const int BPW = (NB + S1_WARPS - 1) / S1_WARPS;
  float accW[S1_MAXB][4];
#pragma unroll
  for (int m = 0; m < S1_MAXB; ++m) accW[m][0] = accW[m][1] = accW[m][2] = accW[m][3] = 0.f;
  const uint32_t ahi_s = smem_u32(Ahi), alo_s = smem_u32(Alo), dhi_s = smem_u32(Dhi), dlo_s = smem_u32(Dlo);

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
    //    stored as bf16 hi / lo planes, and the tile's RoPE angles
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
        split_store(Ahi + tt * PLD + c, Alo + tt * PLD + c, a);
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

    // 2. U = A W^T per head (+ Q-K-Mean's skip terms); a warp per (head, 8 out channels).
    //    A fragments: ldmatrix rows = tokens (lm & 1) * 8 + lr, columns k0 + (lm >> 1) * 8
    const uint32_t frag_off = static_cast<uint32_t>((((lm & 1) * 8 + lr) * PLD + (lm >> 1) * 8) * 2);
    for (int task = warp; task < (G + 1) * NTI; task += S1_WARPS) {
      const int hh = task / NTI, nt = task % NTI;
      const uint2 *wb = p.wsplit + static_cast<size_t>(head_glob(hh)) * DL * (DL / 2);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KST; ++ks) {
        const uint32_t off = frag_off + (hh * DL + ks * 16) * 2;
        uint32_t ah[4], al[4];
        ldsm_x4(ahi_s + off, ah[0], ah[1], ah[2], ah[3]);
        ldsm_x4(alo_s + off, al[0], al[1], al[2], al[3]);
        const uint2 *wr = wb + (nt * 8 + gr) * (DL / 2) + (ks * 16 + 2 * qc) / 2;
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

    // 3. per (token, head): norm statistics, dn = RoPE^-1(dq or dk), du (over U in place, and
    //    into the dU planes); a warp per pair, lane i holding the RoPE pair (i, i + d~/2)
    for (int it = warp; it < TT * (G + 1); it += S1_WARPS) {
      const int tt = it / (G + 1), hh = it % (G + 1);
      float *uu = U + tt * QKP + hh * DL;
      const bool act = lane < HALF;
      const int pc = tt * PLD + hh * DL + lane;
      if (t0 + tt >= S) {                            // past the sequence: no gradient
        if (act) {
          uu[lane] = 0.f;
          uu[lane + HALF] = 0.f;
          split_store(Dhi + pc, Dlo + pc, 0.f);
          split_store(Dhi + pc + HALF, Dlo + pc + HALF, 0.f);
        }
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
        split_store(Dhi + pc, Dlo + pc, d1);
        split_store(Dhi + pc + HALF, Dlo + pc + HALF, d2);
      }
    }
    __syncthreads();

    // 4. dA = dU W per head (the channel conv's transpose); a warp per (head, 8 in channels)
    for (int task = warp; task < (G + 1) * NTI; task += S1_WARPS) {
      const int hh = task / NTI, nt = task % NTI;
      const uint2 *wt = p.wsplitT + static_cast<size_t>(head_glob(hh)) * DL * (DL / 2);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KST; ++ks) {
        const uint32_t off = frag_off + (hh * DL + ks * 16) * 2;
        uint32_t ah[4], al[4];
        ldsm_x4(dhi_s + off, ah[0], ah[1], ah[2], ah[3]);
        ldsm_x4(dlo_s + off, al[0], al[1], al[2], al[3]);
        const uint2 *wr = wt + (nt * 8 + gr) * (DL / 2) + (ks * 16 + 2 * qc) / 2;
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
    for (int c = tid; c < CH; c += S1_THREADS) {
      const bool is_qk = c < QK;
      const int i = is_qk ? c % DL : c - QK;
      const int gc = c < G * DL ? qcol0 + c : (is_qk ? kcol0 + (c - G * DL) : vcol0 + i);
      const int vsh = (!is_qk && (p.flags & F_VALUE_SHIFT) && g * DL + i >= p.VS0) ? 1 : 0;
      for (int tt = 0; tt < TT; ++tt) {
        const int t = t0 + tt;
        if (t >= S) break;
        float val;
        if (is_qk) {
          val = 0.f;
          if (qkm) {
            const float *ur = U + tt * QKP;
            const float duk = ur[G * DL + i];
            if (c < G * DL) {
              val = 0.5f * ur[c] + duk / (2.0f * static_cast<float>(G));
            } else {
              float sq = 0.f;
              for (int h2 = 0; h2 < G; ++h2) sq += ur[h2 * DL + i];
              val = 0.5f * sq + 0.5f * duk;
            }
          }
        } else {
          val = dvs[(tt + vsh) * DL + i];
        }
        p.dPpart[(static_cast<size_t>(b) * S + t) * p.NQKV + gc] = val;
      }
    }
    // 5. dW[h][i][c] += sum over the tile's tokens of dU[t][h][i] A[t][h][c].  A operand dU^T
    //    (16 out channels x 16 tokens): ldmatrix.trans of the dU plane, matrix lm at tokens
    //    (lm >> 1) * 8 + lr, channels (lm & 1) * 8; B operand (16 tokens x 8 in channels):
    //    ldmatrix.trans of the A plane, matrix (lm & 1) at tokens (lm & 1) * 8 + lr
    const uint32_t ta_off = static_cast<uint32_t>((((lm >> 1) * 8 + lr) * PLD + (lm & 1) * 8) * 2);
    const uint32_t tb_off = static_cast<uint32_t>((((lm & 1) * 8 + lr) * PLD) * 2);
#pragma unroll
    for (int m = 0; m < S1_MAXB; ++m) {
      const int blk = warp * BPW + m;
      if (m < BPW && blk < NB) {
        const int hh = blk / (MT * NTI), rem = blk % (MT * NTI);
        const int cu = hh * DL + (rem / NTI) * 16;   // first out channel of the block
        const int ca = hh * DL + (rem % NTI) * 8;    // first in channel
        uint32_t ah[4], al[4], bh[2], bl[2];
        ldsm_x4_t(dhi_s + ta_off + cu * 2, ah[0], ah[1], ah[2], ah[3]);
        ldsm_x4_t(dlo_s + ta_off + cu * 2, al[0], al[1], al[2], al[3]);
        ldsm_x2_t(ahi_s + tb_off + ca * 2, bh[0], bh[1]);
        ldsm_x2_t(alo_s + tb_off + ca * 2, bl[0], bl[1]);
        mma_bf16_16816(accW[m], ah, bh);
        mma_bf16_16816(accW[m], ah, bl);
        mma_bf16_16816(accW[m], al, bh);
      }
    }
    __syncthreads();                                 // planes, U and this buffer reused next
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
// load and store of a warp covers 32 consecutive columns of one row), walked in chunks of 8
// rows whose loads (dPpart, the P rows back to KC-1 before the chunk, the dA rows up to KC-1
// after it) are all issued before any is used; the sequence conv's transpose and its filter
// gradient, then dP in bfloat16 (the value columns converted as they are).  The filter
// gradient is summed over the CTA's warps in shared memory and added once per CTA.
constexpr int S2_COLS = 32;
constexpr int S2_SUB = 32;                           // rows per warp
constexpr int S2_WARPS = 8;
constexpr int S2_KCMAX = 8;
constexpr int S2_CH = 8;                             // rows per chunk

__global__ void __launch_bounds__(256) stencil_bwd2_kernel(
    const float *__restrict__ P, const float *__restrict__ dA, const float *__restrict__ dPpart,
    const float *__restrict__ conv_seq, __nv_bfloat16 *__restrict__ dP, float *__restrict__ dconv_seq,
    int B, int S, int NQ, int NKV, int NQKV, int KC) {
  __shared__ float red[S2_WARPS][S2_KCMAX][S2_COLS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = blockIdx.x * S2_COLS + lane;             // column of dP (all NQKV)
  const long long M = static_cast<long long>(B) * S;
  const long long r_beg = (static_cast<long long>(blockIdx.y) * S2_WARPS + warp) * S2_SUB;
  const int W = NQ + NKV;
  const bool live = c < NQKV;
  const bool qk = live && c < W;
  const int KC1 = KC - 1;
  // per lag (tap j = KC-1 - lag): wl[lag] = w[c][j], dwl[lag] accumulates the gradient of w[c][j]
  float wl[S2_KCMAX], dwl[S2_KCMAX];
#pragma unroll
  for (int l = 0; l < S2_KCMAX; ++l) {
    wl[l] = (qk && l < KC) ? conv_seq[static_cast<size_t>(c) * KC + (KC1 - l)] : 0.f;
    dwl[l] = 0.f;
  }
  constexpr int NW = S2_CH + S2_KCMAX - 1;
  for (int ch = 0; ch < S2_SUB / S2_CH; ++ch) {
    const long long r0 = r_beg + ch * S2_CH;
    if (r0 >= M || !live) break;
    // da[m] = dA[r0 + m], pq[m] = P[r0 + m - (KCMAX-1)] (zero outside [0, M) and outside the
    // halo this chunk needs); the sequence boundaries are applied per use below
    float da[NW], pq[NW], dpp[S2_CH];
#pragma unroll
    for (int e = 0; e < S2_CH; ++e) dpp[e] = r0 + e < M ? dPpart[(r0 + e) * NQKV + c] : 0.f;
    if (qk) {
#pragma unroll
      for (int m = 0; m < NW; ++m) {
        const long long rd = r0 + m, rp = r0 + m - (S2_KCMAX - 1);
        da[m] = (m < S2_CH + KC1 && rd < M) ? dA[rd * W + c] : 0.f;
        pq[m] = (m >= S2_KCMAX - KC && rp >= 0 && rp < M) ? P[rp * NQKV + c] : 0.f;
      }
    }
#pragma unroll
    for (int e = 0; e < S2_CH; ++e) {
      const long long row = r0 + e;
      if (row >= M) break;
      float v = dpp[e];
      if (qk) {
        const int t = static_cast<int>(row % S);
#pragma unroll
        for (int l = 0; l < S2_KCMAX; ++l) {
          if (l < KC) {                                  // output t + l read input t by tap KC-1-l
            if (t + l < S) v = fmaf(wl[l], da[e + l], v);
            if (t - l >= 0) dwl[l] = fmaf(da[e], pq[e + S2_KCMAX - 1 - l], dwl[l]);
          }
        }
      }
      dP[row * NQKV + c] = __float2bfloat16_rn(v);
    }
  }
#pragma unroll
  for (int l = 0; l < S2_KCMAX; ++l) red[warp][l][lane] = dwl[l];
  __syncthreads();
  if (warp == 0 && qk) {
    for (int j = 0; j < KC; ++j) {
      float sum = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < S2_WARPS; ++w2) sum += red[w2][KC1 - j][lane];
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
         (d.G + 2) * d.DL / 4 <= S1_THREADS && s1_smem_bytes(d.G, d.DL, d.KC) <= 200 * 1024;
}

template <int DL>
cudaError_t launch_bwd1(const Dims &d, const S1Params &p, int cpg, int tiles, cudaStream_t st) {
  const size_t smem = s1_smem_bytes(d.G, DL, d.KC);
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
