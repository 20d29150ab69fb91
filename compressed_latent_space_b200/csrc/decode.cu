// Single-token decode step over the compressed cache (gist.science explainer, 1. Problem
// Statement: during generation the cache is streamed once per token; 2. Methodology:
// the cache holds latent keys/values only, Hkv*d~ wide each).
//
// For each sequence b with L = lengths[b] cached tokens, one new token x[b]:
//   D1  p = x W_qkv^T                                   (split-K partial sums, fp32)
//   D2  latent stencil of the new row: the causal conv reads the stored KC-1 pre-conv rows,
//       the value-shift reads the stored upper-half value row; q-k-mean, RMS norm, RoPE at
//       position L; k, v appended at position L; conv / value-shift state advanced
//   D3  attention of the G query heads of each group over keys 0..L, its keys split across
//       CTAs only when the (sequence, group) pairs are fewer than the SMs
//   D3b merge of the splits (log-sum-exp) into o [B, NQ], when there are splits
//   D4  y = o W_o^T, then lengths[b] += 1
// A sequence with L >= max_seq is left untouched (y row zero) and the cache status word is
// set to a "full" code.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int CHUNK = 1024;       // keys per split-KV block

// ------------------------------------------------------------------ D1 / D4 on staged tiles
// C[M, N] = A[M, K] B[N, K]^T (+ A2[M, K] B^T) for M <= 64 per CTA row block, bfloat16
// operands, fp32 accumulation.  Grid (ceil(N / NC), ksplit, ceil(M / 64)): a CTA owns NC
// columns and one K slice, which it walks in 64-wide chunks staged in shared memory by 16-byte
// cp.async through an S-deep ring (S - 1 chunks in flight while one is computed; rows padded
// by 16 bytes so the ldmatrix reads are conflict-free).  Warp w computes rows 16w..16w+15 x
// the NC columns with mma.sync.  Each staged A row serves NC columns, so A crosses from L2
// N / NC times in all.  TWO_A adds a second A operand (the low bf16 halves of an fp32
// A split hi + lo).  OUT_F32: fp32 partial sums to C + ks*M*N; else bf16.  `lengths`
// (optional): block (0, 0, 0) advances lengths[m] for m < M where it is below max_seq (the
// last kernel of a decode step).
constexpr int SK_KC = 64;           // K chunk
constexpr int SK_LD = SK_KC + 8;    // padded row, in elements

template <bool TWO_A, int NC>
__host__ __device__ constexpr int skinny_stage_elems() {
  return ((TWO_A ? 2 : 1) * 64 + NC) * SK_LD;
}

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <bool OUT_F32, bool TWO_A, int S, int NC>
__global__ void __launch_bounds__(128) skinny_mma_kernel(
    const __nv_bfloat16 *__restrict__ A, const __nv_bfloat16 *__restrict__ A2,
    const __nv_bfloat16 *__restrict__ B, void *__restrict__ C, int M, int N, int K,
    int k_per_split, int *lengths, int max_seq) {
  static_assert(NC % 16 == 0, "16 columns per B load");
  constexpr int STAGE = skinny_stage_elems<TWO_A, NC>();
  extern __shared__ __align__(16) __nv_bfloat16 sk_smem[];     // [S][A (A2) B]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * NC, ks = blockIdx.y, m0 = blockIdx.z * 64;
  const int kbeg = ks * k_per_split, kend = min(K, kbeg + k_per_split);
  pdl_launch_dependents();
  {
    // the weight slab does not depend on the previous kernel: pull it towards L2 meanwhile
    const int lines = kend > kbeg ? ((kend - kbeg) * 2 + 127) / 128 : 0;
    for (int i = tid; i < NC * lines; i += 128) {
      const int r = i / lines, c = i % lines;
      if (n0 + r < N) prefetch_l2(B + static_cast<size_t>(n0 + r) * K + kbeg + c * 64);
    }
  }
  pdl_wait();
  if (lengths && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    for (int m = tid; m < M; m += 128)
      if (lengths[m] < max_seq) lengths[m] += 1;
  const int nchunks = kend > kbeg ? (kend - kbeg + SK_KC - 1) / SK_KC : 0;
  auto issue = [&](int c) {                           // an empty group past the last chunk
    if (c < nchunks) {
      const int k0 = kbeg + c * SK_KC;
      __nv_bfloat16 *st = sk_smem + (c % S) * STAGE;
      for (int i = tid; i < 64 * (SK_KC / 8); i += 128) {     // A (and A2): 64 x SK_KC
        const int r = i / (SK_KC / 8), j = i % (SK_KC / 8);
        const int k = k0 + j * 8;
        const bool ok = m0 + r < M && k < kend;
        const size_t off = ok ? static_cast<size_t>(m0 + r) * K + k : 0;
        cp_async16_zfill(st + r * SK_LD + j * 8, A + off, ok);
        if constexpr (TWO_A) cp_async16_zfill(st + (64 + r) * SK_LD + j * 8, A2 + off, ok);
      }
      __nv_bfloat16 *bs = st + (TWO_A ? 128 : 64) * SK_LD;
      for (int i = tid; i < NC * (SK_KC / 8); i += 128) {     // B: NC x SK_KC
        const int r = i / (SK_KC / 8), j = i % (SK_KC / 8);
        const int k = k0 + j * 8;
        const bool ok = n0 + r < N && k < kend;
        cp_async16_zfill(bs + r * SK_LD + j * 8,
                         B + (ok ? static_cast<size_t>(n0 + r) * K + k : 0), ok);
      }
    }
    cp_async_commit();
  };
  float acc[NC / 8][4];
#pragma unroll
  for (int t = 0; t < NC / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
  for (int c = 0; c < S - 1; ++c) issue(c);
  for (int c = 0; c < nchunks; ++c) {
    issue(c + S - 1);
    cp_async_wait_group<S - 1>();                      // chunk c has landed
    __syncthreads();
    const __nv_bfloat16 *st = sk_smem + (c % S) * STAGE;
    const uint32_t a_base = smem_u32(st + (warp * 16 + (lane & 15)) * SK_LD + (lane >> 4) * 8);
    const uint32_t b_base = smem_u32(st + ((TWO_A ? 128 : 64) + (lane & 7) + (lane >> 4) * 8) * SK_LD +
                                     ((lane >> 3) & 1) * 8);
#pragma unroll
    for (int kk = 0; kk < SK_KC / 16; ++kk) {
      uint32_t a[4], a2[4];
      ldsm_x4(a_base + kk * 32, a[0], a[1], a[2], a[3]);
      if constexpr (TWO_A) ldsm_x4(a_base + kk * 32 + 64 * SK_LD * 2, a2[0], a2[1], a2[2], a2[3]);
#pragma unroll
      for (int t = 0; t < NC / 8; t += 2) {           // 16 columns per B load
        uint32_t bq[4];
        ldsm_x4(b_base + t * 8 * SK_LD * 2 + kk * 32, bq[0], bq[1], bq[2], bq[3]);
        const uint32_t b0[2] = {bq[0], bq[1]}, b1[2] = {bq[2], bq[3]};
        mma_bf16_16816(acc[t], a, b0);
        mma_bf16_16816(acc[t + 1], a, b1);
        if constexpr (TWO_A) {
          mma_bf16_16816(acc[t], a2, b0);
          mma_bf16_16816(acc[t + 1], a2, b1);
        }
      }
    }
    __syncthreads();                                  // stage c % S is refilled next
  }
  cp_async_wait_group<0>();
  const int gr = lane >> 2, qc = lane & 3;
#pragma unroll
  for (int t = 0; t < NC / 8; ++t) {
    const int n = n0 + t * 8 + 2 * qc;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = m0 + warp * 16 + gr + h * 8;
      if (m >= M) continue;
      const float v0 = acc[t][2 * h], v1 = acc[t][2 * h + 1];
      if constexpr (OUT_F32) {
        float *cp = static_cast<float *>(C) + (static_cast<size_t>(ks) * M + m) * N + n;
        if (n < N) cp[0] = v0;
        if (n + 1 < N) cp[1] = v1;
      } else {
        __nv_bfloat16 *cp = static_cast<__nv_bfloat16 *>(C) + static_cast<size_t>(m) * N + n;
        if (n + 1 < N) {
          *reinterpret_cast<uint32_t *>(cp) = pack_bf16x2(v0, v1);
        } else if (n < N) {
          cp[0] = __float2bfloat16_rn(v0);
        }
      }
    }
  }
}

template <bool OUT_F32, bool TWO_A, int S, int NC>
static cudaError_t launch_skinny(int ksplit, const __nv_bfloat16 *A, const __nv_bfloat16 *A2,
                                 const __nv_bfloat16 *B, void *C, int M, int N, int K,
                                 int *lengths, int max_seq, cudaStream_t st) {
  const int kps = ((K + ksplit - 1) / ksplit + SK_KC - 1) / SK_KC * SK_KC;
  const dim3 grid((N + NC - 1) / NC, ksplit, (M + 63) / 64);
  const size_t smem = static_cast<size_t>(S) * skinny_stage_elems<TWO_A, NC>() * 2;
  cudaError_t e = ensure_dyn_smem<skinny_mma_kernel<OUT_F32, TWO_A, S, NC>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(skinny_mma_kernel<OUT_F32, TWO_A, S, NC>, grid, dim3(128), smem, st, A, A2,
                    B, C, M, N, K, kps, lengths, max_seq);
}

// ------------------------------------------------------------------ D2 decode stencil
template <typename T>
struct D2Params {
  using TL = typename LatentType<T>::type;
  const float *p_part;
  int ksplit;
  const float *conv_seq, *conv_chan;
  TL *k_cache, *v_cache;
  float *conv_state, *vshift_state;
  int *lengths, *status;
  float *q_new;
  int B, H, Hkv, G, DL, NQ, NKV, NQKV, KC, VS0, max_seq;
  unsigned flags;
  float eps;
  double theta[32];        // RoPE frequencies base^(-2i/d~), i < d~/2, computed on the host
};

// D2 keeps the group's channel filters transposed in shared memory, wt[j][o] = the weight of
// input j for output channel o (o over the G q heads and the k head, d~ each), rows padded to
// an odd length so both the transposing writes and the per-output reads are conflict-free.
// The filters, which no earlier kernel writes, are staged before the grid-dependency wait;
// the sequence's conv state is only prefetched into L2 then (the previous step may still be
// writing it, and L2 keeps a prefetched line coherent).  After the wait the projections and
// the state are loaded together, and the old state stays in shared memory for the shift.
__host__ __device__ constexpr int d2_ld(int QKC) { return QKC | 1; }
__host__ __device__ inline size_t d2_smem_floats(int G, int DL, int KC) {
  const int QKC = (G + 1) * DL, CH = (G + 2) * DL;
  return 64                                     // RoPE frequencies (32 doubles)
         + static_cast<size_t>(DL) * d2_ld(QKC)   // wt
         + QKC * KC                             // sequence filters
         + static_cast<size_t>(QKC) * (KC - 1)  // old conv state
         + CH + 2 * QKC + 16                    // pn, av, uv, inv
         + DL;                                  // the value-shift state of the group's channels
}

// D2's shared-memory carve ([th | wt | wseq | old | pn | a | u | inv | vsh], floats; th holds
// doubles, so `sm` is 8-byte aligned)
template <int DL>
struct D2Smem {
  double *th;
  float *wt, *wseq, *old, *pn, *a, *u, *inv, *vsh;
  __device__ D2Smem(float *sm, int G, int KC) {
    const int QKC = (G + 1) * DL, CH = (G + 2) * DL;
    th = reinterpret_cast<double *>(sm);
    wt = sm + 64;
    wseq = wt + DL * d2_ld(QKC);
    old = wseq + QKC * KC;                           // [KC-1][QKC] conv state before the step
    pn = old + QKC * (KC - 1);
    a = pn + CH;
    u = a + QKC;
    inv = u + QKC;
    vsh = inv + 16;
  }
};

// Before the grid-dependency wait: the group's filters into shared memory (no __syncthreads),
// the sequence's conv and value-shift state towards L2.  The filters are read in batches of
// independent loads, so that a CTA which only becomes resident after the previous kernel's
// CTAs leave (and stages them with nothing to hide behind) pays one or two memory round trips.
template <typename T, int DL, int BATCH = 8>
__device__ __forceinline__ void d2_stage(const D2Params<T> &p, int g, int b, const D2Smem<DL> &m) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int G = p.G, QKC = (G + 1) * DL, KC = p.KC, KC1 = KC - 1;
  const int LD = d2_ld(QKC);
  // filters: q heads g*G.., then k head H+g; W_head[i][j] -> wt[j][head * DL + i], four
  // consecutive j of one (head, i) per load (16-byte loads when the filters are so aligned)
  const int nf4 = (G + 1) * DL * DL / 4;
  const bool vec = (reinterpret_cast<uintptr_t>(p.conv_chan) & 15u) == 0;
  for (int e0 = tid; e0 < nf4; e0 += BATCH * nt) {
    float4 v[BATCH];
#pragma unroll
    for (int k = 0; k < BATCH; ++k) {
      const int e = (e0 + k * nt) * 4;
      if (e0 + k * nt < nf4) {
        const int hh = e / (DL * DL), r = e % (DL * DL);
        const int head = hh < G ? g * G + hh : p.H + g;
        const float *src = p.conv_chan + static_cast<size_t>(head) * DL * DL + r;
        v[k] = vec ? *reinterpret_cast<const float4 *>(src) : make_float4(src[0], src[1], src[2], src[3]);
      }
    }
#pragma unroll
    for (int k = 0; k < BATCH; ++k) {
      const int e = (e0 + k * nt) * 4;
      if (e0 + k * nt < nf4) {
        const int hh = e / (DL * DL), r = e % (DL * DL), i = r / DL, j = r % DL;
        float *dst = m.wt + j * LD + hh * DL + i;
        dst[0] = v[k].x;
        dst[LD] = v[k].y;
        dst[2 * LD] = v[k].z;
        dst[3 * LD] = v[k].w;
      }
    }
  }
  const int qcol0 = g * G * DL, kcol0 = p.NQ + g * DL;
  for (int e0 = tid; e0 < QKC * KC; e0 += BATCH * nt) {
    float v[BATCH];
#pragma unroll
    for (int k = 0; k < BATCH; ++k) {
      const int e = e0 + k * nt;
      if (e < QKC * KC) {
        const int c = e / KC, t = e % KC;
        const int gc = c < G * DL ? qcol0 + c : kcol0 + (c - G * DL);
        v[k] = p.conv_seq[static_cast<size_t>(gc) * KC + t];
      }
    }
#pragma unroll
    for (int k = 0; k < BATCH; ++k)
      if (e0 + k * nt < QKC * KC) m.wseq[e0 + k * nt] = v[k];
  }
  for (int i = tid; i < DL / 2; i += nt) m.th[i] = p.theta[i];   // read once, off the param bank
  if (p.flags & F_VALUE_SHIFT) {                     // the shifted channels of this group
    const float *vs = p.vshift_state + static_cast<size_t>(b) * (p.NKV - p.VS0);
    for (int c = max(g * DL, p.VS0) + tid * 32; c < (g + 1) * DL; c += nt * 32)
      prefetch_l2(vs + (c - p.VS0));
  }
  const int W = p.NQ + p.NKV;
  const float *cs = p.conv_state + static_cast<size_t>(b) * KC1 * W;
  for (int e = tid; e < KC1 * (G + 1); e += nt) {   // the state rows of this group's channels
    const int j = e / (G + 1), part = e % (G + 1);  // (G q heads' DL run is contiguous)
    const float *row = cs + static_cast<size_t>(j) * W;
    const float *seg = part == 0 ? row + qcol0 : row + kcol0;
    const int len = part == 0 ? G * DL : DL;
    for (int off = 0; off < len; off += 32) prefetch_l2(seg + off);
  }
}

// After the wait: the token's projections (sum of the split-K partials), the old conv state and
// the value-shift state into shared memory, thread c taking channel c (the compute below keeps
// that mapping for the projections and the conv state).
template <typename T, int DL>
__device__ __forceinline__ void d2_load(const D2Params<T> &p, int g, int b, const D2Smem<DL> &m,
                                        int tid, int nt) {
  const int G = p.G, CH = (G + 2) * DL, QKC = (G + 1) * DL, KC1 = p.KC - 1;
  const int qcol0 = g * G * DL, kcol0 = p.NQ + g * DL, vcol0 = p.NQ + p.NKV + g * DL;
  const int W = p.NQ + p.NKV;
  const float *cs = p.conv_state + static_cast<size_t>(b) * KC1 * W;
  const size_t kstride = static_cast<size_t>(p.B) * p.NQKV;
  const float *vs = p.vshift_state + static_cast<size_t>(b) * (p.NKV - p.VS0);
  // channel c's first eight split-K partials, state rows (KC <= 8) and value-shift entry
  auto fetch = [&](int c, float (&part)[8], float (&st)[7], float &vsv) {
    const int gc = c < G * DL ? qcol0 + c : (c < QKC ? kcol0 + (c - G * DL) : vcol0 + (c - QKC));
    const float *pp = p.p_part + static_cast<size_t>(b) * p.NQKV + gc;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) part[ks] = c < CH && ks < p.ksplit ? pp[ks * kstride] : 0.f;
#pragma unroll
    for (int j = 0; j < 7; ++j)
      st[j] = c < QKC && j < KC1 ? cs[static_cast<size_t>(j) * W + gc] : 0.f;
    const int vc = g * DL + (c - QKC);              // a value channel's index in N_kv
    const bool shifted = c >= QKC && c < CH && (p.flags & F_VALUE_SHIFT) && vc >= p.VS0;
    vsv = shifted ? vs[vc - p.VS0] : 0.f;
  };
  auto put = [&](int c, const float (&part)[8], const float (&st)[7], float vsv) {
    if (c >= CH) return;
    float v = ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
    if (p.ksplit > 8) {
      const int gc = c < G * DL ? qcol0 + c : (c < QKC ? kcol0 + (c - G * DL) : vcol0 + (c - QKC));
      const float *pp = p.p_part + static_cast<size_t>(b) * p.NQKV + gc;
      for (int ks = 8; ks < p.ksplit; ++ks) v += pp[ks * kstride];
    }
    m.pn[c] = v;
    if (c >= QKC) m.vsh[c - QKC] = vsv;
    if (c < QKC)
#pragma unroll
      for (int j = 0; j < 7; ++j)
        if (j < KC1) m.old[j * QKC + c] = st[j];
  };
  // two channels per thread and pass, both channels' loads issued before either is stored, so
  // that a CTA with more channels than threads still pays one memory round trip
  for (int c = tid; c < CH; c += 2 * nt) {
    float pa[8], sa[7], va, pb[8], sb[7], vb;
    fetch(c, pa, sa, va);
    fetch(c + nt, pb, sb, vb);
    put(c, pa, sa, va);
    put(c + nt, pb, sb, vb);
  }
}

// The stencil of the new token at position L (< max_seq): k and v rows appended to the cache,
// the G query heads' rotated latents to q (head hh at q + hh * DL; global or shared memory),
// conv / value-shift state advanced.  Threads tid = 0..nt-1 (the ones that ran d2_load, with
// the same numbering) take part and meet at named barrier `bar`; kv_keep (optional, shared
// memory [2][DL]) receives the appended key and value as the cache holds them.
template <typename T, int DL>
__device__ __forceinline__ void d2_compute(const D2Params<T> &p, int g, int b, int L,
                                           const D2Smem<DL> &m, float *q, int tid, int nt, int bar,
                                           float *kv_keep = nullptr) {
  using TL = typename D2Params<T>::TL;
  const int G = p.G, QKC = (G + 1) * DL, KC = p.KC, KC1 = KC - 1;
  const int LD = d2_ld(QKC);
  const int qcol0 = g * G * DL, kcol0 = p.NQ + g * DL;
  const int W = p.NQ + p.NKV;
  float *cs = p.conv_state + static_cast<size_t>(b) * KC1 * W;
  constexpr int HALF = DL / 2;
  float rc = 1.f, rs = 0.f;                          // RoPE rotation of this thread's pairs
  if ((p.flags & F_ROPE) && tid < (G + 1) * HALF)
    rope_cos_sin(static_cast<double>(L) * m.th[tid % HALF], rc, rs);
  // the sequence conv of the q|k channels (each thread reads only what it loaded)
  for (int c = tid; c < QKC; c += nt) {
    const float *w = m.wseq + c * KC;
    float acc = 0.f;
    for (int j = 0; j < KC1; ++j) acc = fmaf(w[j], m.old[j * QKC + c], acc);
    m.a[c] = fmaf(w[KC1], m.pn[c], acc);
  }
  bar_sync(bar, nt);
  // channel conv (thread per output) and q-k-mean
  for (int o = tid; o < QKC; o += nt) {
    const int hh = o / DL, i = o % DL;
    const float *ah = m.a + hh * DL;
    float acc = 0.f;
#pragma unroll 8
    for (int j = 0; j < DL; ++j) acc = fmaf(m.wt[j * LD + o], ah[j], acc);
    if (p.flags & F_QK_MEAN) {
      const float pk = m.pn[G * DL + i];
      if (hh < G) {
        acc += 0.5f * (m.pn[o] + pk);
      } else {
        float mq = 0.f;
        for (int h2 = 0; h2 < G; ++h2) mq += m.pn[h2 * DL + i];
        acc += 0.5f * (mq / static_cast<float>(G) + pk);
      }
    }
    m.u[o] = acc;
  }
  bar_sync(bar, nt);
  // RMS norm per head: one warp per head
  const int warp = tid >> 5, lane = tid & 31;
  for (int hh = warp; hh <= G; hh += nt / 32) {
    float ss = 0.f;
    for (int i = lane; i < DL; i += 32) ss += m.u[hh * DL + i] * m.u[hh * DL + i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0)
      m.inv[hh] = (p.flags & F_QK_NORM) ? 1.0f / sqrtf(ss / static_cast<float>(DL) + p.eps) : 1.0f;
  }
  bar_sync(bar, nt);
  // RoPE at position L on (i, i + DL/2) pairs, then store q and k (cache); every pair a thread
  // takes has i = tid mod DL/2 (DL/2 divides the block size), whose rotation it computed above
  for (int o = tid; o < (G + 1) * HALF; o += nt) {
    const int hh = o / HALF, ip = o % HALF;
    float x1 = m.u[hh * DL + ip] * m.inv[hh], x2 = m.u[hh * DL + ip + HALF] * m.inv[hh];
    if (p.flags & F_ROPE) {
      const float y1 = x1 * rc - x2 * rs, y2 = x1 * rs + x2 * rc;
      x1 = y1;
      x2 = y2;
    }
    if (hh < G) {
      q[hh * DL + ip] = x1;
      q[hh * DL + ip + HALF] = x2;
    } else {
      auto *kd = p.k_cache + ((static_cast<size_t>(b) * p.Hkv + g) * p.max_seq + L) * DL;
      check_latent<TL>(x1, p.status);
      check_latent<TL>(x2, p.status);
      const TL k1 = from_f32<TL>(x1), k2 = from_f32<TL>(x2);
      kd[ip] = k1;
      kd[ip + HALF] = k2;
      if (kv_keep) {                                 // the appended key as the cache holds it
        kv_keep[ip] = to_f32(k1);
        kv_keep[ip + HALF] = to_f32(k2);
      }
    }
  }
  // value with the value-shift, appended at position L
  const int vhalf = p.VS0;
  float *vs = p.vshift_state + static_cast<size_t>(b) * (p.NKV - vhalf);
  for (int c = tid; c < DL; c += nt) {
    const int vc = g * DL + c;
    const bool shifted = vc >= vhalf;
    const float val = ((p.flags & F_VALUE_SHIFT) && shifted) ? m.vsh[c] : m.pn[QKC + c];
    check_latent<TL>(val, p.status);
    const TL vv = from_f32<TL>(val);
    p.v_cache[((static_cast<size_t>(b) * p.Hkv + g) * p.max_seq + L) * DL + c] = vv;
    if (kv_keep) kv_keep[DL + c] = to_f32(vv);
  }
  // state advance (thread c rewrites only channel c's state, which it alone read)
  for (int c = tid; c < QKC; c += nt) {
    const int gc = c < G * DL ? qcol0 + c : kcol0 + (c - G * DL);
    for (int j = 0; j + 1 < KC1; ++j) cs[static_cast<size_t>(j) * W + gc] = m.old[(j + 1) * QKC + c];
    if (KC1 > 0) cs[static_cast<size_t>(KC1 - 1) * W + gc] = m.pn[c];
  }
  for (int c = tid; c < DL; c += nt) {
    const int vc = g * DL + c;
    if (vc >= vhalf) vs[vc - vhalf] = m.pn[QKC + c];
  }
}

template <typename T, int DL>
__global__ void __launch_bounds__(256) decode_stencil_kernel(const D2Params<T> p) {
  extern __shared__ __align__(16) float sm[];
  const int g = blockIdx.x, b = blockIdx.y;
  const D2Smem<DL> m(sm, p.G, p.KC);
  pdl_launch_dependents();
  d2_stage(p, g, b, m);
  __syncthreads();                                   // staged filters visible to every thread
  pdl_wait();
  d2_load(p, g, b, m, threadIdx.x, blockDim.x);      // loads in flight before the position
  const int L = p.lengths[b];
  if (L >= p.max_seq) {
    if (threadIdx.x == 0) report(p.status, DEV_CACHE_FULL);
    return;
  }
  d2_compute(p, g, b, L, m, p.q_new + (static_cast<size_t>(b) * p.H + g * p.G) * DL, threadIdx.x,
             blockDim.x, 0);
}

// ------------------------------------------------------------------ D3 split-KV attention
// One CTA per (sequence, kv group, split of CHUNK keys).  The split is walked in sub-chunks of
// SUB keys through a two-deep ring of 16-byte asynchronous copies, so the copy of sub-chunk
// i+1 is in flight while sub-chunk i is computed.  Keys land with their 16-byte pieces
// XOR-swizzled by row (the one-row-per-thread reads below then hit eight bank groups).
// Per sub-chunk:
//   scores  one thread per key, the group's G queries broadcast from shared memory
//   softmax one warp per head: running max m and sum l across sub-chunks; the P V
//           accumulators are rescaled by 2^(m_old - m_new) when the max moves
//   P V     thread (dim pair, key slice) accumulates G heads x 2 dims
// The split's unnormalised o and its (m, l) go to the workspace for the merge.
constexpr int SUB = 256;

template <int CPR>
__device__ __forceinline__ int kv_swz(int r) {       // swizzle of a row's 16-byte pieces
  constexpr int SPAN = CPR < 8 ? CPR : 8;
  constexpr int DIV = CPR < 8 ? 8 / CPR : 1;
  return (r / DIV) & (SPAN - 1);
}

template <int DL, typename TL>
__global__ void __launch_bounds__(128) decode_attn_kernel(
    const float *__restrict__ q_new, const TL *__restrict__ k_cache,
    const TL *__restrict__ v_cache, const int *__restrict__ lengths, float *__restrict__ part_o,
    float *__restrict__ part_ml, int H, int Hkv, int G, int max_seq, int nchunk,
    float scale_log2) {
  constexpr int EPC = 16 / sizeof(TL);               // elements per 16-byte piece
  constexpr int CPR = DL / EPC;                      // pieces per row
  constexpr int PAIRS = DL / 2;
  constexpr int KS = 128 / PAIRS;                    // key slices in the P V phase
  constexpr int GMAX = 8;                            // heads per P V pass
  extern __shared__ __align__(16) uint8_t smraw[];
  TL *Kb = reinterpret_cast<TL *>(smraw);            // [2][SUB][DL], swizzled pieces
  TL *Vb = Kb + 2 * SUB * DL;                        // [2][SUB][DL]
  float *qs = reinterpret_cast<float *>(Vb + 2 * SUB * DL);   // [G][DL], pre-scaled
  float *sc = qs + G * DL;                           // [G][SUB]
  float *red = sc + G * SUB;                         // [KS][G][DL]
  float *mls = red + KS * G * DL;                    // [G][2] running (m, l)
  float *scl = mls + 2 * G;                          // [G] rescale of this sub-chunk
  const int ch = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int L = lengths[b];
  const int s0 = ch * CHUNK;
  const int n = L < max_seq ? min(CHUNK, L + 1 - s0) : 0;
  float *po = part_o + ((static_cast<size_t>(b) * H + g * G) * nchunk + ch) * DL;
  float *pml = part_ml + ((static_cast<size_t>(b) * H + g * G) * nchunk + ch) * 2;
  if (n <= 0) {
    for (int i = tid; i < G * DL; i += blockDim.x)
      po[static_cast<size_t>(i / DL) * nchunk * DL + (i % DL)] = 0.f;
    for (int h = tid; h < G; h += blockDim.x) {
      pml[static_cast<size_t>(h) * nchunk * 2] = -INFINITY;
      pml[static_cast<size_t>(h) * nchunk * 2 + 1] = 0.f;
    }
    return;
  }
  const size_t row0 = (static_cast<size_t>(b) * Hkv + g) * max_seq + s0;
  const int nsub = (n + SUB - 1) / SUB;
  auto issue = [&](int sbi) {                        // copies of sub-chunk sbi into slot sbi&1
    const int base = sbi * SUB, cnt = min(SUB, n - base);
    TL *kd = Kb + (sbi & 1) * SUB * DL, *vd = Vb + (sbi & 1) * SUB * DL;
    for (int i = tid; i < cnt * CPR; i += blockDim.x) {
      const int r = i / CPR, j = i % CPR;
      const size_t src = (row0 + base + r) * DL + j * EPC;
      cp_async16_zfill(kd + r * DL + (j ^ kv_swz<CPR>(r)) * EPC, k_cache + src, true);
      cp_async16_zfill(vd + r * DL + j * EPC, v_cache + src, true);
    }
    cp_async_commit();
  };
  issue(0);
  for (int i = tid; i < G * DL; i += blockDim.x)
    qs[i] = q_new[(static_cast<size_t>(b) * H + g * G) * DL + i] * scale_log2;
  for (int h = tid; h < G; h += blockDim.x) {
    mls[2 * h] = -INFINITY;
    mls[2 * h + 1] = 0.f;
  }
  const int dp = tid % PAIRS, ks = tid / PAIRS;
  float acc[GMAX][2];                                // P V accumulators (G <= 8 here)
#pragma unroll
  for (int h = 0; h < GMAX; ++h) acc[h][0] = acc[h][1] = 0.f;

  for (int sbi = 0; sbi < nsub; ++sbi) {
    if (sbi + 1 < nsub) {
      issue(sbi + 1);
      cp_async_wait_one();                           // sub-chunk sbi has landed
    } else {
      cp_async_wait_none();
    }
    __syncthreads();
    const TL *Ks = Kb + (sbi & 1) * SUB * DL, *Vs = Vb + (sbi & 1) * SUB * DL;
    const int cnt = min(SUB, n - sbi * SUB);
    // scores
    for (int r = tid; r < cnt; r += blockDim.x) {
      float kf[DL];
#pragma unroll
      for (int j = 0; j < CPR; ++j) {
        float e8[EPC];
        const TL *src = Ks + r * DL + (j ^ kv_swz<CPR>(r)) * EPC;
        if constexpr (EPC == 8) {
          load8(src, *reinterpret_cast<float(*)[8]>(e8));
        } else {
          const float4 f = *reinterpret_cast<const float4 *>(src);
          e8[0] = f.x; e8[1] = f.y; e8[2] = f.z; e8[3] = f.w;
        }
#pragma unroll
        for (int e = 0; e < EPC; ++e) kf[j * EPC + e] = e8[e];
      }
      for (int h = 0; h < G; ++h) {
        const float4 *qh = reinterpret_cast<const float4 *>(qs + h * DL);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int d4 = 0; d4 < DL / 4; ++d4) {
          const float4 qv = qh[d4];
          a0 = fmaf(qv.x, kf[4 * d4 + 0], a0);
          a1 = fmaf(qv.y, kf[4 * d4 + 1], a1);
          a2 = fmaf(qv.z, kf[4 * d4 + 2], a2);
          a3 = fmaf(qv.w, kf[4 * d4 + 3], a3);
        }
        sc[h * SUB + r] = (a0 + a1) + (a2 + a3);
      }
    }
    __syncthreads();
    // running max and sum per head
    for (int h = warp; h < G; h += blockDim.x / 32) {
      float mx = -INFINITY;
      for (int r = lane; r < cnt; r += 32) mx = fmaxf(mx, sc[h * SUB + r]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = mls[2 * h];
      const float m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int r = lane; r < cnt; r += 32) {
        const float e = exp2f(sc[h * SUB + r] - m_new);
        sc[h * SUB + r] = e;
        sum += e;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) {
        const float f = exp2f(m_old - m_new);        // 0 on the first sub-chunk
        scl[h] = f;
        mls[2 * h] = m_new;
        mls[2 * h + 1] = mls[2 * h + 1] * f + sum;
      }
    }
    __syncthreads();
    // P V
#pragma unroll
    for (int h = 0; h < GMAX; ++h) {
      if (h < G) {
        const float f = scl[h];
        acc[h][0] *= f;
        acc[h][1] *= f;
      }
    }
    for (int r = ks; r < cnt; r += KS) {
      float2 v;
      if constexpr (sizeof(TL) == 2) {
        v = __half22float2(*reinterpret_cast<const __half2 *>(Vs + r * DL + 2 * dp));
      } else {
        v = *reinterpret_cast<const float2 *>(Vs + r * DL + 2 * dp);
      }
#pragma unroll
      for (int h = 0; h < GMAX; ++h) {
        if (h < G) {
          const float pr = sc[h * SUB + r];
          acc[h][0] = fmaf(pr, v.x, acc[h][0]);
          acc[h][1] = fmaf(pr, v.y, acc[h][1]);
        }
      }
    }
    __syncthreads();                                 // slot sbi&1 and sc are reused next
  }
#pragma unroll
  for (int h = 0; h < GMAX; ++h) {
    if (h < G) {
      red[(ks * G + h) * DL + 2 * dp] = acc[h][0];
      red[(ks * G + h) * DL + 2 * dp + 1] = acc[h][1];
    }
  }
  __syncthreads();
  for (int i = tid; i < G * DL; i += blockDim.x) {
    float o = 0.f;
#pragma unroll
    for (int k = 0; k < KS; ++k) o += red[k * G * DL + i];
    po[static_cast<size_t>(i / DL) * nchunk * DL + (i % DL)] = o;
  }
  for (int h = tid; h < G; h += blockDim.x) {
    pml[static_cast<size_t>(h) * nchunk * 2] = mls[2 * h];
    pml[static_cast<size_t>(h) * nchunk * 2 + 1] = mls[2 * h + 1];
  }
}

// ------------------------------------------------------------------ D3 on tensor cores
// The float16-cache variant of D3.  CTA = sequence x kv group x key split; the split's keys
// stream through an NSLOT-deep ring of TC_SUB-key sub-chunks (NSLOT - 1 sub-chunks in flight
// while one is computed: one CTA has to keep enough bytes in flight to draw its share of the
// memory bandwidth), loaded with an L2 evict-first hint so the stream does not push out the
// weights and activations the step's other kernels read.  Each warp owns a quarter of every
// sub-chunk and runs its own online softmax on mma.sync tiles:
//   S = Q K^T   m16n8k16, rows = the G query heads (rows G..15 zero), 8 keys per n-tile,
//               Q rounded to float16 like the prefill's latent q, in registers; K through
//               ldmatrix; the scores are scaled by log2(e)/sqrt(d~) in fp32
//   P V         the S accumulators of two n-tiles are, after exp2 and rounding to float16,
//               exactly the A fragment of the next m16n8k16 (keys as K); V enters through
//               ldmatrix.trans
// Row max and sum are per head row, reduced over the four lanes that hold a row.  The four
// warps' (m, l, o) are combined in shared memory before the split's partials are written.
constexpr int TC_SUB = 256;                  // keys per sub-chunk
constexpr int TC_RING_BYTES = 96 * 1024;     // copy ring budget (two CTAs per SM at d~ = 32)

template <int DL>
__host__ __device__ constexpr int tc_slots() {
  return TC_RING_BYTES / (TC_SUB * DL * 4) > 2 ? TC_RING_BYTES / (TC_SUB * DL * 4) : 2;
}

template <int DL>
__host__ __device__ constexpr size_t tc_smem_bytes() {
  return static_cast<size_t>(tc_slots<DL>()) * TC_SUB * DL * 4 + 4 * 8 * (DL + 2) * 4;
}

template <int DL>
__global__ void __launch_bounds__(128, 1) decode_attn_tc_kernel(
    const float *__restrict__ q_new, const __half *__restrict__ k_cache,
    const __half *__restrict__ v_cache, const int *__restrict__ lengths,
    float *__restrict__ part_o, float *__restrict__ part_ml, __nv_bfloat16 *__restrict__ o_hi,
    __nv_bfloat16 *__restrict__ o_lo, int H, int Hkv, int G, int max_seq, int chunk, int nchunk,
    float scale_log2, const uint8_t *__restrict__ next_w, size_t next_w_bytes) {
  constexpr int CPR = DL / 8;                        // 16-byte pieces (8 dims) per row
  constexpr int NSLOT = tc_slots<DL>();
  constexpr int NT = TC_SUB / 32;                    // 8-key n-tiles per warp step
  constexpr int WK = NT * 8;                         // keys per warp per sub-chunk
  constexpr int SLOT = 2 * TC_SUB * DL;              // halves per slot: [K | V]
  static_assert(4 * WK == TC_SUB && NT % 2 == 0, "four warps cover a sub-chunk");
  // cp.async.wait_group NSLOT - 2 below: a 12-slot ring (wait_group 10) raised an illegal
  // instruction on this GPU, 6 slots (wait_group 4) run; keep the count of groups in flight small
  static_assert(NSLOT <= 6, "at most five copy groups in flight");
  extern __shared__ __align__(16) uint8_t smraw[];
  __half *ring = reinterpret_cast<__half *>(smraw);  // [NSLOT][K, V][TC_SUB][DL], swizzled
  float *wst = reinterpret_cast<float *>(ring + NSLOT * SLOT);     // [4][8 heads][DL + 2]
  const int ch = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, gr = lane >> 2, qd = lane & 3;
  pdl_launch_dependents();
  {
    // the up-projection weights, which nothing in the step writes, towards L2 for the step's
    // last kernel (the evict-first cache stream leaves them there); an equal share per CTA
    const size_t lines = (next_w_bytes + 127) / 128;
    const size_t ctas = static_cast<size_t>(gridDim.x) * gridDim.y * gridDim.z;
    const size_t id = (static_cast<size_t>(b) * gridDim.y + g) * gridDim.x + ch;
    const size_t per = (lines + ctas - 1) / ctas;
    for (size_t i = id * per + tid; i < min(lines, (id + 1) * per); i += blockDim.x)
      prefetch_l2(next_w + i * 128);
  }
  pdl_wait();
  const int L = lengths[b];
  const int s0 = ch * chunk;
  const int n = L < max_seq ? min(chunk, L + 1 - s0) : 0;   // keys of this split
  float *po = part_o + ((static_cast<size_t>(b) * H + g * G) * nchunk + ch) * DL;
  float *pml = part_ml + ((static_cast<size_t>(b) * H + g * G) * nchunk + ch) * 2;
  const bool whole = nchunk == 1;                    // one split: write the merged o itself
  if (n <= 0) {
    for (int i = tid; i < G * DL; i += blockDim.x) {
      if (whole) {
        o_hi[(static_cast<size_t>(b) * H + g * G) * DL + i] = __float2bfloat16_rn(0.f);
        o_lo[(static_cast<size_t>(b) * H + g * G) * DL + i] = __float2bfloat16_rn(0.f);
      } else {
        po[static_cast<size_t>(i / DL) * nchunk * DL + (i % DL)] = 0.f;
      }
    }
    for (int h = tid; h < G && !whole; h += blockDim.x) {
      pml[static_cast<size_t>(h) * nchunk * 2] = -INFINITY;
      pml[static_cast<size_t>(h) * nchunk * 2 + 1] = 0.f;
    }
    return;
  }
  const size_t row0 = (static_cast<size_t>(b) * Hkv + g) * max_seq + s0;
  const int nsub = (n + TC_SUB - 1) / TC_SUB;
  const uint64_t stream_pol = l2_evict_first_policy();
  auto issue = [&](int sbi) {                        // sub-chunk sbi into slot sbi % NSLOT;
    if (sbi < nsub) {                                // an empty group past the last one
      const int base = sbi * TC_SUB, cnt = min(TC_SUB, n - base);  // rows past cnt: zeros
      __half *kd = ring + (sbi % NSLOT) * SLOT, *vd = kd + TC_SUB * DL;
      for (int i = tid; i < TC_SUB * CPR; i += blockDim.x) {
        const int r = i / CPR, j = i % CPR;
        const bool ok = r < cnt;
        const size_t src = (row0 + base + (ok ? r : 0)) * DL + j * 8;
        const int dst = r * DL + (j ^ kv_swz<CPR>(r)) * 8;
        cp_async16_zfill_stream(kd + dst, k_cache + src, ok, stream_pol);
        cp_async16_zfill_stream(vd + dst, v_cache + src, ok, stream_pol);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int s = 0; s < NSLOT - 1; ++s) issue(s);


  // Q fragments (rows = heads; a1, a3 are rows 8..15 and stay zero)
  uint32_t qa[DL / 16][2];
  {
    const float *qh = q_new + (static_cast<size_t>(b) * H + g * G + gr) * DL;
#pragma unroll
    for (int kk = 0; kk < DL / 16; ++kk) {
      float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
      if (gr < G) {
        v0 = qh[16 * kk + 2 * qd];
        v1 = qh[16 * kk + 2 * qd + 1];
        v2 = qh[16 * kk + 2 * qd + 8];
        v3 = qh[16 * kk + 2 * qd + 9];
      }
      qa[kk][0] = pack_f16x2(v0, v1);
      qa[kk][1] = pack_f16x2(v2, v3);
    }
  }
  float o[DL / 8][4];
#pragma unroll
  for (int t = 0; t < DL / 8; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;              // of head row gr (lanes of one quad agree)

  for (int sbi = 0; sbi < nsub; ++sbi) {
    cp_async_wait_group<NSLOT - 2>();                // sub-chunk sbi has landed
    __syncthreads();                                 // ... for every thread; and every warp
    issue(sbi + NSLOT - 1);                          // is done with the slot refilled here
    const uint32_t ks_base = smem_u32(ring + (sbi % NSLOT) * SLOT);
    const uint32_t vs_base = ks_base + TC_SUB * DL * 2;
    const int kb = warp * WK;                        // this warp's first key in the sub-chunk
    const int valid = n - sbi * TC_SUB - kb;         // keys of this warp's slice that exist
    if (valid > 0) {
      // ---- S = Q K^T over 8 n-tiles
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int m0 = 0; m0 < NT * CPR; m0 += 4) {      // four (n-tile, piece) matrices per load
        const int id = m0 + (lane >> 3);
        const int nt = id / CPR, j = id % CPR;
        const int r = kb + nt * 8 + (lane & 7);
        uint32_t f[4];
        ldsm_x4(ks_base + (r * DL + (j ^ kv_swz<CPR>(r)) * 8) * 2, f[0], f[1], f[2], f[3]);
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          // matrices m0+e, m0+e+1 = pieces (2c, 2c+1) of one n-tile = one 16-dim k step
          const int idm = m0 + e, ntm = idm / CPR, kk = (idm % CPR) / 2;
          const uint32_t a[4] = {qa[kk][0], 0u, qa[kk][1], 0u};
          const uint32_t bb[2] = {f[e], f[e + 1]};
          mma_f16_16816(sc[ntm], a, bb);
        }
      }
      // ---- online softmax of row gr over this warp's 64 keys (scores to log2 units here,
      // after the product, as in the prefill attention)
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          sc[nt][e] = nt * 8 + 2 * qd + e < valid ? sc[nt][e] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, sc[nt][e]);
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);          // finite: key kb of this slice is valid
      const float f = exp2f(m_run - m_new);          // 0 while m_run = -inf
      m_run = m_new;
      float ls = 0.f;
      uint32_t pa[NT / 2][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float p0 = exp2f(sc[nt][0] - m_new), p1 = exp2f(sc[nt][1] - m_new);
        ls += p0 + p1;
        pa[nt / 2][nt & 1] = pack_f16x2(p0, p1);
      }
      l_run = l_run * f + ls;
#pragma unroll
      for (int t = 0; t < DL / 8; ++t) {
        o[t][0] *= f;
        o[t][1] *= f;
      }
      // ---- O += P V: 4 k-steps of 16 keys x DL/8 n-tiles of dims
#pragma unroll
      for (int kk = 0; kk < NT / 2; ++kk) {
        const uint32_t a[4] = {pa[kk][0], 0u, pa[kk][1], 0u};
#pragma unroll
        for (int t0 = 0; t0 < DL / 8; t0 += 2) {      // two dim n-tiles (4 matrices) per load
          const int id = lane >> 3;                  // (dim tile t0 + id/2, key half id&1)
          const int r = kb + kk * 16 + (id & 1) * 8 + (lane & 7);
          const int j = t0 + (id >> 1);
          uint32_t f4[4];
          ldsm_x4_t(vs_base + (r * DL + (j ^ kv_swz<CPR>(r)) * 8) * 2, f4[0], f4[1], f4[2], f4[3]);
          const uint32_t b0[2] = {f4[0], f4[1]}, b1[2] = {f4[2], f4[3]};
          mma_f16_16816(o[t0], a, b0);
          mma_f16_16816(o[t0 + 1], a, b1);
        }
      }
    }
  }
  cp_async_wait_group<0>();                          // only empty groups can be left

  // ---- combine the four warps: each posts (m, l, o) of its head rows
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  constexpr int WS = DL + 2;
  if (gr < G) {
    float *w = wst + (warp * 8 + gr) * WS;
#pragma unroll
    for (int t = 0; t < DL / 8; ++t) {
      w[t * 8 + 2 * qd] = o[t][0];
      w[t * 8 + 2 * qd + 1] = o[t][1];
    }
    if (qd == 0) {
      w[DL] = m_run;
      w[DL + 1] = l_run;
    }
  }
  __syncthreads();
  for (int i = tid; i < G * DL; i += blockDim.x) {
    const int h = i / DL, d = i % DL;
    float mw[4], M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      mw[w] = wst[(w * 8 + h) * WS + DL];
      M = fmaxf(M, mw[w]);
    }
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float c = mw[w] == -INFINITY ? 0.f : exp2f(mw[w] - M);
      acc = fmaf(c, wst[(w * 8 + h) * WS + d], acc);
      lsum = fmaf(c, wst[(w * 8 + h) * WS + DL + 1], lsum);
    }
    if (whole) {
      const float v = acc / lsum;
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      const size_t idx = (static_cast<size_t>(b) * H + g * G) * DL + i;
      o_hi[idx] = hi;
      o_lo[idx] = __float2bfloat16_rn(v - __bfloat162float(hi));
    } else {
      po[static_cast<size_t>(h) * nchunk * DL + d] = acc;
      if (d == 0) {
        pml[static_cast<size_t>(h) * nchunk * 2] = M;
        pml[static_cast<size_t>(h) * nchunk * 2 + 1] = lsum;
      }
    }
  }
}

// ------------------------------------------------------------------ D2 + D3, cache buffered in TMEM
// The stencil of the new token sits on the path to the first score (no score exists before q),
// and in decode_attn_tc_kernel the cache stream meanwhile stops after the two sub-chunks its
// copy ring has free (the third slot holds the stencil's filters).  This kernel adds four
// filler warps (4..7) beside the four compute warps (0..3): while the compute warps run the
// stencil, the fillers stream the first sub-chunks through the two free slots and park each in
// tensor memory already in the compute warps' MMA fragment form (filler warp 4 + w issues
// exactly the ldmatrix reads compute warp w would, and stores the words to the TMEM lanes of
// their common lane quadrant, one column per word), then leave the next sub-chunks in the free
// slots.  The compute warps take the parked sub-chunks from TMEM (tcgen05.ld straight into
// fragments), then continue through the ring as decode_attn_tc_kernel does.  Hand-offs use
// named barriers: FZ_BAR_TM + i (sub-chunk i parked; fillers arrive, compute warps wait),
// FZ_BAR_HO (both sides: the fillers' copies have landed, the compute warps are done with
// TMEM, which warp 4 then frees), FZ_BAR_C / FZ_BAR_F (within the compute / filler warps).
constexpr int FZ_TMEM_COLS = 256;            // per CTA: two CTAs per SM share the 512 columns
constexpr int FZ_BAR_C = 1, FZ_BAR_F = 2, FZ_BAR_TM = 3;

template <int DL>
__host__ __device__ constexpr int fz_words() {   // fragment words per thread per sub-chunk
  return 2 * (TC_SUB / 32) * (DL / 8);
}
// sub-chunks parked in TMEM: as many as the columns hold, rounded down to a multiple of the
// free slots (so the ring positions the fillers leave match the compute warps' ring order)
template <int DL>
__host__ __device__ constexpr int fz_parked() {
  return FZ_TMEM_COLS / fz_words<DL>() / (tc_slots<DL>() - 1) * (tc_slots<DL>() - 1);
}
// the ring and combine area of decode_attn_tc_kernel, then the new token's queries [8][DL],
// key and value [2][DL] (float16-rounded), the G heads' scores of the new key [8] and the TMEM
// address
template <int DL>
__host__ __device__ constexpr size_t fz_smem_bytes() {
  return tc_smem_bytes<DL>() + (8 * DL + 2 * DL + 8) * 4 + 16;
}

template <int DL>
__global__ void __launch_bounds__(256, 2) decode_attn_fused_kernel(
    const __half *__restrict__ k_cache, const __half *__restrict__ v_cache,
    const int *__restrict__ lengths, __nv_bfloat16 *__restrict__ o_hi,
    __nv_bfloat16 *__restrict__ o_lo, int H, int Hkv, int G, int max_seq, float scale_log2,
    const uint8_t *__restrict__ next_w, size_t next_w_bytes, const D2Params<__nv_bfloat16> p2) {
  constexpr int CPR = DL / 8;                        // 16-byte pieces (8 dims) per row
  constexpr int NSLOT = tc_slots<DL>();
  constexpr int NT = TC_SUB / 32;                    // 8-key n-tiles per warp step
  constexpr int WK = NT * 8;                         // keys per warp per sub-chunk
  constexpr int SLOT = 2 * TC_SUB * DL;              // halves per slot: [K | V]
  constexpr int KW = NT * CPR;                       // K (and V) fragment words per thread
  constexpr int FW = 2 * KW;
  constexpr int NPARK = fz_parked<DL>();
  constexpr int FREE = NSLOT - 1;                    // slots free while the stencil runs
  constexpr int FZ_BAR_HO = FZ_BAR_TM + NPARK;
  static_assert(4 * WK == TC_SUB && NT % 2 == 0, "four warps cover a sub-chunk");
  static_assert(KW % 16 == 0, "TMEM stores of 16 columns");
  static_assert(NPARK >= FREE && NPARK * FW <= FZ_TMEM_COLS && FZ_BAR_HO < 16, "TMEM parking");
  static_assert(NSLOT <= 6, "at most five copy groups in flight");
  extern __shared__ __align__(16) uint8_t smraw[];
  __half *ring = reinterpret_cast<__half *>(smraw);  // [NSLOT][K, V][TC_SUB][DL], swizzled
  float *wst = reinterpret_cast<float *>(ring + NSLOT * SLOT);     // [4][8 heads][DL + 2]
  float *qn = wst + 4 * 8 * (DL + 2);                // [8][DL] queries of the new token
  float *kvn = qn + 8 * DL;                          // [2][DL] its key and value
  float *sn = kvn + 2 * DL;                          // [8] scores of the new key
  uint32_t *taddr_s = reinterpret_cast<uint32_t *>(sn + 8);
  float *scratch = reinterpret_cast<float *>(ring + (NSLOT - 1) * SLOT);
  const int g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, gr = lane >> 2, qd = lane & 3;
  const int t = tid & 127;                           // index within the compute or filler half
  const bool filler = warp >= 4;
  {
    // the up-projection weights, which nothing in the step writes, towards L2 for the step's
    // last kernel (the evict-first cache stream leaves them there); an equal share per CTA
    const size_t lines = (next_w_bytes + 127) / 128;
    const size_t ctas = static_cast<size_t>(gridDim.y) * gridDim.z;
    const size_t id = static_cast<size_t>(b) * gridDim.y + g;
    const size_t per = (lines + ctas - 1) / ctas;
    for (size_t i = id * per + tid; i < min(lines, (id + 1) * per); i += blockDim.x)
      prefetch_l2(next_w + i * 128);
  }
  if (warp == 4) {
    tmem_alloc(taddr_s, FZ_TMEM_COLS);
    tmem_relinquish();
  }
  // the dependents launch only once this CTA holds its columns (two CTAs of this kernel fill
  // an SM's shared memory, so their 2 x 256 columns never wait on each other)
  pdl_launch_dependents();
  const D2Smem<DL> m(scratch, p2.G, p2.KC);
  d2_stage<__nv_bfloat16, DL, 5>(p2, g, b, m);       // 5 x 256 loads: a group of 4 + 1 heads of 32
  tc_fence_before();
  __syncthreads();                                   // filters staged, TMEM address posted
  tc_fence_after();
  const uint32_t tmem = *taddr_s + ((static_cast<uint32_t>(warp & 3) * 32) << 16);
  pdl_wait();
  const int L = lengths[b];
  if (!filler) d2_load(p2, g, b, m, t, 128);         // shares the length's round trip
  if (L >= max_seq) {                                // cache full: o = 0, nothing appended
    if (tid == 0) report(p2.status, DEV_CACHE_FULL);
    for (int i = tid; i < G * DL; i += blockDim.x) {
      o_hi[(static_cast<size_t>(b) * H + g * G) * DL + i] = __float2bfloat16_rn(0.f);
      o_lo[(static_cast<size_t>(b) * H + g * G) * DL + i] = __float2bfloat16_rn(0.f);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
      tc_fence_after();
      tmem_dealloc(*taddr_s, FZ_TMEM_COLS);
    }
    return;
  }
  const int n = L;                                   // cache rows 0..L-1; row L is the new key
  const size_t row0 = (static_cast<size_t>(b) * Hkv + g) * max_seq;
  const int nsub = (n + TC_SUB - 1) / TC_SUB;
  const uint64_t stream_pol = l2_evict_first_policy();
  auto issue = [&](int sbi, int slot) {              // sub-chunk sbi into `slot` by this half's
    if (sbi < nsub) {                                // 128 threads; an empty group past the end
      const int base = sbi * TC_SUB, cnt = min(TC_SUB, n - base);  // rows past cnt: zeros
      __half *kd = ring + slot * SLOT, *vd = kd + TC_SUB * DL;
      for (int i = t; i < TC_SUB * CPR; i += 128) {
        const int r = i / CPR, j = i % CPR;
        const bool ok = r < cnt;
        const size_t src = (row0 + base + (ok ? r : 0)) * DL + j * 8;
        const int dst = r * DL + (j ^ kv_swz<CPR>(r)) * 8;
        cp_async16_zfill_stream(kd + dst, k_cache + src, ok, stream_pol);
        cp_async16_zfill_stream(vd + dst, v_cache + src, ok, stream_pol);
      }
    }
    cp_async_commit();
  };
  const int kb = (warp & 3) * WK;                    // the compute warp's first key in a sub-chunk

  if (filler) {
    // ---- park sub-chunks 0..NPARK-1 in TMEM; leave NPARK..NPARK+FREE-1 in slots 0..FREE-1
#pragma unroll
    for (int s = 0; s < FREE; ++s) issue(s, s);
    for (int i = 0; i < NPARK; ++i) {
      const int slot = i % FREE;
      cp_async_wait_group<FREE - 1>();               // sub-chunk i has landed (own copies)
      bar_sync(FZ_BAR_F, 128);                       // ... everyone's
      if (i < nsub) {
        const uint32_t ks_base = smem_u32(ring + slot * SLOT);
        const uint32_t vs_base = ks_base + TC_SUB * DL * 2;
        uint32_t w[FW];
#pragma unroll
        for (int m0 = 0; m0 < KW; m0 += 4) {         // K: the S = Q K^T B fragments
          const int id = m0 + (lane >> 3);
          const int nt = id / CPR, j = id % CPR;
          const int r = kb + nt * 8 + (lane & 7);
          ldsm_x4(ks_base + (r * DL + (j ^ kv_swz<CPR>(r)) * 8) * 2, w[m0], w[m0 + 1], w[m0 + 2],
                  w[m0 + 3]);
        }
#pragma unroll
        for (int kk = 0; kk < NT / 2; ++kk) {        // V: the O += P V B fragments
#pragma unroll
          for (int t0 = 0; t0 < DL / 8; t0 += 2) {
            const int id = lane >> 3;
            const int r = kb + kk * 16 + (id & 1) * 8 + (lane & 7);
            const int j = t0 + (id >> 1);
            const int o = KW + (kk * (DL / 16) + t0 / 2) * 4;
            ldsm_x4_t(vs_base + (r * DL + (j ^ kv_swz<CPR>(r)) * 8) * 2, w[o], w[o + 1], w[o + 2],
                      w[o + 3]);
          }
        }
#pragma unroll
        for (int c = 0; c < FW; c += 16) {
          uint32_t w16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) w16[e] = w[c + e];
          tmem_st16(tmem + i * FW + c, w16);
        }
        tmem_st_wait();
      }
      bar_sync(FZ_BAR_F, 128);                       // every filler is done with the slot
      issue(i + FREE, slot);                         // -> slot (i + FREE) % FREE == slot
      tc_fence_before();
      bar_arrive(FZ_BAR_TM + i, 256);                // sub-chunk i is in TMEM
    }
    cp_async_wait_group<0>();                        // the ring's sub-chunks have landed
    bar_sync(FZ_BAR_HO, 256);                        // ... and the compute warps are off TMEM
    if (warp == 4) {
      tc_fence_after();
      tmem_dealloc(*taddr_s, FZ_TMEM_COLS);
    }
    return;
  }

  // ---- compute warps: the stencil of the new token (the fillers stream meanwhile)
  d2_compute(p2, g, b, L, m, qn, t, 128, FZ_BAR_C, kvn);
  bar_sync(FZ_BAR_C, 128);                           // q, the new key and value are visible

  // Q fragments (rows = heads; a1, a3 are rows 8..15 and stay zero)
  uint32_t qa[DL / 16][2];
  {
    const float *qh = qn + gr * DL;
#pragma unroll
    for (int kk = 0; kk < DL / 16; ++kk) {
      float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
      if (gr < G) {
        v0 = qh[16 * kk + 2 * qd];
        v1 = qh[16 * kk + 2 * qd + 1];
        v2 = qh[16 * kk + 2 * qd + 8];
        v3 = qh[16 * kk + 2 * qd + 9];
      }
      qa[kk][0] = pack_f16x2(v0, v1);
      qa[kk][1] = pack_f16x2(v2, v3);
    }
  }
  float o[DL / 8][4];
#pragma unroll
  for (int u = 0; u < DL / 8; ++u) o[u][0] = o[u][1] = o[u][2] = o[u][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;              // of head row gr (lanes of one quad agree)

  // online softmax of row gr over this warp's keys of one sub-chunk; P as f16 A fragments
  auto softmax = [&](float (&sc)[NT][4], int valid, uint32_t (&pa)[NT / 2][2]) {
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        sc[nt][e] = nt * 8 + 2 * qd + e < valid ? sc[nt][e] * scale_log2 : -INFINITY;
        mx = fmaxf(mx, sc[nt][e]);
      }
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);            // finite: key kb of this slice is valid
    const float f = exp2f(m_run - m_new);            // 0 while m_run = -inf
    m_run = m_new;
    float ls = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float p0 = exp2f(sc[nt][0] - m_new), p1 = exp2f(sc[nt][1] - m_new);
      ls += p0 + p1;
      pa[nt / 2][nt & 1] = pack_f16x2(p0, p1);
    }
    l_run = l_run * f + ls;
#pragma unroll
    for (int u = 0; u < DL / 8; ++u) {
      o[u][0] *= f;
      o[u][1] *= f;
    }
  };

  // ---- the parked sub-chunks, fragments straight from TMEM
  for (int i = 0; i < NPARK; ++i) {
    bar_sync(FZ_BAR_TM + i, 256);
    tc_fence_after();
    const int valid = n - i * TC_SUB - kb;
    if (i < nsub && valid > 0) {
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int h = 0; h < KW; h += 16) {             // K words, 16 columns per load
        uint32_t kw[16];
        tmem_ld16(tmem + i * FW + h, kw);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const int idm = h + e, ntm = idm / CPR, kk = (idm % CPR) / 2;
          const uint32_t a[4] = {qa[kk][0], 0u, qa[kk][1], 0u};
          const uint32_t bb[2] = {kw[e], kw[e + 1]};
          mma_f16_16816(sc[ntm], a, bb);
        }
      }
      uint32_t pa[NT / 2][2];
      softmax(sc, valid, pa);
      constexpr int WPK = DL / 4;                    // V words per 16-key step
#pragma unroll
      for (int h = 0; h < KW; h += 16) {
        uint32_t vw[16];
        tmem_ld16(tmem + i * FW + KW + h, vw);
        tmem_ld_wait();
#pragma unroll
        for (int kk = h / WPK; kk < (h + 16) / WPK; ++kk) {
          const uint32_t a[4] = {pa[kk][0], 0u, pa[kk][1], 0u};
#pragma unroll
          for (int t0 = 0; t0 < DL / 8; t0 += 2) {
            const int w0 = kk * WPK + (t0 / 2) * 4 - h;
            const uint32_t b0[2] = {vw[w0], vw[w0 + 1]}, b1[2] = {vw[w0 + 2], vw[w0 + 3]};
            mma_f16_16816(o[t0], a, b0);
            mma_f16_16816(o[t0 + 1], a, b1);
          }
        }
      }
    }
  }
  tc_fence_before();
  bar_sync(FZ_BAR_HO, 256);                          // slots 0..FREE-1 hold sub-chunks NPARK..

  // ---- the rest through the ring: sub-chunk s >= NPARK in slot (s - NPARK) % NSLOT
#pragma unroll
  for (int s = 0; s < FREE; ++s) cp_async_commit();  // stand-ins for the fillers' groups
  for (int sbi = NPARK; sbi < nsub; ++sbi) {
    cp_async_wait_group<NSLOT - 2>();                // sub-chunk sbi has landed
    bar_sync(FZ_BAR_C, 128);                         // ... for every thread; and every warp
    issue(sbi + NSLOT - 1, (sbi + NSLOT - 1 - NPARK) % NSLOT);  // is done with that slot
    const uint32_t ks_base = smem_u32(ring + ((sbi - NPARK) % NSLOT) * SLOT);
    const uint32_t vs_base = ks_base + TC_SUB * DL * 2;
    const int valid = n - sbi * TC_SUB - kb;         // keys of this warp's slice that exist
    if (valid > 0) {
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int m0 = 0; m0 < KW; m0 += 4) {           // four (n-tile, piece) matrices per load
        const int id = m0 + (lane >> 3);
        const int nt = id / CPR, j = id % CPR;
        const int r = kb + nt * 8 + (lane & 7);
        uint32_t f[4];
        ldsm_x4(ks_base + (r * DL + (j ^ kv_swz<CPR>(r)) * 8) * 2, f[0], f[1], f[2], f[3]);
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const int idm = m0 + e, ntm = idm / CPR, kk = (idm % CPR) / 2;
          const uint32_t a[4] = {qa[kk][0], 0u, qa[kk][1], 0u};
          const uint32_t bb[2] = {f[e], f[e + 1]};
          mma_f16_16816(sc[ntm], a, bb);
        }
      }
      uint32_t pa[NT / 2][2];
      softmax(sc, valid, pa);
#pragma unroll
      for (int kk = 0; kk < NT / 2; ++kk) {
        const uint32_t a[4] = {pa[kk][0], 0u, pa[kk][1], 0u};
#pragma unroll
        for (int t0 = 0; t0 < DL / 8; t0 += 2) {      // two dim n-tiles (4 matrices) per load
          const int id = lane >> 3;
          const int r = kb + kk * 16 + (id & 1) * 8 + (lane & 7);
          const int j = t0 + (id >> 1);
          uint32_t f4[4];
          ldsm_x4_t(vs_base + (r * DL + (j ^ kv_swz<CPR>(r)) * 8) * 2, f4[0], f4[1], f4[2], f4[3]);
          const uint32_t b0[2] = {f4[0], f4[1]}, b1[2] = {f4[2], f4[3]};
          mma_f16_16816(o[t0], a, b0);
          mma_f16_16816(o[t0 + 1], a, b1);
        }
      }
    }
  }
  cp_async_wait_group<0>();                          // only empty groups can be left

  // ---- the new key's score per head, with q rounded to float16 as in the fragments
  for (int h = warp; h < G; h += 4) {
    float acc = 0.f;
    for (int i = lane; i < DL; i += 32)
      acc = fmaf(__half2float(__float2half_rn(qn[h * DL + i])), kvn[i], acc);
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) sn[h] = acc * scale_log2;
  }
  // ---- combine the four warps and the new key (one more partial: m = its score, l = 1)
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  constexpr int WS = DL + 2;
  if (gr < G) {
    float *w = wst + (warp * 8 + gr) * WS;
#pragma unroll
    for (int u = 0; u < DL / 8; ++u) {
      w[u * 8 + 2 * qd] = o[u][0];
      w[u * 8 + 2 * qd + 1] = o[u][1];
    }
    if (qd == 0) {
      w[DL] = m_run;
      w[DL + 1] = l_run;
    }
  }
  bar_sync(FZ_BAR_C, 128);
  for (int i = t; i < G * DL; i += 128) {
    const int h = i / DL, d = i % DL;
    float mw[4], M = sn[h];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      mw[w] = wst[(w * 8 + h) * WS + DL];
      M = fmaxf(M, mw[w]);
    }
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float c = mw[w] == -INFINITY ? 0.f : exp2f(mw[w] - M);
      acc = fmaf(c, wst[(w * 8 + h) * WS + d], acc);
      lsum = fmaf(c, wst[(w * 8 + h) * WS + DL + 1], lsum);
    }
    const float c = exp2f(sn[h] - M);
    acc = fmaf(c, kvn[DL + d], acc);
    lsum += c;
    const float v = acc / lsum;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const size_t idx = (static_cast<size_t>(b) * H + g * G) * DL + i;
    o_hi[idx] = hi;
    o_lo[idx] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
}

// ------------------------------------------------------------------ D3b merge (+ advance)
// One CTA per sequence: all (m, l) of its heads and chunks are staged in shared memory with
// one parallel load, then each thread (head, dim) combines its chunks' partial outputs.  The
// sequence's length advances here, after every kernel of the step that reads it.
__global__ void __launch_bounds__(512) decode_merge_kernel(
    const float *__restrict__ part_o, const float *__restrict__ part_ml, int *__restrict__ lengths,
    float *__restrict__ o, int H, int DL, int max_seq, int nchunk) {
  extern __shared__ float mls[];                      // [H][nused][2]
  const int b = blockIdx.x;
  const int L = lengths[b];
  const bool full = L >= max_seq;
  const int nused = full ? 0 : min(nchunk, (L + 1 + CHUNK - 1) / CHUNK);
  for (int i = threadIdx.x; i < H * nused * 2; i += blockDim.x) {
    const int h = i / (nused * 2), r = i % (nused * 2);
    mls[i] = part_ml[(static_cast<size_t>(b) * H + h) * nchunk * 2 + r];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < H * DL; i += blockDim.x) {
    const int h = i / DL, d = i % DL;
    const float *ml = mls + h * nused * 2;
    float mx = -INFINITY;
    for (int c = 0; c < nused; ++c) mx = fmaxf(mx, ml[2 * c]);
    const float *po = part_o + (static_cast<size_t>(b) * H + h) * nchunk * DL + d;
    float l = 0.f, acc = 0.f;
#pragma unroll 4
    for (int c = 0; c < nused; ++c) {
      const float w = exp2f(ml[2 * c] - mx);
      l = fmaf(w, ml[2 * c + 1], l);
      acc = fmaf(w, po[static_cast<size_t>(c) * DL], acc);
    }
    o[static_cast<size_t>(b) * H * DL + i] = nused > 0 ? acc / l : 0.f;
  }
  __syncthreads();
  if (threadIdx.x == 0 && !full) lengths[b] = L + 1;
}

// D3b for 16-bit layers: one CTA per (head, sequence), one thread per latent dim; the merged
// o is written as bfloat16 hi + lo terms (o = hi + lo to ~16 significand bits), the A operands
// of the D4 projection.
__global__ void __launch_bounds__(64) decode_merge16_kernel(
    const float *__restrict__ part_o, const float *__restrict__ part_ml,
    const int *__restrict__ lengths, __nv_bfloat16 *__restrict__ o_hi,
    __nv_bfloat16 *__restrict__ o_lo, int H, int DL, int max_seq, int chunk, int nchunk) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  if (d >= DL) return;
  const int L = lengths[b];
  const int nused = L >= max_seq ? 0 : min(nchunk, (L + 1 + chunk - 1) / chunk);
  const float *ml = part_ml + (static_cast<size_t>(b) * H + h) * nchunk * 2;
  const float *po = part_o + (static_cast<size_t>(b) * H + h) * nchunk * DL + d;
  float mx = -INFINITY;
  for (int c = 0; c < nused; ++c) mx = fmaxf(mx, ml[2 * c]);
  float l = 0.f, acc = 0.f;
#pragma unroll 4
  for (int c = 0; c < nused; ++c) {
    const float w = exp2f(ml[2 * c] - mx);
    l = fmaf(w, ml[2 * c + 1], l);
    acc = fmaf(w, po[static_cast<size_t>(c) * DL], acc);
  }
  const float v = nused > 0 ? acc / l : 0.f;
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  const size_t idx = (static_cast<size_t>(b) * H + h) * DL + d;
  o_hi[idx] = hi;
  o_lo[idx] = __float2bfloat16_rn(v - __bfloat162float(hi));
}

constexpr int kQkvBlocksPerSm = 1;   // QKV projection blocks per SM (split-K fills the rest)
constexpr int kQkvCols = 32;         // QKV projection columns per block

int decode_ksplit(const Dims &d) {
  // enough blocks to keep every SM streaming the weight matrix
  const int nblk = (d.NQKV + kQkvCols - 1) / kQkvCols;
  int ks = (kQkvBlocksPerSm * num_sms() + nblk - 1) / nblk;
  if (ks < 1) ks = 1;
  while (ks > 1 && d.E / ks < 64) --ks;
  return ks;
}

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

// Keys per split of the attention: 16-bit layers split each (sequence, group) only as far as
// needed for one CTA per SM (a batch with enough groups runs unsplit and skips the merge);
// float32 layers use fixed CHUNK-key splits.
int decode_chunk(const Dims &d, int max_seq) {
  if (!d.bf16) return CHUNK;
  const long units = static_cast<long>(d.B) * d.Hkv;
  const long nsplit = (num_sms() + units - 1) / units;
  const long per = (max_seq + nsplit - 1) / nsplit;
  return static_cast<int>((per + TC_SUB - 1) / TC_SUB * TC_SUB);
}

// 16-bit layers whose keys run unsplit and whose stencil scratch fits one slot of the
// attention's copy ring run the stencil inside the attention kernel.
static bool decode_fused(const Dims &d, int max_seq) {
  const int chunk = decode_chunk(d, max_seq);
  const int nchunk = (max_seq + chunk - 1) / chunk;
  if (!d.bf16 || nchunk != 1 || d.DL > 32) return false;
  const size_t slot_bytes = static_cast<size_t>(2) * TC_SUB * d.DL * 2;
  return d2_smem_floats(d.G, d.DL, d.KC) * 4 <= slot_bytes;
}

// projection, stencil, attention, output projection, and the merge of the attention's key
// splits (16-bit layers merge only when they split; float32 layers always run it); the
// stencil shares the attention's kernel where decode_fused says so
int decode_kernel_count(const Dims &d, int max_seq) {
  const int chunk = decode_chunk(d, max_seq);
  const int nchunk = (max_seq + chunk - 1) / chunk;
  if (decode_fused(d, max_seq)) return 3;
  return d.bf16 && nchunk == 1 ? 4 : 5;
}

size_t decode_workspace_bytes(const Dims &d, int max_seq) {
  const int nchunk = (max_seq + decode_chunk(d, max_seq) - 1) / decode_chunk(d, max_seq);
  const int ks = d.bf16 ? decode_ksplit(d) : 1;
  size_t s = 0;
  s += align256(static_cast<size_t>(ks) * d.B * d.NQKV * 4);
  s += align256(static_cast<size_t>(d.B) * d.H * d.DL * 4);
  s += align256(static_cast<size_t>(d.B) * d.H * nchunk * d.DL * 4);
  s += align256(static_cast<size_t>(d.B) * d.H * nchunk * 2 * 4);
  s += align256(static_cast<size_t>(d.B) * d.NQ * 4);
  return s;
}

void decode_workspace_carve(const Dims &d, int max_seq, void *ws, DecodeArgs &a) {
  const int chunk = decode_chunk(d, max_seq);
  const int nchunk = (max_seq + chunk - 1) / chunk;
  const int ks = d.bf16 ? decode_ksplit(d) : 1;
  char *p = static_cast<char *>(ws);
  a.p_part = reinterpret_cast<float *>(p);
  p += align256(static_cast<size_t>(ks) * d.B * d.NQKV * 4);
  a.q_new = reinterpret_cast<float *>(p);
  p += align256(static_cast<size_t>(d.B) * d.H * d.DL * 4);
  a.part_o = reinterpret_cast<float *>(p);
  p += align256(static_cast<size_t>(d.B) * d.H * nchunk * d.DL * 4);
  a.part_ml = reinterpret_cast<float *>(p);
  p += align256(static_cast<size_t>(d.B) * d.H * nchunk * 2 * 4);
  a.o = p;
  a.ksplit = ks;
  a.nchunk = nchunk;
  a.chunk = chunk;
}

template <int DL>
static cudaError_t launch_decode_tc(const Dims &d, const DecodeArgs &a, float scale_log2,
                                    cudaStream_t st) {
  const size_t smem = tc_smem_bytes<DL>();
  cudaError_t e = ensure_dyn_smem<decode_attn_tc_kernel<DL>>(smem);
  if (e != cudaSuccess) return e;
  __nv_bfloat16 *o_hi = static_cast<__nv_bfloat16 *>(a.o);
  return launch_pdl(decode_attn_tc_kernel<DL>, dim3(a.nchunk, d.Hkv, d.B), dim3(128),
                    smem, st, a.q_new, static_cast<const __half *>(a.k_cache),
                    static_cast<const __half *>(a.v_cache), a.lengths, a.part_o, a.part_ml, o_hi,
                    o_hi + static_cast<size_t>(d.B) * d.NQ, d.H, d.Hkv, d.G, a.max_seq, a.chunk,
                    a.nchunk, scale_log2, static_cast<const uint8_t *>(a.w_o),
                    static_cast<size_t>(d.E) * d.NQ * 2);
}

template <int DL>
static cudaError_t launch_decode_fused(const Dims &d, const DecodeArgs &a, float scale_log2,
                                       const D2Params<__nv_bfloat16> &p2, cudaStream_t st) {
  const size_t smem = fz_smem_bytes<DL>();
  cudaError_t e = ensure_dyn_smem<decode_attn_fused_kernel<DL>>(smem);
  if (e != cudaSuccess) return e;
  __nv_bfloat16 *o_hi = static_cast<__nv_bfloat16 *>(a.o);
  return launch_pdl(decode_attn_fused_kernel<DL>, dim3(1, d.Hkv, d.B), dim3(256), smem, st,
                    static_cast<const __half *>(a.k_cache), static_cast<const __half *>(a.v_cache),
                    a.lengths, o_hi, o_hi + static_cast<size_t>(d.B) * d.NQ, d.H, d.Hkv, d.G,
                    a.max_seq, scale_log2, static_cast<const uint8_t *>(a.w_o),
                    static_cast<size_t>(d.E) * d.NQ * 2, p2);
}

template <int DL, typename TL>
static cudaError_t launch_decode_attn(const Dims &d, const DecodeArgs &a, float scale_log2,
                                      const D2Params<__nv_bfloat16> *p2, cudaStream_t st) {
  if constexpr (sizeof(TL) == 2) {
    if (p2) {
      if constexpr (DL <= 32) return launch_decode_fused<DL>(d, a, scale_log2, *p2, st);
      return cudaErrorInvalidValue;
    }
    return launch_decode_tc<DL>(d, a, scale_log2, st);
  }
  const int KS = 128 / (DL / 2);
  const size_t smem = 4 * static_cast<size_t>(SUB) * DL * sizeof(TL) +
                      (static_cast<size_t>(d.G) * DL + static_cast<size_t>(d.G) * SUB +
                       static_cast<size_t>(KS) * d.G * DL + 3 * d.G) * 4;
  cudaError_t e = ensure_dyn_smem<decode_attn_kernel<DL, TL>>(smem);
  if (e != cudaSuccess) return e;
  decode_attn_kernel<DL, TL><<<dim3(a.nchunk, d.Hkv, d.B), 128, smem, st>>>(
      a.q_new, static_cast<const TL *>(a.k_cache), static_cast<const TL *>(a.v_cache), a.lengths,
      a.part_o, a.part_ml, d.H, d.Hkv, d.G, a.max_seq, a.nchunk, scale_log2);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t decode_typed(const Dims &d, const DecodeArgs &a, cudaStream_t st,
                                const StageMarker &mark) {
  cudaError_t e;
  // D1
  if constexpr (sizeof(T) == 2) {
    e = launch_skinny<true, false, 8, kQkvCols>(
        a.ksplit, static_cast<const __nv_bfloat16 *>(a.x), nullptr,
        static_cast<const __nv_bfloat16 *>(a.w_qkv), a.p_part, d.B, d.NQKV, d.E, nullptr, 0, st);
    if (e != cudaSuccess) return e;
  } else {
    e = gemm_simt(0, a.x, a.w_qkv, a.p_part, d.B, d.NQKV, d.E, st);
    if (e != cudaSuccess) return e;
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  mark();
  // D2
  using TL = typename LatentType<T>::type;
  D2Params<T> p2;
  p2.p_part = a.p_part;
  p2.ksplit = sizeof(T) == 2 ? a.ksplit : 1;
  p2.conv_seq = a.conv_seq;
  p2.conv_chan = a.conv_chan;
  p2.k_cache = static_cast<TL *>(a.k_cache);
  p2.v_cache = static_cast<TL *>(a.v_cache);
  p2.conv_state = a.conv_state;
  p2.vshift_state = a.vshift_state;
  p2.lengths = a.lengths;
  p2.status = a.status;
  p2.q_new = a.q_new;
  p2.B = d.B; p2.H = d.H; p2.Hkv = d.Hkv; p2.G = d.G; p2.DL = d.DL;
  p2.NQ = d.NQ; p2.NKV = d.NKV; p2.NQKV = d.NQKV; p2.KC = d.KC; p2.VS0 = d.VS0;
  p2.max_seq = a.max_seq;
  p2.flags = d.flags;
  p2.eps = d.eps;
  for (int i = 0; i < d.DL / 2; ++i)
    p2.theta[i] = pow(static_cast<double>(d.rope_base), -2.0 * i / d.DL);
  const bool fused = decode_fused(d, a.max_seq);
  if (!fused) {
    const size_t sm2 = d2_smem_floats(d.G, d.DL, d.KC) * 4;
    auto d2 = d.DL == 16 ? decode_stencil_kernel<T, 16>
                         : (d.DL == 32 ? decode_stencil_kernel<T, 32> : decode_stencil_kernel<T, 64>);
    if (sm2 > 48 * 1024) {
      e = d.DL == 16 ? ensure_dyn_smem<decode_stencil_kernel<T, 16>>(sm2)
                     : (d.DL == 32 ? ensure_dyn_smem<decode_stencil_kernel<T, 32>>(sm2)
                                   : ensure_dyn_smem<decode_stencil_kernel<T, 64>>(sm2));
      if (e != cudaSuccess) return e;
    }
    if ((e = launch_pdl(d2, dim3(d.Hkv, d.B), dim3(256), sm2, st, p2)) != cudaSuccess) return e;
    mark();
  }
  // D3 (with D2 inside when fused)
  const float scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(d.DL)));
  const D2Params<__nv_bfloat16> *p2f = nullptr;
  if constexpr (sizeof(T) == 2) p2f = fused ? &p2 : nullptr;
  if (d.DL == 16) e = launch_decode_attn<16, TL>(d, a, scale_log2, p2f, st);
  else if (d.DL == 32) e = launch_decode_attn<32, TL>(d, a, scale_log2, p2f, st);
  else e = launch_decode_attn<64, TL>(d, a, scale_log2, p2f, st);
  if (e != cudaSuccess) return e;
  mark();
  // D3b (+ lengths advance for float32 layers; the 16-bit D4 advances them)
  if constexpr (sizeof(T) == 2) {
    if (a.nchunk > 1) {                              // an unsplit attention wrote o itself
      __nv_bfloat16 *o_hi = static_cast<__nv_bfloat16 *>(a.o);
      e = launch_pdl(decode_merge16_kernel, dim3(d.H, d.B), dim3(d.DL < 32 ? 32 : d.DL), 0, st,
                     a.part_o, a.part_ml, a.lengths, o_hi, o_hi + static_cast<size_t>(d.B) * d.NQ,
                     d.H, d.DL, a.max_seq, a.chunk, a.nchunk);
      if (e != cudaSuccess) return e;
      mark();
    }
  } else {
    const int nused_max = a.nchunk;
    const size_t smm = static_cast<size_t>(d.H) * nused_max * 2 * 4;
    if (smm > 48 * 1024) {
      e = ensure_dyn_smem<decode_merge_kernel>(smm);
      if (e != cudaSuccess) return e;
    }
    const int threads = d.H * d.DL < 512 ? ((d.H * d.DL + 31) / 32) * 32 : 512;
    decode_merge_kernel<<<d.B, threads, smm, st>>>(a.part_o, a.part_ml, a.lengths,
                                                   static_cast<float *>(a.o), d.H, d.DL,
                                                   a.max_seq, a.nchunk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark();
  }
  // D4 (+ lengths advance for 16-bit layers)
  if constexpr (sizeof(T) == 2) {
    const __nv_bfloat16 *o_hi = static_cast<const __nv_bfloat16 *>(a.o);
    e = launch_skinny<false, true, 8, 16>(1, o_hi, o_hi + static_cast<size_t>(d.B) * d.NQ,
                                          static_cast<const __nv_bfloat16 *>(a.w_o), a.y, d.B,
                                          d.E, d.NQ, a.lengths, a.max_seq, st);
    if (e != cudaSuccess) return e;
  } else {
    e = gemm_simt(0, a.o, a.w_o, a.y, d.B, d.E, d.NQ, st);
    if (e != cudaSuccess) return e;
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  mark();
  return cudaSuccess;
}

cudaError_t decode_step(const Dims &d, const DecodeArgs &a, cudaStream_t st,
                        const StageMarker &mark) {
  if (d.B == 0) return cudaSuccess;
  return d.bf16 ? decode_typed<__nv_bfloat16>(d, a, st, mark) : decode_typed<float>(d, a, st, mark);
}

}  // namespace cca
