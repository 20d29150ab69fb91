// Down-projection fused with the latent stencil for 16-bit layers: P = x W_qkv^T never
// leaves the SM.  (gist.science explainer, 2. Methodology, Core Mechanism: down-projection,
// convolutional mixing, Q-K-Mean, Value-Shift, normalisation and RoPE; 3. Key Contributions:
// the convolutions fused into the attention pipeline's kernels.)
//
// A persistent CTA is bound to a set of NG consecutive key/value groups for its whole life and
// walks a contiguous run of (sequence, tile) units.  A tile is 128 consecutive tokens of one
// sequence, the first HALO (= max(conv_kernel - 1, 1)) of which only feed the causal
// convolution and the value-shift of the next ones: tiles overlap by HALO rows, and each
// writes 128 - HALO tokens.  Per tile:
//   warp 0     TMA producer: x rows [t0 - HALO, t0 + 128 - HALO) of the sequence (rows outside
//              the sequence read as zero, the convolution's zero padding) and the group set's
//              W_q / W_k / W_v rows, 32 columns of K per stage, 4 stages (64-byte swizzle).
//   warp 1     TMEM (512 columns) and all MMAs: P[128 x N] = x W^T into columns [0, N)
//              (N = NG (G + 2) d~ <= 384, one or two tcgen05.mma per K step); then per
//              query / key head the channel conv C[128 x d~] = A W_c^T into columns
//              [384, 384 + d~), with A and W_c split into bfloat16 leading terms and
//              remainders (A_hi W_hi + A_lo W_hi + A_hi W_lo, about 16 significand bits); the
//              filters of each head stream in by TMA through a two-deep buffer.
//   warps 2-9  epilogue, one token row per thread (the TMEM lane quadrant of its warp), two
//              warps per row each on half of every head's columns:
//              values with the value-shift (the previous token's row through shared memory),
//              then per head: the causal sequence conv of P's columns (rows exchanged through
//              shared memory), A written as hi / lo bfloat16 in the MMA's swizzled layout, the
//              channel conv's result read back, Q-K-Mean from P's pre-conv columns, RMS norm
//              and RoPE in registers, float16 stores of q, k, v, and the decode state of the
//              sequence's last tokens.
// The accumulator is single-buffered: the next tile's MMAs start once the epilogue has read
// every P column it needs (its TMA loads run ahead meanwhile).  Every wait is bounded; on a
// timeout the CTA records it in the status word, stops and releases its tensor memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int FM = 128;            // rows (tokens, halo included) per tile
constexpr int FBK = 32;            // K columns per stage: 64-byte rows
constexpr int FST = 4;             // stages
constexpr int FN_MAX = 384;        // accumulator columns
constexpr uint32_t FCONV0 = 384;   // TMEM column of the channel-conv result
constexpr int F_EPI_WARPS = 8;     // two per TMEM lane quadrant, each on half of a head's columns
constexpr int F_THREADS = 64 + 32 * F_EPI_WARPS;
constexpr int XS_LD = 17;          // row stride (floats) of a half's row-exchange buffer

struct FusedParams {
  const float *conv_seq;
  __half *q, *k, *v;
  float *conv_state, *vshift_state;
  int *lengths;
  int *status;
  int write_state;
  int B, S, E, H, Hkv, G, NQ, NKV, KC, HALO, VS0, kv_stride;
  int NG, N, nsets, cps, units_per_seq;
  unsigned flags;
  float eps;
  double theta[32];                // RoPE frequencies base^(-2i/d~), i < d~/2
};

struct FusedBars {
  uint64_t full[FST], empty[FST];
  uint64_t acc_full, acc_empty, a_ready, conv_done;
  uint64_t filt_full[2];
  uint32_t tmem_base;
  int abort;
};

// Shared-memory carve (bytes), the same on host and device.
struct FusedSmem {
  int stage_bytes, off_filt, off_abuf, off_xs, off_taps, off_bars, total;
};
__host__ __device__ inline FusedSmem fused_smem(int DL, int N, int NG, int G, int KC) {
  FusedSmem m;
  m.stage_bytes = FM * FBK * 2 + N * FBK * 2;
  int off = FST * m.stage_bytes;
  m.off_filt = off;                              // 2 buffers x {hi, lo} x [d~ x d~] bf16
  off += 4 * DL * DL * 2;
  off = (off + 1023) & ~1023;
  m.off_abuf = off;                              // {hi, lo} x [128 x d~] bf16
  off += 2 * FM * DL * 2;
  m.off_xs = off;                                // one exchange buffer per half, then the
  off += 2 * FM * XS_LD * 4 + 2 * FM * 4;        // halves' norm partial sums
  m.off_taps = off;
  off += NG * (G + 1) * DL * KC * 4;
  off = (off + 15) & ~15;
  m.off_bars = off;
  off += static_cast<int>(sizeof(FusedBars));
  m.total = off + 1024;                          // slack for the 1024-byte alignment
  return m;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void epi_sync() {   // all eight epilogue warps
  asm volatile("bar.sync 1, 256;" ::: "memory");
}
__device__ __forceinline__ void half_sync(int hf) {   // the four epilogue warps of one half
  asm volatile("bar.sync %0, 128;" ::"r"(2 + hf) : "memory");
}
// Byte offset of 16-byte chunk j of row r in a K-major tile with ROWB-byte rows, in the
// 128/64/32-byte swizzled layout that TMA writes and tcgen05.mma reads (ROWB = 128, 64, 32).
template <int ROWB>
__device__ __forceinline__ uint32_t swz_off(int r, int j) {
  constexpr uint32_t BB = ROWB == 128 ? 3 : ROWB == 64 ? 2 : 1;
  const uint32_t o = static_cast<uint32_t>(r) * ROWB + static_cast<uint32_t>(j) * 16;
  return o ^ (((o >> 7) & ((1u << BB) - 1)) << 4);
}
template <int ROWB>
__host__ __device__ constexpr uint32_t swz_mode() {
  return ROWB == 128 ? 2u : ROWB == 64 ? 4u : 6u;
}

template <int W>
__device__ __forceinline__ void tmem_ldw(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 32) tmem_ld32(taddr, r);
  else if constexpr (W == 16) tmem_ld16(taddr, r);
  else if constexpr (W == 8) tmem_ld8(taddr, r);
  else tmem_ld4(taddr, r);
}
// Stores Q (16, 8 or 4) consecutive 16-bit values, as pairs in v, at the 2-byte-aligned dst.
template <int Q>
__device__ __forceinline__ void store_halves(__half *dst, const uint32_t (&v)[Q / 2]) {
  if constexpr (Q == 16) {
    reinterpret_cast<uint4 *>(dst)[0] = make_uint4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<uint4 *>(dst)[1] = make_uint4(v[4], v[5], v[6], v[7]);
  } else if constexpr (Q == 8) {
    *reinterpret_cast<uint4 *>(dst) = make_uint4(v[0], v[1], v[2], v[3]);
  } else {
    *reinterpret_cast<uint2 *>(dst) = make_uint2(v[0], v[1]);
  }
}

template <int DL>
__global__ void __launch_bounds__(F_THREADS, 1)
    qkv_stencil_kernel(const __grid_constant__ CUtensorMap mapX,
                       const __grid_constant__ CUtensorMap mapWq,
                       const __grid_constant__ CUtensorMap mapWkv,
                       const __grid_constant__ CUtensorMap mapFhi,
                       const __grid_constant__ CUtensorMap mapFlo, const FusedParams p) {
  constexpr int CW = DL < 32 ? DL : 32;            // columns per TMEM load / exchange chunk
  constexpr int NCH = DL / CW;
  constexpr int ROWB = DL * 2;                     // bytes per row of A and of the filters
  constexpr int HALF = DL / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int G = p.G, NG = p.NG, N = p.N, KC = p.KC, HALO = p.HALO;
  const FusedSmem L = fused_smem(DL, N, NG, G, KC);
  FusedBars *bars = reinterpret_cast<FusedBars *>(smem + L.off_bars);
  float *xs = reinterpret_cast<float *>(smem + L.off_xs);
  float *taps = reinterpret_cast<float *>(smem + L.off_taps);
  uint8_t *abuf = smem + L.off_abuf;               // hi then lo
  uint8_t *filt = smem + L.off_filt;               // buffer f: hi at 2f, lo at 2f + 1
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // this CTA's group set and run of (sequence, tile) units
  const int gs = blockIdx.x / p.cps, ci = blockIdx.x % p.cps;
  const int nunits = p.B * p.units_per_seq;
  const int u_beg = static_cast<int>(static_cast<long long>(nunits) * ci / p.cps);
  const int u_end = static_cast<int>(static_cast<long long>(nunits) * (ci + 1) / p.cps);
  const int TOUT = FM - HALO;
  const int qrow0 = gs * NG * G * DL, krow0 = p.NQ + gs * NG * DL, vrow0 = p.NQ + p.NKV + gs * NG * DL;
  const int nheads = NG * (G + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < FST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, F_EPI_WARPS);
    mbar_init(&bars->a_ready, F_EPI_WARPS);
    mbar_init(&bars->conv_done, 1);
    mbar_init(&bars->filt_full[0], 1);
    mbar_init(&bars->filt_full[1], 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  // the sequence-conv taps of the group set's query and key channels (CTA-local channel lc:
  // the NG*G*d~ query channels, then the NG*d~ key channels)
  for (int i = threadIdx.x; i < nheads * DL * KC; i += blockDim.x) {
    const int lc = i / KC, tap = i % KC;
    const int gc = lc < NG * G * DL ? qrow0 + lc : p.NQ + gs * NG * DL + (lc - NG * G * DL);
    taps[i] = p.conv_seq[static_cast<size_t>(gc) * KC + tap];
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int *abort = &bars->abort;
  int *status = p.status;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&mapX);
      tma_prefetch_desc(&mapWq);
      tma_prefetch_desc(&mapWkv);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = u_beg; ok && u < u_end; ++u) {
        const int b = u / p.units_per_seq, t0 = (u % p.units_per_seq) * TOUT;
        for (int k0 = 0; k0 < p.E; k0 += FBK) {
          if (!mbar_wait(&bars->empty[stage], phase ^ 1u, abort, status)) { ok = false; break; }
          uint8_t *st = smem + stage * L.stage_bytes;
          mbar_arrive_expect_tx(&bars->full[stage], L.stage_bytes);
          tma_load_3d(st, &mapX, &bars->full[stage], k0, t0 - HALO, b);
          uint8_t *bs = st + FM * FBK * 2;
          tma_load_2d(bs, &mapWq, &bars->full[stage], k0, qrow0);
          tma_load_2d(bs + NG * G * DL * FBK * 2, &mapWkv, &bars->full[stage], k0, krow0);
          tma_load_2d(bs + (NG * G * DL + NG * DL) * FBK * 2, &mapWkv, &bars->full[stage], k0, vrow0);
          if (++stage == FST) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const int N0 = N < 256 ? N : 256, N1 = N - N0;
      const uint32_t idesc0 = idesc_f16_f32(FM, N0, 0, 0, 0);
      const uint32_t idesc1 = idesc_f16_f32(FM, N1 > 0 ? N1 : 16, 0, 0, 0);
      constexpr uint32_t idesc_c = idesc_f16_f32(FM, DL, 0, 0, 0);
      constexpr uint32_t SWC = swz_mode<ROWB>();
      constexpr uint32_t FPLANE = DL * DL * 2;
      const uint32_t filt_tx = 2 * FPLANE;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t fload = 0, fuse = 0, areads = 0;       // filter loads issued / used, A hand-offs
      auto head_glob = [&](int hidx) {                // conv_chan head of CTA-local head hidx
        const int gi = hidx / (G + 1), hh = hidx % (G + 1);
        return hh < G ? (gs * NG + gi) * G + hh : p.H + gs * NG + gi;
      };
      auto load_filter = [&](int hidx) {
        const int f = fload & 1;
        mbar_arrive_expect_tx(&bars->filt_full[f], filt_tx);
        tma_load_2d(filt + (2 * f) * FPLANE, &mapFhi, &bars->filt_full[f], 0, head_glob(hidx) * DL);
        tma_load_2d(filt + (2 * f + 1) * FPLANE, &mapFlo, &bars->filt_full[f], 0, head_glob(hidx) * DL);
        ++fload;
      };
      tma_prefetch_desc(&mapFhi);
      tma_prefetch_desc(&mapFlo);
      int local = 0;
      for (int u = u_beg; ok && u < u_end; ++u, ++local) {
        load_filter(0);
        if (nheads > 1) load_filter(1);
        if (!mbar_wait(&bars->acc_empty, (local & 1) ^ 1u, abort, status)) break;
        tc_fence_after();
        for (int kb = 0; kb * FBK < p.E; ++kb) {
          if (!mbar_wait(&bars->full[stage], phase, abort, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * L.stage_bytes);
          const uint32_t b_addr = a_addr + FM * FBK * 2;
#pragma unroll
          for (int ks = 0; ks < FBK / 16; ++ks) {
            const uint64_t ad = smem_desc(a_addr + ks * 32, 16, 512, 4);
            const uint64_t bd = smem_desc(b_addr + ks * 32, 16, 512, 4);
            umma_f16_ss(tmem, ad, bd, idesc0, (kb > 0 || ks > 0) ? 1u : 0u);
            if (N1 > 0) {
              const uint64_t bd1 = smem_desc(b_addr + 256 * FBK * 2 + ks * 32, 16, 512, 4);
              umma_f16_ss(tmem + 256, ad, bd1, idesc1, (kb > 0 || ks > 0) ? 1u : 0u);
            }
          }
          umma_commit(&bars->empty[stage]);
          if (++stage == FST) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&bars->acc_full);
        // the channel conv of each query / key head, as the epilogue hands A over
        for (int hidx = 0; ok && hidx < nheads; ++hidx) {
          if (!mbar_wait(&bars->a_ready, areads & 1, abort, status)) { ok = false; break; }
          ++areads;
          const int f = fuse & 1;
          if (!mbar_wait(&bars->filt_full[f], (fuse >> 1) & 1, abort, status)) { ok = false; break; }
          ++fuse;
          tc_fence_after();
          const uint32_t ahi = smem_u32(abuf), alo = ahi + FM * ROWB;
          const uint32_t whi = smem_u32(filt + (2 * f) * FPLANE), wlo = whi + FPLANE;
#pragma unroll
          for (int ks = 0; ks < DL / 16; ++ks) {
            const uint64_t dah = smem_desc(ahi + ks * 32, 16, 8 * ROWB, SWC);
            const uint64_t dal = smem_desc(alo + ks * 32, 16, 8 * ROWB, SWC);
            const uint64_t dwh = smem_desc(whi + ks * 32, 16, 8 * ROWB, SWC);
            const uint64_t dwl = smem_desc(wlo + ks * 32, 16, 8 * ROWB, SWC);
            umma_f16_ss(tmem + FCONV0, dah, dwh, idesc_c, ks > 0 ? 1u : 0u);
            umma_f16_ss(tmem + FCONV0, dal, dwh, idesc_c, 1u);
            umma_f16_ss(tmem + FCONV0, dah, dwl, idesc_c, 1u);
          }
          umma_commit(&bars->conv_done);
          // the filter buffer and A are free once these MMAs are done
          if (!mbar_wait(&bars->conv_done, (areads - 1) & 1, abort, status)) { ok = false; break; }
          if (hidx + 2 < nheads) load_filter(hidx + 2);
        }
      }
      // drain: filter loads issued but never consumed (an early exit) are waited out
      while (fuse < fload) {
        const int f = fuse & 1;
        if (!mbar_wait(&bars->filt_full[f], (fuse >> 1) & 1, abort, status)) break;
        ++fuse;
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue warps 2-9
    // Two warps per TMEM lane quadrant; half hf of a head's d~ columns belongs to the warps
    // (2 + 4 hf .. 5 + 4 hf): columns [hf Q, hf Q + Q) and [d~/2 + hf Q, d~/2 + hf Q + Q) with
    // Q = d~/4, so both members of every RoPE pair (i, i + d~/2) stay with one thread.  Rows are
    // exchanged within a half (its own buffer and named barrier); the halves meet at the MMA
    // hand-off and for the norm's sum of squares.
    constexpr int Q = DL / 4;
    const int quad = warp & 3, hf = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tP = tmem + lane_off, tC = tmem + FCONV0 + lane_off;
    uint8_t *ahi = abuf, *alo = abuf + FM * ROWB;
    float *xh = xs + hf * FM * XS_LD;                 // this half's exchange buffer
    float *nrm = xs + 2 * FM * XS_LD;                 // [half][row] partial sums of squares
    // A failed (timed-out) wait sets the CTA's abort flag, after which every wait returns at
    // once; the epilogue still runs its whole loop so that its warps meet at every named
    // barrier, and only its stores are skipped.
    int local = 0;
    uint32_t convs = 0;
    bool ok = true;
    for (int u = u_beg; u < u_end; ++u, ++local) {
      const int b = u / p.units_per_seq, t0 = (u % p.units_per_seq) * TOUT;
      const int t = t0 - HALO + row;                  // this row's token
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->acc_full, local & 1, abort, status)) && ok;
      const bool out = ok && row >= HALO && t < p.S;
      const bool last_tile = ok && p.write_state && t0 <= p.S - 1 && p.S - 1 < t0 + TOUT;
      const bool last_tok = last_tile && t == p.S - 1;
      const int ts = out ? t : 0;                     // a row of the tensors for address math
      tc_fence_after();
      // ---- values, with the value-shift (the previous row's value through shared memory);
      // this half takes the columns [hf d~/2, (hf+1) d~/2), Q at a time
      for (int gi = 0; gi < NG; ++gi) {
        const int g = gs * NG + gi;
        const int vcol = NG * G * DL + NG * DL + gi * DL;
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          const int c0 = hf * (DL / 2) + blk * Q;
          uint32_t r[Q];
          tmem_ldw<Q>(tP + vcol + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < Q; ++j) xh[row * XS_LD + j] = __uint_as_float(r[j]);
          half_sync(hf);
          uint32_t pk[Q / 2];
          bool fits = true;
#pragma unroll
          for (int j = 0; j < Q; j += 2) {
            float val[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int gvc = g * DL + c0 + j + e;
              const bool shifted = (p.flags & F_VALUE_SHIFT) && gvc >= p.VS0;
              val[e] = shifted ? (row > 0 ? xh[(row - 1) * XS_LD + j + e] : 0.f) : __uint_as_float(r[j + e]);
              if (last_tok && gvc >= p.VS0)
                p.vshift_state[static_cast<size_t>(b) * (p.NKV - p.VS0) + (gvc - p.VS0)] = __uint_as_float(r[j + e]);
            }
            fits &= fabsf(val[0]) <= kF16Max && fabsf(val[1]) <= kF16Max;
            pk[j / 2] = pack_f16x2(val[0], val[1]);
          }
          if (out) {
            store_halves<Q>(p.v + ((static_cast<size_t>(b) * p.Hkv + g) * p.kv_stride + ts) * DL + c0, pk);
            if (!fits) report(status, DEV_RANGE);
          }
          half_sync(hf);
        }
      }
      // ---- query and key heads
      for (int hidx = 0; hidx < nheads; ++hidx) {
        const int gi = hidx / (G + 1), hh = hidx % (G + 1);
        const int g = gs * NG + gi;
        const bool is_q = hh < G;
        const int pcol = is_q ? (gi * G + hh) * DL : NG * G * DL + gi * DL;     // P column
        const int kcol = NG * G * DL + gi * DL;                                  // its k head
        const int gch = is_q ? (g * G + hh) * DL : p.NQ + g * DL;             // q|k channel
        // sequence conv of this half's two column blocks, into A (hi / lo) in the MMA's layout
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          const int c0 = blk * (DL / 2) + hf * Q;
          uint32_t r[Q];
          tmem_ldw<Q>(tP + pcol + c0, r);
          tmem_ld_wait();
          if (last_tile && t >= p.S - (KC - 1) && t >= 0 && t < p.S) {   // the last KC-1 tokens
            float *cs = p.conv_state + (static_cast<size_t>(b) * (KC - 1) + (t - (p.S - KC + 1))) *
                                           (p.NQ + p.NKV);
#pragma unroll
            for (int j = 0; j < Q; ++j) cs[gch + c0 + j] = __uint_as_float(r[j]);
          }
#pragma unroll
          for (int j = 0; j < Q; ++j) xh[row * XS_LD + j] = __uint_as_float(r[j]);
          half_sync(hf);
          float a[Q];
#pragma unroll
          for (int j = 0; j < Q; ++j) a[j] = 0.f;
          for (int tap = 0; tap < KC; ++tap) {
            const int rr = max(row - (KC - 1) + tap, 0);
            const float *tp = taps + (pcol + c0) * KC + tap;
#pragma unroll
            for (int j = 0; j < Q; ++j) a[j] = fmaf(tp[j * KC], xh[rr * XS_LD + j], a[j]);
          }
          uint32_t hi[Q / 2], lo[Q / 2];
#pragma unroll
          for (int j = 0; j < Q; j += 2) split_bf16x2(make_float2(a[j], a[j + 1]), hi[j / 2], lo[j / 2]);
          if constexpr (Q >= 8) {
#pragma unroll
            for (int q8 = 0; q8 < Q / 8; ++q8) {
              const uint32_t o = swz_off<ROWB>(row, c0 / 8 + q8);
              *reinterpret_cast<uint4 *>(ahi + o) = make_uint4(hi[4 * q8], hi[4 * q8 + 1], hi[4 * q8 + 2], hi[4 * q8 + 3]);
              *reinterpret_cast<uint4 *>(alo + o) = make_uint4(lo[4 * q8], lo[4 * q8 + 1], lo[4 * q8 + 2], lo[4 * q8 + 3]);
            }
          } else {                                     // 4 columns: half of a 16-byte piece
            const uint32_t o = swz_off<ROWB>(row, c0 / 8) + (c0 % 8) * 2;
            *reinterpret_cast<uint2 *>(ahi + o) = make_uint2(hi[0], hi[1]);
            *reinterpret_cast<uint2 *>(alo + o) = make_uint2(lo[0], lo[1]);
          }
          half_sync(hf);                               // xh is rewritten by the next block
        }
        fence_proxy_async_smem();                      // A visible to the tensor cores
        tc_fence_before();
        epi_sync();
        if (lane == 0) mbar_arrive(&bars->a_ready);
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->conv_done, convs & 1, abort, status)) && ok;
        ++convs;
        tc_fence_after();
        float uu[2 * Q];                               // [low block | high block]
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          const int c0 = blk * (DL / 2) + hf * Q;
          uint32_t r[Q];
          tmem_ldw<Q>(tC + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < Q; ++j) uu[blk * Q + j] = __uint_as_float(r[j]);
        }
        if (p.flags & F_QK_MEAN) {                     // + (pre-conv q + pre-conv k) / 2
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {
            const int c0 = blk * (DL / 2) + hf * Q;
            uint32_t rk[Q], rq[Q];
            tmem_ldw<Q>(tP + kcol + c0, rk);
            float mq[Q];
            if (is_q) {
              tmem_ldw<Q>(tP + pcol + c0, rq);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < Q; ++j) mq[j] = __uint_as_float(rq[j]);
            } else {
#pragma unroll
              for (int j = 0; j < Q; ++j) mq[j] = 0.f;
              for (int h2 = 0; h2 < G; ++h2) {
                tmem_ldw<Q>(tP + (gi * G + h2) * DL + c0, rq);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < Q; ++j) mq[j] += __uint_as_float(rq[j]);
              }
#pragma unroll
              for (int j = 0; j < Q; ++j) mq[j] /= static_cast<float>(G);
            }
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < Q; ++j) uu[blk * Q + j] += 0.5f * (mq[j] + __uint_as_float(rk[j]));
          }
        }
        if (hidx == nheads - 1) {                      // every P column this tile needs is read
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->acc_empty);
        }
        if (p.flags & F_QK_NORM) {
          float ss = 0.f;
#pragma unroll
          for (int i = 0; i < 2 * Q; ++i) ss += uu[i] * uu[i];
          nrm[hf * FM + row] = ss;
          epi_sync();
          ss = nrm[row] + nrm[FM + row];
          const float inv = 1.0f / sqrtf(ss / static_cast<float>(DL) + p.eps);
#pragma unroll
          for (int i = 0; i < 2 * Q; ++i) uu[i] *= inv;
        }
        if ((p.flags & F_ROPE) && out) {
#pragma unroll
          for (int j = 0; j < Q; ++j) {
            float cs, sn;
            rope_cos_sin(static_cast<double>(t) * p.theta[hf * Q + j], cs, sn);
            const float x1 = uu[j], x2 = uu[Q + j];
            uu[j] = x1 * cs - x2 * sn;
            uu[Q + j] = x1 * sn + x2 * cs;
          }
        }
        if (out && ok) {
          __half *dst = is_q ? p.q + ((static_cast<size_t>(b) * p.H + g * G + hh) * p.S + t) * DL
                             : p.k + ((static_cast<size_t>(b) * p.Hkv + g) * p.kv_stride + t) * DL;
          bool fits = true;
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {
            uint32_t pk[Q / 2];
#pragma unroll
            for (int j = 0; j < Q; j += 2) {
              pk[j / 2] = pack_f16x2(uu[blk * Q + j], uu[blk * Q + j + 1]);
              fits &= fabsf(uu[blk * Q + j]) <= kF16Max && fabsf(uu[blk * Q + j + 1]) <= kF16Max;
            }
            store_halves<Q>(dst + blk * (DL / 2) + hf * Q, pk);
          }
          if (!fits) report(status, DEV_RANGE);
        }
      }
      if (last_tile && gs == 0 && row == HALO && hf == 0) p.lengths[b] = p.S;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

__global__ void split_planes_kernel(const float *__restrict__ w, __nv_bfloat16 *__restrict__ hi,
                                    __nv_bfloat16 *__restrict__ lo, size_t n) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float v = w[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

}  // namespace

int fused_group_set(const Dims &d) {
  if (!d.bf16 || (d.flags & F_NO_CONV)) return 0;
  if (d.DL != 16 && d.DL != 32 && d.DL != 64) return 0;
  if (d.KC < 1 || d.KC > 8 || d.E % FBK) return 0;
  const int per = (d.G + 2) * d.DL;
  int best = 0;
  for (int ng = 1; ng <= d.Hkv; ng *= 2) {
    if (d.Hkv % ng) break;
    if (ng * per > FN_MAX || ng * d.G * d.DL > 256) break;
    best = ng;
  }
  if (!best) return 0;
  if (fused_smem(d.DL, best * per, best, d.G, d.KC).total > 227 * 1024) return 0;
  return best;
}

size_t fused_filter_bytes(const Dims &d) {
  return static_cast<size_t>(d.H + d.Hkv) * d.DL * d.DL * 2 * 2;
}

template <int DL>
static cudaError_t launch_fused(const Dims &d, const FusedArgs &a, int NG, cudaStream_t st) {
  const int N = NG * (d.G + 2) * DL;
  const int HALO = d.KC - 1 > 1 ? d.KC - 1 : 1;
  CUtensorMap mx, mwq, mwkv, mfh, mfl;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(d.E), static_cast<uint64_t>(d.S),
                              static_cast<uint64_t>(d.B)};
    const uint64_t strides[2] = {static_cast<uint64_t>(d.E) * 2,
                                 static_cast<uint64_t>(d.E) * 2 * d.S};
    const uint32_t box[3] = {FBK, FM, 1};
    if (!make_tma_16bit(&mx, a.x, 3, dims, strides, box, 64, 0)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(d.E), static_cast<uint64_t>(d.NQKV)};
    const uint64_t strides[1] = {static_cast<uint64_t>(d.E) * 2};
    const uint32_t boxq[2] = {FBK, static_cast<uint32_t>(NG * d.G * DL)};
    const uint32_t boxkv[2] = {FBK, static_cast<uint32_t>(NG * DL)};
    if (!make_tma_16bit(&mwq, a.w_qkv, 2, dims, strides, boxq, 64, 0) ||
        !make_tma_16bit(&mwkv, a.w_qkv, 2, dims, strides, boxkv, 64, 0))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(DL), static_cast<uint64_t>(d.H + d.Hkv) * DL};
    const uint64_t strides[1] = {static_cast<uint64_t>(DL) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(DL), static_cast<uint32_t>(DL)};
    if (!make_tma_16bit(&mfh, a.filt_hi, 2, dims, strides, box, DL * 2, 0) ||
        !make_tma_16bit(&mfl, a.filt_lo, 2, dims, strides, box, DL * 2, 0))
      return cudaErrorInvalidValue;
  }
  FusedParams p;
  p.conv_seq = a.conv_seq;
  p.q = static_cast<__half *>(a.q);
  p.k = static_cast<__half *>(a.k);
  p.v = static_cast<__half *>(a.v);
  p.conv_state = a.conv_state;
  p.vshift_state = a.vshift_state;
  p.lengths = a.lengths;
  p.status = a.status;
  p.write_state = a.write_state ? 1 : 0;
  p.B = d.B; p.S = d.S; p.E = d.E; p.H = d.H; p.Hkv = d.Hkv; p.G = d.G; p.NQ = d.NQ; p.NKV = d.NKV; p.KC = d.KC;
  p.HALO = HALO; p.VS0 = d.VS0; p.kv_stride = a.kv_stride;
  p.NG = NG; p.N = N;
  p.nsets = d.Hkv / NG;
  p.units_per_seq = (d.S + (FM - HALO) - 1) / (FM - HALO);
  p.flags = d.flags;
  p.eps = d.eps;
  for (int i = 0; i < 32; ++i)
    p.theta[i] = i < DL / 2 ? pow(static_cast<double>(d.rope_base), -2.0 * i / DL) : 0.0;
  const int units = d.B * p.units_per_seq;
  int cps = num_sms() / p.nsets;                  // CTAs per group set: one per SM in all
  if (cps < 1) cps = 1;
  if (cps > units) cps = units;
  p.cps = cps;
  const FusedSmem L = fused_smem(DL, N, NG, d.G, d.KC);
  if (cudaError_t e = ensure_dyn_smem<qkv_stencil_kernel<DL>>(L.total); e != cudaSuccess) return e;
  qkv_stencil_kernel<DL><<<p.nsets * cps, F_THREADS, L.total, st>>>(mx, mwq, mwkv, mfh, mfl, p);
  return cudaGetLastError();
}

cudaError_t split_filter_planes(const Dims &d, const float *conv_chan, void *hi, void *lo,
                                cudaStream_t st) {
  const size_t n = static_cast<size_t>(d.H + d.Hkv) * d.DL * d.DL;
  const unsigned blocks = static_cast<unsigned>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
  split_planes_kernel<<<blocks, 256, 0, st>>>(conv_chan, static_cast<__nv_bfloat16 *>(hi),
                                              static_cast<__nv_bfloat16 *>(lo), n);
  return cudaGetLastError();
}

cudaError_t fused_qkv_stencil(const Dims &d, const FusedArgs &a, cudaStream_t st) {
  if (d.B == 0 || d.S == 0) return cudaSuccess;
  const int NG = fused_group_set(d);
  if (!NG) return cudaErrorNotSupported;
  if (d.DL == 16) return launch_fused<16>(d, a, NG, st);
  if (d.DL == 32) return launch_fused<32>(d, a, NG, st);
  return launch_fused<64>(d, a, NG, st);
}

}  // namespace cca
