// The C ABI of libcca (declared in include/cca.h and include/cca_stages.h): argument
// validation on the host, layout of the caller's workspace and cache buffers, and the
// launch sequence of each call.  No device memory is allocated here.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "cca.h"
#include "cca_stages.h"
#include "common.cuh"
#include "kernels.h"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return CCA_OK;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Which kernels a 16-bit prefill with the convolutions uses for the down-projection and the
// stencil: the fused kernel (P stays on chip) wherever it supports the shape; measured on B200
// it is as fast or faster than the separate GEMM + stencil kernels on every workload
// (cca_prefill_4k 0.39 -> 0.22 ms, ccgqa_prefill_16k 0.43 -> 0.39 ms, ccgqa_prefill_32k 0.61 vs
// 0.63 ms).  CCA_PREFILL_PATH=fused or =unfused overrides the choice (for comparing the paths).
bool use_fused(const cca::Dims &d) {
  if (cca::fused_group_set(d) == 0) return false;
  const char *f = getenv("CCA_PREFILL_PATH");
  return !(f && strcmp(f, "unfused") == 0);
}

// Host-side fault injection for the error paths: CCA_FAULT_INJECT=launch makes every call
// that would launch kernels fail with CCA_ERR_CUDA before touching the device.
bool injected_launch_failure() {
  const char *f = getenv("CCA_FAULT_INJECT");
  return f && strcmp(f, "launch") == 0;
}

int cuda_fail(cudaError_t e, const char *what) {
  return fail(CCA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Validates a config and fills the kernel-facing shape (B and S left at zero).
int make_dims(const cca_config_t *cfg, cca::Dims &d) {
  if (!cfg) return fail(CCA_ERR_INVALID_ARG, "config is NULL");
  if (cfg->d_model <= 0 || cfg->n_heads <= 0 || cfg->n_kv_heads <= 0 || cfg->compression <= 0)
    return fail(CCA_ERR_INVALID_ARG, "d_model, n_heads, n_kv_heads and compression must be positive");
  if (cfg->d_model % cfg->n_heads)
    return fail(CCA_ERR_INVALID_ARG, "d_model %d is not a multiple of n_heads %d", cfg->d_model, cfg->n_heads);
  if (cfg->n_heads % cfg->n_kv_heads)
    return fail(CCA_ERR_INVALID_ARG, "n_heads %d is not a multiple of n_kv_heads %d", cfg->n_heads, cfg->n_kv_heads);
  const int hd = cfg->d_model / cfg->n_heads;
  if (hd % cfg->compression)
    return fail(CCA_ERR_INVALID_ARG, "head width %d is not a multiple of compression %d", hd, cfg->compression);
  const int dl = hd / cfg->compression;
  if (dl != 16 && dl != 32 && dl != 64 && dl != 128)
    return fail(CCA_ERR_UNSUPPORTED, "latent head width %d: kernels take 16, 32, 64 or 128", dl);
  if (dl == 128 && cfg->dtype != CCA_BF16)
    return fail(CCA_ERR_UNSUPPORTED, "latent head width 128 is supported for bfloat16 layers only");
  if (cfg->conv_kernel < 1 || cfg->conv_kernel > 8)
    return fail(CCA_ERR_UNSUPPORTED, "conv_kernel %d: kernels take 1..8", cfg->conv_kernel);
  if (cfg->chan_conv_kernel != 1)
    return fail(CCA_ERR_UNSUPPORTED, "chan_conv_kernel %d: kernels take 1 (pointwise)", cfg->chan_conv_kernel);
  if (cfg->dtype != CCA_F32 && cfg->dtype != CCA_BF16)
    return fail(CCA_ERR_INVALID_ARG, "dtype %d is neither CCA_F32 nor CCA_BF16", cfg->dtype);
  if (cfg->flags & ~static_cast<unsigned>(CCA_DEFAULT_FLAGS | CCA_NO_CONV))
    return fail(CCA_ERR_INVALID_ARG, "unknown flag bits 0x%x", cfg->flags);
  if (!(cfg->norm_eps >= 0.f)) return fail(CCA_ERR_INVALID_ARG, "norm_eps must be >= 0");
  if ((cfg->flags & CCA_ROPE) && !(cfg->rope_base > 1.f))
    return fail(CCA_ERR_INVALID_ARG, "rope_base must be > 1");
  const int tp = cfg->tp_size <= 1 ? 1 : cfg->tp_size;
  if (cfg->tp_size < 0 || cfg->tp_rank < 0 || cfg->tp_rank >= tp)
    return fail(CCA_ERR_INVALID_ARG, "tp_rank %d outside [0, tp_size %d)", cfg->tp_rank, tp);
  if (cfg->n_kv_heads % tp)
    return fail(CCA_ERR_INVALID_ARG, "n_kv_heads %d is not a multiple of tp_size %d", cfg->n_kv_heads, tp);
  d.E = cfg->d_model;
  d.H = cfg->n_heads / tp;              // this rank's heads (all of them without TP)
  d.Hkv = cfg->n_kv_heads / tp;
  d.G = d.H / d.Hkv;
  d.DL = dl;
  d.NQ = d.H * dl;
  d.NKV = d.Hkv * dl;
  d.NQKV = d.NQ + 2 * d.NKV;
  d.KC = cfg->conv_kernel;
  {
    // value channels >= n_kv/2 of the whole layer are shifted; this rank holds global value
    // channels [rank * NKV, (rank + 1) * NKV)
    const int vs = cfg->n_kv_heads * dl / 2 - (tp > 1 ? cfg->tp_rank : 0) * d.NKV;
    d.VS0 = vs < 0 ? 0 : vs > d.NKV ? d.NKV : vs;
  }
  d.flags = cfg->flags;
  d.eps = cfg->norm_eps;
  d.rope_base = cfg->rope_base;
  d.bf16 = cfg->dtype == CCA_BF16;
  return CCA_OK;
}

size_t esize(const cca::Dims &d) { return d.bf16 ? 2 : 4; }

struct PrefillLayout {
  size_t status, wo16, wsplit, P, q, k, v, o, total;
};

PrefillLayout prefill_layout(const cca::Dims &d, int B, int S) {
  PrefillLayout L;
  const size_t M = static_cast<size_t>(B) * S, es = esize(d);
  size_t off = 0;
  L.status = off; off += 256;
  L.wo16 = off; off += d.bf16 ? align256(static_cast<size_t>(d.E) * d.NQ * 2) : 0;
  L.wsplit = off; off += (d.flags & CCA_NO_CONV) ? 0 : align256(cca::conv_chan_split_bytes(d));
  L.P = off; off += align256(M * d.NQKV * 4);   // projections stay float32
  L.q = off; off += align256(M * d.NQ * es);
  L.k = off; off += align256(M * d.NKV * es);
  L.v = off; off += align256(M * d.NKV * es);
  L.o = off; off += align256(M * d.NQ * es);
  L.total = off;
  return L;
}

struct CacheLayout {
  size_t k, v, conv, vshift, lengths, status, total;
};

CacheLayout cache_layout(const cca::Dims &d, int B, int max_seq) {
  CacheLayout L;
  const size_t es = esize(d);
  size_t off = 0;
  L.k = off; off += align256(static_cast<size_t>(B) * d.Hkv * max_seq * d.DL * es);
  L.v = off; off += align256(static_cast<size_t>(B) * d.Hkv * max_seq * d.DL * es);
  L.conv = off; off += align256(static_cast<size_t>(B) * (d.KC - 1) * (d.NQ + d.NKV) * 4);
  L.vshift = off; off += align256(static_cast<size_t>(B) * (d.NKV - d.VS0) * 4);
  L.lengths = off; off += align256(static_cast<size_t>(B) * 4);
  L.status = off; off += 256;
  L.total = off;
  return L;
}

// The decode kernels (and so the cache) cover latent widths up to 64 with the convolutions.
int check_decode_shape(const cca::Dims &d) {
  if (d.DL > 64)
    return fail(CCA_ERR_UNSUPPORTED, "decode and the cache take latent head widths 16, 32 or 64");
  if (d.flags & CCA_NO_CONV)
    return fail(CCA_ERR_UNSUPPORTED, "decode and the cache need the convolutions (CCA_NO_CONV is prefill-only)");
  return CCA_OK;
}

// The convolution stencil covers latent widths up to 64; CCA_NO_CONV layers take up to 128.
int check_stencil_shape(const cca::Dims &d) {
  if (d.DL > 64 && !(d.flags & CCA_NO_CONV))
    return fail(CCA_ERR_UNSUPPORTED, "latent head width %d needs CCA_NO_CONV (the convolution "
                "stencil takes 16, 32 or 64)", d.DL);
  return CCA_OK;
}

int check_cache(const cca::Dims &d, const cca_cache_t *c) {
  if (!c->k || !c->v || !c->vshift_state || !c->lengths || !c->status ||
      (d.KC > 1 && !c->conv_state))
    return fail(CCA_ERR_INVALID_ARG, "cache has a NULL region (lay it out with cca_cache_alloc)");
  if (c->batch <= 0 || c->max_seq <= 0) return fail(CCA_ERR_INVALID_ARG, "cache batch/max_seq must be positive");
  if (!aligned16(c->k) || !aligned16(c->v) || !aligned16(c->conv_state) || !aligned16(c->vshift_state))
    return fail(CCA_ERR_ALIGNMENT, "cache regions must be 16-byte aligned");
  return CCA_OK;
}

// dtype of the operands: CCA_F32 (CUDA cores), CCA_BF16 or CCA_F16 (tensor cores).
int gemm_dispatch(int dtype, int out_f32, const void *A, const void *B, void *C, int M, int N,
                  int K, int *status, cudaStream_t st) {
  cudaError_t e;
  if (dtype != CCA_F32)
    e = cca::gemm_tcgen05(A, B, C, M, N, K, dtype == CCA_F16, out_f32, status, st);
  else
    e = cca::gemm_simt(0, A, B, C, M, N, K, st);
  return e == cudaSuccess ? CCA_OK : cuda_fail(e, "projection GEMM launch");
}

// ---------------------------------------------------------------- stage timing
struct StageTiming {
  std::mutex mu;
  bool enabled = false;
  std::vector<std::vector<cudaEvent_t>> calls;
  std::vector<cudaEvent_t> pool;
  static constexpr size_t kMaxCalls = 4096;

  cudaEvent_t take() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
  void clear() {
    for (auto &c : calls)
      for (cudaEvent_t e : c) pool.push_back(e);
    calls.clear();
  }
};
StageTiming g_timing;

// Records the events of one C-ABI call when stage timing is on.
struct CallRecorder {
  cudaStream_t st;
  long idx = -1;
  explicit CallRecorder(cudaStream_t s) : st(s) {
    std::lock_guard<std::mutex> lk(g_timing.mu);
    if (!g_timing.enabled || g_timing.calls.size() >= StageTiming::kMaxCalls) return;
    g_timing.calls.emplace_back();
    idx = static_cast<long>(g_timing.calls.size()) - 1;
  }
  void mark() {
    if (idx < 0) return;
    std::lock_guard<std::mutex> lk(g_timing.mu);
    if (idx >= static_cast<long>(g_timing.calls.size())) return;
    cudaEvent_t e = g_timing.take();
    if (!e) return;
    cudaEventRecord(e, st);
    g_timing.calls[idx].push_back(e);
  }
  static void mark_cb(void *self) { static_cast<CallRecorder *>(self)->mark(); }
  cca::StageMarker marker() {
    cca::StageMarker m;
    m.ctx = this;
    m.fn = &CallRecorder::mark_cb;
    return m;
  }
};

}  // namespace

extern "C" {

CCA_API int cca_stage_timing(int enable) {
  std::lock_guard<std::mutex> lk(g_timing.mu);
  if (enable) g_timing.clear();
  g_timing.enabled = enable != 0;
  return ok();
}

CCA_API int cca_stage_times(double *ms, int n, int *calls) {
  std::lock_guard<std::mutex> lk(g_timing.mu);
  if (n < 0 || (n > 0 && !ms)) return fail(CCA_ERR_INVALID_ARG, "ms is NULL");
  for (int i = 0; i < n; ++i) ms[i] = 0.0;
  size_t slots = 0;
  int used = 0;
  for (auto &c : g_timing.calls) {
    if (c.size() < 2) continue;
    if (slots == 0) slots = c.size() - 1;
    if (c.size() - 1 != slots) continue;
    for (size_t i = 0; i < slots; ++i) {
      float t = 0.f;
      cudaError_t e = cudaEventSynchronize(c[i + 1]);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&t, c[i], c[i + 1]);
      if (e != cudaSuccess) return cuda_fail(e, "stage event");
      if (static_cast<int>(i) < n) ms[i] += t;
    }
    ++used;
  }
  if (calls) *calls = used;
  g_last_error.clear();
  return static_cast<int>(slots);
}


CCA_API const char *cca_last_error_string(void) { return g_last_error.c_str(); }

CCA_API int cca_cache_alloc(const cca_config_t *cfg, int batch, int max_seq, void *dev_buf,
                            size_t *bytes, cca_cache_t *out, void *stream) {
  cca::Dims d;
  int rc = make_dims(cfg, d);
  if (rc) return rc;
  if ((rc = check_decode_shape(d))) return rc;
  if (!bytes) return fail(CCA_ERR_INVALID_ARG, "bytes is NULL");
  if (batch <= 0 || max_seq <= 0) return fail(CCA_ERR_INVALID_ARG, "batch and max_seq must be positive");
  const CacheLayout L = cache_layout(d, batch, max_seq);
  if (!dev_buf) {
    *bytes = L.total;
    return ok();
  }
  if (!out) return fail(CCA_ERR_INVALID_ARG, "out is NULL");
  if (*bytes < L.total)
    return fail(CCA_ERR_WORKSPACE, "cache buffer of %zu bytes, %zu needed", *bytes, L.total);
  if (!aligned16(dev_buf)) return fail(CCA_ERR_ALIGNMENT, "cache buffer must be 16-byte aligned");
  if (injected_launch_failure()) return fail(CCA_ERR_CUDA, "injected launch failure");
  char *base = static_cast<char *>(dev_buf);
  out->k = base + L.k;
  out->v = base + L.v;
  out->conv_state = d.KC > 1 ? base + L.conv : nullptr;
  out->vshift_state = base + L.vshift;
  out->lengths = reinterpret_cast<int *>(base + L.lengths);
  out->status = reinterpret_cast<int *>(base + L.status);
  out->batch = batch;
  out->max_seq = max_seq;
  cudaError_t e = cudaMemsetAsync(dev_buf, 0, L.total, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cache zeroing");
  return ok();
}

CCA_API size_t cca_prefill_workspace_size(const cca_config_t *cfg, int batch, int seq) {
  cca::Dims d;
  if (make_dims(cfg, d) || check_stencil_shape(d) || batch < 0 || seq < 0) return 0;
  return prefill_layout(d, batch, seq).total;
}

CCA_API size_t cca_decode_workspace_size(const cca_config_t *cfg, int batch, int max_seq) {
  cca::Dims d;
  if (make_dims(cfg, d) || check_decode_shape(d) || batch <= 0 || max_seq <= 0) return 0;
  d.B = batch;
  return cca::decode_workspace_bytes(d, max_seq);
}

CCA_API int cca_decode_kernel_count(const cca_config_t *cfg, int batch, int max_seq) {
  cca::Dims d;
  int rc = make_dims(cfg, d);
  if (rc) return rc;
  if ((rc = check_decode_shape(d))) return rc;
  if (batch <= 0 || max_seq <= 0) return fail(CCA_ERR_INVALID_ARG, "batch and max_seq must be positive");
  d.B = batch;
  return cca::decode_kernel_count(d, max_seq);
}

CCA_API int cca_prefill_forward(const cca_config_t *cfg, const cca_weights_t *w, const void *x,
                                int batch, int seq, void *y, cca_cache_t *cache,
                                void *workspace, size_t ws_bytes, void *stream) {
  cca::Dims d;
  int rc = make_dims(cfg, d);
  if (rc) return rc;
  if ((rc = check_stencil_shape(d))) return rc;
  const bool no_conv = (d.flags & CCA_NO_CONV) != 0;
  if (!w || !w->w_qkv || !w->w_o || (!no_conv && (!w->conv_seq || !w->conv_chan)))
    return fail(CCA_ERR_INVALID_ARG, "weights (or one of their pointers) NULL");
  if (batch < 0 || seq < 0) return fail(CCA_ERR_INVALID_ARG, "batch and seq must be >= 0");
  if (batch > 0 && seq > 0 && (!x || !y)) return fail(CCA_ERR_INVALID_ARG, "x or y NULL");
  if (static_cast<long long>(batch) * seq > (1LL << 31) / 4)
    return fail(CCA_ERR_UNSUPPORTED, "batch*seq %lld too large", static_cast<long long>(batch) * seq);
  if (!aligned16(x) || !aligned16(y) || !aligned16(w->w_qkv) || !aligned16(w->w_o) ||
      !aligned16(workspace))
    return fail(CCA_ERR_ALIGNMENT, "x, y, weights and workspace must be 16-byte aligned");
  if (cache) {
    if ((rc = check_decode_shape(d))) return rc;
    if ((rc = check_cache(d, cache))) return rc;
    if (cache->batch != batch)
      return fail(CCA_ERR_INVALID_ARG, "cache batch %d != batch %d", cache->batch, batch);
    if (seq > cache->max_seq)
      return fail(CCA_ERR_CACHE_FULL, "seq %d exceeds cache max_seq %d", seq, cache->max_seq);
  }
  d.B = batch;
  d.S = seq;
  const PrefillLayout L = prefill_layout(d, batch, seq);
  if (!workspace || ws_bytes < L.total)
    return fail(CCA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace ? ws_bytes : 0, L.total);
  if (injected_launch_failure()) return fail(CCA_ERR_CUDA, "injected launch failure");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  int *status = reinterpret_cast<int *>(ws + L.status);
  cudaError_t e = cudaMemsetAsync(status, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "workspace status reset");
  if (batch == 0 || seq == 0) return ok();
  const int M = batch * seq;
  CallRecorder rec(st);
  rec.mark();
  // The projection fused with the stencil where the kernel supports the shape (16-bit layers
  // with the convolutions); P then never reaches global memory.
  const bool fused = d.bf16 && !no_conv && use_fused(d);
  // 16-bit layers: the up-projection runs on float16 operands (the attention output is
  // float16), so W_o is converted once per call.
  void *wo = const_cast<void *>(w->w_o);
  char *fhi = ws + L.wsplit, *flo = fhi + static_cast<size_t>(d.H + d.Hkv) * d.DL * d.DL * 2;
  if (d.bf16) {
    wo = ws + L.wo16;
    if ((e = cca::convert_bf16_to_f16(w->w_o, wo, static_cast<size_t>(d.E) * d.NQ, status, st)) !=
        cudaSuccess)
      return cuda_fail(e, "W_o conversion launch");
    if (fused)
      e = cca::split_filter_planes(d, w->conv_chan, fhi, flo, st);
    else if (!no_conv)
      e = cca::split_conv_chan(d, w->conv_chan, ws + L.wsplit, st);
    if (e != cudaSuccess) return cuda_fail(e, "channel-conv weight split launch");
  }
  rec.mark();
  void *P = ws + L.P, *q = ws + L.q, *o = ws + L.o;
  void *k = cache ? cache->k : ws + L.k;
  void *v = cache ? cache->v : ws + L.v;
  const int kv_stride = cache ? cache->max_seq : seq;

  if (fused) {
    cca::FusedArgs fa;
    fa.x = x;
    fa.w_qkv = w->w_qkv;
    fa.conv_seq = w->conv_seq;
    fa.filt_hi = fhi;
    fa.filt_lo = flo;
    fa.q = q;
    fa.k = k;
    fa.v = v;
    fa.kv_stride = kv_stride;
    fa.conv_state = cache ? static_cast<float *>(cache->conv_state) : nullptr;
    fa.vshift_state = cache ? static_cast<float *>(cache->vshift_state) : nullptr;
    fa.lengths = cache ? cache->lengths : nullptr;
    fa.write_state = cache != nullptr;
    fa.status = status;
    if ((e = cca::fused_qkv_stencil(d, fa, st)) != cudaSuccess)
      return cuda_fail(e, "fused projection + stencil launch");
    rec.mark();
    if ((e = cca::latent_attention(d, q, k, v, kv_stride, o, status, st)) != cudaSuccess)
      return cuda_fail(e, "attention launch");
    rec.mark();
    if ((rc = gemm_dispatch(CCA_F16, 0, o, wo, y, M, d.E, d.NQ, status, st))) return rc;
    rec.mark();
    return ok();
  }

  const int dt = d.bf16 ? CCA_BF16 : CCA_F32;
  if ((rc = gemm_dispatch(dt, 1, x, w->w_qkv, P, M, d.NQKV, d.E, status, st))) return rc;
  rec.mark();
  cca::StencilArgs sa;
  sa.P = static_cast<const float *>(P);
  sa.conv_seq = w->conv_seq;
  sa.conv_chan = w->conv_chan;
  sa.conv_chan_split = ws + L.wsplit;
  sa.q = q;
  sa.k = k;
  sa.v = v;
  sa.kv_stride = kv_stride;
  sa.conv_state = cache ? static_cast<float *>(cache->conv_state) : nullptr;
  sa.vshift_state = cache ? static_cast<float *>(cache->vshift_state) : nullptr;
  sa.lengths = cache ? cache->lengths : nullptr;
  sa.write_state = cache != nullptr;
  sa.status = status;
  if ((e = cca::latent_stencil(d, sa, st)) != cudaSuccess) return cuda_fail(e, "stencil launch");
  rec.mark();
  if ((e = cca::latent_attention(d, q, k, v, kv_stride, o, status, st)) != cudaSuccess)
    return cuda_fail(e, "attention launch");
  rec.mark();
  if ((rc = gemm_dispatch(d.bf16 ? CCA_F16 : CCA_F32, 0, o, wo, y, M, d.E, d.NQ, status, st)))
    return rc;
  rec.mark();
  return ok();
}

}  // extern "C"

namespace {
// ------------------------------------------------------------------ backward pass
struct BackwardLayout {
  size_t status, wsplit, wsplitT, P, q, k, v, o, lse, D, woT, dO, oB, dq, dk, dv, dA, dPpart,
      dP, total;
};

BackwardLayout backward_layout(const cca::Dims &d, int B, int S) {
  BackwardLayout L;
  const size_t M = static_cast<size_t>(B) * S;
  const size_t rows = static_cast<size_t>(B) * d.H * S;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off += align256(bytes); return o; };
  L.status = take(256);
  L.wsplit = take(cca::conv_chan_split_bytes(d));
  L.wsplitT = take(cca::conv_chan_split_bytes(d));
  L.P = take(M * d.NQKV * 4);
  L.q = take(M * d.NQ * 2);
  L.k = take(M * d.NKV * 2);
  L.v = take(M * d.NKV * 2);
  L.o = take(M * d.NQ * 2);
  L.lse = take(rows * 4);
  L.D = take(rows * 4);
  L.woT = take(static_cast<size_t>(d.NQ) * d.E * 2);
  L.dO = take(M * d.NQ * 2);
  L.oB = take(M * d.NQ * 2);
  L.dq = take(M * d.NQ * 4);
  L.dk = take(M * d.NKV * 4);
  L.dv = take(M * d.NKV * 4);
  L.dA = take(M * (d.NQ + d.NKV) * 4);
  L.dPpart = take(M * d.NQKV * 4);
  L.dP = take(M * d.NQKV * 2);
  L.total = off;
  return L;
}

int check_backward_shape(const cca::Dims &d) {
  if (!d.bf16) return fail(CCA_ERR_UNSUPPORTED, "the backward pass runs bfloat16 layers");
  if (!cca::stencil_backward_supported(d))
    return fail(CCA_ERR_UNSUPPORTED, "backward pass: needs the convolutions, latent width <= 64 "
                "and (H/Hkv + 1) * d~^2 <= 20480");
  if (d.E % 8) return fail(CCA_ERR_UNSUPPORTED, "backward pass: d_model must be a multiple of 8");
  return CCA_OK;
}
}  // namespace

extern "C" {

CCA_API size_t cca_backward_workspace_size(const cca_config_t *cfg, int batch, int seq) {
  cca::Dims d;
  if (make_dims(cfg, d) || check_backward_shape(d) || batch < 0 || seq < 0) return 0;
  return backward_layout(d, batch, seq).total;
}

CCA_API int cca_backward(const cca_config_t *cfg, const cca_weights_t *w, const void *x,
                         const void *dy, int batch, int seq, void *dx, float *dw_qkv,
                         float *dw_o, float *dconv_seq, float *dconv_chan, void *workspace,
                         size_t ws_bytes, void *stream) {
  cca::Dims d;
  int rc = make_dims(cfg, d);
  if (rc) return rc;
  if ((rc = check_backward_shape(d))) return rc;
  if (!w || !w->w_qkv || !w->w_o || !w->conv_seq || !w->conv_chan)
    return fail(CCA_ERR_INVALID_ARG, "weights (or one of their pointers) NULL");
  if (batch <= 0 || seq <= 0) return fail(CCA_ERR_INVALID_ARG, "batch and seq must be positive");
  if (!x || !dy || !dx || !dw_qkv || !dw_o || !dconv_seq || !dconv_chan)
    return fail(CCA_ERR_INVALID_ARG, "x, dy or an output NULL");
  if (static_cast<long long>(batch) * seq > (1LL << 31) / 4)
    return fail(CCA_ERR_UNSUPPORTED, "batch*seq %lld too large", static_cast<long long>(batch) * seq);
  if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || !aligned16(dw_qkv) || !aligned16(dw_o) ||
      !aligned16(w->w_qkv) || !aligned16(w->w_o) || !aligned16(workspace))
    return fail(CCA_ERR_ALIGNMENT, "tensors and workspace must be 16-byte aligned");
  d.B = batch;
  d.S = seq;
  const BackwardLayout L = backward_layout(d, batch, seq);
  if (!workspace || ws_bytes < L.total)
    return fail(CCA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace ? ws_bytes : 0, L.total);
  if (injected_launch_failure()) return fail(CCA_ERR_CUDA, "injected launch failure");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  int *status = reinterpret_cast<int *>(ws + L.status);
  const int M = batch * seq;
  cudaError_t e = cudaMemsetAsync(status, 0, 256, st);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(dconv_seq, 0, static_cast<size_t>(d.NQ + d.NKV) * d.KC * 4, st);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(dconv_chan, 0, static_cast<size_t>(d.H + d.Hkv) * d.DL * d.DL * 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "backward set-up");
  CallRecorder rec(st);
  rec.mark();
  // forward recomputation: projections (kept), latents, attention output and log-sum-exp
  void *P = ws + L.P, *q = ws + L.q, *k = ws + L.k, *v = ws + L.v, *o = ws + L.o;
  float *lse = reinterpret_cast<float *>(ws + L.lse), *Dd = reinterpret_cast<float *>(ws + L.D);
  if ((rc = gemm_dispatch(CCA_BF16, 1, x, w->w_qkv, P, M, d.NQKV, d.E, status, st))) return rc;
  if ((e = cca::split_conv_chan(d, w->conv_chan, ws + L.wsplit, st)) != cudaSuccess)
    return cuda_fail(e, "channel-conv weight split launch");
  cca::StencilArgs sa{};
  sa.P = static_cast<const float *>(P);
  sa.conv_seq = w->conv_seq;
  sa.conv_chan = w->conv_chan;
  sa.conv_chan_split = ws + L.wsplit;
  sa.q = q;
  sa.k = k;
  sa.v = v;
  sa.kv_stride = seq;
  sa.status = status;
  if ((e = cca::latent_stencil(d, sa, st)) != cudaSuccess) return cuda_fail(e, "stencil launch");
  if ((e = cca::latent_attention_tc(d, q, k, v, seq, o, status, st, lse)) != cudaSuccess)
    return cuda_fail(e, "attention launch");
  rec.mark();
  // dO = dy W_o (float16, the attention backward's operand type), D = rowsum(dO * O)
  void *woT = ws + L.woT, *dO = ws + L.dO;
  if ((e = cca::transpose16(w->w_o, woT, d.E, d.NQ, d.E, false, st)) != cudaSuccess)
    return cuda_fail(e, "W_o transpose launch");
  if ((e = cca::gemm_tcgen05_f16out(dy, woT, dO, M, d.NQ, d.E, 0, status, st)) != cudaSuccess)
    return cuda_fail(e, "dO GEMM launch");
  if ((e = cca::attention_rowdot(d, dO, o, Dd, st)) != cudaSuccess)
    return cuda_fail(e, "rowdot launch");
  rec.mark();
  // attention backward
  cca::AttnBwdArgs ab;
  ab.q = q;
  ab.k = k;
  ab.v = v;
  ab.dO = dO;
  ab.kv_stride = seq;
  ab.lse = lse;
  ab.D = Dd;
  ab.dq = reinterpret_cast<float *>(ws + L.dq);
  ab.dk = reinterpret_cast<float *>(ws + L.dk);
  ab.dv = reinterpret_cast<float *>(ws + L.dv);
  ab.status = status;
  if ((e = cca::latent_attention_backward(d, ab, st)) != cudaSuccess)
    return cuda_fail(e, "attention backward launch");
  rec.mark();
  // stencil backward -> dP (bf16) and the conv filters' gradients
  cca::StencilBwdArgs sb;
  sb.P = static_cast<const float *>(P);
  sb.dq = ab.dq;
  sb.dk = ab.dk;
  sb.dv = ab.dv;
  sb.conv_seq = w->conv_seq;
  sb.conv_chan = w->conv_chan;
  sb.conv_chan_split = ws + L.wsplit;
  sb.conv_chan_split_t = ws + L.wsplitT;
  sb.dA = reinterpret_cast<float *>(ws + L.dA);
  sb.dPpart = reinterpret_cast<float *>(ws + L.dPpart);
  sb.dP = ws + L.dP;
  sb.dconv_seq = dconv_seq;
  sb.dconv_chan = dconv_chan;
  if ((e = cca::stencil_backward(d, sb, st)) != cudaSuccess)
    return cuda_fail(e, "stencil backward launch");
  rec.mark();
  // dx = dP W_qkv, dW_qkv = dP^T x, dW_o = dy^T o: the operands read as stored (row-major
  // activations as MN-major tiles of the products over tokens); o in bfloat16 for dW_o
  void *oB = ws + L.oB;
  if ((e = cca::convert_f16_to_bf16(o, oB, static_cast<size_t>(M) * d.NQ, st)) != cudaSuccess)
    return cuda_fail(e, "attention output conversion launch");
  if ((e = cca::gemm_tcgen05_t(ws + L.dP, w->w_qkv, dx, M, d.E, d.NQKV, 0, 1, 0, status, st)) != cudaSuccess ||
      (e = cca::gemm_tcgen05_t(ws + L.dP, x, dw_qkv, d.NQKV, d.E, M, 1, 1, 1, status, st)) != cudaSuccess ||
      (e = cca::gemm_tcgen05_t(dy, oB, dw_o, d.E, d.NQ, M, 1, 1, 1, status, st)) != cudaSuccess)
    return cuda_fail(e, "gradient GEMM launch");
  rec.mark();
  return ok();
}

CCA_API int cca_decode_step(const cca_config_t *cfg, const cca_weights_t *w, const void *x,
                            void *y, cca_cache_t *cache, void *workspace, size_t ws_bytes,
                            void *stream) {
  cca::Dims d;
  int rc = make_dims(cfg, d);
  if (rc) return rc;
  if (!w || !w->w_qkv || !w->w_o || !w->conv_seq || !w->conv_chan)
    return fail(CCA_ERR_INVALID_ARG, "weights (or one of their pointers) NULL");
  if ((rc = check_decode_shape(d))) return rc;
  if (!cache) return fail(CCA_ERR_INVALID_ARG, "cache is NULL");
  if ((rc = check_cache(d, cache))) return rc;
  if (d.G > 8)
    return fail(CCA_ERR_UNSUPPORTED, "decode takes at most 8 query heads per kv head (got %d)", d.G);
  if (!x || !y) return fail(CCA_ERR_INVALID_ARG, "x or y NULL");
  if (!aligned16(x) || !aligned16(y) || !aligned16(w->w_qkv) || !aligned16(w->w_o) ||
      !aligned16(workspace))
    return fail(CCA_ERR_ALIGNMENT, "x, y, weights and workspace must be 16-byte aligned");
  d.B = cache->batch;
  const size_t need = cca::decode_workspace_bytes(d, cache->max_seq);
  if (!workspace || ws_bytes < need)
    return fail(CCA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace ? ws_bytes : 0, need);
  if (injected_launch_failure()) return fail(CCA_ERR_CUDA, "injected launch failure");
  cca::DecodeArgs a;
  cca::decode_workspace_carve(d, cache->max_seq, workspace, a);
  a.x = x;
  a.w_qkv = w->w_qkv;
  a.w_o = w->w_o;
  a.conv_seq = w->conv_seq;
  a.conv_chan = w->conv_chan;
  a.y = y;
  a.k_cache = cache->k;
  a.v_cache = cache->v;
  a.conv_state = static_cast<float *>(cache->conv_state);
  a.vshift_state = static_cast<float *>(cache->vshift_state);
  a.lengths = cache->lengths;
  a.status = cache->status;
  a.max_seq = cache->max_seq;
  CallRecorder rec(static_cast<cudaStream_t>(stream));
  rec.mark();
  cudaError_t e = cca::decode_step(d, a, static_cast<cudaStream_t>(stream), rec.marker());
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return ok();
}

CCA_API int cca_cache_check(cca_cache_t *cache, void *stream) {
  if (!cache || !cache->status) return fail(CCA_ERR_INVALID_ARG, "cache (or its status word) is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int s = 0;
  if ((e = cudaMemcpy(&s, cache->status, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "status read");
  if (s == 0) return ok();
  if ((e = cudaMemset(cache->status, 0, sizeof(int))) != cudaSuccess) return cuda_fail(e, "status clear");
  if (s == cca::DEV_CACHE_FULL) return fail(CCA_ERR_CACHE_FULL, "a sequence reached max_seq");
  if (s == cca::DEV_RANGE) return fail(CCA_ERR_RANGE, "a latent key or value exceeded the float16 range");
  return fail(CCA_ERR_DEVICE, "kernel status %d", s);
}

CCA_API int cca_workspace_status(const void *workspace, void *stream) {
  if (!workspace) return fail(CCA_ERR_INVALID_ARG, "workspace is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int s = 0;
  if ((e = cudaMemcpy(&s, workspace, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "status read");
  if (s == cca::DEV_RANGE) return fail(CCA_ERR_RANGE, "a latent query, key or value exceeded the float16 range");
  if (s) return fail(CCA_ERR_DEVICE, "kernel status %d (bounded wait ran out)", s);
  return ok();
}

CCA_API int cca_gemm(int dtype, int out_dtype, const void *A, const void *B, void *C, int M, int N, int K,
                     int *status, void *stream) {
  if ((dtype != CCA_F32 && dtype != CCA_BF16 && dtype != CCA_F16) ||
      (out_dtype != CCA_F32 && out_dtype != CCA_BF16))
    return fail(CCA_ERR_INVALID_ARG, "bad dtype %d / %d", dtype, out_dtype);
  if (M < 0 || N < 0 || K <= 0) return fail(CCA_ERR_INVALID_ARG, "bad shape %d x %d x %d", M, N, K);
  if (M > 0 && N > 0 && (!A || !B || !C)) return fail(CCA_ERR_INVALID_ARG, "NULL operand");
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return fail(CCA_ERR_ALIGNMENT, "operands must be 16-byte aligned");
  if (injected_launch_failure()) return fail(CCA_ERR_CUDA, "injected launch failure");
  if (dtype == CCA_F32 && out_dtype != CCA_F32)
    return fail(CCA_ERR_UNSUPPORTED, "float32 operands give a float32 result");
  if (dtype != CCA_F32 && K % 8 != 0)
    return fail(CCA_ERR_UNSUPPORTED, "16-bit rows must be a multiple of 16 bytes (K %% 8 == 0)");
  int rc = gemm_dispatch(dtype, out_dtype == CCA_F32, A, B, C, M, N, K, status,
                         static_cast<cudaStream_t>(stream));
  return rc ? rc : ok();
}

CCA_API int cca_gemm_t(int out_dtype, const void *A, const void *B, void *C, int M, int N, int K,
                       int a_trans, int b_trans, int *status, void *stream) {
  if (out_dtype != CCA_F32 && out_dtype != CCA_BF16)
    return fail(CCA_ERR_INVALID_ARG, "bad out dtype %d", out_dtype);
  if (M < 0 || N < 0 || K <= 0) return fail(CCA_ERR_INVALID_ARG, "bad shape %d x %d x %d", M, N, K);
  if (M > 0 && N > 0 && (!A || !B || !C)) return fail(CCA_ERR_INVALID_ARG, "NULL operand");
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return fail(CCA_ERR_ALIGNMENT, "operands must be 16-byte aligned");
  if ((a_trans ? M : K) % 8 != 0 || (b_trans ? N : K) % 8 != 0)
    return fail(CCA_ERR_UNSUPPORTED, "each operand's contiguous extent must be a multiple of 8");
  if (injected_launch_failure()) return fail(CCA_ERR_CUDA, "injected launch failure");
  const cudaError_t e = cca::gemm_tcgen05_t(A, B, C, M, N, K, a_trans ? 1 : 0, b_trans ? 1 : 0,
                                            out_dtype == CCA_F32, status,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "GEMM launch");
}

CCA_API size_t cca_stage_stencil_workspace_size(const cca_config_t *cfg) {
  cca::Dims d;
  if (make_dims(cfg, d)) return 0;
  return align256(cca::conv_chan_split_bytes(d)) + 256;
}

CCA_API int cca_stage_stencil(const cca_config_t *cfg, const void *P, int batch, int seq,
                              const float *conv_seq, const float *conv_chan, void *q, void *k,
                              void *v, int kv_stride, void *workspace, size_t ws_bytes,
                              void *stream) {
  cca::Dims d;
  int rc = make_dims(cfg, d);
  if (rc) return rc;
  if ((rc = check_stencil_shape(d))) return rc;
  const bool no_conv = (d.flags & CCA_NO_CONV) != 0;
  if (batch < 0 || seq < 0 || kv_stride < seq) return fail(CCA_ERR_INVALID_ARG, "bad batch/seq/kv_stride");
  if (batch > 0 && seq > 0 && (!P || (!no_conv && (!conv_seq || !conv_chan)) || !q || !k || !v))
    return fail(CCA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(P)) return fail(CCA_ERR_ALIGNMENT, "P must be 16-byte aligned");
  if (injected_launch_failure()) return fail(CCA_ERR_CUDA, "injected launch failure");
  d.B = batch;
  d.S = seq;
  const size_t need = align256(cca::conv_chan_split_bytes(d)) + 256;
  if (!workspace || ws_bytes < need)
    return fail(CCA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace ? ws_bytes : 0, need);
  if (!aligned16(workspace)) return fail(CCA_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char *wsp = static_cast<char *>(workspace);
  int *status = reinterpret_cast<int *>(wsp);
  cudaError_t e0 = cudaMemsetAsync(status, 0, 256, st);
  if (e0 == cudaSuccess && d.bf16 && !no_conv) e0 = cca::split_conv_chan(d, conv_chan, wsp + 256, st);
  if (e0 != cudaSuccess) return cuda_fail(e0, "stencil preparation");
  cca::StencilArgs sa{};
  sa.P = static_cast<const float *>(P);
  sa.conv_seq = conv_seq;
  sa.conv_chan = conv_chan;
  sa.conv_chan_split = wsp + 256;
  sa.status = status;
  sa.q = q;
  sa.k = k;
  sa.v = v;
  sa.kv_stride = kv_stride;
  cudaError_t e = cca::latent_stencil(d, sa, st);
  return e == cudaSuccess ? ok() : cuda_fail(e, "stencil launch");
}

CCA_API int cca_stage_attention(const cca_config_t *cfg, const void *q, const void *k,
                                const void *v, int batch, int seq, int kv_stride, void *o,
                                int *status, void *stream) {
  cca::Dims d;
  int rc = make_dims(cfg, d);
  if (rc) return rc;
  if (batch < 0 || seq < 0 || kv_stride < seq) return fail(CCA_ERR_INVALID_ARG, "bad batch/seq/kv_stride");
  if (batch > 0 && seq > 0 && (!q || !k || !v || !o)) return fail(CCA_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(CCA_ERR_ALIGNMENT, "q, k, v, o must be 16-byte aligned");
  if (injected_launch_failure()) return fail(CCA_ERR_CUDA, "injected launch failure");
  d.B = batch;
  d.S = seq;
  cudaError_t e = cca::latent_attention(d, q, k, v, kv_stride, o, status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "attention launch");
}

}  // extern "C"

namespace cca {
// Records `msg` as the calling thread's last error and returns `code`.
int set_last_error(int code, const char *msg) { return fail(code, "%s", msg); }
}  // namespace cca
