/*
 * cca.h -- C ABI of the B200 (sm_100a) implementation of Compressed Convolutional
 * Attention (CCA) and its grouped variant CCGQA.
 *
 * The operator (arXiv 2510.04476, "Compressed Convolutional Attention: Efficient
 * Attention in a Compressed Latent Space"; gist.science explainer, 2. Methodology, Core
 * Mechanism and Extension: CCGQA; arXiv abstract):
 *   1. x [tokens, E] is projected to latent q (H heads), k and v (Hkv heads), each head
 *      d~ = (E/H)/C wide, so the query latent is E/C wide ("Down-Projection").
 *   2. q and k pass a causal depthwise convolution along the sequence (conv_kernel taps,
 *      tap conv_kernel-1 on the current token) and a per-head channel convolution
 *      (d~ x d~ per head, pointwise in time) ("Convolutional Mixing"); half of
 *      (pre-conv q + pre-conv k) is added back to both ("Q-K-Mean"); the upper half of the
 *      value channels of token t is taken from token t-1 ("Value-Shift"); q and k are
 *      RMS-normalised per head and rotated by RoPE ("RoPE Integration").
 *   3. causal softmax attention runs on the latent heads, query head h reading key/value
 *      head h / (H/Hkv) (CCGQA), scale 1/sqrt(d~).
 *   4. the latent result [tokens, E/C] is projected back to E.
 *
 * Conventions for every entry point:
 *   - All device pointers are caller-owned; the library never allocates or frees device
 *     memory.  Scratch comes from the caller's `workspace`, sized by the *_size queries.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as void*; NULL =
 *     the legacy default stream).  Arguments are validated on the host before any launch;
 *     a failed check returns an error and launches nothing.
 *   - Return value: CCA_OK (0) or a negative CCA_ERR_* code; the text of the last error of
 *     the calling thread is in cca_last_error_string().  No C++ exception crosses the ABI.
 *   - Tensors are dense and row-major in the listed index order.  Activations x, y and the
 *     projection weights use the config's dtype (float32 or bfloat16); conv filters and the
 *     conv / value-shift state are always float32.  The latent queries, keys and values (and
 *     so the K/V cache) are float32 in float32 layers and float16 in bfloat16 layers: the
 *     same size and tensor-core rate as bfloat16 with three more significand bits (after
 *     the per-head RMS norm q and k are bounded by sqrt(d~); a latent beyond the float16
 *     range is reported as CCA_ERR_RANGE through cca_workspace_status / cca_cache_check).
 *     Device pointers must be 16-byte aligned (CCA_ERR_ALIGNMENT).
 */
#ifndef CCA_H
#define CCA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CCA_API __attribute__((visibility("default")))

/* Element types.  A layer is CCA_F32 or CCA_BF16; CCA_F16 (the latent type of bfloat16
 * layers) is accepted only by the stage entry points of cca_stages.h. */
typedef enum { CCA_F32 = 0, CCA_BF16 = 1, CCA_F16 = 2 } cca_dtype_t;

enum {
  CCA_OK = 0,
  CCA_ERR_INVALID_ARG = -1,   /* null pointer, non-positive size, inconsistent shape      */
  CCA_ERR_UNSUPPORTED = -2,   /* valid operator, but outside what the kernels implement   */
  CCA_ERR_WORKSPACE = -3,     /* workspace pointer null or smaller than the size query    */
  CCA_ERR_CACHE_FULL = -4,    /* a sequence would pass max_seq                             */
  CCA_ERR_ALIGNMENT = -5,     /* a device pointer is not 16-byte aligned                  */
  CCA_ERR_CUDA = -6,          /* a CUDA call or kernel launch failed                      */
  CCA_ERR_DEVICE = -7,        /* a kernel reported an internal error (bounded wait ran out) */
  CCA_ERR_RANGE = -8          /* a latent q, k or v exceeded the float16 range (16-bit layers) */
};

/* Switches of the method's three expressivity steps and of normalisation / RoPE.
 * CCA_NO_CONV makes both convolutions the identity (Convolutional Mixing off; not part of
 * CCA_DEFAULT_FLAGS).  With compression 1 and CCA_ROPE alone the layer is plain multi-head
 * (Hkv == H) or grouped-query attention with rotary embeddings, the systems the pages compare
 * CCA against (gist.science explainer, 4. Experimental Results: prefill against MHA and GQA-8
 * at 16k); such layers run up to a latent width of 128, prefill only (no cache, no decode). */
enum {
  CCA_QK_MEAN = 1u,
  CCA_VALUE_SHIFT = 2u,
  CCA_QK_NORM = 4u,
  CCA_ROPE = 8u,
  CCA_DEFAULT_FLAGS = 15u,
  CCA_NO_CONV = 16u
};

/* One CCA / CCGQA layer.  d_model = E, n_heads = H, n_kv_heads = Hkv (H % Hkv == 0;
 * Hkv == H is CCA), compression = C with (E/H) % C == 0.  Queries are compressed by C (latent
 * width E/C) and keys / values by C * H/Hkv (latent width Hkv * d~): CCGQA's decoupled
 * compression rates (gist.science explainer, Extension: CCGQA).  Supported by the kernels:
 * d~ = E/H/C in {16, 32, 64} (and 128 for bfloat16 CCA_NO_CONV prefill), conv_kernel in
 * [1, 8], chan_conv_kernel == 1.  norm_eps is added to the mean square before the square
 * root (1e-6 by default). */
typedef struct {
  int d_model;
  int n_heads;
  int n_kv_heads;
  int compression;
  int conv_kernel;
  int chan_conv_kernel;
  float rope_base;
  float norm_eps;
  unsigned flags;
  int dtype;                /* cca_dtype_t */
  int tp_size;              /* tensor-parallel ranks sharing the layer (0 or 1: none)       */
  int tp_rank;              /* this rank, 0 <= tp_rank < tp_size                            */
} cca_config_t;

/* Tensor parallelism by key/value group (gist.science explainer, 5. Significance and
 * Implications, Scalability: the method works with tensor parallelism).  Every step before the
 * up-projection is local to a key/value group (the channel conv is per head, Q-K-Mean pairs a
 * query head with its group's key head, attention reads only its group), so with
 * tp_size = R (Hkv % R == 0) rank r holds query heads [r H/R, (r+1) H/R) and key/value heads
 * [r Hkv/R, (r+1) Hkv/R) and computes them alone.  All sizes (workspace, cache, decode) are
 * then the rank's own, and the weights passed are the rank's slices:
 *   w_qkv     its query rows, then its key rows, then its value rows (of the global W_q, W_k, W_v)
 *   w_o       [E, n_q / R]: its columns of the global W_o
 *   conv_seq  its query channels' rows, then its key channels' rows
 *   conv_chan its query heads' filters, then its key heads' filters
 * y is the rank's share of the up-projection; the layer's output is the sum of y over the
 * ranks (one all-reduce of [tokens, E], done by the caller).  The value-shift keeps the
 * global split: value channel c of the layer comes from the previous token when
 * c >= n_kv / 2 of the whole layer, whichever rank holds it. */

/* Layer parameters (device pointers).
 *   w_qkv     [n_q + 2*n_kv, E]  rows: W_q (n_q = H*d~), W_k (n_kv = Hkv*d~), W_v
 *   w_o       [E, n_q]
 *   conv_seq  [n_q + n_kv, conv_kernel] float32, one causal filter per latent q/k channel
 *   conv_chan [H + Hkv, d~, d~, chan_conv_kernel] float32 (head, out, in, tap)          */
typedef struct {
  const void *w_qkv;
  const void *w_o;
  const float *conv_seq;
  const float *conv_chan;
} cca_weights_t;

/* Compressed decode state, laid out by cca_cache_alloc inside one caller buffer.
 *   k, v          [batch, Hkv, max_seq, d~]  final latent keys (after conv, q-k-mean, norm
 *                 and RoPE) and values (after value-shift), latent element type (above)
 *   conv_state    [batch, conv_kernel-1, n_q + n_kv] float32: pre-conv q|k projections of
 *                 the last conv_kernel-1 tokens, oldest first, zero before position 0
 *   vshift_state  [batch, n_kv - n_kv/2] float32: upper-half value projection of the last
 *                 token
 *   lengths       [batch] int32, tokens held per sequence (the RoPE position of the next)
 *   status        int32 sticky error word set by kernels that met a full sequence       */
typedef struct {
  void *k;
  void *v;
  void *conv_state;
  void *vshift_state;
  int *lengths;
  int *status;
  int batch;
  int max_seq;
} cca_cache_t;

/* Lays out a decode cache for `batch` sequences of up to `max_seq` tokens.  The cache holds
 * the compressed latent keys and values, the thing decoding streams per generated token
 * (gist.science explainer, 1. Problem Statement), Hkv heads of d~ each (Extension: CCGQA:
 * grouped key/value heads in the compressed space), plus the conv and value-shift state that
 * the causal convolutions and Value-Shift of the next token need (2. Methodology, Core
 * Mechanism).
 * dev_buf == NULL: only writes the byte count to *bytes.  Otherwise *bytes must be at
 * least that count; fills *out with pointers into dev_buf and enqueues on `stream` the
 * zeroing of the whole buffer (lengths = 0, status = 0).  Errors: INVALID_ARG,
 * UNSUPPORTED, WORKSPACE (buffer too small), ALIGNMENT, CUDA. */
CCA_API int cca_cache_alloc(const cca_config_t *cfg, int batch, int max_seq, void *dev_buf,
                            size_t *bytes, cca_cache_t *out, void *stream);

/* Scratch bytes needed by cca_prefill_forward (0 if the config is invalid). */
CCA_API size_t cca_prefill_workspace_size(const cca_config_t *cfg, int batch, int seq);

/* Scratch bytes needed by cca_decode_step for a cache of this shape (0 if invalid). */
CCA_API size_t cca_decode_workspace_size(const cca_config_t *cfg, int batch, int max_seq);

/* Kernels one cca_decode_step launches for a cache of this shape, on the current device
 * (the split of the attention's keys depends on its SM count); for launch accounting and
 * profiling.  (Not in the paper.)  Negative CCA_ERR_* code if the config is invalid. */
CCA_API int cca_decode_kernel_count(const cca_config_t *cfg, int batch, int max_seq);

/* Full layer forward of `batch` sequences of `seq` tokens each, from position 0: the
 * down-projection, convolutional mixing, Q-K-Mean, Value-Shift, normalisation and RoPE,
 * attention in the compressed space and the up-projection (gist.science explainer,
 * 2. Methodology, Core Mechanism; Extension: CCGQA for Hkv < H).
 *   x [batch, seq, E] -> y [batch, seq, E]   (x and y must not overlap)
 * In bfloat16 layers the up-projection runs on float16 operands (the attention output is
 * float16), so W_o is converted to float16 in the workspace on every call: an entry beyond
 * the float16 range (|w| > 65504) sets CCA_ERR_RANGE in the workspace status word
 * (cca_workspace_status), and entries below 2^-14 keep float16's subnormal spacing of 2^-24
 * (an absolute change below 3e-8 per weight).
 * cache == NULL: keys/values live in the workspace only.  Otherwise (cache->batch ==
 * batch, seq <= max_seq) the final keys/values of every token are written to the cache,
 * the conv and value-shift state of the last token are stored and lengths[b] = seq.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CACHE_FULL (seq > max_seq), ALIGNMENT, CUDA. */
CCA_API int cca_prefill_forward(const cca_config_t *cfg, const cca_weights_t *w, const void *x,
                                int batch, int seq, void *y, cca_cache_t *cache,
                                void *workspace, size_t ws_bytes, void *stream);

/* One new token per sequence over the compressed cache: the same operator as
 * cca_prefill_forward evaluated for the next position only, reading the cached latent keys
 * and values that decoding streams (gist.science explainer, 1. Problem Statement; Extension:
 * CCGQA: the grouped latent cache is what shrinks).
 * x [batch, E] -> y [batch, E], batch = cache->batch.
 * The token's key/value are appended at position lengths[b], its query attends to
 * positions 0..lengths[b], the conv / value-shift state advance and lengths[b] += 1.
 * A sequence already holding max_seq tokens is left untouched, its y row is zero and the
 * cache status word is set to CCA_ERR_CACHE_FULL (read it with cca_cache_check).  The decode
 * kernels take at most 8 query heads per kv head (CCA_ERR_UNSUPPORTED otherwise).  A new
 * latent key or value beyond the float16 range sets it to CCA_ERR_RANGE.
 * Where the stencil runs inside the attention kernel (bfloat16 layers, d~ <= 32, keys unsplit:
 * cca_decode_kernel_count == 3), each CTA of that kernel holds 256 tensor-memory columns of its
 * SM while it buffers the first cache rows; a kernel of another stream that allocates tensor
 * memory on the same SM meanwhile waits for them to be released.
 * Errors (host): INVALID_ARG, UNSUPPORTED, WORKSPACE, ALIGNMENT, CUDA. */
CCA_API int cca_decode_step(const cca_config_t *cfg, const cca_weights_t *w, const void *x,
                            void *y, cca_cache_t *cache, void *workspace, size_t ws_bytes,
                            void *stream);

/* cca_decode_step without a caller workspace; it allocates nothing.  (The paper has no
 * counterpart: this exists for callers.)  Meant for callers that cannot allocate device
 * memory on their decode path, e.g. a serving loop whose memory is fixed at start-up, or a
 * program running under another framework's allocator that it does not control.  Inputs,
 * outputs, weights and the cache are the caller's as in cca_decode_step; the step's scratch
 * lives in an 8 MiB array built into the library, held by every GPU that loads the library
 * until the process exits.  A step that needs more scratch (cca_decode_workspace_size above
 * 8 MiB, e.g. more than 451 sequences of 16 heads with d~ = 32 and 4 kv heads) is rejected
 * with CCA_ERR_WORKSPACE before anything is launched.  The first call on each device looks
 * up the array's device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture.  Every call uses the same array and leaves its
 * contents there; nothing in it needs to start at zero, but two calls whose kernels overlap
 * on the GPU (different streams without ordering) race on it.  The looked-up address is kept
 * for the life of the process: after cudaDeviceReset on a device, this entry point must not be
 * called again on that device.  Errors as cca_decode_step. */
CCA_API int cca_decode_step_static(const cca_config_t *cfg, const cca_weights_t *w,
                                   const void *x, void *y, cca_cache_t *cache, void *stream);

/* Scratch bytes needed by cca_backward (0 if the config is invalid or outside what the
 * backward kernels take). */
CCA_API size_t cca_backward_workspace_size(const cca_config_t *cfg, int batch, int seq);

/* Backward pass of the layer for `batch` sequences of `seq` tokens from position 0 (the pages
 * measure it against MHA's: gist.science explainer, 4. Experimental Results, "Backward Pass").
 * Given x [batch, seq, E] and dy = dL/dy [batch, seq, E] (bfloat16), writes
 *   dx         [batch, seq, E] bfloat16
 *   dw_qkv     [n_q + 2 n_kv, E] float32     dw_o [E, n_q] float32
 *   dconv_seq  [n_q + n_kv, conv_kernel] float32
 *   dconv_chan [H + Hkv, d~, d~, 1] float32
 * (every output overwritten).  The forward's intermediates are recomputed in the workspace (the
 * projections, the latents, the attention output and its per-row log-sum-exp); then the
 * gradient of the up-projection, the attention's backward pass (probabilities recomputed from
 * the log-sum-exp), the stencil's (RoPE, norm, Q-K-Mean, value-shift and both convolutions
 * taken back), and the down-projection's.  With tp_size > 1 the gradients are the rank's, and
 * dx is the rank's share (the caller sums it over the ranks).  bfloat16 layers with the
 * convolutions, d~ in {16, 32, 64}, conv_kernel <= 8, (H/Hkv + 1) d~^2 <= 20480,
 * (H/Hkv + 2) d~ <= 2048, E % 8 == 0, and the stencil backward's per-CTA tiles within 200 KB of
 * shared memory (CCA_ERR_UNSUPPORTED otherwise; cca_backward_workspace_size returns 0 then).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, ALIGNMENT, CUDA. */
CCA_API int cca_backward(const cca_config_t *cfg, const cca_weights_t *w, const void *x,
                         const void *dy, int batch, int seq, void *dx, float *dw_qkv,
                         float *dw_o, float *dconv_seq, float *dconv_chan, void *workspace,
                         size_t ws_bytes, void *stream);

/* Waits for `stream`, then returns the cache's sticky status word (CCA_OK or
 * CCA_ERR_CACHE_FULL) and clears it. */
CCA_API int cca_cache_check(cca_cache_t *cache, void *stream);

/* Text of the calling thread's last error ("" if none). */
CCA_API const char *cca_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* CCA_H */
