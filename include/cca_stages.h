/*
 * cca_stages.h -- the kernels of the CCA forward one at a time, for per-stage testing and
 * timing.  Same conventions as cca.h (caller-owned device memory, asynchronous on
 * `stream`, host-side validation, CCA_* status codes).  `status` is an optional device
 * int (may be NULL) in which a kernel whose bounded wait ran out records a nonzero code.
 */
#ifndef CCA_STAGES_H
#define CCA_STAGES_H

#include "cca.h"

#ifdef __cplusplus
extern "C" {
#endif

/* C[m, n] = sum_k A[m, k] * B[n, k]  (A [M, K], B [N, K], C [M, N], all row-major; A and B
 * of `dtype`, C of `out_dtype`).  bf16 or f16 operands run on the tcgen05 tensor-core kernel
 * (K % 8 == 0, result bf16 or float32), float32 operands on CUDA cores (result float32).
 * This is the contraction of the down-projection (x W_qkv^T) and of the up-projection
 * (o W_o^T) of the layer (gist.science explainer, 2. Methodology, Core Mechanism,
 * "Down-Projection"). */
CCA_API int cca_gemm(int dtype, int out_dtype, const void *A, const void *B, void *C, int M,
                     int N, int K, int *status, void *stream);

/* The same contraction on bfloat16 operands either of which may be stored transposed:
 * C[m, n] = sum_k A'[m, k] * B'[n, k] with A' = A [M, K] (a_trans == 0) or A stored [K, M]
 * (a_trans == 1), B' = B [N, K] (b_trans == 0) or B stored [K, N] (b_trans == 1); C [M, N]
 * float32 (out_dtype CCA_F32) or bfloat16.  The contiguous extent of each operand (K, or M /
 * N when transposed) must be a multiple of 8.  The backward pass's gradient products
 * (dx = dP W_qkv, dW_qkv = dP^T x, dW_o = dy^T o) read their operands this way, untransposed
 * in memory.  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED (extents), CUDA. */
CCA_API int cca_gemm_t(int out_dtype, const void *A, const void *B, void *C, int M, int N, int K,
                       int a_trans, int b_trans, int *status, void *stream);

/* Latent stencil: P [batch*seq, n_q + 2 n_kv] (the projections, float32) ->
 * q [batch, H, seq, d~], k and v [batch, Hkv, kv_stride, d~] with kv_stride >= seq
 * (q, k and v of the latent element type of cca.h: float16 for bfloat16 layers).
 * Sequence conv, channel conv, q-k-mean, value-shift, RMS norm and RoPE (positions 0..seq-1),
 * as selected by cfg->flags (gist.science explainer, 2. Methodology, Core Mechanism). */
CCA_API int cca_stage_stencil(const cca_config_t *cfg, const void *P, int batch, int seq,
                              const float *conv_seq, const float *conv_chan, void *q, void *k,
                              void *v, int kv_stride, void *workspace, size_t ws_bytes,
                              void *stream);

/* Scratch bytes cca_stage_stencil needs (its first 256 bytes are a status word read by
 * cca_workspace_status; the rest holds the channel-conv weights split for the tensor cores). */
CCA_API size_t cca_stage_stencil_workspace_size(const cca_config_t *cfg);

/* Causal latent attention: q [batch, H, seq, d~], k/v [batch, Hkv, kv_stride, d~] ->
 * o [batch*seq, H*d~] (token-major; q, k, v and o of the latent element type of cca.h), scale 1/sqrt(d~), query head h reads kv head
 * h / (H/Hkv) (gist.science/de explainer, 2. Methodik: Softmax(QK^T)V in the compressed
 * space; gist.science explainer, Extension: CCGQA). */
CCA_API int cca_stage_attention(const cca_config_t *cfg, const void *q, const void *k,
                                const void *v, int batch, int seq, int kv_stride, void *o,
                                int *status, void *stream);

/* Waits for `stream` and returns CCA_OK, CCA_ERR_RANGE if the last cca_prefill_forward
 * that used this workspace met a latent beyond the float16 range, or CCA_ERR_DEVICE if one
 * of its kernels recorded an internal error. */
CCA_API int cca_workspace_status(const void *workspace, void *stream);

/* y[i] = 2^x[i] for i < n (n even; x, y caller-owned device float32 arrays, enqueued on
 * `stream`) by the cubic on the FMA pipes that the latent attention uses for part of its
 * softmax probabilities (gist.science/de explainer, 2. Methodik: Softmax(QK^T)V): x = n + f,
 * f in [-1/2, 1/2], 2^f by the minimax cubic under relative error, 2^n into the exponent;
 * relative error below 1e-4 for x in [-125, 126], arguments below -125 treated as -125.
 * Errors: INVALID_ARG (odd or negative n, NULL pointers), CUDA (launch). */
CCA_API int cca_stage_exp2_poly(const float *x, float *y, int n, void *stream);

/* Failure-detection diagnostic (the paper has no counterpart).  Launches one CTA that runs
 * the bounded mbarrier wait of the tcgen05 kernels on a shared-memory barrier, with a limit of
 * limit_ns nanoseconds (1e3 .. 1e9) instead of the kernels' 2 s.  arm == 0: nothing ever
 * arrives on the barrier, so the wait gives up after the limit, writes DEV_WAIT_TIMEOUT (1) to
 * *status (a caller-owned device int, expected to hold 0) and the kernel returns; the context
 * stays usable.  arm != 0: one thread arrives first, the wait completes and *status is left
 * unchanged.  Errors: INVALID_ARG (limit out of range, status NULL), CUDA (launch). */
CCA_API int cca_stage_wait_probe(long long limit_ns, int arm, int *status, void *stream);

/* Per-kernel timing for benchmarks.  cca_stage_timing(1) starts a session: from then on
 * every cca_prefill_forward / cca_decode_step records a CUDA event on its stream before its
 * first kernel and after each kernel (events only; nothing else changes).
 * cca_stage_timing(0) ends recording.  cca_stage_times waits for the recorded events and
 * writes, for up to n kernels of the recorded calls (in launch order), the summed
 * milliseconds to ms[] and the number of recorded calls to *calls; it returns the number
 * of kernel slots per call.  Recording holds at most 4096 calls. */
CCA_API int cca_stage_timing(int enable);
CCA_API int cca_stage_times(double *ms, int n, int *calls);

#ifdef __cplusplus
}
#endif

#endif /* CCA_STAGES_H */
