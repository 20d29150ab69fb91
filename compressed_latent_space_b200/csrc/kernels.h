// Host-side launchers of the CCA kernels (internal to libcca; not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace cca {

// Shape of one layer plus the switches, as the kernels consume it.
struct Dims {
  int B = 0, S = 0;              // batch, tokens per sequence (prefill)
  int E = 0, H = 0, Hkv = 0;     // d_model, query heads, key/value heads
  int G = 0, DL = 0;             // group size H/Hkv, latent head width
  int NQ = 0, NKV = 0, NQKV = 0; // H*DL, Hkv*DL, NQ + 2*NKV
  int KC = 0;                    // sequence-conv taps
  int VS0 = 0;                   // first value channel taken from the previous token (value-shift)
  unsigned flags = 0;
  float eps = 1e-6f;
  float rope_base = 10000.f;
  int bf16 = 1;                  // activations and weights bf16 (latents and cache float16)
};

// Called after each kernel launch of a C-ABI call; records a timing event when stage
// timing is on (see cca_stage_timing).
struct StageMarker {
  void *ctx = nullptr;
  void (*fn)(void *) = nullptr;
  void operator()() const {
    if (fn) fn(ctx);
  }
};

enum : unsigned { F_QK_MEAN = 1u, F_VALUE_SHIFT = 2u, F_QK_NORM = 4u, F_ROPE = 8u, F_NO_CONV = 16u };

// C[M, N] = A[M, K] * B[N, K]^T, bf16 (or f16 with ab_f16) in, fp32 accumulate, bf16 or fp32
// out (tcgen05 + TMA).
cudaError_t gemm_tcgen05(const void *A, const void *B, void *C, int M, int N, int K, int ab_f16,
                         int out_f32, int *status, cudaStream_t st);
// C[M, N] = sum_k A'[m, k] B'[n, k] on bf16 operands, A' = A [M, K] (a_mn == 0) or the
// transpose of A stored [K, M] (a_mn == 1), B' likewise ([N, K] or [K, N]); fp32 or bf16 out.
// The contiguous extent of each operand must be a multiple of 8.
cudaError_t gemm_tcgen05_t(const void *A, const void *B, void *C, int M, int N, int K, int a_mn,
                           int b_mn, int out_f32, int *status, cudaStream_t st);
// The same contraction with a float16 result (the backward pass's dO, an operand of the
// float16 attention-backward MMAs).
cudaError_t gemm_tcgen05_f16out(const void *A, const void *B, void *C, int M, int N, int K,
                                int ab_f16, int *status, cudaStream_t st);
// dst[i] = float16(src[i]) for a bf16 tensor of n elements (n % 8 == 0); a value beyond the
// float16 range records DEV_RANGE in *status.
cudaError_t convert_bf16_to_f16(const void *src, void *dst, size_t n, int *status, cudaStream_t st);
// dst[i] = bfloat16(src[i]) for a float16 tensor of n elements (n % 8 == 0).
cudaError_t convert_f16_to_bf16(const void *src, void *dst, size_t n, cudaStream_t st);
// Same contraction on CUDA cores; element type float (bf16 == 0) or bf16.
cudaError_t gemm_simt(int bf16, const void *A, const void *B, void *C, int M, int N, int K,
                      cudaStream_t st);

// Latent stencil of a prefill: P [B*S, NQKV] (float32) -> q [B, H, S, DL],
// k/v [B, Hkv, kv_stride, DL] (float16 for 16-bit layers) (kv_stride >= S: the cache's max_seq, or S for workspace
// buffers).  With write_state the last KC-1 pre-conv q|k rows and the last upper-half value
// row are stored (float32) and lengths[b] = S.
struct StencilArgs {
  const float *P;
  const float *conv_seq;
  const float *conv_chan;
  const void *conv_chan_split = nullptr;   // 16-bit layers: output of split_conv_chan
  void *q, *k, *v;
  int kv_stride;
  float *conv_state;    // [B, KC-1, NQ+NKV]
  float *vshift_state;  // [B, NKV - NKV/2]
  int *lengths;         // [B]
  int *status = nullptr;  // receives DEV_RANGE for a latent beyond the float16 range
  bool write_state = false;
};
cudaError_t latent_stencil(const Dims &d, const StencilArgs &a, cudaStream_t st);
// The channel-conv weights of a 16-bit layer as {bf16x2 hi, bf16x2 lo} per pair of inputs
// (conv_chan_split_bytes of scratch); the stencil's tensor-core path reads them.
size_t conv_chan_split_bytes(const Dims &d);
cudaError_t split_conv_chan(const Dims &d, const float *conv_chan, void *out, cudaStream_t st);

// Down-projection fused with the latent stencil (16-bit layers): x [B, S, E] and W_qkv ->
// q, k, v as latent_stencil writes them (and the decode state with write_state), without P
// ever reaching global memory.  fused_group_set: the key/value groups one CTA takes (0 when
// the shape is not supported by the fused kernel).  filt_hi / filt_lo: the channel filters as
// bf16 leading terms and remainders, [(H + Hkv) * DL, DL] each (split_filter_planes, into
// fused_filter_bytes of scratch).
struct FusedArgs {
  const void *x, *w_qkv;
  const float *conv_seq;
  const void *filt_hi, *filt_lo;
  void *q, *k, *v;
  int kv_stride;
  float *conv_state, *vshift_state;
  int *lengths;
  bool write_state;
  int *status;
};
int fused_group_set(const Dims &d);
size_t fused_filter_bytes(const Dims &d);
cudaError_t split_filter_planes(const Dims &d, const float *conv_chan, void *hi, void *lo,
                                cudaStream_t st);
cudaError_t fused_qkv_stencil(const Dims &d, const FusedArgs &a, cudaStream_t st);

// Causal latent attention: q [B, H, S, DL], k/v [B, Hkv, kv_stride, DL] -> o [B*S, NQ].
cudaError_t latent_attention(const Dims &d, const void *q, const void *k, const void *v,
                             int kv_stride, void *o, int *status, cudaStream_t st);
// The tcgen05 kernel behind latent_attention for 16-bit layers (float16 q, k, v, o).
// lse (optional, [B, H, S] float32): per query row, the log2-domain log-sum-exp of its scaled
// scores (the backward pass recomputes the probabilities from it).
cudaError_t latent_attention_tc(const Dims &d, const void *q, const void *k, const void *v,
                                int kv_stride, void *o, int *status, cudaStream_t st,
                                float *lse = nullptr);

// Backward pass of the latent attention (16-bit layers): q [B, H, S, DL], k / v
// [B, Hkv, kv_stride, DL], dO [B*S, NQ] (float16, the layout of the forward's o), lse [B, H, S]
// (from the forward), D = rowsum(dO * O) [B, H, S] -> dq [B, H, S, DL], dk / dv [B, Hkv, S, DL]
// (float32).
struct AttnBwdArgs {
  const void *q, *k, *v, *dO;
  int kv_stride;
  const float *lse, *D;
  float *dq, *dk, *dv;
  int *status;
};
cudaError_t latent_attention_backward(const Dims &d, const AttnBwdArgs &a, cudaStream_t st);
cudaError_t attention_rowdot(const Dims &d, const void *dO, const void *O, float *D,
                             cudaStream_t st);

// Backward pass of the latent stencil: P (the forward's projections), dq / dk / dv (float32,
// the attention backward's layouts) -> dP [B*S, NQKV] bfloat16, and the conv filters'
// gradients added to dconv_seq [NQ+NKV, KC] and dconv_chan [H+Hkv, DL, DL] (float32, zeroed by
// the caller).  dA and dPpart are float32 scratch, [B*S, NQ+NKV] and [B*S, NQKV].
struct StencilBwdArgs {
  const float *P, *dq, *dk, *dv, *conv_seq, *conv_chan;
  const void *conv_chan_split;     // split_conv_chan's output for these filters
  void *conv_chan_split_t;         // scratch of conv_chan_split_bytes: the transposed split
  float *dA, *dPpart;
  void *dP;
  float *dconv_seq, *dconv_chan;
};
bool stencil_backward_supported(const Dims &d);
cudaError_t stencil_backward(const Dims &d, const StencilBwdArgs &a, cudaStream_t st);
// out[c][r] = in[r][c] for 16-bit elements ([R, C] -> [C, R8], rows R..R8-1 of the output
// zero), float16 converted to bfloat16 when from_f16.
cudaError_t transpose16(const void *in, void *out, int R, int C, int R8, bool from_f16,
                        cudaStream_t st);

// Decode step kernels.
struct DecodeArgs {
  const void *x;            // [B, E]
  const void *w_qkv;        // [NQKV, E]
  const void *w_o;          // [E, NQ]
  const float *conv_seq;
  const float *conv_chan;
  void *y;                  // [B, E]
  void *k_cache, *v_cache;  // [B, Hkv, max_seq, DL]
  float *conv_state;        // [B, KC-1, NQ+NKV]
  float *vshift_state;      // [B, NKV - NKV/2]
  int *lengths;             // [B]
  int *status;              // cache status word
  int max_seq;
  // workspace
  float *p_part;            // [ksplit, B, NQKV]
  float *q_new;             // [B, H, DL]
  float *part_o;            // [B, H, nchunk, DL]
  float *part_ml;           // [B, H, nchunk, 2]
  void *o;                  // [B, NQ]
  int ksplit;
  int nchunk;
  int chunk;
};
size_t decode_workspace_bytes(const Dims &d, int max_seq);
int decode_kernel_count(const Dims &d, int max_seq);
void decode_workspace_carve(const Dims &d, int max_seq, void *ws, DecodeArgs &a);
cudaError_t decode_step(const Dims &d, const DecodeArgs &a, cudaStream_t st,
                        const StageMarker &mark);

int num_sms();

// Tiled TMA descriptor of a 16-bit tensor of `rank` dims (dims[0] innermost, in elements;
// strides_bytes[i] is the byte stride of dim i+1), box in elements, swizzle span in bytes
// (0, 32, 64 or 128); out-of-range elements of a box read as zero.
bool make_tma_16bit(CUtensorMap *map, const void *ptr, int rank, const uint64_t *dims,
                    const uint64_t *strides_bytes, const uint32_t *box, int swizzle_bytes,
                    int f16);

// Records `msg` as the calling thread's last error (cca_last_error_string) and returns `code`.
int set_last_error(int code, const char *msg);

}  // namespace cca
