// Projection GEMM on the 5th-generation tensor cores: C[M,N] = A[M,K] * B[N,K]^T.
//
// Used for the down-projection x W_qkv^T and the up-projection o W_o^T of the layer
// (gist.science explainer, 2. Methodology, Core Mechanism: "Down-Projection"; the result of
// the latent attention returns to width E through one output matrix), and for the backward
// pass's gradient products.  Operands are K-major (PyTorch Linear layout) or, per operand,
// MN-major (stored [K][M] / [K][N], as a row-major activation is for a product over its
// rows), bf16 or f16, accumulated in fp32 in tensor memory.  An MN-major tile is TMA-loaded
// as 64-element (128-byte) column chunks of 64 K rows in the 128-byte swizzle, which is the
// UMMA MN-major layout with the chunks LBO = 8 KB apart and 8-row groups SBO = 1 KB apart.
//
// Persistent, warp-specialised kernel, one CTA per SM:
//   warp 0  : TMA producer, 4-stage ring of 128x64 (A) + 256x64 (B) tiles, 128B swizzle
//   warp 1  : allocates 512 TMEM columns (two 128x256 fp32 accumulators) and issues
//             tcgen05.mma (M=128, N=256, K=16) from one thread
//   warps 2-5: epilogue, tcgen05.ld of its 32-lane quadrant, convert, store
// The epilogue of tile i overlaps the main loop of tile i+1 (double-buffered accumulator).
// Every wait is bounded (see mbar_wait); a timeout sets the status word and the CTA exits
// after releasing its tensor memory.
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;

struct Bars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  int abort;
};
constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + sizeof(Bars);

constexpr int MN_CHUNK_BYTES = 64 * BK * 2;         // one 64-element MN chunk of a stage

template <typename OutT, int AB_F16, int A_MN, int B_MN>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap mapA,
                     const __grid_constant__ CUtensorMap mapB, OutT *__restrict__ C,
                     int M, int N, int K, int *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = ((M + BM - 1) / BM) * n_tiles;
  const int num_kb = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->tfull[a], 1);
      mbar_init(&bars->tempty[a], 4);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int *abort = &bars->abort;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int m0 = (tile / n_tiles) * BM;
        const int n0 = (tile % n_tiles) * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&bars->empty[stage], phase ^ 1u, abort, status)) { ok = false; break; }
          uint8_t *sa = smem + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&bars->full[stage], STAGE_BYTES);
          if constexpr (A_MN) {
#pragma unroll
            for (int c = 0; c < BM / 64; ++c)
              tma_load_2d(sa + c * MN_CHUNK_BYTES, &mapA, &bars->full[stage], m0 + 64 * c, kb * BK);
          } else {
            tma_load_2d(sa, &mapA, &bars->full[stage], kb * BK, m0);
          }
          if constexpr (B_MN) {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c)
              tma_load_2d(sa + A_BYTES + c * MN_CHUNK_BYTES, &mapB, &bars->full[stage], n0 + 64 * c,
                          kb * BK);
          } else {
            tma_load_2d(sa + A_BYTES, &mapB, &bars->full[stage], kb * BK, n0);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN, A_MN, B_MN, AB_F16);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        if (!mbar_wait(&bars->tempty[acc], aphase ^ 1u, abort, status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&bars->full[stage], phase, abort, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // K-major: 16 K elements are 32 bytes along the row; MN-major: 16 K rows are two
            // 8-row (1 KB) groups
            const uint64_t ad = A_MN ? smem_desc(a_addr + k * 2048, MN_CHUNK_BYTES, 1024, 2)
                                     : smem_desc(a_addr + k * 32, 16, 1024, 2);
            const uint64_t bd = B_MN ? smem_desc(b_addr + k * 2048, MN_CHUNK_BYTES, 1024, 2)
                                     : smem_desc(b_addr + k * 32, 16, 1024, 2);
            umma_f16_ss(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&bars->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit(&bars->tfull[acc]);
      }
    }
  } else {
    // Epilogue: warp w may only touch TMEM lanes 32*(w%4) .. 32*(w%4)+31.
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    int local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      const bool got = mbar_wait(&bars->tfull[acc], aphase, abort, status);
      if (!__all_sync(0xffffffffu, got)) break;   // also reconverges the warp for tcgen05.ld
      tc_fence_after();
      const int m = (tile / n_tiles) * BM + row;
      const int n0 = (tile % n_tiles) * BN;
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + ((quad * 32) << 16) + acc * BN + c * 32, r);
        tmem_ld_wait();
        if (c == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->tempty[acc]);
        }
        const int n = n0 + c * 32;
        if (m < M && n < N) {
          OutT *dst = C + static_cast<size_t>(m) * N + n;
          if (n + 32 <= N && (N & 7) == 0) {
            if constexpr (sizeof(OutT) == 2) {
              constexpr bool kHalf = std::is_same<OutT, __half>::value;
              auto pk = [](float a, float b2) { return kHalf ? pack_f16x2(a, b2) : pack_bf16x2(a, b2); };
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint4 u;
                u.x = pk(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                u.y = pk(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                u.z = pk(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                u.w = pk(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                reinterpret_cast<uint4 *>(dst)[v] = u;
              }
            } else {
#pragma unroll
              for (int v = 0; v < 8; ++v)
                reinterpret_cast<uint4 *>(dst)[v] =
                    make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < N) dst[j] = from_f32<OutT>(__uint_as_float(r[j]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 row-major tensor [rows, cols] -> box [box_rows, 64 cols], 128B swizzle (a
// K-major operand: box_rows MN rows of 64 K; an MN-major one: 64 K rows of 64 MN columns).
bool make_map_2d(CUtensorMap *map, const void *ptr, int rows, int cols, int box_rows, int f16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <typename OutT, int AB_F16, int A_MN = 0, int B_MN = 0>
static cudaError_t launch_gemm(const CUtensorMap &ma, const CUtensorMap &mb, void *C, int M,
                               int N, int K, int *status, cudaStream_t st) {
  if (cudaError_t e = ensure_dyn_smem<gemm_bf16_kernel<OutT, AB_F16, A_MN, B_MN>>(SMEM_BYTES);
      e != cudaSuccess)
    return e;
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  gemm_bf16_kernel<OutT, AB_F16, A_MN, B_MN><<<grid, THREADS, SMEM_BYTES, st>>>(
      ma, mb, static_cast<OutT *>(C), M, N, K, status);
  return cudaGetLastError();
}

cudaError_t gemm_tcgen05_t(const void *A, const void *B, void *C, int M, int N, int K, int a_mn,
                           int b_mn, int out_f32, int *status, cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  // every TMA row pitch a multiple of 16 bytes: the contiguous extent of each operand % 8
  if ((a_mn ? M : K) % 8 != 0 || (b_mn ? N : K) % 8 != 0) return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  const bool okA = a_mn ? make_map_2d(&ma, A, K, M, BK, 0) : make_map_2d(&ma, A, M, K, BM, 0);
  const bool okB = b_mn ? make_map_2d(&mb, B, K, N, BK, 0) : make_map_2d(&mb, B, N, K, BN, 0);
  if (!okA || !okB) return cudaErrorInvalidValue;
  const int sel = (a_mn ? 2 : 0) + (b_mn ? 1 : 0);
  if (out_f32) {
    switch (sel) {
      case 0: return launch_gemm<float, 0, 0, 0>(ma, mb, C, M, N, K, status, st);
      case 1: return launch_gemm<float, 0, 0, 1>(ma, mb, C, M, N, K, status, st);
      case 2: return launch_gemm<float, 0, 1, 0>(ma, mb, C, M, N, K, status, st);
      default: return launch_gemm<float, 0, 1, 1>(ma, mb, C, M, N, K, status, st);
    }
  }
  switch (sel) {
    case 0: return launch_gemm<__nv_bfloat16, 0, 0, 0>(ma, mb, C, M, N, K, status, st);
    case 1: return launch_gemm<__nv_bfloat16, 0, 0, 1>(ma, mb, C, M, N, K, status, st);
    case 2: return launch_gemm<__nv_bfloat16, 0, 1, 0>(ma, mb, C, M, N, K, status, st);
    default: return launch_gemm<__nv_bfloat16, 0, 1, 1>(ma, mb, C, M, N, K, status, st);
  }
}

cudaError_t gemm_tcgen05_f16out(const void *A, const void *B, void *C, int M, int N, int K,
                                int ab_f16, int *status, cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (K % 8 != 0) return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  if (!make_map_2d(&ma, A, M, K, BM, ab_f16) || !make_map_2d(&mb, B, N, K, BN, ab_f16))
    return cudaErrorInvalidValue;
  return ab_f16 ? launch_gemm<__half, 1>(ma, mb, C, M, N, K, status, st)
                : launch_gemm<__half, 0>(ma, mb, C, M, N, K, status, st);
}

cudaError_t gemm_tcgen05(const void *A, const void *B, void *C, int M, int N, int K, int ab_f16,
                         int out_f32, int *status, cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (K % 8 != 0) return cudaErrorInvalidValue;   // TMA row pitch must be a multiple of 16 B
  CUtensorMap ma, mb;
  if (!make_map_2d(&ma, A, M, K, BM, ab_f16) || !make_map_2d(&mb, B, N, K, BN, ab_f16))
    return cudaErrorInvalidValue;
  if (ab_f16)
    return out_f32 ? launch_gemm<float, 1>(ma, mb, C, M, N, K, status, st)
                   : launch_gemm<__nv_bfloat16, 1>(ma, mb, C, M, N, K, status, st);
  return out_f32 ? launch_gemm<float, 0>(ma, mb, C, M, N, K, status, st)
                 : launch_gemm<__nv_bfloat16, 0>(ma, mb, C, M, N, K, status, st);
}

}  // namespace cca

namespace cca {
namespace {

__global__ void __launch_bounds__(256) bf16_to_f16_kernel(const __nv_bfloat16 *__restrict__ src,
                                                          __half *__restrict__ dst, size_t n8,
                                                          int *status) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float v[8];
    load8(src + i * 8, v);
    bool ok = true;
#pragma unroll
    for (int e = 0; e < 8; ++e) ok = ok && (fabsf(v[e]) <= kF16Max);
    if (!ok) report(status, DEV_RANGE);
    uint4 u;
    u.x = pack_f16x2(v[0], v[1]);
    u.y = pack_f16x2(v[2], v[3]);
    u.z = pack_f16x2(v[4], v[5]);
    u.w = pack_f16x2(v[6], v[7]);
    reinterpret_cast<uint4 *>(dst)[i] = u;
  }
}

__global__ void __launch_bounds__(256) f16_to_bf16_kernel(const __half *__restrict__ src,
                                                          __nv_bfloat16 *__restrict__ dst, size_t n8) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4 *>(src)[i];
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
    uint4 o;
    uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h[e]);
      ow[e] = pack_bf16x2(f.x, f.y);
    }
    reinterpret_cast<uint4 *>(dst)[i] = o;
  }
}

}  // namespace

cudaError_t convert_f16_to_bf16(const void *src, void *dst, size_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  if (n % 8) return cudaErrorInvalidValue;
  const size_t n8 = n / 8;
  size_t blocks = (n8 + 255) / 256;
  const size_t cap = static_cast<size_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  f16_to_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      static_cast<const __half *>(src), static_cast<__nv_bfloat16 *>(dst), n8);
  return cudaGetLastError();
}

cudaError_t convert_bf16_to_f16(const void *src, void *dst, size_t n, int *status, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  if (n % 8) return cudaErrorInvalidValue;
  const size_t n8 = n / 8;
  size_t blocks = (n8 + 255) / 256;
  const size_t cap = static_cast<size_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  bf16_to_f16_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      static_cast<const __nv_bfloat16 *>(src), static_cast<__half *>(dst), n8, status);
  return cudaGetLastError();
}

}  // namespace cca

namespace cca {

bool make_tma_16bit(CUtensorMap *map, const void *ptr, int rank, const uint64_t *dims,
                    const uint64_t *strides_bytes, const uint32_t *box, int swizzle_bytes,
                    int f16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) s[i] = strides_bytes[i];
  }
  const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  rank, const_cast<void *>(ptr), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace cca
