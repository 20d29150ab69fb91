// Stage entry of the attention's FMA-pipe exponential (ex2_poly2), so that its error bound is
// tested on the device, and the diagnostic of the kernels' failure detection: one CTA runs the same bounded mbarrier wait
// the tcgen05 kernels use, on a barrier that nothing arrives on unless the caller asks for it,
// with a limit the caller chooses.  It shows, on the device, that a wait which can never
// complete gives up after its limit, records DEV_WAIT_TIMEOUT in the status word and lets the
// kernel return, so the context stays usable.  (The paper has no counterpart.)
#include "cca_stages.h"
#include "common.cuh"
#include "kernels.h"

namespace cca {
namespace {

__global__ void wait_probe_kernel(unsigned long long limit_ns, int arm, int *status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (arm && threadIdx.x == 0) mbar_arrive(&bar);   // completes phase 0: the wait succeeds
  __syncwarp();
  mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
  __syncthreads();
}

__global__ void exp2_poly_kernel(const float *__restrict__ x, float *__restrict__ y, int npairs) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < npairs; i += gridDim.x * blockDim.x) {
    float p0, p1;
    ex2_poly2(f2(x[2 * i], x[2 * i + 1]), p0, p1);
    y[2 * i] = p0;
    y[2 * i + 1] = p1;
  }
}

}  // namespace
}  // namespace cca

extern "C" CCA_API int cca_stage_exp2_poly(const float *x, float *y, int n, void *stream) {
  if (n < 0 || (n & 1)) return cca::set_last_error(CCA_ERR_INVALID_ARG, "n must be even and >= 0");
  if (n > 0 && (!x || !y)) return cca::set_last_error(CCA_ERR_INVALID_ARG, "x or y is NULL");
  if (n > 0) {
    const int pairs = n / 2, blocks = (pairs + 255) / 256 < 1024 ? (pairs + 255) / 256 : 1024;
    cca::exp2_poly_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, pairs);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cca::set_last_error(CCA_ERR_CUDA, cudaGetErrorString(e));
  }
  return cca::set_last_error(CCA_OK, "");
}

extern "C" CCA_API int cca_stage_wait_probe(long long limit_ns, int arm, int *status,
                                            void *stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000LL)
    return cca::set_last_error(CCA_ERR_INVALID_ARG, "limit_ns must be in [1e3, 1e9]");
  if (!status) return cca::set_last_error(CCA_ERR_INVALID_ARG, "status is NULL");
  cca::wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_ns), arm ? 1 : 0, status);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cca::set_last_error(CCA_ERR_CUDA, cudaGetErrorString(e));
  return cca::set_last_error(CCA_OK, "");
}
