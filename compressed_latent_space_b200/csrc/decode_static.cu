// cca_decode_step_static: the decode step with its scratch in a fixed device array that is
// part of this library, for callers that cannot hand the library a workspace.
//
// Some callers cannot allocate device memory on their decode path: a serving loop whose
// memory is planned once at start-up and must not grow per request, a host program that
// runs inside another framework's allocator it does not control, or code called back from a
// context where an allocation could block or fail at an arbitrary moment.  Such a caller
// still owns the inputs, outputs, weights and the cache; only the decode step's scratch
// (partial projections, the new queries, split-KV partial results, the merged attention
// output) moves into `g_decode_scratch` below.
//
// The array holds kStaticScratchBytes (8 MiB) on each GPU; every GPU that loads the library
// keeps it until the process exits.  In host code `g_decode_scratch` names a host-side
// stand-in, not device memory, so its device address is looked up with cudaGetSymbolAddress,
// once per device, with that device current, on the first call made on that device.
#include <stdio.h>

#include <mutex>

#include "cca.h"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" CCA_API int cca_decode_step_static(const cca_config_t *cfg, const cca_weights_t *w,
                                              const void *x, void *y, cca_cache_t *cache,
                                              void *stream) {
  if (!cfg || !cache)
    return cca::set_last_error(CCA_ERR_INVALID_ARG, "config or cache is NULL");
  const size_t need = cca_decode_workspace_size(cfg, cache->batch, cache->max_seq);
  if (need == 0)   // invalid config or cache shape: the regular entry point names the problem
    return cca_decode_step(cfg, w, x, y, cache, nullptr, 0, stream);
  if (need > kStaticScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "this decode step needs %zu bytes of scratch; the built-in array holds %zu "
             "(use cca_decode_step with a caller workspace)",
             need, kStaticScratchBytes);
    return cca::set_last_error(CCA_ERR_WORKSPACE, msg);
  }
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cca::set_last_error(CCA_ERR_CUDA, cudaGetErrorString(e));
  if (device < 0 || device >= kMaxDevices)
    return cca::set_last_error(CCA_ERR_UNSUPPORTED, "device index beyond 63");
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_ptr[device]) {
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_decode_scratch);
      if (e != cudaSuccess) return cca::set_last_error(CCA_ERR_CUDA, cudaGetErrorString(e));
      g_scratch_ptr[device] = p;
    }
    scratch = g_scratch_ptr[device];
  }
  // Nothing in the scratch has to start at zero: every byte a decode step reads there was
  // written earlier in the same step.
  return cca_decode_step(cfg, w, x, y, cache, scratch, kStaticScratchBytes, stream);
}
