// noalloc.cu -- latent attention over a contiguous cache for callers that cannot allocate
// device memory.  Such a caller may be a plugin inside a host runtime that owns all device
// memory and hands its plugins no workspace, or a runtime that fixes its memory plan at
// start-up and forbids any later allocation.  This entry point runs the same attend and
// combine kernels as mla_attend_dense, but takes its scratch from a fixed array compiled
// into the library instead of a caller-provided workspace.
#include <cuda_runtime.h>

#include "internal.h"
#include "mla.h"

namespace {

// 32 MiB of scratch: enough for mla_attend_workspace_bytes(B, Q, 64, 512) up to 32 MiB
// (for example B * Q up to about 100 on a 148-SM device).  The runtime reserves it on a
// device when it loads this file's code module there: with lazy module loading (the
// default), at the first cudaGetSymbolAddress below, i.e. the first call on that device.
// It is held until the process exits.
constexpr size_t kScratchBytes = size_t(32) << 20;
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of g_scratch on the current device.  In host code the name g_scratch is
// only a host-side stand-in for the symbol, so the address is looked up once per device
// (with that device current) and cached.
void *scratch_on_current_device(cudaError_t *err) {
  static void *addr[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *err = e;
    return nullptr;
  }
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) {
      *err = e;
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" mla_status mla_attend_dense_noalloc(const uint16_t *q_tilde, const uint16_t *cache,
                                               const int32_t *seq_lens, int B, int Q, int H, int R, int Lmax,
                                               float scale, uint16_t *o_latent, float *lse, int32_t *status,
                                               void *stream) {
  const size_t need = mla_attend_workspace_bytes(B, Q, H, R);
  if (need == 0) return (H != mla::kHeads || R != mla::kLatent) ? MLA_ERR_UNSUPPORTED : MLA_ERR_ARG;
  if (need > kScratchBytes) return MLA_ERR_WORKSPACE;
  cudaError_t err = cudaSuccess;
  void *ws = scratch_on_current_device(&err);
  if (ws == nullptr) return mla::record_cuda_error(err);
  return mla_attend_dense(q_tilde, cache, seq_lens, B, Q, H, R, Lmax, scale, ws, kScratchBytes, o_latent, lse,
                          status, stream);
}
