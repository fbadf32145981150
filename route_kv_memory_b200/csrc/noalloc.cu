// mka_session_ema_noalloc: the L2 session-memory EMA for callers that cannot
// allocate device memory.
//
// mka_session_ema needs a caller-provided scratch buffer (per-chunk EMA end
// states and carries).  Some host programs cannot provide one: a plugin running
// inside a host application whose memory manager owns every device allocation
// and does not let plugins call cudaMalloc, or a caller whose device memory is
// fully reserved up front.  This variant takes its scratch from a fixed array
// that lives in the library's own device image instead.
#include <mutex>
#include <stdio.h>

#include "../../include/mka.h"
#include "kernels.h"

namespace {

// The scratch: every GPU that loads the library holds these bytes until the
// process exits.  All calls share it, so calls that overlap on the GPU (two
// streams, two host threads) race on it and must be serialised by the caller.
// Each call writes every scratch byte it reads before reading it, so nothing
// needs clearing between calls.
__device__ __align__(256) unsigned char g_ema_scratch[MKA_NOALLOC_SCRATCH_BYTES];

// Host code may not use g_ema_scratch as a device address (in host code the
// name is a host-side stand-in).  Its device address is looked up once per
// device, with that device current, and cached.  The address belongs to the
// device's primary context: the cache does not follow cudaDeviceReset or a
// non-primary context, which load the image again elsewhere.
void* scratch_address(int* err) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) {
    char msg[160];
    snprintf(msg, sizeof(msg), "mka_session_ema_noalloc: no usable CUDA device (%s)", cudaGetErrorString(e));
    *err = mka::set_last_error(MKA_ERR_CUDA, msg);
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_ema_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[160];
      snprintf(msg, sizeof(msg), "mka_session_ema_noalloc: cudaGetSymbolAddress failed (%s)", cudaGetErrorString(e));
      *err = mka::set_last_error(MKA_ERR_CUDA, msg);
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" {

int mka_session_ema_noalloc(const mka_config* cfg, const void* x, const float* carry_in, float* m2, float* carry_out,
                            void* stream) {
  size_t need = mka_session_ema_workspace_size(cfg);
  if (need > (size_t)MKA_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "mka_session_ema_noalloc: this shape needs %zu bytes of scratch, the built-in scratch holds %zu; "
             "use mka_session_ema with a caller buffer", need, (size_t)MKA_NOALLOC_SCRATCH_BYTES);
    return mka::set_last_error(MKA_ERR_WORKSPACE, msg);
  }
  int err = MKA_OK;
  void* ws = scratch_address(&err);
  if (!ws) return err;
  // need == 0 means an invalid cfg: mka_session_ema reports which field.
  return mka_session_ema(cfg, x, carry_in, m2, carry_out, ws, (size_t)MKA_NOALLOC_SCRATCH_BYTES, stream);
}

}  // extern "C"
