// Decode step without a caller-provided workspace: its scratch lives in a
// file-scope device buffer, so the call allocates nothing.
#include <mutex>

#include "kernels.h"

namespace {

// The scratch buffer.  In host code this name is a host-side stand-in, not a
// device address: the address kernels may use comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[HYMBA_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" HYMBA_API hymba_status hymba_layer_decode_step_static(hymba_layer *layer, int batch,
                                                                 int64_t pos, const void *x_t,
                                                                 void *y_t, hymba_kv_cache *kv_cache,
                                                                 hymba_ssm_cache *ssm_cache,
                                                                 hymba_stream_t stream) {
  size_t need = 0;
  hymba_status st = hymba_layer_decode_workspace(layer, batch, pos, &need);
  if (st != HYMBA_OK) return st;
  if (need > HYMBA_DECODE_STATIC_SCRATCH_BYTES) {
    hymba::set_error("this decode step needs %zu bytes of scratch; the static buffer holds %u "
                     "(use hymba_layer_decode_step with a workspace)",
                     need, HYMBA_DECODE_STATIC_SCRATCH_BYTES);
    return HYMBA_ERR_WORKSPACE;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    hymba::set_error("no current CUDA device");
    return HYMBA_ERR_DEVICE;
  }
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> g(g_mu);
    if (!g_scratch_addr[dev]) {
      void *p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
      if (e != cudaSuccess || !p) {
        hymba::set_error("cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
        return HYMBA_ERR_CUDA;
      }
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  return hymba_layer_decode_step(layer, batch, pos, x_t, y_t, kv_cache, ssm_cache, scratch,
                                 HYMBA_DECODE_STATIC_SCRATCH_BYTES, stream);
}
