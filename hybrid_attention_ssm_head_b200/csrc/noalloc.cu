// Decode step without a caller-provided workspace: its scratch lives in a
// file-scope device buffer, so the call allocates nothing.
#include <cuda.h>

#include <mutex>

#include "kernels.h"

namespace {

// The scratch buffer.  In host code this name is a host-side stand-in, not a
// device address: the address kernels may use comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[HYMBA_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// The address is looked up once per device and CUDA context: a context torn down and
// created again (cudaDeviceReset) maps the module afresh, so the cached address is
// re-derived whenever the current context is not the one it was taken in.
void *g_scratch_addr[kMaxDevices] = {};
void *g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
void *current_context() {
  static std::once_flag once;
  static CtxGetCurrentFn fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

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
    // the runtime makes the device's primary context current on its first call above
    void *ctx = current_context();
    if (!g_scratch_addr[dev] || ctx != g_scratch_ctx[dev]) {
      void *p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
      if (e != cudaSuccess || !p) {
        hymba::set_error("cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
        return HYMBA_ERR_CUDA;
      }
      g_scratch_addr[dev] = p;
      g_scratch_ctx[dev] = ctx;
    }
    scratch = g_scratch_addr[dev];
  }
  return hymba_layer_decode_step(layer, batch, pos, x_t, y_t, kv_cache, ssm_cache, scratch,
                                 HYMBA_DECODE_STATIC_SCRATCH_BYTES, stream);
}
