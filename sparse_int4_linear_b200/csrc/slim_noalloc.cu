// slim_linear_noalloc: the forward for callers that cannot allocate device
// memory.  slim_linear needs a small scratch buffer for the adapter's
// T = X L product and asks the caller for it; some callers have no way to
// provide one (an engine plugin whose device memory is planned up front,
// code running where cudaMalloc is not allowed or would synchronize the
// device).  This variant keeps that scratch in a fixed-size array in the
// library's own device memory instead.
#include <mutex>

#include "slim_common.cuh"
#include "slim_internal.h"

namespace {

// The adapter scratch of every slim_linear_noalloc call.  Every GPU that
// loads the library holds it until the process exits.  Host code must not
// use the symbol itself as a device address: its device address is looked
// up once per device below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SLIM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the scratch array on the current device (looked up on
// the first call per device, with that device current).
slim_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    slim::set_last_cuda_error(e);
    return SLIM_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return SLIM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      slim::set_last_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
      return SLIM_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SLIM_OK;
}

}  // namespace

extern "C" slim_status slim_linear_noalloc(const slim_layer* layer, const uint16_t* X, int M, uint16_t* Y,
                                           void* stream) {
  slim::NvtxRange nv("slim_linear_noalloc");
  if (!layer || layer->magic != slim::kLayerMagic || !layer->base || !layer->status) return SLIM_ERR_STATE;
  if (M < 0) return SLIM_ERR_ARG;
  if (M == 0) return SLIM_OK;
  if (!X || !Y) return SLIM_ERR_ARG;
  if (!aligned16(X) || !aligned16(Y)) return SLIM_ERR_ALIGN;
  {
    const uintptr_t x0 = reinterpret_cast<uintptr_t>(X), x1 = x0 + (size_t)M * layer->K * 2;
    const uintptr_t y0 = reinterpret_cast<uintptr_t>(Y), y1 = y0 + (size_t)M * layer->N * 2;
    if (x0 < y1 && y0 < x1) return SLIM_ERR_ARG;
  }
  // The workspace must fit the fixed array: the prefill path's dequantized
  // weight images never would, so M > 16 stays on the token-tiled decode
  // kernels, and M <= 16 uses the streaming kernel only when its workspace
  // fits.
  const size_t need = slim::forward_workspace_bytes(*layer, M, false, SLIM_NOALLOC_SCRATCH_BYTES);
  if (need > SLIM_NOALLOC_SCRATCH_BYTES) return SLIM_ERR_WORKSPACE;
  const int major = slim::device_cc_major();
  if (major < 0) return SLIM_ERR_CUDA;
  if (major != 10) return SLIM_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (need > 0) {
    slim_status st = scratch_address(&scratch);
    if (st != SLIM_OK) return st;
  }
  cudaError_t e = slim::launch_forward(*layer, X, M, Y, scratch, false, SLIM_NOALLOC_SCRATCH_BYTES,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    slim::set_last_cuda_error(e);
    return SLIM_ERR_CUDA;
  }
  return SLIM_OK;
}
