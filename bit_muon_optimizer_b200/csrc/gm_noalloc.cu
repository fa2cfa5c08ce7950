// gm_newton_schulz_noalloc: standard Newton-Schulz without any device
// allocation, for callers that must not allocate GPU memory themselves.
//
// Some callers cannot call cudaMalloc (or torch's allocator) at the point where
// they need the orthogonalisation: code running inside a host framework that
// owns every allocation through its own pool, plugins that may not touch the
// device allocator, or paths where an allocation would synchronise the device.
// This entry point serves them: its scratch is a fixed file-scope device array
// that exists as soon as the library's kernels are loaded on a device, and it
// calls no allocating routine (no cudaMalloc, no cudaFree, no library that
// allocates).

#include <mutex>

#include "gm_common.cuh"
#include "gm_internal.h"

namespace gm {
namespace {

constexpr size_t kNoallocScratchBytes = GM_NOALLOC_SCRATCH_BYTES;   // 64 MiB per device

// Every GPU that loads this library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array for the current device. The host-side
// name of the array is only a stand-in, so the address is looked up once per
// device (with that device current) and cached.
gm_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(GM_E_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return set_error(GM_E_UNSUPPORTED, "device index %d too large", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return set_error(GM_E_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return GM_OK;
}

}  // namespace
}  // namespace gm

using namespace gm;

extern "C" gm_status gm_newton_schulz_noalloc(int B, int m, int n, const void* X, gm_dtype xdt,
                                              const float* abc, int T, float eps, void* O,
                                              gm_dtype odt, gm_stream_t stream) {
  const size_t need = gm_workspace_bytes(GM_OP_NEWTON_SCHULZ, B, m, n, 0, 0);
  if (need == 0) return set_error(GM_E_ARG, "bad shape B=%d m=%d n=%d", B, m, n);
  if (need > kNoallocScratchBytes)
    return set_error(GM_E_WORKSPACE,
                     "B=%d m=%d n=%d needs %zu bytes of scratch; the built-in scratch holds %zu "
                     "(use gm_newton_schulz with a caller-provided workspace instead)",
                     B, m, n, need, kNoallocScratchBytes);
  void* ws = nullptr;
  const gm_status st = noalloc_scratch(&ws);
  if (st != GM_OK) return st;
  return gm_newton_schulz(B, m, n, X, xdt, abc, T, eps, O, odt, ws, kNoallocScratchBytes, stream);
}
