// nsa_forward_noalloc: the NSA prefill forward for callers that cannot allocate
// device memory themselves.  The scratch that nsa_forward takes from the caller's
// workspace (compressed K/V, chosen block indices, the fp32 branch accumulator)
// lives here in one fixed file-scope device array instead.
//
// The array is a __device__ variable: in host code its name is only a host-side
// stand-in, not a device address.  Its device address is looked up per device
// with cudaGetSymbolAddress, with that device current, and that address is what
// the kernels receive.  Only a successful lookup is kept: after a failed one (for
// example a first call made while a stream is being captured) the next call on
// that device tries again.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/nsa.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 32ull << 20;   // 32 MiB, held by every GPU that loads the library
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu[kMaxDevices];
void* g_addr[kMaxDevices];   // device address of the array per device; null until a lookup succeeds

// Device address of the scratch array on the current device.
cudaError_t scratch_address(void** addr) {
  *addr = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu[dev]);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();   // leave no error behind for the caller's next runtime call
      return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    }
    g_addr[dev] = p;
  }
  *addr = g_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" NSA_API nsa_status nsa_forward_noalloc(const void* q, const void* k, const void* v, const void* gates,
                                                  const nsa_config* cfg, void* out, void* stream) {
  if (!cfg) return NSA_ERR_INVALID_ARG;
  if (cfg->mode == NSA_MODE_DSA) return NSA_ERR_INVALID_ARG;   // as nsa_forward
  const size_t need = nsa_workspace_size(cfg, 0);
  if (need == 0) {
    // an invalid configuration: let nsa_forward report exactly what is wrong
    nsa_config c = *cfg;
    c.workspace = nullptr;
    c.workspace_bytes = 0;
    return nsa_forward(q, k, v, gates, &c, out, stream);
  }
  if (need > kNoAllocScratchBytes) return NSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return NSA_ERR_CUDA;
  nsa_config c = *cfg;
  c.workspace = scratch;
  c.workspace_bytes = kNoAllocScratchBytes;
  return nsa_forward(q, k, v, gates, &c, out, stream);
}

extern "C" NSA_API nsa_status nsa_device_status_noalloc(int32_t* code_out, void* stream) {
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return NSA_ERR_CUDA;
  return nsa_device_status(scratch, code_out, stream);   // the status word leads the array
}
