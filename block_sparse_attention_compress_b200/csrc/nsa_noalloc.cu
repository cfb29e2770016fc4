// nsa_forward_noalloc: the NSA prefill forward for callers that cannot allocate
// device memory themselves.  The scratch that nsa_forward takes from the caller's
// workspace (compressed K/V, chosen block indices, the fp32 branch accumulator)
// lives here in one fixed file-scope device array instead.
//
// The array is a __device__ variable: in host code its name is only a host-side
// stand-in, so its device address is looked up once per device with
// cudaGetSymbolAddress (on the first call made with that device current) and that
// address is what the kernels receive.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/nsa.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 32ull << 20;   // 32 MiB, held by every GPU that loads the library
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::once_flag g_once[kMaxDevices];
void* g_addr[kMaxDevices];
cudaError_t g_addr_err[kMaxDevices];

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t scratch_address(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_once[dev], [dev] {
    void* p = nullptr;
    g_addr_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_addr[dev] = g_addr_err[dev] == cudaSuccess ? p : nullptr;
  });
  *addr = g_addr[dev];
  return g_addr_err[dev];
}

}  // namespace

extern "C" NSA_API nsa_status nsa_forward_noalloc(const void* q, const void* k, const void* v, const void* gates,
                                                  const nsa_config* cfg, void* out, void* stream) {
  if (!cfg) return NSA_ERR_INVALID_ARG;
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
  if (scratch_address(&scratch) != cudaSuccess || !scratch) return NSA_ERR_CUDA;
  nsa_config c = *cfg;
  c.workspace = scratch;
  c.workspace_bytes = kNoAllocScratchBytes;
  return nsa_forward(q, k, v, gates, &c, out, stream);
}
