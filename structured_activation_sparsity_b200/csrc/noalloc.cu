// sparsesam_rcmlp_noalloc: the Residual-Consistency MLP with its scratch in a fixed, library-owned
// device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the block: hosts whose
// allocator owns all device memory and hands none to plug-ins, and latency-bound loops that must not
// pay cudaMalloc's implicit device-wide synchronisation. For them this entry point takes only inputs
// and outputs; the two scratch buffers the MLP needs (the gathered kept rows and the hidden
// activation) live in `g_rcmlp_scratch` below.
//
// The array is a file-scope __device__ variable: every GPU that loads this library holds its
// kRcmlpScratchBytes until the process exits. Host code may not use its name as a device address;
// the address is looked up once per device with cudaGetSymbolAddress (with that device current)
// and passed to the kernels. That cached address (like the status word's) is not looked up again,
// so it is stale after a cudaDeviceReset of the device.
#include <mutex>

#include "kernels.h"

namespace ss {
namespace {

constexpr size_t kRcmlpScratchBytes = size_t(32) << 20;   // 32 MiB
static __device__ __align__(256) uint8_t g_rcmlp_scratch[kRcmlpScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[128] = {};

// Device address of g_rcmlp_scratch on the current device (set up on the first call per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return SS_ECUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_rcmlp_scratch) != cudaSuccess || p == nullptr) return SS_ECUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SS_OK;
}

}  // namespace
}  // namespace ss

extern "C" int sparsesam_rcmlp_noalloc(const ss_cfg* cfg, uint16_t* x, int32_t C, int32_t hidden,
                                       const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                                       const uint16_t* b2, const int32_t* keep, int32_t K,
                                       void* stream) {
  // The same argument checks as sparsesam_rcmlp, then the size check, all on the host: a shape
  // whose scratch exceeds the fixed array is rejected before any CUDA call.
  size_t need = 0;
  int rc0 = ss::rcmlp_validate(cfg, x, C, hidden, w1, b1, w2, b2, keep, K, &need);
  if (rc0) return rc0;
  if (need > ss::kRcmlpScratchBytes) return SS_EWORKSPACE;
  void* scratch = nullptr;
  int rc = ss::scratch_address(&scratch);
  if (rc) return rc;
  // Every scratch byte the MLP reads is written earlier in the same call (the gather fills the
  // kept rows, fc1 fills the hidden rows it covers, TMA zero-fills rows past the end), so nothing
  // left from a previous call has to be cleared.
  return sparsesam_rcmlp(cfg, x, C, hidden, w1, b1, w2, b2, keep, K, scratch,
                         ss::kRcmlpScratchBytes, stream);
}
