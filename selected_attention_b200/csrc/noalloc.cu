// bsa_fwd_noalloc: the block-sparse attention forward for callers that cannot allocate device
// memory.  Some hosts own every byte of device memory themselves — an inference engine that hands
// its plugins pre-planned buffers and no scratch, or a latency-critical loop where a cudaMalloc
// (which may synchronise the device) is not acceptable — so they cannot provide the workspace
// bsa_fwd asks for.  This entry point takes the same problem and tensors as bsa_fwd and keeps
// the metadata scratch (status word and KV lists) in a fixed-size array of device memory that is
// part of the library image, so it allocates nothing.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds its own
// copy until the process exits.  Host code cannot use the symbol's name as a device address, so
// the first call on each device looks up that device's address with cudaGetSymbolAddress (with
// the device current) and remembers it; that first call should come before any stream capture.
// All calls on a device share the one array and leave their contents behind (the status word at
// its start is cleared by every call); calls whose GPU work overlaps in time race on it, so
// callers must order them (one stream, or synchronise between streams).
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_fwd_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_fwd_scratch on the current device; looked up once per device.
bsa_status scratch_on_current_device(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) return BSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return BSA_OK;
}

}  // namespace

extern "C" bsa_status bsa_fwd_noalloc(const bsa_params* p, const void* q, const void* k, const void* v, void* out,
                                      float* lse, void* stream) {
  size_t need = 0;
  bsa_status s = bsa_fwd_workspace_size(p, &need);  // validates the problem (no launch)
  if (s != BSA_OK) return s;
  if (need > kNoAllocScratchBytes) return BSA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  if ((s = scratch_on_current_device(&scratch)) != BSA_OK) return s;
  return bsa_fwd(p, q, k, v, out, lse, scratch, kNoAllocScratchBytes, stream);
}
