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
// the first call in each CUDA context looks up that context's address with cudaGetSymbolAddress
// (with the device current) and remembers it together with the context's id; a later call in
// another context (a device reset creates a new one, and the array may then sit elsewhere) looks
// it up again.  The first call on a device should come before any stream capture.  All calls on a
// device share the one array and leave their contents behind (the status word at its start is
// cleared by every call); calls whose GPU work overlaps in time race on it, so callers must order
// them (one stream, or synchronise between streams).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_fwd_scratch[kNoAllocScratchBytes];

struct ScratchEntry {
  unsigned long long ctx_id;  // id of the CUDA context the address belongs to
  void* addr;                 // device address of g_fwd_scratch in that context
};

std::mutex g_scratch_mu;
ScratchEntry g_scratch[kMaxDevices] = {};

// Driver calls that name the current context and its process-unique id, fetched through the
// runtime's driver entry point (the library does not link libcuda).
struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const CtxFns& ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return f;
}

// Device address of g_fwd_scratch in the current context; looked up once per context.
bsa_status scratch_in_current_context(void** addr) {
  const CtxFns& f = ctx_fns();
  if (!f.get_current || !f.get_id) return BSA_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BSA_ERR_UNSUPPORTED;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS) return BSA_ERR_CUDA;
  if (ctx == nullptr) {
    // no context is current yet: the lookup makes the runtime create the device's primary context
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) return BSA_ERR_CUDA;
    if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return BSA_ERR_CUDA;
  }
  unsigned long long id = 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return BSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchEntry& e = g_scratch[dev];
  if (e.addr == nullptr || e.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) return BSA_ERR_CUDA;
    e.ctx_id = id;
    e.addr = p;
  }
  *addr = e.addr;
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
  if ((s = scratch_in_current_context(&scratch)) != BSA_OK) return s;
  return bsa_fwd(p, q, k, v, out, lse, scratch, kNoAllocScratchBytes, stream);
}

// The device status word of the last bsa_fwd_noalloc call on the current device sits at the
// start of the library's array; this reads it like bsa_get_status reads a workspace (it
// synchronises `stream`).
extern "C" bsa_status bsa_fwd_noalloc_get_status(void* stream, uint32_t* dev_bits) {
  if (!dev_bits) return BSA_ERR_NULLPTR;
  void* scratch = nullptr;
  bsa_status s = scratch_in_current_context(&scratch);
  if (s != BSA_OK) return s;
  return bsa_get_status(scratch, stream, dev_bits);
}
