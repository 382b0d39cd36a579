// Kernel timing (off by default).  While enabled, each kernel launch the library makes is bracketed
// by a pair of CUDA events on the launch stream; bsa_profile_collect synchronises those events and
// sums the device time per kernel name.  Events come from a pool that grows on first use and is
// reused afterwards; with timing off the launch path only tests one flag.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace sa {
namespace {

struct Rec {
  const char* name;
  cudaEvent_t start, stop;
};

std::mutex g_mu;
bool g_on = false;
std::vector<cudaEvent_t> g_pool;
size_t g_pool_next = 0;
std::vector<Rec> g_recs;
int g_open = -1;
int g_depth = 0;  // open brackets (nested ones are not recorded)
uint64_t* g_cta_buf = nullptr;  // caller-owned device array [3][g_cta_cap][2]
int g_cta_cap = 0;

cudaEvent_t take_event() {
  if (g_pool_next == g_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    g_pool.push_back(e);
  }
  return g_pool[g_pool_next++];
}

}  // namespace

// A bracket opened inside another one (a launcher that times itself, called from a launcher that
// times a group of kernels) is counted in the outer bracket only.
void prof_begin(const char* name, cudaStream_t st) {
  if (!g_on) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_depth++ > 0) return;
  Rec r{name, take_event(), take_event()};
  if (r.start && r.stop && cudaEventRecord(r.start, st) == cudaSuccess) {
    g_recs.push_back(r);
    g_open = static_cast<int>(g_recs.size()) - 1;
  }
}

void prof_end(cudaStream_t st) {
  if (!g_on) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_depth > 0 && --g_depth > 0) return;
  if (g_open >= 0 && cudaEventRecord(g_recs[g_open].stop, st) != cudaSuccess) g_recs.pop_back();
  g_open = -1;
}

uint64_t* prof_cta_clock(int slot, int grid) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_cta_buf || grid > g_cta_cap || slot < 0 || slot > 2) return nullptr;
  return g_cta_buf + static_cast<size_t>(slot) * g_cta_cap * 2;
}

}  // namespace sa

extern "C" {

bsa_status bsa_profile_cta_clock(uint64_t* dev_buf, int32_t capacity) {
  if (dev_buf && capacity <= 0) return BSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(sa::g_mu);
  sa::g_cta_buf = dev_buf;
  sa::g_cta_cap = dev_buf ? capacity : 0;
  return BSA_OK;
}

bsa_status bsa_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(sa::g_mu);
  sa::g_on = on != 0;
  sa::g_recs.clear();
  sa::g_pool_next = 0;
  sa::g_open = -1;
  sa::g_depth = 0;
  return BSA_OK;
}

bsa_status bsa_profile_collect(bsa_kernel_time* out, int32_t max_entries, int32_t* n_entries) {
  if (!out || !n_entries) return BSA_ERR_NULLPTR;
  std::lock_guard<std::mutex> lk(sa::g_mu);
  std::vector<std::string> names;
  std::vector<double> ms;
  std::vector<int32_t> cnt;
  for (const auto& r : sa::g_recs) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return BSA_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess) return BSA_ERR_CUDA;
    size_t i = 0;
    while (i < names.size() && names[i] != r.name) ++i;
    if (i == names.size()) {
      names.emplace_back(r.name);
      ms.push_back(0.0);
      cnt.push_back(0);
    }
    ms[i] += t;
    cnt[i] += 1;
  }
  const int32_t n = static_cast<int32_t>(names.size());
  for (int32_t i = 0; i < n && i < max_entries; ++i) {
    std::memset(out[i].name, 0, sizeof(out[i].name));
    std::strncpy(out[i].name, names[i].c_str(), sizeof(out[i].name) - 1);
    out[i].launches = cnt[i];
    out[i].total_ms = ms[i];
  }
  *n_entries = n;
  sa::g_recs.clear();
  sa::g_pool_next = 0;
  return BSA_OK;
}

}  // extern "C"
