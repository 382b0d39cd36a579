// Diagnostic: one 128 x 128 x 128 tcgen05 tile, C = A B^T with A K-major and B either K-major
// ([N][K]) or MN-major ([K][N]); modes 2 and 3 take A from tensor memory (written with
// tcgen05.st) with B K-major (2) or MN-major (3); modes 4 and 5 give A MN-major (the buffer holds
// A^T, [K][M]) with B K-major (4) or MN-major (5).  Exercises exactly the building blocks the attention kernels use
// (TMA 128B-swizzled loads, smem descriptors of both majors, TMEM accumulate, tcgen05.ld), so a
// parity failure in attention can be narrowed to the tile machinery or the attention logic.
#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

struct __align__(1024) DiagSmem {
  uint8_t a[2][128 * 128];  // two 64-column sub-tiles of A: [128 rows][64] each
  uint8_t b[2][128 * 128];  // two sub-tiles of B
  uint64_t bar_load;
  uint64_t bar_mma;
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(128) diag_mma_kernel(const __grid_constant__ CUtensorMap tm_a,
                                                       const __grid_constant__ CUtensorMap tm_b, float* c,
                                                       int b_mn_major, uint32_t* status, const void* a_ptr) {
  extern __shared__ uint8_t smem_raw[];
  DiagSmem& s = *reinterpret_cast<DiagSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (tid == 0) {
    mbar_init(&s.bar_load, 1);
    mbar_init(&s.bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  bool ok = true;
  if (b_mn_major == 2 || b_mn_major == 3) {
    // A row (warp*32 + lane) from global into TMEM columns [128, 192): 64 packed bf16 pairs
    const uint32_t* arow = reinterpret_cast<const uint32_t*>(a_ptr) + (warp * 32 + lane) * 64;
    uint32_t r[16];
    for (int c = 0; c < 64; c += 16) {
      for (int i = 0; i < 16; ++i) r[i] = arow[c + i];
      tmem_st16(tmem_addr(tmem, warp * 32, 128 + c), r);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    mbar_arrive_expect_tx(&s.bar_load, 4 * 128 * 128);
    tma_load_2d(s.a[0], &tm_a, &s.bar_load, 0, 0);
    tma_load_2d(s.a[1], &tm_a, &s.bar_load, 64, 0);
    tma_load_2d(s.b[0], &tm_b, &s.bar_load, 0, 0);
    tma_load_2d(s.b[1], &tm_b, &s.bar_load, 64, 0);
    ok = mbar_wait(&s.bar_load, 0, status);
    if (ok) {
      tc_fence_after();
      const bool a_mn = b_mn_major >= 4;
      const uint32_t idesc =
          idesc_bf16_f32(128, 128, a_mn, b_mn_major == 1 || b_mn_major == 3 || b_mn_major == 5);
      for (int ks = 0; ks < 8; ++ks) {
        // A MN-major: sub-tile = M chunk of 64, K step = 16 rows
        const uint64_t ad = a_mn ? sdesc_sw128(smem_u32(s.a[0]) + ks * 2048, 128 * 128, 1024)
                                 : sdesc_sw128(smem_u32(s.a[ks / 4]) + (ks % 4) * 32, 0, 1024);
        uint64_t bd;
        if (b_mn_major == 2 || b_mn_major == 3) {  // A from TMEM; B K-major (2) or MN-major (3)
          bd = b_mn_major == 3 ? sdesc_sw128(smem_u32(s.b[0]) + ks * 2048, 128 * 128, 1024)
                               : sdesc_sw128(smem_u32(s.b[ks / 4]) + (ks % 4) * 32, 0, 1024);
          mma_bf16_ts(tmem, tmem + 128 + ks * 8, bd, idesc, ks > 0 ? 1u : 0u);
          continue;
        }
        if (b_mn_major == 1 || b_mn_major == 5)  // B tile is [K rows][N cols]: sub-tile = N chunk, K step = 16 rows
          bd = sdesc_sw128(smem_u32(s.b[0]) + ks * 2048, 128 * 128, 1024);
        else
          bd = sdesc_sw128(smem_u32(s.b[ks / 4]) + (ks % 4) * 32, 0, 1024);
        mma_bf16_ss(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
      }
      tc_commit(&s.bar_mma);
    }
  }
  __syncwarp();
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  __syncthreads();
  if (!aborted(status)) ok = mbar_wait(&s.bar_mma, 0, status);
  else ok = false;
  tc_fence_after();
  if (ok) {
    const int row = warp * 32 + lane;
    for (int cc = 0; cc < 128; cc += 32) {
      uint32_t r[32];
      tmem_ld32(tmem_addr(tmem, warp * 32, cc), r);
      tmem_ld_wait(r);
#pragma unroll
      for (int i = 0; i < 32; ++i) c[row * 128 + cc + i] = __uint_as_float(r[i]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// Failure detection: one warp waits on an mbarrier of one arrival with the kernels' bounded wait.
// With `arrive` lane 0 arrives first and the wait succeeds; without it nothing ever arrives, the
// wait gives up after kWaitLimitNs and sets SA_DEV_TIMEOUT, and the kernel returns normally, so the
// context stays usable (no trap, no fault).
__global__ void diag_wait_kernel(uint32_t* status, int arrive) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (arrive && threadIdx.x == 0) mbar_arrive(&bar);
  __syncwarp();
  mbar_wait(&bar, 0, status);
}

__global__ void diag_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int n, int degree) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
  float y0, y1;
  if (degree == 3) ex2_poly_pair<3>(x0, x1, y0, y1);
  else ex2_poly_pair<4>(x0, x1, y0, y1);
  y[i] = y0;
  if (i + 1 < n) y[i + 1] = y1;
}

}  // namespace

cudaError_t diag_exp2_launch(const float* x, float* y, int n, int degree, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int pairs = (n + 1) / 2;
  diag_exp2_kernel<<<(pairs + 255) / 256, 256, 0, st>>>(x, y, n, degree);
  return cudaGetLastError();
}

cudaError_t diag_mma_tile_launch(const void* a, const void* b, float* c, int n, int b_mn_major, uint32_t* status,
                                 cudaStream_t st) {
  if (n != 128) return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (!make_tmap_2d_bf16(&ta, a, 128, 128, 128, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d_bf16(&tb, b, 128, 128, 128, 128)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(DiagSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(diag_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  prof_begin("diag_mma", st);
  diag_mma_kernel<<<1, 128, smem, st>>>(ta, tb, c, b_mn_major, status, a);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t diag_wait_launch(uint32_t* status, int arrive, cudaStream_t st) {
  diag_wait_kernel<<<1, 32, 0, st>>>(status, arrive);
  return cudaGetLastError();
}

}  // namespace sa
