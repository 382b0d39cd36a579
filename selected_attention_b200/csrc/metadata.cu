// Metadata kernels: selections -> per-unit KV block lists and transposed lists.
//
// SparseAttnSharedkvMetadata page (function description): an operator run ahead of the
// attention call that lays out each core's share of the work.  Here the products are CSR lists:
//   * BSA: for unit (b, h, qb), the KV blocks its BlockSparseMask row selects, ascending
//     (BlockSparseAttentionGrad page, parameter description of the mask: one row of selected KV
//     blocks per Q block).
//   * BSA transposed: for (b, g, kb), ascending h_local * nqb + qb over the group's query heads
//     that selected kb; the dK/dV pass (dV = P^T dOut, dK = dS^T Q scale) walks these.
// All products are integers and deterministic (no atomics decide an order).
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

constexpr int kWarps = 8;

// One warp per row: count nonzero bytes.
__global__ void count_rows_kernel(const uint8_t* __restrict__ rows, int n_rows, int row_len,
                                  int32_t* __restrict__ counts) {
  griddep_wait();  // launched with programmatic dependent launch: the predecessor must be complete
  griddep_launch_dependents();
  const int warp = blockIdx.x * kWarps + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (warp >= n_rows) return;
  const uint8_t* r = rows + static_cast<size_t>(warp) * row_len;
  int c = 0;
  for (int i = lane; i < row_len; i += 32) c += (r[i] != 0);
#pragma unroll
  for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) counts[warp] = c;
}

// One warp per row: write the indices of nonzero bytes, ascending, at col[row_ptr[row]...].
__global__ void fill_rows_kernel(const uint8_t* __restrict__ rows, int n_rows, int row_len,
                                 const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col) {
  griddep_wait();
  griddep_launch_dependents();
  const int warp = blockIdx.x * kWarps + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (warp >= n_rows) return;
  const uint8_t* r = rows + static_cast<size_t>(warp) * row_len;
  int pos = row_ptr[warp];
  const unsigned lt = (1u << lane) - 1u;
  for (int base = 0; base < row_len; base += 32) {
    const int i = base + lane;
    const bool on = i < row_len && r[i] != 0;
    const unsigned bal = __ballot_sync(0xffffffffu, on);
    if (on) col[pos + __popc(bal & lt)] = i;
    pos += __popc(bal);
  }
}

// Single-CTA exclusive scan (1024 threads), chunk by chunk.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ counts, int n,
                                                    int32_t* __restrict__ row_ptr) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  griddep_wait();
  griddep_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + tid;
    const int v = i < n ? counts[i] : 0;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
      int s = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sums[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int c0 = carry;
    const int excl = c0 + (w ? warp_sums[w - 1] : 0) + x - v;
    if (i < n) row_ptr[i] = excl;
    __syncthreads();
    if (tid == 1023) carry = excl + v;
    __syncthreads();
  }
  if (tid == 0) row_ptr[n] = carry;
}

// mask [B, N1, nqb, nkb] -> maskT [B, N2, nkb, G*nqb] with entry (hl*nqb + qb), 32x32 tiles.
__global__ void transpose_mask_kernel(const uint8_t* __restrict__ mask, int N1, int N2, int nqb, int nkb,
                                      uint8_t* __restrict__ maskT) {
  __shared__ uint8_t tile[32][33];
  griddep_wait();
  griddep_launch_dependents();
  const int bh = blockIdx.z;  // b * N1 + h
  const int b = bh / N1, h = bh % N1;
  const int G = N1 / N2, g = h / G, hl = h % G;
  const int q0 = blockIdx.y * 32, k0 = blockIdx.x * 32;
  const uint8_t* src = mask + static_cast<size_t>(bh) * nqb * nkb;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int qb = q0 + r, kb = k0 + threadIdx.x;
    tile[r][threadIdx.x] = (qb < nqb && kb < nkb) ? src[static_cast<size_t>(qb) * nkb + kb] : 0;
  }
  __syncthreads();
  const size_t row_len = static_cast<size_t>(G) * nqb;
  uint8_t* dst = maskT + (static_cast<size_t>(b) * N2 + g) * nkb * row_len;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int kb = k0 + r, qb = q0 + threadIdx.x;
    if (kb < nkb && qb < nqb) dst[static_cast<size_t>(kb) * row_len + static_cast<size_t>(hl) * nqb + qb] =
        tile[threadIdx.x][r];
  }
}

inline int div_up(int a, int b) { return (a + b - 1) / b; }

}  // namespace

cudaError_t exclusive_scan(const int32_t* counts, int n, int32_t* row_ptr, cudaStream_t st) {
  prof_begin("meta_scan", st);
  cudaError_t e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, st, counts, n, row_ptr);
  prof_end(st);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t bsa_kv_lists(const uint8_t* mask, int units, int nkb, int32_t* counts, int32_t* row_ptr, int32_t* col,
                         cudaStream_t st) {
  if (units <= 0) return cudaSuccess;
  const int grid = div_up(units, kWarps);
  prof_begin("meta_count", st);
  cudaError_t e = launch_pdl(count_rows_kernel, dim3(grid), dim3(kWarps * 32), 0, st, mask, units, nkb, counts);
  prof_end(st);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if ((e = exclusive_scan(counts, units, row_ptr, st)) != cudaSuccess) return e;
  prof_begin("meta_fill", st);
  e = launch_pdl(fill_rows_kernel, dim3(grid), dim3(kWarps * 32), 0, st, mask, units, nkb,
                 static_cast<const int32_t*>(row_ptr), col);
  prof_end(st);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t bsa_q_lists(const uint8_t* mask, int B, int N1, int N2, int nqb, int nkb, uint8_t* maskT,
                        int32_t* counts, int32_t* row_ptr, int32_t* col, cudaStream_t st) {
  const int G = N1 / N2;
  dim3 grid(div_up(nkb, 32), div_up(nqb, 32), B * N1);
  prof_begin("meta_transpose", st);
  cudaError_t e = launch_pdl(transpose_mask_kernel, grid, dim3(32, 8), 0, st, mask, N1, N2, nqb, nkb, maskT);
  prof_end(st);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return bsa_kv_lists(maskT, B * N2 * nkb, G * nqb, counts, row_ptr, col, st);
}

}  // namespace sa
