// Sparse-decode metadata (SparseFlashAttention page: the selected sparse blocks map to pages of a
// paged KV cache; sparse_block_size is a multiple of block_size) and the balanced work list
// (SparseAttnSharedkvMetadata page: each core gets the start and end of its share of the tasks).
//
//   sfa_page_list   per (b, kv head g): the physical pages of the selected sparse blocks, in list
//                   order, compacted (empty slots and pages past seqused_kv dropped), with the
//                   number of valid tokens of each page.  A sparse block id at or past the
//                   sequence's block count sets SA_DEV_BAD_INDEX and is skipped.
//   sfa_work_list   units (b, g, head half) share the page list of (b, g); one CTA computes a
//                   piece of at most `chunk` consecutive pages of one unit, with chunk the smallest
//                   size whose pieces fit one wave of CTAs (so the longest piece is as short as
//                   possible).  Pieces are numbered unit by unit.
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

// One warp per (b, g): each lane takes a slot of the sparse-index row, counts its valid pages,
// and a warp scan places them, so the compacted list keeps the row's order.
__global__ void sfa_page_list_kernel(const int32_t* __restrict__ sparse_indices, const int32_t* __restrict__ block_table,
                                     const int32_t* __restrict__ seqused_kv, int B, int N2, int K, int ppb,
                                     int page_size, int max_pages_per_seq, int num_pages, int32_t* __restrict__ pages,
                                     int32_t* __restrict__ tokens, int32_t* __restrict__ count,
                                     uint32_t* __restrict__ status) {
  griddep_launch_dependents();  // the work list may launch now; it waits for this grid's results
  const int bg = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bg >= B * N2) return;
  const int b = bg / N2;
  const int used = seqused_kv[b];
  const int sbs = ppb * page_size;
  const int n_sb = used > 0 ? (used + sbs - 1) / sbs : 0;
  const int32_t* idx = sparse_indices + static_cast<size_t>(bg) * K;  // row 0 of Sq
  const int cap = K * ppb;
  int base = 0;
  uint32_t bad = 0;
  for (int s0 = 0; s0 < K; s0 += 32) {
    const int i = s0 + lane;
    const int j = i < K ? idx[i] : -1;
    // valid pages of this slot: logical pages j*ppb .. j*ppb+ppb-1 that start below `used`
    int nvalid = 0;
    if (j >= n_sb) bad |= SA_DEV_BAD_INDEX;
    if (j >= 0 && j < n_sb) {
      for (int p = 0; p < ppb; ++p) {
        const int lp = j * ppb + p;
        if (lp * page_size >= used) break;
        const int phys = lp < max_pages_per_seq ? block_table[static_cast<size_t>(b) * max_pages_per_seq + lp] : -1;
        if (phys < 0 || phys >= num_pages) { bad |= SA_DEV_BAD_INDEX; break; }
        ++nvalid;
      }
    }
    int incl = nvalid;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = base + incl - nvalid;
    for (int p = 0; p < nvalid; ++p) {
      const int lp = j * ppb + p;
      pages[static_cast<size_t>(bg) * cap + pos] = block_table[static_cast<size_t>(b) * max_pages_per_seq + lp];
      tokens[static_cast<size_t>(bg) * cap + pos] = min(page_size, used - lp * page_size);
      ++pos;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) count[bg] = base;
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (lane == 0 && bad) raise_status(status, bad);
}

// One CTA: choose the piece size and lay out the pieces.
//   units u = (b * N2 + g) * per + head_half; n_u = count[b, g]
//   chunk = the smallest c >= 1 with sum_u ceil(n_u / c) <= G (binary search; with more units
//   than G it ends at c = max n_u, one piece per unit, and the piece arrays, sized G + units,
//   still hold them)
//   piece records: unit, first page, page count; unit_first[u], unit_pieces[u]
__global__ void __launch_bounds__(1024) sfa_work_list_kernel(const int32_t* __restrict__ count, int units, int per,
                                                             int G,
                                                             int32_t* __restrict__ piece_unit,
                                                             int32_t* __restrict__ piece_begin,
                                                             int32_t* __restrict__ piece_len,
                                                             int32_t* __restrict__ unit_first,
                                                             int32_t* __restrict__ unit_pieces,
                                                             int32_t* __restrict__ n_pieces) {
  __shared__ int s_pieces, s_max;
  __shared__ int s_chunk;
  __shared__ int warp_tot[32];
  __shared__ int carry;
  griddep_launch_dependents();
  griddep_wait();  // launched early (programmatic dependent launch): the page counts must be complete
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) s_max = 1;
  __syncthreads();
  int mx = 1;
  for (int u = tid; u < units; u += blockDim.x) mx = max(mx, count[u / per]);
  atomicMax(&s_max, mx);
  __syncthreads();
  int lo = 1, hi = s_max;  // pieces(hi) = units <= G
  while (lo < hi) {        // uniform across the block
    const int mid = (lo + hi) >> 1;
    if (tid == 0) s_pieces = 0;
    __syncthreads();
    int loc = 0;
    for (int u = tid; u < units; u += blockDim.x) {
      const int n = count[u / per];
      loc += n > 0 ? (n + mid - 1) / mid : 0;
    }
    atomicAdd(&s_pieces, loc);  // integer sum: order does not matter
    __syncthreads();
    const int total = s_pieces;
    __syncthreads();
    if (total <= G) hi = mid;
    else lo = mid + 1;
  }
  if (tid == 0) {
    s_chunk = lo;
    carry = 0;
  }
  __syncthreads();
  const int chunk = s_chunk;
  // exclusive scan of pieces per unit, in unit order
  for (int base = 0; base < units; base += blockDim.x) {
    const int u = base + tid;
    const int n = u < units ? count[u / per] : 0;
    const int pcs = u < units ? (n > 0 ? (n + chunk - 1) / chunk : 0) : 0;
    int x = pcs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
      int t = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_tot[lane] = t;
    }
    __syncthreads();
    const int first = carry + (w ? warp_tot[w - 1] : 0) + x - pcs;
    if (u < units) {
      unit_first[u] = first;
      unit_pieces[u] = pcs;
      for (int p = 0; p < pcs; ++p) {
        piece_unit[first + p] = u;
        piece_begin[first + p] = p * chunk;
        piece_len[first + p] = min(chunk, n - p * chunk);
      }
    }
    __syncthreads();
    if (tid == blockDim.x - 1) carry = first + pcs;
    __syncthreads();
  }
  if (tid == 0) *n_pieces = carry;
}

}  // namespace

cudaError_t sfa_page_list(const SfaMetaArgs& a, cudaStream_t st) {
  const int n = a.B * a.N2;
  if (n == 0) return cudaSuccess;
  prof_begin("sfa_page_list", st);
  sfa_page_list_kernel<<<(n + 3) / 4, 128, 0, st>>>(a.sparse_indices, a.block_table, a.seqused_kv, a.B, a.N2,
                                                        a.K, a.ppb, a.page_size, a.max_pages_per_seq, a.num_pages,
                                                        a.pages, a.tokens, a.count, a.status);
  prof_end(st);
  return cudaGetLastError();
}

cudaError_t sfa_work_list(const int32_t* count, int units, int per, int G, int32_t* piece_unit,
                          int32_t* piece_begin, int32_t* piece_len, int32_t* unit_first, int32_t* unit_pieces,
                          int32_t* n_pieces, cudaStream_t st) {
  prof_begin("sfa_work_list", st);
  cudaError_t e = launch_pdl(sfa_work_list_kernel, dim3(1), dim3(1024), 0, st, count, units, per, G, piece_unit,
                             piece_begin, piece_len, unit_first, unit_pieces, n_pieces);
  prof_end(st);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sa
