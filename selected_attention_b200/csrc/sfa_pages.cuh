// The compacted page list of one (batch, kv head) row of a sparse decode (SparseFlashAttention
// page: the selected sparse blocks of sparse_block_size tokens map, page by page, to physical pages
// of the paged cache through block_table; sparse_block_size is a multiple of the page size).
// Shared by the stand-alone metadata kernel and the decode kernel's prologue, so the list the
// decode uses is the one the metadata op exposes.
#pragma once
#include <stdint.h>

#include "status_bits.h"

namespace sa {

// One warp.  Slots of the row are taken in order; a slot with id j (>= 0) contributes the logical
// pages j*ppb .. j*ppb+ppb-1 that start below `used` (the sequence's token count), each mapped
// through the table.  An id at or past the sequence's sparse-block count, or a table entry outside
// [0, num_pages), sets SA_DEV_BAD_INDEX in *bad and contributes nothing (for the table, from that
// page on).  Every valid page is written at its position in the compacted list: pages[pos] = its
// physical page, tokens[pos] = its tokens in use.  Returns the number of valid pages (all lanes).
__device__ __forceinline__ int sfa_row_page_list(const int32_t* __restrict__ idx, int K, int ppb, int page_size,
                                                 int used, const int32_t* __restrict__ table_row,
                                                 int max_pages_per_seq, int num_pages, int32_t* __restrict__ pages,
                                                 int32_t* __restrict__ tokens, uint32_t* bad) {
  const int lane = threadIdx.x & 31;
  const int sbs = ppb * page_size;
  const int n_sb = used > 0 ? (used + sbs - 1) / sbs : 0;
  int base = 0;
  uint32_t flags = 0;
  for (int s0 = 0; s0 < K; s0 += 32) {
    const int i = s0 + lane;
    const int j = i < K ? idx[i] : -1;
    int nvalid = 0;
    if (j >= n_sb) flags |= SA_DEV_BAD_INDEX;
    if (j >= 0 && j < n_sb) {
      for (int p = 0; p < ppb; ++p) {
        const int lp = j * ppb + p;
        if (lp * page_size >= used) break;
        const int phys = lp < max_pages_per_seq ? table_row[lp] : -1;
        if (phys < 0 || phys >= num_pages) {
          flags |= SA_DEV_BAD_INDEX;
          break;
        }
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
      pages[pos] = table_row[lp];
      tokens[pos] = min(page_size, used - lp * page_size);
      ++pos;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  *bad = __reduce_or_sync(0xffffffffu, flags);
  return base;
}

// The balanced split of a unit's n pages over its P pieces: piece p takes the pages
// [floor(p n / P), floor((p + 1) n / P)) of the compacted list.
__host__ __device__ __forceinline__ void sfa_piece_range(int n, int P, int p, int* begin, int* len) {
  const long long b0 = static_cast<long long>(p) * n / P, b1 = static_cast<long long>(p + 1) * n / P;
  *begin = static_cast<int>(b0);
  *len = static_cast<int>(b1 - b0);
}

}  // namespace sa

namespace sa {

// Pieces of a sparse decode: unit u = (b * N2 + g) * HH + head half; piece = u * P + p.  The
// piece's set-up, run by one warp: the unit's compacted page list into its own region
// (pages / tokens, cap entries), then its share [begin, begin + len) of the list.  Device status
// bits go to *status.
__device__ __forceinline__ void sfa_piece_setup(int piece, int P, int HH, int N2, int K, int ppb, int page_size,
                                                int max_pages_per_seq, int num_pages,
                                                const int32_t* __restrict__ sparse_indices,
                                                const int32_t* __restrict__ block_table,
                                                const int32_t* __restrict__ seqused_kv, int32_t* __restrict__ pages,
                                                int32_t* __restrict__ tokens, int* n, int* begin, int* len,
                                                uint32_t* status) {
  const int u = piece / P, p = piece % P;
  const int bg = u / HH, b = bg / N2;
  uint32_t bad = 0;
  const int cnt = sfa_row_page_list(sparse_indices + static_cast<size_t>(bg) * K, K, ppb, page_size, seqused_kv[b],
                                    block_table + static_cast<size_t>(b) * max_pages_per_seq, max_pages_per_seq,
                                    num_pages, pages, tokens, &bad);
  if ((threadIdx.x & 31) == 0 && bad && status) atomicOr(status, bad);
  *n = cnt;
  sfa_piece_range(cnt, P, p, begin, len);
}

}  // namespace sa
