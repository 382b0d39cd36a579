// Sparse-decode metadata (SparseFlashAttention page: the selected sparse blocks map to pages of a
// paged KV cache; sparse_block_size is a multiple of block_size) and the balanced split of each
// unit's pages over its pieces (SparseAttnSharedkvMetadata page: each core gets the start and end
// of its share of the tasks).
//
//   sfa_page_list   per (b, kv head g): the physical pages of the selected sparse blocks, in list
//                   order, compacted (empty slots and pages past seqused_kv dropped), with the
//                   number of valid tokens of each page.  A sparse block id at or past the
//                   sequence's block count sets SA_DEV_BAD_INDEX and is skipped.
//   sfa_pieces      the decode's own set-up for every piece (unit u, piece p of P): the unit's
//                   page list in the piece's region and the piece's range [begin, begin + len)
//                   with begin = floor(p n / P); the decode kernel runs the same code in its
//                   prologue, this launch exposes it (metadata op BSA_META_SFA_WORK).
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"
#include "sfa_pages.cuh"

namespace sa {
namespace {

// One warp per (b, g).
__global__ void sfa_page_list_kernel(const int32_t* __restrict__ sparse_indices, const int32_t* __restrict__ block_table,
                                     const int32_t* __restrict__ seqused_kv, int B, int N2, int K, int ppb,
                                     int page_size, int max_pages_per_seq, int num_pages, int32_t* __restrict__ pages,
                                     int32_t* __restrict__ tokens, int32_t* __restrict__ count,
                                     uint32_t* __restrict__ status) {
  const int bg = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (bg >= B * N2) return;
  const int b = bg / N2;
  const int cap = K * ppb;
  uint32_t bad = 0;
  const int n = sfa_row_page_list(sparse_indices + static_cast<size_t>(bg) * K, K, ppb, page_size, seqused_kv[b],
                                  block_table + static_cast<size_t>(b) * max_pages_per_seq, max_pages_per_seq,
                                  num_pages, pages + static_cast<size_t>(bg) * cap, tokens + static_cast<size_t>(bg) * cap,
                                  &bad);
  if (lane == 0) {
    count[bg] = n;
    if (bad) raise_status(status, bad);
  }
}

// One warp per piece.
__global__ void sfa_pieces_kernel(SfaMetaArgs a, int P, int HH, int n_pieces, int32_t* __restrict__ rec) {
  const int piece = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (piece >= n_pieces) return;
  const int cap = a.K * a.ppb;
  int n, begin, len;
  sfa_piece_setup(piece, P, HH, a.N2, a.K, a.ppb, a.page_size, a.max_pages_per_seq, a.num_pages, a.sparse_indices,
                  a.block_table, a.seqused_kv, a.pages + static_cast<size_t>(piece) * cap,
                  a.tokens + static_cast<size_t>(piece) * cap, &n, &begin, &len, a.status);
  if ((threadIdx.x & 31) == 0) {
    rec[3 * piece] = n;
    rec[3 * piece + 1] = begin;
    rec[3 * piece + 2] = len;
  }
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

cudaError_t sfa_pieces(const SfaMetaArgs& a, int P, int HH, int n_pieces, int32_t* rec, cudaStream_t st) {
  if (n_pieces == 0) return cudaSuccess;
  prof_begin("sfa_pieces", st);
  sfa_pieces_kernel<<<(n_pieces + 3) / 4, 128, 0, st>>>(a, P, HH, n_pieces, rec);
  prof_end(st);
  return cudaGetLastError();
}

int sfa_pieces_per_unit(int units, int sms) {
  int P = units > 0 ? sms / units : 1;
  return P < 1 ? 1 : (P > kSfaMaxPieces ? kSfaMaxPieces : P);
}

}  // namespace sa
