// NSA selected-attention metadata (NsaSelectedAttention page: selected_key = Gather(key,
// topk_indices[i]) for 0 <= i < selected_block_count; TND layout with per-batch lengths).
//
//   nsa_check_seqlens  cu_seqlens must start at 0, be non-decreasing, end at T and hold no batch
//                      longer than the declared maximum length; otherwise SA_DEV_BAD_SEQLEN is set
//                      and every kernel skips all work.
//   nsa_kv_lists       per (token, kv head): the valid block ids ascending (-1 dropped; ids at or
//                      past the batch's block count dropped and flagged SA_DEV_BAD_INDEX;
//                      duplicates kept), their count and whether an id repeats.  For the
//                      backward it also sets bit t of the bit-row (g, kb) of a bitmap
//                      [N2][nblk_max][ceil(T/32)] words.
//   nsa_token_lists    per (b, g, kb) (kb padded to the longest batch): the tokens whose list holds
//                      kb, ascending, each once.  One warp per (b, g, kb) reads the batch's span of
//                      the bit-row, a word per lane, so the order is fixed without sorting.
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

__global__ void nsa_check_seqlens_kernel(const int32_t* __restrict__ cu, int B, int T, int max_len,
                                         int32_t* __restrict__ ok_flag, uint32_t* __restrict__ status) {
  int bad = (cu[0] != 0 || cu[B] != T) ? 1 : 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x)
    if (cu[b + 1] < cu[b] || cu[b + 1] - cu[b] > max_len) bad = 1;
  bad = __syncthreads_or(bad);
  if (threadIdx.x == 0) {
    *ok_flag = bad ? 0 : 1;
    if (bad) raise_status(status, SA_DEV_BAD_SEQLEN);
  }
}

__device__ __forceinline__ int batch_of(const int32_t* __restrict__ cu, int B, int t) {
  int lo = 0, hi = B - 1;  // largest b with cu[b] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__global__ void nsa_kv_lists_kernel(const int32_t* __restrict__ topk, const int32_t* __restrict__ cu, int B, int T,
                                    int N2, int K, int sel_block, int nblk_max, int words,
                                    const int32_t* __restrict__ ok_flag,
                                    int32_t* __restrict__ ids, int32_t* __restrict__ cnt, int32_t* __restrict__ dup,
                                    uint32_t* __restrict__ bitmap, uint32_t* __restrict__ status) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;  // (t, g)
  if (row >= T * N2) return;
  const int t = row / N2;
  int32_t* out = ids + static_cast<size_t>(row) * K;
  if (!*ok_flag) {
    for (int i = 0; i < K; ++i) out[i] = -1;
    cnt[row] = 0;
    dup[row] = 0;
    return;
  }
  const int b = batch_of(cu, B, t);
  const int len = cu[b + 1] - cu[b];
  const int nblk = (len + sel_block - 1) / sel_block;
  const int g = row - t * N2;
  const int32_t* in = topk + static_cast<size_t>(row) * K;
  int n = 0;
  bool bad = false;
  for (int i = 0; i < K; ++i) {
    const int v = in[i];
    if (v < 0) continue;
    if (v >= nblk) { bad = true; continue; }
    // insertion into the ascending prefix out[0..n)
    int p = n;
    while (p > 0 && out[p - 1] > v) {
      out[p] = out[p - 1];
      --p;
    }
    out[p] = v;
    ++n;
    if (bitmap)  // v < nblk <= nblk_max: the batch is no longer than the maximum length
      atomicOr(&bitmap[(static_cast<size_t>(g) * nblk_max + v) * words + (t >> 5)], 1u << (t & 31));
  }
  int d = 0;
  for (int i = 1; i < n; ++i) d |= out[i] == out[i - 1];
  for (int i = n; i < K; ++i) out[i] = -1;
  cnt[row] = n;
  dup[row] = d;
  if (bad) raise_status(status, SA_DEV_BAD_INDEX);
}

// rows r = (b * N2 + g) * nblk_max + kb; lane i takes word w0 + i of the bit-row, w0 stepping by 32
template <bool kFill>
__global__ void nsa_column_kernel(const uint32_t* __restrict__ bitmap, const int32_t* __restrict__ cu, int B, int N2,
                                  int sel_block, int nblk_max, int words, const int32_t* __restrict__ ok_flag,
                                  int32_t* __restrict__ counts, const int32_t* __restrict__ row_ptr,
                                  int32_t* __restrict__ col) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= B * N2 * nblk_max) return;
  const int kb = r % nblk_max;
  const int bg = r / nblk_max;
  const int b = bg / N2, g = bg % N2;
  int pos = kFill ? row_ptr[r] : 0;
  const int t0 = cu[b], t1 = cu[b + 1];
  if (*ok_flag && kb * sel_block < t1 - t0) {
    const uint32_t* bits = bitmap + (static_cast<size_t>(g) * nblk_max + kb) * words;
    const int wlo = t0 >> 5, whi = (t1 - 1) >> 5;
    for (int w0 = wlo; w0 <= whi; w0 += 32) {
      const int w = w0 + lane;
      uint32_t x = w <= whi ? bits[w] : 0u;
      if (w == wlo) x &= ~0u << (t0 & 31);                       // tokens of earlier batches
      if (w == whi && (t1 & 31)) x &= (1u << (t1 & 31)) - 1u;    // tokens of later batches
      const int c = __popc(x);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (kFill) {
        int q = pos + incl - c;
        while (x) {
          col[q++] = w * 32 + (__ffs(x) - 1);
          x &= x - 1u;
        }
      }
      pos += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (!kFill && lane == 0) counts[r] = pos;
}

}  // namespace

cudaError_t nsa_metadata(const NsaMetaArgs& a, cudaStream_t st) {
  cudaError_t e;
  prof_begin("nsa_check_seqlens", st);
  nsa_check_seqlens_kernel<<<1, 256, 0, st>>>(a.cu_seqlens, a.B, a.T, a.max_len, a.ok_flag, a.status);
  prof_end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  uint32_t* bitmap = a.token_lists ? a.bitmap : nullptr;
  if (bitmap) {
    const size_t bitmap_words = static_cast<size_t>(a.N2) * a.nblk_max * a.words;
    if ((e = cudaMemsetAsync(bitmap, 0, bitmap_words * sizeof(uint32_t), st)) != cudaSuccess) return e;
  }
  const int rows = a.T * a.N2;
  if (rows > 0) {
    prof_begin("nsa_kv_lists", st);
    nsa_kv_lists_kernel<<<(rows + 127) / 128, 128, 0, st>>>(a.topk, a.cu_seqlens, a.B, a.T, a.N2, a.K, a.sel_block,
                                                            a.nblk_max, a.words, a.ok_flag, a.ids, a.cnt, a.dup, bitmap,
                                                            a.status);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (!a.token_lists) return cudaSuccess;
  const int trows = a.B * a.N2 * a.nblk_max;
  const int grid = (trows + 7) / 8;
  prof_begin("nsa_token_count", st);
  nsa_column_kernel<false><<<grid, 256, 0, st>>>(a.bitmap, a.cu_seqlens, a.B, a.N2, a.sel_block, a.nblk_max, a.words,
                                                 a.ok_flag, a.t_counts, nullptr, nullptr);
  prof_end(st);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = exclusive_scan(a.t_counts, trows, a.t_row_ptr, st)) != cudaSuccess) return e;
  prof_begin("nsa_token_fill", st);
  nsa_column_kernel<true><<<grid, 256, 0, st>>>(a.bitmap, a.cu_seqlens, a.B, a.N2, a.sel_block, a.nblk_max, a.words,
                                                a.ok_flag, nullptr, a.t_row_ptr, a.t_col);
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace sa
