// NSA selected attention, backward preprocess and the block-major dK / dV pass for the shapes the
// tensor-core dK / dV kernel does not cover (NsaSelectedAttention page, forward formula:
// selected_key/value = Gather(key/value, topk_indices[i]); the backward applies the
// BlockSparseAttentionGrad formulas to the gathered blocks).  The token-major forward and dQ
// passes run on tcgen05 (nsa_tc.cu), dK / dV for 64-token blocks and G in {8, ..., 128} too
// (nsa_dkdv.cu).
//
// The fallback dK/dV pass here is block-major: one CTA per (b, g, kv block) walks the ascending
// token list of that block (nsa_meta.cu), warps each owning 16 of the block's keys with warp-level
// mma.sync (m16n8k16); a block listed twice by a token (literal Gather) counts twice.  P and dS
// enter the products that accumulate dV and dK as two bf16 parts (hi + lo).  It also serves
// 192-dim q / k (v and dOut keep 128), which the tensor-core dK / dV kernel's staging does not fit.
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

constexpr int kDV = 128;  // head dim of v, Out, dOut (q / k: 128 or 192)
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------------------------
// warp-level MMA and shared-memory helpers
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // zero-fill rows past the sequence
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// A [rows][W] bf16 tile in shared memory (W = 128 or 192, rows of 2W bytes), 16-byte chunks
// XOR-swizzled by row % 8 within each group of 8 (ldmatrix reads 8 rows of one chunk column
// conflict-free).
template <int W>
__device__ __forceinline__ uint32_t tile_off(int row, int chunk) {
  return static_cast<uint32_t>(row * (2 * W) + (((chunk ^ row) & 7) | (chunk & ~7)) * 16);
}

// B fragments for n = 16 rows of the tile, k = 16 columns starting at k0 (tile rows = n):
// non-transposed ldmatrix, two n8 tiles: {b0,b1} of rows 0-7 and of rows 8-15.
template <int W>
__device__ __forceinline__ void ldsm_b_rows(uint32_t (&r)[4], uint32_t tile, int k0, int lane) {
  const int row = (lane & 7) + ((lane >> 4) << 3);
  const int chunk = (k0 >> 3) + ((lane >> 3) & 1);
  ldsm_x4(r, tile + tile_off<W>(row, chunk));  // r0,r1: rows 0-7 (k lo, k hi); r2,r3: rows 8-15
}
// B fragments for k = 16 rows of the tile (keys), n = 16 columns starting at n0: transposed
// ldmatrix; r0,r1 = {b0,b1} of columns n0..n0+7, r2,r3 = of columns n0+8..n0+15.
template <int W>
__device__ __forceinline__ void ldsm_b_cols(uint32_t (&r)[4], uint32_t tile, int n0, int lane) {
  const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
  const int chunk = (n0 >> 3) + (lane >> 4);
  ldsm_x4_t(r, tile + tile_off<W>(row, chunk));
}
// A fragment (16 rows x 16 columns from k0) of a tile.
template <int W>
__device__ __forceinline__ void ldsm_a(uint32_t (&r)[4], uint32_t tile, int row0, int k0, int lane) {
  const int row = row0 + (lane & 7) + (((lane >> 3) & 1) << 3);
  const int chunk = (k0 >> 3) + (lane >> 4);
  ldsm_x4(r, tile + tile_off<W>(row, chunk));
}

__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(x0, x1);
  lo = pack_bf16(x0 - bf16lo(hi), x1 - bf16hi(hi));
}

struct NsaParams {
  int B, T, N1, N2, G, K, sel_block, mask_mode, head_tiles;
  float scale, scale_log2;
  const int32_t* cu;
  const int32_t* ok_flag;
  const int32_t* ids;  // [T][N2][K] ascending, -1 padded
  const int32_t* cnt;  // [T][N2]
  const int32_t* t_row_ptr;
  const int32_t* t_col;
  int nblk_max;
  const __nv_bfloat16 *q, *k, *v, *out, *dout;
  const float* lse;
  const float* lse2;   // [T][N1] LSE * log2(e), +inf for rows without keys
  const float* dvec;   // [T][N1] rowsum(dOut o Out)
  __nv_bfloat16 *o, *dq, *dk, *dv;
  float* lse_out;
  uint32_t* status;
};


// softmax_grad D = rowsum(dOut o Out) and LSE * log2(e) per (token, head); 8 threads per row
__global__ void nsa_prep_kernel(const NsaParams prm) {
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gid >> 3;
  const int part = static_cast<int>(gid & 7);
  const long long n_rows = static_cast<long long>(prm.T) * prm.N1;
  const bool live = row < n_rows;  // whole warps stay for the shuffles below
  const uint4* po = reinterpret_cast<const uint4*>(prm.out + (live ? row : 0) * kDV + part * 16);
  const uint4* pd = reinterpret_cast<const uint4*>(prm.dout + (live ? row : 0) * kDV + part * 16);
  float d = 0.f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint4 a = po[k], b = pd[k];
    d += bf16lo(a.x) * bf16lo(b.x) + bf16hi(a.x) * bf16hi(b.x);
    d += bf16lo(a.y) * bf16lo(b.y) + bf16hi(a.y) * bf16hi(b.y);
    d += bf16lo(a.z) * bf16lo(b.z) + bf16hi(a.z) * bf16hi(b.z);
    d += bf16lo(a.w) * bf16lo(b.w) + bf16hi(a.w) * bf16hi(b.w);
  }
  d += __shfl_xor_sync(0xffffffffu, d, 1);
  d += __shfl_xor_sync(0xffffffffu, d, 2);
  d += __shfl_xor_sync(0xffffffffu, d, 4);
  if (live && part == 0) {
    const_cast<float*>(prm.dvec)[row] = d;
    const float l = prm.lse[row];
    const_cast<float*>(prm.lse2)[row] = l == -INFINITY ? INFINITY : l * kLog2e;
  }
}

// ---------------------------------------------------------------------------------------------
// block-major dK / dV
// ---------------------------------------------------------------------------------------------
// one warp per 16 keys of the block (sel_block / 16 warps, at most 8); DQK = head dim of q / k
template <int DQK>
__global__ void __launch_bounds__(256) nsa_dkdv_kernel(const NsaParams prm) {
  constexpr int kQB = 16 * DQK * 2;  // bytes of a stage's Q tile (16 heads); dO follows it (4096)
  extern __shared__ __align__(128) uint8_t dsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x;  // (b, g, kb)
  const int kb = r % prm.nblk_max;
  const int bg = r / prm.nblk_max;
  const int b = bg / prm.N2, g = bg % prm.N2;
  if (!*prm.ok_flag) return;
  const int t0 = prm.cu[b], len = prm.cu[b + 1] - t0;
  const int nkeys = min(prm.sel_block, len - kb * prm.sel_block);  // keys of this block in the batch
  if (nkeys <= 0) return;
  const int nb = prm.sel_block;  // block tile rows (rows past nkeys are zero)
  const int rp = prm.t_row_ptr[r], n_tok = prm.t_row_ptr[r + 1] - rp;
  // shared memory: K [nb][DQK], V [nb][128] of the block; Q [16][DQK], dO [16][128] of one token's
  // 16 heads x 2 stages
  const uint32_t k_t = smem_u32(dsm), v_t = k_t + nb * DQK * 2;
  const uint32_t qd0 = v_t + nb * 256;  // stage s: Q at qd0 + s (kQB + 4096), dO at + kQB
  float* vec = reinterpret_cast<float*>(dsm + nb * (DQK * 2 + 256) + 2 * (kQB + 4096));  // [stage][lse2 16 | dvec 16]
  const int r0 = lane >> 2, cq = (lane & 3) * 2;
  const int key0 = warp * 16;  // this warp's keys within the block
  {
    const size_t row = static_cast<size_t>(t0 + kb * prm.sel_block) * prm.N2 + g;
    // every warp loads a quarter of K and V
    for (int i = threadIdx.x; i < nb * (DQK / 8); i += blockDim.x) {
      const int rr = i / (DQK / 8), c = i % (DQK / 8);
      const bool ok = rr < nkeys;
      cp_async16(k_t + tile_off<DQK>(rr, c), prm.k + (row + static_cast<size_t>(ok ? rr : 0) * prm.N2) * DQK + c * 8, ok);
    }
    for (int i = threadIdx.x; i < nb * 16; i += blockDim.x) {
      const int rr = i >> 4, c = i & 15;
      const bool ok = rr < nkeys;
      cp_async16(v_t + tile_off<kDV>(rr, c), prm.v + (row + static_cast<size_t>(ok ? rr : 0) * prm.N2) * kDV + c * 8, ok);
    }
    cp_commit();
  }
  const int items = n_tok * prm.head_tiles;
  auto issue = [&](int it) {
    const int tok = prm.t_col[rp + it / prm.head_tiles];
    const int ht = it % prm.head_tiles;
    const int h0 = g * prm.G + ht * 16;
    const int rows = min(16, prm.G - ht * 16);
    const uint32_t qs = qd0 + (it & 1) * (kQB + 4096);
    for (int i = threadIdx.x; i < 16 * (DQK / 8); i += blockDim.x) {
      const int rr = i / (DQK / 8), c = i % (DQK / 8);
      const bool ok = rr < rows;
      const size_t off = (static_cast<size_t>(tok) * prm.N1 + h0 + (ok ? rr : 0)) * DQK + c * 8;
      cp_async16(qs + tile_off<DQK>(rr, c), prm.q + off, ok);
    }
    for (int i = threadIdx.x; i < 16 * 16; i += blockDim.x) {
      const int rr = i >> 4, c = i & 15;
      const bool ok = rr < rows;
      const size_t off = (static_cast<size_t>(tok) * prm.N1 + h0 + (ok ? rr : 0)) * kDV + c * 8;
      cp_async16(qs + kQB + tile_off<kDV>(rr, c), prm.dout + off, ok);
    }
    if (threadIdx.x < 16) {
      const bool ok = threadIdx.x < rows;
      const size_t o = static_cast<size_t>(tok) * prm.N1 + h0 + threadIdx.x;
      vec[(it & 1) * 32 + threadIdx.x] = ok ? prm.lse2[o] : INFINITY;
      vec[(it & 1) * 32 + 16 + threadIdx.x] = ok ? prm.dvec[o] : 0.f;
    }
    cp_commit();
  };
  float dk[DQK / 8][4], dv[16][4];
#pragma unroll
  for (int n = 0; n < DQK / 8; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) dk[n][i] = 0.f;
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) dv[n][i] = 0.f;
  if (items > 0) issue(0);
  for (int it = 0; it < items; ++it) {
    if (it + 1 < items) {
      __syncthreads();  // stage (it+1)&1 was last read in iteration it-1
      issue(it + 1);
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const int tok = prm.t_col[rp + it / prm.head_tiles];
    const int qpos = tok - t0;
    // multiplicity of this block in the token's list (literal Gather counts duplicates)
    int mult = 0;
    {
      const int32_t* sl = prm.ids + (static_cast<size_t>(tok) * prm.N2 + g) * prm.K;
      const int nsl = prm.cnt[static_cast<size_t>(tok) * prm.N2 + g];
      for (int i = 0; i < nsl; ++i) mult += sl[i] == kb;
    }
    const uint32_t qs = qd0 + (it & 1) * (kQB + 4096), ds = qs + kQB;
    const float* l2 = vec + (it & 1) * 32;
    const float* dvv = l2 + 16;
    // S^T = K Q^T and dP^T = V dO^T: this warp's 16 keys x the token's 16 heads
    float st[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float dpt[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < DQK / 16; ++ks) {
      uint32_t ka[4], bq[4];
      ldsm_a<DQK>(ka, k_t, key0, ks * 16, lane);
      ldsm_b_rows<DQK>(bq, qs, ks * 16, lane);
      mma16816(st[0], ka, bq[0], bq[1]);
      mma16816(st[1], ka, bq[2], bq[3]);
    }
#pragma unroll
    for (int ks = 0; ks < kDV / 16; ++ks) {
      uint32_t va[4], bd[4];
      ldsm_a<kDV>(va, v_t, key0, ks * 16, lane);
      ldsm_b_rows<kDV>(bd, ds, ks * 16, lane);
      mma16816(dpt[0], va, bd[0], bd[1]);
      mma16816(dpt[1], va, bd[2], bd[3]);
    }
    // P^T, dS^T: rows = keys (key0 + r0 (+8)), columns = heads (n*8 + cq (+1))
    uint32_t p_hi[4], p_lo[4], s_hi[4], s_lo[4];
    float pv[2][4], sv[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int kr = key0 + r0 + (i >> 1) * 8;   // key row within the block
        const int hc = n * 8 + cq + (i & 1);       // head column
        const bool vis = kr < nkeys && (prm.mask_mode != 2 || kb * prm.sel_block + kr <= qpos);
        const float p = vis ? ex2(fmaf(st[n][i], prm.scale_log2, -l2[hc])) * static_cast<float>(mult) : 0.f;
        pv[n][i] = p;
        sv[n][i] = p * (dpt[n][i] - dvv[hc]);
      }
    split2(pv[0][0], pv[0][1], p_hi[0], p_lo[0]);
    split2(pv[0][2], pv[0][3], p_hi[1], p_lo[1]);
    split2(pv[1][0], pv[1][1], p_hi[2], p_lo[2]);
    split2(pv[1][2], pv[1][3], p_hi[3], p_lo[3]);
    split2(sv[0][0], sv[0][1], s_hi[0], s_lo[0]);
    split2(sv[0][2], sv[0][3], s_hi[1], s_lo[1]);
    split2(sv[1][0], sv[1][1], s_hi[2], s_lo[2]);
    split2(sv[1][2], sv[1][3], s_hi[3], s_lo[3]);
    // dV += P^T dO, dK += dS^T Q  (B = [16 heads][128 dims], transposed loads)
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
      uint32_t bdo[4];
      ldsm_b_cols<kDV>(bdo, ds, n * 8, lane);
      mma16816(dv[n], p_hi, bdo[0], bdo[1]);
      mma16816(dv[n + 1], p_hi, bdo[2], bdo[3]);
      mma16816(dv[n], p_lo, bdo[0], bdo[1]);
      mma16816(dv[n + 1], p_lo, bdo[2], bdo[3]);
    }
#pragma unroll
    for (int n = 0; n < DQK / 8; n += 2) {
      uint32_t bqq[4];
      ldsm_b_cols<DQK>(bqq, qs, n * 8, lane);
      mma16816(dk[n], s_hi, bqq[0], bqq[1]);
      mma16816(dk[n + 1], s_hi, bqq[2], bqq[3]);
      mma16816(dk[n], s_lo, bqq[0], bqq[1]);
      mma16816(dk[n + 1], s_lo, bqq[2], bqq[3]);
    }
  }
  if (items == 0) cp_wait<0>();
  // write dK (scaled) and dV for this warp's keys
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int kr = key0 + r0 + i * 8;
    if (kr >= nkeys) continue;
    const size_t krow = static_cast<size_t>(t0 + kb * prm.sel_block + kr) * prm.N2 + g;
#pragma unroll
    for (int n = 0; n < DQK / 8; ++n)
      *reinterpret_cast<uint32_t*>(prm.dk + krow * DQK + n * 8 + cq) =
          pack_bf16(dk[n][2 * i] * prm.scale, dk[n][2 * i + 1] * prm.scale);
#pragma unroll
    for (int n = 0; n < 16; ++n)
      *reinterpret_cast<uint32_t*>(prm.dv + krow * kDV + n * 8 + cq) = pack_bf16(dv[n][2 * i], dv[n][2 * i + 1]);
  }
}

// dK/dV rows of keys that no token selected stay zero: clear everything first (a: n8a chunks of
// 8 values, b: n8b)
__global__ void nsa_zero_kernel(__nv_bfloat16* __restrict__ a, long long n8a, __nv_bfloat16* __restrict__ b,
                                long long n8b) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n8a) reinterpret_cast<uint4*>(a)[i] = make_uint4(0, 0, 0, 0);
  if (i < n8b) reinterpret_cast<uint4*>(b)[i] = make_uint4(0, 0, 0, 0);
}

NsaParams make_params(const NsaArgs& a) {
  NsaParams p;
  p.B = a.B; p.T = a.T; p.N1 = a.N1; p.N2 = a.N2; p.G = a.N1 / a.N2; p.K = a.K; p.sel_block = a.sel_block;
  p.mask_mode = a.mask_mode; p.head_tiles = (p.G + 15) / 16;
  p.scale = a.scale; p.scale_log2 = a.scale * kLog2e;
  p.cu = a.cu_seqlens; p.ok_flag = a.ok_flag; p.ids = a.ids; p.cnt = a.cnt;
  p.t_row_ptr = a.t_row_ptr; p.t_col = a.t_col; p.nblk_max = a.nblk_max;
  p.q = static_cast<const __nv_bfloat16*>(a.q); p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.v = static_cast<const __nv_bfloat16*>(a.v); p.out = static_cast<const __nv_bfloat16*>(a.out_in);
  p.dout = static_cast<const __nv_bfloat16*>(a.dout);
  p.lse = a.lse_in; p.lse2 = a.lse2; p.dvec = a.dvec;
  p.o = static_cast<__nv_bfloat16*>(a.out); p.dq = static_cast<__nv_bfloat16*>(a.dq);
  p.dk = static_cast<__nv_bfloat16*>(a.dk); p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.lse_out = a.lse_out; p.status = a.status;
  return p;
}

}  // namespace

cudaError_t nsa_fwd_launch(const NsaArgs& a, cudaStream_t st) { return nsa_fwd_tc_launch(a, st); }

cudaError_t nsa_bwd_launch(const NsaArgs& a, cudaStream_t st) {
  const NsaParams p = make_params(a);
  cudaError_t e;
  const long long rows = static_cast<long long>(a.T) * a.N1;
  if (rows > 0) {
    prof_begin("nsa_bwd_prep", st);
    nsa_prep_kernel<<<static_cast<unsigned>((rows * 8 + 255) / 256), 256, 0, st>>>(p);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const long long n8k = static_cast<long long>(a.T) * a.N2 * a.D / 8;
  const long long n8v = static_cast<long long>(a.T) * a.N2 * kDV / 8;
  if (n8k > 0) {
    nsa_zero_kernel<<<static_cast<unsigned>((n8k + 255) / 256), 256, 0, st>>>(p.dk, n8k, p.dv, n8v);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int kv_rows = a.B * a.N2 * a.nblk_max;
  if (kv_rows > 0 && nsa_dkdv_tc_supported(a)) {
    if ((e = nsa_dkdv_tc_launch(a, st)) != cudaSuccess) return e;
  } else if (kv_rows > 0) {
    auto kern = a.D == 192 ? nsa_dkdv_kernel<192> : nsa_dkdv_kernel<128>;
    const size_t smem = static_cast<size_t>(a.sel_block) * (a.D * 2 + 256) + 2 * (16 * a.D * 2 + 4096) +
                        2 * 32 * sizeof(float);
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
      return e;
    prof_begin("nsa_bwd_dkdv_warp", st);
    kern<<<kv_rows, (a.sel_block / 16) * 32, smem, st>>>(p);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return nsa_dq_tc_launch(a, st);
}

}  // namespace sa
