// Sparse flash attention decode over a paged KV cache (SparseFlashAttention page, formula):
//   Out = softmax((q k~^T + q_rope k_rope~^T) * scale) v~,  D = Dv = 512, Dr = 64, q_len = 1
// where k~ / v~ are the tokens of the selected sparse blocks (sfa_meta.cu turns them into page
// lists and a work list of pieces).
//
// One CTA per piece: the G = N1/N2 query heads of one (batch, kv head) as the 128 rows of the MMA
// against a run of pages, for one half of Dv (O[:, 256*h .. +256]: the full 128 x 512 fp32 O
// would fill all of tensor memory).  Both Dv halves recompute S.  Tensor memory:
//   O half [0,256) | Q dims 0-255 as the A operand [256,384) | S0 [384,416) | S1 [416,448)
// Shared memory: Q dims 256-511 and the rope part (5 x 16 KB), K tiles of 32 tokens x 576 dims
// (2 stages x 9 boxes of 4 KB) and V tiles of 32 tokens x 256 dims (2 stages x 4 boxes).
// Warps 0-7 softmax (lane quarter = head rows, half = 16 of the tile's 32 keys), warp 8 TMA
// producer, warp 9 issues O += P V, warp 10 issues S (tcgen05.mma issue blocks while the tensor
// pipe's queue is full, so with one thread O += P_t V_t would wait behind the issue of S_{t+1}).  A piece covering a whole unit writes Out and LSE; otherwise it
// writes (O, m, l) partials that sfa_combine merges in piece order.
#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

constexpr int kM = 128;       // MMA rows (query heads of one kv head, padded)
constexpr int kTile = 32;     // tokens per KV tile
constexpr int kDQ = 512;      // q / k head dim
constexpr int kDR = 64;       // rope dim
constexpr int kDVH = 256;     // Dv half per CTA
constexpr int kKBoxes = 9;    // 8 boxes of k (64 dims) + 1 of k_rope
constexpr int kVBoxes = 4;    // 4 boxes of v (64 dims) per Dv half
constexpr int kVecWarps = 8;
constexpr int kThreads = (kVecWarps + 3) * 32;
constexpr uint32_t kColO = 0, kColQ = 256, kColS0 = 384, kColS1 = 416;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(1024) DecSmem {
  uint8_t qhi[5][kM * 128];              // Q dims 256-511 (4 boxes) + rope (1 box), [128 rows][64]
  uint8_t k[2][kKBoxes][kTile * 128];    // [stage][box] [32 tokens][64 dims]
  uint8_t v[2][kVBoxes][kTile * 128];
  float red[2][2][kM];
  uint64_t bar_q, bar_qlo, bar_k[2], bar_k_empty[2], bar_v[2], bar_v_empty[2], bar_s_full[2];
  uint64_t bar_p_full[2];   // per S buffer: P of its tile is written (256 arrivals)
  uint64_t bar_pv_done[2];  // per S buffer: the O += P V that read it has completed
  uint64_t bar_o_done, bar_done, bar_pair[4];
  uint32_t tmem_base;
};

struct DecParams {
  int B, N1, N2, G, page_size, cap;
  float scale_log2;
  const int32_t* pages;
  const int32_t* tokens;
  const int32_t* piece_unit;
  const int32_t* piece_begin;
  const int32_t* piece_len;
  const int32_t* unit_pieces;
  const int32_t* n_pieces;
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  float* lse;
  float* part_o;  // [piece][128][256]
  float* part_m;  // [piece][128]
  float* part_l;
  uint32_t* status;
};

__device__ __forceinline__ bool pair_sync(uint64_t* bar, int& exchanges, uint32_t* status) {
  tc_fence_before();
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, exchanges & 1, status);
  ++exchanges;
  tc_fence_after();
  return ok;
}

__global__ void __launch_bounds__(kThreads, 1)
    sfa_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kr,
                      const __grid_constant__ CUtensorMap tm_v, const DecParams prm) {
  griddep_launch_dependents();  // the combine may launch now; it waits for this grid's results
  griddep_wait();               // launched early: the work list must be complete
  const int piece = blockIdx.x;
  if (piece >= *prm.n_pieces) return;  // uniform for the whole CTA
  extern __shared__ uint8_t smem_raw[];
  DecSmem& s = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = prm.piece_unit[piece];
  const int bg = u >> 1, dvh = u & 1;
  const int b = bg / prm.N2, g = bg % prm.N2;
  const int pbeg = prm.piece_begin[piece];
  const int npages = prm.piece_len[piece];
  const int tiles_per_page = prm.page_size / kTile;
  const int n_tiles = npages * tiles_per_page;
  const int32_t* plist = prm.pages + static_cast<size_t>(bg) * prm.cap + pbeg;
  const int32_t* tlist = prm.tokens + static_cast<size_t>(bg) * prm.cap + pbeg;
  const int qrow0 = b * prm.N1 + g * prm.G;  // first query row (head) of this kv head

  if (tid == 0) {
    mbar_init(&s.bar_q, 1);
    mbar_init(&s.bar_qlo, kVecWarps * 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.bar_k[i], 1);
      mbar_init(&s.bar_k_empty[i], 1);
      mbar_init(&s.bar_v[i], 1);
      mbar_init(&s.bar_v_empty[i], 1);
      mbar_init(&s.bar_s_full[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.bar_p_full[i], kVecWarps * 32);
      mbar_init(&s.bar_pv_done[i], 1);
    }
    mbar_init(&s.bar_o_done, 1);
    mbar_init(&s.bar_done, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&s.bar_pair[i], 64);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == kVecWarps) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
      mbar_arrive_expect_tx(&s.bar_q, 5 * kM * 128);
      for (int c = 0; c < 4; ++c) tma_load_2d(s.qhi[c], &tm_q, &s.bar_q, 256 + c * 64, qrow0);
      tma_load_2d(s.qhi[4], &tm_qr, &s.bar_q, 0, qrow0);
      int issued = 0;
      bool ok = true;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j & 1, use = j >> 1;
        const int page = plist[j / tiles_per_page];
        const int tok = page * prm.page_size + (j % tiles_per_page) * kTile;
        if (j >= 2 && !(ok = mbar_wait(&s.bar_k_empty[st], (use - 1) & 1, prm.status))) break;
        mbar_arrive_expect_tx(&s.bar_k[st], kKBoxes * kTile * 128);
        for (int c = 0; c < 8; ++c) tma_load_3d(s.k[st][c], &tm_k, &s.bar_k[st], c * 64, g, tok);
        tma_load_3d(s.k[st][8], &tm_kr, &s.bar_k[st], 0, g, tok);
        if (j >= 2 && !(ok = mbar_wait(&s.bar_v_empty[st], (use - 1) & 1, prm.status))) {
          issued = -(j + 1);
          break;
        }
        mbar_arrive_expect_tx(&s.bar_v[st], kVBoxes * kTile * 128);
        for (int c = 0; c < kVBoxes; ++c) tma_load_3d(s.v[st][c], &tm_v, &s.bar_v[st], dvh * kDVH + c * 64, g, tok);
        issued = j + 1;
      }
      const int nk = issued < 0 ? -issued : issued;
      const int nv = issued < 0 ? -issued - 1 : issued;
      for (int j = (nk > 2 ? nk - 2 : 0); j < nk; ++j) mbar_wait(&s.bar_k[j & 1], (j >> 1) & 1, prm.status);
      for (int j = (nv > 2 ? nv - 2 : 0); j < nv; ++j) mbar_wait(&s.bar_v[j & 1], (j >> 1) & 1, prm.status);
      mbar_wait(&s.bar_q, 0, prm.status);
    }
  } else if (warp == kVecWarps + 1 || warp == kVecWarps + 2) {
    // ------------------------------------------------------------------ MMA issuers
    if (lane == 0 && n_tiles > 0) {
      const bool pv_thread = warp == kVecWarps + 1;
      bool ok = true;
      if (pv_thread) {
        const uint32_t id_o = idesc_bf16_f32(kM, kDVH, false, true);
        const uint64_t dv0 = sdesc_sw128(smem_u32(s.v[0][0]), kTile * 128, 1024);
        constexpr uint32_t kV16 = (kVBoxes * kTile * 128) >> 4;
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int st = j & 1;
          // one barrier per S buffer: its next phase needs S_{j+2}, which waits for this product
          if (!(ok = mbar_wait(&s.bar_p_full[st], (j >> 1) & 1, prm.status))) break;
          if (!(ok = mbar_wait(&s.bar_v[st], (j >> 1) & 1, prm.status))) break;
          tc_fence_after();
          const uint32_t p_col = st ? kColS1 : kColS0;
          const uint64_t dv = dv0 + static_cast<uint64_t>(st) * kV16;
#pragma unroll
          for (int ks = 0; ks < kTile / 16; ++ks)
            mma_bf16_ts(tmem + kColO, tmem + p_col + ks * 8, sdesc_add(dv, ks * 2048), id_o,
                        (j > 0 || ks > 0) ? 1u : 0u);
          tc_commit(&s.bar_o_done);
          tc_commit(&s.bar_v_empty[st]);
          tc_commit(&s.bar_pv_done[st]);
        }
        if (ok) tc_commit(&s.bar_done);
      } else {
        const uint32_t id_s = idesc_bf16_f32(kM, kTile, false, false);
        // descriptors of stage 0 / box 0; stages, boxes and K steps are added offsets
        const uint64_t dqh = sdesc_sw128(smem_u32(s.qhi[0]), 0, 1024);
        const uint64_t dk0 = sdesc_sw128(smem_u32(s.k[0][0]), 0, 1024);
        constexpr uint32_t kK16 = (kKBoxes * kTile * 128) >> 4;
        ok = mbar_wait(&s.bar_q, 0, prm.status) && mbar_wait(&s.bar_qlo, 0, prm.status);
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int st = j & 1;
          // S buffer st last held P_{j-2}; exact parity: pv_done's next phase needs P_j
          if (j >= 2 && !(ok = mbar_wait(&s.bar_pv_done[st], ((j >> 1) - 1) & 1, prm.status))) break;
          if (!(ok = mbar_wait(&s.bar_k[st], (j >> 1) & 1, prm.status))) break;
          tc_fence_after();
          const uint32_t d = tmem + (st ? kColS1 : kColS0);
          const uint64_t dk = dk0 + static_cast<uint64_t>(st) * kK16;
          // dims 0-255: A = Q from tensor memory; dims 256-575: A = Q from shared memory
#pragma unroll
          for (int ks = 0; ks < 16; ++ks)
            mma_bf16_ts(d, tmem + kColQ + ks * 8, sdesc_add(dk, (ks >> 2) * (kTile * 128) + (ks & 3) * 32), id_s,
                        ks > 0 ? 1u : 0u);
#pragma unroll
          for (int ks = 16; ks < 36; ++ks) {
            const int qs = ks - 16;
            mma_bf16_ss(d, sdesc_add(dqh, (qs >> 2) * (kM * 128) + (qs & 3) * 32),
                        sdesc_add(dk, (ks >> 2) * (kTile * 128) + (ks & 3) * 32), id_s, 1u);
          }
          tc_commit(&s.bar_s_full[st]);
          tc_commit(&s.bar_k_empty[st]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // head row == TMEM lane
    const bool row_valid = r < prm.G;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    // Q dims [hf*128, hf*128+128) of this row into TMEM as packed bf16 pairs (A operand of S)
    {
      const uint4* src = reinterpret_cast<const uint4*>(prm.q + static_cast<size_t>(qrow0 + r) * kDQ + hf * 128);
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 4 x 16 packed columns = 128 dims
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v4 = row_valid ? src[c * 4 + i] : make_uint4(0, 0, 0, 0);
          w[4 * i] = v4.x;
          w[4 * i + 1] = v4.y;
          w[4 * i + 2] = v4.z;
          w[4 * i + 3] = v4.w;
        }
        tmem_st16(tmem + lane_base + kColQ + hf * 64 + c * 16, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&s.bar_qlo);
    }
    const uint32_t o_col = kColO + hf * (kDVH / 2);
    float m = -INFINITY, l = 0.f;
    int exchanges = 0;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_s_full[st], (j >> 1) & 1, prm.status));
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_col = st ? kColS1 : kColS0;
      // valid keys of this tile: tokens [t0, t0 + 32) of the page, of which `valid` are in use
      const int valid = tlist[j / tiles_per_page] - (j % tiles_per_page) * kTile;
      float x[16];
      {
        uint32_t rr[16];
        tmem_ld16(tmem + lane_base + s_col + hf * 16, rr);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          reg_fence(rr[i]);
          x[i] = (row_valid && hf * 16 + i < valid) ? __uint_as_float(rr[i]) : -INFINITY;
        }
      }
      float mx = x[0];
#pragma unroll
      for (int i = 1; i < 16; ++i) mx = fmaxf(mx, x[i]);
      s.red[st][hf][r] = mx;
      ok = __all_sync(0xffffffffu, pair_sync(&s.bar_pair[quarter], exchanges, prm.status));
      if (!ok) break;
      mx = fmaxf(mx, s.red[st][hf ^ 1][r]) * prm.scale_log2;
      float m_new = m;
      bool need = false;
      if (mx > m + 8.f) {
        need = (m != -INFINITY);
        m_new = mx;
      }
      if (__any_sync(0xffffffffu, need)) {
        // o_done phase j-1 (O += P_{j-1} V_{j-1}); phase j-2 is complete (S_j waited for it)
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_o_done, (j - 1) & 1, prm.status));
        if (!ok) break;
        tc_fence_after();
        const float alpha = need ? ex2(m - m_new) : 1.f;
        l *= alpha;
#pragma unroll
        for (int c = 0; c < kDVH / 2; c += 32) {
          uint32_t rr[32];
          tmem_ld32(tmem + lane_base + o_col + c, rr);
          tmem_ld_wait(rr);
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
          tmem_st32(tmem + lane_base + o_col + c, rr);
        }
        tmem_st_wait();
      }
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      uint32_t hv[8];
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float e0 = ex2(fmaf(x[2 * i], prm.scale_log2, -m_use));
        const float e1 = ex2(fmaf(x[2 * i + 1], prm.scale_log2, -m_use));
        rs += e0 + e1;
        hv[i] = pack_bf16(e0, e1);
      }
      tmem_st8(tmem + lane_base + s_col + hf * 8, hv);
      tmem_st_wait();
      l += rs;
      m = m_new;
      tc_fence_before();
      mbar_arrive(&s.bar_p_full[st]);
    }
    // ---- epilogue
    bool have = ok && n_tiles > 0;
    if (have) {
      have = __all_sync(0xffffffffu, mbar_wait(&s.bar_done, 0, prm.status));
      tc_fence_after();
    }
    s.red[n_tiles & 1][hf][r] = l;
    if (ok) have = __all_sync(0xffffffffu, pair_sync(&s.bar_pair[quarter], exchanges, prm.status)) && have;
    l += s.red[n_tiles & 1][hf ^ 1][r];
    const bool single = prm.unit_pieces[u] == 1;
    const bool any = have && l > 0.f;
    const float inv_l = any ? 1.f / l : 0.f;
    const size_t orow = static_cast<size_t>(qrow0 + r);
#pragma unroll
    for (int c = 0; c < kDVH / 2; c += 32) {
      uint32_t rr[32];
      if (have) {
        tmem_ld32(tmem + lane_base + o_col + c, rr);
        tmem_ld_wait(rr);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) rr[i] = 0u;
      }
      if (!row_valid) continue;
      const int d0 = dvh * kDVH + hf * (kDVH / 2) + c;
      if (single) {
        __nv_bfloat16* dst = prm.out + orow * kDQ + d0;
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint4 pk;
          pk.x = pack_bf16(__uint_as_float(rr[i + 0]) * inv_l, __uint_as_float(rr[i + 1]) * inv_l);
          pk.y = pack_bf16(__uint_as_float(rr[i + 2]) * inv_l, __uint_as_float(rr[i + 3]) * inv_l);
          pk.z = pack_bf16(__uint_as_float(rr[i + 4]) * inv_l, __uint_as_float(rr[i + 5]) * inv_l);
          pk.w = pack_bf16(__uint_as_float(rr[i + 6]) * inv_l, __uint_as_float(rr[i + 7]) * inv_l);
          *reinterpret_cast<uint4*>(dst + i) = pk;
        }
      } else {
        float* dst = prm.part_o + (static_cast<size_t>(piece) * kM + r) * kDVH + hf * (kDVH / 2) + c;
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(dst + i) = make_float4(__uint_as_float(rr[i]), __uint_as_float(rr[i + 1]),
                                                            __uint_as_float(rr[i + 2]), __uint_as_float(rr[i + 3]));
      }
    }
    if (row_valid && hf == 0) {
      if (single) {
        if (dvh == 0) prm.lse[orow] = any ? (m * kLn2 + logf(l)) : -INFINITY;
      } else {
        prm.part_m[static_cast<size_t>(piece) * kM + r] = (have && l > 0.f) ? m : -INFINITY;
        prm.part_l[static_cast<size_t>(piece) * kM + r] = have ? l : 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Merge the pieces of each unit in piece order:  M = max m_p, L = sum l_p 2^(m_p - M),
// Out = sum O_p 2^(m_p - M) / L,  LSE = (M + log2 L) ln 2.  One warp per (unit, head row); each
// lane owns 8 of the 256 Dv columns, so every partial row is read with coalesced 16-byte loads.
__global__ void __launch_bounds__(256) sfa_combine_kernel(const DecParams prm, const int32_t* __restrict__ unit_first) {
  griddep_wait();  // launched early: the decode pieces must be complete
  const int u = blockIdx.x;
  const int r = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= prm.G) return;
  const int pcs = prm.unit_pieces[u];
  if (pcs == 1) return;  // written by its single piece
  const int bg = u >> 1, dvh = u & 1;
  const int b = bg / prm.N2, g = bg % prm.N2;
  const int p0 = unit_first[u];
  const size_t orow = static_cast<size_t>(b * prm.N1 + g * prm.G + r);
  __nv_bfloat16* dst = prm.out + orow * kDQ + dvh * kDVH + lane * 8;
  float M = -INFINITY;
  for (int p = 0; p < pcs; ++p) M = fmaxf(M, prm.part_m[static_cast<size_t>(p0 + p) * kM + r]);
  float L = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int p = 0; p < pcs; ++p) {
    const float mp = prm.part_m[static_cast<size_t>(p0 + p) * kM + r];
    if (mp == -INFINITY) continue;
    const float wgt = ex2(mp - M);
    L += prm.part_l[static_cast<size_t>(p0 + p) * kM + r] * wgt;
    const float4* src = reinterpret_cast<const float4*>(prm.part_o + (static_cast<size_t>(p0 + p) * kM + r) * kDVH +
                                                        lane * 8);
    const float4 a = src[0], c = src[1];
    acc[0] += a.x * wgt; acc[1] += a.y * wgt; acc[2] += a.z * wgt; acc[3] += a.w * wgt;
    acc[4] += c.x * wgt; acc[5] += c.y * wgt; acc[6] += c.z * wgt; acc[7] += c.w * wgt;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;  // pcs == 0 (no selected key): Out = 0, LSE = -inf
  uint4 pk;
  pk.x = pack_bf16(acc[0] * inv, acc[1] * inv);
  pk.y = pack_bf16(acc[2] * inv, acc[3] * inv);
  pk.z = pack_bf16(acc[4] * inv, acc[5] * inv);
  pk.w = pack_bf16(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(dst) = pk;
  if (lane == 0 && dvh == 0) prm.lse[orow] = L > 0.f ? (M * kLn2 + logf(L)) : -INFINITY;
}

}  // namespace

cudaError_t sfa_decode_launch(const SfaDecodeArgs& a, cudaStream_t st) {
  CUtensorMap tq, tqr, tk, tkr, tv;
  const uint64_t qrows = static_cast<uint64_t>(a.B) * a.N1;
  const uint64_t tokens = static_cast<uint64_t>(a.num_pages) * a.page_size;
  if (!make_tmap_2d_bf16(&tq, a.q, qrows, kDQ, kDQ, kM) || !make_tmap_2d_bf16(&tqr, a.q_rope, qrows, kDR, kDR, kM) ||
      !make_tmap_3d_bf16(&tk, a.k_cache, kDQ, a.N2, tokens, kDQ, static_cast<uint64_t>(a.N2) * kDQ, 1, kTile) ||
      !make_tmap_3d_bf16(&tkr, a.k_rope_cache, kDR, a.N2, tokens, kDR, static_cast<uint64_t>(a.N2) * kDR, 1, kTile) ||
      !make_tmap_3d_bf16(&tv, a.v_cache, kDQ, a.N2, tokens, kDQ, static_cast<uint64_t>(a.N2) * kDQ, 1, kTile))
    return cudaErrorInvalidValue;
  DecParams p;
  p.B = a.B; p.N1 = a.N1; p.N2 = a.N2; p.G = a.N1 / a.N2; p.page_size = a.page_size; p.cap = a.cap;
  p.scale_log2 = a.scale * kLog2e;
  p.pages = a.pages; p.tokens = a.tokens; p.piece_unit = a.piece_unit; p.piece_begin = a.piece_begin;
  p.piece_len = a.piece_len; p.unit_pieces = a.unit_pieces; p.n_pieces = a.n_pieces;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.out = static_cast<__nv_bfloat16*>(a.out); p.lse = a.lse;
  p.part_o = a.part_o; p.part_m = a.part_m; p.part_l = a.part_l; p.status = a.status;
  const size_t smem = sizeof(DecSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(sfa_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  prof_begin("sfa_decode", st);
  e = launch_pdl(sfa_decode_kernel, dim3(a.max_pieces), dim3(kThreads), smem, st, tq, tqr, tk, tkr, tv, p);
  prof_end(st);
  if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
  prof_begin("sfa_combine", st);
  e = launch_pdl(sfa_combine_kernel, dim3(a.units, (p.G + 7) / 8), dim3(256), 0, st, p, a.unit_first);
  prof_end(st);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sa
