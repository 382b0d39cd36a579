// Block-sparse attention backward on tcgen05 (BlockSparseAttentionGrad page, backward formulas):
//   softmax_grad = rowsum(dOut o Out);  dP = dOut V^T;  dS = P o (dP - softmax_grad)
//   dV = P^T dOut;  dQ = (dS K) scale;  dK = (dS^T Q) scale
// P is recomputed from the forward's LSE: P = exp(scale q.k - LSE).
//
// Three kernels, no atomics (run-to-run bit identical):
//   bwd_prep     softmax_grad (D) and LSE*log2(e) per query row, written into 128-row padded
//                tiles so the passes below can bulk-load a tile's vectors.
//   bwd_kv       one CTA per KV block (b, g, kb) walking its transposed list of Q tiles (the
//                group's query heads included, in a fixed order): S^T = K Q^T, P^T, dP^T = V dO^T,
//                dV += P^T dO, dS^T = P^T o (dP^T - D), dK += dS^T Q.  TMEM holds S^T, dP^T, dV, dK.
//   bwd_q        one CTA per Q tile (b, h, qb) walking its KV list: S = Q K^T, P, dP = dO V^T,
//                dS, dQ += dS K.  TMEM holds two S buffers, dP and dQ.
#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

constexpr int kT = 128;  // rows of a Q tile and of a KV tile in the MMAs (M and N)
constexpr int kD = 128;
constexpr int kVecWarps = 8;  // element-wise warps: lane quarter = warp % 4, column half = warp / 4
constexpr int kThreads = (kVecWarps + 2) * 32;
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------------------------------------
// preprocess: D_i = sum_d dOut_id Out_id ; L2_i = LSE_i * log2(e)  (+inf where the row has no key
// or the tile row is padding, which makes exp2(s - L2) = 0 there)
// ------------------------------------------------------------------------------------------------
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                                const float* __restrict__ lse, int S_q, int bx, int nqb, long long n_rows,
                                float* __restrict__ dvec, float* __restrict__ lse2) {
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row = gid >> 3;  // 8 threads per row, 16 elements each
  const int part = static_cast<int>(gid & 7);
  if (row >= n_rows) return;
  const long long tile = row / kT;
  const int i = static_cast<int>(row % kT);
  const long long bh = tile / nqb;
  const int qb = static_cast<int>(tile % nqb);
  const int qpos = qb * bx + i;
  const bool valid = i < bx && qpos < S_q;
  float d = 0.f;
  if (valid) {
    const size_t g = (static_cast<size_t>(bh) * S_q + qpos) * kD + part * 16;
    const uint4* po = reinterpret_cast<const uint4*>(out + g);
    const uint4* pd = reinterpret_cast<const uint4*>(dout + g);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint4 a = po[k], b = pd[k];
      d += bf16lo(a.x) * bf16lo(b.x) + bf16hi(a.x) * bf16hi(b.x);
      d += bf16lo(a.y) * bf16lo(b.y) + bf16hi(a.y) * bf16hi(b.y);
      d += bf16lo(a.z) * bf16lo(b.z) + bf16hi(a.z) * bf16hi(b.z);
      d += bf16lo(a.w) * bf16lo(b.w) + bf16hi(a.w) * bf16hi(b.w);
    }
  }
  d += __shfl_xor_sync(0xffffffffu, d, 1);
  d += __shfl_xor_sync(0xffffffffu, d, 2);
  d += __shfl_xor_sync(0xffffffffu, d, 4);
  if (part == 0) {
    dvec[row] = valid ? d : 0.f;
    float l2 = INFINITY;
    if (valid) {
      const float l = lse[static_cast<size_t>(bh) * S_q + qpos];
      l2 = (l == -INFINITY) ? INFINITY : l * kLog2e;
    }
    lse2[row] = l2;
  }
}

struct BwdParams {
  int B, N1, N2, S_q, S_kv, bx, by, nqb, nkb, mask_mode, win_left, win_right;
  float scale, scale_log2;
  const int32_t* row_ptr;  // KV lists (Q-major pass) or transposed lists (KV-major pass)
  const int32_t* col;
  const float* dvec;       // [B*N1*nqb*128]
  const float* lse2;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  uint32_t* status;
};

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const uint32_t (&rr)[32], float mul) {
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    uint4 pk;
    pk.x = pack_bf16(__uint_as_float(rr[i + 0]) * mul, __uint_as_float(rr[i + 1]) * mul);
    pk.y = pack_bf16(__uint_as_float(rr[i + 2]) * mul, __uint_as_float(rr[i + 3]) * mul);
    pk.z = pack_bf16(__uint_as_float(rr[i + 4]) * mul, __uint_as_float(rr[i + 5]) * mul);
    pk.w = pack_bf16(__uint_as_float(rr[i + 6]) * mul, __uint_as_float(rr[i + 7]) * mul);
    *reinterpret_cast<uint4*>(dst + i) = pk;
  }
}

// Exchange point of the two element-wise warps that share a TMEM lane quarter (64 arrivals,
// bounded wait).  Orders each side's tensor-memory reads before the other side's writes.
__device__ __forceinline__ bool pair_sync(uint64_t* bar, int& exchanges, uint32_t* status) {
  tc_fence_before();
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, exchanges & 1, status);
  ++exchanges;
  tc_fence_after();
  return ok;
}

// Split x into bf16 hi + lo (x ~= hi + lo to about 2^-17 relative): the dK and dQ products run as
// two MMAs, hi then lo, so dS enters the tensor cores with ~16 significant bits.
__device__ __forceinline__ void split_pack(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(x0, x1);
  lo = pack_bf16(x0 - bf16lo(hi), x1 - bf16hi(hi));
}

// ------------------------------------------------------------------------------------------------
// KV-major pass: dK, dV
// TMEM columns: S^T [0,128) | dP^T [128,256) | dV [256,384) | dK [384,512).
// After the P/dS warpgroup has read S^T and dP^T, it writes back the bf16 MMA A operands over
// the consumed columns: P^T hi/lo -> S^T[0,64)/[64,128), dS^T hi/lo -> dP^T[0,64)/[64,128).
// ------------------------------------------------------------------------------------------------
struct __align__(1024) KvSmem {
  uint8_t k[2][kT * 128];        // K tile [128 keys][64 d] x 2
  uint8_t v[2][kT * 128];
  uint8_t q[2][2][kT * 128];     // [stage][sub-tile] Q tile [128 queries][64 d]
  uint8_t dout[2][2][kT * 128];  // [stage][sub-tile] dO tile
  float lse2[2][kT];             // per Q stage
  float dvec[2][kT];
  uint64_t bar_kv, bar_q[2], bar_do[2];
  uint64_t bar_s_full, bar_dp_full, bar_p_ready, bar_ds_ready, bar_done;
  uint64_t bar_q_empty[2], bar_do_empty[2];
  uint64_t bar_pair[4];
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(kThreads, 1)
    bsa_bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const BwdParams prm) {
  constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384;
  extern __shared__ uint8_t smem_raw[];
  KvSmem& s = *reinterpret_cast<KvSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bg = blockIdx.x / prm.nkb;
  const int kb = static_cast<int>(blockIdx.x % prm.nkb);  // early KV blocks have the longest lists
  const int b = bg / prm.N2, g = bg % prm.N2;
  const int G = prm.N1 / prm.N2;
  const int unit = bg * prm.nkb + kb;
  const int rp = prm.row_ptr[unit];
  const int n = prm.row_ptr[unit + 1] - rp;
  const int kv_row0 = bg * prm.S_kv + kb * prm.by;

  if (tid == 0) {
    mbar_init(&s.bar_kv, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.bar_q[i], 1);
      mbar_init(&s.bar_do[i], 1);
      mbar_init(&s.bar_q_empty[i], 1);
      mbar_init(&s.bar_do_empty[i], 1);
    }
    mbar_init(&s.bar_s_full, 1);
    mbar_init(&s.bar_dp_full, 1);
    mbar_init(&s.bar_p_ready, kVecWarps * 32);
    mbar_init(&s.bar_ds_ready, kVecWarps * 32);
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

  auto entry_rows = [&](int i, int& qrow, int& tile, int& qpos0) {
    const int e = prm.col[rp + i];
    const int hl = e / prm.nqb, qb = e % prm.nqb;
    const int bh = b * prm.N1 + g * G + hl;
    qrow = bh * prm.S_q + qb * prm.bx;
    tile = bh * prm.nqb + qb;
    qpos0 = qb * prm.bx;
  };

  if (warp == kVecWarps) {
    // ------------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      mbar_arrive_expect_tx(&s.bar_kv, 4 * kT * 128);
      tma_load_2d(s.k[0], &tm_k, &s.bar_kv, 0, kv_row0);
      tma_load_2d(s.k[1], &tm_k, &s.bar_kv, 64, kv_row0);
      tma_load_2d(s.v[0], &tm_v, &s.bar_kv, 0, kv_row0);
      tma_load_2d(s.v[1], &tm_v, &s.bar_kv, 64, kv_row0);
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i & 1;
        int qrow, tile, qpos0;
        entry_rows(i, qrow, tile, qpos0);
        if (i >= 2 && !mbar_wait(&s.bar_q_empty[st], ((i - 2) >> 1) & 1, prm.status)) break;
        mbar_arrive_expect_tx(&s.bar_q[st], 2 * kT * 128 + 2 * kT * 4);
        tma_load_2d(s.q[st][0], &tm_q, &s.bar_q[st], 0, qrow);
        tma_load_2d(s.q[st][1], &tm_q, &s.bar_q[st], 64, qrow);
        bulk_load(s.lse2[st], prm.lse2 + static_cast<size_t>(tile) * kT, kT * 4, &s.bar_q[st]);
        bulk_load(s.dvec[st], prm.dvec + static_cast<size_t>(tile) * kT, kT * 4, &s.bar_q[st]);
        if (i >= 2 && !mbar_wait(&s.bar_do_empty[st], ((i - 2) >> 1) & 1, prm.status)) {
          issued = -(i + 1);  // Q issued, dO not
          break;
        }
        mbar_arrive_expect_tx(&s.bar_do[st], 2 * kT * 128);
        tma_load_2d(s.dout[st][0], &tm_do, &s.bar_do[st], 0, qrow);
        tma_load_2d(s.dout[st][1], &tm_do, &s.bar_do[st], 64, qrow);
        issued = i + 1;
      }
      const int nq = issued < 0 ? -issued : issued;
      const int ndo = issued < 0 ? -issued - 1 : issued;
      for (int i = (nq > 2 ? nq - 2 : 0); i < nq; ++i) mbar_wait(&s.bar_q[i & 1], (i >> 1) & 1, prm.status);
      for (int i = (ndo > 2 ? ndo - 2 : 0); i < ndo; ++i) mbar_wait(&s.bar_do[i & 1], (i >> 1) & 1, prm.status);
      mbar_wait(&s.bar_kv, 0, prm.status);
    }
  } else if (warp == kVecWarps + 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      const uint32_t id_kmaj = idesc_bf16_f32(kT, kT, false, false);  // S^T, dP^T
      const uint32_t id_mnb = idesc_bf16_f32(kT, kD, false, true);    // dV, dK (B = [queries][d])
      auto mma_ss = [&](uint32_t d, const uint8_t (*a)[kT * 128], const uint8_t (*bm)[kT * 128]) {
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t ad = sdesc_sw128(smem_u32(a[ks >> 2]) + (ks & 3) * 32, 0, 1024);
          const uint64_t bd = sdesc_sw128(smem_u32(bm[ks >> 2]) + (ks & 3) * 32, 0, 1024);
          mma_bf16_ss(d, ad, bd, id_kmaj, ks > 0 ? 1u : 0u);
        }
      };
      auto mma_ts = [&](uint32_t d, uint32_t a_col, const uint8_t (*bm)[kT * 128], bool acc) {
#pragma unroll
        for (int ks = 0; ks < kT / 16; ++ks) {
          const uint64_t bd = sdesc_sw128(smem_u32(bm[0]) + ks * 2048, kT * 128, 1024);
          mma_bf16_ts(d, tmem + a_col + ks * 8, bd, id_mnb, (acc || ks > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(&s.bar_kv, 0, prm.status) && mbar_wait(&s.bar_q[0], 0, prm.status);
      if (ok) {
        tc_fence_after();
        mma_ss(tmem + kColS, s.k, s.q[0]);
        tc_commit(&s.bar_s_full);
        ok = mbar_wait(&s.bar_do[0], 0, prm.status);
      }
      if (ok) {
        tc_fence_after();
        mma_ss(tmem + kColDP, s.v, s.dout[0]);
        tc_commit(&s.bar_dp_full);
      }
      for (int i = 0; ok && i < n; ++i) {
        const int st = i & 1;
        if (!(ok = mbar_wait(&s.bar_p_ready, i & 1, prm.status))) break;
        tc_fence_after();
        mma_ts(tmem + kColDV, kColS, s.dout[st], i > 0);       // dV += P^T_hi dO
        mma_ts(tmem + kColDV, kColS + 64, s.dout[st], true);   // dV += P^T_lo dO
        tc_commit(&s.bar_do_empty[st]);
        if (!(ok = mbar_wait(&s.bar_ds_ready, i & 1, prm.status))) break;
        tc_fence_after();
        mma_ts(tmem + kColDK, kColDP, s.q[st], i > 0);       // dK += dS^T_hi Q
        mma_ts(tmem + kColDK, kColDP + 64, s.q[st], true);   // dK += dS^T_lo Q
        tc_commit(&s.bar_q_empty[st]);
        if (i + 1 < n) {
          if (!(ok = mbar_wait(&s.bar_q[st ^ 1], ((i + 1) >> 1) & 1, prm.status))) break;
          tc_fence_after();
          mma_ss(tmem + kColS, s.k, s.q[st ^ 1]);
          tc_commit(&s.bar_s_full);
          if (!(ok = mbar_wait(&s.bar_do[st ^ 1], ((i + 1) >> 1) & 1, prm.status))) break;
          tc_fence_after();
          mma_ss(tmem + kColDP, s.v, s.dout[st ^ 1]);
          tc_commit(&s.bar_dp_full);
        }
      }
      if (ok) tc_commit(&s.bar_done);
    }
  } else {
    // ------------------------------------------------------------------ P / dS warps
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // key row within the KV tile == TMEM lane
    const int c0 = hf * (kT / 2);       // this thread's query columns [c0, c0 + 64)
    const int kpos = kb * prm.by + r;
    const bool key_valid = r < prm.by && kpos < prm.S_kv;
    // query positions that see this key: [qlo, qhi]
    int qlo = -0x40000000, qhi = 0x3fffffff;
    const int shift = prm.S_kv - prm.S_q;
    if (prm.mask_mode == 2) qlo = kpos;
    else if (prm.mask_mode == 3) qlo = kpos - shift;
    else if (prm.mask_mode == 4) { qlo = kpos - shift - prm.win_right; qhi = kpos - shift + prm.win_left; }
    if (!key_valid) { qlo = 1; qhi = 0; }
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int exchanges = 0;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int st = i & 1;
      int qrow, tile, qpos0;
      entry_rows(i, qrow, tile, qpos0);
      ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_q[st], (i >> 1) & 1, prm.status) &&
                                       mbar_wait(&s.bar_s_full, i & 1, prm.status));
      if (!ok) break;
      tc_fence_after();
      const bool full = qpos0 + c0 >= qlo && qpos0 + c0 + kT / 2 - 1 <= qhi;
      const float* l2 = s.lse2[st] + c0;
      float p[kT / 2];
#pragma unroll
      for (int c = 0; c < kT / 2; c += 32) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + kColS + c0 + c, rr);
        tmem_ld_wait(rr);
#pragma unroll
        for (int k2 = 0; k2 < 32; ++k2) p[c + k2] = ex2(__uint_as_float(rr[k2]) * prm.scale_log2 - l2[c + k2]);
      }
      if (!full) {
#pragma unroll
        for (int c = 0; c < kT / 2; ++c) {
          const int qp = qpos0 + c0 + c;
          if (qp < qlo || qp > qhi) p[c] = 0.f;
        }
      }
      // both halves have read S^T before either overwrites it:
      // P^T hi -> S^T[c0/2, +32), P^T lo -> S^T[64 + c0/2, +32): A operands of dV += P^T dO
      ok = __all_sync(0xffffffffu, pair_sync(&s.bar_pair[quarter], exchanges, prm.status));
      if (!ok) break;
#pragma unroll
      for (int c = 0; c < kT / 2; c += 32) {
        uint32_t hv[16], lv[16];
#pragma unroll
        for (int k2 = 0; k2 < 16; ++k2) split_pack(p[c + 2 * k2], p[c + 2 * k2 + 1], hv[k2], lv[k2]);
        tmem_st16(tmem + lane_base + kColS + (c0 + c) / 2, hv);
        tmem_st16(tmem + lane_base + kColS + 64 + (c0 + c) / 2, lv);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&s.bar_p_ready);
      ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_dp_full, i & 1, prm.status));
      if (!ok) break;
      tc_fence_after();
      const float* dvv = s.dvec[st] + c0;
      // dS^T = P^T o (dP^T - D); hi -> dP^T[c0/2, +32), lo -> dP^T[64 + c0/2, +32)
      uint32_t hv[32], lv[32];
#pragma unroll
      for (int c = 0; c < kT / 2; c += 32) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + kColDP + c0 + c, rr);
        tmem_ld_wait(rr);
#pragma unroll
        for (int k2 = 0; k2 < 16; ++k2) {
          const int cc = c + 2 * k2;
          split_pack(p[cc] * (__uint_as_float(rr[2 * k2]) - dvv[cc]),
                     p[cc + 1] * (__uint_as_float(rr[2 * k2 + 1]) - dvv[cc + 1]), hv[cc / 2], lv[cc / 2]);
        }
      }
      ok = __all_sync(0xffffffffu, pair_sync(&s.bar_pair[quarter], exchanges, prm.status));
      if (!ok) break;
      tmem_st16(tmem + lane_base + kColDP + c0 / 2, hv);
      tmem_st16(tmem + lane_base + kColDP + c0 / 2 + 16, hv + 16);
      tmem_st16(tmem + lane_base + kColDP + 64 + c0 / 2, lv);
      tmem_st16(tmem + lane_base + kColDP + 64 + c0 / 2 + 16, lv + 16);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&s.bar_ds_ready);
    }
    // ---- epilogue: dK = scale * acc, dV = acc (this thread: head-dim columns [c0, c0 + 64))
    bool have = ok && n > 0;
    if (have) {
      have = __all_sync(0xffffffffu, mbar_wait(&s.bar_done, 0, prm.status));
      tc_fence_after();
    }
    __nv_bfloat16* dkrow = prm.dk + static_cast<size_t>(kv_row0 + r) * kD + c0;
    __nv_bfloat16* dvrow = prm.dv + static_cast<size_t>(kv_row0 + r) * kD + c0;
#pragma unroll
    for (int c = 0; c < kD / 2; c += 32) {
      uint32_t rk[32], rv[32];
      if (have) {
        tmem_ld32(tmem + lane_base + kColDK + c0 + c, rk);
        tmem_ld32(tmem + lane_base + kColDV + c0 + c, rv);
        tmem_ld_wait(rk);
#pragma unroll
        for (int i = 0; i < 32; ++i) reg_fence(rv[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) rk[i] = rv[i] = 0u;
      }
      if (key_valid) {
        store_row_bf16(dkrow + c, rk, prm.scale);
        store_row_bf16(dvrow + c, rv, 1.f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------------------------------------
// Q-major pass: dQ
// TMEM columns: S0 [0,BN) | S1 [BN,2BN) | dP [2BN,3BN) | dQ [3BN, 3BN+128).
// dS for tile j is written back as bf16 hi -> S_j[0,BN/2) and lo -> S_j[BN/2,BN), the A operands
// of dQ += dS K.
// ------------------------------------------------------------------------------------------------
constexpr int kQKStages = 3, kQVStages = 2;  // K is held by S and dQ, V only by dP

template <int BN>
struct __align__(1024) QSmem {
  uint8_t q[2][kT * 128];
  uint8_t dout[2][kT * 128];
  uint8_t k[kQKStages][2][BN * 128];  // [stage][sub-tile] [BN keys][64 d]
  uint8_t v[kQVStages][2][BN * 128];
  uint64_t bar_qdo, bar_k[kQKStages], bar_k_empty[kQKStages], bar_v[kQVStages], bar_v_empty[kQVStages];
  uint64_t bar_s_full[2], bar_dp_full, bar_ds_ready, bar_done;
  uint64_t bar_pair[4];
  uint32_t tmem_base;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    bsa_bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BwdParams prm) {
  constexpr uint32_t kColS0 = 0, kColS1 = BN, kColDP = 2 * BN, kColDQ = 3 * BN;
  extern __shared__ uint8_t smem_raw[];
  QSmem<BN>& s = *reinterpret_cast<QSmem<BN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / prm.nqb;
  const int qb = prm.nqb - 1 - static_cast<int>(blockIdx.x % prm.nqb);
  const int b = bh / prm.N1, h = bh % prm.N1;
  const int g = h / (prm.N1 / prm.N2);
  const int unit = bh * prm.nqb + qb;
  const int rp = prm.row_ptr[unit];
  const int n = prm.row_ptr[unit + 1] - rp;
  const int q_row0 = bh * prm.S_q + qb * prm.bx;
  const int kv_row0 = (b * prm.N2 + g) * prm.S_kv;

  if (tid == 0) {
    mbar_init(&s.bar_qdo, 1);
    for (int i = 0; i < kQKStages; ++i) {
      mbar_init(&s.bar_k[i], 1);
      mbar_init(&s.bar_k_empty[i], 1);
    }
    for (int i = 0; i < kQVStages; ++i) {
      mbar_init(&s.bar_v[i], 1);
      mbar_init(&s.bar_v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&s.bar_s_full[i], 1);
    mbar_init(&s.bar_dp_full, 1);
    mbar_init(&s.bar_ds_ready, kVecWarps * 32);
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
    if (lane == 0 && n > 0) {
      mbar_arrive_expect_tx(&s.bar_qdo, 4 * kT * 128);
      tma_load_2d(s.q[0], &tm_q, &s.bar_qdo, 0, q_row0);
      tma_load_2d(s.q[1], &tm_q, &s.bar_qdo, 64, q_row0);
      tma_load_2d(s.dout[0], &tm_do, &s.bar_qdo, 0, q_row0);
      tma_load_2d(s.dout[1], &tm_do, &s.bar_qdo, 64, q_row0);
      int issued_k = 0, issued_v = 0;
      bool ok = true;
      auto load_v = [&](int jv) -> bool {
        const int sv = jv % kQVStages, uv = jv / kQVStages;
        if (jv >= kQVStages && !mbar_wait(&s.bar_v_empty[sv], (uv - 1) & 1, prm.status)) return false;
        const int vrow = kv_row0 + prm.col[rp + jv] * prm.by;
        mbar_arrive_expect_tx(&s.bar_v[sv], 2 * BN * 128);
        tma_load_2d(s.v[sv][0], &tm_v, &s.bar_v[sv], 0, vrow);
        tma_load_2d(s.v[sv][1], &tm_v, &s.bar_v[sv], 64, vrow);
        issued_v = jv + 1;
        return true;
      };
      for (int j = 0; ok && j < n; ++j) {
        const int sk = j % kQKStages, uk = j / kQKStages;
        if (j >= kQKStages && !(ok = mbar_wait(&s.bar_k_empty[sk], (uk - 1) & 1, prm.status))) break;
        const int row = kv_row0 + prm.col[rp + j] * prm.by;
        mbar_arrive_expect_tx(&s.bar_k[sk], 2 * BN * 128);
        tma_load_2d(s.k[sk][0], &tm_k, &s.bar_k[sk], 0, row);
        tma_load_2d(s.k[sk][1], &tm_k, &s.bar_k[sk], 64, row);
        issued_k = j + 1;
        const int jv = j - (kQKStages - kQVStages);  // V trails K by one tile
        if (jv >= 0) ok = load_v(jv);
      }
      for (int jv = issued_v; ok && jv < n; ++jv) ok = load_v(jv);
      for (int j = (issued_k > kQKStages ? issued_k - kQKStages : 0); j < issued_k; ++j)
        mbar_wait(&s.bar_k[j % kQKStages], (j / kQKStages) & 1, prm.status);
      for (int j = (issued_v > kQVStages ? issued_v - kQVStages : 0); j < issued_v; ++j)
        mbar_wait(&s.bar_v[j % kQVStages], (j / kQVStages) & 1, prm.status);
      mbar_wait(&s.bar_qdo, 0, prm.status);
    }
  } else if (warp == kVecWarps + 1) {
    if (lane == 0 && n > 0) {
      const uint32_t id_s = idesc_bf16_f32(kT, BN, false, false);
      const uint32_t id_dq = idesc_bf16_f32(kT, kD, false, true);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1, sk = j % kQKStages;
        if (!mbar_wait(&s.bar_k[sk], (j / kQKStages) & 1, prm.status)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t ad = sdesc_sw128(smem_u32(s.q[ks >> 2]) + (ks & 3) * 32, 0, 1024);
          const uint64_t bd = sdesc_sw128(smem_u32(s.k[sk][ks >> 2]) + (ks & 3) * 32, 0, 1024);
          mma_bf16_ss(tmem + (st ? kColS1 : kColS0), ad, bd, id_s, ks > 0 ? 1u : 0u);
        }
        tc_commit(&s.bar_s_full[st]);
        return true;
      };
      auto issue_dp = [&](int j) -> bool {
        const int sv = j % kQVStages;
        if (!mbar_wait(&s.bar_v[sv], (j / kQVStages) & 1, prm.status)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t ad = sdesc_sw128(smem_u32(s.dout[ks >> 2]) + (ks & 3) * 32, 0, 1024);
          const uint64_t bd = sdesc_sw128(smem_u32(s.v[sv][ks >> 2]) + (ks & 3) * 32, 0, 1024);
          mma_bf16_ss(tmem + kColDP, ad, bd, id_s, ks > 0 ? 1u : 0u);
        }
        tc_commit(&s.bar_dp_full);
        tc_commit(&s.bar_v_empty[sv]);
        return true;
      };
      bool ok = mbar_wait(&s.bar_qdo, 0, prm.status);
      if (ok) ok = issue_s(0);
      if (ok) ok = issue_dp(0);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j & 1;
        if (j + 1 < n && !(ok = issue_s(j + 1))) break;
        if (!(ok = mbar_wait(&s.bar_ds_ready, j & 1, prm.status))) break;
        tc_fence_after();
        const uint32_t s_col = st ? kColS1 : kColS0;
        const int sk = j % kQKStages;
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            const uint64_t bd = sdesc_sw128(smem_u32(s.k[sk][0]) + ks * 2048, BN * 128, 1024);
            mma_bf16_ts(tmem + kColDQ, tmem + s_col + half * (BN / 2) + ks * 8, bd, id_dq,
                        (j > 0 || half > 0 || ks > 0) ? 1u : 0u);
          }
        tc_commit(&s.bar_k_empty[sk]);
        if (j + 1 < n && !(ok = issue_dp(j + 1))) break;
      }
      if (ok) tc_commit(&s.bar_done);
    }
  } else {
    constexpr int kHalf = BN / 2;
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // query row == TMEM lane
    const int c0 = hf * kHalf;          // this thread's key columns [c0, c0 + BN/2)
    const int qpos = qb * prm.bx + r;
    const bool row_valid = r < prm.bx && qpos < prm.S_q;
    int lo = 0, hi = prm.S_kv - 1;
    const int qq = qpos + prm.S_kv - prm.S_q;
    if (prm.mask_mode == 2) hi = min(hi, qpos);
    else if (prm.mask_mode == 3) hi = min(hi, qq);
    else if (prm.mask_mode == 4) { lo = qq - prm.win_left; hi = min(hi, qq + prm.win_right); }
    if (!row_valid) { lo = 1; hi = 0; }
    const size_t trow = static_cast<size_t>(unit) * kT + r;
    const float l2 = prm.lse2[trow];
    const float dval = prm.dvec[trow];
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int exchanges = 0;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int st = j & 1;
      const uint32_t s_col = st ? kColS1 : kColS0;
      ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_s_full[st], (j >> 1) & 1, prm.status));
      if (!ok) break;
      tc_fence_after();
      const int kpos0 = prm.col[rp + j] * prm.by + c0;
      const bool full = kpos0 >= lo && kpos0 + kHalf - 1 <= hi;
      float p[kHalf];
#pragma unroll
      for (int c = 0; c < kHalf; c += 32) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + s_col + c0 + c, rr);
        tmem_ld_wait(rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) p[c + i] = ex2(__uint_as_float(rr[i]) * prm.scale_log2 - l2);
      }
      if (!full) {
#pragma unroll
        for (int c = 0; c < kHalf; ++c) {
          const int kp = kpos0 + c;
          if (kp < lo || kp > hi) p[c] = 0.f;
        }
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_dp_full, j & 1, prm.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t hv[kHalf / 2], lv[kHalf / 2];
#pragma unroll
      for (int c = 0; c < kHalf; c += 32) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + kColDP + c0 + c, rr);
        tmem_ld_wait(rr);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          split_pack(p[c + 2 * i] * (__uint_as_float(rr[2 * i]) - dval),
                     p[c + 2 * i + 1] * (__uint_as_float(rr[2 * i + 1]) - dval), hv[c / 2 + i], lv[c / 2 + i]);
      }
      // both halves have read S_j before either writes dS over it:
      // hi -> S_j[c0/2, +BN/4), lo -> S_j[BN/2 + c0/2, +BN/4)
      ok = __all_sync(0xffffffffu, pair_sync(&s.bar_pair[quarter], exchanges, prm.status));
      if (!ok) break;
#pragma unroll
      for (int c = 0; c < kHalf / 2; c += 16) {
        tmem_st16(tmem + lane_base + s_col + c0 / 2 + c, hv + c);
        tmem_st16(tmem + lane_base + s_col + BN / 2 + c0 / 2 + c, lv + c);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&s.bar_ds_ready);
    }
    bool have = ok && n > 0;
    if (have) {
      have = __all_sync(0xffffffffu, mbar_wait(&s.bar_done, 0, prm.status));
      tc_fence_after();
    }
    const int d0 = hf * (kD / 2);  // this thread's head-dim columns of dQ
    __nv_bfloat16* dqrow = prm.dq + static_cast<size_t>(q_row0 + r) * kD + d0;
#pragma unroll
    for (int c = 0; c < kD / 2; c += 32) {
      uint32_t rr[32];
      if (have) {
        tmem_ld32(tmem + lane_base + kColDQ + d0 + c, rr);
        tmem_ld_wait(rr);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) rr[i] = 0u;
      }
      if (row_valid) store_row_bf16(dqrow + c, rr, prm.scale);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int BN>
cudaError_t launch_q(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, int grid, cudaStream_t st) {
  const size_t smem = sizeof(QSmem<BN>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(bsa_bwd_q_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  prof_begin("bsa_bwd_q", st);
  bsa_bwd_q_kernel<BN><<<grid, kThreads, smem, st>>>(tq, tk, tv, tdo, p);
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t bsa_bwd_launch(const BsaBwdArgs& a, const void* q, const void* k, const void* v, const void* out,
                           const void* dout, const float* lse, cudaStream_t st) {
  const long long n_rows = static_cast<long long>(a.B) * a.N1 * a.nqb * kT;
  {
    const long long threads = n_rows * 8;
    const int blk = 256;
    prof_begin("bsa_bwd_prep", st);
    bwd_prep_kernel<<<static_cast<unsigned>((threads + blk - 1) / blk), blk, 0, st>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse, a.S_q, a.bx, a.nqb,
        n_rows, a.dvec, a.lse2);
    prof_end(st);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tq, tk, tv, tdo, tk128, tv128;
  const uint64_t q_rows = static_cast<uint64_t>(a.B) * a.N1 * a.S_q;
  const uint64_t kv_rows = static_cast<uint64_t>(a.B) * a.N2 * a.S_kv;
  if (!make_tmap_2d_bf16(&tq, q, q_rows, kD, kD, kT) || !make_tmap_2d_bf16(&tdo, dout, q_rows, kD, kD, kT) ||
      !make_tmap_2d_bf16(&tk, k, kv_rows, kD, kD, a.by) || !make_tmap_2d_bf16(&tv, v, kv_rows, kD, kD, a.by) ||
      !make_tmap_2d_bf16(&tk128, k, kv_rows, kD, kD, kT) || !make_tmap_2d_bf16(&tv128, v, kv_rows, kD, kD, kT))
    return cudaErrorInvalidValue;
  BwdParams p;
  p.B = a.B; p.N1 = a.N1; p.N2 = a.N2; p.S_q = a.S_q; p.S_kv = a.S_kv; p.bx = a.bx; p.by = a.by;
  p.nqb = a.nqb; p.nkb = a.nkb; p.mask_mode = a.mask_mode; p.win_left = a.win_left; p.win_right = a.win_right;
  p.scale = a.scale; p.scale_log2 = a.scale * kLog2e;
  p.dvec = a.dvec; p.lse2 = a.lse2;
  p.dq = static_cast<__nv_bfloat16*>(a.dq);
  p.dk = static_cast<__nv_bfloat16*>(a.dk);
  p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.status = a.status;
  // KV-major pass
  {
    BwdParams pk = p;
    pk.row_ptr = a.t_row_ptr;
    pk.col = a.t_col;
    const size_t smem = sizeof(KvSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(bsa_bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = a.B * a.N2 * a.nkb;
    prof_begin("bsa_bwd_kv", st);
    bsa_bwd_kv_kernel<<<grid, kThreads, smem, st>>>(tq, tk128, tv128, tdo, pk);
    prof_end(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // Q-major pass
  p.row_ptr = a.row_ptr;
  p.col = a.col;
  const int grid = a.B * a.N1 * a.nqb;
  if (a.by == 128) return launch_q<128>(p, tq, tk, tv, tdo, grid, st);
  return launch_q<64>(p, tq, tk, tv, tdo, grid, st);
}

}  // namespace sa
