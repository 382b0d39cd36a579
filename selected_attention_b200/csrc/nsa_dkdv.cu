// NSA dK / dV on tcgen05 (NsaSelectedAttention page: selected_key/value = Gather(key/value,
// topk_indices[i]); the gradients follow the BlockSparseAttentionGrad backward formulas on the
// gathered keys, scattered back to the source rows).
//
// One CTA per kv block (b, g, kb) of 64 keys walks the ascending list of tokens that selected
// the block (nsa_meta.cu), 128 / G tokens per step, so that a step is a 128-row tile of
// (token, head) rows: in TND the G query heads of a kv-head group are contiguous rows.
//   S  = Q K^T,  dP = dO V^T            M = 128 rows, N = 64 keys, K = 128 head dims
//   P  = exp2(S scale log2e - LSE log2e) * multiplicity, masked;  dS = P o (dP - D)
//   dV^T += dO^T P,  dK^T += Q^T dS      M = 128 head dims, N = 64 keys, K = 128 rows
// P and dS reach the tensor cores from shared memory as bf16 hi + lo (MN-major B operands);
// dO^T and Q^T are the staged tiles read as MN-major A operands.  TMEM holds S, dP and the two
// accumulators; the list order is fixed, so results are run-to-run identical without atomics.
//
// Warps 0-7 compute P and dS (TMEM lane quarter = warp % 4, key half = warp / 4), warp 8 issues
// the TMA loads, warp 9 issues the MMAs.  Every wait is bounded (SA_DEV_TIMEOUT).
// With 192-dim q / k (v and dO keep 128) the Q rows of a step are three 64-dim chunks, Q / dO have
// one stage instead of two (227 KB), and dK^T takes two M = 128 accumulators over dims 0-127 and
// 64-191, the second's rows 64-127 giving dims 128-191.
#include <cuda.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

constexpr int kRows = 128;  // (token, head) rows of a step
constexpr int kKeys = 64;   // keys of a block
constexpr int kDV = 128;    // head dim of v / dO (q / k: DQK)
constexpr int kEw = 8;      // element-wise warps
constexpr int kThreads = (kEw + 2) * 32;
constexpr uint32_t kColS = 0, kColDP = 64, kColDV = 128, kColDK = 192, kColDK2 = 256;  // TMEM columns
constexpr float kLog2e = 1.4426950408889634f;

template <int DQK>
struct __align__(1024) DkdvSmem {
  static constexpr int kQC = DQK / 64;             // 64-dim chunks of q / k
  static constexpr int kNst = DQK == 128 ? 2 : 1;  // Q / dO stages
  uint8_t k[kQC][kKeys * 128];        // K block: [64 keys][64 d] per head-dim chunk
  uint8_t v[2][kKeys * 128];
  uint8_t q[kNst][kQC][kRows * 128];  // [stage][chunk] [128 rows][64 d]
  uint8_t dout[kNst][2][kRows * 128];
  uint8_t p[2][kRows * 128];          // P hi, lo: [128 rows][64 keys]
  uint8_t ds[2][kRows * 128];         // dS hi, lo
  uint64_t bar_kv, bar_qdo[kNst], bar_qdo_empty[kNst];
  uint64_t bar_s_full, bar_p_ready, bar_p_free, bar_done;
  uint32_t tmem_base;
};

struct DkdvParams {
  int B, N1, N2, G, K, nblk_max, mask_mode, tok_per_step;
  float scale, scale_log2;
  const int32_t *cu, *ok_flag, *ids, *cnt, *dup, *t_row_ptr, *t_col;
  const float *lse2, *dvec;  // [T][N1]: LSE * log2(e) (+inf without keys), rowsum(dO o Out)
  __nv_bfloat16 *dk, *dv;
  uint32_t* status;
};

// 8 floats -> bf16 hi (round to nearest) and lo = x - hi, packed in pairs
__device__ __forceinline__ void split2x4(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    h[i] = pack_bf16(x[2 * i], x[2 * i + 1]);
    l[i] = pack_bf16(x[2 * i] - bf16lo(h[i]), x[2 * i + 1] - bf16hi(h[i]));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// byte offset of (row, 16-byte chunk) in a [rows][128 B] tile written with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int DQK>
__global__ void __launch_bounds__(kThreads, 1)
    nsa_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const DkdvParams prm) {
  using Sm = DkdvSmem<DQK>;
  constexpr int kQC = Sm::kQC, kNst = Sm::kNst;
  constexpr bool kTwoAcc = DQK == 192;
  constexpr uint32_t kTmemCols = kTwoAcc ? 512 : 256;
  extern __shared__ uint8_t smem_raw[];
  Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // CTA order: batches from the last one (longest lists first in causal workloads), kv head,
  // then blocks ascending; CTAs that run together share the batch's Q / dO rows in L2
  const int kb = static_cast<int>(blockIdx.x % prm.nblk_max);
  const int bg = static_cast<int>(blockIdx.x / prm.nblk_max);
  const int b = prm.B - 1 - bg / prm.N2, g = bg % prm.N2;
  if (!*prm.ok_flag) return;
  const int t0 = prm.cu[b], len = prm.cu[b + 1] - t0;
  const int nkeys = min(kKeys, len - kb * kKeys);
  if (nkeys <= 0) return;
  const int row = (b * prm.N2 + g) * prm.nblk_max + kb;
  const int rp = prm.t_row_ptr[row];
  const int n_tok = prm.t_row_ptr[row + 1] - rp;
  if (n_tok == 0) return;  // no token selected the block: its dK / dV rows stay zero
  const int tps = prm.tok_per_step;
  const int steps = (n_tok + tps - 1) / tps;
  const int key_tok0 = t0 + kb * kKeys;  // token index of the block's first key

  if (tid == 0) {
    mbar_init(&s.bar_kv, 1);
    for (int i = 0; i < kNst; ++i) {
      mbar_init(&s.bar_qdo[i], 1);
      mbar_init(&s.bar_qdo_empty[i], 1);
    }
    mbar_init(&s.bar_s_full, 1);
    mbar_init(&s.bar_p_ready, kEw * 32);
    mbar_init(&s.bar_p_free, 1);
    mbar_init(&s.bar_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == kEw) {
    // ------------------------------------------------------------------ TMA producer
    // Lane j < tps loads the token of slot j and issues that slot's four row copies, so the token
    // reads of a step are one round trip, not tps dependent ones.
    if (lane == 0) {
      mbar_arrive_expect_tx(&s.bar_kv, (kQC + 2) * kKeys * 128);
      for (int c = 0; c < kQC; ++c) tma_load_3d(s.k[c], &tm_k, &s.bar_kv, c * 64, g, key_tok0);
      tma_load_3d(s.v[0], &tm_v, &s.bar_kv, 0, g, key_tok0);
      tma_load_3d(s.v[1], &tm_v, &s.bar_kv, 64, g, key_tok0);
    }
    int issued = 0;
    for (int i = 0; i < steps; ++i) {
      const int st = i % kNst;
      // slots past the list repeat its last token (finite data; their rows are masked)
      const int qrow = lane < tps ? prm.t_col[rp + min(i * tps + lane, n_tok - 1)] * prm.N1 + g * prm.G : 0;
      bool ok = true;
      if (lane == 0) {
        if (i >= kNst) ok = mbar_wait(&s.bar_qdo_empty[st], ((i - kNst) / kNst) & 1, prm.status);
        if (ok) mbar_arrive_expect_tx(&s.bar_qdo[st], (kQC + 2) * kRows * 128);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;  // the expected bytes are set before any copy
      if (lane < tps) {
        const uint32_t off = static_cast<uint32_t>(lane * prm.G * 128);
        for (int c = 0; c < kQC; ++c) tma_load_2d(s.q[st][c] + off, &tm_q, &s.bar_qdo[st], c * 64, qrow);
        tma_load_2d(s.dout[st][0] + off, &tm_do, &s.bar_qdo[st], 0, qrow);
        tma_load_2d(s.dout[st][1] + off, &tm_do, &s.bar_qdo[st], 64, qrow);
      }
      issued = i + 1;
    }
    // wait for this CTA's own copies still in flight before it may exit
    if (lane == 0) {
      for (int i = (issued > kNst ? issued - kNst : 0); i < issued; ++i)
        mbar_wait(&s.bar_qdo[i % kNst], (i / kNst) & 1, prm.status);
      mbar_wait(&s.bar_kv, 0, prm.status);
    }
  } else if (warp == kEw + 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(kRows, kKeys, false, false);  // S, dP
      const uint32_t id_g = idesc_bf16_f32(128, kKeys, true, true);      // dV^T, dK^T (M = 128 dims)
      // descriptors of stage 0 / sub-tile 0; stages, sub-tiles and K steps are added offsets
      const uint64_t dq0 = sdesc_sw128(smem_u32(s.q[0][0]), 0, 1024);
      const uint64_t ddo0 = sdesc_sw128(smem_u32(s.dout[0][0]), 0, 1024);
      const uint64_t dk = sdesc_sw128(smem_u32(s.k[0]), 0, 1024);
      const uint64_t dv = sdesc_sw128(smem_u32(s.v[0]), 0, 1024);
      const uint64_t dqm0 = sdesc_sw128(smem_u32(s.q[0][0]), kRows * 128, 1024);    // MN-major A
      const uint64_t ddom0 = sdesc_sw128(smem_u32(s.dout[0][0]), kRows * 128, 1024);
      const uint64_t dph = sdesc_sw128(smem_u32(s.p[0]), kRows * 128, 1024), dpl = sdesc_add(dph, kRows * 128);
      const uint64_t dsh = sdesc_sw128(smem_u32(s.ds[0]), kRows * 128, 1024), dsl = sdesc_add(dsh, kRows * 128);
      constexpr uint32_t kStageQ16 = (kQC * kRows * 128) >> 4;  // one Q stage, in 16-byte units
      constexpr uint32_t kStageD16 = (2 * kRows * 128) >> 4;    // one dO stage
      // [128 rows] x [64 keys] += A [128 rows][KD] . B [64 keys][KD]^T, both K-major (KD = DQK for S,
      // 128 for dP)
      auto mma_s = [&](uint32_t d, uint64_t a, uint64_t b, auto kd) {
        constexpr int KD = decltype(kd)::value;
#pragma unroll
        for (int ks = 0; ks < KD / 16; ++ks)
          mma_bf16_ss(d, sdesc_add(a, (ks >> 2) * (kRows * 128) + (ks & 3) * 32),
                      sdesc_add(b, (ks >> 2) * (kKeys * 128) + (ks & 3) * 32), id_s, ks > 0 ? 1u : 0u);
      };
      // [128 d] x [64 keys] += A^T . B with A the [128 rows][128 d] tile (MN-major, two 64-d
      // chunks 16 KB apart) and B the [128 rows][64 keys] tile (MN-major, one chunk)
      auto mma_g = [&](uint32_t d, uint64_t a, uint64_t b, bool acc) {
#pragma unroll
        for (int ks = 0; ks < kRows / 16; ++ks)
          mma_bf16_ss(d, sdesc_add(a, ks * 2048), sdesc_add(b, ks * 2048), id_g, (acc || ks > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(&s.bar_kv, 0, prm.status) && mbar_wait(&s.bar_qdo[0], 0, prm.status);
      if (ok) {
        tc_fence_after();
        mma_s(tmem + kColS, dq0, dk, std::integral_constant<int, DQK>{});
        mma_s(tmem + kColDP, ddo0, dv, std::integral_constant<int, kDV>{});
        tc_commit(&s.bar_s_full);
      }
      for (int i = 0; ok && i < steps; ++i) {
        const int st = i % kNst;
        if (!(ok = mbar_wait(&s.bar_p_ready, i & 1, prm.status))) break;
        tc_fence_after();
        const uint64_t ddom = ddom0 + static_cast<uint64_t>(st) * kStageD16;
        const uint64_t dqm = dqm0 + static_cast<uint64_t>(st) * kStageQ16;
        mma_g(tmem + kColDV, ddom, dph, i > 0);   // dV^T += dO^T P_hi
        mma_g(tmem + kColDV, ddom, dpl, true);    // dV^T += dO^T P_lo
        mma_g(tmem + kColDK, dqm, dsh, i > 0);    // dK^T += Q^T dS_hi  (dims 0..127)
        mma_g(tmem + kColDK, dqm, dsl, true);     // dK^T += Q^T dS_lo
        if (kTwoAcc) {                             // dims 64..191: Q^T from chunks 1 and 2
          const uint64_t dqm1 = sdesc_add(dqm, kRows * 128);
          mma_g(tmem + kColDK2, dqm1, dsh, i > 0);
          mma_g(tmem + kColDK2, dqm1, dsl, true);
        }
        tc_commit(&s.bar_p_free);
        tc_commit(&s.bar_qdo_empty[st]);
        if (i + 1 < steps) {
          const int sn = (i + 1) % kNst;
          if (!(ok = mbar_wait(&s.bar_qdo[sn], ((i + 1) / kNst) & 1, prm.status))) break;
          tc_fence_after();
          mma_s(tmem + kColS, dq0 + static_cast<uint64_t>(sn) * kStageQ16, dk, std::integral_constant<int, DQK>{});
          mma_s(tmem + kColDP, ddo0 + static_cast<uint64_t>(sn) * kStageD16, dv, std::integral_constant<int, kDV>{});
          tc_commit(&s.bar_s_full);
        }
      }
      if (ok) tc_commit(&s.bar_done);
    }
  } else {
    // ------------------------------------------------------------------ P / dS warps
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;       // tile row == TMEM lane
    const int c0 = hf * 32;                  // this thread's keys [c0, c0 + 32)
    const int slot = r / prm.G;              // token slot of the row within a step
    const int h = g * prm.G + r % prm.G;     // query head of the row
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int kpos0 = kb * kKeys + c0;       // key position (in the batch) of column c0
    bool ok = true;
    for (int i = 0; i < steps; ++i) {
      const int idx = i * tps + slot;
      const bool row_ok = idx < n_tok;
      float l2 = INFINITY, dd = 0.f, mult = 0.f;
      int qpos = -1;
      if (row_ok) {
        const int tok = prm.t_col[rp + idx];
        qpos = tok - t0;
        l2 = prm.lse2[static_cast<size_t>(tok) * prm.N1 + h];
        dd = prm.dvec[static_cast<size_t>(tok) * prm.N1 + h];
        mult = 1.f;
        if (prm.dup[static_cast<size_t>(tok) * prm.N2 + g]) {  // an id listed twice counts twice
          const int32_t* sl = prm.ids + (static_cast<size_t>(tok) * prm.N2 + g) * prm.K;
          const int nsl = prm.cnt[static_cast<size_t>(tok) * prm.N2 + g];
          int m = 0;
          for (int x = 0; x < nsl; ++x) m += sl[x] == kb;
          mult = static_cast<float>(m);
        }
      }
      // keys visible to this row: position < len, and <= the query position under the mask
      int lim = len - 1 - kpos0;
      if (prm.mask_mode == 2) lim = min(lim, qpos - kpos0);
      if (!row_ok) lim = -1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_s_full, i & 1, prm.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[32], dr[32];
      tmem_ld32(tmem + lane_base + kColS + c0, sr);
      tmem_ld32(tmem + lane_base + kColDP + c0, dr);
      tmem_ld_wait(sr);
#pragma unroll
      for (int c = 0; c < 32; ++c) reg_fence(dr[c]);
      float p[32], ds[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        p[c] = c <= lim ? ex2(fmaf(__uint_as_float(sr[c]), prm.scale_log2, -l2)) * mult : 0.f;
        ds[c] = p[c] * (__uint_as_float(dr[c]) - dd);
      }
      // P / dS buffers are free once the previous step's dV / dK products have read them
      if (i > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_p_free, (i - 1) & 1, prm.status));
        if (!ok) break;
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint4 ph, pl, sh, sl;
        split2x4(p + cc * 8, ph, pl);
        split2x4(ds + cc * 8, sh, sl);
        const uint32_t off = sw128(r, hf * 4 + cc);
        *reinterpret_cast<uint4*>(s.p[0] + off) = ph;
        *reinterpret_cast<uint4*>(s.p[1] + off) = pl;
        *reinterpret_cast<uint4*>(s.ds[0] + off) = sh;
        *reinterpret_cast<uint4*>(s.ds[1] + off) = sl;
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&s.bar_p_ready);
    }
    // ---- epilogue: TMEM lane r = head dim r; columns = keys [c0, c0 + 32)
    bool have = ok;
    if (have) {
      have = __all_sync(0xffffffffu, mbar_wait(&s.bar_done, 0, prm.status));
      tc_fence_after();
    }
    if (have) {
      uint32_t rk[32], rv[32];
      tmem_ld32(tmem + lane_base + kColDK + c0, rk);
      tmem_ld32(tmem + lane_base + kColDV + c0, rv);
      tmem_ld_wait(rk);
#pragma unroll
      for (int i = 0; i < 32; ++i) reg_fence(rv[i]);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        if (c0 + c >= nkeys) break;
        const size_t krow = static_cast<size_t>(key_tok0 + c0 + c) * prm.N2 + g;
        prm.dk[krow * DQK + r] = __float2bfloat16_rn(__uint_as_float(rk[c]) * prm.scale);
        prm.dv[krow * kDV + r] = __float2bfloat16_rn(__uint_as_float(rv[c]));
      }
      if (kTwoAcc && quarter >= 2) {  // rows 64..127 of the second accumulator: dims 128..191
        tmem_ld32(tmem + lane_base + kColDK2 + c0, rk);
        tmem_ld_wait(rk);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c0 + c >= nkeys) break;
          const size_t krow = static_cast<size_t>(key_tok0 + c0 + c) * prm.N2 + g;
          prm.dk[krow * DQK + 64 + r] = __float2bfloat16_rn(__uint_as_float(rk[c]) * prm.scale);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

bool nsa_dkdv_tc_supported(const NsaArgs& a) {
  const int G = a.N1 / a.N2;
  return (a.D == 128 || a.D == 192) && a.sel_block == kKeys && G >= 8 && G <= 128 && 128 % G == 0;
}

cudaError_t nsa_dkdv_tc_launch(const NsaArgs& a, cudaStream_t st) {
  if (!nsa_dkdv_tc_supported(a)) return cudaErrorNotSupported;
  const int G = a.N1 / a.N2;
  const int rows = a.B * a.N2 * a.nblk_max;
  if (rows == 0 || a.T == 0) return cudaSuccess;
  CUtensorMap tq, tdo, tk, tv;
  const uint64_t qrows = static_cast<uint64_t>(a.T) * a.N1;
  const int D = a.D;
  if (!make_tmap_2d_bf16(&tq, a.q, qrows, D, D, G) || !make_tmap_2d_bf16(&tdo, a.dout, qrows, kDV, kDV, G) ||
      !make_tmap_3d_bf16(&tk, a.k, D, a.N2, a.T, D, static_cast<uint64_t>(a.N2) * D, 1, kKeys) ||
      !make_tmap_3d_bf16(&tv, a.v, kDV, a.N2, a.T, kDV, static_cast<uint64_t>(a.N2) * kDV, 1, kKeys))
    return cudaErrorInvalidValue;
  DkdvParams p;
  p.B = a.B; p.N1 = a.N1; p.N2 = a.N2; p.G = G; p.K = a.K; p.nblk_max = a.nblk_max; p.mask_mode = a.mask_mode;
  p.tok_per_step = kRows / G;
  p.scale = a.scale; p.scale_log2 = a.scale * kLog2e;
  p.cu = a.cu_seqlens; p.ok_flag = a.ok_flag; p.ids = a.ids; p.cnt = a.cnt; p.dup = a.dup;
  p.t_row_ptr = a.t_row_ptr; p.t_col = a.t_col;
  p.lse2 = a.lse2; p.dvec = a.dvec;
  p.dk = static_cast<__nv_bfloat16*>(a.dk); p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.status = a.status;
  static_assert(sizeof(DkdvSmem<192>) + 1024 <= 227 * 1024, "shared memory of one CTA (227 KB on sm_100)");
  static_assert(sizeof(DkdvSmem<128>) + 1024 <= 227 * 1024, "shared memory of one CTA (227 KB on sm_100)");
  const size_t smem = (D == 192 ? sizeof(DkdvSmem<192>) : sizeof(DkdvSmem<128>)) + 1024;
  auto kern = D == 192 ? nsa_dkdv_tc_kernel<192> : nsa_dkdv_tc_kernel<128>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  prof_begin("nsa_bwd_dkdv", st);
  kern<<<rows, kThreads, smem, st>>>(tq, tdo, tk, tv, p);
  prof_end(st);
  return cudaGetLastError();
}

}  // namespace sa
