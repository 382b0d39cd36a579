// NSA selected attention on tcgen05: the token-major passes (NsaSelectedAttention page, forward
// formula: selected_key/value = Gather(key/value, topk_indices[i]); Out = Softmax(Mask(scale q
// K_sel^T)) V_sel; the dQ pass applies the BlockSparseAttentionGrad formulas dP = dOut V^T,
// dS = P o (dP - softmax_grad), dQ = dS K scale to the gathered blocks).
//
// An item is (token t, kv head g, head tile): the NH <= 32 query heads of the tile against the
// token's gathered keys.  A token's keys are its own selection, so no two items share a key set
// and the query side is only NH rows: the products are taken transposed, with 128 gathered keys as
// the MMA's M and the heads as N (the form the paged decode uses):
//   forward  S^T [128 keys][NH] = K~ . Q^T          O^T [128 dv][NH] += V~^T . P^T
//   dQ pass  S^T = K~ . Q^T, dP^T = V~ . dO^T        dQ^T [d][NH] += K~^T . dS^T (bf16 hi + lo)
// P^T (dS^T) is written to shared memory as the B operand, K-major ([NH heads][128 keys]).
// q / k have DQK = 128 or 192 dims (v, Out, dO 128): with 192 a K tile is three 64-dim chunks and
// dQ^T takes two M = 128 accumulators, over dims 0-127 and 64-191 (the second's rows 64-127 are
// dims 128-191).
//
// Gather: the visible chunks (16 keys, or 64 when the block size is a multiple of 64) of the
// token's listed blocks (a block's chunks past the last visible key, the query under the causal
// mask or the batch end, are skipped; a block listed twice is gathered twice) are laid out in
// order by the list warp into a per-item list in shared memory; a 128-key tile is loaded by TMA
// ({64 dims, 1 head, chunk tokens} boxes, 128-byte swizzle) into K and V rings.  A tile's unused
// chunk slots repeat its first chunk and are masked.
//
// Warps: 0-15 softmax (TMEM lane quarter = 32 keys, or 32 rows of the accumulator in the epilogue,
// and a quarter of the tile's heads), 16 builds the item lists (up to two items ahead) and loads Q
// (dO), 17 and 18 load the K and V tiles (each on its own ring, so K runs ahead of the V slots the
// later products still hold), 19 issues S^T (and dP^T), 20 issues O^T (dQ^T).  Persistent CTAs
// take items round-robin.  Every wait is bounded; on a timeout the kernel sets SA_DEV_TIMEOUT and
// stops.
#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

constexpr int kTok = 128;     // keys per tile: MMA M
constexpr int kDV = 128;      // head dim of v, Out and dOut (q and k: DQK, 128 or 192)
// Keys per gather chunk (one TMA box per head-dim half): 64 when the selected block size is a
// multiple of 64 (a block's visible prefix then ends inside its last chunk and is masked there),
// else 16.  A 128-key tile holds kTok / chunk chunks.
constexpr int kMaxChunks = 512;  // count * size <= 8192 keys per (token, kv head)
constexpr int kSoftWarps = 16;
constexpr int kHeadGroups = kSoftWarps / 4;
// warps: 0-15 softmax (lane quarter = warp % 4, head group = warp / 4), 16 item lists + Q loads,
// 17 K producer, 18 V producer, 19 S^T issuer, 20 O^T issuer
constexpr int kWList = kSoftWarps, kWK = kSoftWarps + 1, kWV = kSoftWarps + 2, kWS = kSoftWarps + 3,
              kWO = kSoftWarps + 4;
constexpr int kThreads = (kSoftWarps + 5) * 32;
constexpr int kTileBytes = kTok * 128;  // [128 keys][64 dims] bf16, one head-dim half
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLazy = 8.f;  // log2 units a tile may exceed the running maximum without a rescale

// Ring depths: an operand held until the last product of its tile (V in the forward, K in the dQ
// pass) gets the deeper ring, the one released by the first product the shallower.
// A 32-head tile's Q, dO and P buffers take one stage of the deeper ring (227 KB per CTA); with
// 192-dim q / k (16-head tiles only) a K stage is 48 KB and the rings are two or three deep.
template <bool kDq, int NH, int DQK>
struct TcCfg {
  static constexpr int kQC = DQK / 64;  // 64-wide chunks of q / k
  static constexpr int kDeep = !kDq ? (NH == 16 ? 4 : 3) : (NH == 16 ? 3 : 2);
  static constexpr int kKR = DQK == 128 ? (kDq ? kDeep : 2) : 2;  // K ring (S^T, and dQ^T in the dQ pass)
  static constexpr int kVR = DQK == 128 ? (kDq ? 2 : kDeep) : (kDq ? 2 : 3);  // V ring (O^T, or dP^T)
};

struct ItemDesc {
  int32_t t, g, h0, rows, pos, len, t0, n_vis;
  float lse2[32];  // dQ pass: LSE * log2(e) per head (+inf: no key); forward: unused
  float dvec[32];  // dQ pass: softmax_grad per head
  int32_t kp0[kMaxChunks];  // first key (within the batch) of each visible chunk
};

template <bool kDq, int NH, int DQK>
struct __align__(1024) TcSmem {
  using Cfg = TcCfg<kDq, NH, DQK>;
  // operand buffers start on 1024-byte boundaries (the 128-byte swizzle's pattern)
  alignas(1024) uint8_t k[Cfg::kKR][Cfg::kQC][kTileBytes];
  alignas(1024) uint8_t v[Cfg::kVR][2][kTileBytes];
  alignas(1024) uint8_t q[2][Cfg::kQC][NH * 128];   // [item slot][64-dim chunk][NH rows][64 dims]
  // P^T (dS^T hi, lo) per tile parity: [tile & 1][part][key half][NH rows][64 keys]
  alignas(1024) uint8_t p[2][kDq ? 2 : 1][2][NH * 128];
  alignas(1024) uint8_t dout[kDq ? 2 : 1][2][kDq ? NH * 128 : 16];  // dQ pass only
  ItemDesc desc[2];
  float red[2][4][NH];                       // per tile parity: column maxima of each lane quarter
  float red_l[4][NH];
  uint64_t bar_desc_full[2], bar_desc_empty[2];
  uint64_t bar_q[2], bar_q_empty[2];
  uint64_t bar_k[Cfg::kKR], bar_k_empty[Cfg::kKR];
  uint64_t bar_v[Cfg::kVR], bar_v_empty[Cfg::kVR];
  uint64_t bar_s_full[2], bar_s_free[2];     // score buffers (S^T, and dP^T in the dQ pass)
  uint64_t bar_p_full[2], bar_pv_done[2];    // the P^T (dS^T) buffers: written / consumed, per tile parity
  uint64_t bar_x;                            // softmax warps exchange tile maxima, then sums
  uint64_t bar_acc_free;                     // the epilogue has read the accumulator
  uint32_t tmem_base;
};

struct TcParams {
  int B, T, N1, N2, G, K, sel_block, mask_mode, head_tiles;
  int chunk, chunk_shift;  // keys per gather chunk (16 or 64) and its log2
  long long items;
  float scale, scale_log2;
  const int32_t* cu;
  const int32_t* ok_flag;
  const int32_t* ids;  // [T][N2][K] valid ids ascending, -1 padded
  const int32_t* cnt;  // [T][N2]
  const float* lse2;   // [T][N1] LSE * log2(e), +inf for rows without keys (dQ pass)
  const float* dvec;   // [T][N1] softmax_grad (dQ pass)
  __nv_bfloat16* out;  // forward Out, or dQ
  float* lse_out;
  uint32_t* status;
};

__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ int batch_of(const int32_t* __restrict__ cu, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// NH consecutive 32-bit TMEM columns of this thread's lane (NH = 16 or 32)
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
template <int N>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 4) tmem_ld4(taddr, r);
  else if constexpr (N == 8) tmem_ld8(taddr, r);
  else tmem_ld16(taddr, r);
}
template <int N>
__device__ __forceinline__ void tmem_st_row(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 4) tmem_st4(taddr, r);
  else if constexpr (N == 8) tmem_st8(taddr, r);
  else tmem_st16(taddr, r);
}

// byte offset of (row, 16-byte chunk) in a [rows][128 B] tile written with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <bool kDq, int NH, int DQK>
__global__ void __launch_bounds__(kThreads, 1)
    nsa_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const TcParams prm) {
  using Cfg = TcCfg<kDq, NH, DQK>;
  constexpr int kKR = Cfg::kKR, kVR = Cfg::kVR, kQC = Cfg::kQC;
  // 192-dim dQ: a second accumulator over dims 64..191 (its rows 64..127 are dims 128..191)
  constexpr bool kTwoAcc = kDq && DQK == 192;
  // TMEM columns: score buffers at [0, NH) and [NH, 2NH); dP^T buffers after them (dQ pass); the
  // O^T / dQ^T accumulator(s) last
  constexpr uint32_t kColS = 0, kColDP = 2 * NH, kColAcc = kDq ? 4 * NH : 2 * NH;
  constexpr uint32_t kTmemCols = kDq ? ((kTwoAcc ? 6 : 5) * NH <= 128 ? 128 : 256) : 128;
  griddep_launch_dependents();
  griddep_wait();  // launched early: the metadata (and the preprocess) must be complete
  extern __shared__ uint8_t smem_raw[];
  TcSmem<kDq, NH, DQK>& s =
      *reinterpret_cast<TcSmem<kDq, NH, DQK>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool run = *prm.ok_flag != 0;  // cu_seqlens valid (uniform)
  // this CTA's items: blockIdx.x, blockIdx.x + gridDim.x, ...
  const long long n_my = run && blockIdx.x < prm.items ? (prm.items - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.bar_desc_full[i], 1);
      mbar_init(&s.bar_desc_empty[i], kSoftWarps * 32 + 4);  // softmax threads, K, V, S, O warps' lane 0
      mbar_init(&s.bar_q[i], 1);
      mbar_init(&s.bar_q_empty[i], 1);
      mbar_init(&s.bar_s_full[i], 1);
      mbar_init(&s.bar_s_free[i], kSoftWarps * 32);
      mbar_init(&s.bar_p_full[i], kSoftWarps * 32);
      mbar_init(&s.bar_pv_done[i], 1);
    }
    for (int i = 0; i < kKR; ++i) {
      mbar_init(&s.bar_k[i], 1);
      mbar_init(&s.bar_k_empty[i], 1);
    }
    for (int i = 0; i < kVR; ++i) {
      mbar_init(&s.bar_v[i], 1);
      mbar_init(&s.bar_v_empty[i], 1);
    }
    mbar_init(&s.bar_x, kSoftWarps * 32);
    mbar_init(&s.bar_acc_free, kSoftWarps * 32);
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

  // consumers: the descriptor of this CTA's item number k (slot k & 1)
  auto desc_wait = [&](long long k) -> bool {
    return mbar_wait(&s.bar_desc_full[k & 1], (k >> 1) & 1, prm.status);
  };

  if (warp == kWList) {
    // ------------------------------------------------------------------ item lists + Q (dO) loads
    bool ok = true;
    for (long long k = 0; ok && k < n_my; ++k) {
      const int slot = static_cast<int>(k & 1);
      // exact parity: the slot's next phase needs this item's arrivals
      if (k >= 2 && !(ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_desc_empty[slot], ((k >> 1) - 1) & 1,
                                                              prm.status))))
        break;
      const long long item = blockIdx.x + k * gridDim.x;
      // items (g, t, head tile), kv-head major: the CTAs sweep one kv head's tokens at a time, so
      // that head's K / V (the blocks the neighbouring tokens gather) stay in L2
      const int ht = static_cast<int>(item % prm.head_tiles);
      const int t = static_cast<int>((item / prm.head_tiles) % prm.T);
      const int g = static_cast<int>(item / (static_cast<long long>(prm.head_tiles) * prm.T));
      const int b = batch_of(prm.cu, prm.B, t);
      const int t0 = prm.cu[b], len = prm.cu[b + 1] - t0, pos = t - t0;
      const int last_key = prm.mask_mode == 2 ? pos : len - 1;
      const int n_sel = prm.cnt[static_cast<size_t>(t) * prm.N2 + g];
      const int32_t* sel = prm.ids + (static_cast<size_t>(t) * prm.N2 + g) * prm.K;
      const int cpb = prm.sel_block >> prm.chunk_shift;
      ItemDesc& d = s.desc[slot];
      // visible chunks of each listed block (a prefix of its chunks), laid out in list order
      int base = 0;
      for (int i0 = 0; i0 < n_sel; i0 += 32) {
        const int i = i0 + lane;
        const int j = i < n_sel ? sel[i] : -1;
        const int first = j * prm.sel_block;
        const int nc = (j >= 0 && first <= last_key) ? min(cpb, ((last_key - first) >> prm.chunk_shift) + 1) : 0;
        int incl = nc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int at = base + incl - nc;
        for (int c = 0; c < nc; ++c) d.kp0[at + c] = first + (c << prm.chunk_shift);
        base += __shfl_sync(0xffffffffu, incl, 31);
      }
      const int h0 = g * prm.G + ht * NH;
      const int rows = min(NH, prm.G - ht * NH);
      if (kDq && lane < NH) {
        const bool live = lane < rows;
        const size_t o = static_cast<size_t>(t) * prm.N1 + h0 + lane;
        d.lse2[lane] = live ? prm.lse2[o] : INFINITY;
        d.dvec[lane] = live ? prm.dvec[o] : 0.f;
      }
      if (lane == 0) {
        d.t = t; d.g = g; d.h0 = h0; d.rows = rows; d.pos = pos; d.len = len; d.t0 = t0; d.n_vis = base;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.bar_desc_full[slot]);  // release: the list and header above
      // Q (and dO) of the item's heads; the slot was last read by item k - 2's score products
      if (lane == 0) {
        if (k >= 2) ok = mbar_wait(&s.bar_q_empty[slot], ((k >> 1) - 1) & 1, prm.status);
        if (ok) {
          mbar_arrive_expect_tx(&s.bar_q[slot], (kQC + (kDq ? 2 : 0)) * NH * 128);
          const int qrow = t * prm.N1 + h0;
#pragma unroll
          for (int c = 0; c < kQC; ++c) tma_load_2d(s.q[slot][c], &tm_q, &s.bar_q[slot], c * 64, qrow);
          if (kDq) {
            tma_load_2d(s.dout[kDq ? slot : 0][0], &tm_do, &s.bar_q[slot], 0, qrow);
            tma_load_2d(s.dout[kDq ? slot : 0][1], &tm_do, &s.bar_q[slot], 64, qrow);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    // do not leave the CTA with copies in flight
    if (lane == 0)
      for (long long k = (n_my > 2 ? n_my - 2 : 0); k < n_my; ++k)
        mbar_wait(&s.bar_q[k & 1], (k >> 1) & 1, prm.status);
  } else if (warp == kWK || warp == kWV) {
    // ------------------------------------------------------------------ K / V producers
    // lane c < 8 loads chunk c of each tile (a tile's unused chunk slots repeat its chunk 0)
    const bool is_k = warp == kWK;
    const CUtensorMap* map = is_k ? &tm_k : &tm_v;
    constexpr int kRK = Cfg::kKR, kRV = Cfg::kVR;
    const int R = is_k ? kRK : kRV;
    uint64_t* full = is_k ? s.bar_k : s.bar_v;
    uint64_t* empty = is_k ? s.bar_k_empty : s.bar_v_empty;
    bool ok = true;
    long long use = 0;  // tiles loaded into this ring (this CTA)
    for (long long k = 0; ok && k < n_my; ++k) {
      const int slot = static_cast<int>(k & 1);
      if (!(ok = __all_sync(0xffffffffu, desc_wait(k)))) break;
      const ItemDesc& d = s.desc[slot];
      const int n_vis = d.n_vis, t0 = d.t0, g = d.g;
      const int cpt = kTok >> prm.chunk_shift;  // chunks per tile
      const int n_tiles = (n_vis + cpt - 1) / cpt;
      for (int j = 0; ok && j < n_tiles; ++j, ++use) {
        const int c = j * cpt + (lane & 7);
        const int tok = t0 + (lane < cpt ? d.kp0[c < n_vis ? c : j * cpt] : 0);
        const int st = static_cast<int>(use % R);
        if (lane == 0 && use >= R) ok = mbar_wait(&empty[st], ((use / R) - 1) & 1, prm.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* dst = is_k ? s.k[st % kRK][0] : s.v[st % kRV][0];
        const int nc = is_k ? kQC : 2;  // 64-wide chunks of a key row
        if (lane == 0) mbar_arrive_expect_tx(&full[st], nc * kTileBytes);
        __syncwarp();
        if (lane < cpt)
          for (int c = 0; c < nc; ++c)
            tma_load_3d(dst + c * kTileBytes + lane * prm.chunk * 128, map, &full[st], c * 64, g, tok);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.bar_desc_empty[slot]);  // this warp is done with the item's list
    }
    // do not leave the CTA with copies in flight
    if (lane == 0)
      for (long long u = (use > R ? use - R : 0); u < use; ++u) mbar_wait(&full[u % R], (u / R) & 1, prm.status);
  } else if (warp == kWS) {
    // ------------------------------------------------------------------ S^T (and dP^T) issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(kTok, NH, false, false);
      const uint64_t dk0 = sdesc_sw128(smem_u32(s.k[0][0]), 0, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(s.v[0][0]), 0, 1024);
      const uint64_t dq0 = sdesc_sw128(smem_u32(s.q[0][0]), 0, 1024);
      const uint64_t ddo0 = sdesc_sw128(smem_u32(s.dout[0][0]), 0, 1024);
      bool ok = true;
      long long J = 0;  // tiles issued (this CTA): S buffer J & 1, K stage J % kKR, V stage J % kVR
      for (long long k = 0; ok && k < n_my; ++k) {
        const int slot = static_cast<int>(k & 1);
        if (!(ok = desc_wait(k))) break;
        const int n_vis = s.desc[slot].n_vis;
        mbar_arrive(&s.bar_desc_empty[slot]);
        const int n_tiles = (n_vis + (kTok >> prm.chunk_shift) - 1) / (kTok >> prm.chunk_shift);
        // every item's Q slot is loaded (and released below), with or without tiles
        if (!(ok = mbar_wait(&s.bar_q[slot], (k >> 1) & 1, prm.status))) break;
        const uint64_t dq = dq0 + static_cast<uint64_t>(slot) * ((kQC * NH * 128) >> 4);
        const uint64_t ddo = ddo0 + static_cast<uint64_t>(kDq ? slot : 0) * ((2 * NH * 128) >> 4);
        for (int j = 0; ok && j < n_tiles; ++j, ++J) {
          const int st = static_cast<int>(J & 1);
          // S buffer st last held tile J-2; exact parity: s_free's next phase needs this tile
          if (J >= 2 && !(ok = mbar_wait(&s.bar_s_free[st], ((J >> 1) - 1) & 1, prm.status))) break;
          const int ks_ = static_cast<int>(J % kKR);
          if (!(ok = mbar_wait(&s.bar_k[ks_], (J / kKR) & 1, prm.status))) break;
          tc_fence_after();
          const uint64_t dk = dk0 + static_cast<uint64_t>(ks_) * ((kQC * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < DQK / 16; ++kk)
            mma_bf16_ss(tmem + kColS + st * NH, sdesc_add(dk, (kk >> 2) * kTileBytes + (kk & 3) * 32),
                        sdesc_add(dq, (kk >> 2) * (NH * 128) + (kk & 3) * 32), id_s, kk > 0 ? 1u : 0u);
          if (!kDq) tc_commit(&s.bar_k_empty[ks_]);  // forward: K is read by S^T only
          if (kDq) {
            const int vs = static_cast<int>(J % kVR);
            if (!(ok = mbar_wait(&s.bar_v[vs], (J / kVR) & 1, prm.status))) break;
            tc_fence_after();
            const uint64_t dv = dv0 + static_cast<uint64_t>(vs) * ((2 * kTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kDV / 16; ++kk)
              mma_bf16_ss(tmem + kColDP + st * NH, sdesc_add(dv, (kk >> 2) * kTileBytes + (kk & 3) * 32),
                          sdesc_add(ddo, (kk >> 2) * (NH * 128) + (kk & 3) * 32), id_s, kk > 0 ? 1u : 0u);
            tc_commit(&s.bar_v_empty[vs]);  // dQ pass: V is read by dP^T only
          }
          tc_commit(&s.bar_s_full[st]);
        }
        if (ok) tc_commit(&s.bar_q_empty[slot]);  // after the item's last read of Q / dO
      }
    }
  } else if (warp == kWO) {
    // ------------------------------------------------------------------ O^T (dQ^T) issuer
    if (lane == 0) {
      const uint32_t id_o = idesc_bf16_f32(kTok, NH, true, false);  // A = V^T / K^T MN-major, B K-major
      // A: the two 64-wide dv (d) halves of a stage are kTileBytes apart; K step = 16 keys = 2048 B
      const uint64_t da0 = sdesc_sw128(smem_u32(kDq ? s.k[0][0] : s.v[0][0]), kTileBytes, 1024);
      const uint64_t dp0 = sdesc_sw128(smem_u32(s.p[0][0][0]), 0, 1024);
      constexpr uint32_t kPBuf16 = ((kDq ? 2 : 1) * 2 * NH * 128) >> 4;  // one tile's P buffer, 16-byte units
      constexpr int kAR = kDq ? kKR : kVR;
      bool ok = true;
      long long J = 0, tiled = 0;
      for (long long k = 0; ok && k < n_my; ++k) {
        const int slot = static_cast<int>(k & 1);
        if (!(ok = desc_wait(k))) break;
        const int n_vis = s.desc[slot].n_vis;
        mbar_arrive(&s.bar_desc_empty[slot]);
        const int n_tiles = (n_vis + (kTok >> prm.chunk_shift) - 1) / (kTok >> prm.chunk_shift);
        if (n_tiles == 0) continue;
        // the accumulator is overwritten by this item's first product: the epilogue of the last item
        // with tiles has read it (exact parity: acc_free's next phase needs this item's products)
        if (tiled > 0 && !(ok = mbar_wait(&s.bar_acc_free, (tiled - 1) & 1, prm.status))) break;
        ++tiled;
        for (int j = 0; ok && j < n_tiles; ++j, ++J) {
          const int st = static_cast<int>(J & 1);
          // exact parity: p_full[st]'s next phase needs tile J + 2, written after this product
          if (!(ok = mbar_wait(&s.bar_p_full[st], (J >> 1) & 1, prm.status))) break;
          const int as = static_cast<int>(J % kAR);
          if (!kDq && !(ok = mbar_wait(&s.bar_v[as], (J / kAR) & 1, prm.status))) break;
          tc_fence_after();
          const uint64_t da = da0 + static_cast<uint64_t>(as) * (((kDq ? kQC : 2) * kTileBytes) >> 4);
#pragma unroll
          for (int acc_i = 0; acc_i < (kTwoAcc ? 2 : 1); ++acc_i) {  // 192-dim dQ: dims 0..127, 64..191
            const uint64_t da_i = da + static_cast<uint64_t>(acc_i) * (kTileBytes >> 4);
#pragma unroll
            for (int part = 0; part < (kDq ? 2 : 1); ++part) {  // dQ pass: dS^T hi, then lo
              const uint64_t dp = dp0 + static_cast<uint64_t>(st) * kPBuf16 + static_cast<uint64_t>(part) * ((2 * NH * 128) >> 4);
#pragma unroll
              for (int kk = 0; kk < kTok / 16; ++kk)
                mma_bf16_ss(tmem + kColAcc + acc_i * NH, sdesc_add(da_i, kk * 2048),
                            sdesc_add(dp, (kk >> 2) * (NH * 128) + (kk & 3) * 32), id_o,
                            (j > 0 || part > 0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(kDq ? &s.bar_k_empty[as] : &s.bar_v_empty[as]);
          tc_commit(&s.bar_pv_done[st]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    // warp = (head group hg, lane quarter): its 32 keys of a tile (TMEM lanes) and HW = NH / 4 of
    // the heads (TMEM columns), so each tile's chain is split over four warps per sub-partition
    constexpr int HW = NH / kHeadGroups;
    const int quarter = warp & 3, hg = warp >> 2;
    const int hb = hg * HW;             // this warp's first head of the tile
    const int r = quarter * 32 + lane;  // key row of a tile == TMEM lane (and accumulator row)
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;
    long long J = 0;
    int xph = 0;  // phases of bar_x completed
    for (long long k = 0; ok && k < n_my; ++k) {
      const int slot = static_cast<int>(k & 1);
      if (!(ok = __all_sync(0xffffffffu, desc_wait(k)))) break;
      const ItemDesc& d = s.desc[slot];
      const int n_vis = d.n_vis, pos = d.pos, len = d.len, rows = d.rows, h0 = d.h0, t = d.t;
      const int cpt = kTok >> prm.chunk_shift;  // chunks per tile
      const int n_tiles = (n_vis + cpt - 1) / cpt;
      float m[HW], l[HW];
#pragma unroll
      for (int h = 0; h < HW; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
      }
      for (int j = 0; j < n_tiles; ++j, ++J) {
        const int st = static_cast<int>(J & 1);
        const int c = j * cpt + (r >> prm.chunk_shift);
        const int kpos = c < n_vis ? d.kp0[c] + (r & (prm.chunk - 1)) : 0x7fffffff;
        const bool vis = kpos < len && (prm.mask_mode != 2 || kpos <= pos);
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_s_full[st], (J >> 1) & 1, prm.status));
        if (!ok) break;
        tc_fence_after();
        float x[HW];
        uint32_t dpr[HW];
        {
          uint32_t rr[HW];
          tmem_ld_row<HW>(tmem + lane_base + kColS + st * NH + hb, rr);
          if constexpr (kDq) tmem_ld_row<HW>(tmem + lane_base + kColDP + st * NH + hb, dpr);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < HW; ++h) {
            reg_fence(rr[h]);
            if (kDq) reg_fence(dpr[h]);
            x[h] = vis ? __uint_as_float(rr[h]) * prm.scale_log2 : -INFINITY;
          }
        }
        tc_fence_before();
        mbar_arrive(&s.bar_s_free[st]);
        if (!kDq) {
          // column maxima of the tile: over the warp's 32 keys, then over the four lane quarters
#pragma unroll
          for (int h = 0; h < HW; ++h) {
            const float mx = warp_max(x[h]);
            if (lane == 0) s.red[st][quarter][hb + h] = mx;
          }
          mbar_arrive(&s.bar_x);
          ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_x, xph & 1, prm.status));
          ++xph;
          if (!ok) break;
        }
        // this tile's P buffer is free once the product of tile J-2 has completed (exact parity:
        // the buffer's next product needs this tile's P)
        if (J >= 2) {
          ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_pv_done[st], ((J >> 1) - 1) & 1, prm.status));
          if (!ok) break;
        }
        bool any = false;
        float alpha[HW];
        if (!kDq) {
#pragma unroll
          for (int h = 0; h < HW; ++h) {
            const float tm = fmaxf(fmaxf(s.red[st][0][hb + h], s.red[st][1][hb + h]),
                                   fmaxf(s.red[st][2][hb + h], s.red[st][3][hb + h]));
            alpha[h] = 1.f;
            if (tm > m[h] + kLazy) {  // uniform over the warps of this head group
              alpha[h] = ex2(m[h] - tm);
              l[h] *= alpha[h];
              m[h] = tm;
              any = true;
            }
          }
        }
        // P^T (forward) or dS^T hi / lo (dQ pass) of this key row, K-major [NH rows][keys]
        const int khalf = r >> 6, kcol = r & 63;
        uint8_t* pb = s.p[st][0][khalf];
#pragma unroll
        for (int h = 0; h < HW; ++h) {
          const uint32_t off = sw128(hb + h, kcol >> 3) + (kcol & 7) * 2;
          if (!kDq) {
            const float mu = m[h] == -INFINITY ? 0.f : m[h];
            const float e = ex2(x[h] - mu);
            l[h] += e;
            *reinterpret_cast<__nv_bfloat16*>(pb + off) = __float2bfloat16_rn(e);
          } else {
            const float p = vis ? ex2(x[h] - d.lse2[hb + h]) : 0.f;  // per-head values from shared memory
            const float ds = p * (__uint_as_float(dpr[h]) - d.dvec[hb + h]);
            const __nv_bfloat16 hi = __float2bfloat16_rn(ds);
            const __nv_bfloat16 lo = __float2bfloat16_rn(ds - __bfloat162float(hi));
            *reinterpret_cast<__nv_bfloat16*>(pb + off) = hi;
            *reinterpret_cast<__nv_bfloat16*>(s.p[st][kDq ? 1 : 0][khalf] + off) = lo;
          }
        }
        if (!kDq && __any_sync(0xffffffffu, any) && j > 0) {
          // rescale this head group's O^T columns (accumulator row r) once the product of tile J-1
          // has completed (exact parity: that buffer's next product needs P of tile J+1)
          ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_pv_done[st ^ 1], ((J - 1) >> 1) & 1, prm.status));
          if (!ok) break;
          tc_fence_after();
          uint32_t rr[HW];
          tmem_ld_row<HW>(tmem + lane_base + kColAcc + hb, rr);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < HW; ++h) {
            reg_fence(rr[h]);
            rr[h] = __float_as_uint(__uint_as_float(rr[h]) * alpha[h]);
          }
          tmem_st_row<HW>(tmem + lane_base + kColAcc + hb, rr);
          tmem_st_wait();
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&s.bar_p_full[st]);
      }
      if (!ok) break;
      // ---- epilogue of the item: accumulator row r = dv (d) index, columns = heads
      float L[HW];
      if (!kDq) {
        // l over the 128 keys of each head: warp sums, then the four quarters
#pragma unroll
        for (int h = 0; h < HW; ++h) {
          float v = l[h];
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) s.red_l[quarter][hb + h] = v;
        }
        mbar_arrive(&s.bar_x);
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_x, xph & 1, prm.status));
        ++xph;
        if (!ok) break;
#pragma unroll
        for (int h = 0; h < HW; ++h)
          L[h] = (s.red_l[0][hb + h] + s.red_l[1][hb + h]) + (s.red_l[2][hb + h] + s.red_l[3][hb + h]);
      }
      uint32_t acc[HW], acc2[HW];
      const bool hi_rows = kTwoAcc && quarter >= 2;  // this warp's rows 64..127 also hold dims 128..191
      if (n_tiles > 0) {
        const long long jl = J - 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_pv_done[jl & 1], (jl >> 1) & 1, prm.status));
        if (!ok) break;
        tc_fence_after();
        tmem_ld_row<HW>(tmem + lane_base + kColAcc + hb, acc);
        if (hi_rows) tmem_ld_row<HW>(tmem + lane_base + kColAcc + NH + hb, acc2);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < HW; ++h) {
          reg_fence(acc[h]);
          if (hi_rows) reg_fence(acc2[h]);
        }
        tc_fence_before();
        mbar_arrive(&s.bar_acc_free);
      } else {
#pragma unroll
        for (int h = 0; h < HW; ++h) acc[h] = acc2[h] = 0u;
      }
      // the descriptor slot is no longer needed
      mbar_arrive(&s.bar_desc_empty[slot]);
      constexpr int kDO = kDq ? DQK : kDV;  // row length of the output (dQ or Out)
      __nv_bfloat16* base = prm.out + static_cast<size_t>(t) * prm.N1 * kDO;
#pragma unroll
      for (int h = 0; h < HW; ++h) {
        if (hb + h >= rows) break;
        float mul;
        if (kDq) mul = prm.scale;
        else mul = L[h] > 0.f ? 1.f / L[h] : 0.f;
        base[static_cast<size_t>(h0 + hb + h) * kDO + r] = __float2bfloat16_rn(__uint_as_float(acc[h]) * mul);
        if (hi_rows)
          base[static_cast<size_t>(h0 + hb + h) * kDO + 64 + r] = __float2bfloat16_rn(__uint_as_float(acc2[h]) * mul);
      }
      if (!kDq && quarter == 0 && lane < HW && hb + lane < rows) {
        float mh = m[0], lh = L[0];
#pragma unroll
        for (int h = 1; h < HW; ++h)
          if (lane == h) {
            mh = m[h];
            lh = L[h];
          }
        prm.lse_out[static_cast<size_t>(t) * prm.N1 + h0 + hb + lane] = lh > 0.f ? (mh * kLn2 + logf(lh)) : -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

template <bool kDq, int NH, int DQK>
cudaError_t launch_tc(const NsaArgs& a, const TcParams& p, const char* name, cudaStream_t st) {
  CUtensorMap tq, tdo, tk, tv;
  const uint64_t qrows = static_cast<uint64_t>(a.T) * a.N1;
  if (!make_tmap_2d_bf16(&tq, a.q, qrows, DQK, DQK, NH) ||
      (kDq && !make_tmap_2d_bf16(&tdo, a.dout, qrows, kDV, kDV, NH)) || (!kDq && !make_tmap_2d_bf16(&tdo, a.q, qrows, DQK, DQK, NH)) ||
      !make_tmap_3d_bf16(&tk, a.k, DQK, a.N2, a.T, DQK, static_cast<uint64_t>(a.N2) * DQK, 1, p.chunk) ||
      !make_tmap_3d_bf16(&tv, a.v, kDV, a.N2, a.T, kDV, static_cast<uint64_t>(a.N2) * kDV, 1, p.chunk))
    return cudaErrorInvalidValue;
  static_assert(sizeof(TcSmem<kDq, NH, DQK>) + 1024 <= 227 * 1024, "shared memory of one CTA (227 KB on sm_100)");
  const size_t smem = sizeof(TcSmem<kDq, NH, DQK>) + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(nsa_tc_kernel<kDq, NH, DQK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = static_cast<int>(p.items < sms ? p.items : sms);
  if (grid == 0) return cudaSuccess;
  prof_begin(name, st);
  e = launch_pdl(nsa_tc_kernel<kDq, NH, DQK>, dim3(grid), dim3(kThreads), smem, st, tq, tdo, tk, tv, p);
  prof_end(st);
  return e != cudaSuccess ? e : cudaGetLastError();
}

TcParams tc_params(const NsaArgs& a, int NH) {
  TcParams p;
  p.B = a.B; p.T = a.T; p.N1 = a.N1; p.N2 = a.N2; p.G = a.N1 / a.N2; p.K = a.K; p.sel_block = a.sel_block;
  p.mask_mode = a.mask_mode; p.head_tiles = (p.G + NH - 1) / NH;
  p.chunk = a.sel_block % 64 == 0 ? 64 : 16;
  p.chunk_shift = p.chunk == 64 ? 6 : 4;
  p.items = static_cast<long long>(a.T) * a.N2 * p.head_tiles;
  p.scale = a.scale; p.scale_log2 = a.scale * kLog2e;
  p.cu = a.cu_seqlens; p.ok_flag = a.ok_flag; p.ids = a.ids; p.cnt = a.cnt;
  p.lse2 = a.lse2; p.dvec = a.dvec; p.status = a.status;
  return p;
}

}  // namespace

cudaError_t nsa_fwd_tc_launch(const NsaArgs& a, cudaStream_t st) {
  const int G = a.N1 / a.N2;
  TcParams p = tc_params(a, G <= 16 ? 16 : 32);
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse_out = a.lse_out;
  if (a.D == 192) return G <= 16 ? launch_tc<false, 16, 192>(a, p, "nsa_fwd", st) : cudaErrorNotSupported;
  if (G <= 16) return launch_tc<false, 16, 128>(a, p, "nsa_fwd", st);
  return launch_tc<false, 32, 128>(a, p, "nsa_fwd", st);
}

cudaError_t nsa_dq_tc_launch(const NsaArgs& a, cudaStream_t st) {
  const int G = a.N1 / a.N2;
  TcParams p = tc_params(a, G <= 16 ? 16 : 32);
  p.out = static_cast<__nv_bfloat16*>(a.dq);
  p.lse_out = nullptr;
  if (a.D == 192) return G <= 16 ? launch_tc<true, 16, 192>(a, p, "nsa_bwd_dq", st) : cudaErrorNotSupported;
  if (G <= 16) return launch_tc<true, 16, 128>(a, p, "nsa_bwd_dq", st);
  return launch_tc<true, 32, 128>(a, p, "nsa_bwd_dq", st);
}

}  // namespace sa
