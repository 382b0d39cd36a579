// Sparse flash attention decode over a paged KV cache (SparseFlashAttention page, formula):
//   Out = softmax((q k~^T + q_rope k_rope~^T) * scale) v~,  D = Dv = 512, Dr = 64, q_len = 1
// where k~ / v~ are the tokens of the selected sparse blocks (sfa_meta.cu turns them into page
// lists and a work list of pieces).
//
// The query side of a decode step is small (the G = N1/N2 heads of one kv head, one row each) and
// the key side long, so the products are taken transposed, with the tokens as the MMA's M = 128
// rows and the heads as N:
//   S^T [128 tokens][64 heads]  = K~ [128][576] . Q^T          (Q of 64 heads stays in shared memory)
//   O^T [512 dv][64 heads]     += V~^T [512][128] . P^T [128][64] (four M = 128 tiles of dv)
// One CTA per piece: a run of pages of one unit (batch, kv head, half of the G heads).  O^T takes
// 256 TMEM columns and the two S^T buffers 128, so every head of the CTA keeps all 512 dv columns
// and S is computed once per head.  K streams through a ring of [128 tokens][64 dims] slots and V
// through a ring of [2 x 64 dv][64 tokens] slots, each ring with its own producer and consumer.
// P^T has a single shared-memory buffer (written once O^T += V^T P^T of the previous tile has
// completed); the 16 KB that a second one would take hold a fourth V slot instead.
//
// The softmax runs across tokens, i.e. across TMEM lanes: each softmax thread owns one token of a
// tile and 32 heads.  Per tile the four warps of a head half reduce their maxima with redux.sync
// and exchange them through shared memory (an mbarrier with bounded waits, not a named barrier,
// so a timed-out warp cannot leave the others blocked); the running maximum of a head moves only
// when the tile exceeds it by more than 2^8, and then O^T's columns of that head are rescaled.
// Per-thread partial sums l are reduced over the tokens once, in the epilogue.
//
// Warps: 0-7 softmax (lane quarter = TMEM lanes, warp >> 2 = head half of 32), 8 K producer,
// 9 V producer, 10 issues S^T, 11 issues O^T += V^T P^T.  A piece covering a whole unit writes
// Out and LSE; otherwise it writes (O, m, l) partials that sfa_combine merges in piece order.
#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

constexpr int kTok = 128;     // tokens per tile: MMA M of S^T, K of O^T
constexpr int kHeads = 64;    // query heads per CTA: MMA N
constexpr int kDQ = 512;      // q / k / v head dim
constexpr int kDR = 64;       // rope dim
constexpr int kKChunks = 9;   // 8 x 64 dims of k + 1 of k_rope
constexpr int kVUses = 8;     // V slots per tile: 4 dv tiles of 128 x 2 token halves of 64
constexpr int kKR = 4;        // K ring depth
constexpr int kVR = 4;        // V ring depth
constexpr int kSmWarps = 8;
constexpr int kThreads = (kSmWarps + 4) * 32;
constexpr uint32_t kColO = 0, kColS = 256;  // O^T: 4 x 64 columns; S^T buffers at 256 and 320
constexpr uint32_t kSlot = kTok * 128;      // 16 KB
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLazy = 8.f;  // log2 units a tile may exceed the running maximum without a rescale

struct __align__(1024) DecSmem {
  uint8_t q[kKChunks][kHeads * 128];  // Q rows (heads) x 64 dims per chunk, 128-byte swizzle
  uint8_t k[kKR][kSlot];              // [128 tokens][64 dims]
  uint8_t v[kVR][kSlot];              // [2 dv chunks][64 tokens][64 dv]
  uint8_t p[kSlot];                   // P^T [128 tokens][64 heads] bf16 (one buffer)
  float red_m[2][2][4][32];           // [tile parity][head half][lane quarter][head]
  float red_l[2][4][32];              // [head half][lane quarter][head]
  uint64_t bar_q, bar_k[kKR], bar_k_empty[kKR], bar_v[kVR], bar_v_empty[kVR];
  uint64_t bar_s_full[2], bar_s_free[2], bar_p_full[2], bar_pv_done[2];
  uint64_t bar_x[2];  // per head half: maxima (one phase per tile), then the sums
  uint32_t tmem_base;
};

struct DecParams {
  int B, N1, N2, G, HH, page_size, cap, sub_rows;
  float scale_log2;
  const int32_t* pages;
  const int32_t* tokens;
  const int32_t* piece_unit;
  const int32_t* piece_begin;
  const int32_t* piece_len;
  const int32_t* unit_pieces;
  const int32_t* n_pieces;
  __nv_bfloat16* out;
  float* lse;
  float* part_o;  // [piece][64 heads][512]
  float* part_m;  // [piece][64]
  float* part_l;
  uint32_t* status;
};

__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// byte offset of (row, 16-byte chunk) in a [rows][128 B] tile written with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Sum v[0..31] over the 32 lanes of the warp; lane i returns the total of element i.  Each round
// halves the elements a lane keeps: it adds its partner's copy of the half it keeps (31 shuffles).
__device__ __forceinline__ float transpose_sum(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float keep = up ? v[i + w] : v[i];
      const float send = up ? v[i] : v[i + w];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
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
  const int bg = u / prm.HH, hh = u % prm.HH;
  const int b = bg / prm.N2, g = bg % prm.N2;
  const int pbeg = prm.piece_begin[piece];
  const int npages = prm.piece_len[piece];
  const int sub = prm.sub_rows;             // tokens per TMA box (32 or 64, divides the page)
  const int spp = prm.page_size / sub;      // boxes per page
  const int n_sub = kTok / sub;             // boxes per tile
  const int n_chunks = npages * spp;
  const int n_tiles = (n_chunks + n_sub - 1) / n_sub;
  const int32_t* plist = prm.pages + static_cast<size_t>(bg) * prm.cap + pbeg;
  const int32_t* tlist = prm.tokens + static_cast<size_t>(bg) * prm.cap + pbeg;
  const int head0 = hh * kHeads;                       // first head of this CTA within the group
  const int nh = min(kHeads, prm.G - head0);           // heads of the group this CTA owns
  const int qrow0 = b * prm.N1 + g * prm.G + head0;    // their first query row

  if (tid == 0) {
    mbar_init(&s.bar_q, 1);
    for (int i = 0; i < kKR; ++i) {
      mbar_init(&s.bar_k[i], 1);
      mbar_init(&s.bar_k_empty[i], 1);
    }
    for (int i = 0; i < kVR; ++i) {
      mbar_init(&s.bar_v[i], 1);
      mbar_init(&s.bar_v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.bar_s_full[i], 1);
      mbar_init(&s.bar_s_free[i], kSmWarps * 32);
      mbar_init(&s.bar_p_full[i], kSmWarps * 32);
      mbar_init(&s.bar_pv_done[i], 1);
      mbar_init(&s.bar_x[i], 4 * 32);
    }
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

  // Box t of tile j: its page-list entry and its token offset inside the page; a box past the
  // piece's end repeats the tile's first box (its rows are masked, and the copy stays in bounds).
  // The producers load the entry one tile ahead and use it one iteration later, so the load's
  // latency is not paid at the start of every tile.
  auto box_entry = [&](int j, int t) -> int {
    const int qb = j * n_sub + t;
    return qb < n_chunks ? qb : j * n_sub;
  };

  if (warp == kSmWarps) {
    // ------------------------------------------------------------------ K producer
    int issued = 0;
    bool ok = true;
    if (n_tiles > 0) {
      if (lane == 0) {
        mbar_arrive_expect_tx(&s.bar_q, kKChunks * kHeads * 128);
        for (int c = 0; c < 8; ++c) tma_load_2d(s.q[c], &tm_q, &s.bar_q, c * 64, qrow0);
        tma_load_2d(s.q[8], &tm_qr, &s.bar_q, 0, qrow0);
      }
      int nxt_page = 0, nxt_off = 0;  // page id (loaded, used next iteration) and token offset
      if (lane < n_sub) {
        const int qb = box_entry(0, lane);
        nxt_page = plist[qb / spp];
        nxt_off = (qb % spp) * sub;
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int tok = nxt_page * prm.page_size + nxt_off;
        if (j + 1 < n_tiles && lane < n_sub) {
          const int qb = box_entry(j + 1, lane);
          nxt_page = plist[qb / spp];
          nxt_off = (qb % spp) * sub;
        }
        for (int c = 0; c < kKChunks; ++c) {
          const int use = j * kKChunks + c, slot = use % kKR;
          if (lane == 0 && use >= kKR) ok = mbar_wait(&s.bar_k_empty[slot], ((use / kKR) - 1) & 1, prm.status);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (lane == 0) mbar_arrive_expect_tx(&s.bar_k[slot], kSlot);
          __syncwarp();
          if (lane < n_sub) {
            uint8_t* dst = s.k[slot] + lane * sub * 128;
            if (c < 8) tma_load_3d(dst, &tm_k, &s.bar_k[slot], c * 64, g, tok);
            else tma_load_3d(dst, &tm_kr, &s.bar_k[slot], 0, g, tok);
          }
          ++issued;
        }
      }
      // wait for this CTA's own copies still in flight before it may exit
      if (lane == 0) {
        for (int use = (issued > kKR ? issued - kKR : 0); use < issued; ++use)
          mbar_wait(&s.bar_k[use % kKR], (use / kKR) & 1, prm.status);
        mbar_wait(&s.bar_q, 0, prm.status);
      }
    }
  } else if (warp == kSmWarps + 1) {
    // ------------------------------------------------------------------ V producer
    int issued = 0;
    bool ok = true;
    if (n_tiles > 0) {
      const int half_boxes = n_sub / 2;  // boxes per token half
      int nxt_page = 0, nxt_off = 0;  // page id (loaded, used next iteration) and token offset
      if (lane < n_sub) {
        const int qb = box_entry(0, lane);
        nxt_page = plist[qb / spp];
        nxt_off = (qb % spp) * sub;
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int tok = nxt_page * prm.page_size + nxt_off;
        if (j + 1 < n_tiles && lane < n_sub) {
          const int qb = box_entry(j + 1, lane);
          nxt_page = plist[qb / spp];
          nxt_off = (qb % spp) * sub;
        }
        for (int x = 0; x < kVUses; ++x) {
          const int mt = x >> 1, th = x & 1;
          const int use = j * kVUses + x, slot = use % kVR;
          if (lane == 0 && use >= kVR) ok = mbar_wait(&s.bar_v_empty[slot], ((use / kVR) - 1) & 1, prm.status);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (lane == 0) mbar_arrive_expect_tx(&s.bar_v[slot], kSlot);
          __syncwarp();
          if (lane < n_sub && lane / half_boxes == th) {
            uint8_t* dst = s.v[slot] + (lane - th * half_boxes) * sub * 128;
            tma_load_3d(dst, &tm_v, &s.bar_v[slot], mt * 128, g, tok);
            tma_load_3d(dst + 64 * 128, &tm_v, &s.bar_v[slot], mt * 128 + 64, g, tok);
          }
          ++issued;
        }
      }
      if (lane == 0)
        for (int use = (issued > kVR ? issued - kVR : 0); use < issued; ++use)
          mbar_wait(&s.bar_v[use % kVR], (use / kVR) & 1, prm.status);
    }
  } else if (warp == kSmWarps + 2) {
    // ------------------------------------------------------------------ S^T issuer
    if (lane == 0 && n_tiles > 0) {
      const uint32_t id_s = idesc_bf16_f32(kTok, kHeads, false, false);
      const uint64_t dq = sdesc_sw128(smem_u32(s.q[0]), 0, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(s.k[0]), 0, 1024);
      bool ok = mbar_wait(&s.bar_q, 0, prm.status);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j & 1;
        // S buffer st last held S^T_{j-2}; exact parity: s_free's next phase needs S^T_j
        if (j >= 2 && !(ok = mbar_wait(&s.bar_s_free[st], ((j >> 1) - 1) & 1, prm.status))) break;
        const uint32_t d = tmem + kColS + st * kHeads;
        for (int c = 0; c < kKChunks; ++c) {
          const int use = j * kKChunks + c, slot = use % kKR;
          if (!(ok = mbar_wait(&s.bar_k[slot], (use / kKR) & 1, prm.status))) break;
          tc_fence_after();
          const uint64_t dk = sdesc_add(dk0, slot * kSlot);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_bf16_ss(d, sdesc_add(dk, ks * 32), sdesc_add(dq, c * (kHeads * 128) + ks * 32), id_s,
                        (c > 0 || ks > 0) ? 1u : 0u);
          tc_commit(&s.bar_k_empty[slot]);
        }
        if (ok) tc_commit(&s.bar_s_full[st]);
      }
    }
  } else if (warp == kSmWarps + 3) {
    // ------------------------------------------------------------------ O^T issuer
    if (lane == 0 && n_tiles > 0) {
      const uint32_t id_o = idesc_bf16_f32(kTok, kHeads, true, true);
      // A = V^T: MN-major, the two 64-dv chunks of a slot 8 KB apart; B = P^T: MN-major, one chunk
      const uint64_t dv0 = sdesc_sw128(smem_u32(s.v[0]), 64 * 128, 1024);
      const uint64_t dp0 = sdesc_sw128(smem_u32(s.p), kSlot, 1024);
      bool ok = true;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j & 1;
        // one barrier per tile parity: its next phase needs P_{j+2}, written after this product
        if (!(ok = mbar_wait(&s.bar_p_full[st], (j >> 1) & 1, prm.status))) break;
        for (int x = 0; x < kVUses; ++x) {
          const int mt = x >> 1, th = x & 1;
          const int use = j * kVUses + x, slot = use % kVR;
          if (!(ok = mbar_wait(&s.bar_v[slot], (use / kVR) & 1, prm.status))) break;
          tc_fence_after();
          const uint64_t dv = sdesc_add(dv0, slot * kSlot);
          const uint64_t dp = sdesc_add(dp0, th * (64 * 128));
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_bf16_ss(tmem + kColO + mt * kHeads, sdesc_add(dv, ks * 2048), sdesc_add(dp, ks * 2048), id_o,
                        (j > 0 || th > 0 || ks > 0) ? 1u : 0u);
          tc_commit(&s.bar_v_empty[slot]);
        }
        if (ok) tc_commit(&s.bar_pv_done[st]);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int quarter = warp & 3, hc = warp >> 2;
    const int r = quarter * 32 + lane;  // token row of the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int rt = r / sub, rin = r % sub;  // box of the row, row inside the box
    // the row holds a token in use when its box lies in the piece and rin + the box's offset in
    // the page is below the page's token count; the count is loaded one tile ahead (cnt) and
    // compared one iteration later, so the load's latency is not paid at the start of every tile
    int cnt = 0, cnt_off = 0;
    auto load_count = [&](int j) {
      const int qb = j * n_sub + rt;
      if (qb < n_chunks) {
        cnt = tlist[qb / spp];
        cnt_off = (qb % spp) * sub;
      } else {
        cnt = 0;
        cnt_off = 0;
      }
    };
    float m[32], l[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      m[i] = -INFINITY;
      l[i] = 0.f;
    }
    bool ok = true;
    if (n_tiles > 0) load_count(0);
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j & 1;
      const bool tv = rin + cnt_off < cnt;
      if (j + 1 < n_tiles) load_count(j + 1);
      ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_s_full[st], (j >> 1) & 1, prm.status));
      if (!ok) break;
      tc_fence_after();
      float t[32];
      {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + kColS + st * kHeads + hc * 32, rr);
        tmem_ld_wait(rr);
#pragma unroll
        for (int i = 0; i < 32; ++i) t[i] = tv ? __uint_as_float(rr[i]) * prm.scale_log2 : -INFINITY;
      }
      tc_fence_before();
      mbar_arrive(&s.bar_s_free[st]);
      // tile maxima per head: over the warp's 32 tokens, then over the four lane quarters
      {
        float* dst = s.red_m[st][hc][quarter];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float a0 = warp_max(t[i]), a1 = warp_max(t[i + 1]), a2 = warp_max(t[i + 2]),
                      a3 = warp_max(t[i + 3]);
          if (lane == 0) *reinterpret_cast<float4*>(dst + i) = make_float4(a0, a1, a2, a3);
        }
      }
      mbar_arrive(&s.bar_x[hc]);
      ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_x[hc], j & 1, prm.status));
      if (!ok) break;
      bool any = false;
      float my_alpha = 1.f;
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 mx = *reinterpret_cast<const float4*>(&s.red_m[st][hc][0][i]);
#pragma unroll
        for (int qq = 1; qq < 4; ++qq) {
          const float4 o = *reinterpret_cast<const float4*>(&s.red_m[st][hc][qq][i]);
          mx.x = fmaxf(mx.x, o.x);
          mx.y = fmaxf(mx.y, o.y);
          mx.z = fmaxf(mx.z, o.z);
          mx.w = fmaxf(mx.w, o.w);
        }
        const float tm[4] = {mx.x, mx.y, mx.z, mx.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (tm[e] > m[i + e] + kLazy) {  // uniform over the four warps of this head half
            const float alpha = ex2(m[i + e] - tm[e]);
            l[i + e] *= alpha;
            if (lane == i + e) my_alpha = alpha;
            m[i + e] = tm[e];
            any = true;
          }
        }
      }
      // the P buffer is free once O^T += V^T P^T_{j-1} has completed
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_pv_done[st ^ 1], ((j - 1) >> 1) & 1, prm.status));
        if (!ok) break;
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {  // heads [8cc, 8cc + 8) of the warp's 32: one 16-byte chunk
        uint32_t hv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = cc * 8 + 2 * e;
          const float m0 = m[i] == -INFINITY ? 0.f : m[i];
          const float m1 = m[i + 1] == -INFINITY ? 0.f : m[i + 1];
          const float e0 = ex2(t[i] - m0), e1 = ex2(t[i + 1] - m1);
          l[i] += e0;
          l[i + 1] += e1;
          hv[e] = pack_bf16(e0, e1);
        }
        *reinterpret_cast<uint4*>(s.p + sw128(r, hc * 4 + cc)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      }
      if (any && j > 0) {
        // O^T holds P_{j-1} V_{j-1} once pv_done of tile j-1 has its phase (already waited for
        // above, before P_j was written); the phase before it completed before P_{j-1} was
        // written, so the parity is exact
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_pv_done[st ^ 1], ((j - 1) >> 1) & 1, prm.status));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t rr[32];
          const uint32_t addr = tmem + lane_base + kColO + mt * kHeads + hc * 32;
          tmem_ld32(addr, rr);
          tmem_ld_wait(rr);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            rr[i] = __float_as_uint(__uint_as_float(rr[i]) * __shfl_sync(0xffffffffu, my_alpha, i));
          tmem_st32(addr, rr);
        }
        tmem_st_wait();
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&s.bar_p_full[st]);
    }
    // ---- epilogue: TMEM lane = dv row of each 128-row tile; columns = this warp's 32 heads
    bool have = ok && n_tiles > 0;
    if (have) {
      const int jl = n_tiles - 1;
      have = __all_sync(0xffffffffu, mbar_wait(&s.bar_pv_done[jl & 1], (jl >> 1) & 1, prm.status));
      tc_fence_after();
    }
    // l over the 128 tokens: lane i gets the warp's total of head i, then the four quarters add
    float lw = transpose_sum(l, lane);
    s.red_l[hc][quarter][lane] = lw;
    if (ok) {
      mbar_arrive(&s.bar_x[hc]);
      have = __all_sync(0xffffffffu, mbar_wait(&s.bar_x[hc], n_tiles & 1, prm.status)) && have;
    }
    float L = 0.f;
    if (have)
      L = ((s.red_l[hc][0][lane] + s.red_l[hc][1][lane]) + s.red_l[hc][2][lane]) + s.red_l[hc][3][lane];
    float mh = m[0];
#pragma unroll
    for (int i = 1; i < 32; ++i)
      if (lane == i) mh = m[i];
    const bool single = prm.unit_pieces[u] == 1;
    const bool any = have && L > 0.f;
    const float inv_l = any ? 1.f / L : 0.f;
    const int hl = hc * 32;  // this warp's first head (of the CTA's 64)
#pragma unroll 1
    for (int mt = 0; mt < 4; ++mt) {
      uint32_t rr[32];
      if (have) {
        tmem_ld32(tmem + lane_base + kColO + mt * kHeads + hl, rr);
        tmem_ld_wait(rr);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) rr[i] = 0u;
      }
      const int dv = mt * 128 + r;
      if (single) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float sc = __shfl_sync(0xffffffffu, inv_l, i);
          if (hl + i < nh)
            prm.out[static_cast<size_t>(qrow0 + hl + i) * kDQ + dv] = __float2bfloat16_rn(__uint_as_float(rr[i]) * sc);
        }
      } else {
        float* dst = prm.part_o + (static_cast<size_t>(piece) * kHeads + hl) * kDQ + dv;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (hl + i < nh) dst[static_cast<size_t>(i) * kDQ] = __uint_as_float(rr[i]);
      }
    }
    if (quarter == 0 && hl + lane < nh) {
      const size_t orow = static_cast<size_t>(qrow0 + hl + lane);
      if (single) {
        prm.lse[orow] = any ? (mh * kLn2 + logf(L)) : -INFINITY;
      } else {
        prm.part_m[static_cast<size_t>(piece) * kHeads + hl + lane] = any ? mh : -INFINITY;
        prm.part_l[static_cast<size_t>(piece) * kHeads + hl + lane] = have ? L : 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Merge the pieces of each unit in piece order:  M = max m_p, L = sum l_p 2^(m_p - M),
// Out = sum O_p 2^(m_p - M) / L,  LSE = (M + log2 L) ln 2.  One warp per (unit, head); each lane
// owns 16 of the 512 Dv columns, so every partial row is read with coalesced 16-byte loads.
__global__ void __launch_bounds__(256) sfa_combine_kernel(const DecParams prm, const int32_t* __restrict__ unit_first) {
  griddep_wait();  // launched early: the decode pieces must be complete
  const int u = blockIdx.x;
  const int hcol = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int bg = u / prm.HH, hh = u % prm.HH;
  const int head = hh * kHeads + hcol;
  if (hcol >= kHeads || head >= prm.G) return;
  const int pcs = prm.unit_pieces[u];
  if (pcs == 1) return;  // written by its single piece
  const int b = bg / prm.N2, g = bg % prm.N2;
  const int p0 = unit_first[u];
  const size_t orow = static_cast<size_t>(b * prm.N1 + g * prm.G + head);
  __nv_bfloat16* dst = prm.out + orow * kDQ + lane * 16;
  float M = -INFINITY;
  for (int p = 0; p < pcs; ++p) M = fmaxf(M, prm.part_m[static_cast<size_t>(p0 + p) * kHeads + hcol]);
  float L = 0.f, acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int p = 0; p < pcs; ++p) {
    const float mp = prm.part_m[static_cast<size_t>(p0 + p) * kHeads + hcol];
    if (mp == -INFINITY) continue;
    const float wgt = ex2(mp - M);
    L += prm.part_l[static_cast<size_t>(p0 + p) * kHeads + hcol] * wgt;
    const float4* src =
        reinterpret_cast<const float4*>(prm.part_o + (static_cast<size_t>(p0 + p) * kHeads + hcol) * kDQ + lane * 16);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 a = src[c];
      acc[4 * c] += a.x * wgt;
      acc[4 * c + 1] += a.y * wgt;
      acc[4 * c + 2] += a.z * wgt;
      acc[4 * c + 3] += a.w * wgt;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;  // pcs == 0 (no selected key): Out = 0, LSE = -inf
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint4 pk;
    pk.x = pack_bf16(acc[8 * c] * inv, acc[8 * c + 1] * inv);
    pk.y = pack_bf16(acc[8 * c + 2] * inv, acc[8 * c + 3] * inv);
    pk.z = pack_bf16(acc[8 * c + 4] * inv, acc[8 * c + 5] * inv);
    pk.w = pack_bf16(acc[8 * c + 6] * inv, acc[8 * c + 7] * inv);
    *reinterpret_cast<uint4*>(dst + 8 * c) = pk;
  }
  if (lane == 0) prm.lse[orow] = L > 0.f ? (M * kLn2 + logf(L)) : -INFINITY;
}

}  // namespace

int sfa_head_halves(int G) { return G > kHeads ? 2 : 1; }

cudaError_t sfa_decode_launch(const SfaDecodeArgs& a, cudaStream_t st) {
  CUtensorMap tq, tqr, tk, tkr, tv;
  const int sub = a.page_size % 64 == 0 ? 64 : 32;
  const uint64_t qrows = static_cast<uint64_t>(a.B) * a.N1;
  const uint64_t tokens = static_cast<uint64_t>(a.num_pages) * a.page_size;
  if (!make_tmap_2d_bf16(&tq, a.q, qrows, kDQ, kDQ, kHeads) ||
      !make_tmap_2d_bf16(&tqr, a.q_rope, qrows, kDR, kDR, kHeads) ||
      !make_tmap_3d_bf16(&tk, a.k_cache, kDQ, a.N2, tokens, kDQ, static_cast<uint64_t>(a.N2) * kDQ, 1, sub) ||
      !make_tmap_3d_bf16(&tkr, a.k_rope_cache, kDR, a.N2, tokens, kDR, static_cast<uint64_t>(a.N2) * kDR, 1, sub) ||
      !make_tmap_3d_bf16(&tv, a.v_cache, kDQ, a.N2, tokens, kDQ, static_cast<uint64_t>(a.N2) * kDQ, 1, sub))
    return cudaErrorInvalidValue;
  DecParams p;
  p.B = a.B; p.N1 = a.N1; p.N2 = a.N2; p.G = a.N1 / a.N2; p.HH = sfa_head_halves(p.G);
  p.page_size = a.page_size; p.cap = a.cap; p.sub_rows = sub;
  p.scale_log2 = a.scale * kLog2e;
  p.pages = a.pages; p.tokens = a.tokens; p.piece_unit = a.piece_unit; p.piece_begin = a.piece_begin;
  p.piece_len = a.piece_len; p.unit_pieces = a.unit_pieces; p.n_pieces = a.n_pieces;
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
  e = launch_pdl(sfa_combine_kernel, dim3(a.units, kHeads / 8), dim3(256), 0, st, p, a.unit_first);
  prof_end(st);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sa
