// Sparse flash attention decode over a paged KV cache (SparseFlashAttention page, formula):
//   Out = softmax((q k~^T + q_rope k_rope~^T) * scale) v~,  D = Dv = 512, Dr = 64, q_len = 1
// where k~ / v~ are the tokens of the selected sparse blocks.
//
// The query side of a decode step is small (the G = N1/N2 heads of one kv head, one row each) and
// the key side long, so the products are taken transposed, with the tokens as the MMA's M = 128
// rows and the heads as N:
//   S^T [128 tokens][64 heads]  = K~ [128][576] . Q^T          (Q of 64 heads stays in shared memory)
//   O^T [512 dv][64 heads]     += V~^T [512][128] . P^T [128][64] (four M = 128 tiles of dv)
// A unit is (batch, kv head, half of the G heads).  Its compacted page list (sfa_pages.cuh, the
// code the metadata op runs too) is built in the kernel's prologue while Q is loaded, and its n
// pages are split evenly over P pieces (P = the thread-block cluster size, up to 4): piece p takes
// pages [floor(p n / P), floor((p + 1) n / P)).  One CTA per piece.  O^T takes
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
// 9 V producer, 10 builds the page list then issues S^T, 11 issues O^T += V^T P^T (and first zeroes
// the V rows of a partly used page past its tokens in use: those rows get weight 0, but a
// non-finite value there would still turn 0 * x into NaN).  With P = 1 the CTA writes Out and LSE;
// otherwise the P CTAs of a cluster leave their (O, m, l) in shared memory and each merges a
// 512 / P slice of the head dim from all of them over distributed shared memory, in rank order.
#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"
#include "sfa_pages.cuh"

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
  float cl_m[kHeads], cl_l[kHeads];        // this piece's running max (log2 units) and sum per head
  float cl_w[kHeads][kSfaMaxPieces];       // merge weights of the cluster's pieces per head
  int32_t setup[3];                        // n, begin, len of this piece
  uint32_t tmem_base;
};

struct DecParams {
  int B, N1, N2, G, HH, P, K, ppb, page_size, max_pages_per_seq, num_pages, cap, sub_rows;
  float scale_log2;
  const int32_t* sparse_indices;
  const int32_t* block_table;
  const int32_t* seqused_kv;
  int32_t* pages;   // [piece][cap]: the unit's compacted page list, built by the piece itself
  int32_t* tokens;  // [piece][cap]: tokens in use of each listed page
  int32_t* rec;     // [piece][3]: n, begin, len
  __nv_bfloat16* out;
  float* lse;
  uint32_t* status;
};

// ---- thread-block cluster: distributed shared memory and the cluster barrier --------------------
__device__ __forceinline__ uint32_t cluster_map(const void* p, int rank) {  // own smem -> rank's copy
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a)
               : "memory");
  return v;
}
// Every thread of every CTA of the cluster: shared-memory writes before it are visible to the
// cluster's reads after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

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
  griddep_launch_dependents();
  griddep_wait();  // launched early (programmatic dependent launch): the inputs must be complete
  const int piece = blockIdx.x;  // unit * P + its rank in the cluster
  extern __shared__ uint8_t smem_raw[];
  DecSmem& s = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = piece / prm.P, rank = piece % prm.P;
  const int bg = u / prm.HH, hh = u % prm.HH;
  const int b = bg / prm.N2, g = bg % prm.N2;
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
  // Q does not depend on the page list: its load overlaps the list's construction
  if (warp == kSmWarps && lane == 0) {
    mbar_arrive_expect_tx(&s.bar_q, kKChunks * kHeads * 128);
    for (int c = 0; c < 8; ++c) tma_load_2d(s.q[c], &tm_q, &s.bar_q, c * 64, qrow0);
    tma_load_2d(s.q[8], &tm_qr, &s.bar_q, 0, qrow0);
  }
  if (warp == kSmWarps + 2) {
    int n, begin, len;
    sfa_piece_setup(piece, prm.P, prm.HH, prm.N2, prm.K, prm.ppb, prm.page_size, prm.max_pages_per_seq,
                    prm.num_pages, prm.sparse_indices, prm.block_table, prm.seqused_kv,
                    prm.pages + static_cast<size_t>(piece) * prm.cap, prm.tokens + static_cast<size_t>(piece) * prm.cap,
                    &n, &begin, &len, prm.status);
    if (lane == 0) {
      s.setup[0] = n;
      s.setup[1] = begin;
      s.setup[2] = len;
      prm.rec[3 * piece] = n;
      prm.rec[3 * piece + 1] = begin;
      prm.rec[3 * piece + 2] = len;
    }
  }
  __syncthreads();  // the page list (global, written by this CTA) and the piece's range are ready
  const int pbeg = s.setup[1];
  const int npages = s.setup[2];
  const int sub = prm.sub_rows;             // tokens per TMA box (32 or 64, divides the page)
  const int spp = prm.page_size / sub;      // boxes per page
  const int n_sub = kTok / sub;             // boxes per tile
  const int n_chunks = npages * spp;
  const int n_tiles = (n_chunks + n_sub - 1) / n_sub;
  const int32_t* plist = prm.pages + static_cast<size_t>(piece) * prm.cap + pbeg;
  const int32_t* tlist = prm.tokens + static_cast<size_t>(piece) * prm.cap + pbeg;

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
      if (lane == 0)
        for (int use = (issued > kKR ? issued - kKR : 0); use < issued; ++use)
          mbar_wait(&s.bar_k[use % kKR], (use / kKR) & 1, prm.status);
    }
    if (lane == 0) mbar_wait(&s.bar_q, 0, prm.status);
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
    // Lane 0 issues; the warp first zeroes the V rows of a box past its page's tokens in use (the
    // last page of a sequence, or a box past the piece's end that repeats the tile's first box).
    if (n_tiles > 0) {
      const uint32_t id_o = idesc_bf16_f32(kTok, kHeads, true, true);
      // A = V^T: MN-major, the two 64-dv chunks of a slot 8 KB apart; B = P^T: MN-major, one chunk
      const uint64_t dv0 = sdesc_sw128(smem_u32(s.v[0]), 64 * 128, 1024);
      const uint64_t dp0 = sdesc_sw128(smem_u32(s.p), kSlot, 1024);
      const int half_boxes = n_sub / 2;  // boxes per token half of a tile
      bool ok = true;
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j & 1;
        // rows in use of each box of the tile (lane t < n_sub: box t)
        int valid = sub;
        if (lane < n_sub) {
          const int qb = j * n_sub + lane;
          valid = qb < n_chunks ? max(0, min(sub, tlist[qb / spp] - (qb % spp) * sub)) : 0;
        }
        const uint32_t partial = __ballot_sync(0xffffffffu, lane < n_sub && valid < sub);
        if (partial == 0) {
          // every box of the tile is fully in use: lane 0 alone waits and issues
          if (lane == 0) {
            ok = mbar_wait(&s.bar_p_full[st], (j >> 1) & 1, prm.status);
            for (int x = 0; ok && x < kVUses; ++x) {
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
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (ok && lane == 0) tc_commit(&s.bar_pv_done[st]);
          continue;
        }
        // one barrier per tile parity: its next phase needs P_{j+2}, written after this product
        if (lane == 0) ok = mbar_wait(&s.bar_p_full[st], (j >> 1) & 1, prm.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        for (int x = 0; x < kVUses; ++x) {
          const int mt = x >> 1, th = x & 1;
          const int use = j * kVUses + x, slot = use % kVR;
          if (lane == 0) ok = mbar_wait(&s.bar_v[slot], (use / kVR) & 1, prm.status);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          const uint32_t mine = (partial >> (th * half_boxes)) & ((1u << half_boxes) - 1u);
          if (mine) {
            // every lane observes the copy's completion itself before it overwrites part of it
            ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_v[slot], (use / kVR) & 1, prm.status));
            if (!ok) break;
            for (int t = 0; t < half_boxes; ++t) {
              if (!((mine >> t) & 1u)) continue;
              const int v0 = __shfl_sync(0xffffffffu, valid, th * half_boxes + t);
              uint8_t* box = s.v[slot] + t * sub * 128;
              const int n16 = (sub - v0) * 8;  // 16-byte chunks per 64-dv chunk to clear
              for (int c = lane; c < 2 * n16; c += 32) {
                const int chunk = c / n16, e = c % n16;
                *reinterpret_cast<uint4*>(box + chunk * (64 * 128) + v0 * 128 + e * 16) = make_uint4(0u, 0u, 0u, 0u);
              }
            }
            fence_async_smem();
            __syncwarp();
          }
          if (lane == 0) {
            tc_fence_after();
            const uint64_t dv = sdesc_add(dv0, slot * kSlot);
            const uint64_t dp = sdesc_add(dp0, th * (64 * 128));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16_ss(tmem + kColO + mt * kHeads, sdesc_add(dv, ks * 2048), sdesc_add(dp, ks * 2048), id_o,
                          (j > 0 || th > 0 || ks > 0) ? 1u : 0u);
            tc_commit(&s.bar_v_empty[slot]);
          }
          __syncwarp();
        }
        if (ok && lane == 0) tc_commit(&s.bar_pv_done[st]);
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
    const bool any = have && L > 0.f;
    const int hl = hc * 32;  // this warp's first head (of the CTA's 64)
    if (prm.P == 1) {
      const float inv_l = any ? 1.f / L : 0.f;
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
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float sc = __shfl_sync(0xffffffffu, inv_l, i);
          if (hl + i < nh)
            prm.out[static_cast<size_t>(qrow0 + hl + i) * kDQ + dv] = __float2bfloat16_rn(__uint_as_float(rr[i]) * sc);
        }
      }
      if (quarter == 0 && hl + lane < nh)
        prm.lse[static_cast<size_t>(qrow0 + hl + lane)] = any ? (mh * kLn2 + logf(L)) : -INFINITY;
    } else {
      // O^T (unnormalised) into this CTA's shared memory as [64 heads][512 dv] fp32 over the K and
      // V rings (all their copies and products have completed); m and l per head beside it
      float* so = reinterpret_cast<float*>(s.k[0]);
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
#pragma unroll
        for (int i = 0; i < 32; ++i) so[(hl + i) * kDQ + mt * 128 + r] = __uint_as_float(rr[i]);
      }
      if (quarter == 0) {
        s.cl_m[hl + lane] = any ? mh : -INFINITY;
        s.cl_l[hl + lane] = any ? L : 0.f;
      }
    }
  }
  if (prm.P > 1) {
    // ---- merge of the cluster's pieces (all threads of every CTA of the cluster take part)
    const int P = prm.P;
    cluster_sync_all();
    if (tid < kHeads) {  // per head: M = max m_q, L = sum l_q 2^(m_q - M), weight 2^(m_q - M) / L
      float mq[kSfaMaxPieces], lq[kSfaMaxPieces];
      float M = -INFINITY;
      for (int q = 0; q < P; ++q) {
        mq[q] = ld_cluster_f32(cluster_map(&s.cl_m[tid], q));
        lq[q] = ld_cluster_f32(cluster_map(&s.cl_l[tid], q));
        M = fmaxf(M, mq[q]);
      }
      float Lt = 0.f;
      for (int q = 0; q < P; ++q)
        if (mq[q] != -INFINITY) Lt += lq[q] * ex2(mq[q] - M);
      const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
      for (int q = 0; q < P; ++q) s.cl_w[tid][q] = (mq[q] != -INFINITY) ? ex2(mq[q] - M) * inv : 0.f;
      if (rank == 0 && tid < nh)
        prm.lse[static_cast<size_t>(qrow0 + tid)] = Lt > 0.f ? (M + log2f(Lt)) * kLn2 : -INFINITY;
    }
    __syncthreads();
    // this CTA's slice of the head dim: float4 columns [f0, f1) of the 128 per row
    const int f0 = rank * (kDQ / 4) / P, f1 = (rank + 1) * (kDQ / 4) / P, nf = f1 - f0;
    const float* so = reinterpret_cast<const float*>(s.k[0]);
    for (int idx = tid; idx < nh * nf; idx += kThreads) {
      const int h = idx / nf, f = f0 + idx % nf;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < P; ++q) {
        const float w = s.cl_w[h][q];
        const float4 o = ld_cluster_f32x4(cluster_map(so + h * kDQ + 4 * f, q));
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
      }
      uint2 pk;
      pk.x = pack_bf16(acc.x, acc.y);
      pk.y = pack_bf16(acc.z, acc.w);
      *reinterpret_cast<uint2*>(prm.out + static_cast<size_t>(qrow0 + h) * kDQ + 4 * f) = pk;
    }
    cluster_sync_all();  // no CTA leaves while another still reads its shared memory
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
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
  p.B = a.B; p.N1 = a.N1; p.N2 = a.N2; p.G = a.N1 / a.N2; p.HH = sfa_head_halves(p.G); p.P = a.P;
  p.K = a.K; p.ppb = a.ppb; p.page_size = a.page_size; p.max_pages_per_seq = a.max_pages_per_seq;
  p.num_pages = a.num_pages; p.cap = a.K * a.ppb; p.sub_rows = sub;
  p.scale_log2 = a.scale * kLog2e;
  p.sparse_indices = a.sparse_indices; p.block_table = a.block_table; p.seqused_kv = a.seqused_kv;
  p.pages = a.pages; p.tokens = a.tokens; p.rec = a.rec;
  p.out = static_cast<__nv_bfloat16*>(a.out); p.lse = a.lse; p.status = a.status;
  const size_t smem = sizeof(DecSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(sfa_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = a.units * a.P;
  if (grid == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = a.P;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.P > 1 ? 2 : 1;
  prof_begin("sfa_decode", st);
  e = cudaLaunchKernelEx(&cfg, sfa_decode_kernel, tq, tqr, tk, tkr, tv, p);
  prof_end(st);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sa
