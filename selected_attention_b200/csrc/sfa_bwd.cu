// Backward of the paged sparse decode (SparseFlashAttention page, formula; the gradient formulas
// are the BlockSparseAttentionGrad page's, applied to the gathered keys with the rope-split score
// s = scale (q.k + q_rope.k_rope)):
//   P  = exp(s - LSE),   D = rowsum(dOut o Out),   dP = dOut v~^T,   dS = P o (dP - D)
//   dQ = scale dS k~,  dQ_rope = scale dS k_rope~,  dk~ = scale dS^T q,  dk_rope~ = scale dS^T q_rope,
//   dv~ = P^T dOut
// and the gradient of every cache row the step read is the sum of its gathered rows' gradients.
//
// The key side of a decode step is long and the query side one row per head, so, as in the
// forward, the products are taken with 128 gathered tokens as the MMA's M:
//   S^T [128 tok][G]  = [k~ | k_rope~] . [q | q_rope]^T      (9 chunks of 64 dims)
//   dP^T [128 tok][G] = v~ . dOut^T                           (8 chunks)
//   dv~ [128 tok][512] = P^T . dOut                           (4 column chunks of 128)
//   dk~ [128 tok][576] = dS^T . [q | q_rope]                  (4 chunks of 128 + 1 of 64)
// One CTA per (batch, kv head, tile of 128 gathered tokens).  S^T and dP^T take TMEM columns
// [0, 256); the element-wise warps turn them into P^T and dS^T (bf16) in shared memory, the
// K-major A operands of dv~ / dk~, and the tile's dS^T is also stored for the dQ kernel.  The 9
// column chunks of the two gradient products alternate between two 128-column TMEM buffers, so the
// warps write one chunk out while the next is computed: each warp stages its 32 rows x 64 columns
// in shared memory and writes them with one TMA store (rows of the outputs are 1 KB or more apart,
// so the TMEM layout, one row per thread, would otherwise cost a separate 32-byte sector per thread
// and store).  Every operand tile streams through one ring of 32 KB stages (two 16 KB [128 rows][64]
// tiles, 128-byte swizzle) in the order the products use them; q and dOut are read twice
// (L2-resident: one batch's q and dOut are 272 KB).
//
// dv~ and dk~ rows (bf16) go straight into the cache gradients when their page has one reader (the
// common case), else into a gathered-order scratch.  The dQ kernel accumulates
//   dQ [G][64-dim chunk] = sum over the unit's tiles of dS . [k~ | k_rope~]
// in TMEM (one CTA per (batch, kv head, 64-dim chunk), tiles in order), and a third kernel writes
// the rows of every page with two or more readers: the sum, in a fixed order, of the gathered rows
// read from it (a page listed twice, or reached from two batches, adds its contributions), so no
// result depends on scheduling.  Every row of a page the step read is written (rows past the
// sequence's end get zero).  Rows of a page past its tokens in use are masked (P = dS = 0), and the
// dQ kernel zeroes the k~ rows there (a non-finite value in a cache tail would turn 0 * x into NaN).
#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

constexpr int kTok = 128;      // gathered tokens per tile
constexpr int kDQ = 512;       // q / k / v head dim
constexpr int kDR = 64;        // rope dim
constexpr int kDK = kDQ + kDR;  // q|q_rope, k|k_rope
constexpr int kQC = 9;         // 64-wide chunks of q|q_rope
constexpr int kVC = 8;         // 64-wide chunks of v / dOut
constexpr int kRing = 3;       // ring stages
constexpr int kCw = 8;         // element-wise / epilogue warps
constexpr int kThreads = (kCw + 2) * 32;  // + producer, MMA issuer
constexpr uint32_t kTile = kTok * 128;    // [128 rows][64 bf16], 16 KB
constexpr int kStages = kQC + kVC + 4 + 5;  // 26 per tile
constexpr int kChunks = 9;                 // 4 dv~ + 5 dk~
constexpr uint32_t kColS = 0, kColDP = 128, kColOut = 256;
constexpr float kLog2e = 1.4426950408889634f;

struct __align__(1024) BwdSmem {
  uint8_t ring[kRing][2][kTile];   // stages of two tiles
  uint8_t pt[2][kTile];            // P^T  [128 tok][2 x 64 heads] bf16 (K-major atoms of 64 heads)
  uint8_t dst[2][kTile];           // dS^T
  uint8_t stage_out[kCw][4096];    // per epilogue warp: [32 rows][128 B] of output, then a TMA store
  float lse2[128], dvec[128];      // per head: LSE log2(e), rowsum(dOut o Out)
  int32_t vrow[kTok];              // gathered row in use (1) or masked (0)
  uint64_t full[kRing], empty[kRing];
  uint64_t bar_scores, bar_ops, chunk_full[2], chunk_free[2];
  uint32_t tmem_base;
};

struct BwdParams {
  int B, N1, N2, G, Gp, K, ppb, page_size, cap, sub_rows, T;
  float scale, scale_log2;
  const int32_t* pages;
  const int32_t* tokens;
  const int32_t* count;
  const float* lse2;
  const float* dvec;
  int rows_u;              // cap * page_size: gathered rows per unit
  const int32_t* refs;     // [num_pages * N2]: readers of each cache row-block (page, kv head)
  uint32_t* status;
};

// The ring's stage s of a tile: which tiles it holds.  kind: 0 K~ chunk, 1 V~ chunk, 2 Q chunk,
// 3 dOut chunk; (kind0, c0) is the first tile, (kind1, c1) the second (c1 < 0: none).
struct StageDef {
  int kind0, c0, kind1, c1;
};
__device__ __forceinline__ StageDef stage_def(int s) {
  if (s < kQC) return {0, s, 2, s};                       // S^T: K~_c, Q_c
  if (s < kQC + kVC) return {1, s - kQC, 3, s - kQC};     // dP^T: V~_c, dOut_c
  s -= kQC + kVC;
  if (s < 4) return {3, 2 * s, 3, 2 * s + 1};             // dv~ chunk: dOut pair
  s -= 4;
  return {2, 2 * s, 2, s < 4 ? 2 * s + 1 : -1};           // dk~ chunk: Q pair (the last: q_rope)
}

__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads, 1)
    sfa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                   const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_gk, const __grid_constant__ CUtensorMap tm_gv,
                   const __grid_constant__ CUtensorMap tm_ds, const __grid_constant__ CUtensorMap tm_dkc,
                   const __grid_constant__ CUtensorMap tm_dkrc, const __grid_constant__ CUtensorMap tm_dvc,
                   const BwdParams prm) {
  griddep_launch_dependents();
  griddep_wait();  // page lists and the preprocess must be complete
  const int u = blockIdx.y, t = blockIdx.x;  // unit (b, g), tile
  const int b = u / prm.N2, g = u % prm.N2;
  const int sub = prm.sub_rows, spp = prm.page_size / sub, n_sub = kTok / sub;
  const int n_chunks = prm.count[u] * spp;
  const int n_tiles = (n_chunks + n_sub - 1) / n_sub;
  if (t >= n_tiles) return;  // uniform over the CTA, before any barrier or TMEM use
  extern __shared__ uint8_t smem_raw[];
  BwdSmem& s = *reinterpret_cast<BwdSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qrow0 = b * prm.N1 + g * prm.G;
  const int32_t* plist = prm.pages + static_cast<size_t>(u) * prm.cap;
  const int32_t* tlist = prm.tokens + static_cast<size_t>(u) * prm.cap;

  if (tid == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.bar_scores, 1);
    mbar_init(&s.bar_ops, kCw * 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.chunk_full[i], 1);
      mbar_init(&s.chunk_free[i], kCw * 32);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  // per head and per row set-up (the rows of box q of the tile: entry qb / spp, offset)
  for (int h = tid; h < 128; h += kThreads) {
    s.lse2[h] = h < prm.G ? prm.lse2[qrow0 + h] : 0.f;
    s.dvec[h] = h < prm.G ? prm.dvec[qrow0 + h] : 0.f;
  }
  for (int r = tid; r < kTok; r += kThreads) {
    const int qb = t * n_sub + r / sub, off = (qb % spp) * sub + r % sub;
    s.vrow[r] = (qb < n_chunks && off < tlist[qb / spp]) ? 1 : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == kCw) {
    // ------------------------------------------------------------------ producer
    // Box q of the tile is gathered from entry qb / spp at token offset (qb % spp) * sub; a box past
    // the unit's end repeats the tile's first box (its rows are masked; the copy stays in bounds).
    int tok = 0;
    if (lane < n_sub) {
      const int qb0 = t * n_sub + lane;
      const int qb = qb0 < n_chunks ? qb0 : t * n_sub;
      tok = plist[qb / spp] * prm.page_size + (qb % spp) * sub;
    }
    bool ok = true;
    for (int st = 0; ok && st < kStages; ++st) {
      const int slot = st % kRing;
      if (lane == 0 && st >= kRing) ok = mbar_wait(&s.empty[slot], ((st / kRing) - 1) & 1, prm.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const StageDef d = stage_def(st);
      if (lane == 0) mbar_arrive_expect_tx(&s.full[slot], (d.c1 >= 0 ? 2u : 1u) * kTile);
      __syncwarp();
      for (int x = 0; x < 2; ++x) {
        const int kind = x ? d.kind1 : d.kind0, c = x ? d.c1 : d.c0;
        if (c < 0) continue;
        uint8_t* dst = s.ring[slot][x];
        if (kind <= 1) {  // gathered rows: n_sub boxes of sub tokens
          if (lane < n_sub) {
            uint8_t* bx = dst + lane * sub * 128;
            if (kind == 0) {
              if (c < 8) tma_load_3d(bx, &tm_k, &s.full[slot], c * 64, g, tok);
              else tma_load_3d(bx, &tm_kr, &s.full[slot], 0, g, tok);
            } else {
              tma_load_3d(bx, &tm_v, &s.full[slot], c * 64, g, tok);
            }
          }
        } else if (lane == 0) {  // the unit's 128 query rows
          if (kind == 2) {
            if (c < 8) tma_load_2d(dst, &tm_q, &s.full[slot], c * 64, qrow0);
            else tma_load_2d(dst, &tm_qr, &s.full[slot], 0, qrow0);
          } else {
            tma_load_2d(dst, &tm_do, &s.full[slot], c * 64, qrow0);
          }
        }
      }
      __syncwarp();
    }
    // wait for this CTA's own copies still in flight before it may exit
    if (lane == 0)
      for (int st = kStages - kRing; st < kStages; ++st) mbar_wait(&s.full[st % kRing], (st / kRing) & 1, prm.status);
  } else if (warp == kCw + 1) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t id_s = idesc_bf16_f32(kTok, prm.Gp, false, false);
    const uint64_t ring0 = sdesc_sw128(smem_u32(s.ring[0][0]), 0, 1024);
    bool ok = true;
    int st = 0;
    auto wait_stage = [&](int stg) -> bool {
      bool r = true;
      if (lane == 0) r = mbar_wait(&s.full[stg % kRing], (stg / kRing) & 1, prm.status);
      return __shfl_sync(0xffffffffu, r, 0);
    };
    // S^T and dP^T: A = the gathered tile (K-major), B = the query-side tile (K-major)
    for (; ok && st < kQC + kVC; ++st) {
      if (!(ok = wait_stage(st))) break;
      if (lane == 0) {
        tc_fence_after();
        const uint64_t a = sdesc_add(ring0, (st % kRing) * 2 * kTile);
        const uint64_t bq = sdesc_add(a, kTile);
        const uint32_t d = tmem + (st < kQC ? kColS : kColDP);
        const bool first = st == 0 || st == kQC;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16_ss(d, sdesc_add(a, ks * 32), sdesc_add(bq, ks * 32), id_s, (!first || ks > 0) ? 1u : 0u);
        tc_commit(&s.empty[st % kRing]);
      }
      __syncwarp();
    }
    if (ok && lane == 0) tc_commit(&s.bar_scores);
    // the three gradient products, once P^T and dS^T are in shared memory
    if (ok && lane == 0) ok = mbar_wait(&s.bar_ops, 0, prm.status);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok && lane == 0) {  // the tile's dS^T for the dQ kernel: two [128 tok][64 heads] boxes
      tma_store_3d(&tm_ds, s.dst[0], 0, t * kTok, u);
      tma_store_3d(&tm_ds, s.dst[1], 64, t * kTok, u);
      bulk_commit();
    }
    const uint64_t dpt = sdesc_sw128(smem_u32(s.pt[0]), 0, 1024);  // K-major A, atoms 16 KB apart
    const uint64_t dds = sdesc_sw128(smem_u32(s.dst[0]), 0, 1024);
    const int ksteps = prm.Gp / 16;
    for (int j = 0; ok && j < kChunks; ++j, ++st) {
      const int buf = j & 1;
      if (j >= 2 && lane == 0) ok = mbar_wait(&s.chunk_free[buf], ((j >> 1) - 1) & 1, prm.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (!(ok = wait_stage(st))) break;
      const int slot = st % kRing;
      const bool rope = j == 8;  // the 64-wide last chunk of dk~
      const int n = rope ? 64 : 128;
      if (lane == 0) {
        tc_fence_after();
        const uint64_t bst = sdesc_sw128(smem_u32(s.ring[slot][0]), kTile, 1024);  // MN-major B, N chunks 16 KB apart
        const uint32_t d = tmem + kColOut + buf * 128;
        // dv~ / dk~: M = tokens, K = heads: A = P^T or dS^T (K-major), B = dOut / Q pair (MN-major)
        const uint32_t id = idesc_bf16_f32(kTok, n, false, true);
        const uint64_t a0 = j < 4 ? dpt : dds;
        for (int ks = 0; ks < ksteps; ++ks)
          mma_bf16_ss(d, sdesc_add(a0, (ks >> 2) * kTile + (ks & 3) * 32), sdesc_add(bst, ks * 2048), id,
                      ks > 0 ? 1u : 0u);
        tc_commit(&s.empty[slot]);
        tc_commit(&s.chunk_full[buf]);
      }
      __syncwarp();
    }
    if (lane == 0) bulk_wait_all();  // the dS^T store is complete before the CTA exits
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ element-wise and epilogue warps
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // TMEM lane: token row (S^T, dv~, dk~) or head (dQ_t)
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = mbar_wait(&s.bar_scores, 0, prm.status);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const bool vr = s.vrow[r] != 0;
      const float c_s = prm.scale_log2;
      // 64 heads per thread, in two loads of 32
      for (int hc = 0; hc < 2; ++hc) {
        const int h0 = half * 64 + hc * 32;
        uint32_t sr[32], dr[32];
        tmem_ld32(tmem + lane_base + kColS + h0, sr);
        tmem_ld32(tmem + lane_base + kColDP + h0, dr);
        tmem_ld_wait(sr);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float p2[2], d2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = h0 + i + e;
            const float l2 = s.lse2[h];
            const bool on = vr && h < prm.G && l2 != -INFINITY;
            const float p = on ? ex2(fmaf(__uint_as_float(sr[i + e]), c_s, -l2)) : 0.f;
            p2[e] = p;
            d2[e] = on ? p * (__uint_as_float(dr[i + e]) - s.dvec[h]) : 0.f;
          }
          pk[i / 2] = pack_bf16(p2[0], p2[1]);
          dk[i / 2] = pack_bf16(d2[0], d2[1]);
        }
        // row r of the K-major atom `half`: heads h0 - half * 64 .. +32 are 16-byte chunks 4 hc .. 4 hc + 3
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t off = sw128(r, hc * 4 + c);
          *reinterpret_cast<uint4*>(s.pt[half] + off) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          *reinterpret_cast<uint4*>(s.dst[half] + off) = make_uint4(dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3]);
        }
      }
      fence_async_smem();  // the MMA (async proxy) reads P^T / dS^T
      tc_fence_before();
    }
    mbar_arrive(&s.bar_ops);
    // epilogue of the 9 column chunks: rows 32 quarter .. +31 and columns 64 half .. +63 of each
    uint8_t* so = s.stage_out[warp];
    const int row0 = t * kTok + quarter * 32;  // gathered row of lane 0 (dv~, dk~)
    auto flush = [&]() {  // the staged block has been read by its TMA store; the buffer is free
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
    };
    for (int j = 0; ok && j < kChunks; ++j) {
      const int buf = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s.chunk_full[buf], (j >> 1) & 1, prm.status));
      if (!ok) break;
      tc_fence_after();
      const bool rope = j == 8;
      if (!(rope && half == 1)) {
        uint32_t v[32], w[32];
        const uint32_t col = tmem + lane_base + kColOut + buf * 128 + half * 64;
        tmem_ld32(col, v);
        tmem_ld32(col + 32, w);
        tmem_ld_wait(v);
        {
          // dv~ (j < 4) or dk~ (scaled) rows, bf16, gathered order: row lane of the block
          const float mul = j < 4 ? 1.f : prm.scale;
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            pk[i] = pack_bf16(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
            pk[16 + i] = pack_bf16(__uint_as_float(w[2 * i]) * mul, __uint_as_float(w[2 * i + 1]) * mul);
          }
          flush();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(so + sw128(lane, c)) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          fence_async_smem();
          __syncwarp();
          // the block's 32 rows lie in one page of the unit's list (32 divides the page size)
          const int entry = row0 / prm.page_size;
          if (lane == 0 && entry < prm.count[u]) {
            const int page = plist[entry];
            if (prm.refs[page * prm.N2 + g] == 1) {
              // the page's only reader: straight into the cache gradients
              const int crow = page * prm.page_size + row0 % prm.page_size;
              if (j < 4) tma_store_3d(&tm_dvc, so, j * 128 + half * 64, g, crow);
              else if (j < 8) tma_store_3d(&tm_dkc, so, (j - 4) * 128 + half * 64, g, crow);
              else tma_store_3d(&tm_dkrc, so, 0, g, crow);
            } else {
              // a page with several readers: gathered order, summed by the scatter
              if (j < 4) tma_store_3d(&tm_gv, so, j * 128 + half * 64, row0, u);
              else tma_store_3d(&tm_gk, so, (j - 4) * 128 + half * 64, row0, u);
            }
            bulk_commit();
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&s.chunk_free[buf]);
    }
    if (lane == 0) bulk_wait_all();  // the stores are complete before the CTA exits
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// D = rowsum(dOut o Out) and LSE log2(e) per query row; one warp per row of 512.
__global__ void sfa_bwd_prep_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                                    const float* __restrict__ lse, int rows, float* __restrict__ dvec,
                                    float* __restrict__ lse2) {
  griddep_wait();
  griddep_launch_dependents();
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint4* o = reinterpret_cast<const uint4*>(out + static_cast<size_t>(row) * kDQ);
  const uint4* d = reinterpret_cast<const uint4*>(dout + static_cast<size_t>(row) * kDQ);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 a = o[lane + 32 * i], c = d[lane + 32 * i];
    acc += bf16lo(a.x) * bf16lo(c.x) + bf16hi(a.x) * bf16hi(c.x) + bf16lo(a.y) * bf16lo(c.y) +
           bf16hi(a.y) * bf16hi(c.y) + bf16lo(a.z) * bf16lo(c.z) + bf16hi(a.z) * bf16hi(c.z) +
           bf16lo(a.w) * bf16lo(c.w) + bf16hi(a.w) * bf16hi(c.w);
  }
#pragma unroll
  for (int x = 16; x >= 1; x >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, x);
  if (lane == 0) {
    dvec[row] = acc;
    lse2[row] = lse[row] * kLog2e;
  }
}

// dQ of one (unit, 64-dim chunk of q | q_rope): D [128 heads][64 dims] = sum over the unit's tiles
// t (in order) of dS_t [heads][128 tok] . k~_t [128 tok][64 dims], accumulated in TMEM.  A = the
// stored dS^T tile read MN-major (M = heads), B = the tile's gathered k~ chunk read MN-major.
// Warps: 0-3 epilogue (TMEM lane quarter = 32 heads), 4 producer, 5 issuer (it first zeroes the k~
// rows past a page's tokens in use: those rows have dS = 0, but a non-finite cache value would
// still turn 0 * x into NaN).
constexpr int kDqRing = 3;
constexpr int kDqThreads = 6 * 32;

struct __align__(1024) DqSmem {
  uint8_t ds[kDqRing][2][kTile];  // dS^T [128 tok][2 x 64 heads]
  uint8_t k[kDqRing][kTile];      // k~ chunk [128 tok][64 dims]
  uint64_t full[kDqRing], empty[kDqRing], done;
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(kDqThreads, 1)
    sfa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_ds, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_kr, const BwdParams prm, __nv_bfloat16* __restrict__ dq,
                      __nv_bfloat16* __restrict__ dqr) {
  griddep_launch_dependents();
  griddep_wait();  // the dS^T tiles must be complete
  const int c = blockIdx.x, u = blockIdx.y;  // 64-dim chunk (8: q_rope), unit (b, g)
  const int b = u / prm.N2, g = u % prm.N2;
  const int sub = prm.sub_rows, spp = prm.page_size / sub, n_sub = kTok / sub;
  const int n_chunks = prm.count[u] * spp;
  const int n_tiles = (n_chunks + n_sub - 1) / n_sub;
  extern __shared__ uint8_t smem_raw[];
  DqSmem& s = *reinterpret_cast<DqSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t* plist = prm.pages + static_cast<size_t>(u) * prm.cap;
  const int32_t* tlist = prm.tokens + static_cast<size_t>(u) * prm.cap;
  if (tid == 0) {
    for (int i = 0; i < kDqRing; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  if (warp == 4) {
    // ------------------------------------------------------------------ producer
    bool ok = true;
    for (int t = 0; ok && t < n_tiles; ++t) {
      const int slot = t % kDqRing;
      if (lane == 0 && t >= kDqRing) ok = mbar_wait(&s.empty[slot], ((t / kDqRing) - 1) & 1, prm.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&s.full[slot], 3 * kTile);
        tma_load_3d(s.ds[slot][0], &tm_ds, &s.full[slot], 0, t * kTok, u);
        tma_load_3d(s.ds[slot][1], &tm_ds, &s.full[slot], 64, t * kTok, u);
      }
      __syncwarp();
      if (lane < n_sub) {  // box lane of the tile; a box past the unit's end repeats the first
        const int qb0 = t * n_sub + lane;
        const int qb = qb0 < n_chunks ? qb0 : t * n_sub;
        const int tok = plist[qb / spp] * prm.page_size + (qb % spp) * sub;
        uint8_t* bx = s.k[slot] + lane * sub * 128;
        if (c < 8) tma_load_3d(bx, &tm_k, &s.full[slot], c * 64, g, tok);
        else tma_load_3d(bx, &tm_kr, &s.full[slot], 0, g, tok);
      }
      __syncwarp();
    }
    if (lane == 0)
      for (int t = (n_tiles > kDqRing ? n_tiles - kDqRing : 0); t < n_tiles; ++t)
        mbar_wait(&s.full[t % kDqRing], (t / kDqRing) & 1, prm.status);
  } else if (warp == 5) {
    // ------------------------------------------------------------------ zeroing + issuer
    const uint32_t id = idesc_bf16_f32(kTok, 64, true, true);
    bool ok = true;
    for (int t = 0; ok && t < n_tiles; ++t) {
      const int slot = t % kDqRing;
      // rows in use: lane covers rows lane, lane + 32, lane + 64, lane + 96
      uint32_t masked = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;
        const int qb = t * n_sub + r / sub, off = (qb % spp) * sub + r % sub;
        if (!(qb < n_chunks && off < tlist[qb / spp])) masked |= 1u << i;
      }
      const bool any = __any_sync(0xffffffffu, masked != 0);
      // every lane observes the copy's completion itself before it may overwrite part of it
      ok = __all_sync(0xffffffffu, mbar_wait(&s.full[slot], (t / kDqRing) & 1, prm.status));
      if (!ok) break;
      if (any) {
        for (int i = 0; i < 4; ++i) {
          const uint32_t rows = __ballot_sync(0xffffffffu, (masked >> i) & 1u);
          for (uint32_t m = rows; m; m &= m - 1) {
            const int r = (__ffs(m) - 1) + 32 * i;
            if (lane < 8) *reinterpret_cast<uint4*>(s.k[slot] + r * 128 + lane * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        fence_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        tc_fence_after();
        const uint64_t da = sdesc_sw128(smem_u32(s.ds[slot][0]), kTile, 1024);  // M chunks (64 heads) 16 KB apart
        const uint64_t db = sdesc_sw128(smem_u32(s.k[slot]), kTile, 1024);
#pragma unroll
        for (int ks = 0; ks < kTok / 16; ++ks)
          mma_bf16_ss(tmem, sdesc_add(da, ks * 2048), sdesc_add(db, ks * 2048), id, (t > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&s.empty[slot]);
      }
      __syncwarp();
    }
    if (ok && lane == 0 && n_tiles > 0) tc_commit(&s.done);
  } else {
    // ------------------------------------------------------------------ epilogue: head h = TMEM lane
    const int h = warp * 32 + lane;
    uint32_t v[32], w[32];
    bool have = false;
    if (n_tiles > 0) {
      have = __all_sync(0xffffffffu, mbar_wait(&s.done, 0, prm.status));
      if (have) {
        tc_fence_after();
        const uint32_t lb = static_cast<uint32_t>(warp * 32) << 16;
        tmem_ld32(tmem + lb, v);
        tmem_ld32(tmem + lb + 32, w);
        tmem_ld_wait(v);
      }
    }
    if (h < prm.G && (have || n_tiles == 0)) {
      const size_t row = static_cast<size_t>(b) * prm.N1 + g * prm.G + h;
      uint4* o = c < 8 ? reinterpret_cast<uint4*>(dq + row * kDQ + c * 64) : reinterpret_cast<uint4*>(dqr + row * kDR);
      const float sc = prm.scale;
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        pk[i] = have ? pack_bf16(__uint_as_float(v[2 * i]) * sc, __uint_as_float(v[2 * i + 1]) * sc) : 0u;
        pk[16 + i] = have ? pack_bf16(__uint_as_float(w[2 * i]) * sc, __uint_as_float(w[2 * i + 1]) * sc) : 0u;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) o[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 64);
}

// Readers of every cache row-block (physical page, kv head): entry e = u * cap + i (page i of unit
// u's compacted list) is counted, then listed, under key page * N2 + g.
__global__ void sfa_refs_count_kernel(const int32_t* __restrict__ pages, const int32_t* __restrict__ count, int U,
                                      int N2, int cap, int32_t* __restrict__ cnt) {
  griddep_wait();
  griddep_launch_dependents();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= U * cap) return;
  const int u = e / cap, i = e % cap;
  if (i >= count[u]) return;
  atomicAdd(&cnt[pages[e] * N2 + u % N2], 1);
}

__global__ void sfa_refs_fill_kernel(const int32_t* __restrict__ pages, const int32_t* __restrict__ count, int U,
                                     int N2, int cap, const int32_t* __restrict__ ptr, int32_t* __restrict__ cursor,
                                     int32_t* __restrict__ list) {
  griddep_wait();
  griddep_launch_dependents();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= U * cap) return;
  const int u = e / cap, i = e % cap;
  if (i >= count[u]) return;
  const int key = pages[e] * N2 + u % N2;
  list[ptr[key] + atomicAdd(&cursor[key], 1)] = e;
}

// Each key's readers in ascending entry order (insertion sort; lists are short), so the sums below
// do not depend on the order the fill's atomics ran in.
__global__ void sfa_refs_sort_kernel(const int32_t* __restrict__ ptr, int n_keys, int32_t* __restrict__ list) {
  griddep_wait();
  griddep_launch_dependents();
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n_keys) return;
  const int a = ptr[k], z = ptr[k + 1];
  for (int i = a + 1; i < z; ++i) {
    const int v = list[i];
    int j = i - 1;
    while (j >= a && list[j] > v) {
      list[j + 1] = list[j];
      --j;
    }
    list[j + 1] = v;
  }
}

// One CTA per entry; for a key with two or more readers, the first reader writes the key's rows:
// row x of the page gets the sum, over the key's readers in order, of their gathered row x
// (readers whose page has fewer tokens in use skip it), and zero where no reader has the row in
// use.  (A key with one reader was written by the backward kernel itself.)
__global__ void sfa_scatter_kernel(const int32_t* __restrict__ pages, const int32_t* __restrict__ tokens,
                                   const int32_t* __restrict__ count, int U, int N2, int cap, int page_size,
                                   const int32_t* __restrict__ ptr, const int32_t* __restrict__ list,
                                   const __nv_bfloat16* __restrict__ gk, const __nv_bfloat16* __restrict__ gv,
                                   __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dkr,
                                   __nv_bfloat16* __restrict__ dv) {
  griddep_wait();
  griddep_launch_dependents();
  const int e = blockIdx.x;
  const int u = e / cap, i = e % cap;
  if (i >= count[u]) return;
  const int g = u % N2, page = pages[e];
  const int key = page * N2 + g;
  const int a = ptr[key], z = ptr[key + 1];
  if (z - a < 2 || list[a] != e) return;  // a single reader, or not the key's first reader
  // 8 bf16 per step: 72 steps of k|k_rope and 64 of v per row
  constexpr int kStepsK = kDK / 8, kStepsV = kDQ / 8;
  for (int x = threadIdx.x; x < page_size * (kStepsK + kStepsV); x += blockDim.x) {
    const int row = x / (kStepsK + kStepsV), c = x % (kStepsK + kStepsV);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    bool any = false;
    for (int m = a; m < z; ++m) {
      const int e2 = list[m], u2 = e2 / cap, i2 = e2 % cap;
      if (row >= tokens[e2]) continue;
      any = true;
      const size_t grow = static_cast<size_t>(u2) * cap * page_size + static_cast<size_t>(i2) * page_size + row;
      const uint4 w = c < kStepsK ? reinterpret_cast<const uint4*>(gk + grow * kDK)[c]
                                  : reinterpret_cast<const uint4*>(gv + grow * kDQ)[c - kStepsK];
      acc[0] += bf16lo(w.x); acc[1] += bf16hi(w.x);
      acc[2] += bf16lo(w.y); acc[3] += bf16hi(w.y);
      acc[4] += bf16lo(w.z); acc[5] += bf16hi(w.z);
      acc[6] += bf16lo(w.w); acc[7] += bf16hi(w.w);
    }
    const uint4 o = any ? make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]), pack_bf16(acc[4], acc[5]),
                                     pack_bf16(acc[6], acc[7]))
                        : make_uint4(0u, 0u, 0u, 0u);
    const size_t crow = (static_cast<size_t>(page) * page_size + row) * N2 + g;
    if (c < kDQ / 8) reinterpret_cast<uint4*>(dk + crow * kDQ)[c] = o;
    else if (c < kStepsK) reinterpret_cast<uint4*>(dkr + crow * kDR)[c - kDQ / 8] = o;
    else reinterpret_cast<uint4*>(dv + crow * kDQ)[c - kStepsK] = o;
  }
}

}  // namespace

int sfa_bwd_tiles(int cap, int page_size) {
  const int sub = page_size % 64 == 0 ? 64 : 32;
  const int spp = page_size / sub, n_sub = kTok / sub;
  return (cap * spp + n_sub - 1) / n_sub;
}

cudaError_t sfa_bwd_launch(const SfaBwdArgs& a, cudaStream_t st) {
  const int U = a.B * a.N2, cap = a.cap, G = a.N1 / a.N2;
  const int sub = a.page_size % 64 == 0 ? 64 : 32;
  const int T = sfa_bwd_tiles(cap, a.page_size);
  const int n_keys = a.num_pages * a.N2;
  cudaError_t e = cudaSuccess;
  // page lists, their readers per cache row-block
  if ((e = sfa_page_list(a.meta, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.cnt, 0, sizeof(int32_t) * 2 * static_cast<size_t>(n_keys), st)) != cudaSuccess) return e;
  const int ne = U * cap, tb = 256;
  // (the scan times itself, so it stays outside this kernel group's timing brackets)
  prof_begin("sfa_bwd_refs", st);
  e = launch_pdl(sfa_refs_count_kernel, dim3((ne + tb - 1) / tb), dim3(tb), 0, st,
                 static_cast<const int32_t*>(a.meta.pages), static_cast<const int32_t*>(a.meta.count), U, a.N2, cap,
                 a.cnt);
  prof_end(st);
  if (e == cudaSuccess) e = exclusive_scan(a.cnt, n_keys, a.ptr, st);
  if (e != cudaSuccess) return e;
  prof_begin("sfa_bwd_refs", st);
  e = launch_pdl(sfa_refs_fill_kernel, dim3((ne + tb - 1) / tb), dim3(tb), 0, st,
                 static_cast<const int32_t*>(a.meta.pages), static_cast<const int32_t*>(a.meta.count), U, a.N2, cap,
                 static_cast<const int32_t*>(a.ptr), a.cnt + n_keys, a.list);
  if (e == cudaSuccess)
    e = launch_pdl(sfa_refs_sort_kernel, dim3((n_keys + tb - 1) / tb), dim3(tb), 0, st,
                   static_cast<const int32_t*>(a.ptr), n_keys, a.list);
  prof_end(st);
  if (e != cudaSuccess) return e;
  // preprocess
  const int rows = a.B * a.N1;
  prof_begin("sfa_bwd_prep", st);
  e = launch_pdl(sfa_bwd_prep_kernel, dim3((rows + 7) / 8), dim3(256), 0, st,
                 static_cast<const __nv_bfloat16*>(a.out), static_cast<const __nv_bfloat16*>(a.dout), a.lse, rows,
                 a.dvec, a.lse2);
  prof_end(st);
  if (e != cudaSuccess) return e;
  // the token-major products
  CUtensorMap tq, tqr, tdo, tk, tkr, tv;
  const uint64_t qrows = static_cast<uint64_t>(a.B) * a.N1;
  const uint64_t tokens = static_cast<uint64_t>(a.num_pages) * a.page_size;
  if (!make_tmap_2d_bf16(&tq, a.q, qrows, kDQ, kDQ, kTok) || !make_tmap_2d_bf16(&tqr, a.q_rope, qrows, kDR, kDR, kTok) ||
      !make_tmap_2d_bf16(&tdo, a.dout, qrows, kDQ, kDQ, kTok) ||
      !make_tmap_3d_bf16(&tk, a.k_cache, kDQ, a.N2, tokens, kDQ, static_cast<uint64_t>(a.N2) * kDQ, 1, sub) ||
      !make_tmap_3d_bf16(&tkr, a.k_rope_cache, kDR, a.N2, tokens, kDR, static_cast<uint64_t>(a.N2) * kDR, 1, sub) ||
      !make_tmap_3d_bf16(&tv, a.v_cache, kDQ, a.N2, tokens, kDQ, static_cast<uint64_t>(a.N2) * kDQ, 1, sub))
    return cudaErrorInvalidValue;
  // outputs: gathered rows [U][cap * page_size][576 | 512] bf16, dS^T [U][T * 128 tok][128 heads] bf16
  CUtensorMap tgk, tgv, tds;
  const uint64_t rows_u = static_cast<uint64_t>(cap) * a.page_size;
  if (!make_tmap_3d_bf16(&tgk, a.gk, kDK, rows_u, U, kDK, rows_u * kDK, 32, 1) ||
      !make_tmap_3d_bf16(&tgv, a.gv, kDQ, rows_u, U, kDQ, rows_u * kDQ, 32, 1) ||
      !make_tmap_3d_bf16(&tds, a.ds, 128, static_cast<uint64_t>(T) * kTok, U, 128, static_cast<uint64_t>(T) * kTok * 128,
                         kTok, 1))
    return cudaErrorInvalidValue;
  // the cache gradients, written directly for pages with one reader: boxes of 32 rows of one head
  CUtensorMap tdkc, tdkrc, tdvc;
  if (!make_tmap_3d_bf16(&tdkc, a.dk_cache, kDQ, a.N2, tokens, kDQ, static_cast<uint64_t>(a.N2) * kDQ, 1, 32) ||
      !make_tmap_3d_bf16(&tdkrc, a.dk_rope_cache, kDR, a.N2, tokens, kDR, static_cast<uint64_t>(a.N2) * kDR, 1, 32) ||
      !make_tmap_3d_bf16(&tdvc, a.dv_cache, kDQ, a.N2, tokens, kDQ, static_cast<uint64_t>(a.N2) * kDQ, 1, 32))
    return cudaErrorInvalidValue;
  BwdParams p;
  p.B = a.B; p.N1 = a.N1; p.N2 = a.N2; p.G = G; p.Gp = (G + 15) / 16 * 16; p.K = a.meta.K; p.ppb = a.meta.ppb;
  p.page_size = a.page_size; p.cap = cap; p.sub_rows = sub; p.T = T;
  p.scale = a.scale; p.scale_log2 = a.scale * kLog2e;
  p.pages = a.meta.pages; p.tokens = a.meta.tokens; p.count = a.meta.count;
  p.lse2 = a.lse2; p.dvec = a.dvec; p.rows_u = cap * a.page_size; p.status = a.meta.status; p.refs = a.cnt;
  const size_t smem = sizeof(BwdSmem) + 1024;
  if ((e = cudaFuncSetAttribute(sfa_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
    return e;
  if (T > 0 && U > 0) {
    prof_begin("sfa_bwd", st);
    e = launch_pdl(sfa_bwd_kernel, dim3(T, U), dim3(kThreads), smem, st, tq, tqr, tdo, tk, tkr, tv, tgk, tgv, tds,
                   tdkc, tdkrc, tdvc, p);
    prof_end(st);
    if (e != cudaSuccess) return e;
  }
  // dQ (9 chunks of 64 dims per unit), then the rows of pages with several readers
  const size_t dq_smem = sizeof(DqSmem) + 1024;
  if ((e = cudaFuncSetAttribute(sfa_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dq_smem)) !=
      cudaSuccess)
    return e;
  if (U > 0) {
    prof_begin("sfa_bwd_dq", st);
    e = launch_pdl(sfa_bwd_dq_kernel, dim3(kDK / 64, U), dim3(kDqThreads), dq_smem, st, tds, tk, tkr, p,
                   static_cast<__nv_bfloat16*>(a.dq), static_cast<__nv_bfloat16*>(a.dq_rope));
    prof_end(st);
    if (e != cudaSuccess) return e;
  }
  if (ne > 0) {
    prof_begin("sfa_bwd_scatter", st);
    e = launch_pdl(sfa_scatter_kernel, dim3(ne), dim3(256), 0, st, static_cast<const int32_t*>(a.meta.pages),
                   static_cast<const int32_t*>(a.meta.tokens), static_cast<const int32_t*>(a.meta.count), U, a.N2, cap,
                   a.page_size, static_cast<const int32_t*>(a.ptr), static_cast<const int32_t*>(a.list),
                   static_cast<const __nv_bfloat16*>(a.gk), static_cast<const __nv_bfloat16*>(a.gv),
                   static_cast<__nv_bfloat16*>(a.dk_cache), static_cast<__nv_bfloat16*>(a.dk_rope_cache),
                   static_cast<__nv_bfloat16*>(a.dv_cache));
    prof_end(st);
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sa
