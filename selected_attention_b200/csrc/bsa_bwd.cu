// Block-sparse attention backward on tcgen05 (BlockSparseAttentionGrad page, backward formulas):
//   softmax_grad = rowsum(dOut o Out);  dP = dOut V^T;  dS = P o (dP - softmax_grad)
//   dV = P^T dOut;  dQ = (dS K) scale;  dK = (dS^T Q) scale
// P is recomputed from the forward's LSE: P = exp(scale q.k - LSE).
//
// Operands: the passes run their products on fp16 copies of Q, K, V and dOut, each scaled by a
// power of two s_x (1 when 2^-8 <= max|x| < 2^14, else chosen so max|x| s_x <= 2^14; bf16 values have
// 8 significant bits, so the copies are exact unless a value falls below fp16's normal range); P (in [0, 1]) and dS (scaled by a power of
// two from the bound |dS| <= 256 max|dOut| max|V|) enter the gradient products as single fp16
// operands, 11 significant bits.  The scales are undone in fp32: in the exponent of P, on dP
// before dS, and in the dQ / dK / dV epilogues (all exact, being powers of two).
//
// Kernels, no atomics on the results (run-to-run bit identical):
//   bwd_to_f16   fp16 copies of Q, K, V, dOut and their max |x| (an integer atomic max on the float
//                bits: order-free); bwd_f16_fixup re-converts, scaled, a tensor whose max lies
//                outside [2^-8, 2^14), and returns at once otherwise.
//   bwd_prep     softmax_grad (D, times the dS scale) and LSE*log2(e) per query row, written into 128-row padded
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
// fp16 operand copies
// ------------------------------------------------------------------------------------------------
// The four tensors of the backward's products, blockIdx.y = 0 Q, 1 K, 2 V, 3 dOut; n8 = elements / 8.
struct F16Copy {
  const uint4* src[4];
  uint4* dst[4];
  long long n8[4];
};

__device__ __forceinline__ float bf16_pair_absmax(uint32_t w) {
  return fmaxf(fabsf(bf16lo(w)), fabsf(bf16hi(w)));
}

// Plain conversion (scale 1) of the four tensors and their max |x| in one sweep.
__global__ void bwd_to_f16_kernel(const F16Copy c, uint32_t* __restrict__ amax) {
  griddep_wait();
  griddep_launch_dependents();
  const int t = blockIdx.y;
  // selected by comparisons, not a dynamic index, so the parameter block is not copied to local memory
  const uint4* __restrict__ src = t == 0 ? c.src[0] : t == 1 ? c.src[1] : t == 2 ? c.src[2] : c.src[3];
  uint4* __restrict__ dst = t == 0 ? c.dst[0] : t == 1 ? c.dst[1] : t == 2 ? c.dst[2] : c.dst[3];
  const long long n8 = t == 0 ? c.n8[0] : t == 1 ? c.n8[1] : t == 2 ? c.n8[2] : c.n8[3];
  float m = 0.f;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 w = src[i];
    m = fmaxf(m, fmaxf(fmaxf(bf16_pair_absmax(w.x), bf16_pair_absmax(w.y)),
                       fmaxf(bf16_pair_absmax(w.z), bf16_pair_absmax(w.w))));
    uint4 o;
    o.x = pack_f16(bf16lo(w.x), bf16hi(w.x));
    o.y = pack_f16(bf16lo(w.y), bf16hi(w.y));
    o.z = pack_f16(bf16lo(w.z), bf16hi(w.z));
    o.w = pack_f16(bf16lo(w.w), bf16hi(w.w));
    dst[i] = o;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0 && m > 0.f) atomicMax(&amax[t], __float_as_uint(m));  // m >= 0: bits order as values
}

// The per-tensor scales and the factors that undo them.
struct BwdScales {
  float s[4];    // Q, K, V, dOut copy scales
  float s_ds;    // dS scale
  float c_s;     // multiplies a score accumulator: scale * log2(e) / (s_Q s_K)
  float c_dp;    // multiplies a dP accumulator: s_dS / (s_dO s_V)
  float dq_mul;  // dQ = acc * scale / (s_dS s_K)
  float dk_mul;  // dK = acc * scale / (s_dS s_Q)
  float dv_mul;  // dV = acc / s_dO
};

__device__ __forceinline__ BwdScales bwd_scales(const uint32_t* __restrict__ amax, float scale, float scale_log2) {
  BwdScales r;
  float a[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    a[t] = __uint_as_float(amax[t]);
    r.s[t] = copy_scale(a[t]);
  }
  r.s_ds = pow2_scale(256.f * a[3] * a[2]);
  r.c_s = scale_log2 / (r.s[0] * r.s[1]);
  r.c_dp = r.s_ds / (r.s[3] * r.s[2]);
  r.dq_mul = scale / (r.s_ds * r.s[1]);
  r.dk_mul = scale / (r.s_ds * r.s[0]);
  r.dv_mul = 1.f / r.s[3];
  return r;
}

// Re-conversion of a tensor whose max |x| asks for a scale other than 1 (very large or very small
// values); the whole grid returns at once otherwise.
__global__ void bwd_f16_fixup_kernel(const F16Copy c, const uint32_t* __restrict__ amax) {
  griddep_wait();  // the conversion and its maxima must be complete
  griddep_launch_dependents();
  const int t = blockIdx.y;
  const float sc = copy_scale(__uint_as_float(amax[t]));
  if (sc == 1.f) return;
  const uint4* __restrict__ src = t == 0 ? c.src[0] : t == 1 ? c.src[1] : t == 2 ? c.src[2] : c.src[3];
  uint4* __restrict__ dst = t == 0 ? c.dst[0] : t == 1 ? c.dst[1] : t == 2 ? c.dst[2] : c.dst[3];
  const long long n8 = t == 0 ? c.n8[0] : t == 1 ? c.n8[1] : t == 2 ? c.n8[2] : c.n8[3];
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 w = src[i];
    uint4 o;
    o.x = pack_f16(bf16lo(w.x) * sc, bf16hi(w.x) * sc);
    o.y = pack_f16(bf16lo(w.y) * sc, bf16hi(w.y) * sc);
    o.z = pack_f16(bf16lo(w.z) * sc, bf16hi(w.z) * sc);
    o.w = pack_f16(bf16lo(w.w) * sc, bf16hi(w.w) * sc);
    dst[i] = o;
  }
}

// ------------------------------------------------------------------------------------------------
// preprocess: -D_i = -sum_d dOut_id Out_id ; -L2_i = -LSE_i * log2(e)  (-inf where the row has no
// key or the tile row is padding, which makes exp2(s + (-L2)) = 0 there).  Stored negated so that
// P = exp2(s * scale * log2(e) + (-L2)) is one fused multiply-add and dS = P * (dP + (-D)).
// ------------------------------------------------------------------------------------------------
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                                const float* __restrict__ lse, int N1, int S_q, int bx, int nqb, long long n_rows,
                                BsaStrides qs, BsaStrides ls, const uint32_t* __restrict__ amax,
                                float* __restrict__ dvec, float* __restrict__ lse2) {
  griddep_wait();  // launched with programmatic dependent launch: the lists before it must be complete
  griddep_launch_dependents();
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
    const long long b = bh / N1, h = bh % N1;
    const size_t g = static_cast<size_t>(b * qs.b + h * qs.h + qpos * qs.s) + part * 16;
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
    // -D in the dS scale (the dP accumulators are brought to it by c_dp)
    const float s_ds = pow2_scale(256.f * __uint_as_float(amax[3]) * __uint_as_float(amax[2]));
    dvec[row] = valid ? -d * s_ds : 0.f;
    float l2 = -INFINITY;
    if (valid) {
      const long long b = bh / N1, h = bh % N1;
      const float l = lse[static_cast<size_t>(b * ls.b + h * ls.h + qpos * ls.s)];
      l2 = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
    }
    lse2[row] = l2;
  }
}

struct BwdParams {
  int B, N1, N2, S_q, S_kv, bx, by, nqb, nkb, mask_mode, win_left, win_right;
  float scale, scale_log2;
  int32_t* next_unit;      // persistent-kernel work counter, zero at launch
  int pdl_wait;            // wait for the previous grid (0: the dQ pass right after the KV pass,
                           // which it does not read: it may fill the KV pass's tail)
  const int32_t* row_ptr;  // KV lists (Q-major pass) or transposed lists (KV-major pass)
  const int32_t* col;
  const float* dvec;       // [B*N1*nqb*128]: -softmax_grad per padded query row
  const float* lse2;       // -LSE*log2(e) per padded query row (-inf: no key or padding)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  uint32_t* status;
  uint64_t* cta_clock;  // optional [grid][2] start / finish times (ns), see bsa_profile_cta_clock
  BsaStrides qs, kvs;   // element strides of dq (heads N1) and of dk / dv (heads N2)
  const uint8_t* amask; // optional dense atten_mask [S_q][S_kv], nonzero = masked out
  const uint32_t* amax; // max |x| of Q, K, V, dOut (the fp16 copies' scales)
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


// ------------------------------------------------------------------------------------------------
// KV-major pass: dK, dV.  Persistent: one CTA per SM takes KV blocks (b, g, kb) from a device
// counter (head-major, earliest block first: with causal masks those have the longest lists) and
// walks each block's transposed list.  Every entry (a 128-row Q tile of one of the group's heads)
// runs as two 64-row halves, so the element-wise work on one half overlaps the tensor-core work of
// the neighbouring halves:
//   TMEM columns: two score buffers, b = half % 2, each S^T [128b, 128b+64) | dP^T [128b+64,
//   128b+128) of one half (128 keys x 64 query rows); dV [256,384), dK [384,512).  The fp16 A
//   operands of the products are written in place: each element-wise thread, which loaded the
//   32 query columns [32h, 32h+32) of S^T and of dP^T, writes its 16 packed columns of P^T over
//   [128b+32h, +16) and of dS^T over [128b+64+32h, +16), so no thread overwrites columns another
//   thread still has to load.  The products of half x read buffer x % 2 and release it for the
//   scores of half x + 2, so those of half x + 1 are already in the other buffer when the warps
//   finish half x: the chain "warps load half x, then the scores of x + 1 start" of a single
//   score buffer is gone, and the score MMAs of x + 1 overlap the warps' work on x.
//   Each hand-off is split in two, so the critical loop (products of x -> scores of x + 2 ->
//   element-wise work on x + 2 -> its products) moves in smaller steps: the warps turn S^T into
//   P^T and store it as soon as S^T has landed (dV += P^T dO may start), then wait for dP^T and
//   write dS^T (dK += dS^T Q); S^T of half x + 2 waits only for dV of half x (which read the S^T
//   columns), dP^T of x + 2 only for dK of x.
//   Shared memory: the block's K and V tiles, and a 4-stage ring of half entries (64 rows of Q
//   and dO with their D and LSE*log2e values), so loads run two half-steps ahead.
// ------------------------------------------------------------------------------------------------
constexpr int kHalfRows = 64;
constexpr int kKvRing = 4;
constexpr int kSchedKv = 4;
// warps: 0-7 element-wise, 8 scheduler + TMA, 9 issues dV / dK products, 10 issues S^T, 11 dP^T.
// One thread issues a tcgen05.mma about every 70 clocks whatever its shape (measured: chains of
// M = 128 MMAs with N = 64 or 128 from one thread run at 70-77 clocks each, two threads together
// at 55), while an N = 64 MMA with both operands in shared memory occupies the tensor pipe ~48
// clocks: the 16 score MMAs of a half from one thread would pace the whole pass, so S^T and dP^T
// have a thread each.  The dQ pass's MMAs are N = 128 (64 clocks), and two issuers keep up there.
constexpr int kKvThreads = (kVecWarps + 3) * 32;       // the Q-major pass
constexpr int kKvPassThreads = (kVecWarps + 4) * 32;   // the KV-major pass

struct __align__(1024) KvSmem {
  uint8_t k[2][kT * 128];                 // K tile [128 keys][64 d] x 2
  uint8_t v[2][kT * 128];
  uint8_t q[kKvRing][2][kHalfRows * 128];     // [stage][d half] [64 query rows][64 d]
  uint8_t dout[kKvRing][2][kHalfRows * 128];
  float lse2[kKvRing][kHalfRows];
  float dvec[kKvRing][kHalfRows];
  int32_t sched[kSchedKv];
  uint64_t bar_kv, bar_kv_empty;
  uint64_t bar_qdo[kKvRing], bar_qdo_empty[kKvRing];
  // one of each per score buffer b (one phase per half of b): a warp may start half x + 1 before a
  // slower one has arrived for half x (never x + 2, whose scores need the products of x), so its
  // arrivals must not count toward x's phase; and a score thread may wait for the next block's K / V
  // between two halves, so its release barrier must not run two phases past it
  uint64_t bar_s_full[2];    // S^T of a half has landed in buffer b
  uint64_t bar_dp_full[2];   // dP^T of a half has landed
  uint64_t bar_p_ready[2];   // P^T written in place (256 arrivals)
  uint64_t bar_ds_ready[2];  // dS^T written in place (256 arrivals)
  uint64_t bar_dv_done[2];   // dV += P^T dO of the half has completed (the S^T columns are free)
  uint64_t bar_dk_done[2];   // dK += dS^T Q has completed (the dP^T columns are free)
  uint64_t bar_done;
  uint64_t bar_sched_full[kSchedKv], bar_sched_empty[kSchedKv];
  uint32_t tmem_base;
};

template <bool kMask>  // kMask: a dense atten_mask is applied
__global__ void __launch_bounds__(kKvPassThreads, 1)
    bsa_bwd_kv_kernel(const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do64,
                      const BwdParams prm) {
  griddep_wait();  // the D / LSE tiles of the preprocess must be complete
  griddep_launch_dependents();  // after the wait: the dQ pass then starts only once its inputs exist
  if (prm.cta_clock && threadIdx.x == 0) prm.cta_clock[2 * blockIdx.x] = globaltimer_ns();
  const BwdScales sc = bwd_scales(prm.amax, prm.scale, prm.scale_log2);
  constexpr uint32_t kColBuf = 128, kColDP = 64, kColDV = 256, kColDK = 384;
  extern __shared__ uint8_t smem_raw[];
  KvSmem& s = *reinterpret_cast<KvSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = prm.N1 / prm.N2;
  const int units = prm.B * prm.N2 * prm.nkb;

  if (tid == 0) {
    mbar_init(&s.bar_kv, 1);
    mbar_init(&s.bar_kv_empty, 2);  // the block's last S^T and last dP^T
    for (int i = 0; i < kKvRing; ++i) {
      mbar_init(&s.bar_qdo[i], 1);
      mbar_init(&s.bar_qdo_empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s.bar_s_full[b], 1);
      mbar_init(&s.bar_dp_full[b], 1);
      mbar_init(&s.bar_p_ready[b], kVecWarps * 32);
      mbar_init(&s.bar_ds_ready[b], kVecWarps * 32);
      mbar_init(&s.bar_dv_done[b], 1);
      mbar_init(&s.bar_dk_done[b], 1);
    }
    mbar_init(&s.bar_done, 1);
    for (int i = 0; i < kSchedKv; ++i) {
      mbar_init(&s.bar_sched_full[i], 1);
      mbar_init(&s.bar_sched_empty[i], 3 + kVecWarps * 32);
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

  // Schedule number i -> (b*N2 + g, kv block), its transposed list [rp, rp + n).  The first
  // kLead KV blocks of every (b, g) come first, interleaved across heads (under causal selection
  // the earliest blocks are selected by the most q blocks: the longest lists, a sink block by all
  // of them), then each head's remaining blocks in order, so no long list starts near the end.
  auto unit_of = [&](int i, int& bg, int& kb, int& rp, int& n) {
    constexpr int kLead = 16;
    const int bgs = prm.B * prm.N2, lead = min(prm.nkb, kLead);
    if (i < bgs * lead) {
      kb = i / bgs;
      bg = i % bgs;
    } else {
      const int j = i - bgs * lead, rest = prm.nkb - lead;
      bg = j / rest;
      kb = lead + j % rest;
    }
    const int unit = bg * prm.nkb + kb;
    rp = prm.row_ptr[unit];
    n = prm.row_ptr[unit + 1] - rp;
  };
  // list entry -> its query head, its padded tile index and the position of its first query row
  auto entry_rows = [&](int bg, int e_code, int& qh, int& tile, int& qpos0) {
    const int b = bg / prm.N2, g = bg % prm.N2;
    const int hl = e_code / prm.nqb, qb = e_code % prm.nqb;
    qh = g * G + hl;
    tile = (b * prm.N1 + qh) * prm.nqb + qb;
    qpos0 = qb * prm.bx;
  };
  auto next_from_ring = [&](int k) -> int {
    const int slot = k % kSchedKv;
    if (!mbar_wait(&s.bar_sched_full[slot], (k / kSchedKv) & 1, prm.status)) return -1;
    const int u = *reinterpret_cast<volatile int32_t*>(&s.sched[slot]);
    mbar_arrive(&s.bar_sched_empty[slot]);
    return u;
  };

  if (warp == kVecWarps) {
    // ------------------------------------------------------------------ scheduler + TMA producer
    if (lane == 0) {
      int hq = 0, ucount = 0;  // half entries loaded, K/V loads (this CTA)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % kSchedKv;
        if (k >= kSchedKv && !(ok = mbar_wait(&s.bar_sched_empty[slot], ((k / kSchedKv) - 1) & 1, prm.status)))
          break;
        int i = atomicAdd(prm.next_unit, 1);
        if (i >= units) i = -1;
        s.sched[slot] = i;
        mbar_arrive(&s.bar_sched_full[slot]);
        if (i < 0) break;
        int bg, kb, rp, n;
        unit_of(i, bg, kb, rp, n);
        if (n == 0) continue;
        const int b = bg / prm.N2, g = bg % prm.N2, kpos0 = kb * prm.by;
        if (ucount > 0 && !(ok = mbar_wait(&s.bar_kv_empty, (ucount - 1) & 1, prm.status))) break;
        mbar_arrive_expect_tx(&s.bar_kv, 4 * kT * 128);
        tma_load_4d(s.k[0], &tm_k, &s.bar_kv, 0, g, kpos0, b);
        tma_load_4d(s.k[1], &tm_k, &s.bar_kv, 64, g, kpos0, b);
        tma_load_4d(s.v[0], &tm_v, &s.bar_kv, 0, g, kpos0, b);
        tma_load_4d(s.v[1], &tm_v, &s.bar_kv, 64, g, kpos0, b);
        ++ucount;
        for (int e = 0; ok && e < 2 * n; ++e) {
          const int h = e & 1;
          int qh, tile, qpos0;  // the entry's query head (hq counts the half entries loaded)
          entry_rows(bg, prm.col[rp + (e >> 1)], qh, tile, qpos0);
          const int hs = hq % kKvRing;
          if (hq >= kKvRing && !(ok = mbar_wait(&s.bar_qdo_empty[hs], ((hq / kKvRing) - 1) & 1, prm.status))) break;
          mbar_arrive_expect_tx(&s.bar_qdo[hs], 4 * kHalfRows * 128 + 2 * kHalfRows * 4);
          const int qp = qpos0 + h * kHalfRows;
          tma_load_4d(s.q[hs][0], &tm_q64, &s.bar_qdo[hs], 0, qh, qp, b);
          tma_load_4d(s.q[hs][1], &tm_q64, &s.bar_qdo[hs], 64, qh, qp, b);
          tma_load_4d(s.dout[hs][0], &tm_do64, &s.bar_qdo[hs], 0, qh, qp, b);
          tma_load_4d(s.dout[hs][1], &tm_do64, &s.bar_qdo[hs], 64, qh, qp, b);
          const size_t voff = static_cast<size_t>(tile) * kT + h * kHalfRows;
          bulk_load(s.lse2[hs], prm.lse2 + voff, kHalfRows * 4, &s.bar_qdo[hs]);
          bulk_load(s.dvec[hs], prm.dvec + voff, kHalfRows * 4, &s.bar_qdo[hs]);
          ++hq;
        }
      }
      // do not leave the CTA with copies in flight
      for (int j = (hq > kKvRing ? hq - kKvRing : 0); j < hq; ++j)
        mbar_wait(&s.bar_qdo[j % kKvRing], (j / kKvRing) & 1, prm.status);
      if (ucount > 0) mbar_wait(&s.bar_kv, (ucount - 1) & 1, prm.status);
    }
  } else if (warp >= kVecWarps + 1) {
    // ------------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const bool grads_thread = warp == kVecWarps + 1;
      const bool dp_thread = warp == kVecWarps + 3;  // else S^T
      const uint32_t id_sdp = idesc_f16_f32(kT, kHalfRows, false, false);  // S^T, dP^T of a half
      const uint32_t id_mnb = idesc_f16_f32(kT, kD, false, true);          // dV, dK (B = [queries][d])
      int G0 = 0, ucount = 0;
      bool ok = true;
      // descriptors of stage 0 / sub-tile 0; stages, sub-tiles and K steps are added offsets
      const uint64_t dk0 = sdesc_sw128(smem_u32(s.k[0]), 0, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(s.v[0]), 0, 1024);
      const uint64_t dq0 = sdesc_sw128(smem_u32(s.q[0][0]), 0, 1024);
      const uint64_t ddo0 = sdesc_sw128(smem_u32(s.dout[0][0]), 0, 1024);
      const uint64_t dqm0 = sdesc_sw128(smem_u32(s.q[0][0]), kHalfRows * 128, 1024);      // MN-major
      const uint64_t ddom0 = sdesc_sw128(smem_u32(s.dout[0][0]), kHalfRows * 128, 1024);
      constexpr uint32_t kStage16 = (2 * kHalfRows * 128) >> 4;  // one ring stage, in 16-byte units
      // S^T = K Q_h^T (the S^T thread) or dP^T = V dO_h^T (the dP^T thread) of global half hx into
      // score buffer hx % 2
      const uint64_t da0 = dp_thread ? dv0 : dk0, db0 = dp_thread ? ddo0 : dq0;
      const uint32_t dcol = dp_thread ? kColDP : 0u;
      auto sdp = [&](int hx) -> bool {
        const int hs = hx % kKvRing;
        if (!mbar_wait(&s.bar_qdo[hs], (hx / kKvRing) & 1, prm.status)) return false;
        tc_fence_after();
        const uint32_t d = tmem + (hx & 1) * kColBuf + dcol;
        const uint64_t db = db0 + static_cast<uint64_t>(hs) * kStage16;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t ko = (ks >> 2) * (kT * 128) + (ks & 3) * 32, qo = (ks >> 2) * (kHalfRows * 128) + (ks & 3) * 32;
          mma_bf16_ss(d, sdesc_add(da0, ko), sdesc_add(db, qo), id_sdp, ks > 0 ? 1u : 0u);
        }
        tc_commit(dp_thread ? &s.bar_dp_full[hx & 1] : &s.bar_s_full[hx & 1]);
        return true;
      };
      // acc += A (TMEM, 128 keys x 64 query rows) . B (the half's [64 rows][128 d], MN-major).  A's
      // query rows 16 ks .. 16 ks + 15 sit in columns a_col + 8 (ks & 1) + 32 (ks >> 1): the 16
      // packed columns of query rows [0,32) start at a_col, those of [32,64) at a_col + 32.
      auto grad = [&](uint32_t d, uint32_t a_col, uint64_t bdesc, bool acc) {
#pragma unroll
        for (int ks = 0; ks < kHalfRows / 16; ++ks)
          mma_bf16_ts(d, tmem + a_col + (ks & 1) * 8 + (ks >> 1) * 32, sdesc_add(bdesc, ks * 2048), id_mnb,
                      (acc || ks > 0) ? 1u : 0u);
      };
      for (int k = 0; ok; ++k) {
        const int i = next_from_ring(k);
        if (i < 0) break;
        int bg, kb, rp, n;
        unit_of(i, bg, kb, rp, n);
        if (n == 0) continue;
        const int nh = 2 * n;
        if (grads_thread) {
          // dV += P^T dO and dK += dS^T Q as soon as the element-wise warps have a half
          for (int x = 0; ok && x < nh; ++x) {
            const int hx = G0 + x, hs = hx % kKvRing;
            // exact parity: the next phase of p_ready[hx % 2] needs the warps' P of half hx + 2,
            // whose S^T waits for the dV product of half hx, issued after this wait (the same for
            // ds_ready, dP^T and dK)
            const uint32_t buf = (hx & 1) * kColBuf;
            if (!(ok = mbar_wait(&s.bar_p_ready[hx & 1], (hx >> 1) & 1, prm.status))) break;
            tc_fence_after();
            grad(tmem + kColDV, buf, ddom0 + static_cast<uint64_t>(hs) * kStage16, x > 0);  // dV += P^T dO
            tc_commit(&s.bar_dv_done[hx & 1]);
            if (!(ok = mbar_wait(&s.bar_ds_ready[hx & 1], (hx >> 1) & 1, prm.status))) break;
            tc_fence_after();
            grad(tmem + kColDK, buf + kColDP, dqm0 + static_cast<uint64_t>(hs) * kStage16, x > 0);  // dK += dS^T Q
            tc_commit(&s.bar_qdo_empty[hs]);
            tc_commit(&s.bar_dk_done[hx & 1]);
          }
          if (ok) tc_commit(&s.bar_done);
        } else {
          // S^T (dP^T) of each half once the dV (dK) product of half hx - 2 has released its
          // columns of the score buffer.  Exact parity: the next phase of dv_done[hx % 2] (dV of
          // half hx) needs the scores this thread issues after the wait.
          if (!(ok = mbar_wait(&s.bar_kv, ucount & 1, prm.status))) break;
          ++ucount;
          for (int x = 0; ok && x < nh; ++x) {
            const int hx = G0 + x;
            if (hx >= 2 && !(ok = mbar_wait(dp_thread ? &s.bar_dk_done[hx & 1] : &s.bar_dv_done[hx & 1],
                                            ((hx - 2) >> 1) & 1, prm.status)))
              break;
            if (!(ok = sdp(hx))) break;
            if (x + 1 == nh) tc_commit(&s.bar_kv_empty);  // the block's last read of K (or V)
          }
        }
        G0 += nh;
      }
    }
  } else {
    // ------------------------------------------------------------------ P / dS warps
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // key row within the KV tile == TMEM lane
    const int c0 = hf * 32;             // this thread's query columns [c0, c0 + 32) of a half
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int shift = prm.S_kv - prm.S_q;
    int G0 = 0, done_count = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int i = __shfl_sync(0xffffffffu, next_from_ring(k), 0);
      if (i < 0) break;
      int bg, kb, rp, n;
      unit_of(i, bg, kb, rp, n);
      const int kpos = kb * prm.by + r;
      const bool key_valid = r < prm.by && kpos < prm.S_kv;
      // query positions that see this key: [qlo, qhi]
      int qlo = -0x40000000, qhi = 0x3fffffff;
      if (prm.mask_mode == 2) qlo = kpos;
      else if (prm.mask_mode == 3) qlo = kpos - shift;
      else if (prm.mask_mode == 4) { qlo = kpos - shift - prm.win_right; qhi = kpos - shift + prm.win_left; }
      if (!key_valid) { qlo = 1; qhi = 0; }
      // the list entry of the next half is read one half ahead: a global load on this loop's
      // critical path otherwise (~350 clocks per half)
      int code_next = n > 0 ? prm.col[rp] : 0;
      for (int x = 0; x < 2 * n; ++x) {
        const int hx = G0 + x, hs = hx % kKvRing;
        const int code = code_next;
        if (x + 1 < 2 * n) code_next = prm.col[rp + ((x + 1) >> 1)];
        int qh, tile, qpos0;
        entry_rows(bg, code, qh, tile, qpos0);
        const int qp0 = qpos0 + (x & 1) * kHalfRows + c0;  // query position of column c0
        // exact parity: the next phase of s_full[hx % 2] (S^T of half hx + 2) waits for the dV
        // product of half hx, which needs the p_ready arrival below (the same for dp_full)
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_qdo[hs], (hx / kKvRing) & 1, prm.status) &&
                                         mbar_wait(&s.bar_s_full[hx & 1], (hx >> 1) & 1, prm.status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t buf = tmem + lane_base + (hx & 1) * kColBuf + c0;  // this thread's S^T columns
        uint32_t sr[32], dr[32];
        tmem_ld32(buf, sr);
        tmem_ld_wait(sr);
        const float4* nl2 = reinterpret_cast<const float4*>(s.lse2[hs] + c0);  // -LSE*log2e per query row
        const float4* nd = reinterpret_cast<const float4*>(s.dvec[hs] + c0);   // -D s_dS per query row
        const uint64_t sc2 = f2_pack(sc.c_s, sc.c_s), cdp2 = f2_pack(sc.c_dp, sc.c_dp);
        // the dense atten_mask: bit c set when query column c of the chunk may not see this key
        uint32_t mbits = 0;
        if (kMask && key_valid) {
#pragma unroll 4
          for (int c = 0; c < 32; ++c) {
            const int qp = qp0 + c;
            if (qp < prm.S_q && prm.amask[static_cast<size_t>(qp) * prm.S_kv + kpos] != 0) mbits |= 1u << c;
          }
        }
        const bool full = qp0 >= qlo && qp0 + 31 <= qhi && mbits == 0;
        uint32_t ph[16], dh[16];
        // P = exp2(S c_s - LSE log2e), kept in fp32 (over the scores) for dS
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 L = nl2[c4];
#pragma unroll
          for (int hp = 0; hp < 2; ++hp) {
            const int c = c4 * 4 + hp * 2;
            float t0, t1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2,
                             hp ? f2_pack(L.z, L.w) : f2_pack(L.x, L.y)),
                      t0, t1);
            float p0 = ex2(t0), p1 = ex2(t1);
            if (!full) {
              if (qp0 + c < qlo || qp0 + c > qhi || ((mbits >> c) & 1u)) p0 = 0.f;
              if (qp0 + c + 1 < qlo || qp0 + c + 1 > qhi || ((mbits >> (c + 1)) & 1u)) p1 = 0.f;
            }
            sr[c] = __float_as_uint(p0);
            sr[c + 1] = __float_as_uint(p1);
            ph[c / 2] = pack_f16(p0, p1);
          }
        }
        // in place, over the first 16 of the 32 S^T columns this thread loaded
        tmem_st16(buf, ph);  // P^T
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&s.bar_p_ready[hx & 1]);
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_dp_full[hx & 1], (hx >> 1) & 1, prm.status));
        if (!ok) break;
        tc_fence_after();
        tmem_ld32(buf + kColDP, dr);
        tmem_ld_wait(dr);
        // dS (in its fp16 scale) = P (dP c_dp - D s_dS)
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 Dn = nd[c4];
#pragma unroll
          for (int hp = 0; hp < 2; ++hp) {
            const int c = c4 * 4 + hp * 2;
            float g0, g1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                             f2_fma(f2_pack(__uint_as_float(dr[c]), __uint_as_float(dr[c + 1])), cdp2,
                                    hp ? f2_pack(Dn.z, Dn.w) : f2_pack(Dn.x, Dn.y))),
                      g0, g1);
            dh[c / 2] = pack_f16(g0, g1);
          }
        }
        tmem_st16(buf + kColDP, dh);  // dS^T, over the first 16 of this thread's dP^T columns
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&s.bar_ds_ready[hx & 1]);
      }
      if (!ok) break;
      // ---- epilogue: dK = scale * acc, dV = acc (this thread: head-dim columns [hf*64, +64))
      bool have = n > 0;
      if (have) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_done, done_count & 1, prm.status));
        ++done_count;
        if (!ok) break;
        tc_fence_after();
      }
      const size_t krow = static_cast<size_t>((bg / prm.N2) * prm.kvs.b + (bg % prm.N2) * prm.kvs.h +
                                              static_cast<long long>(kb * prm.by + r) * prm.kvs.s);
      __nv_bfloat16* dkrow = prm.dk + krow + hf * 64;
      __nv_bfloat16* dvrow = prm.dv + krow + hf * 64;
#pragma unroll
      for (int c = 0; c < kD / 2; c += 32) {
        uint32_t rk[32], rv[32];
        if (have) {
          tmem_ld32(tmem + lane_base + kColDK + hf * 64 + c, rk);
          tmem_ld32(tmem + lane_base + kColDV + hf * 64 + c, rv);
          tmem_ld_wait(rk);
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) reg_fence(rv[i2]);
        } else {
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) rk[i2] = rv[i2] = 0u;
        }
        if (key_valid) {
          store_row_bf16(dkrow + c, rk, sc.dk_mul);
          store_row_bf16(dvrow + c, rv, sc.dv_mul);
        }
      }
      // dK / dV have been read: the next block's first products wait for its P / dS, which come
      // after this
      tc_fence_before();
      G0 += 2 * n;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
  if (prm.cta_clock && threadIdx.x == 0) prm.cta_clock[2 * blockIdx.x + 1] = globaltimer_ns();
}

// ------------------------------------------------------------------------------------------------
// Q-major pass: dQ
// TMEM columns: S0 [0,BN) | S1 [BN,2BN) | dP [2BN,3BN) | dQ [3BN, 3BN+128).
// dS for tile j is written back as packed bf16 over the S_j columns its warp has read: the warp of
// key half h (columns [h*BN/2, +BN/2)) puts dS hi of its keys at [h*BN/2, +BN/4) and lo at
// [h*BN/2 + BN/4, +BN/4); these are the A operands of dQ += dS K (one MMA per 16 keys, so the A
// columns of each K step are addressed individually).
// ------------------------------------------------------------------------------------------------
constexpr int kQKStages = 3, kQVStages = 2;  // K is held by S and dQ, V only by dP

template <int BN>
struct __align__(1024) QSmem {
  uint8_t q[2][kT * 128];
  uint8_t dout[2][kT * 128];
  uint8_t k[kQKStages][2][BN * 128];  // [stage][sub-tile] [BN keys][64 d]
  uint8_t v[kQVStages][2][BN * 128];
  int32_t sched[kSchedKv];
  uint64_t bar_qdo, bar_qdo_empty, bar_k[kQKStages], bar_k_empty[kQKStages], bar_v[kQVStages], bar_v_empty[kQVStages];
  uint64_t bar_s_full[2], bar_dp_full, bar_ds_ready[2], bar_dq_done[2], bar_done;
  uint64_t bar_dp_free;  // the element-wise warps have loaded dP of the current tile (256 arrivals)
  uint64_t bar_sched_full[kSchedKv], bar_sched_empty[kSchedKv];
  uint32_t tmem_base;
};

// Persistent: one CTA per SM takes Q tiles (b, h, qb) from a device counter (head-major, latest
// q block first).  Warps: 0-7 element-wise, 8 scheduler + TMA, 9 issues dQ += dS K (hi, lo),
// 10 issues S = Q K^T and dP = dO V^T.  Per-buffer barriers (ds_ready, dq_done per S buffer) keep
// every parity wait exact with two issuing threads.
template <int BN, bool kMask>  // kMask: a dense atten_mask is applied
__global__ void __launch_bounds__(kKvThreads, 1)
    bsa_bwd_q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BwdParams prm) {
  if (prm.pdl_wait) griddep_wait();
  griddep_launch_dependents();
  if (prm.cta_clock && threadIdx.x == 0) prm.cta_clock[2 * blockIdx.x] = globaltimer_ns();
  const BwdScales sc = bwd_scales(prm.amax, prm.scale, prm.scale_log2);
  constexpr uint32_t kColS0 = 0, kColS1 = BN, kColDP = 2 * BN, kColDQ = 3 * BN;
  extern __shared__ uint8_t smem_raw[];
  QSmem<BN>& s = *reinterpret_cast<QSmem<BN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int units = prm.B * prm.N1 * prm.nqb;

  if (tid == 0) {
    mbar_init(&s.bar_qdo, 1);
    mbar_init(&s.bar_qdo_empty, 1);
    for (int i = 0; i < kQKStages; ++i) {
      mbar_init(&s.bar_k[i], 1);
      mbar_init(&s.bar_k_empty[i], 1);
    }
    for (int i = 0; i < kQVStages; ++i) {
      mbar_init(&s.bar_v[i], 1);
      mbar_init(&s.bar_v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.bar_s_full[i], 1);
      mbar_init(&s.bar_ds_ready[i], kVecWarps * 32);
      mbar_init(&s.bar_dq_done[i], 1);
    }
    mbar_init(&s.bar_dp_full, 1);
    mbar_init(&s.bar_dp_free, kVecWarps * 32);
    mbar_init(&s.bar_done, 1);
    for (int i = 0; i < kSchedKv; ++i) {
      mbar_init(&s.bar_sched_full[i], 1);
      mbar_init(&s.bar_sched_empty[i], 2 + kVecWarps * 32);
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

  // schedule number i -> (b*N1 + h, q block), its KV list [rp, rp + n)
  auto unit_of = [&](int i, int& bh, int& qb, int& rp, int& n) {
    bh = i / prm.nqb;
    qb = prm.nqb - 1 - i % prm.nqb;
    const int unit = bh * prm.nqb + qb;
    rp = prm.row_ptr[unit];
    n = prm.row_ptr[unit + 1] - rp;
  };
  auto next_from_ring = [&](int k) -> int {
    const int slot = k % kSchedKv;
    if (!mbar_wait(&s.bar_sched_full[slot], (k / kSchedKv) & 1, prm.status)) return -1;
    const int u = *reinterpret_cast<volatile int32_t*>(&s.sched[slot]);
    mbar_arrive(&s.bar_sched_empty[slot]);
    return u;
  };

  if (warp == kVecWarps) {
    // ------------------------------------------------------------------ scheduler + TMA producer
    if (lane == 0) {
      int jk = 0, jv = 0, ucount = 0;
      bool ok = true;
      auto load_v = [&](int rp, int b, int g, int j) -> bool {
        const int sv = jv % kQVStages, uv = jv / kQVStages;
        if (jv >= kQVStages && !mbar_wait(&s.bar_v_empty[sv], (uv - 1) & 1, prm.status)) return false;
        const int vpos = prm.col[rp + j] * prm.by;
        mbar_arrive_expect_tx(&s.bar_v[sv], 2 * BN * 128);
        tma_load_4d(s.v[sv][0], &tm_v, &s.bar_v[sv], 0, g, vpos, b);
        tma_load_4d(s.v[sv][1], &tm_v, &s.bar_v[sv], 64, g, vpos, b);
        ++jv;
        return true;
      };
      for (int k = 0; ok; ++k) {
        const int slot = k % kSchedKv;
        if (k >= kSchedKv && !(ok = mbar_wait(&s.bar_sched_empty[slot], ((k / kSchedKv) - 1) & 1, prm.status)))
          break;
        int i = atomicAdd(prm.next_unit, 1);
        if (i >= units) i = -1;
        s.sched[slot] = i;
        mbar_arrive(&s.bar_sched_full[slot]);
        if (i < 0) break;
        int bh, qb, rp, n;
        unit_of(i, bh, qb, rp, n);
        if (n == 0) continue;
        const int b = bh / prm.N1, g = (bh % prm.N1) / (prm.N1 / prm.N2);
        const int h = bh % prm.N1, q_pos0 = qb * prm.bx;
        if (ucount > 0 && !(ok = mbar_wait(&s.bar_qdo_empty, (ucount - 1) & 1, prm.status))) break;
        mbar_arrive_expect_tx(&s.bar_qdo, 4 * kT * 128);
        tma_load_4d(s.q[0], &tm_q, &s.bar_qdo, 0, h, q_pos0, b);
        tma_load_4d(s.q[1], &tm_q, &s.bar_qdo, 64, h, q_pos0, b);
        tma_load_4d(s.dout[0], &tm_do, &s.bar_qdo, 0, h, q_pos0, b);
        tma_load_4d(s.dout[1], &tm_do, &s.bar_qdo, 64, h, q_pos0, b);
        ++ucount;
        for (int j = 0; ok && j < n; ++j) {
          const int sk = jk % kQKStages, uk = jk / kQKStages;
          if (jk >= kQKStages && !(ok = mbar_wait(&s.bar_k_empty[sk], (uk - 1) & 1, prm.status))) break;
          const int kpos = prm.col[rp + j] * prm.by;
          mbar_arrive_expect_tx(&s.bar_k[sk], 2 * BN * 128);
          tma_load_4d(s.k[sk][0], &tm_k, &s.bar_k[sk], 0, g, kpos, b);
          tma_load_4d(s.k[sk][1], &tm_k, &s.bar_k[sk], 64, g, kpos, b);
          ++jk;
          if (j >= kQKStages - kQVStages) ok = load_v(rp, b, g, j - (kQKStages - kQVStages));  // V trails K
        }
        for (int j = n - (kQKStages - kQVStages); ok && j < n; ++j)
          if (j >= 0) ok = load_v(rp, b, g, j);
      }
      // do not leave the CTA with copies in flight
      for (int j = (jk > kQKStages ? jk - kQKStages : 0); j < jk; ++j)
        mbar_wait(&s.bar_k[j % kQKStages], (j / kQKStages) & 1, prm.status);
      for (int j = (jv > kQVStages ? jv - kQVStages : 0); j < jv; ++j)
        mbar_wait(&s.bar_v[j % kQVStages], (j / kQVStages) & 1, prm.status);
      if (ucount > 0) mbar_wait(&s.bar_qdo, (ucount - 1) & 1, prm.status);
    }
  } else if (warp == kVecWarps + 1 || warp == kVecWarps + 2) {
    // ------------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const bool dq_thread = warp == kVecWarps + 1;
      const uint32_t id_s = idesc_f16_f32(kT, BN, false, false);
      const uint32_t id_dq = idesc_f16_f32(kT, kD, false, true);
      // descriptors of stage 0 / sub-tile 0; stages, sub-tiles and K steps are added offsets
      const uint64_t dq0 = sdesc_sw128(smem_u32(s.q[0]), 0, 1024);
      const uint64_t ddo0 = sdesc_sw128(smem_u32(s.dout[0]), 0, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(s.k[0][0]), 0, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(s.v[0][0]), 0, 1024);
      const uint64_t dkm0 = sdesc_sw128(smem_u32(s.k[0][0]), BN * 128, 1024);  // K as MN-major B of dQ
      constexpr uint32_t kKv16 = (2 * BN * 128) >> 4;  // one K or V stage, in 16-byte units
      int J0 = 0, ucount = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int i = next_from_ring(k);
        if (i < 0) break;
        int bh, qb, rp, n;
        unit_of(i, bh, qb, rp, n);
        if (n == 0) continue;
        if (dq_thread) {
          for (int j = 0; ok && j < n; ++j) {
            const int J = J0 + j, st = J & 1, sk = J % kQKStages;
            if (!(ok = mbar_wait(&s.bar_ds_ready[st], (J >> 1) & 1, prm.status))) break;
            tc_fence_after();
            const uint32_t s_col = st ? kColS1 : kColS0;
            const uint64_t dkm = dkm0 + static_cast<uint64_t>(sk) * kKv16;
            constexpr int kStepsPerHalf = BN / 32;  // 16-key K steps in a warp's key half
#pragma unroll
#pragma unroll
            for (int ks = 0; ks < BN / 16; ++ks) {
              const uint32_t a_col = s_col + (ks / kStepsPerHalf) * (BN / 2) + (ks % kStepsPerHalf) * 8;
              mma_bf16_ts(tmem + kColDQ, tmem + a_col, sdesc_add(dkm, ks * 2048), id_dq, (j > 0 || ks > 0) ? 1u : 0u);
            }
            tc_commit(&s.bar_k_empty[sk]);
            tc_commit(&s.bar_dq_done[st]);
          }
          if (ok) tc_commit(&s.bar_done);
        } else {
          if (!(ok = mbar_wait(&s.bar_qdo, ucount & 1, prm.status))) break;
          ++ucount;
          for (int j = 0; ok && j < n; ++j) {
            const int J = J0 + j, st = J & 1, sk = J % kQKStages, sv = J % kQVStages;
            // S buffer st last held dS_{J-2}, read by dQ_{J-2}
            if (J >= 2 && !(ok = mbar_wait(&s.bar_dq_done[st], ((J >> 1) - 1) & 1, prm.status))) break;
            if (!(ok = mbar_wait(&s.bar_k[sk], (J / kQKStages) & 1, prm.status))) break;
            tc_fence_after();
            const uint64_t dk = dk0 + static_cast<uint64_t>(sk) * kKv16;
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks)
              mma_bf16_ss(tmem + (st ? kColS1 : kColS0), sdesc_add(dq0, (ks >> 2) * (kT * 128) + (ks & 3) * 32),
                          sdesc_add(dk, (ks >> 2) * (BN * 128) + (ks & 3) * 32), id_s, ks > 0 ? 1u : 0u);
            tc_commit(&s.bar_s_full[st]);
            // dP has one buffer: the warps have loaded dP_{J-1} (exact parity: the next phase of
            // dp_free needs dP_J, issued after the wait)
            if (J >= 1 && !(ok = mbar_wait(&s.bar_dp_free, (J - 1) & 1, prm.status))) break;
            if (!(ok = mbar_wait(&s.bar_v[sv], (J / kQVStages) & 1, prm.status))) break;
            tc_fence_after();
            const uint64_t dv = dv0 + static_cast<uint64_t>(sv) * kKv16;
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks)
              mma_bf16_ss(tmem + kColDP, sdesc_add(ddo0, (ks >> 2) * (kT * 128) + (ks & 3) * 32),
                          sdesc_add(dv, (ks >> 2) * (BN * 128) + (ks & 3) * 32), id_s, ks > 0 ? 1u : 0u);
            tc_commit(&s.bar_dp_full);
            tc_commit(&s.bar_v_empty[sv]);
            if (j + 1 == n) tc_commit(&s.bar_qdo_empty);  // the unit's last read of Q and dO
          }
        }
        J0 += n;
      }
    }
  } else {
    // ------------------------------------------------------------------ P / dS warps
    constexpr int kHalf = BN / 2;
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // query row == TMEM lane
    const int c0 = hf * kHalf;          // this thread's key columns [c0, c0 + BN/2)
    const uint64_t sc2 = f2_pack(sc.c_s, sc.c_s), cdp2 = f2_pack(sc.c_dp, sc.c_dp);
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int J0 = 0, done_count = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int i = __shfl_sync(0xffffffffu, next_from_ring(k), 0);
      if (i < 0) break;
      int bh, qb, rp, n;
      unit_of(i, bh, qb, rp, n);
      const int qpos = qb * prm.bx + r;
      const bool row_valid = r < prm.bx && qpos < prm.S_q;
      int lo = 0, hi = prm.S_kv - 1;
      const int qq = qpos + prm.S_kv - prm.S_q;
      if (prm.mask_mode == 2) hi = min(hi, qpos);
      else if (prm.mask_mode == 3) hi = min(hi, qq);
      else if (prm.mask_mode == 4) { lo = qq - prm.win_left; hi = min(hi, qq + prm.win_right); }
      if (!row_valid) { lo = 1; hi = 0; }
      const size_t trow = static_cast<size_t>(bh * prm.nqb + qb) * kT + r;
      const uint64_t nl2 = f2_pack(prm.lse2[trow], prm.lse2[trow]);  // -LSE*log2e of the row, twice
      const uint64_t nd2 = f2_pack(prm.dvec[trow], prm.dvec[trow]);  // -D s_dS of the row, twice
      int col_next = n > 0 ? prm.col[rp] : 0;  // read one tile ahead, before the wait
      for (int j = 0; j < n; ++j) {
        const int J = J0 + j, st = J & 1;
        const uint32_t s_col = st ? kColS1 : kColS0;
        const int cj = col_next;
        if (j + 1 < n) col_next = prm.col[rp + j + 1];
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_s_full[st], (J >> 1) & 1, prm.status));
        if (!ok) break;
        tc_fence_after();
        const int kpos0 = cj * prm.by + c0;
        const bool full = kpos0 >= lo && kpos0 + kHalf - 1 <= hi;
        float p[kHalf];
#pragma unroll
        for (int c = 0; c < kHalf; c += 32) {
          uint32_t rr[32];
          tmem_ld32(tmem + lane_base + s_col + c0 + c, rr);
          tmem_ld_wait(rr);
#pragma unroll
          for (int i2 = 0; i2 < 32; i2 += 2) {
            float t0, t1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(rr[i2]), __uint_as_float(rr[i2 + 1])), sc2, nl2), t0, t1);
            p[c + i2] = ex2(t0);
            p[c + i2 + 1] = ex2(t1);
          }
        }
        if (!full) {
#pragma unroll
          for (int c = 0; c < kHalf; ++c) {
            const int kp = kpos0 + c;
            if (kp < lo || kp > hi) p[c] = 0.f;
          }
        }
        if (kMask && row_valid) {
          // the dense atten_mask inside the selected block: this row's bytes of the tile's columns
          const uint64_t mbits =
              dense_mask_bits<kHalf>(prm.amask + static_cast<size_t>(qpos) * prm.S_kv, kpos0, prm.S_kv);
#pragma unroll
          for (int c = 0; c < kHalf; ++c)
            if ((mbits >> c) & 1ull) p[c] = 0.f;
        }
        // dp_full has one phase per tile; its next phase needs the dp_free arrival below
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_dp_full, J & 1, prm.status));
        if (!ok) break;
        tc_fence_after();
        uint32_t hv[kHalf / 2];
#pragma unroll
        for (int c = 0; c < kHalf; c += 32) {
          uint32_t rr[32];
          tmem_ld32(tmem + lane_base + kColDP + c0 + c, rr);
          tmem_ld_wait(rr);
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2) {
            // dS (in its fp16 scale) = P (dP c_dp - D s_dS)
            float g0, g1;
            f2_unpack(f2_mul(f2_pack(p[c + 2 * i2], p[c + 2 * i2 + 1]),
                             f2_fma(f2_pack(__uint_as_float(rr[2 * i2]), __uint_as_float(rr[2 * i2 + 1])), cdp2, nd2)),
                      g0, g1);
            hv[c / 2 + i2] = pack_f16(g0, g1);
          }
        }
        tc_fence_before();
        mbar_arrive(&s.bar_dp_free);  // dP of tile J has been read: the next dP may overwrite it
        // dS (fp16) over the S_J columns this warp has read: [c0, +BN/4)
#pragma unroll
        for (int c = 0; c < kHalf / 2; c += 16) tmem_st16(tmem + lane_base + s_col + c0 + c, hv + c);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&s.bar_ds_ready[st]);
      }
      if (!ok) break;
      // ---- epilogue: dQ = scale * acc (this thread: head-dim columns [hf*64, +64))
      const bool have = n > 0;
      if (have) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_done, done_count & 1, prm.status));
        ++done_count;
        if (!ok) break;
        tc_fence_after();
      }
      const int d0 = hf * (kD / 2);
      __nv_bfloat16* dqrow =
          prm.dq + static_cast<size_t>((bh / prm.N1) * prm.qs.b + (bh % prm.N1) * prm.qs.h +
                                       static_cast<long long>(qpos) * prm.qs.s) + d0;
#pragma unroll
      for (int c = 0; c < kD / 2; c += 32) {
        uint32_t rr[32];
        if (have) {
          tmem_ld32(tmem + lane_base + kColDQ + d0 + c, rr);
          tmem_ld_wait(rr);
        } else {
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) rr[i2] = 0u;
        }
        if (row_valid) store_row_bf16(dqrow + c, rr, sc.dq_mul);
      }
      // dQ has been read: the next unit's first dQ product waits for its dS, which comes after
      tc_fence_before();
      J0 += n;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
  if (prm.cta_clock && threadIdx.x == 0) prm.cta_clock[2 * blockIdx.x + 1] = globaltimer_ns();
}

template <int BN>
cudaError_t launch_q(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, int grid, cudaStream_t st) {
  const size_t smem = sizeof(QSmem<BN>) + 1024;
  auto kernel = p.amask ? bsa_bwd_q_kernel<BN, true> : bsa_bwd_q_kernel<BN, false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  prof_begin("bsa_bwd_q", st);
  if (grid > 0) e = launch_pdl(kernel, dim3(grid), dim3(kKvThreads), smem, st, tq, tk, tv, tdo, p);
  prof_end(st);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t bsa_bwd_launch(const BsaBwdArgs& a, const void* q, const void* k, const void* v, const void* out,
                           const void* dout, const float* lse, cudaStream_t st) {
  // the scaled fp16 copies of Q, K, V, dOut (same layouts)
  {
    F16Copy c;
    const long long nq8 = static_cast<long long>(a.B) * a.N1 * a.S_q * kD / 8;
    const long long nk8 = static_cast<long long>(a.B) * a.N2 * a.S_kv * kD / 8;
    const void* src[4] = {q, k, v, dout};
    void* dst[4] = {a.q16, a.k16, a.v16, a.do16};
    const long long n8[4] = {nq8, nk8, nk8, nq8};
    for (int t = 0; t < 4; ++t) {
      c.src[t] = static_cast<const uint4*>(src[t]);
      c.dst[t] = static_cast<uint4*>(dst[t]);
      c.n8[t] = n8[t];
    }
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const dim3 grid(static_cast<unsigned>(sms * 4), 4);
    prof_begin("bsa_bwd_f16", st);
    cudaError_t e = launch_pdl(bwd_to_f16_kernel, grid, dim3(256), 0, st, c, a.amax);
    if (e == cudaSuccess)
      e = launch_pdl(bwd_f16_fixup_kernel, grid, dim3(256), 0, st, c, static_cast<const uint32_t*>(a.amax));
    prof_end(st);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const long long n_rows = static_cast<long long>(a.B) * a.N1 * a.nqb * kT;
  {
    const long long threads = n_rows * 8;
    const int blk = 256;
    prof_begin("bsa_bwd_prep", st);
    cudaError_t e = launch_pdl(bwd_prep_kernel, dim3(static_cast<unsigned>((threads + blk - 1) / blk)), dim3(blk), 0,
                               st, static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout),
                               lse, a.N1, a.S_q, a.bx, a.nqb, n_rows, a.qs, a.lse_s,
                               static_cast<const uint32_t*>(a.amax), a.dvec, a.lse2);
    prof_end(st);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // the fp16 copies as (head dim, head, position, batch), whichever of BNSD / BSND is in memory
  CUtensorMap tq, tk, tv, tdo, tk128, tv128, tq64, tdo64;
  auto qmap = [&](CUtensorMap* m, const void* base, uint32_t rows) {
    return make_tmap_4d_bf16(m, base, kD, a.N1, a.S_q, a.B, a.qs.h, a.qs.s, a.qs.b, rows);
  };
  auto kvmap = [&](CUtensorMap* m, const void* base, uint32_t rows) {
    return make_tmap_4d_bf16(m, base, kD, a.N2, a.S_kv, a.B, a.kvs.h, a.kvs.s, a.kvs.b, rows);
  };
  if (!qmap(&tq, a.q16, kT) || !qmap(&tdo, a.do16, kT) || !kvmap(&tk, a.k16, a.by) || !kvmap(&tv, a.v16, a.by) ||
      !kvmap(&tk128, a.k16, kT) || !kvmap(&tv128, a.v16, kT) || !qmap(&tq64, a.q16, kHalfRows) ||
      !qmap(&tdo64, a.do16, kHalfRows))
    return cudaErrorInvalidValue;
  BwdParams p;
  bool kv_launched = false;
  p.B = a.B; p.N1 = a.N1; p.N2 = a.N2; p.S_q = a.S_q; p.S_kv = a.S_kv; p.bx = a.bx; p.by = a.by;
  p.nqb = a.nqb; p.nkb = a.nkb; p.mask_mode = a.mask_mode; p.win_left = a.win_left; p.win_right = a.win_right;
  p.scale = a.scale; p.scale_log2 = a.scale * kLog2e;
  p.dvec = a.dvec; p.lse2 = a.lse2;
  p.dq = static_cast<__nv_bfloat16*>(a.dq);
  p.dk = static_cast<__nv_bfloat16*>(a.dk);
  p.dv = static_cast<__nv_bfloat16*>(a.dv);
  p.status = a.status;
  p.cta_clock = nullptr;
  p.qs = a.qs;
  p.kvs = a.kvs;
  p.amask = a.atten_mask;
  p.amax = a.amax;
  // KV-major pass
  {
    BwdParams pk = p;
    pk.row_ptr = a.t_row_ptr;
    pk.col = a.t_col;
    pk.next_unit = a.next_kv;
    const size_t smem = sizeof(KvSmem) + 1024;
    auto kv_kernel = a.atten_mask ? bsa_bwd_kv_kernel<true> : bsa_bwd_kv_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int units = a.B * a.N2 * a.nkb;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = units < sms ? units : sms;  // persistent: one CTA per SM
    prof_begin("bsa_bwd_kv", st);
    pk.pdl_wait = 1;
    pk.cta_clock = prof_cta_clock(1, grid);
    if (grid > 0) e = launch_pdl(kv_kernel, dim3(grid), dim3(kKvPassThreads), smem, st, tq64, tk128, tv128, tdo64, pk);
    prof_end(st);
    if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
    kv_launched = grid > 0;
  }
  // Q-major pass (persistent)
  p.row_ptr = a.row_ptr;
  p.col = a.col;
  p.next_unit = a.next_q;
  // The dQ pass reads the preprocess and the KV lists, not the KV pass: launched right after a KV
  // pass (which signals dependents only after its own wait on the preprocess), it need not wait
  // and its CTAs take the SMs the KV pass leaves; otherwise it waits for the preprocess.
  p.pdl_wait = kv_launched ? 0 : 1;
  const int q_units = a.B * a.N1 * a.nqb;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = q_units < sms ? q_units : sms;
  p.cta_clock = prof_cta_clock(2, grid);
  if (a.by == 128) return launch_q<128>(p, tq, tk, tv, tdo, grid, st);
  return launch_q<64>(p, tq, tk, tv, tdo, grid, st);
}

}  // namespace sa
