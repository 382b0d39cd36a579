// Block-sparse attention forward on tcgen05 (BlockSparseAttentionGrad page, forward formula):
//   Out = softmax(Mask(scale * Q K_sparse^T, atten_mask)) V_sparse,   LSE = m + ln(l)
// A unit is (b, h, q block): 128 query rows against the KV blocks its BlockSparseMask row selects
// (CSR lists from metadata.cu).  The kernel is persistent: one CTA per SM takes units from a
// device counter (head-major, longest q block of each head first) until none is left, so the
// next unit's Q load and first score tiles overlap the current unit's epilogue.  Every unit is
// computed whole by one CTA in list order, so results do not depend on the assignment.
//
// Warp roles (352 threads: 11 warps):
//   warps 0-7  softmax: warp w reads TMEM lane quarter w % 4 (query rows 32*(w%4) .. +31) and the
//              column half w / 4 of each S tile, so each row is shared by two threads that
//              exchange their partial row max through shared memory.  They mask, keep the
//              running max/sum, rescale their half of O in TMEM when needed, write P (bf16)
//              back over the consumed S columns (the A operand of O += P V), and write the
//              unit's Out and LSE.
//   warp 8     scheduler and TMA producer: takes the next unit, hands it to the other warps
//              through a small ring in shared memory, then loads Q (once the previous unit's
//              last S has read the old Q), the K tiles into a 2-stage ring and the V tiles into
//              a 2-stage ring.  A K stage is released when its S = Q K^T has run, a V stage
//              after its O += P V.
//   warp 9     issues O += P_j V_j into the TMEM O accumulator as soon as P_j is ready.
//   warp 10    issues S_j = Q K_j^T into TMEM S buffer j % 2 as soon as K_j is loaded and the
//              buffer's previous O += P V has completed.  Two issuing threads: tcgen05.mma issue
//              blocks while the tensor pipe's queue is full, so one thread would hold each
//              O += P V back behind the next tile's score MMAs.
// Tile counters run across units, so rings, S buffers and barrier phases carry over.
// The row max is taken on the raw scores (scale > 0 is required by the host checks), so each
// probability costs one fused multiply-add (packed in pairs) and one exp2.
// Every wait is bounded (sa_common.cuh); on a timeout the kernel sets SA_DEV_TIMEOUT and stops.
#include <cuda.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sa_common.cuh"

namespace sa {
namespace {

constexpr int kBM = 128;  // query rows per CTA tile (the MMA M)
constexpr int kD = 128;   // head dim of Q/K and V
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = (kSoftmaxWarps + 3) * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr int kKStages = 2, kVStages = 2;
constexpr int kSched = 4;  // unit ring between the scheduler and the other warps

template <int BN>
struct __align__(1024) FwdSmem {
  uint8_t q[2][kBM * 128];            // Q sub-tiles (head-dim columns 0-63, 64-127), 128B swizzle
  uint8_t k[kKStages][2][BN * 128];   // [stage][sub-tile] K rows of one KV block
  uint8_t v[kVStages][2][BN * 128];   // [stage][sub-tile] V rows
  uint8_t ostage[2][kBM * 128];       // Out tile staged for the TMA store (head-dim halves)
  float red[2][2][kBM];               // [tile parity][column half][row]: partial row max
  float red_l[2][2][kBM];             // [unit parity][column half][row]: partial row sum
  int32_t sched[kSched];              // unit ring (-1: no more units)
  uint64_t bar_q, bar_q_empty;
  uint64_t bar_k[kKStages], bar_k_empty[kKStages], bar_v[kVStages], bar_v_empty[kVStages], bar_s_full[2];
  uint64_t bar_p_full[2];             // per S buffer: P of its tile is written (256 arrivals)
  uint64_t bar_o_done;
  uint64_t bar_pv_done[2];            // per S buffer: the O += P V that read it has completed
  uint64_t bar_done;                  // one phase per non-empty unit: its last O += P V has completed
  uint64_t bar_sched_full[kSched], bar_sched_empty[kSched];
  uint64_t bar_pair[4];               // the two softmax warps of each TMEM lane quarter
  uint64_t bar_epi;                   // the unit's Out tile is staged (256 arrivals)
  uint64_t bar_stage_free;            // the previous store has read the staging buffer
  uint32_t tmem_base;
};

struct FwdParams {
  int B, N1, N2, S_q, S_kv, bx, by, nqb, mask_mode, win_left, win_right, units;
  float scale_log2;
  const int32_t* row_ptr;
  const int32_t* col;
  __nv_bfloat16* out;
  float* lse;
  int32_t* next_unit;  // scheduler counter, zero at launch
  uint32_t* status;
  uint64_t* cta_clock;  // optional [grid][2] start / finish times (ns), see bsa_profile_cta_clock
  long long lse_sb, lse_sh, lse_ss;  // LSE element strides of (b, head, position)
  const uint8_t* amask;  // optional dense atten_mask [S_q][S_kv], nonzero = masked out
};

// Unit number i of the schedule -> (b*N1 + h, q block): head-major, latest q block first.
struct UnitInfo {
  int bh, qb, rp, n;
};
__device__ __forceinline__ UnitInfo unit_info(const FwdParams& prm, int i) {
  UnitInfo u;
  u.bh = i / prm.nqb;
  u.qb = prm.nqb - 1 - i % prm.nqb;
  const int unit = u.bh * prm.nqb + u.qb;
  u.rp = prm.row_ptr[unit];
  u.n = prm.row_ptr[unit + 1] - u.rp;
  return u;
}

// Exchange point of the two softmax warps that share a TMEM lane quarter: an mbarrier of 64
// arrivals with a bounded wait (a plain bar.sync could not give up if the partner stopped early).
// The tcgen05 fences order each side's tensor-memory reads before the other side's writes.
__device__ __forceinline__ bool pair_sync(uint64_t* bar, int& exchanges, uint32_t* status) {
  tc_fence_before();
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, exchanges & 1, status);
  ++exchanges;
  tc_fence_after();
  return ok;
}

// kMask: a dense atten_mask is applied (a separate instantiation keeps the mask-free loop unchanged)
template <int BN, bool kMask>
__global__ void __launch_bounds__(kThreads, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const FwdParams prm) {
  griddep_wait();  // launched with programmatic dependent launch: the KV lists must be complete
  if (prm.cta_clock && threadIdx.x == 0) prm.cta_clock[2 * blockIdx.x] = globaltimer_ns();
  griddep_launch_dependents();
  constexpr uint32_t kTmemCols = (2 * BN + kD) <= 256 ? 256 : 512;
  constexpr uint32_t kColS0 = 0, kColS1 = BN, kColO = 2 * BN;
  constexpr int kHalf = BN / 2;  // S columns per softmax thread
  extern __shared__ uint8_t smem_raw[];
  FwdSmem<BN>& s = *reinterpret_cast<FwdSmem<BN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&s.bar_q, 1);
    mbar_init(&s.bar_q_empty, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&s.bar_k[i], 1);
      mbar_init(&s.bar_k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&s.bar_v[i], 1);
      mbar_init(&s.bar_v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&s.bar_s_full[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&s.bar_p_full[i], kSoftmaxWarps * 32);
    mbar_init(&s.bar_o_done, 1);
    for (int i = 0; i < 2; ++i) mbar_init(&s.bar_pv_done[i], 1);
    mbar_init(&s.bar_done, 1);
    for (int i = 0; i < kSched; ++i) {
      mbar_init(&s.bar_sched_full[i], 1);
      mbar_init(&s.bar_sched_empty[i], 2 + kSoftmaxWarps * 32);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&s.bar_pair[i], 64);
    mbar_init(&s.bar_epi, kSoftmaxWarps * 32);
    mbar_init(&s.bar_stage_free, 1);
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

  // the k-th unit of this CTA from the ring (consumers); -1 when the work is done or on timeout
  auto next_from_ring = [&](int k) -> int {
    const int slot = k % kSched;
    if (!mbar_wait(&s.bar_sched_full[slot], (k / kSched) & 1, prm.status)) return -1;
    const int u = *reinterpret_cast<volatile int32_t*>(&s.sched[slot]);
    mbar_arrive(&s.bar_sched_empty[slot]);
    return u;
  };

  if (warp == kSoftmaxWarps) {
    // ------------------------------------------------------------------ scheduler + TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int jk = 0, jv = 0, qcount = 0;  // K / V tiles issued, Q loads issued (this CTA)
      bool ok = true;
      // TMA coordinates (head dim, head, position, batch) of the 4-D maps
      auto load_v = [&](int rp, int b, int g, int j) -> bool {  // V of the unit's tile j (global jv)
        const int sv = jv % kVStages, uv = jv / kVStages;
        if (jv >= kVStages && !mbar_wait(&s.bar_v_empty[sv], (uv - 1) & 1, prm.status)) return false;
        const int vpos = prm.col[rp + j] * prm.by;
        mbar_arrive_expect_tx(&s.bar_v[sv], 2 * BN * 128);
        tma_load_4d(s.v[sv][0], &tm_v, &s.bar_v[sv], 0, g, vpos, b);
        tma_load_4d(s.v[sv][1], &tm_v, &s.bar_v[sv], 64, g, vpos, b);
        ++jv;
        return true;
      };
      for (int k = 0; ok; ++k) {
        const int slot = k % kSched;
        if (k >= kSched && !(ok = mbar_wait(&s.bar_sched_empty[slot], ((k / kSched) - 1) & 1, prm.status))) break;
        int i = atomicAdd(prm.next_unit, 1);
        if (i >= prm.units) i = -1;
        s.sched[slot] = i;
        mbar_arrive(&s.bar_sched_full[slot]);  // release: the ring entry is visible to its readers
        if (i < 0) break;
        const UnitInfo u = unit_info(prm, i);
        if (u.n == 0) continue;
        const int b = u.bh / prm.N1, h = u.bh % prm.N1;
        const int g = h / (prm.N1 / prm.N2);
        const int q_pos0 = u.qb * prm.bx;
        // Q: the previous unit's last S = Q K^T must have read the old Q
        if (qcount > 0 && !(ok = mbar_wait(&s.bar_q_empty, (qcount - 1) & 1, prm.status))) break;
        mbar_arrive_expect_tx(&s.bar_q, 2 * kBM * 128);
        tma_load_4d(s.q[0], &tm_q, &s.bar_q, 0, h, q_pos0, b);
        tma_load_4d(s.q[1], &tm_q, &s.bar_q, 64, h, q_pos0, b);
        ++qcount;
        // K runs up to kKStages tiles ahead, V trails K by one tile
        for (int j = 0; ok && j < u.n; ++j) {
          const int kpos = prm.col[u.rp + j] * prm.by;
          const int sk = jk % kKStages, uk = jk / kKStages;
          if (jk >= kKStages && !(ok = mbar_wait(&s.bar_k_empty[sk], (uk - 1) & 1, prm.status))) break;
          mbar_arrive_expect_tx(&s.bar_k[sk], 2 * BN * 128);
          tma_load_4d(s.k[sk][0], &tm_k, &s.bar_k[sk], 0, g, kpos, b);
          tma_load_4d(s.k[sk][1], &tm_k, &s.bar_k[sk], 64, g, kpos, b);
          ++jk;
          if (j >= kKStages - kVStages) ok = load_v(u.rp, b, g, j - (kKStages - kVStages));
        }
        for (int j = u.n - (kKStages - kVStages); ok && j < u.n; ++j)
          if (j >= 0) ok = load_v(u.rp, b, g, j);
      }
      // do not leave the CTA with copies in flight
      for (int j = (jk > kKStages ? jk - kKStages : 0); j < jk; ++j)
        mbar_wait(&s.bar_k[j % kKStages], (j / kKStages) & 1, prm.status);
      for (int j = (jv > kVStages ? jv - kVStages : 0); j < jv; ++j)
        mbar_wait(&s.bar_v[j % kVStages], (j / kVStages) & 1, prm.status);
      if (qcount > 0) mbar_wait(&s.bar_q, (qcount - 1) & 1, prm.status);
    }
  } else if (warp == kSoftmaxWarps + 1 || warp == kSoftmaxWarps + 2) {
    // ------------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const bool pv_thread = warp == kSoftmaxWarps + 1;
      const uint32_t idesc_s = idesc_bf16_f32(kBM, BN, false, false);
      const uint32_t idesc_o = idesc_bf16_f32(kBM, kD, false, true);
      // descriptors of stage 0 / sub-tile 0; other stages, sub-tiles and K steps are added offsets
      const uint64_t dq0 = sdesc_sw128(smem_u32(s.q[0]), 0, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(s.k[0][0]), 0, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(s.v[0][0]), BN * 128, 1024);
      int J0 = 0, qcount = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int i = next_from_ring(k);
        if (i < 0) break;
        const UnitInfo u = unit_info(prm, i);
        if (u.n == 0) continue;
        if (pv_thread) {
          for (int j = 0; ok && j < u.n; ++j) {
            const int J = J0 + j, st = J & 1, sv = J % kVStages;
            // one barrier per S buffer: its next phase needs S_{J+2}, which waits for this PV
            if (!(ok = mbar_wait(&s.bar_p_full[st], (J >> 1) & 1, prm.status))) break;
            if (!(ok = mbar_wait(&s.bar_v[sv], (J / kVStages) & 1, prm.status))) break;
            tc_fence_after();
            const uint32_t p_col = st ? kColS1 : kColS0;
            const uint64_t dv = dv0 + static_cast<uint64_t>(sv) * ((2 * BN * 128) >> 4);
#pragma unroll
            for (int ks = 0; ks < BN / 16; ++ks)
              mma_bf16_ts(tmem + kColO, tmem + p_col + ks * 8, sdesc_add(dv, ks * 2048), idesc_o,
                          (j > 0 || ks > 0) ? 1u : 0u);
            tc_commit(&s.bar_o_done);
            tc_commit(&s.bar_v_empty[sv]);
            tc_commit(&s.bar_pv_done[st]);
          }
          if (ok) tc_commit(&s.bar_done);
        } else {
          if (!(ok = mbar_wait(&s.bar_q, qcount & 1, prm.status))) break;
          ++qcount;
          for (int j = 0; ok && j < u.n; ++j) {
            const int J = J0 + j, st = J & 1, sk = J % kKStages;
            // S buffer st last held P_{J-2}; one barrier per buffer keeps the parity wait exact
            if (J >= 2 && !(ok = mbar_wait(&s.bar_pv_done[st], ((J >> 1) - 1) & 1, prm.status))) break;
            if (!(ok = mbar_wait(&s.bar_k[sk], (J / kKStages) & 1, prm.status))) break;
            tc_fence_after();
            const uint32_t d = tmem + (st ? kColS1 : kColS0);
            const uint64_t dk = dk0 + static_cast<uint64_t>(sk) * ((2 * BN * 128) >> 4);
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks)
              mma_bf16_ss(d, sdesc_add(dq0, (ks >> 2) * (kBM * 128) + (ks & 3) * 32),
                          sdesc_add(dk, (ks >> 2) * (BN * 128) + (ks & 3) * 32), idesc_s, ks > 0 ? 1u : 0u);
            tc_commit(&s.bar_s_full[st]);
            tc_commit(&s.bar_k_empty[sk]);
            if (j + 1 == u.n) tc_commit(&s.bar_q_empty);  // the unit's last read of Q
          }
        }
        J0 += u.n;
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t o_col = kColO + hf * (kD / 2);  // this thread's half of the O row
    int exchanges = 0, J0 = 0, done_count = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int i = __shfl_sync(0xffffffffu, next_from_ring(k), 0);
      if (i < 0) break;
      const UnitInfo u = unit_info(prm, i);
      const int n = u.n, rp = u.rp, qb = u.qb;
      const int ub = u.bh / prm.N1, uh = u.bh % prm.N1;
      const int qpos = qb * prm.bx + r;
      const bool row_valid = r < prm.bx && qpos < prm.S_q;
      // visible key interval [lo, hi] for this row (mask modes 0/2/3/4)
      int lo = 0, hi = prm.S_kv - 1;
      const int qq = qpos + prm.S_kv - prm.S_q;
      if (prm.mask_mode == 2) hi = min(hi, qpos);
      else if (prm.mask_mode == 3) hi = min(hi, qq);
      else if (prm.mask_mode == 4) { lo = qq - prm.win_left; hi = min(hi, qq + prm.win_right); }
      if (!row_valid) { lo = 1; hi = 0; }
      float m = -INFINITY, l = 0.f;  // l: partial sum over this thread's columns
      int col_next = n > 0 ? prm.col[rp] : 0;  // read one tile ahead, before the wait
      for (int j = 0; j < n; ++j) {
        const int J = J0 + j;
        const int st = J & 1;
        const int cj = col_next;
        if (j + 1 < n) col_next = prm.col[rp + j + 1];
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_s_full[st], (J >> 1) & 1, prm.status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_col = st ? kColS1 : kColS0;
        const int kpos0 = cj * prm.by + hf * kHalf;
        // the dense atten_mask inside the selected block: bit c = this row may not see column c
        const uint64_t mbits = kMask && row_valid
                                   ? dense_mask_bits<kHalf>(prm.amask + static_cast<size_t>(qpos) * prm.S_kv, kpos0,
                                                           prm.S_kv)
                                   : 0ull;
        float x[kHalf];  // raw scores
#pragma unroll
        for (int c = 0; c < kHalf; c += 32) {
          uint32_t rr[32];
          tmem_ld32(tmem + lane_base + s_col + hf * kHalf + c, rr);
          tmem_ld_wait(rr);
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) x[c + i2] = __uint_as_float(rr[i2]);
        }
        const bool full = kpos0 >= lo && kpos0 + kHalf - 1 <= hi;
        if (!full) {
#pragma unroll
          for (int c = 0; c < kHalf; ++c) {
            const int kp = kpos0 + c;
            if (kp < lo || kp > hi) x[c] = -INFINITY;
          }
        }
        if (kMask && mbits != 0) {
#pragma unroll
          for (int c = 0; c < kHalf; ++c)
            if ((mbits >> c) & 1ull) x[c] = -INFINITY;
        }
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < kHalf; c += 4) {
          mx4[0] = fmaxf(mx4[0], x[c]);
          mx4[1] = fmaxf(mx4[1], x[c + 1]);
          mx4[2] = fmaxf(mx4[2], x[c + 2]);
          mx4[3] = fmaxf(mx4[3], x[c + 3]);
        }
        float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        // row max = max of the two halves; the barrier also orders both threads' S reads before
        // either writes P over the S columns
        s.red[st][hf][r] = mx;
        ok = __all_sync(0xffffffffu, pair_sync(&s.bar_pair[quarter], exchanges, prm.status));
        if (!ok) break;
        mx = fmaxf(mx, s.red[st][hf ^ 1][r]) * prm.scale_log2;  // log2 units of the scaled score
        // Lazy rescaling: the exponent reference m only moves when the row max exceeds it by
        // more than 8 (p <= 2^8 otherwise); numerator and l share the same reference, so the
        // final O / l is unchanged.  Only then must the previous O += P V have landed.
        float m_new = m;
        bool need = false;
        if (mx > m + 8.f) {
          need = (m != -INFINITY);
          m_new = mx;
        }
        if (__any_sync(0xffffffffu, need)) {  // tcgen05.ld/st are warp-collective
          // O += P_{J-1} V_{J-1} is o_done phase J-1 (need implies j > 0).  S_J was issued after
          // O += P_{J-2} V_{J-2} completed (the S buffer's pv_done), so phase J-2 is complete,
          // and phase J needs this thread's P_J: a parity wait tells J-1 from J.
          ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_o_done, (J - 1) & 1, prm.status));
          if (!ok) break;
          tc_fence_after();
          const float alpha = need ? ex2(m - m_new) : 1.f;
          l *= alpha;
#pragma unroll
          for (int c = 0; c < kD / 2; c += 32) {
            uint32_t rr[32];
            tmem_ld32(tmem + lane_base + o_col + c, rr);
            tmem_ld_wait(rr);
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) rr[i2] = __float_as_uint(__uint_as_float(rr[i2]) * alpha);
            tmem_st32(tmem + lane_base + o_col + c, rr);
          }
          tmem_st_wait();
        }
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        // p = 2^(s * scale * log2(e) - m): one packed fma per pair, one exp2 per element
        const uint64_t sc2 = f2_pack(prm.scale_log2, prm.scale_log2), nm2 = f2_pack(-m_use, -m_use);
        uint64_t acc0 = 0, acc1 = 0;  // packed partial row sums (0 bits == 0.0f, 0.0f)
#pragma unroll
        for (int c = 0; c < kHalf; c += 32) {
          uint32_t hv[16];
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2) {
            float t0, t1;
            f2_unpack(f2_fma(f2_pack(x[c + 2 * i2], x[c + 2 * i2 + 1]), sc2, nm2), t0, t1);
            const float e0 = ex2(t0), e1 = ex2(t1);
            if (i2 & 1) acc1 = f2_add(acc1, f2_pack(e0, e1));
            else acc0 = f2_add(acc0, f2_pack(e0, e1));
            hv[i2] = pack_bf16(e0, e1);
          }
          // packed pairs: element column e -> TMEM column e/2 of the S buffer
          tmem_st16(tmem + lane_base + s_col + (hf * kHalf + c) / 2, hv);
        }
        tmem_st_wait();
        {
          float a0, a1, b0, b1;
          f2_unpack(acc0, a0, a1);
          f2_unpack(acc1, b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
        m = m_new;
        tc_fence_before();
        mbar_arrive(&s.bar_p_full[st]);
      }
      if (!ok) break;
      // ---- epilogue.  bar_done has one phase per non-empty unit and this thread has waited on
      // every earlier one, so a parity wait is exact (o_done is not: lazy rescaling skips phases).
      bool have_o = n > 0;
      if (have_o) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_done, done_count & 1, prm.status));
        ++done_count;
        if (!ok) break;
        tc_fence_after();
      }
      // full row sum from the two halves (slot by unit parity: the partner may still be reading
      // the previous unit's entry when this thread writes the next one)
      s.red_l[k & 1][hf][r] = l;
      ok = __all_sync(0xffffffffu, pair_sync(&s.bar_pair[quarter], exchanges, prm.status));
      if (!ok) break;
      l += s.red_l[k & 1][hf ^ 1][r];
      const bool any = have_o && l > 0.f;
      const float inv_l = any ? 1.f / l : 0.f;
      // Out goes through a 128-byte-swizzled staging tile and two TMA stores (one per head-dim
      // half), so global writes are whole rows; the box of block_x rows of a [B*N1][S_q][128] map
      // stops at the q block and at the head's end.  The previous unit's store must have read
      // the staging tile first.
      if (k > 0) {
        if (warp == 0 && lane == 0) {  // the thread that issued the previous unit's stores
          bulk_wait_read_all();
          mbar_arrive(&s.bar_stage_free);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_stage_free, (k - 1) & 1, prm.status));
        if (!ok) break;
      }
      uint8_t* ost = s.ostage[hf];
#pragma unroll
      for (int c = 0; c < kD / 2; c += 32) {
        uint32_t rr[32];
        if (have_o) {  // warp-uniform: every lane joins the collective load
          tmem_ld32(tmem + lane_base + o_col + c, rr);
          tmem_ld_wait(rr);
        } else {
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) rr[i2] = 0u;
        }
#pragma unroll
        for (int i2 = 0; i2 < 32; i2 += 8) {
          uint4 pk;
          pk.x = pack_bf16(__uint_as_float(rr[i2 + 0]) * inv_l, __uint_as_float(rr[i2 + 1]) * inv_l);
          pk.y = pack_bf16(__uint_as_float(rr[i2 + 2]) * inv_l, __uint_as_float(rr[i2 + 3]) * inv_l);
          pk.z = pack_bf16(__uint_as_float(rr[i2 + 4]) * inv_l, __uint_as_float(rr[i2 + 5]) * inv_l);
          pk.w = pack_bf16(__uint_as_float(rr[i2 + 6]) * inv_l, __uint_as_float(rr[i2 + 7]) * inv_l);
          const int chunk = (c + i2) >> 3;  // 16-byte chunk of this row's 64 columns
          *reinterpret_cast<uint4*>(ost + r * 128 + ((chunk ^ (r & 7)) << 4)) = pk;
        }
      }
      fence_async_smem();
      mbar_arrive(&s.bar_epi);
      if (warp == 0 && lane == 0) {
        ok = mbar_wait(&s.bar_epi, k & 1, prm.status);
        if (ok) {
          tma_store_4d(&tm_o, s.ostage[0], 0, uh, qb * prm.bx, ub);
          tma_store_4d(&tm_o, s.ostage[1], 64, uh, qb * prm.bx, ub);
          bulk_commit();  // read completion is awaited at the next unit's epilogue, off the critical path
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (row_valid && hf == 0)
        prm.lse[ub * prm.lse_sb + uh * prm.lse_sh + qpos * prm.lse_ss] = any ? (m * kLn2 + logf(l)) : -INFINITY;
      // O has been read: the next unit's first O += P V waits for P, which comes after this
      tc_fence_before();
      J0 += n;
    }
  }
  if (warp == 0 && lane == 0) bulk_wait_all();  // the last Out stores have completed
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
  if (prm.cta_clock && threadIdx.x == 0) prm.cta_clock[2 * blockIdx.x + 1] = globaltimer_ns();
}

template <int BN>
cudaError_t launch_fwd(const BsaFwdArgs& a, const void* q, const void* k, const void* v, cudaStream_t st) {
  // Q, K, V and Out as (head dim, head, position, batch), whichever of BNSD / BSND is in memory;
  // the Out box stops at the q block (block_x rows) and the tensor's positions
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_4d_bf16(&tq, q, kD, a.N1, a.S_q, a.B, a.qs.h, a.qs.s, a.qs.b, kBM) ||
      !make_tmap_4d_bf16(&tk, k, kD, a.N2, a.S_kv, a.B, a.kvs.h, a.kvs.s, a.kvs.b, BN) ||
      !make_tmap_4d_bf16(&tv, v, kD, a.N2, a.S_kv, a.B, a.kvs.h, a.kvs.s, a.kvs.b, BN) ||
      !make_tmap_4d_bf16(&to, a.out, kD, a.N1, a.S_q, a.B, a.qs.h, a.qs.s, a.qs.b, a.bx))
    return cudaErrorInvalidValue;
  FwdParams p;
  p.B = a.B; p.N1 = a.N1; p.N2 = a.N2; p.S_q = a.S_q; p.S_kv = a.S_kv; p.bx = a.bx; p.by = a.by;
  p.nqb = a.nqb; p.mask_mode = a.mask_mode; p.win_left = a.win_left; p.win_right = a.win_right;
  p.units = a.B * a.N1 * a.nqb;
  p.scale_log2 = a.scale * kLog2e;
  p.row_ptr = a.row_ptr; p.col = a.col;
  p.out = static_cast<__nv_bfloat16*>(a.out); p.lse = a.lse; p.next_unit = a.next_unit; p.status = a.status;
  p.cta_clock = nullptr;
  p.lse_sb = a.lse_s.b; p.lse_sh = a.lse_s.h; p.lse_ss = a.lse_s.s;
  p.amask = a.atten_mask;
  const size_t smem = sizeof(FwdSmem<BN>) + 1024;
  auto kernel = a.atten_mask ? bsa_fwd_kernel<BN, true> : bsa_fwd_kernel<BN, false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (p.units == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.units < sms ? p.units : sms;  // persistent: one CTA per SM
  p.cta_clock = prof_cta_clock(0, grid);
  prof_begin("bsa_fwd", st);
  e = launch_pdl(kernel, dim3(grid), dim3(kThreads), smem, st, tq, tk, tv, to, p);
  prof_end(st);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t bsa_fwd_launch(const BsaFwdArgs& a, const void* q, const void* k, const void* v, cudaStream_t st) {
  if (a.by == 128) return launch_fwd<128>(a, q, k, v, st);
  if (a.by == 64) return launch_fwd<64>(a, q, k, v, st);
  return cudaErrorInvalidValue;
}

}  // namespace sa
