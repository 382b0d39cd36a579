// Internal (non-ABI) declarations shared by the .cu files of the library.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "selected_attention.h"

namespace sa {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Carves a caller workspace into aligned arrays, in a fixed order, so the size query and the
// op call agree.  With base == nullptr it only measures.
struct Carver {
  char* base;
  size_t off = 256;  // bytes [0, 256) hold the status word
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t n) {
    off = align_up(off, 256);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
  size_t bytes() const { return align_up(off, 256); }
  size_t next() const { return align_up(off, 256); }  // offset of the next take
};

// ---- kernel timing (profile.cu): brackets a launch with events when timing is enabled ----------
void prof_begin(const char* name, cudaStream_t st);
void prof_end(cudaStream_t st);
// Per-CTA start / finish record of the persistent block-sparse kernels (slot 0 bsa_fwd, 1
// bsa_bwd_kv, 2 bsa_bwd_q): the device array to write for a launch of `grid` CTAs, or nullptr
// when recording is off or the caller's buffer is too small.
uint64_t* prof_cta_clock(int slot, int grid);

// ---- metadata (metadata.cu) -------------------------------------------------------------------
// BSA KV lists: units (b, h, qb) -> ascending kv block ids.
cudaError_t bsa_kv_lists(const uint8_t* mask, int units, int nkb, int32_t* counts, int32_t* row_ptr, int32_t* col,
                         cudaStream_t st);
// BSA transposed lists: rows (b, g, kb) -> ascending h_local*nqb + qb.  maskT is scratch of
// B*N1*nqb*nkb bytes.
cudaError_t bsa_q_lists(const uint8_t* mask, int B, int N1, int N2, int nqb, int nkb, uint8_t* maskT,
                        int32_t* counts, int32_t* row_ptr, int32_t* col, cudaStream_t st);
// Exclusive scan of n counts into row_ptr[n+1].
cudaError_t exclusive_scan(const int32_t* counts, int n, int32_t* row_ptr, cudaStream_t st);

// ---- tensor maps (tma.cpp) ---------------------------------------------------------------------
// 2D bf16 map over rows x cols (cols contiguous), row stride in elements, box {64, box_rows},
// 128-byte swizzle.
bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride,
                       uint32_t box_rows);
// 3D bf16 map over [d2][d1][d0] (d0 contiguous) with strides in elements, box {64, box1, box2}.
bool make_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t stride1, uint64_t stride2, uint32_t box1, uint32_t box2);

// 3D fp32 map over [d2][d1][d0] (d0 contiguous), strides in elements, box {box0, box1, box2}
// (box0 * 4 bytes <= 128: the 128-byte swizzle).
bool make_tmap_3d_f32(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1,
                      uint64_t stride2, uint32_t box0, uint32_t box1, uint32_t box2);

// 4D bf16 map over (d0 contiguous, d1, d2, d3) with strides in elements, box {64, 1, box2, 1}: a
// [B][..][..][D] attention tensor seen as (head dim, head, position, batch) whatever the order of
// head and position in memory (BNSD or BSND).  Rows past d2 read as zero and are not stored.
bool make_tmap_4d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                       uint64_t stride1, uint64_t stride2, uint64_t stride3, uint32_t box2);

// Element strides of a BSA tensor (b, head, position, d): BNSD [B][N][S][D] or BSND [B][S][N][D];
// the LSE [b][head][position] is [B][N][S] for BNSD and [B][S][N] for BSND.
struct BsaStrides {
  long long b, h, s;
};
// Strides of a [B][heads][S][D] (BNSD) or [B][S][heads][D] (BSND) tensor, and of its [B][heads][S]
// or [B][S][heads] LSE.
inline BsaStrides bsa_strides(int layout, int heads, int S, int D) {
  if (layout == BSA_LAYOUT_BSND) return {1LL * S * heads * D, D, 1LL * heads * D};
  return {1LL * heads * S * D, 1LL * S * D, D};
}

// ---- BSA forward (bsa_fwd.cu) --------------------------------------------------------------------
struct BsaFwdArgs {
  int B, N1, N2, S_q, S_kv, bx, by, nqb, nkb, mask_mode, win_left, win_right;
  float scale;
  BsaStrides qs, kvs, lse_s;  // element strides of q / out, of k / v, of the LSE
  const uint8_t* atten_mask;  // optional dense [S_q][S_kv] mask (nonzero = masked out) or nullptr
  const int32_t* row_ptr;
  const int32_t* col;
  void* out;
  float* lse;
  int32_t* next_unit;  // persistent-kernel work counter, zeroed before the launch
  uint32_t* status;
};

// The first 256 bytes of every workspace: the device status word, then the work counters of the
// persistent kernels (zeroed with the status word before each call).
struct WsHeader {
  uint32_t status;
  int32_t next_fwd, next_bwd_kv, next_bwd_q;
  uint32_t amax[4];  // backward: max |x| (float bits) of Q, K, V, dOut
};
cudaError_t bsa_fwd_launch(const BsaFwdArgs& a, const void* q, const void* k, const void* v, cudaStream_t st);

// ---- BSA backward (bsa_bwd.cu) -------------------------------------------------------------------
struct BsaBwdArgs {
  int B, N1, N2, S_q, S_kv, bx, by, nqb, nkb, mask_mode, win_left, win_right;
  float scale;
  BsaStrides qs, kvs, lse_s;  // element strides of q / out / dout / dq, of k / v / dk / dv, of the LSE
  const uint8_t* atten_mask;  // optional dense [S_q][S_kv] mask (nonzero = masked out) or nullptr
  const int32_t* row_ptr;    // KV lists per (b, h, qb)
  const int32_t* col;
  const int32_t* t_row_ptr;  // transposed lists per (b, g, kb)
  const int32_t* t_col;
  float* dvec;               // scratch [B*N1*nqb*128]
  float* lse2;               // scratch [B*N1*nqb*128]
  void *q16, *k16, *v16, *do16;  // scratch: fp16 copies of Q, K, V, dOut (same layout), scaled by powers of 2
  uint32_t* amax;            // WsHeader::amax, zeroed before the launch
  int32_t* next_kv;          // work counters of the persistent passes, zeroed before the launch
  int32_t* next_q;
  void* dq;
  void* dk;
  void* dv;
  uint32_t* status;
};
cudaError_t bsa_bwd_launch(const BsaBwdArgs& a, const void* q, const void* k, const void* v, const void* out,
                           const void* dout, const float* lse, cudaStream_t st);

// ---- sparse decode (sfa_meta.cu, sfa_decode.cu) ------------------------------------------------
struct SfaMetaArgs {
  const int32_t* sparse_indices;  // [B, 1, N2, K] (row 0 used)
  const int32_t* block_table;     // [B, max_pages_per_seq]
  const int32_t* seqused_kv;      // [B]
  int B, N2, K, ppb, page_size, max_pages_per_seq, num_pages;
  int32_t* pages;   // [B*N2][K*ppb] compacted physical pages
  int32_t* tokens;  // valid tokens of each listed page
  int32_t* count;   // [B*N2]
  uint32_t* status;
};
cudaError_t sfa_page_list(const SfaMetaArgs& a, cudaStream_t st);
// Decode pieces: unit u = (b * N2 + g) * HH + head half is cut into P pieces (P = the cluster size
// of the decode launch); piece u * P + p takes pages [floor(p n / P), floor((p + 1) n / P)) of the
// unit's n.  sfa_pieces runs the decode prologue's set-up for every piece: a.pages / a.tokens are
// [n_pieces][K * ppb] regions, rec is int32 [n_pieces][3] = (n, begin, len).
constexpr int kSfaMaxPieces = 4;
int sfa_pieces_per_unit(int units, int sms);
cudaError_t sfa_pieces(const SfaMetaArgs& a, int P, int HH, int n_pieces, int32_t* rec, cudaStream_t st);
// head halves of 64 per kv head: 2 when the group has more than 64 query heads
int sfa_head_halves(int G);
struct SfaDecodeArgs {
  int B, N1, N2, K, ppb, page_size, max_pages_per_seq, num_pages, units, P;
  float scale;
  const void *q, *q_rope, *k_cache, *k_rope_cache, *v_cache;
  const int32_t *sparse_indices, *block_table, *seqused_kv;
  int32_t *pages, *tokens, *rec;  // per-piece regions, as for sfa_pieces
  void* out;
  float* lse;
  uint32_t* status;
};
cudaError_t sfa_decode_launch(const SfaDecodeArgs& a, cudaStream_t st);

// ---- SFA backward (sfa_bwd.cu) --------------------------------------------------------------------
// Unit u = b * N2 + g (all G heads of a kv head); meta holds the page lists ([U][cap], count [U]).
struct SfaBwdArgs {
  SfaMetaArgs meta;
  int B, N1, N2, page_size, num_pages, cap;  // cap = K * ppb pages per unit
  float scale;
  const void *q, *q_rope, *k_cache, *k_rope_cache, *v_cache, *out, *dout;
  const float* lse;
  void *dq, *dq_rope, *dk_cache, *dk_rope_cache, *dv_cache;
  // workspace
  float *lse2, *dvec;  // [B * N1]
  void* ds;            // [U][T * 128][128] bf16: each tile's dS^T (T = tiles of 128 gathered tokens per unit)
  void *gk, *gv;       // gathered-order row gradients [U][cap * page_size][576] / [..][512] bf16
  int32_t *cnt;        // [2][num_pages * N2]: readers per cache row-block, then the fill cursor
  int32_t *ptr;        // [num_pages * N2 + 1]
  int32_t *list;       // [U * cap]
};
cudaError_t sfa_bwd_launch(const SfaBwdArgs& a, cudaStream_t st);
// tiles of 128 gathered tokens per unit for a list of cap pages (the same rule the kernel uses)
int sfa_bwd_tiles(int cap, int page_size);

// ---- NSA selected attention (nsa_meta.cu, nsa.cu) ----------------------------------------------
struct NsaMetaArgs {
  const int32_t* topk;        // [T, N2, K]
  const int32_t* cu_seqlens;  // [B+1]
  int B, T, N2, K, sel_block, max_len, nblk_max, words;  // words = ceil(T / 32)
  bool token_lists;           // also build the transposed lists (backward)
  int32_t* ok_flag;           // 1 if cu_seqlens is valid
  int32_t* ids;               // [T, N2, K]
  int32_t* cnt;               // [T, N2]
  int32_t* dup;               // [T, N2] 1 if the valid list holds an id twice
  uint32_t* bitmap;           // [N2, nblk_max, words] (backward only)
  int32_t *t_counts, *t_row_ptr, *t_col;  // rows (b, g, kb) with kb < nblk_max
  uint32_t* status;
};
cudaError_t nsa_metadata(const NsaMetaArgs& a, cudaStream_t st);
struct NsaArgs {
  int B, T, N1, N2, K, sel_block, nblk_max, mask_mode;
  int D;  // head dim of q and k: 128, or 192 (with G <= 16); v, Out and dOut have 128
  float scale;
  const int32_t *cu_seqlens, *ok_flag, *ids, *cnt, *dup, *t_row_ptr, *t_col;
  const void *q, *k, *v, *out_in, *dout;
  const float* lse_in;
  float *lse2, *dvec;
  void *out, *dq, *dk, *dv;
  float* lse_out;
  uint32_t* status;
};
cudaError_t nsa_fwd_launch(const NsaArgs& a, cudaStream_t st);
// token-major passes on tcgen05 (nsa_tc.cu): Out / LSE, and dQ (needs lse2 / dvec from the
// backward preprocess)
cudaError_t nsa_fwd_tc_launch(const NsaArgs& a, cudaStream_t st);
cudaError_t nsa_dq_tc_launch(const NsaArgs& a, cudaStream_t st);
cudaError_t nsa_bwd_launch(const NsaArgs& a, cudaStream_t st);
// dK/dV on tcgen05 (nsa_dkdv.cu) for 64-token blocks and G in {8, 16, 32, 64, 128};
// cudaErrorNotSupported for other shapes.  Needs lse2/dvec from the backward preprocess.
bool nsa_dkdv_tc_supported(const NsaArgs& a);
cudaError_t nsa_dkdv_tc_launch(const NsaArgs& a, cudaStream_t st);

// ---- diagnostics (diag.cu) -----------------------------------------------------------------------
cudaError_t diag_mma_tile_launch(const void* a, const void* b, float* c, int n, int b_mn_major, uint32_t* status,
                                 cudaStream_t st);
cudaError_t diag_exp2_launch(const float* x, float* y, int n, int degree, cudaStream_t st);
cudaError_t diag_wait_launch(uint32_t* status, int arrive, cudaStream_t st);

}  // namespace sa
