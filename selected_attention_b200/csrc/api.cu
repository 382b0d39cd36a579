// C ABI entry points: host validation (the pages' constraints), workspace layout, launches.
// Nothing here allocates memory or synchronises, except bsa_get_status.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>

#include "internal.h"

using namespace sa;

namespace {

inline int div_up(int a, int b) { return (a + b - 1) / b; }

// ---- BSA (BlockSparseAttentionGrad page constraints) -------------------------------------------
// N1 at least N2 and a multiple of it (the GQA rule), head dim 128; layouts BNSD.  Block shape:
// block_x <= 128 (one 128-row MMA tile per Q block), block_y 64 or 128.
bsa_status check_bsa(const bsa_params* p) {
  if (!p) return BSA_ERR_NULLPTR;
  if (p->q_layout != BSA_LAYOUT_BNSD && p->q_layout != BSA_LAYOUT_BSND) return BSA_ERR_UNSUPPORTED;
  if (p->kv_layout != p->q_layout) return BSA_ERR_UNSUPPORTED;
  if (p->B <= 0 || p->N1 <= 0 || p->N2 <= 0 || p->S_q <= 0 || p->S_kv <= 0) return BSA_ERR_INVALID_ARG;
  if (p->N1 < p->N2 || p->N1 % p->N2 != 0) return BSA_ERR_INVALID_ARG;
  if (p->D != 128 || p->Dv != 128) return BSA_ERR_UNSUPPORTED;
  if (p->block_x <= 0 || p->block_y <= 0) return BSA_ERR_INVALID_ARG;
  if (p->block_x > 128 || (p->block_y != 64 && p->block_y != 128)) return BSA_ERR_UNSUPPORTED;
  if (p->mask_mode != BSA_MASK_NONE && p->mask_mode != BSA_MASK_CAUSAL && p->mask_mode != BSA_MASK_RIGHT_DOWN_CAUSAL &&
      p->mask_mode != BSA_MASK_BAND)
    return BSA_ERR_INVALID_ARG;
  if (p->mask_mode == BSA_MASK_BAND && (p->win_left < 0 || p->win_right < 0)) return BSA_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale) || p->scale <= 0.f) return BSA_ERR_INVALID_ARG;  // a positive softmax scale
  const long long rows_q = 1LL * p->B * p->N1 * p->S_q, rows_kv = 1LL * p->B * p->N2 * p->S_kv;
  if (rows_q + 256 >= (1LL << 31) || rows_kv + 256 >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  const long long nqb = div_up(p->S_q, p->block_x), nkb = div_up(p->S_kv, p->block_y);
  if (1LL * p->B * p->N1 * nqb * nkb >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  if (1LL * p->B * p->N1 > 65535) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

// A metadata plan passed in bsa_params::plan: 256-byte aligned and made by one of the ops `a`, `b`.
bsa_status check_plan(const bsa_params* p, int32_t a, int32_t b) {
  if (!p->plan) return BSA_OK;
  if (reinterpret_cast<uintptr_t>(p->plan) % 256 != 0) return BSA_ERR_INVALID_ARG;
  return (p->plan_op == a || p->plan_op == b) ? BSA_OK : BSA_ERR_INVALID_ARG;
}

// Array `i` of a plan made by `op` for problem `p` (the layout sparse_attn_metadata_layout gives).
template <class T>
T* plan_array(const bsa_params* p, int32_t op, int i) {
  bsa_meta_layout L;
  if (sparse_attn_metadata_layout(p, op, &L) != BSA_OK) return nullptr;
  return reinterpret_cast<T*>(static_cast<char*>(const_cast<void*>(p->plan)) + L.offsets[i]);
}

// Without a plan the forward builds its KV lists in the workspace; with one it needs only the
// workspace header.
struct BsaFwdWs {
  uint32_t* status;
  int32_t *counts, *row_ptr, *col;
};

size_t carve_bsa_fwd(const bsa_params* p, void* ws, BsaFwdWs* w) {
  Carver c(ws);
  const int nqb = div_up(p->S_q, p->block_x), nkb = div_up(p->S_kv, p->block_y);
  const size_t units = static_cast<size_t>(p->B) * p->N1 * nqb;
  w->status = static_cast<uint32_t*>(ws);
  w->counts = w->row_ptr = w->col = nullptr;
  if (!p->plan) {
    w->counts = c.take<int32_t>(units);
    w->row_ptr = c.take<int32_t>(units + 1);
    w->col = c.take<int32_t>(units * nkb);
  } else if (ws) {
    w->row_ptr = plan_array<int32_t>(p, p->plan_op, 1);
    w->col = plan_array<int32_t>(p, p->plan_op, 2);
  }
  return c.bytes();
}

struct BsaBwdWs {
  uint32_t* status;
  int32_t *counts, *row_ptr, *col;
  uint8_t* maskT;
  int32_t *t_counts, *t_row_ptr, *t_col;
  float *dvec, *lse2;
  uint16_t *q16, *k16, *v16, *do16;
};

size_t carve_bsa_bwd(const bsa_params* p, void* ws, BsaBwdWs* w) {
  Carver c(ws);
  const int nqb = div_up(p->S_q, p->block_x), nkb = div_up(p->S_kv, p->block_y);
  const size_t units = static_cast<size_t>(p->B) * p->N1 * nqb;
  const size_t t_rows = static_cast<size_t>(p->B) * p->N2 * nkb;
  w->status = static_cast<uint32_t*>(ws);
  w->counts = w->row_ptr = w->col = w->t_counts = w->t_row_ptr = w->t_col = nullptr;
  w->maskT = nullptr;
  if (!p->plan) {
    w->counts = c.take<int32_t>(units);
    w->row_ptr = c.take<int32_t>(units + 1);
    w->col = c.take<int32_t>(units * nkb);
    w->maskT = c.take<uint8_t>(units * nkb);
    w->t_counts = c.take<int32_t>(t_rows);
    w->t_row_ptr = c.take<int32_t>(t_rows + 1);
    w->t_col = c.take<int32_t>(units * nkb);
  } else if (ws) {  // a BSA_META_BSA_BWD plan
    w->row_ptr = plan_array<int32_t>(p, BSA_META_BSA_BWD, 1);
    w->col = plan_array<int32_t>(p, BSA_META_BSA_BWD, 2);
    w->t_row_ptr = plan_array<int32_t>(p, BSA_META_BSA_BWD, 3);
    w->t_col = plan_array<int32_t>(p, BSA_META_BSA_BWD, 4);
  }
  w->dvec = c.take<float>(units * 128);
  w->lse2 = c.take<float>(units * 128);
  const size_t nq = static_cast<size_t>(p->B) * p->N1 * p->S_q * p->D;
  const size_t nk = static_cast<size_t>(p->B) * p->N2 * p->S_kv * p->D;
  w->q16 = c.take<uint16_t>(nq);
  w->do16 = c.take<uint16_t>(nq);
  w->k16 = c.take<uint16_t>(nk);
  w->v16 = c.take<uint16_t>(nk);
  return c.bytes();
}

// ---- SFA (SparseFlashAttention page constraints) ----------------------------------------------------
// query / key / value dims 512 with a 64-dim rope part; the page size a multiple of 16 up to 1024
// (this library's TMA boxes of 32 or 64 tokens must divide the page, hence a multiple of 32);
// the sparse block size must be a whole number of pages; decode: one query row per batch.
bsa_status check_sfa(const bsa_params* p) {
  if (!p) return BSA_ERR_NULLPTR;
  if (p->kv_layout != BSA_LAYOUT_PA_ND) return BSA_ERR_UNSUPPORTED;
  if (p->B <= 0 || p->N1 <= 0 || p->N2 <= 0) return BSA_ERR_INVALID_ARG;
  if (p->N1 < p->N2 || p->N1 % p->N2 != 0) return BSA_ERR_INVALID_ARG;
  if (p->N1 / p->N2 > 128) return BSA_ERR_UNSUPPORTED;
  if (p->S_q != 1) return BSA_ERR_UNSUPPORTED;
  if (p->D != 512 || p->Dv != 512 || p->D_rope != 64) return BSA_ERR_UNSUPPORTED;
  if (p->page_size <= 0 || p->page_size % 16 != 0 || p->page_size > 1024) return BSA_ERR_INVALID_ARG;
  if (p->page_size % 32 != 0) return BSA_ERR_UNSUPPORTED;
  if (p->sparse_block_size <= 0 || p->sparse_block_size % p->page_size != 0) return BSA_ERR_INVALID_ARG;
  if (p->sparse_count <= 0 || p->max_pages_per_seq <= 0 || p->num_pages <= 0) return BSA_ERR_INVALID_ARG;
  if (1LL * p->num_pages * p->page_size * p->N2 >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  if (!std::isfinite(p->scale) || p->scale <= 0.f) return BSA_ERR_INVALID_ARG;
  return BSA_OK;
}

// ---- NSA (NsaSelectedAttention page constraints) -------------------------------------------------
// TND only; sparseMode 0 or 2; selected_block_size <= 128 and a multiple of 16; selected block
// count in [1, 128] with count * size <= 8K; B in [1, 1024], N1 in [1, 128], N2 in [1, 32]; each
// batch's length up to 128K (S_q carries the longest one); query and key lengths equal.
bsa_status check_nsa(const bsa_params* p) {
  if (!p) return BSA_ERR_NULLPTR;
  if (p->q_layout != BSA_LAYOUT_TND || p->kv_layout != BSA_LAYOUT_TND) return BSA_ERR_UNSUPPORTED;
  if (p->B < 1 || p->B > 1024 || p->N1 < 1 || p->N1 > 128 || p->N2 < 1 || p->N2 > 32) return BSA_ERR_INVALID_ARG;
  if (p->N1 < p->N2 || p->N1 % p->N2 != 0) return BSA_ERR_INVALID_ARG;
  // head dims: 128 / 128, or 192 for q / k with 128 for v (query groups of at most 16 heads)
  if (p->Dv != 128 || (p->D != 128 && p->D != 192)) return BSA_ERR_UNSUPPORTED;
  if (p->D == 192 && p->N1 / p->N2 > 16) return BSA_ERR_UNSUPPORTED;
  if (p->T_q <= 0 || p->T_q != p->T_kv) return BSA_ERR_INVALID_ARG;
  if (p->S_q <= 0 || p->S_q > 128 * 1024 || p->S_q > p->T_q) return BSA_ERR_INVALID_ARG;
  if (p->sel_block_size <= 0 || p->sel_block_size > 128 || p->sel_block_size % 16 != 0) return BSA_ERR_INVALID_ARG;
  if (p->sel_block_count < 1 || p->sel_block_count > 128 || p->sel_block_count * p->sel_block_size > 8192)
    return BSA_ERR_INVALID_ARG;
  if (p->mask_mode != BSA_MASK_NONE && p->mask_mode != BSA_MASK_CAUSAL) return BSA_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale) || p->scale <= 0.f) return BSA_ERR_INVALID_ARG;
  if (1LL * p->T_q * p->N1 * 128 >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

struct NsaWs {
  uint32_t* status;
  int32_t *ok_flag, *ids, *cnt, *dup;
  uint32_t* bitmap;
  int32_t *t_counts, *t_row_ptr, *t_col;
  float *lse2, *dvec;
  int nblk_max, words;
  size_t off_ids, off_cnt, off_t_row_ptr, off_t_col;  // byte offsets, for the metadata layout
};

// The NSA workspace without a plan (and the layout of an NSA plan: the metadata op writes the
// same arrays).
size_t carve_nsa_lists(const bsa_params* p, void* ws, NsaWs* w, bool bwd) {
  Carver c(ws);
  w->nblk_max = div_up(p->S_q, p->sel_block_size);
  w->words = div_up(p->T_q, 32);
  const size_t rows = static_cast<size_t>(p->T_q) * p->N2;
  w->status = static_cast<uint32_t*>(ws);
  w->ok_flag = c.take<int32_t>(1);
  w->off_ids = c.next();
  w->ids = c.take<int32_t>(rows * p->sel_block_count);
  w->off_cnt = c.next();
  w->cnt = c.take<int32_t>(rows);
  w->dup = c.take<int32_t>(rows);
  w->bitmap = nullptr;
  w->off_t_row_ptr = w->off_t_col = 0;
  w->t_counts = w->t_row_ptr = w->t_col = nullptr;
  w->lse2 = w->dvec = nullptr;
  if (bwd) {
    w->bitmap = c.take<uint32_t>(static_cast<size_t>(p->N2) * w->nblk_max * w->words);
    const size_t trows = static_cast<size_t>(p->B) * p->N2 * w->nblk_max;
    w->t_counts = c.take<int32_t>(trows);
    w->off_t_row_ptr = c.next();
    w->t_row_ptr = c.take<int32_t>(trows + 1);
    w->off_t_col = c.next();
    w->t_col = c.take<int32_t>(rows * p->sel_block_count);
    w->lse2 = c.take<float>(static_cast<size_t>(p->T_q) * p->N1);
    w->dvec = c.take<float>(static_cast<size_t>(p->T_q) * p->N1);
  }
  return c.bytes();
}

// An op's workspace: with a plan the lists (and the cu_seqlens check flag) are the plan's, laid
// out as a plan-less workspace of op plan_op, and the workspace keeps only the backward's scratch.
size_t carve_nsa(const bsa_params* p, void* ws, NsaWs* w, bool bwd) {
  if (!p->plan) return carve_nsa_lists(p, ws, w, bwd);
  bsa_params lists = *p;
  lists.plan = nullptr;
  carve_nsa_lists(&lists, const_cast<void*>(p->plan), w, p->plan_op == BSA_META_NSA_TOKENS);
  Carver c(ws);
  w->status = static_cast<uint32_t*>(ws);
  w->bitmap = nullptr;
  w->t_counts = nullptr;
  w->lse2 = w->dvec = nullptr;
  if (bwd) {
    w->lse2 = c.take<float>(static_cast<size_t>(p->T_q) * p->N1);
    w->dvec = c.take<float>(static_cast<size_t>(p->T_q) * p->N1);
  }
  return c.bytes();
}

NsaMetaArgs nsa_meta_args(const bsa_params* p, const NsaWs& w, bool token_lists) {
  NsaMetaArgs m;
  m.topk = p->topk_indices; m.cu_seqlens = p->cu_seqlens_q;
  m.B = p->B; m.T = p->T_q; m.N2 = p->N2; m.K = p->sel_block_count; m.sel_block = p->sel_block_size;
  m.max_len = p->S_q; m.nblk_max = w.nblk_max; m.words = w.words; m.token_lists = token_lists;
  m.ok_flag = w.ok_flag; m.ids = w.ids; m.cnt = w.cnt; m.dup = w.dup; m.bitmap = w.bitmap;
  m.t_counts = w.t_counts; m.t_row_ptr = w.t_row_ptr; m.t_col = w.t_col; m.status = w.status;
  return m;
}

NsaArgs nsa_args(const bsa_params* p, const NsaWs& w) {
  NsaArgs a;
  a.B = p->B; a.T = p->T_q; a.N1 = p->N1; a.N2 = p->N2; a.K = p->sel_block_count; a.sel_block = p->sel_block_size;
  a.D = p->D;
  a.nblk_max = w.nblk_max; a.mask_mode = p->mask_mode; a.scale = p->scale;
  a.cu_seqlens = p->cu_seqlens_q; a.ok_flag = w.ok_flag; a.ids = w.ids; a.cnt = w.cnt; a.dup = w.dup;
  a.t_row_ptr = w.t_row_ptr; a.t_col = w.t_col;
  a.q = a.k = a.v = a.out_in = a.dout = nullptr;
  a.lse_in = nullptr; a.lse2 = w.lse2; a.dvec = w.dvec;
  a.out = a.dq = a.dk = a.dv = nullptr; a.lse_out = nullptr; a.status = w.status;
  return a;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Decode workspace: per piece, the unit's compacted page list (pages, tokens; K * ppb entries
// each) and its set-up record (n, begin, len).  The metadata op BSA_META_SFA_WORK fills the same
// arrays with the same device code.
struct SfaWs {
  uint32_t* status;
  int32_t *pages, *tokens, *rec;
  int cap, per, units, P, pieces;
  size_t off_pages, off_tokens, off_rec;
};

size_t carve_sfa(const bsa_params* p, void* ws, SfaWs* w) {
  Carver c(ws);
  const int ppb = p->sparse_block_size / p->page_size;
  w->cap = p->sparse_count * ppb;
  w->per = sfa_head_halves(p->N1 / p->N2);
  w->units = p->B * p->N2 * w->per;
  w->P = sfa_pieces_per_unit(w->units, sm_count());
  w->pieces = w->units * w->P;
  w->status = static_cast<uint32_t*>(ws);
  w->off_pages = c.next();
  w->pages = c.take<int32_t>(static_cast<size_t>(w->pieces) * w->cap);
  w->off_tokens = c.next();
  w->tokens = c.take<int32_t>(static_cast<size_t>(w->pieces) * w->cap);
  w->off_rec = c.next();
  w->rec = c.take<int32_t>(static_cast<size_t>(w->pieces) * 3);
  return c.bytes();
}

SfaMetaArgs sfa_meta_args(const bsa_params* p) {
  SfaMetaArgs m;
  m.sparse_indices = p->sparse_indices; m.block_table = p->block_table; m.seqused_kv = p->seqused_kv;
  m.B = p->B; m.N2 = p->N2; m.K = p->sparse_count; m.ppb = p->sparse_block_size / p->page_size;
  m.page_size = p->page_size; m.max_pages_per_seq = p->max_pages_per_seq; m.num_pages = p->num_pages;
  m.pages = m.tokens = m.count = nullptr;
  m.status = nullptr;
  return m;
}

bsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

bsa_status check_ws(void* ws, size_t have, size_t need) {
  if (!ws) return BSA_ERR_NULLPTR;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return BSA_ERR_INVALID_ARG;
  if (have < need) return BSA_ERR_WORKSPACE_TOO_SMALL;
  return BSA_OK;
}

}  // namespace

extern "C" {

const char* bsa_version(void) { return "selected_attention_b200 0.1 (sm_100a)"; }

bsa_status bsa_fwd_workspace_size(const bsa_params* p, size_t* bytes) {
  if (!bytes) return BSA_ERR_NULLPTR;
  bsa_status s = check_bsa(p);
  if (s == BSA_OK) s = check_plan(p, BSA_META_BSA_KV, BSA_META_BSA_BWD);
  if (s != BSA_OK) return s;
  BsaFwdWs w;
  *bytes = carve_bsa_fwd(p, nullptr, &w);
  return BSA_OK;
}

bsa_status bsa_fwd(const bsa_params* p, const void* q, const void* k, const void* v, void* out, float* lse,
                   void* workspace, size_t workspace_bytes, void* stream) {
  bsa_status s = check_bsa(p);
  if (s == BSA_OK) s = check_plan(p, BSA_META_BSA_KV, BSA_META_BSA_BWD);
  if (s != BSA_OK) return s;
  if (!q || !k || !v || !out || !lse || !p->block_mask) return BSA_ERR_NULLPTR;
  BsaFwdWs w;
  const size_t need = carve_bsa_fwd(p, nullptr, &w);
  if ((s = check_ws(workspace, workspace_bytes, need)) != BSA_OK) return s;
  carve_bsa_fwd(p, workspace, &w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nqb = div_up(p->S_q, p->block_x), nkb = div_up(p->S_kv, p->block_y);
  const int units = p->B * p->N1 * nqb;
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(WsHeader), st);
  if (e == cudaSuccess && !p->plan) e = bsa_kv_lists(p->block_mask, units, nkb, w.counts, w.row_ptr, w.col, st);
  if (e != cudaSuccess) return BSA_ERR_CUDA;
  BsaFwdArgs a;
  a.next_unit = &reinterpret_cast<WsHeader*>(w.status)->next_fwd;
  a.B = p->B; a.N1 = p->N1; a.N2 = p->N2; a.S_q = p->S_q; a.S_kv = p->S_kv;
  a.bx = p->block_x; a.by = p->block_y; a.nqb = nqb; a.nkb = nkb;
  a.mask_mode = p->mask_mode; a.win_left = p->win_left; a.win_right = p->win_right; a.scale = p->scale;
  a.qs = bsa_strides(p->q_layout, p->N1, p->S_q, p->D);
  a.kvs = bsa_strides(p->kv_layout, p->N2, p->S_kv, p->D);
  a.lse_s = bsa_strides(p->q_layout, p->N1, p->S_q, 1);
  a.atten_mask = p->atten_mask;
  a.row_ptr = w.row_ptr; a.col = w.col; a.out = out; a.lse = lse; a.status = w.status;
  return cuda_status(bsa_fwd_launch(a, q, k, v, st));
}

bsa_status bsa_bwd_workspace_size(const bsa_params* p, size_t* bytes) {
  if (!bytes) return BSA_ERR_NULLPTR;
  bsa_status s = check_bsa(p);
  if (s == BSA_OK) s = check_plan(p, BSA_META_BSA_BWD, BSA_META_BSA_BWD);
  if (s != BSA_OK) return s;
  BsaBwdWs w;
  *bytes = carve_bsa_bwd(p, nullptr, &w);
  return BSA_OK;
}

bsa_status bsa_bwd(const bsa_params* p, const void* q, const void* k, const void* v, const void* out,
                   const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, void* stream) {
  bsa_status s = check_bsa(p);
  if (s == BSA_OK) s = check_plan(p, BSA_META_BSA_BWD, BSA_META_BSA_BWD);
  if (s != BSA_OK) return s;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !p->block_mask) return BSA_ERR_NULLPTR;
  BsaBwdWs w;
  const size_t need = carve_bsa_bwd(p, nullptr, &w);
  if ((s = check_ws(workspace, workspace_bytes, need)) != BSA_OK) return s;
  carve_bsa_bwd(p, workspace, &w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int nqb = div_up(p->S_q, p->block_x), nkb = div_up(p->S_kv, p->block_y);
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(WsHeader), st);
  if (e == cudaSuccess && !p->plan)
    e = bsa_kv_lists(p->block_mask, p->B * p->N1 * nqb, nkb, w.counts, w.row_ptr, w.col, st);
  if (e == cudaSuccess && !p->plan)
    e = bsa_q_lists(p->block_mask, p->B, p->N1, p->N2, nqb, nkb, w.maskT, w.t_counts, w.t_row_ptr, w.t_col, st);
  if (e != cudaSuccess) return BSA_ERR_CUDA;
  BsaBwdArgs a;
  a.B = p->B; a.N1 = p->N1; a.N2 = p->N2; a.S_q = p->S_q; a.S_kv = p->S_kv;
  a.bx = p->block_x; a.by = p->block_y; a.nqb = nqb; a.nkb = nkb;
  a.mask_mode = p->mask_mode; a.win_left = p->win_left; a.win_right = p->win_right; a.scale = p->scale;
  a.qs = bsa_strides(p->q_layout, p->N1, p->S_q, p->D);
  a.kvs = bsa_strides(p->kv_layout, p->N2, p->S_kv, p->D);
  a.lse_s = bsa_strides(p->q_layout, p->N1, p->S_q, 1);
  a.atten_mask = p->atten_mask;
  a.row_ptr = w.row_ptr; a.col = w.col; a.t_row_ptr = w.t_row_ptr; a.t_col = w.t_col;
  a.dvec = w.dvec; a.lse2 = w.lse2; a.dq = dq; a.dk = dk; a.dv = dv; a.status = w.status;
  a.q16 = w.q16; a.k16 = w.k16; a.v16 = w.v16; a.do16 = w.do16;
  a.amax = reinterpret_cast<WsHeader*>(w.status)->amax;
  a.next_kv = &reinterpret_cast<WsHeader*>(w.status)->next_bwd_kv;
  a.next_q = &reinterpret_cast<WsHeader*>(w.status)->next_bwd_q;
  return cuda_status(bsa_bwd_launch(a, q, k, v, out, dout, lse, st));
}
bsa_status nsa_selected_fwd_workspace_size(const bsa_params* p, size_t* bytes) {
  if (!bytes) return BSA_ERR_NULLPTR;
  bsa_status s = check_nsa(p);
  if (s == BSA_OK) s = check_plan(p, BSA_META_NSA_KV, BSA_META_NSA_TOKENS);
  if (s != BSA_OK) return s;
  NsaWs w;
  *bytes = carve_nsa(p, nullptr, &w, false);
  return BSA_OK;
}

bsa_status nsa_selected_bwd_workspace_size(const bsa_params* p, size_t* bytes) {
  if (!bytes) return BSA_ERR_NULLPTR;
  bsa_status s = check_nsa(p);
  if (s == BSA_OK) s = check_plan(p, BSA_META_NSA_TOKENS, BSA_META_NSA_TOKENS);
  if (s != BSA_OK) return s;
  NsaWs w;
  *bytes = carve_nsa(p, nullptr, &w, true);
  return BSA_OK;
}

bsa_status nsa_selected_fwd(const bsa_params* p, const void* q, const void* k, const void* v, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream) {
  bsa_status s = check_nsa(p);
  if (s == BSA_OK) s = check_plan(p, BSA_META_NSA_KV, BSA_META_NSA_TOKENS);
  if (s != BSA_OK) return s;
  if (!q || !k || !v || !out || !lse || !p->topk_indices || !p->cu_seqlens_q) return BSA_ERR_NULLPTR;
  NsaWs w;
  const size_t need = carve_nsa(p, nullptr, &w, false);
  if ((s = check_ws(workspace, workspace_bytes, need)) != BSA_OK) return s;
  carve_nsa(p, workspace, &w, false);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st) != cudaSuccess) return BSA_ERR_CUDA;
  if (!p->plan && nsa_metadata(nsa_meta_args(p, w, false), st) != cudaSuccess) return BSA_ERR_CUDA;
  NsaArgs a = nsa_args(p, w);
  a.q = q; a.k = k; a.v = v; a.out = out; a.lse_out = lse;
  return cuda_status(nsa_fwd_launch(a, st));
}

bsa_status nsa_selected_bwd(const bsa_params* p, const void* q, const void* k, const void* v, const void* out,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                            size_t workspace_bytes, void* stream) {
  bsa_status s = check_nsa(p);
  if (s == BSA_OK) s = check_plan(p, BSA_META_NSA_TOKENS, BSA_META_NSA_TOKENS);
  if (s != BSA_OK) return s;
  if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !p->topk_indices || !p->cu_seqlens_q)
    return BSA_ERR_NULLPTR;
  NsaWs w;
  const size_t need = carve_nsa(p, nullptr, &w, true);
  if ((s = check_ws(workspace, workspace_bytes, need)) != BSA_OK) return s;
  carve_nsa(p, workspace, &w, true);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st) != cudaSuccess) return BSA_ERR_CUDA;
  if (!p->plan && nsa_metadata(nsa_meta_args(p, w, true), st) != cudaSuccess) return BSA_ERR_CUDA;
  NsaArgs a = nsa_args(p, w);
  a.q = q; a.k = k; a.v = v; a.out_in = out; a.dout = dout; a.lse_in = lse; a.dq = dq; a.dk = dk; a.dv = dv;
  return cuda_status(nsa_bwd_launch(a, st));
}
bsa_status sfa_sparse_decode_workspace_size(const bsa_params* p, size_t* bytes) {
  if (!bytes) return BSA_ERR_NULLPTR;
  bsa_status s = check_sfa(p);
  if (s != BSA_OK) return s;
  if (p->plan) return BSA_ERR_UNSUPPORTED;  // the decode builds its page lists in its prologue
  SfaWs w;
  *bytes = carve_sfa(p, nullptr, &w);
  return BSA_OK;
}

bsa_status sfa_sparse_decode(const bsa_params* p, const void* q, const void* q_rope, const void* k_cache,
                             const void* k_rope_cache, const void* v_cache, void* out, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream) {
  bsa_status s = check_sfa(p);
  if (s != BSA_OK) return s;
  if (p->plan) return BSA_ERR_UNSUPPORTED;
  if (!q || !q_rope || !k_cache || !k_rope_cache || !v_cache || !out || !lse || !p->block_table ||
      !p->sparse_indices || !p->seqused_kv)
    return BSA_ERR_NULLPTR;
  SfaWs w;
  const size_t need = carve_sfa(p, nullptr, &w);
  if ((s = check_ws(workspace, workspace_bytes, need)) != BSA_OK) return s;
  carve_sfa(p, workspace, &w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return BSA_ERR_CUDA;
  SfaDecodeArgs a;
  a.B = p->B; a.N1 = p->N1; a.N2 = p->N2; a.K = p->sparse_count; a.ppb = p->sparse_block_size / p->page_size;
  a.page_size = p->page_size; a.max_pages_per_seq = p->max_pages_per_seq; a.num_pages = p->num_pages;
  a.units = w.units; a.P = w.P; a.scale = p->scale;
  a.q = q; a.q_rope = q_rope; a.k_cache = k_cache; a.k_rope_cache = k_rope_cache; a.v_cache = v_cache;
  a.sparse_indices = p->sparse_indices; a.block_table = p->block_table; a.seqused_kv = p->seqused_kv;
  a.pages = w.pages; a.tokens = w.tokens; a.rec = w.rec;
  a.out = out; a.lse = lse; a.status = w.status;
  return cuda_status(sfa_decode_launch(a, st));
}

// Backward of the decode: the unit's page lists, the preprocess, the per-tile dQ parts, the
// gathered-order row gradients and the readers of every cache row-block.
struct SfaBwdWs {
  uint32_t* status;
  int32_t *pages, *tokens, *count, *cnt, *ptr, *list;
  float *lse2, *dvec;
  uint16_t *ds, *gk, *gv;
};

size_t carve_sfa_bwd(const bsa_params* p, void* ws, SfaBwdWs* w) {
  Carver c(ws);
  const size_t U = static_cast<size_t>(p->B) * p->N2;
  const size_t cap = static_cast<size_t>(p->sparse_count) * (p->sparse_block_size / p->page_size);
  const size_t rows = U * cap * p->page_size;
  const size_t keys = static_cast<size_t>(p->num_pages) * p->N2;
  const size_t T = static_cast<size_t>(sfa_bwd_tiles(static_cast<int>(cap), p->page_size));
  w->status = static_cast<uint32_t*>(ws);
  w->pages = c.take<int32_t>(U * cap);
  w->tokens = c.take<int32_t>(U * cap);
  w->count = c.take<int32_t>(U);
  w->cnt = c.take<int32_t>(2 * keys);
  w->ptr = c.take<int32_t>(keys + 1);
  w->list = c.take<int32_t>(U * cap);
  w->lse2 = c.take<float>(static_cast<size_t>(p->B) * p->N1);
  w->dvec = c.take<float>(static_cast<size_t>(p->B) * p->N1);
  w->ds = c.take<uint16_t>(U * T * 128 * 128);
  w->gk = c.take<uint16_t>(rows * 576);
  w->gv = c.take<uint16_t>(rows * 512);
  return c.bytes();
}

bsa_status sfa_sparse_decode_bwd_workspace_size(const bsa_params* p, size_t* bytes) {
  if (!bytes) return BSA_ERR_NULLPTR;
  bsa_status s = check_sfa(p);
  if (s != BSA_OK) return s;
  if (p->plan) return BSA_ERR_UNSUPPORTED;
  if (1LL * p->num_pages * p->N2 >= (1LL << 30)) return BSA_ERR_UNSUPPORTED;
  SfaBwdWs w;
  *bytes = carve_sfa_bwd(p, nullptr, &w);
  return BSA_OK;
}

bsa_status sfa_sparse_decode_bwd(const bsa_params* p, const void* q, const void* q_rope, const void* k_cache,
                                 const void* k_rope_cache, const void* v_cache, const void* out, const void* dout,
                                 const float* lse, void* dq, void* dq_rope, void* dk_cache, void* dk_rope_cache,
                                 void* dv_cache, void* workspace, size_t workspace_bytes, void* stream) {
  size_t need = 0;
  bsa_status s = sfa_sparse_decode_bwd_workspace_size(p, &need);
  if (s != BSA_OK) return s;
  if (!q || !q_rope || !k_cache || !k_rope_cache || !v_cache || !out || !dout || !lse || !dq || !dq_rope ||
      !dk_cache || !dk_rope_cache || !dv_cache || !p->block_table || !p->sparse_indices || !p->seqused_kv)
    return BSA_ERR_NULLPTR;
  if ((s = check_ws(workspace, workspace_bytes, need)) != BSA_OK) return s;
  SfaBwdWs w;
  carve_sfa_bwd(p, workspace, &w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st) != cudaSuccess) return BSA_ERR_CUDA;
  SfaBwdArgs a;
  a.meta = sfa_meta_args(p);
  a.meta.pages = w.pages; a.meta.tokens = w.tokens; a.meta.count = w.count; a.meta.status = w.status;
  a.B = p->B; a.N1 = p->N1; a.N2 = p->N2; a.page_size = p->page_size; a.num_pages = p->num_pages;
  a.cap = p->sparse_count * (p->sparse_block_size / p->page_size);
  a.scale = p->scale;
  a.q = q; a.q_rope = q_rope; a.k_cache = k_cache; a.k_rope_cache = k_rope_cache; a.v_cache = v_cache;
  a.out = out; a.dout = dout; a.lse = lse;
  a.dq = dq; a.dq_rope = dq_rope; a.dk_cache = dk_cache; a.dk_rope_cache = dk_rope_cache; a.dv_cache = dv_cache;
  a.lse2 = w.lse2; a.dvec = w.dvec; a.ds = w.ds; a.gk = w.gk; a.gv = w.gv;
  a.cnt = w.cnt; a.ptr = w.ptr; a.list = w.list;
  return cuda_status(sfa_bwd_launch(a, st));
}

// ---- metadata -------------------------------------------------------------------------------------
bsa_status sparse_attn_metadata_layout(const bsa_params* p, int32_t op, bsa_meta_layout* layout) {
  if (!layout) return BSA_ERR_NULLPTR;
  std::memset(layout, 0, sizeof(*layout));
  if (op == BSA_META_BSA_BWD) {
    bsa_status s = check_bsa(p);
    if (s != BSA_OK) return s;
    const int nqb = div_up(p->S_q, p->block_x), nkb = div_up(p->S_kv, p->block_y);
    const size_t units = static_cast<size_t>(p->B) * p->N1 * nqb;
    const size_t t_rows = static_cast<size_t>(p->B) * p->N2 * nkb;
    const size_t ents = units * nkb;
    Carver c(nullptr);
    layout->offsets[0] = 0;
    layout->offsets[1] = c.next();  // row_ptr (per (b, h, qb))
    c.take<int32_t>(units + 1);
    layout->offsets[2] = c.next();  // col
    c.take<int32_t>(ents);
    layout->offsets[3] = c.next();  // transposed row_ptr (per (b, g, kb))
    c.take<int32_t>(t_rows + 1);
    layout->offsets[4] = c.next();  // transposed col
    c.take<int32_t>(ents);
    layout->offsets[5] = c.next();  // scratch: counts, transposed counts, transposed mask
    c.take<int32_t>(units);
    c.take<int32_t>(t_rows);
    c.take<uint8_t>(ents);
    layout->count = 6;
    layout->total_bytes = c.bytes();
    return BSA_OK;
  }
  if (op == BSA_META_BSA_KV || op == BSA_META_BSA_Q) {
    bsa_status s = check_bsa(p);
    if (s != BSA_OK) return s;
    const int nqb = div_up(p->S_q, p->block_x), nkb = div_up(p->S_kv, p->block_y);
    Carver c(nullptr);
    const size_t rows = op == BSA_META_BSA_KV ? static_cast<size_t>(p->B) * p->N1 * nqb
                                              : static_cast<size_t>(p->B) * p->N2 * nkb;
    const size_t ents = static_cast<size_t>(p->B) * p->N1 * nqb * nkb;
    layout->offsets[0] = 0;
    c.take<int32_t>(0);
    layout->offsets[1] = c.off;  // row_ptr
    c.take<int32_t>(rows + 1);
    c.off = align_up(c.off, 256);
    layout->offsets[2] = c.off;  // col
    c.take<int32_t>(ents);
    c.off = align_up(c.off, 256);
    layout->offsets[3] = c.off;  // counts (scratch)
    c.take<int32_t>(rows);
    if (op == BSA_META_BSA_Q) {
      c.off = align_up(c.off, 256);
      layout->offsets[4] = c.off;  // transposed mask (scratch)
      c.take<uint8_t>(ents);
    }
    layout->count = op == BSA_META_BSA_Q ? 5 : 4;
    layout->total_bytes = c.bytes();
    return BSA_OK;
  }
  if (op == BSA_META_NSA_KV || op == BSA_META_NSA_TOKENS) {
    bsa_status s = check_nsa(p);
    if (s != BSA_OK) return s;
    NsaWs w;
    const bool tok = op == BSA_META_NSA_TOKENS;
    layout->total_bytes = carve_nsa_lists(p, nullptr, &w, tok);
    layout->offsets[1] = w.off_ids;
    layout->offsets[2] = w.off_cnt;
    layout->offsets[3] = w.off_t_row_ptr;
    layout->offsets[4] = w.off_t_col;
    layout->offsets[0] = 0;
    layout->count = tok ? 5 : 3;
    return BSA_OK;
  }
  if (op == BSA_META_SFA_PAGES) {
    bsa_status s = check_sfa(p);
    if (s != BSA_OK) return s;
    const size_t lists = static_cast<size_t>(p->B) * p->N2 * p->sparse_count * (p->sparse_block_size / p->page_size);
    Carver c(nullptr);
    layout->offsets[0] = 0;
    c.off = align_up(c.off, 256);
    layout->offsets[1] = c.off;  // pages [B*N2][cap], compacted
    c.take<int32_t>(lists);
    c.off = align_up(c.off, 256);
    layout->offsets[2] = c.off;  // tokens [B*N2][cap]
    c.take<int32_t>(lists);
    c.off = align_up(c.off, 256);
    layout->offsets[3] = c.off;  // count [B*N2]
    c.take<int32_t>(static_cast<size_t>(p->B) * p->N2);
    layout->count = 4;
    layout->total_bytes = c.bytes();
    return BSA_OK;
  }
  if (op == BSA_META_SFA_WORK) {
    bsa_status s = check_sfa(p);
    if (s != BSA_OK) return s;
    SfaWs w;
    layout->total_bytes = carve_sfa(p, nullptr, &w);
    layout->offsets[0] = 0;
    layout->offsets[1] = w.off_pages;   // pages [pieces][cap]
    layout->offsets[2] = w.off_tokens;  // tokens [pieces][cap]
    layout->offsets[3] = w.off_rec;     // (n, begin, len) [pieces][3]
    layout->count = 4;
    layout->info[0] = static_cast<size_t>(w.pieces);
    layout->info[1] = static_cast<size_t>(w.P);
    return BSA_OK;
  }
  return BSA_ERR_UNSUPPORTED;
}

bsa_status sparse_attn_metadata(const bsa_params* p, int32_t op, void* plan, size_t plan_bytes, void* stream) {
  bsa_meta_layout L;
  bsa_status s = sparse_attn_metadata_layout(p, op, &L);
  if (s != BSA_OK) return s;
  if ((s = check_ws(plan, plan_bytes, L.total_bytes)) != BSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(plan);
  if (op == BSA_META_NSA_KV || op == BSA_META_NSA_TOKENS) {
    if (!p->topk_indices || !p->cu_seqlens_q) return BSA_ERR_NULLPTR;
    if (cudaMemsetAsync(plan, 0, sizeof(uint32_t), st) != cudaSuccess) return BSA_ERR_CUDA;
    NsaWs w;
    carve_nsa_lists(p, plan, &w, op == BSA_META_NSA_TOKENS);
    return cuda_status(nsa_metadata(nsa_meta_args(p, w, op == BSA_META_NSA_TOKENS), st));
  }
  if (op == BSA_META_SFA_PAGES || op == BSA_META_SFA_WORK) {
    if (!p->block_table || !p->sparse_indices || !p->seqused_kv) return BSA_ERR_NULLPTR;
    if (cudaMemsetAsync(plan, 0, sizeof(uint32_t), st) != cudaSuccess) return BSA_ERR_CUDA;
    SfaMetaArgs m = sfa_meta_args(p);
    m.status = static_cast<uint32_t*>(plan);
    m.pages = reinterpret_cast<int32_t*>(base + L.offsets[1]);
    m.tokens = reinterpret_cast<int32_t*>(base + L.offsets[2]);
    if (op == BSA_META_SFA_PAGES) {
      m.count = reinterpret_cast<int32_t*>(base + L.offsets[3]);
      return cuda_status(sfa_page_list(m, st));
    }
    SfaWs w;
    carve_sfa(p, nullptr, &w);
    return cuda_status(sfa_pieces(m, w.P, w.per, w.pieces, reinterpret_cast<int32_t*>(base + L.offsets[3]), st));
  }
  if (!p->block_mask) return BSA_ERR_NULLPTR;
  const int nqb = div_up(p->S_q, p->block_x), nkb = div_up(p->S_kv, p->block_y);
  cudaError_t e = cudaMemsetAsync(plan, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return BSA_ERR_CUDA;
  int32_t* row_ptr = reinterpret_cast<int32_t*>(base + L.offsets[1]);
  int32_t* col = reinterpret_cast<int32_t*>(base + L.offsets[2]);
  if (op == BSA_META_BSA_BWD) {
    Carver c(base + L.offsets[5]);
    c.off = 0;
    const size_t units = static_cast<size_t>(p->B) * p->N1 * nqb;
    int32_t* counts = c.take<int32_t>(units);
    int32_t* t_counts = c.take<int32_t>(static_cast<size_t>(p->B) * p->N2 * nkb);
    uint8_t* maskT = c.take<uint8_t>(units * nkb);
    e = bsa_kv_lists(p->block_mask, static_cast<int>(units), nkb, counts, row_ptr, col, st);
    if (e == cudaSuccess)
      e = bsa_q_lists(p->block_mask, p->B, p->N1, p->N2, nqb, nkb, maskT, t_counts,
                      reinterpret_cast<int32_t*>(base + L.offsets[3]), reinterpret_cast<int32_t*>(base + L.offsets[4]),
                      st);
    return cuda_status(e);
  }
  int32_t* counts = reinterpret_cast<int32_t*>(base + L.offsets[3]);
  if (op == BSA_META_BSA_KV)
    e = bsa_kv_lists(p->block_mask, p->B * p->N1 * nqb, nkb, counts, row_ptr, col, st);
  else
    e = bsa_q_lists(p->block_mask, p->B, p->N1, p->N2, nqb, nkb, reinterpret_cast<uint8_t*>(base + L.offsets[4]),
                    counts, row_ptr, col, st);
  return cuda_status(e);
}

bsa_status bsa_partition(const int64_t* weights, int32_t n, int32_t parts, int32_t* starts) {
  if (!starts || (n > 0 && !weights)) return BSA_ERR_NULLPTR;
  if (n < 0 || parts < 1) return BSA_ERR_INVALID_ARG;
  __int128 total = 0;
  for (int32_t i = 0; i < n; ++i) {
    if (weights[i] < 0) return BSA_ERR_INVALID_ARG;
    total += weights[i];
  }
  int32_t t = 0;
  __int128 prefix = 0;  // prefix(t)
  for (int32_t s = 0; s < parts; ++s) {
    const __int128 target = (static_cast<__int128>(s) * total + parts - 1) / parts;  // ceil(s W / parts)
    while (prefix < target && t < n) prefix += weights[t++];
    starts[s] = t;
  }
  starts[parts] = n;
  return BSA_OK;
}

bsa_status bsa_get_status(const void* workspace, void* stream, uint32_t* dev_bits) {
  if (!workspace || !dev_bits) return BSA_ERR_NULLPTR;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return BSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return BSA_ERR_CUDA;
  *dev_bits = v;
  return BSA_OK;
}

// ---- diagnostics ------------------------------------------------------------------------------------
bsa_status bsa_diag_mma_tile(const void* a, const void* b, float* c, int32_t b_mn_major, void* workspace,
                             void* stream) {
  if (!a || !b || !c || !workspace) return BSA_ERR_NULLPTR;
  if (b_mn_major < 0 || b_mn_major > 5) return BSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess) return BSA_ERR_CUDA;
  return cuda_status(diag_mma_tile_launch(a, b, c, 128, b_mn_major, static_cast<uint32_t*>(workspace), st));
}

bsa_status bsa_diag_wait(void* workspace, int32_t arrive, void* stream) {
  if (!workspace) return BSA_ERR_NULLPTR;
  if (arrive != 0 && arrive != 1) return BSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess) return BSA_ERR_CUDA;
  return cuda_status(diag_wait_launch(static_cast<uint32_t*>(workspace), arrive, st));
}

bsa_status bsa_diag_exp2(const float* x, float* y, int32_t n, int32_t degree, void* stream) {
  if (!x || !y) return BSA_ERR_NULLPTR;
  if (n < 0 || (degree != 3 && degree != 4)) return BSA_ERR_INVALID_ARG;
  return cuda_status(diag_exp2_launch(x, y, n, degree, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
