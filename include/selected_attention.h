/*
 * selected_attention.h — C ABI of the B200 (sm_100a) block-sparse attention library.
 *
 * Operations (each cites the page that defines what it computes):
 *   bsa_fwd / bsa_bwd           block-sparse attention, KV blocks chosen per Q block by a
 *                               BlockSparseMask bitmap ("aclnnBlockSparseAttentionGrad" page,
 *                               forward formula and backward formulas).
 *   nsa_selected_fwd / _bwd     NSA selected attention: per-token topk_indices gather, TND
 *                               varlen, GQA ("aclnnNsaSelectedAttention" page, forward formula;
 *                               the backward applies the BlockSparseAttentionGrad formulas to the
 *                               gathered blocks).
 *   sfa_sparse_decode / _bwd    sparse flash attention decode over a paged KV cache with a rope
 *                               sub-head ("aclnnSparseFlashAttention" page, formula and
 *                               constraints); the backward applies the BlockSparseAttentionGrad
 *                               formulas to the gathered keys.
 *   sparse_attn_metadata        selection -> per-unit KV lists, transposed lists and per-page
 *                               lists, consumed by the ops above ("SparseAttnSharedkvMetadata"
 *                               page, function description: a task list built ahead of the
 *                               attention call).
 *
 * Conventions
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  The library allocates
 *     nothing, never synchronises (except bsa_get_status), and launches only on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *   - Dtypes: Q, K, V, dOut, Out, dQ, dK, dV are bf16 (uint16 storage); LSE is fp32 natural-log
 *     log-sum-exp of the scaled scores; masks are uint8; indices, tables, cu_seqlens are int32.
 *   - Layouts (row-major, last dimension contiguous):
 *       BNSD  q/dout/out/dq [B, N1, S_q, D], k/v/dk/dv [B, N2, S_kv, D], lse [B, N1, S_q]
 *       TND   q/dout/out/dq [T, N1, D],      k/v/dk/dv [T, N2, D],       lse [T, N1]
 *       PA_ND caches [num_pages, page_size, N2, D]; q [B, 1, N1, D]; out [B, 1, N1, Dv];
 *             lse [B, 1, N1]
 *   - GQA: query head h uses kv head h / (N1 / N2); N1 % N2 == 0 is required.
 *   - Two-phase use, as on the pages: *_workspace_size() validates the problem on the host and
 *     returns the scratch size; the op call re-validates, then launches.  Host validation
 *     errors return before any launch.  Device-side problems (an index past the sequence, a
 *     non-monotone cu_seqlens, a wait that exceeded its limit) set bits in a status word at the
 *     start of the workspace; the offending block is skipped and the call still returns
 *     BSA_OK.  bsa_get_status() reads the word.
 *   - The workspace must be 256-byte aligned and is overwritten by every call.  Calls that
 *     share one workspace must be ordered on the GPU (same stream or synchronised).
 */
#ifndef SELECTED_ATTENTION_H_
#define SELECTED_ATTENTION_H_

#include <stddef.h>
#include <stdint.h>

#include "status_bits.h"

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_NULLPTR = 1,            /* a required pointer is NULL */
  BSA_ERR_INVALID_ARG = 2,        /* a size, layout or rule from the pages is violated */
  BSA_ERR_UNSUPPORTED = 3,        /* valid on the pages, not implemented by this library */
  BSA_ERR_WORKSPACE_TOO_SMALL = 4,
  BSA_ERR_CUDA = 5                /* a CUDA runtime call failed (launch, attribute, ...) */
} bsa_status;

typedef enum { BSA_LAYOUT_BNSD = 0, BSA_LAYOUT_TND = 1, BSA_LAYOUT_BSND = 2, BSA_LAYOUT_PA_ND = 3 } bsa_layout;

/* Mask modes: 0 = no mask (all selected keys computed; NsaSelectedAttention sparseMode 0),
 * 2 = causal, key position <= query position (sparseMode 2), 3 = right-down causal and
 * 4 = band [q' - win_left, q' + win_right] with q' = q + S_kv - S_q (SparseAttnSharedkvMetadata
 * cmp_mask_mode / ori_mask_mode). */
typedef enum { BSA_MASK_NONE = 0, BSA_MASK_CAUSAL = 2, BSA_MASK_RIGHT_DOWN_CAUSAL = 3, BSA_MASK_BAND = 4 } bsa_mask_mode;

typedef struct bsa_params {
  int32_t q_layout, kv_layout; /* bsa_layout */
  int32_t B, N1, N2;           /* batch, query heads, kv heads */
  int32_t S_q, S_kv;           /* BNSD: sequence lengths.  TND: ignored (see T_q / cu_seqlens) */
  int32_t T_q, T_kv;           /* TND: total tokens (host-side sizes) */
  int32_t D, Dv, D_rope;       /* head dims of Q/K, V, and the rope part (SFA) */
  const int32_t* cu_seqlens_q; /* TND: device int32 [B+1] prefix sums */
  const int32_t* cu_seqlens_kv;
  const int32_t* seqused_kv;   /* PA_ND: device int32 [B], tokens of each sequence in use */
  /* BSA: BlockSparseMask, device uint8 [B, N1, ceil(S_q/block_x), ceil(S_kv/block_y)] */
  int32_t block_x, block_y;
  const uint8_t* block_mask;
  /* NSA: topk_indices, device int32 [T, N2, sel_block_count]; ids count sel_block_size-token
   * blocks from the batch's start; -1 = empty slot */
  int32_t sel_block_size, sel_block_count;
  const int32_t* topk_indices;
  /* SFA: paged cache.  block_table device int32 [B, max_pages_per_seq]; sparse_indices device
   * int32 [B, 1, N2, sparse_count] (logical sparse-block ids, -1 = empty) */
  int32_t page_size, max_pages_per_seq, num_pages;
  const int32_t* block_table;
  int32_t sparse_block_size, sparse_count;
  const int32_t* sparse_indices;
  int32_t mask_mode, win_left, win_right; /* bsa_mask_mode */
  float scale;                            /* multiplies q.k (SFA: the whole q.k + q_r.k_r) */
  /* BSA only: optional dense atten_mask, device uint8 [S_q, S_kv] shared by every batch and head,
   * nonzero = masked out; applied inside the selected blocks on top of mask_mode (the
   * Mask(., atten_mask) step of the BlockSparseAttentionGrad formulas).  NULL = none. */
  const uint8_t* atten_mask;
  /* Optional metadata plan (SparseAttnSharedkvMetadata page: the metadata op's output is the
   * attention ops' input), device, 256-byte aligned, written by sparse_attn_metadata with op
   * plan_op for this same problem (the same params and the same selection tensor, unchanged since).
   * NULL = the op builds its lists in its own workspace.  With a plan the op launches no metadata
   * kernel and its workspace shrinks (the *_workspace_size calls see the plan).  Accepted ops:
   *   bsa_fwd: BSA_META_BSA_KV or BSA_META_BSA_BWD;  bsa_bwd: BSA_META_BSA_BWD;
   *   nsa_selected_fwd: BSA_META_NSA_KV or BSA_META_NSA_TOKENS;  nsa_selected_bwd: BSA_META_NSA_TOKENS.
   * Another plan_op returns BSA_ERR_INVALID_ARG; a plan given to sfa_sparse_decode returns
   * BSA_ERR_UNSUPPORTED (the decode builds its page lists in its own prologue).  Device status bits
   * the metadata raised (bad ids, bad cu_seqlens) stay in the plan's status word: read them with
   * bsa_get_status(plan).  The library cannot tell a stale plan from a current one. */
  const void* plan;
  int32_t plan_op; /* bsa_meta_op */
} bsa_params;

/* ---- workspace sizing (phase 1: host validation, no launch) ------------------------------ */
BSA_API bsa_status bsa_fwd_workspace_size(const bsa_params* p, size_t* bytes);
BSA_API bsa_status bsa_bwd_workspace_size(const bsa_params* p, size_t* bytes);
BSA_API bsa_status nsa_selected_fwd_workspace_size(const bsa_params* p, size_t* bytes);
BSA_API bsa_status nsa_selected_bwd_workspace_size(const bsa_params* p, size_t* bytes);
BSA_API bsa_status sfa_sparse_decode_workspace_size(const bsa_params* p, size_t* bytes);

/* ---- BSA (BlockSparseAttentionGrad page), BNSD, D = Dv = 128 -------------------------------
 * Forward: Out = softmax(Mask(scale * Q K_sparse^T, atten_mask)) V_sparse, LSE per row.
 * Rows with no visible key produce Out = 0 and LSE = -inf. */
BSA_API bsa_status bsa_fwd(const bsa_params* p, const void* q, const void* k, const void* v, void* out, float* lse,
                   void* workspace, size_t workspace_bytes, void* stream);
/* Same as bsa_fwd, for callers that cannot allocate device memory (a host that owns all device
 * memory and gives its plugins no scratch, or a path where a cudaMalloc is not acceptable).  The
 * paper has no counterpart: this entry point exists for such callers only.  It needs no
 * workspace: its scratch (status word and KV lists) is a fixed 8 MiB device array inside the
 * library, held by every GPU that loads the library until the process exits.  The first call in a
 * CUDA context looks up that array's device address there (cudaGetSymbolAddress) and keeps it for
 * the context; the first call on a device should come before any stream capture.  Problems whose
 * bsa_fwd workspace exceeds 8 MiB return BSA_ERR_WORKSPACE_TOO_SMALL before any launch.  All calls
 * on a device share the array: calls whose GPU work overlaps race and must be ordered by the
 * caller.  The device status bits of the last call stay in the array: read them with
 * bsa_fwd_noalloc_get_status. */
BSA_API bsa_status bsa_fwd_noalloc(const bsa_params* p, const void* q, const void* k, const void* v, void* out,
                                   float* lse, void* stream);
/* Device status bits (SA_DEV_*) of the last bsa_fwd_noalloc call on the current device, after
 * synchronising `stream` (as bsa_get_status).  No counterpart in the paper. */
BSA_API bsa_status bsa_fwd_noalloc_get_status(void* stream, uint32_t* dev_bits);
/* Backward: softmax_grad = rowsum(dOut o Out); dP = dOut V^T; dS = P o (dP - softmax_grad);
 * dV = P^T dOut; dQ = dS K scale; dK = dS^T Q scale.  `out` and `lse` are the forward's
 * outputs.  dK/dV are accumulated in a fixed order (run-to-run bit identical, no atomics). */
BSA_API bsa_status bsa_bwd(const bsa_params* p, const void* q, const void* k, const void* v, const void* out,
                   const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, void* stream);

/* ---- NSA selected attention (NsaSelectedAttention page), TND, GQA, D = 128 or 192, Dv = 128 -
 * Forward formula of the page: for token t and kv head g, selected_key/value = Gather(key/value,
 * topk_indices[t, g, i]) for the listed blocks; Out = softmax(Mask(scale q K_sel^T)) V_sel for
 * each of the group's G = N1/N2 query heads (heads g*G .. g*G+G-1); LSE per (t, head).
 *   p->q_layout = p->kv_layout = BSA_LAYOUT_TND; q/dq [T, N1, D], out/dout [T, N1, 128], k/dk
 *   [T, N2, D], v/dv [T, N2, 128], lse [T, N1]; (D, Dv) = (128, 128), or (192, 128) (the page's
 *   head-dim pair for query and key vs value) with G = N1 / N2 <= 16.
 *   T_q = T_kv = T; cu_seqlens_q (= cu_seqlens_kv) [B+1] device int32
 *   with per-batch lengths (query and key lengths equal); S_q = the longest batch's length.
 *   topk_indices [T, N2, sel_block_count] int32: block ids of sel_block_size tokens, counted
 *   from the batch's first token; -1 = empty slot; a duplicated id is gathered twice.
 *   mask_mode BSA_MASK_NONE or BSA_MASK_CAUSAL (key position <= query position in the batch).
 *   Host errors (INVALID_ARG / UNSUPPORTED): sel_block_size not a multiple of 16 in [16, 128],
 *   sel_block_count not in [1, 128] or count * size > 8192, N1 % N2 != 0, N2 > 32, N1 > 128,
 *   (D, Dv) other than (128, 128) or (192, 128), D = 192 with G > 16, S_q > 128K, T_q != T_kv,
 *   scale <= 0.
 *   Device status bits: SA_DEV_BAD_INDEX for an id at or past the batch's block count (the id
 *   is skipped); SA_DEV_BAD_SEQLEN if cu_seqlens is not a non-decreasing 0..T sequence or a
 *   batch is longer than S_q (nothing is computed).
 *   Rows with no visible key produce Out = 0 and LSE = -inf.  The backward produces dK/dV rows
 *   of unselected keys as zeros, accumulates dK/dV in a fixed order (no atomics), and counts a
 *   duplicated id once per occurrence. */
BSA_API bsa_status nsa_selected_fwd(const bsa_params* p, const void* q, const void* k, const void* v, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream);
BSA_API bsa_status nsa_selected_bwd(const bsa_params* p, const void* q, const void* k, const void* v, const void* out,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ---- SFA sparse decode (SparseFlashAttention page), PA_ND caches, D = Dv = 512, D_rope = 64 -
 * Out = softmax((q k~^T + q_rope k_rope~^T) * scale) v~ over the selected sparse blocks.
 *   p->kv_layout = BSA_LAYOUT_PA_ND, S_q = 1.  q [B, 1, N1, 512], q_rope [B, 1, N1, 64];
 *   k_cache, v_cache [num_pages, page_size, N2, 512] and k_rope_cache [num_pages, page_size, N2,
 *   64]; out [B, 1, N1, 512] bf16, lse [B, 1, N1] fp32.  block_table [B, max_pages_per_seq] maps
 *   a sequence's logical page to its physical page; sparse_indices [B, 1, N2, sparse_count]
 *   holds logical sparse-block ids (sparse_block_size tokens each, a whole number of pages;
 *   -1 = empty slot); seqused_kv [B] is each sequence's token count: keys at or past it are not
 *   attended.  Query head h uses kv head h / (N1 / N2).
 *   Cache rows past seqused_kv inside a selected page are masked, and their V rows are zeroed in
 *   shared memory before the products, so any value there (NaN included) leaves Out unchanged;
 *   rows of pages that no selected block reaches are never read.
 *   Host errors: UNSUPPORTED for S_q != 1, D / Dv / D_rope other than 512 / 512 / 64, N1 / N2 >
 *   128, page_size not a multiple of 32, or num_pages * page_size * N2 >= 2^31; INVALID_ARG for
 *   non-positive sizes, N1 % N2 != 0, page_size not a multiple of 16 in [16, 1024],
 *   sparse_block_size not a multiple of page_size, or a non-finite or non-positive scale.
 *   Device status bits: SA_DEV_BAD_INDEX for a sparse id at or past the sequence's block count,
 *   or a table entry outside [0, num_pages) (the block is skipped).
 *   A sequence with no selected key produces Out = 0 and LSE = -inf. */
BSA_API bsa_status sfa_sparse_decode(const bsa_params* p, const void* q, const void* q_rope, const void* k_cache,
                             const void* k_rope_cache, const void* v_cache, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Backward of sfa_sparse_decode: the BlockSparseAttentionGrad page's backward formulas applied to
 * the gathered keys, with the score s = scale (q.k + q_rope.k_rope) split as in the forward:
 *   P = exp(s - LSE), D = rowsum(dOut o Out), dP = dOut v~^T, dS = P o (dP - D),
 *   dq = scale dS k~, dq_rope = scale dS k_rope~, dk~ = scale dS^T q, dk_rope~ = scale dS^T q_rope,
 *   dv~ = P^T dOut.
 *   Inputs as for sfa_sparse_decode, plus out (the forward's Out, bf16 [B, 1, N1, 512]), dout
 *   (bf16, same shape) and lse (fp32 [B, 1, N1], natural log).  Outputs (bf16): dq [B, 1, N1, 512],
 *   dq_rope [B, 1, N1, 64], and dk_cache, dv_cache [num_pages, page_size, N2, 512], dk_rope_cache
 *   [num_pages, page_size, N2, 64], laid out as the caches.
 *   Every row of a page the step read (kv head g of a page holding a selected block of batch b) is
 *   SET: a row in use gets the sum of its gathered rows' gradients (a page listed twice, or reached
 *   from two batches' block tables, adds each read; the sum runs in a fixed order, so the result is
 *   deterministic), a row past the sequence's end gets zero.  Rows of pages the step did not read
 *   are NOT written: zero the three gradient caches first to obtain the full cache gradient.  P and
 *   dS enter the tensor cores as bf16.
 *   Host errors: as sfa_sparse_decode, plus BSA_ERR_UNSUPPORTED when p->plan is set or
 *   num_pages * N2 >= 2^30.  Device status bits: as sfa_sparse_decode.  The workspace holds the
 *   page lists, per-tile parts of dq and the gathered-order row gradients (about
 *   B N2 sparse_count sparse_block_size x 2.2 KB). */
BSA_API bsa_status sfa_sparse_decode_bwd_workspace_size(const bsa_params* p, size_t* bytes);
BSA_API bsa_status sfa_sparse_decode_bwd(const bsa_params* p, const void* q, const void* q_rope, const void* k_cache,
                                 const void* k_rope_cache, const void* v_cache, const void* out,
                                 const void* dout, const float* lse, void* dq, void* dq_rope, void* dk_cache,
                                 void* dk_rope_cache, void* dv_cache, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* ---- metadata (SparseAttnSharedkvMetadata page) -------------------------------------------
 * Writes the integer plan the attention kernels consume into `plan` (device, plan_bytes from
 * sparse_attn_metadata_size).  op selects the product:
 *   BSA_META_BSA_KV     int32 row_ptr[U+1] then col[...]: per (b, h, qb) unit, ascending KV
 *                       block ids of its BlockSparseMask row (U = B*N1*nqb).
 *   BSA_META_BSA_Q      transposed lists: per (b, g, kb) row, ascending h_local*nqb + qb.
 *   BSA_META_BSA_BWD    both: offsets[1] row_ptr and [2] col as BSA_META_BSA_KV, [3] row_ptr and
 *                       [4] col as BSA_META_BSA_Q (the backward's two passes), [5] scratch.
 *   BSA_META_NSA_KV     int32 ids[T, N2, K] (valid ids ascending, then -1) and cnt[T, N2].
 *   BSA_META_NSA_TOKENS also, per (b, g, kb) row (kb < ceil(S_q / sel_block_size)), the
 *                       ascending global token indices whose list holds kb, each token once:
 *                       int32 row_ptr[B*N2*nblk+1] and col[...].
 *   BSA_META_SFA_PAGES  int32 pages[B, N2, cap] (compacted: the physical pages of the selected
 *                       sparse blocks in list order, empty slots and pages past seqused_kv
 *                       dropped; cap = sparse_count * sparse_block_size / page_size), tokens[B, N2,
 *                       cap] (tokens in use of each listed page) and count[B, N2].
 *   BSA_META_SFA_WORK   the sparse decode's split of its work (SparseAttnSharedkvMetadata page:
 *                       each core's share of the task list): unit u = (b * N2 + g) * HH + head half
 *                       (HH = 2 when N1 / N2 > 64, else 1) is cut into P pieces, piece u * P + p
 *                       taking pages [floor(p n / P), floor((p + 1) n / P)) of the unit's n.  Per
 *                       piece: int32 pages[pieces][cap] and tokens[pieces][cap] (the unit's
 *                       compacted list, as BSA_META_SFA_PAGES) and rec[pieces][3] = (n, begin,
 *                       len); layout.info[0] = pieces, info[1] = P.  The decode runs this same
 *                       code in its prologue; P = min(4, max(1, SMs / units)).
 * The plan layout for each op is given by sparse_attn_metadata_layout(). */
typedef enum {
  BSA_META_BSA_KV = 0,
  BSA_META_BSA_Q = 1,
  BSA_META_NSA_KV = 2,
  BSA_META_NSA_TOKENS = 3,
  BSA_META_SFA_PAGES = 4,
  BSA_META_SFA_WORK = 5,
  BSA_META_BSA_BWD = 6
} bsa_meta_op;

/* Offsets (bytes from `plan`) of the arrays an op writes: offsets[0] = status word,
 * offsets[1..4] = op-specific arrays (see bsa_meta_op), count = number used; info = op-specific
 * sizes (BSA_META_SFA_WORK: pieces, pieces per unit), zero otherwise. */
typedef struct bsa_meta_layout {
  size_t total_bytes;
  size_t offsets[6];
  int32_t count;
  size_t info[2];
} bsa_meta_layout;

BSA_API bsa_status sparse_attn_metadata_layout(const bsa_params* p, int32_t op, bsa_meta_layout* layout);
BSA_API bsa_status sparse_attn_metadata(const bsa_params* p, int32_t op, void* plan, size_t plan_bytes, void* stream);

/* ---- multi-GPU split (host only) -----------------------------------------------------------
 * Contiguous balanced split of n work items into `parts` ranges (SparseAttnSharedkvMetadata
 * page, function description: each core gets the start and end of its share of the task list).
 * Used to give each rank a contiguous range of (batch, kv head) slices weighted by their selected
 * tiles.  With W the total weight and prefix(t) = weights[0] + ... + weights[t-1]:
 *   starts[s] = min { t : prefix(t) >= ceil(s W / parts) } for s < parts, starts[parts] = n;
 * part s takes items [starts[s], starts[s+1]).  weights: host int64 [n], each >= 0; starts: host
 * int32 [parts + 1], written by the call.  Touches no device state.  Errors: NULL pointers ->
 * BSA_ERR_NULLPTR; n < 0, parts < 1 or a negative weight -> BSA_ERR_INVALID_ARG (starts untouched). */
BSA_API bsa_status bsa_partition(const int64_t* weights, int32_t n, int32_t parts, int32_t* starts);

/* ---- status --------------------------------------------------------------------------------
 * Copies the device status word at the start of `workspace` (or of a metadata plan) to
 * *dev_bits after synchronising `stream`.  Bits: SA_DEV_BAD_INDEX, SA_DEV_BAD_SEQLEN,
 * SA_DEV_TIMEOUT (status_bits.h). */
BSA_API bsa_status bsa_get_status(const void* workspace, void* stream, uint32_t* dev_bits);

/* ---- kernel timing (for benchmarks; off by default) ---------------------------------------
 * bsa_profile_enable(1) starts recording a pair of CUDA events around every kernel launch the
 * library makes (events come from a pool the library creates on first use; 0 stops and clears).
 * bsa_profile_collect() synchronises on the recorded events and returns, per kernel name, the
 * number of launches and their summed device time in milliseconds; it then clears the records.
 * *n_entries receives the number of names (entries beyond max_entries are not written). */
typedef struct bsa_kernel_time {
  char name[32];
  int32_t launches;
  double total_ms;
} bsa_kernel_time;
BSA_API bsa_status bsa_profile_enable(int32_t on);
BSA_API bsa_status bsa_profile_collect(bsa_kernel_time* out, int32_t max_entries, int32_t* n_entries);

/* Schedule record (for benchmarks; off by default).  With dev_buf set (a caller-owned device
 * array of 3 * capacity * 2 uint64), every later launch of the three persistent block-sparse
 * kernels writes, per CTA c < capacity, its start and finish time in ns (the GPU's global timer)
 * to dev_buf[(slot * capacity + c) * 2 + {0, 1}], slot 0 = forward, 1 = KV-major backward pass,
 * 2 = Q-major backward pass; each launch overwrites its slot.  Launches with more CTAs than
 * capacity write nothing.  dev_buf = NULL stops recording.  Not part of the pages' operations. */
BSA_API bsa_status bsa_profile_cta_clock(uint64_t* dev_buf, int32_t capacity);

/* Library version string. */
BSA_API const char* bsa_version(void);

/* ---- diagnostics ---------------------------------------------------------------------------
 * One 128x128x128 tcgen05 tile: c[128][128] (fp32, device) = A B^T with A bf16 [128 rows][128 K]
 * and B bf16 [128 N][128 K] (b_mn_major = 0, 2, 4) or [128 K][128 N] (b_mn_major = 1, 3, 5); modes 2
 * and 3 stage A in tensor memory instead of shared memory; modes 4 and 5 read `a` as A^T
 * ([128 K][128 M], the MN-major A operand).  Other modes return BSA_ERR_INVALID_ARG.  Runs the same
 * TMA / shared-memory-descriptor / TMEM machinery as the attention kernels, so a tile-level
 * fault can be told apart from an attention-level one.  workspace: >= 256 bytes (status word).
 * Not part of the pages' operations. */
BSA_API bsa_status bsa_diag_mma_tile(const void* a, const void* b, float* c, int32_t b_mn_major, void* workspace,
                             void* stream);

/* Diagnostic: y[i] = 2^x[i] (device arrays of n floats) by an exp2 on the FMA pipe (Cody-Waite
 * reduction to [-1/2, 1/2], fitted polynomial of degree 3 or 4, exponent add); the attention
 * kernels use the special-function unit's exp2.  x must lie in [-126, 128).  Not part of the pages'
 * operations.  Returns BSA_ERR_INVALID_ARG for another degree or n < 0. */
BSA_API bsa_status bsa_diag_exp2(const float* x, float* y, int32_t n, int32_t degree, void* stream);

/* Diagnostic for failure detection: one warp waits on a device barrier with the bounded wait every
 * kernel uses.  arrive = 1: the barrier is satisfied first and the status word stays 0.  arrive = 0:
 * nothing arrives; after the wait limit (about one second) the kernel sets SA_DEV_TIMEOUT in the
 * status word at the start of `workspace` (>= 4 bytes, device) and returns normally, so the CUDA
 * context stays usable; read the bits with bsa_get_status.  Other values of arrive return
 * BSA_ERR_INVALID_ARG.  Not part of the pages' operations. */
BSA_API bsa_status bsa_diag_wait(void* workspace, int32_t arrive, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SELECTED_ATTENTION_H_ */
