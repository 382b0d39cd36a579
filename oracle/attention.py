"""fp64 CPU oracle for block-sparse, NSA-selected and sparse-decode attention.

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
import this module.  It shares no code with the CUDA path and must never serve as a fallback.

Everything is computed in float64 on the bf16 inputs widened exactly.  The arithmetic is the
plain definition, with no blocking, online rescaling or reordering:

  * Forward (BlockSparseAttentionGrad page, section stating the forward formula; the
    NsaSelectedAttention page's forward formula is the same after its Gather step):
        S = Mask(scale * Q K_sel^T, atten_mask);  P = softmax(S);  Out = P V_sel
    The softmax is the two-pass form m = max S, l = sum exp(S - m), P = exp(S - m) / l.
    LSE = m + ln l (natural log of the scaled scores).
  * Backward (BlockSparseAttentionGrad page, backward formulas):
        softmax_grad = rowsum(dOut o Out);  dP = dOut V^T;  dS = P o (dP - softmax_grad)
        dV = P^T dOut;  dQ = (dS K) scale;  dK = (dS^T Q) scale
    with dK/dV summed over every query row (and every query head of the GQA group) that used
    the key.
  * Sparse decode (SparseFlashAttention page, formula): softmax(Q K~^T / sqrt(d_k)) V~ with the
    rope split scoring (q.k + q_rope.k_rope) / sqrt(D + Dr).  Its backward (no CUDA counterpart
    yet) applies the backward formulas above to the gathered keys, the rope parts included, and
    adds each key's gradient to the cache row it came from.

Readings of points the pages leave open (each also listed in the design notes):
  * GQA: query head h uses kv head h // (N1 / N2) (contiguous groups; N1 % N2 == 0 rule).
  * BlockSparseMask is per query head, uint8 [B, N1, ceil(Sq/bx), ceil(Skv/by)], nonzero = selected.
  * topk ids count sel_block_size-token blocks from the batch's own start; -1 marks an empty slot;
    a duplicated id is gathered twice (literal Gather).
  * Masked scores are -inf; a row with no visible key gives Out = 0, LSE = -inf, zero gradients.
  * softmax_grad = softmaxGrad(dOut, attentionOut) uses attentionOut as the backward operator
    receives it: the forward output stored in the input dtype.  With bf16 inputs (uint16 bit
    patterns) the oracle rounds its own fp64 Out to bf16 before the rowsum; with float inputs it
    uses Out unrounded.
  * Mask modes: 0 = none, 2 = causal (key pos <= query pos), 3 = right-down causal
    (key pos <= query pos + Skv - Sq), 4 = band [q' - win_left, q' + win_right] with
    q' = query pos + Skv - Sq.  Keys at or past the sequence's kv length are never visible.

Pins: tests/test_oracle_pins.py checks these functions against torch's scaled-dot-product
attention in float64 (forward and autograd backward), finite differences, closed forms,
invariants and hand-worked fixtures under tests/golden/.
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> the nearest bf16 value (round half to even), returned as float64.

    One rounding of the exact value: bf16 keeps 8 significant bits, so a value in the binade
    [2^(e-1), 2^e) is rounded to a multiple of 2^(e-8); below the normal range (|x| < 2^-126) the
    step stays 2^-133 (the subnormal spacing).  Results of magnitude 2^128 or more become +-inf;
    zeros keep their sign, infinities and NaN pass through."""
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    fin = np.isfinite(x) & (x != 0)
    xf = x[fin]
    _, e = np.frexp(xf)                              # xf = m * 2^e with 0.5 <= |m| < 1
    step_exp = np.maximum(e - 8, -133)
    y = np.ldexp(np.rint(np.ldexp(xf, -step_exp)), step_exp)   # np.rint: half to even
    y = np.where(np.abs(y) >= 2.0 ** 128, np.copysign(np.inf, xf), y)
    out[fin] = y
    return out


def stored_out(o: np.ndarray, out_storage) -> np.ndarray:
    """attentionOut as the backward operator receives it (see module notes)."""
    return round_to_bf16(o) if out_storage == "bf16" else o


# ----------------------------------------------------------------------------------------------
# mask rule (BlockSparseAttentionGrad forward formula, its Mask(., atten_mask) step; NsaSelectedAttention
# sparseMode 0 / 2; SparseAttnSharedkvMetadata mask modes 3 and 4 with ori_win_left/right)
# ----------------------------------------------------------------------------------------------
def visible(pos_q: np.ndarray, pos_k: np.ndarray, mode: int, s_q: int, s_kv: int,
            kv_len: int, win_left: int = 0, win_right: int = 0, atten_mask=None) -> np.ndarray:
    """Boolean [len(pos_q), len(pos_k)]: key k is visible to query q.  atten_mask, when given, is
    the dense [S_q, S_kv] mask of the Mask(., atten_mask) step (nonzero = masked out), applied on
    top of the mode."""
    pq = np.asarray(pos_q, dtype=np.int64)[:, None]
    pk = np.asarray(pos_k, dtype=np.int64)[None, :]
    ok = (pk >= 0) & (pk < kv_len)
    if atten_mask is not None:
        am = np.asarray(atten_mask)
        inside = (pq >= 0) & (pq < am.shape[0]) & (pk >= 0) & (pk < am.shape[1])
        ok = ok & inside & (am[np.clip(pq, 0, am.shape[0] - 1), np.clip(pk, 0, am.shape[1] - 1)] == 0)
    if mode == 0:
        return ok & np.ones_like(pq, dtype=bool)
    if mode == 2:
        return ok & (pk <= pq)
    if mode == 3:
        return ok & (pk <= pq + (s_kv - s_q))
    if mode == 4:
        qq = pq + (s_kv - s_q)
        return ok & (pk >= qq - win_left) & (pk <= qq + win_right)
    raise ValueError(f"mask mode {mode}")


# ----------------------------------------------------------------------------------------------
# one group of query rows against one gathered key list
# ----------------------------------------------------------------------------------------------
def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, vis: np.ndarray, scale: float,
           q_extra: np.ndarray | None = None, k_extra: np.ndarray | None = None):
    """Forward formula on gathered keys.

    q [R, D], k [L, D], v [L, Dv], vis [R, L] bool.  Optional q_extra [R, Dr] / k_extra [L, Dr]
    add the rope part of the score (SparseFlashAttention: D plus Dr).
    Returns Out [R, Dv], LSE [R], P [R, L].
    """
    s = q @ k.T
    if q_extra is not None:
        s = s + q_extra @ k_extra.T
    s = scale * s
    s = np.where(vis, s, NEG_INF)
    m = s.max(axis=1, initial=NEG_INF)
    any_vis = np.isfinite(m)
    m_safe = np.where(any_vis, m, 0.0)
    e = np.where(vis, np.exp(s - m_safe[:, None]), 0.0)
    l = e.sum(axis=1)
    p = np.where(any_vis[:, None], e / np.where(any_vis, l, 1.0)[:, None], 0.0)
    out = p @ v
    lse = np.where(any_vis, m_safe + np.log(np.where(any_vis, l, 1.0)), NEG_INF)
    return out, lse, p


def attend_grad(q, k, v, dout, out, p, scale, q_extra=None, k_extra=None):
    """Backward formulas on gathered keys; returns dQ [R,D], dK [L,D], dV [L,Dv] (and the rope
    parts dQ_extra, dK_extra when the score had them)."""
    softmax_grad = np.sum(dout * out, axis=1)          # rowsum(dOut o Out)
    dp = dout @ v.T                                    # dP = dOut V^T
    ds = p * (dp - softmax_grad[:, None])              # dS = P o (dP - softmax_grad)
    dv = p.T @ dout                                    # dV = P^T dOut
    dq = (ds @ k) * scale                              # dQ = (dS K) scale
    dk = (ds.T @ q) * scale                            # dK = (dS^T Q) scale
    if q_extra is None:
        return dq, dk, dv
    return dq, dk, dv, (ds @ k_extra) * scale, (ds.T @ q_extra) * scale


# ----------------------------------------------------------------------------------------------
# BSA: BNSD, BlockSparseMask (BlockSparseAttentionGrad page)
# ----------------------------------------------------------------------------------------------
def bsa_unit_keys(mask_row: np.ndarray, by: int, s_kv: int) -> np.ndarray:
    """Key positions of one Q block: the selected KV blocks in ascending order, concatenated."""
    blocks = np.nonzero(mask_row)[0]
    if len(blocks) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(j * by, min(s_kv, (j + 1) * by)) for j in blocks])


def bsa_slice_forward(q_g, k_g, v_g, mask_g, bx, by, mode, scale, win_left=0, win_right=0,
                      q_blocks=None, atten_mask=None):
    """One (batch, kv-head) slice.  q_g [G, Sq, D] (the group's query heads), k_g [Skv, D],
    v_g [Skv, Dv], mask_g [G, nqb, nkb].  Returns Out [G, Sq, Dv], LSE [G, Sq]; with q_blocks
    given, only those Q blocks are filled (the rest stay NaN)."""
    G, s_q, _ = q_g.shape
    s_kv = k_g.shape[0]
    out = np.full((G, s_q, v_g.shape[1]), np.nan)
    lse = np.full((G, s_q), np.nan)
    nqb = mask_g.shape[1]
    for h in range(G):
        for qb in (range(nqb) if q_blocks is None else q_blocks):
            rows = np.arange(qb * bx, min(s_q, (qb + 1) * bx))
            keys = bsa_unit_keys(mask_g[h, qb], by, s_kv)
            vis = visible(rows, keys, mode, s_q, s_kv, s_kv, win_left, win_right, atten_mask)
            o, l, _ = attend(q_g[h, rows], k_g[keys], v_g[keys], vis, scale)
            out[h, rows] = o
            lse[h, rows] = l
    return out, lse


def bsa_slice_backward(q_g, k_g, v_g, dout_g, mask_g, bx, by, mode, scale, win_left=0,
                       win_right=0, q_blocks=None, kv_blocks=None, out_storage=None, out_in_g=None,
                       atten_mask=None):
    """One (batch, kv-head) slice of the backward pass.  Returns dQ [G,Sq,D], dK [Skv,D],
    dV [Skv,Dv], Out, LSE.  Units (h, qb) are skipped only when they contribute neither to a
    requested dQ block nor to a requested KV block, so every requested entry is exact.
    out_in_g [G,Sq,Dv] (float64), when given, is the attentionOut input of the backward operator:
    softmax_grad = rowsum(dOut o attentionOut) then uses it as given instead of the oracle's own
    forward output."""
    G, s_q, _ = q_g.shape
    s_kv = k_g.shape[0]
    nqb = mask_g.shape[1]
    dq = np.zeros_like(q_g, dtype=np.float64)
    dk = np.zeros(k_g.shape)
    dv = np.zeros(v_g.shape)
    out = np.full((G, s_q, v_g.shape[1]), np.nan)
    lse = np.full((G, s_q), np.nan)
    want_q = None if q_blocks is None else set(q_blocks)
    want_kv = None if kv_blocks is None else np.asarray(list(kv_blocks))
    for h in range(G):
        for qb in range(nqb):
            if want_q is not None or want_kv is not None:
                hit_q = want_q is not None and qb in want_q
                hit_kv = want_kv is not None and bool(np.any(mask_g[h, qb, want_kv]))
                if not (hit_q or hit_kv):
                    continue
            rows = np.arange(qb * bx, min(s_q, (qb + 1) * bx))
            keys = bsa_unit_keys(mask_g[h, qb], by, s_kv)
            vis = visible(rows, keys, mode, s_q, s_kv, s_kv, win_left, win_right, atten_mask)
            qr, kr, vr = q_g[h, rows], k_g[keys], v_g[keys]
            o, l, p = attend(qr, kr, vr, vis, scale)
            o_in = stored_out(o, out_storage) if out_in_g is None else out_in_g[h, rows]
            g_q, g_k, g_v = attend_grad(qr, kr, vr, dout_g[h, rows], o_in, p, scale)
            out[h, rows] = o
            lse[h, rows] = l
            dq[h, rows] = g_q
            np.add.at(dk, keys, g_k)
            np.add.at(dv, keys, g_v)
    return dq, dk, dv, out, lse


def _f64(x):
    return bf16_to_f64(x) if np.asarray(x).dtype == np.uint16 else np.asarray(x, dtype=np.float64)


def bsa_forward(q, k, v, block_mask, bx, by, mode, scale, win_left=0, win_right=0, atten_mask=None):
    """Full BNSD forward: q [B,N1,Sq,D], k/v [B,N2,Skv,D*] (bf16 bits or floats); atten_mask an
    optional dense [Sq, Skv] mask (nonzero = masked out) shared by every batch and head."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N1, s_q, _ = q.shape
    N2 = k.shape[1]
    G = N1 // N2
    out = np.zeros((B, N1, s_q, v.shape[3]))
    lse = np.zeros((B, N1, s_q))
    for b in range(B):
        for g in range(N2):
            hs = slice(g * G, (g + 1) * G)
            o, l = bsa_slice_forward(q[b, hs], k[b, g], v[b, g], block_mask[b, hs], bx, by, mode,
                                     scale, win_left, win_right, atten_mask=atten_mask)
            out[b, hs], lse[b, hs] = o, l
    return out, lse


def bsa_backward(q, k, v, dout, block_mask, bx, by, mode, scale, win_left=0, win_right=0, out_in=None,
                 atten_mask=None):
    """Full BNSD backward; returns dQ, dK, dV, Out, LSE.  out_in [B,N1,Sq,Dv] (bf16 bits or
    floats), when given, is the backward operator's attentionOut input (softmax_grad =
    rowsum(dOut o attentionOut)); by default the oracle's own Out, stored in the input dtype."""
    out_storage = "bf16" if np.asarray(q).dtype == np.uint16 else None
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    out_in = None if out_in is None else _f64(out_in)
    B, N1, s_q, _ = q.shape
    N2 = k.shape[1]
    G = N1 // N2
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    out = np.zeros((B, N1, s_q, v.shape[3]))
    lse = np.zeros((B, N1, s_q))
    for b in range(B):
        for g in range(N2):
            hs = slice(g * G, (g + 1) * G)
            r = bsa_slice_backward(q[b, hs], k[b, g], v[b, g], dout[b, hs], block_mask[b, hs],
                                   bx, by, mode, scale, win_left, win_right, out_storage=out_storage,
                                   out_in_g=None if out_in is None else out_in[b, hs], atten_mask=atten_mask)
            dq[b, hs], dk[b, g], dv[b, g], out[b, hs], lse[b, hs] = r
    return dq, dk, dv, out, lse


# ----------------------------------------------------------------------------------------------
# NSA selected attention: TND varlen, topk_indices, GQA (NsaSelectedAttention page)
# ----------------------------------------------------------------------------------------------
def nsa_token_keys(ids: np.ndarray, sel_block: int, seq_len: int) -> np.ndarray:
    """Gather(key, topk_indices[i]) for 0 <= i < selected_block_count: the key positions (within
    the batch) of the listed blocks, in list order; -1 slots are empty; ids past the sequence
    contribute no keys."""
    parts = [np.arange(j * sel_block, min(seq_len, (j + 1) * sel_block)) for j in ids if j >= 0]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def nsa_slice(q_g, k_g, v_g, topk_g, sel_block, mode, scale, dout_g=None, tokens=None,
              out_storage=None, out_in_g=None):
    """One (batch, kv-head) slice: q_g [S, G, D], k_g [S, D], v_g [S, Dv], topk_g [S, K].
    Forward for every listed token (all by default); with dout_g also the backward pass.
    Returns Out [S,G,Dv], LSE [S,G] (+ dQ [S,G,D], dK [S,D], dV [S,Dv]); unlisted tokens are NaN
    in Out/LSE/dQ, and dK/dV then hold only the listed tokens' contributions.  out_in_g [S,G,Dv]
    (float64), when given, is the backward's attentionOut input (used for softmax_grad as given)."""
    S, G, _ = q_g.shape
    out = np.full((S, G, v_g.shape[1]), np.nan)
    lse = np.full((S, G), np.nan)
    if dout_g is not None:
        dq = np.full(q_g.shape, np.nan)
        dk = np.zeros(k_g.shape)
        dv = np.zeros(v_g.shape)
    for t in (range(S) if tokens is None else tokens):
        keys = nsa_token_keys(topk_g[t], sel_block, S)
        vis = visible(np.full(G, t), keys, mode, S, S, S)
        qr, kr, vr = q_g[t], k_g[keys], v_g[keys]
        o, l, p = attend(qr, kr, vr, vis, scale)
        out[t], lse[t] = o, l
        if dout_g is not None:
            o_in = stored_out(o, out_storage) if out_in_g is None else out_in_g[t]
            g_q, g_k, g_v = attend_grad(qr, kr, vr, dout_g[t], o_in, p, scale)
            dq[t] = g_q
            np.add.at(dk, keys, g_k)
            np.add.at(dv, keys, g_v)
    if dout_g is None:
        return out, lse
    return out, lse, dq, dk, dv


def nsa_forward(q, k, v, topk, cu_seqlens, sel_block, mode, scale):
    """Full TND forward: q [T,N1,D], k/v [T,N2,D*], topk [T,N2,K] int32, cu_seqlens [B+1]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, N1, _ = q.shape
    N2 = k.shape[1]
    G = N1 // N2
    out = np.zeros((T, N1, v.shape[2]))
    lse = np.zeros((T, N1))
    for b in range(len(cu_seqlens) - 1):
        t0, t1 = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        for g in range(N2):
            hs = slice(g * G, (g + 1) * G)
            o, l = nsa_slice(q[t0:t1, hs], k[t0:t1, g], v[t0:t1, g], topk[t0:t1, g], sel_block,
                             mode, scale)
            out[t0:t1, hs], lse[t0:t1, hs] = o, l
    return out, lse


def nsa_backward(q, k, v, dout, topk, cu_seqlens, sel_block, mode, scale, out_in=None):
    """Full TND backward; returns dQ, dK, dV, Out, LSE.  out_in [T,N1,Dv], when given, is the
    backward's attentionOut input (as in bsa_backward)."""
    out_storage = "bf16" if np.asarray(q).dtype == np.uint16 else None
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    out_in = None if out_in is None else _f64(out_in)
    T, N1, _ = q.shape
    N2 = k.shape[1]
    G = N1 // N2
    out = np.zeros((T, N1, v.shape[2]))
    lse = np.zeros((T, N1))
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(len(cu_seqlens) - 1):
        t0, t1 = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        for g in range(N2):
            hs = slice(g * G, (g + 1) * G)
            o, l, gq, gk, gv = nsa_slice(q[t0:t1, hs], k[t0:t1, g], v[t0:t1, g], topk[t0:t1, g],
                                         sel_block, mode, scale, dout_g=dout[t0:t1, hs],
                                         out_storage=out_storage,
                                         out_in_g=None if out_in is None else out_in[t0:t1, hs])
            out[t0:t1, hs], lse[t0:t1, hs], dq[t0:t1, hs] = o, l, gq
            dk[t0:t1, g], dv[t0:t1, g] = gk, gv
    return dq, dk, dv, out, lse


# ----------------------------------------------------------------------------------------------
# SFA: sparse decode over a paged KV cache with a rope sub-head (SparseFlashAttention page)
# ----------------------------------------------------------------------------------------------
def sfa_token_positions(ids: np.ndarray, sparse_block: int, kv_len: int) -> np.ndarray:
    """Logical token positions of the selected sparse blocks, in list order (-1 = empty)."""
    parts = [np.arange(j * sparse_block, min(kv_len, (j + 1) * sparse_block)) for j in ids if j >= 0]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def sfa_decode_slice(q_g, qr_g, page_of, k_pages, kr_pages, v_pages, positions, page_size, scale):
    """One (batch, kv-head) decode slice.  q_g [Sq, G, D], qr_g [Sq, G, Dr]; page_of maps a
    logical page index to a key into k_pages / kr_pages / v_pages ([page, D*] per entry).
    All selected keys are visible (decode, no mask).  Returns Out [Sq,G,Dv], LSE [Sq,G]."""
    Sq, G, _ = q_g.shape
    kk = np.stack([k_pages[page_of(p // page_size)][p % page_size] for p in positions]) \
        if len(positions) else np.zeros((0, q_g.shape[2]))
    kr = np.stack([kr_pages[page_of(p // page_size)][p % page_size] for p in positions]) \
        if len(positions) else np.zeros((0, qr_g.shape[2]))
    vv = np.stack([v_pages[page_of(p // page_size)][p % page_size] for p in positions]) \
        if len(positions) else np.zeros((0, q_g.shape[2]))
    out = np.zeros((Sq, G, vv.shape[1]))
    lse = np.zeros((Sq, G))
    for s in range(Sq):
        vis = np.ones((G, len(positions)), dtype=bool)
        o, l, _ = attend(q_g[s], kk, vv, vis, scale, q_extra=qr_g[s], k_extra=kr)
        out[s], lse[s] = o, l
    return out, lse


def sfa_decode(q, q_rope, k_cache, k_rope_cache, v_cache, block_table, sparse_indices,
               seqused_kv, page_size, sparse_block, scale, batches=None):
    """q [B,Sq,N1,D], q_rope [B,Sq,N1,Dr]; caches [pages, page_size, N2, D*]; block_table
    [B, max_pages]; sparse_indices [B, Sq, N2, K] (row 0 used for every query row of a batch);
    seqused_kv [B].  The caches may be dicts {physical page: [page_size, N2, D*]} holding only
    the pages that are read.  Returns Out [B,Sq,N1,Dv], LSE [B,Sq,N1] (NaN for skipped batches)."""
    B, Sq, N1, D = q.shape
    N2 = sparse_indices.shape[2]
    G = N1 // N2
    Dv = (v_cache[next(iter(v_cache))] if isinstance(v_cache, dict) else v_cache).shape[-1]
    out = np.full((B, Sq, N1, Dv), np.nan)
    lse = np.full((B, Sq, N1), np.nan)
    for b in (range(B) if batches is None else batches):
        for g in range(N2):
            hs = slice(g * G, (g + 1) * G)
            pos = sfa_token_positions(sparse_indices[b, 0, g], sparse_block, int(seqused_kv[b]))

            def page_of(lp, b=b):
                return int(block_table[b, lp])

            kp = {p: _f64(k_cache[p])[:, g] for p in {page_of(x // page_size) for x in pos}}
            krp = {p: _f64(k_rope_cache[p])[:, g] for p in kp}
            vp = {p: _f64(v_cache[p])[:, g] for p in kp}
            o, l = sfa_decode_slice(_f64(q[b, :, hs]), _f64(q_rope[b, :, hs]), page_of, kp, krp, vp,
                                    pos, page_size, scale)
            out[b, :, hs], lse[b, :, hs] = o, l
    return out, lse


def sfa_backward(q, q_rope, k_cache, k_rope_cache, v_cache, dout, block_table, sparse_indices,
                 seqused_kv, page_size, sparse_block, scale):
    """Backward of sfa_decode: the BlockSparseAttentionGrad backward formulas applied to the
    gathered keys with the rope split score s = scale (q.k + q_rope.k_rope), so
        dQ = (dS K~) scale,  dQ_rope = (dS K~_rope) scale,
        dK~ = (dS^T Q) scale, dK~_rope = (dS^T Q_rope) scale, dV~ = P^T dOut,
    and each gathered key's gradient is added to the cache row it was read from (a sparse block
    listed twice adds twice; rows never read stay zero).  Arrays as in sfa_decode, caches as
    arrays.  Returns dQ, dQ_rope, dK_cache, dK_rope_cache, dV_cache, Out, LSE."""
    out_storage = "bf16" if np.asarray(q).dtype == np.uint16 else None
    q, q_rope, dout = _f64(q), _f64(q_rope), _f64(dout)
    k_cache, k_rope_cache, v_cache = _f64(k_cache), _f64(k_rope_cache), _f64(v_cache)
    B, Sq, N1, _ = q.shape
    N2 = sparse_indices.shape[2]
    G = N1 // N2
    dq, dqr = np.zeros(q.shape), np.zeros(q_rope.shape)
    dk, dkr, dv = np.zeros(k_cache.shape), np.zeros(k_rope_cache.shape), np.zeros(v_cache.shape)
    out = np.zeros((B, Sq, N1, v_cache.shape[-1]))
    lse = np.zeros((B, Sq, N1))
    for b in range(B):
        for g in range(N2):
            hs = slice(g * G, (g + 1) * G)
            pos = sfa_token_positions(sparse_indices[b, 0, g], sparse_block, int(seqused_kv[b]))
            pages = np.array([int(block_table[b, p // page_size]) for p in pos], dtype=np.int64)
            offs = np.asarray(pos, dtype=np.int64) % page_size
            kk, kr, vv = k_cache[pages, offs, g], k_rope_cache[pages, offs, g], v_cache[pages, offs, g]
            for s in range(Sq):
                vis = np.ones((G, len(pos)), dtype=bool)
                o, l, p = attend(q[b, s, hs], kk, vv, vis, scale, q_extra=q_rope[b, s, hs], k_extra=kr)
                gq, gk, gv, gqr, gkr = attend_grad(q[b, s, hs], kk, vv, dout[b, s, hs], stored_out(o, out_storage),
                                                   p, scale, q_extra=q_rope[b, s, hs], k_extra=kr)
                out[b, s, hs], lse[b, s, hs] = o, l
                dq[b, s, hs], dqr[b, s, hs] = gq, gqr
                np.add.at(dk, (pages, offs, g), gk)
                np.add.at(dkr, (pages, offs, g), gkr)
                np.add.at(dv, (pages, offs, g), gv)
    return dq, dqr, dk, dkr, dv, out, lse
