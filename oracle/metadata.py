"""CPU reference for the sparse-attention metadata (selection -> per-unit KV lists, transposed
lists, per-page lists and the balanced per-SM work list).

TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
import this module; it shares no code with the CUDA path.

The SparseAttnSharedkvMetadata page describes an operator that, ahead of the attention call,
writes a task list giving each compute core the start and end (batch, head, Q block, K block) of
its share of the work.  The reference here defines the integer products our device metadata
must reproduce bit-exactly:

  * BSA KV lists (BlockSparseAttentionGrad page: "BlockSparseMask specifies the KV block
    selected by each Q block"): units in (b, h, qb) order; each unit's KV block ids ascending.
  * BSA transposed lists (needed by dK/dV, backward formulas dV = P^T dOut, dK = dS^T Q scale):
    per (b, kv head g, kv block kb) the ascending entries h_local * nqb + qb of the query blocks
    (of the group's query heads) that selected kb.
  * NSA lists (NsaSelectedAttention page, Gather(key, topk_indices[i])): per (token, kv head) the
    valid ids ascending (duplicates kept, -1 dropped, ids past the batch's block count dropped
    and flagged); per (b, g, kb), kb < the longest batch's block count, the ascending global
    token indices whose list holds kb, each token once (a duplicated id is weighted by its
    multiplicity in the dK/dV computation instead).
  * SFA page lists (SparseFlashAttention page: sparse_block_size is a multiple of block_size):
    per (b, kv head) the physical pages of the selected sparse blocks, in list order.
  * Work list: see `work_cuts`.
"""
from __future__ import annotations

import numpy as np

BAD_INDEX = 1  # device status bit: an index at or past the sequence's block count was dropped


def csr_from_lists(lists):
    row_ptr = np.zeros(len(lists) + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum([len(x) for x in lists])
    col = np.array([c for x in lists for c in x], dtype=np.int32)
    return row_ptr, col


def bsa_kv_csr(mask: np.ndarray):
    """mask uint8 [B, N1, nqb, nkb] -> (row_ptr [B*N1*nqb+1], col) ascending per unit.

    Units are the rows of the mask in (b, h, qb) order; a row's list is the positions of its
    nonzero bytes, which np.nonzero returns in ascending row-major order."""
    B, N1, nqb, nkb = mask.shape
    rows = mask.reshape(B * N1 * nqb, nkb) != 0
    row_ptr = np.zeros(rows.shape[0] + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum(rows.sum(axis=1))
    col = np.nonzero(rows)[1].astype(np.int32)
    return row_ptr, col


def bsa_q_csr(mask: np.ndarray, N2: int):
    """Transposed lists: rows (b, g, kb); entries h_local * nqb + qb ascending, i.e. the nonzero
    positions of the mask rearranged to [B, N2, nkb, G, nqb]."""
    B, N1, nqb, nkb = mask.shape
    G = N1 // N2
    t = mask.reshape(B, N2, G, nqb, nkb).transpose(0, 1, 4, 2, 3).reshape(B * N2 * nkb, G * nqb)
    return bsa_kv_csr(t.reshape(B * N2 * nkb, 1, 1, G * nqb))


def nsa_blocks_per_batch(cu_seqlens, sel_block):
    lens = np.diff(np.asarray(cu_seqlens, dtype=np.int64))
    return (lens + sel_block - 1) // sel_block


def nsa_kv_lists(topk: np.ndarray, cu_seqlens, sel_block: int):
    """topk int32 [T, N2, K] -> (ids [T, N2, K] valid ids ascending then -1 padding,
    count [T, N2] int32, status bits)."""
    T, N2, K = topk.shape
    nblk = nsa_blocks_per_batch(cu_seqlens, sel_block)
    batch_of = np.zeros(T, dtype=np.int64)
    for b in range(len(nblk)):
        batch_of[cu_seqlens[b]:cu_seqlens[b + 1]] = b
    ids = np.full((T, N2, K), -1, dtype=np.int32)
    cnt = np.zeros((T, N2), dtype=np.int32)
    status = 0
    for t in range(T):
        nb = nblk[batch_of[t]]
        for g in range(N2):
            row = [int(x) for x in topk[t, g] if x >= 0]
            if any(x >= nb for x in row):
                status |= BAD_INDEX
            row = sorted(x for x in row if x < nb)
            ids[t, g, :len(row)] = row
            cnt[t, g] = len(row)
    return ids, cnt, status


def nsa_token_csr(ids: np.ndarray, cnt: np.ndarray, cu_seqlens, sel_block: int, nblk_max: int):
    """Rows (b, g, kb) for kb < nblk_max (rows past the batch's own block count are empty):
    ascending global token indices whose valid list holds kb, each token once."""
    T, N2, _ = ids.shape
    B = len(cu_seqlens) - 1
    lists = []
    for b in range(B):
        t0, t1 = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        for g in range(N2):
            per = [[] for _ in range(nblk_max)]
            for t in range(t0, t1):
                for kb in sorted(set(int(x) for x in ids[t, g, :int(cnt[t, g])])):
                    per[kb].append(t)
            lists.extend(per)
    return csr_from_lists(lists)


def sfa_page_lists(sparse_indices: np.ndarray, block_table: np.ndarray, seqused_kv,
                   sparse_block: int, page_size: int):
    """sparse_indices [B, Sq, N2, K] (row 0 of Sq used) -> (pages [B, N2, K*ppb] physical pages
    in list order with -1 for empty slots, status).  ppb = sparse_block / page_size."""
    B, _, N2, K = sparse_indices.shape
    ppb = sparse_block // page_size
    pages = np.full((B, N2, K * ppb), -1, dtype=np.int32)
    status = 0
    for b in range(B):
        nsb = (int(seqused_kv[b]) + sparse_block - 1) // sparse_block
        for g in range(N2):
            for i in range(K):
                j = int(sparse_indices[b, 0, g, i])
                if j < 0:
                    continue
                if j >= nsb:
                    status |= BAD_INDEX
                    continue
                for p in range(ppb):
                    lp = j * ppb + p
                    if lp * page_size < int(seqused_kv[b]):
                        pages[b, g, i * ppb + p] = block_table[b, lp]
    return pages, status


def work_cuts(weights: np.ndarray, n_parts: int) -> np.ndarray:
    """Balanced split of a sequence of work items (SparseAttnSharedkvMetadata page: each core
    gets the start and end of its share of the task list).

    weights: int [U] per-unit cost.  Returns cuts int32 [n_parts + 1] in units of the
    linearised item index: part s covers prefix positions [ceil(s*W/n), ceil((s+1)*W/n)) of the
    total weight W, so cut[s] = ceil(s * W / n_parts)."""
    W = int(np.sum(weights))
    return np.array([-(-(s * W) // n_parts) for s in range(n_parts + 1)], dtype=np.int64)


def slice_cuts(weights, n_parts: int) -> np.ndarray:
    """Whole-item version of work_cuts: the first item of each part when items may not be cut
    (the multi-GPU split of (batch, kv head) slices; SparseAttnSharedkvMetadata page, each core's
    start and end in the task list).  Part s starts at the smallest t whose prefix weight
    w[0] + ... + w[t-1] reaches ceil(s*W/n_parts); the last cut is the item count.  Plain loops."""
    w = [int(x) for x in weights]
    W = sum(w)
    starts = []
    for s in range(n_parts):
        target = -(-(s * W) // n_parts)
        t, prefix = 0, 0
        while prefix < target and t < len(w):
            prefix += w[t]
            t += 1
        starts.append(t)
    starts.append(len(w))
    return np.array(starts, dtype=np.int32)


def sfa_pieces_per_unit(units: int, sms: int, max_pieces: int = 4) -> int:
    """Pieces per decode unit: as many as one wave of the GPU's SMs allows, at most `max_pieces`
    (the pieces of a unit merge their partial results inside one thread-block cluster)."""
    return min(max_pieces, max(1, sms // max(units, 1)))


def sfa_pieces(count: np.ndarray, HH: int, P: int):
    """Split of the sparse decode's work (SparseAttnSharedkvMetadata page: each core gets the start
    and end of its share of the task list).  count [B*N2]: compacted pages per (b, kv head); a unit
    u = bg * HH + head half shares its (b, kv head)'s list.  Unit u's n pages are cut into P
    consecutive pieces; piece u * P + p gets pages [floor(p n / P), floor((p + 1) n / P)).
    Returns int32 [units * P, 3] = (n, begin, len)."""
    units = len(count) * HH
    rec = np.zeros((units * P, 3), dtype=np.int32)
    for u in range(units):
        n = int(count[u // HH])
        for p in range(P):
            b0, b1 = (p * n) // P, ((p + 1) * n) // P
            rec[u * P + p] = (n, b0, b1 - b0)
    return rec
