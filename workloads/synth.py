"""Seeded synthetic inputs for the block-sparse / selected / sparse-decode attention workloads.

This module holds no attention arithmetic: it only draws random numbers and random selections.
Both the fp64 oracle (tests, CPU baseline) and the CUDA path (tests, bench) take their inputs
from here.

Values are fp32 N(0, 1) draws from numpy's PCG64, rounded to bf16 (round to nearest, ties to
even) and kept as uint16 bit patterns.  Every tensor is produced in chunks of rows; each chunk
has its own stream keyed by (seed, tensor tag, chunk index), so any slice of a large tensor can
be regenerated on its own (the oracle re-creates only the heads or pages it checks).

Selections follow the structure of the pages' problem statements:
  * BlockSparseMask rows (BlockSparseAttentionGrad page, "BlockSparseMask specifies the KV block
    selected by each Q block"): uint8 [B, N1, ceil(Sq/bx), ceil(Skv/by)], nonzero = selected.
  * topk_indices (NsaSelectedAttention page, forward formula, Gather(key, topk_indices[i])):
    int32 [T, N2, selected_block_count], block ids relative to the batch start, -1 = empty slot.
  * sparse block ids + block table for a paged KV cache (SparseFlashAttention page, constraints
    on block_size / sparse_block_size).
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np


# ----------------------------------------------------------------------------------------------
# bf16 bit patterns
# ----------------------------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _tag_id(tag: str) -> int:
    return zlib.crc32(tag.encode("utf-8"))


def chunk_rng(seed: int, tag: str, chunk: int) -> np.random.Generator:
    return np.random.default_rng([seed, _tag_id(tag), chunk])


def normal_rows_bf16(seed: int, tag: str, n_rows: int, row_elems: int, rows_per_chunk: int,
                     lo: int = 0, hi: int | None = None) -> np.ndarray:
    """Rows [lo, hi) of an [n_rows, row_elems] bf16 tensor of N(0,1) draws.

    Chunk c covers rows [c*rows_per_chunk, (c+1)*rows_per_chunk) and is drawn from its own
    stream, so the result does not depend on lo/hi.
    """
    hi = n_rows if hi is None else hi
    assert 0 <= lo <= hi <= n_rows
    out = np.empty((hi - lo, row_elems), dtype=np.uint16)
    c0, c1 = lo // rows_per_chunk, (hi + rows_per_chunk - 1) // rows_per_chunk
    for c in range(c0, c1):
        r0 = c * rows_per_chunk
        r1 = min(n_rows, r0 + rows_per_chunk)
        vals = chunk_rng(seed, tag, c).standard_normal((r1 - r0) * row_elems, dtype=np.float32)
        vals = f32_to_bf16_bits(vals).reshape(r1 - r0, row_elems)
        a, b = max(lo, r0), min(hi, r1)
        out[a - lo:b - lo] = vals[a - r0:b - r0]
    return out


def _selection_rng(seed: int, tag: str) -> np.random.Generator:
    return np.random.default_rng([seed, _tag_id("select:" + tag)])


# ----------------------------------------------------------------------------------------------
# selections
# ----------------------------------------------------------------------------------------------
def bsa_mask_fixed_extra(seed: int, B: int, N: int, nqb: int, nkb: int, extra: int) -> np.ndarray:
    """Diagonal block plus min(extra, qb) distinct earlier blocks, uniform without replacement."""
    rng = _selection_rng(seed, "bsa_fixed_extra")
    m = np.zeros((B, N, nqb, nkb), dtype=np.uint8)
    for b in range(B):
        for h in range(N):
            for qb in range(nqb):
                m[b, h, qb, qb] = 1
                r = min(extra, qb)
                if r:
                    m[b, h, qb, rng.choice(qb, size=r, replace=False)] = 1
    return m


def bsa_mask_bernoulli(seed: int, B: int, N: int, nb: int, p: float) -> np.ndarray:
    """Diagonal always on; every earlier (causal) block on independently with probability p."""
    rng = _selection_rng(seed, "bsa_bernoulli")
    u = rng.random((B, N, nb, nb))
    m = (u < p) & np.tril(np.ones((nb, nb), dtype=bool), k=-1)
    m |= np.eye(nb, dtype=bool)
    return m.astype(np.uint8)


def bsa_mask_local_sink_random(seed: int, B: int, N: int, nb: int, budget: int,
                               local: int) -> np.ndarray:
    """min(budget, qb+1) blocks per Q block: diagonal, `local` previous blocks, block 0 (sink),
    the rest uniform without replacement from the remaining causal blocks."""
    rng = _selection_rng(seed, "bsa_local_sink")
    m = np.zeros((B, N, nb, nb), dtype=np.uint8)
    for qb in range(nb):
        fixed = {qb, 0} | {qb - i for i in range(1, local + 1) if qb - i >= 0}
        fixed = np.array(sorted(fixed), dtype=np.int64)
        m[:, :, qb, fixed] = 1
        want = min(budget, qb + 1) - len(fixed)
        if want <= 0:
            continue
        cand = np.setdiff1d(np.arange(qb + 1), fixed)
        keys = rng.random((B, N, len(cand)))
        pick = np.argpartition(keys, want - 1, axis=-1)[..., :want] if want < len(cand) else \
            np.broadcast_to(np.arange(len(cand)), (B, N, len(cand)))
        bi, hi = np.meshgrid(np.arange(B), np.arange(N), indexing="ij")
        m[bi[..., None], hi[..., None], qb, cand[pick]] = 1
    return m


def _distinct_below(rng: np.random.Generator, m: np.ndarray, r: np.ndarray, rmax: int) -> np.ndarray:
    """Per row, r[i] distinct integers drawn uniformly from [0, m[i]) (Floyd's method);
    unused slots hold -1.  Requires r <= m."""
    n = m.shape[0]
    out = np.full((n, rmax), -1, dtype=np.int64)
    for s in range(rmax):
        active = s < r
        j = m - r + s  # Floyd: j runs over [m-r, m)
        t = np.floor(rng.random(n) * (j + 1)).astype(np.int64)
        seen = (out[:, :s] == t[:, None]).any(axis=1) if s else np.zeros(n, dtype=bool)
        val = np.where(seen, j, t)
        out[:, s] = np.where(active, val, -1)
    return out


def nsa_topk(seed: int, seqlens: list[int], N2: int, block: int, count: int) -> np.ndarray:
    """topk_indices [T, N2, count] int32: the token's own block plus min(count-1, own) distinct
    earlier blocks, uniform; valid ids in random order, then -1 padding at the end."""
    rng = _selection_rng(seed, "nsa_topk")
    pos = np.concatenate([np.arange(s) for s in seqlens])
    own = np.repeat(pos // block, N2)
    rows = own.shape[0]
    r = np.minimum(count - 1, own)
    picks = _distinct_below(rng, own, r, count - 1)
    sel = np.concatenate([own[:, None], picks], axis=1)  # [rows, count], -1 at the tail of picks
    nvalid = r + 1
    keys = rng.random((rows, count))
    keys[np.arange(count)[None, :] >= nvalid[:, None]] = 2.0  # padding sorts last
    order = np.argsort(keys, axis=1, kind="stable")
    sel = np.take_along_axis(sel, order, axis=1)
    return sel.reshape(len(pos), N2, count).astype(np.int32)


def sfa_selection(seed: int, B: int, N2: int, n_logical: int, count: int, n_pages: int):
    """block_table [B, n_logical] (a permutation of the physical pages) and
    sparse_indices [B, 1, N2, count] (distinct logical blocks, uniform, random order)."""
    rng = _selection_rng(seed, "sfa")
    table = rng.permutation(n_pages)[: B * n_logical].reshape(B, n_logical).astype(np.int32)
    idx = np.empty((B, 1, N2, count), dtype=np.int32)
    for b in range(B):
        for g in range(N2):
            idx[b, 0, g] = rng.choice(n_logical, size=count, replace=False)
    return table, idx


# ----------------------------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------------------------
MASK_NONE, MASK_CAUSAL, MASK_RIGHT_DOWN_CAUSAL, MASK_BAND = 0, 2, 3, 4


@dataclass
class BsaWorkload:
    """BNSD block-sparse attention problem (BlockSparseAttentionGrad page)."""
    name: str
    seed: int
    B: int
    N1: int
    N2: int
    S: int
    D: int
    block: int
    selection: str                      # "fixed_extra" | "bernoulli" | "local_sink"
    sel_args: dict = field(default_factory=dict)
    mask_mode: int = MASK_CAUSAL

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    @property
    def nb(self) -> int:
        return (self.S + self.block - 1) // self.block

    def block_mask(self) -> np.ndarray:
        if self.selection == "fixed_extra":
            return bsa_mask_fixed_extra(self.seed, self.B, self.N1, self.nb, self.nb, **self.sel_args)
        if self.selection == "bernoulli":
            return bsa_mask_bernoulli(self.seed, self.B, self.N1, self.nb, **self.sel_args)
        if self.selection == "local_sink":
            return bsa_mask_local_sink_random(self.seed, self.B, self.N1, self.nb, **self.sel_args)
        raise ValueError(self.selection)

    def tensor(self, tag: str, b: int | None = None, h: int | None = None) -> np.ndarray:
        """bf16 bits of q/k/v/dout, BNSD.  With b and h given, only that [S, D] head slice."""
        heads = self.N1 if tag in ("q", "dout") else self.N2
        if b is None:
            rows = normal_rows_bf16(self.seed, tag, self.B * heads * self.S, self.D, self.S)
            return rows.reshape(self.B, heads, self.S, self.D)
        lo = (b * heads + h) * self.S
        return normal_rows_bf16(self.seed, tag, self.B * heads * self.S, self.D, self.S, lo, lo + self.S)


@dataclass
class NsaWorkload:
    """TND varlen selected attention problem (NsaSelectedAttention page)."""
    name: str
    seed: int
    seqlens: list
    N1: int
    N2: int
    D: int
    sel_block: int
    sel_count: int
    mask_mode: int = MASK_CAUSAL
    Dv: int = 0  # head dim of v / Out / dOut; 0: the same as q / k (D)

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    @property
    def dv(self) -> int:
        return self.Dv or self.D

    @property
    def T(self) -> int:
        return int(sum(self.seqlens))

    @property
    def B(self) -> int:
        return len(self.seqlens)

    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)

    def topk(self) -> np.ndarray:
        return nsa_topk(self.seed, self.seqlens, self.N2, self.sel_block, self.sel_count)

    def tensor(self, tag: str, lo: int = 0, hi: int | None = None) -> np.ndarray:
        """bf16 bits of q/k/v/dout, TND, tokens [lo, hi)."""
        heads = self.N1 if tag in ("q", "dout") else self.N2
        d = self.D if tag in ("q", "k") else self.dv
        hi = self.T if hi is None else hi
        rows = normal_rows_bf16(self.seed, tag, self.T, heads * d, 64, lo, hi)
        return rows.reshape(hi - lo, heads, d)


@dataclass
class SfaWorkload:
    """Paged sparse decode problem (SparseFlashAttention page)."""
    name: str
    seed: int
    B: int
    N1: int
    N2: int
    D: int
    Dr: int
    context: int
    page: int
    sparse_block: int
    count: int

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D + self.Dr))

    @property
    def n_logical(self) -> int:
        return self.context // self.page

    @property
    def n_pages(self) -> int:
        return self.B * self.n_logical

    def selection(self):
        return sfa_selection(self.seed, self.B, self.N2, self.context // self.sparse_block,
                             self.count, self.n_pages)

    def query(self, tag: str) -> np.ndarray:
        d = self.D if tag == "q" else self.Dr
        rows = normal_rows_bf16(self.seed, tag, self.B, self.N1 * d, 1)
        return rows.reshape(self.B, 1, self.N1, d)

    def pages(self, tag: str, page_ids) -> np.ndarray:
        """bf16 bits of the listed physical pages of k_cache / k_rope_cache / v_cache:
        [len(page_ids), page, N2, d]."""
        d = self.Dr if tag == "k_rope" else self.D
        page_ids = np.asarray(page_ids, dtype=np.int64)
        out = np.empty((len(page_ids), self.page * self.N2 * d), dtype=np.uint16)
        for i, p in enumerate(page_ids):
            out[i] = normal_rows_bf16(self.seed, tag, self.n_pages, self.page * self.N2 * d, 1,
                                      int(p), int(p) + 1)[0]
        return out.reshape(len(page_ids), self.page, self.N2, d)


def workload(config: int):
    """The five synthetic problems, keyed 1..5 (seed 20260000 + number)."""
    seed = 20260000 + config
    if config == 1:
        return BsaWorkload("bsa_tiny_S512", seed, B=1, N1=2, N2=2, S=512, D=128, block=64,
                           selection="fixed_extra", sel_args={"extra": 3})
    if config == 2:
        return BsaWorkload("bsa_S8192", seed, B=2, N1=16, N2=16, S=8192, D=128, block=128,
                           selection="bernoulli", sel_args={"p": 0.25})
    if config == 3:
        return NsaWorkload("nsa_tnd_gqa", seed, seqlens=[4096, 8192, 16384, 32768], N1=64, N2=4,
                           D=128, sel_block=64, sel_count=16)
    if config == 4:
        return SfaWorkload("sfa_paged_decode", seed, B=32, N1=128, N2=1, D=512, Dr=64,
                           context=65536, page=64, sparse_block=64, count=32)
    if config == 5:
        return BsaWorkload("bsa_S131072", seed, B=1, N1=32, N2=32, S=131072, D=128, block=128,
                           selection="local_sink", sel_args={"budget": 64, "local": 4})
    raise ValueError(config)
