"""Pins for the CPU metadata reference: a hand-written fixture, brute force over every mask of a
tiny shape (the lists must rebuild the mask exactly), and NSA / SFA list properties."""
import itertools
import json
import os

import numpy as np

from oracle import metadata as M

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_bsa_lists():
    with open(os.path.join(GOLDEN, "bsa_metadata_3x3.json")) as f:
        g = json.load(f)
    mask = np.array(g["mask"], np.uint8)
    rp, col = M.bsa_kv_csr(mask)
    assert rp.tolist() == g["kv_row_ptr"] and col.tolist() == g["kv_col"]
    rp, col = M.bsa_q_csr(mask, g["N2"])
    assert rp.tolist() == g["q_row_ptr"] and col.tolist() == g["q_col"]


def test_bsa_lists_rebuild_every_2x3_mask():
    """Brute force over all 2^6 masks of one head with 2 Q blocks x 3 KV blocks, two heads."""
    for bits in itertools.product([0, 1], repeat=6):
        m1 = np.array(bits, np.uint8).reshape(2, 3)
        mask = np.stack([m1, 1 - m1])[None]           # [1, 2, 2, 3]
        rp, col = M.bsa_kv_csr(mask)
        rebuilt = np.zeros_like(mask)
        for u in range(len(rp) - 1):
            b, h, qb = np.unravel_index(u, mask.shape[:3])
            ids = col[rp[u]:rp[u + 1]]
            assert np.all(np.diff(ids) > 0)
            rebuilt[b, h, qb, ids] = 1
        assert np.array_equal(rebuilt, mask)
        for n2 in (1, 2):
            rp2, col2 = M.bsa_q_csr(mask, n2)
            G = 2 // n2
            rebuilt = np.zeros_like(mask)
            for r in range(len(rp2) - 1):
                b, g, kb = np.unravel_index(r, (1, n2, 3))
                e = col2[rp2[r]:rp2[r + 1]]
                assert np.all(np.diff(e) > 0)
                rebuilt[b, g * G + e // 2, e % 2, kb] = 1
            assert np.array_equal(rebuilt, mask)


def test_nsa_lists_properties():
    rng = np.random.default_rng(0)
    seqlens = [20, 9, 33]
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    T, N2, K, bs = sum(seqlens), 2, 4, 8
    topk = rng.integers(-1, 6, size=(T, N2, K)).astype(np.int32)
    ids, cnt, status = M.nsa_kv_lists(topk, cu, bs)
    nblk = M.nsa_blocks_per_batch(cu, bs)
    assert status == M.BAD_INDEX          # ids up to 5 exceed the 2-block batch
    for b in range(len(seqlens)):
        for t in range(cu[b], cu[b + 1]):
            for g in range(N2):
                want = sorted(int(x) for x in topk[t, g] if 0 <= x < nblk[b])
                assert ids[t, g, :cnt[t, g]].tolist() == want
                assert np.all(ids[t, g, cnt[t, g]:] == -1)
    nmax = int(nblk.max())
    rp, col = M.nsa_token_csr(ids, cnt, cu, bs, nmax)
    distinct = sum(len(set(ids[t, g, :cnt[t, g]].tolist())) for t in range(T) for g in range(N2))
    assert rp[-1] == distinct and len(rp) == len(seqlens) * N2 * nmax + 1
    # every (token, g, id) pair appears exactly once, tokens ascending
    r = 0
    for b in range(len(seqlens)):
        for g in range(N2):
            for kb in range(nmax):
                toks = col[rp[r]:rp[r + 1]]
                assert np.all(np.diff(toks) > 0)
                want = [t for t in range(cu[b], cu[b + 1]) if kb in set(ids[t, g, :cnt[t, g]].tolist())]
                assert toks.tolist() == want
                r += 1


def test_sfa_page_lists():
    table = np.array([[5, 3, 0, 7], [1, 2, 6, 4]], np.int32)
    idx = np.array([[[[2, 0, -1]]], [[[3, 1, 4]]]], np.int32)   # [B=2, Sq=1, N2=1, K=3]
    pages, status = M.sfa_page_lists(idx, table, [256, 200], 64, 64)
    assert pages[0, 0].tolist() == [0, 5, -1]
    assert pages[1, 0].tolist() == [4, 2, -1] and status == M.BAD_INDEX
    # sparse blocks of two pages each: block j covers logical pages 2j, 2j+1
    pages, status = M.sfa_page_lists(idx[:, :, :, :2], table, [256, 256], 128, 64)
    assert pages[0, 0].tolist() == [-1, -1, 5, 3] and pages[1, 0].tolist() == [-1, -1, 6, 4]
    assert status == M.BAD_INDEX


def test_work_cuts():
    w = np.array([3, 1, 4, 1, 5, 9, 2, 6])
    cuts = M.work_cuts(w, 4)
    assert cuts[0] == 0 and cuts[-1] == w.sum()
    assert np.all(np.diff(cuts) >= 0) and np.max(np.diff(cuts)) - np.min(np.diff(cuts)) <= 1


def test_slice_cuts_golden():
    with open(os.path.join(GOLDEN, "slice_cuts.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        assert M.slice_cuts(np.array(c["weights"], np.int64), c["parts"]).tolist() == c["starts"], c["why"]


def test_slice_cuts_uniform_closed_form_and_balance():
    """Equal weights give starts ceil(s n / parts) (the textbook even split); for any weights each
    part's total stays within one slice's weight of W / parts (brute force over small random
    weight vectors, zeros included)."""
    for n in range(0, 13):
        for parts in range(1, 7):
            got = M.slice_cuts(np.full(n, 3, np.int64), parts)
            assert got.tolist() == [-(-(s * n) // parts) for s in range(parts)] + [n]
    rng = np.random.default_rng(5)
    for _ in range(300):
        n, parts = int(rng.integers(1, 12)), int(rng.integers(1, 6))
        w = rng.integers(0, 9, n)
        st = M.slice_cuts(w, parts)
        assert st[0] == 0 and st[-1] == n and np.all(np.diff(st) >= 0)
        part_w = [int(w[st[s]:st[s + 1]].sum()) for s in range(parts)]
        assert sum(part_w) == w.sum()
        assert max(part_w) <= -(-int(w.sum()) // parts) + int(w.max()) if n else True
        # each cut is the first place the running total reaches its share: no earlier cut works
        pre = np.concatenate([[0], np.cumsum(w)])
        for s in range(1, parts):
            target = -(-(s * int(w.sum())) // parts)
            assert min(t for t in range(n + 1) if pre[t] >= target or t == n) == st[s]


def test_sfa_pieces_cover_each_unit_evenly():
    """Brute-force properties of the decode split, independent of its formula: the pieces of a
    unit are consecutive, start at 0, end at n, and their lengths differ by at most one (the
    most even split of n pages into P runs); units of one (b, kv head) share its count."""
    rng = np.random.default_rng(3)
    for _ in range(200):
        bgs, HH, P = int(rng.integers(1, 9)), int(rng.integers(1, 3)), int(rng.integers(1, 5))
        count = rng.integers(0, 70, size=bgs).astype(np.int32)
        rec = M.sfa_pieces(count, HH, P)
        assert rec.shape == (bgs * HH * P, 3)
        for u in range(bgs * HH):
            r = rec[u * P:(u + 1) * P]
            n = int(count[u // HH])
            assert (r[:, 0] == n).all()
            assert r[0, 1] == 0 and int(r[-1, 1] + r[-1, 2]) == n
            assert (r[1:, 1] == r[:-1, 1] + r[:-1, 2]).all()
            assert r[:, 2].max() - r[:, 2].min() <= 1 and r[:, 2].min() >= 0
    assert M.sfa_pieces_per_unit(64, 148) == 2 and M.sfa_pieces_per_unit(160, 148) == 1
    assert M.sfa_pieces_per_unit(40, 148) == 3 and M.sfa_pieces_per_unit(1, 148) == 4
