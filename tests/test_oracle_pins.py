"""Pins for the fp64 oracle: each test checks it against something other than itself.

  * torch's scaled_dot_product_attention in float64 on CPU (forward) and its autograd gradients
    (backward), with the selection expanded to a dense boolean mask: BSA, NSA and SFA.
  * central finite differences of L = sum(dOut o Out) for dQ, dK, dV.
  * closed forms and invariants (single visible key, constant V, key shift, rowsum(dS) = 0,
    sum dV = sum dOut, sum dK = 0, LSE = logsumexp of the visible scores).
  * hand-worked fixtures in tests/golden/.
"""
import json
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import attention as A
from workloads import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _dense_mask_bsa(mask, bx, by, s_q, s_kv, mode, wl=0, wr=0):
    """Boolean [B, N1, Sq, Skv], built by expanding blocks (independent of the oracle's gather)."""
    B, N1, nqb, nkb = mask.shape
    blk = np.repeat(np.repeat(mask.astype(bool), bx, axis=2), by, axis=3)[:, :, :s_q, :s_kv]
    i = np.arange(s_q)[:, None]
    j = np.arange(s_kv)[None, :]
    if mode == 0:
        rule = np.ones((s_q, s_kv), dtype=bool)
    elif mode == 2:
        rule = j <= i
    elif mode == 3:
        rule = j <= i + (s_kv - s_q)
    else:
        c = i + (s_kv - s_q)
        rule = (j >= c - wl) & (j <= c + wr)
    return blk & rule[None, None]


def _torch_sdpa(q, k, v, dense, scale, dout=None, q2=None, k2=None):
    """Reference via torch SDPA (float64, CPU).  q [B,N1,Sq,D], k/v [B,N2,Skv,*], dense bool mask
    [B,N1,Sq,Skv].  GQA by repeating kv heads.  Returns out, lse, (dq, dk, dv)."""
    tq = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    tk = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    tv = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    G = q.shape[1] // k.shape[1]
    kk = tk.repeat_interleave(G, dim=1)
    vv = tv.repeat_interleave(G, dim=1)
    qq = tq
    if q2 is not None:
        tq2 = torch.tensor(q2, dtype=torch.float64)
        tk2 = torch.tensor(k2, dtype=torch.float64).repeat_interleave(G, dim=1)
        qq = torch.cat([tq, tq2], dim=-1)
        kk = torch.cat([kk, tk2], dim=-1)
    m = torch.tensor(dense)
    out = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=m, scale=scale)
    scores = (qq @ kk.transpose(-1, -2)) * scale
    lse = torch.logsumexp(scores.masked_fill(~m, float("-inf")), dim=-1)
    res = [out.detach().numpy(), lse.detach().numpy()]
    if dout is not None:
        out.backward(torch.tensor(dout, dtype=torch.float64))
        res += [tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()]
    return res


# ---------------------------------------------------------------------------------------------
# BSA vs dense SDPA
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("mode,s_q,s_kv,bx,by,N1,N2", [
    (2, 64, 64, 16, 16, 2, 2),     # causal, MHA
    (2, 50, 50, 8, 16, 4, 2),      # ragged tail, bx != by, GQA
    (0, 40, 56, 8, 8, 2, 1),       # no mask, Sq != Skv
    (3, 24, 40, 8, 8, 2, 2),       # right-down causal
    (4, 48, 48, 8, 8, 2, 2),       # band
])
def test_bsa_matches_dense_sdpa(mode, s_q, s_kv, bx, by, N1, N2):
    rng = np.random.default_rng(1)
    B, D = 2, 8
    q, k, v, do = _rand(rng, B, N1, s_q, D), _rand(rng, B, N2, s_kv, D), \
        _rand(rng, B, N2, s_kv, D), _rand(rng, B, N1, s_q, D)
    nqb, nkb = -(-s_q // bx), -(-s_kv // by)
    mask = (rng.random((B, N1, nqb, nkb)) < 0.5).astype(np.uint8)
    wl, wr = 9, 2
    dense = _dense_mask_bsa(mask, bx, by, s_q, s_kv, mode, wl, wr)
    scale = 0.37
    dq, dk, dv, out, lse = A.bsa_backward(q, k, v, do, mask, bx, by, mode, scale, wl, wr)
    ok = dense.any(-1)   # rows with no visible key are compared separately below
    r_out, r_lse, r_dq, r_dk, r_dv = _torch_sdpa(q, k, v, np.where(ok[..., None], dense, True), scale,
                                                 np.where(ok[..., None], do, 0.0))
    assert np.allclose(out[ok], r_out[ok], atol=1e-12)
    assert np.allclose(lse[ok], r_lse[ok], atol=1e-12)
    assert np.allclose(dq[ok], r_dq[ok], atol=1e-11)
    assert np.allclose(dk, r_dk, atol=1e-11)
    assert np.allclose(dv, r_dv, atol=1e-11)
    # rows with no visible key: Out = 0, LSE = -inf (reading: fully masked rows)
    assert np.all(out[~ok] == 0) and np.all(np.isneginf(lse[~ok]))
    # the forward-only entry agrees with the backward's recomputed forward
    o2, l2 = A.bsa_forward(q, k, v, mask, bx, by, mode, scale, wl, wr)
    assert np.array_equal(o2, out) and np.array_equal(l2, lse)


def test_bsa_all_blocks_is_dense_causal():
    """Every causal block selected + causal mask == textbook dense causal attention."""
    rng = np.random.default_rng(2)
    B, N, S, D, bs = 1, 2, 64, 16, 16
    q, k, v, do = (_rand(rng, B, N, S, D) for _ in range(4))
    nb = S // bs
    mask = np.broadcast_to(np.tril(np.ones((nb, nb), np.uint8)), (B, N, nb, nb)).copy()
    scale = 1 / np.sqrt(D)
    dq, dk, dv, out, lse = A.bsa_backward(q, k, v, do, mask, bs, bs, 2, scale)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
    o.backward(torch.tensor(do))
    assert np.allclose(out, o.detach().numpy(), atol=1e-12)
    assert np.allclose(dq, tq.grad.numpy(), atol=1e-11)
    assert np.allclose(dk, tk.grad.numpy(), atol=1e-11)
    assert np.allclose(dv, tv.grad.numpy(), atol=1e-11)


# ---------------------------------------------------------------------------------------------
# NSA vs dense SDPA
# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("mode,Dv", [(2, 8), (0, 8), (2, 6)])   # Dv != D: the next scope row's split
def test_nsa_matches_dense_sdpa(mode, Dv):
    rng = np.random.default_rng(3)
    seqlens = [40, 17, 64]
    N1, N2, D, bs, K = 4, 2, 8, 8, 3
    T = sum(seqlens)
    cu = np.concatenate([[0], np.cumsum(seqlens)])
    q, do = _rand(rng, T, N1, D), _rand(rng, T, N1, Dv)
    k, v = _rand(rng, T, N2, D), _rand(rng, T, N2, Dv)
    topk = np.full((T, N2, K), -1, np.int32)
    for b, s in enumerate(seqlens):
        for t in range(s):
            nb = -(-s // bs)
            for g in range(N2):
                own = t // bs
                cand = [x for x in range(nb) if x != own]
                pick = list(rng.choice(cand, size=min(K - 1, len(cand)), replace=False))
                row = [own] + pick
                if rng.random() < 0.3:
                    row = row[:-1]   # leave an empty (-1) slot
                rng.shuffle(row)
                topk[cu[b] + t, g, :len(row)] = row
    scale = 0.41
    dq, dk, dv, out, lse = A.nsa_backward(q, k, v, do, topk, cu, bs, mode, scale)
    for b, s in enumerate(seqlens):
        t0 = cu[b]
        dense = np.zeros((1, N1, s, s), dtype=bool)
        for t in range(s):
            for g in range(N2):
                for j in topk[t0 + t, g]:
                    if j >= 0:
                        dense[0, g * (N1 // N2):(g + 1) * (N1 // N2), t, j * bs:(j + 1) * bs] = True
        if mode == 2:
            dense &= np.tril(np.ones((s, s), dtype=bool))[None, None]
        tr = lambda x: x[t0:t0 + s].transpose(1, 0, 2)[None]  # noqa: E731  TND -> BNSD
        r_out, r_lse, r_dq, r_dk, r_dv = _torch_sdpa(tr(q), tr(k), tr(v), dense, scale, tr(do))
        assert np.allclose(out[t0:t0 + s], r_out[0].transpose(1, 0, 2), atol=1e-12)
        assert np.allclose(lse[t0:t0 + s], r_lse[0].T, atol=1e-12)
        assert np.allclose(dq[t0:t0 + s], r_dq[0].transpose(1, 0, 2), atol=1e-11)
        assert np.allclose(dk[t0:t0 + s], r_dk[0].transpose(1, 0, 2), atol=1e-11)
        assert np.allclose(dv[t0:t0 + s], r_dv[0].transpose(1, 0, 2), atol=1e-11)


def test_nsa_topk_order_and_duplicates():
    """Permuting a topk row changes nothing; a duplicated id is gathered twice (literal Gather):
    it equals attention over the key list with that block repeated."""
    rng = np.random.default_rng(4)
    S, N1, N2, D, bs = 32, 2, 1, 4, 8
    q, k, v = _rand(rng, S, N1, D), _rand(rng, S, N2, D), _rand(rng, S, N2, D)
    cu = np.array([0, S])
    topk = np.array([[[0, 1, 2, 3]]] * S, np.int32)
    o1, l1 = A.nsa_forward(q, k, v, topk, cu, bs, 0, 0.5)
    o2, l2 = A.nsa_forward(q, k, v, topk[:, :, ::-1].copy(), cu, bs, 0, 0.5)
    assert np.allclose(o1, o2, atol=1e-14) and np.allclose(l1, l2, atol=1e-14)
    dup = np.array([[[0, 0, -1, -1]]] * S, np.int32)
    o3, l3 = A.nsa_forward(q, k, v, dup, cu, bs, 0, 0.5)
    s = 0.5 * q[:, 0] @ k[:8, 0].T                      # block 0 scores, head 0
    ref_lse = logsumexp(np.concatenate([s, s], axis=1), axis=1)
    assert np.allclose(l3[:, 0], ref_lse, atol=1e-13)


# ---------------------------------------------------------------------------------------------
# SFA vs dense SDPA on the logical sequence
# ---------------------------------------------------------------------------------------------
def test_sfa_matches_dense_sdpa():
    rng = np.random.default_rng(5)
    B, N1, N2, D, Dr, page, n_logical, K = 2, 4, 2, 16, 4, 8, 6, 3
    n_pages = B * n_logical + 3
    table = rng.permutation(n_pages)[:B * n_logical].reshape(B, n_logical).astype(np.int32)
    kc, krc, vc = _rand(rng, n_pages, page, N2, D), _rand(rng, n_pages, page, N2, Dr), \
        _rand(rng, n_pages, page, N2, D)
    q, qr = _rand(rng, B, 1, N1, D), _rand(rng, B, 1, N1, Dr)
    seqused = np.array([n_logical * page, n_logical * page - 5])
    idx = np.full((B, 1, N2, K), -1, np.int32)
    for b in range(B):
        for g in range(N2):
            idx[b, 0, g] = rng.choice(n_logical, size=K, replace=False)
    idx[1, 0, 1, 2] = -1
    scale = 1 / np.sqrt(D + Dr)
    out, lse = A.sfa_decode(q, qr, kc, krc, vc, table, idx, seqused, page, page, scale)
    for b in range(B):
        # logical K/V of batch b
        lk = np.concatenate([kc[table[b, lp]] for lp in range(n_logical)])       # [L, N2, D]
        lkr = np.concatenate([krc[table[b, lp]] for lp in range(n_logical)])
        lv = np.concatenate([vc[table[b, lp]] for lp in range(n_logical)])
        dense = np.zeros((1, N1, 1, n_logical * page), dtype=bool)
        G = N1 // N2
        for g in range(N2):
            for j in idx[b, 0, g]:
                if j >= 0:
                    dense[0, g * G:(g + 1) * G, 0, j * page:(j + 1) * page] = True
        dense[..., seqused[b]:] = False
        tr = lambda x: x.transpose(1, 0, 2)[None]  # noqa: E731
        r_out, r_lse = _torch_sdpa(q[b].transpose(1, 0, 2)[None], tr(lk), tr(lv), dense, scale,
                                   q2=qr[b].transpose(1, 0, 2)[None], k2=tr(lkr))
        assert np.allclose(out[b, 0], r_out[0, :, 0], atol=1e-12)
        assert np.allclose(lse[b, 0], r_lse[0, :, 0], atol=1e-12)


def test_sfa_readings_multi_page_blocks_duplicates_and_empty():
    """Sparse blocks of two scattered pages each, a sequence cut inside a page, a duplicated id
    (gathered twice, the literal reading) and a row with no valid id (Out = 0, LSE = -inf), against
    dense SDPA over an explicitly built key list."""
    rng = np.random.default_rng(9)
    B, N1, N2, D, Dr, page, ppb, n_logical, K = 2, 4, 1, 8, 4, 4, 2, 8, 3
    sbs = page * ppb
    n_pages = B * n_logical + 2
    table = rng.permutation(n_pages)[:B * n_logical].reshape(B, n_logical).astype(np.int32)
    kc, krc, vc = _rand(rng, n_pages, page, N2, D), _rand(rng, n_pages, page, N2, Dr), \
        _rand(rng, n_pages, page, N2, D)
    q, qr = _rand(rng, B, 1, N1, D), _rand(rng, B, 1, N1, Dr)
    seqused = np.array([n_logical * page - 3, 0])        # batch 0 ends inside its last page
    idx = np.array([[[[3, 1, 3]]], [[[-1, -1, -1]]]], np.int32)  # block 3 listed twice; batch 1 empty
    scale = 0.4
    out, lse = A.sfa_decode(q, qr, kc, krc, vc, table, idx, seqused, page, sbs, scale)
    # batch 0: keys of blocks 3, 1, 3 in that order, each block = logical pages 2j, 2j + 1
    toks = [j * sbs + t for j in (3, 1, 3) for t in range(sbs) if j * sbs + t < seqused[0]]
    kk = np.stack([kc[table[0, t // page], t % page] for t in toks])      # [L, N2, D]
    kr = np.stack([krc[table[0, t // page], t % page] for t in toks])
    vv = np.stack([vc[table[0, t // page], t % page] for t in toks])
    tr = lambda x: x.transpose(1, 0, 2)[None]  # noqa: E731
    dense = np.ones((1, N1, 1, len(toks)), dtype=bool)
    r_out, r_lse = _torch_sdpa(q[0].transpose(1, 0, 2)[None], tr(kk), tr(vv), dense, scale,
                               q2=qr[0].transpose(1, 0, 2)[None], k2=tr(kr))
    assert len(toks) == 3 * sbs - 2 * 3  # block 3 holds the cut page (3 tokens past the end), twice
    assert np.allclose(out[0, 0], r_out[0, :, 0], atol=1e-12)
    assert np.allclose(lse[0, 0], r_lse[0, :, 0], atol=1e-12)
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1]))


def _sfa_small(rng, Sq=1):
    B, N1, N2, D, Dr, page, ppb, n_logical, K = 2, 4, 2, 8, 4, 4, 2, 8, 3
    n_pages = B * n_logical + 2
    table = rng.permutation(n_pages)[:B * n_logical].reshape(B, n_logical).astype(np.int32)
    kc, krc, vc = _rand(rng, n_pages, page, N2, D), _rand(rng, n_pages, page, N2, Dr), \
        _rand(rng, n_pages, page, N2, D)
    q, qr, do = _rand(rng, B, Sq, N1, D), _rand(rng, B, Sq, N1, Dr), _rand(rng, B, Sq, N1, D)
    seqused = np.array([n_logical * page - 3, n_logical * page])
    idx = np.array([[[[3, 1, 3], [0, -1, 2]]], [[[2, 0, -1], [1, 3, 2]]]], np.int32)  # a duplicate, empty slots
    return dict(q=q, qr=qr, do=do, kc=kc, krc=krc, vc=vc, table=table, idx=idx, seqused=seqused,
                page=page, sbs=page * ppb)


def test_sfa_backward_matches_autograd():
    """Sparse-decode backward against torch float64 autograd through an explicit gather from
    leaf cache tensors (torch's indexing backward does the scatter-add, duplicates included)."""
    rng = np.random.default_rng(10)
    for Sq in (1, 2):
        pb = _sfa_small(rng, Sq)
        scale = 0.35
        dq, dqr, dk, dkr, dv, out, lse = A.sfa_backward(pb["q"], pb["qr"], pb["kc"], pb["krc"], pb["vc"],
                                                        pb["do"], pb["table"], pb["idx"], pb["seqused"],
                                                        pb["page"], pb["sbs"], scale)
        t = {n: torch.tensor(pb[n], dtype=torch.float64, requires_grad=True) for n in ("q", "qr", "kc", "krc", "vc")}
        B, _, N1, _ = pb["q"].shape
        N2 = pb["kc"].shape[2]
        G = N1 // N2
        loss = 0.0
        for b in range(B):
            for g in range(N2):
                toks = [j * pb["sbs"] + i for j in pb["idx"][b, 0, g] if j >= 0 for i in range(pb["sbs"])
                        if j * pb["sbs"] + i < pb["seqused"][b]]
                pages = torch.tensor([int(pb["table"][b, x // pb["page"]]) for x in toks])
                offs = torch.tensor([x % pb["page"] for x in toks])
                kk = torch.cat([t["kc"][pages, offs, g], t["krc"][pages, offs, g]], dim=-1)
                vv = t["vc"][pages, offs, g]
                qq = torch.cat([t["q"][b, :, g * G:(g + 1) * G], t["qr"][b, :, g * G:(g + 1) * G]], dim=-1)
                o = torch.nn.functional.scaled_dot_product_attention(qq.transpose(0, 1), kk[None], vv[None],
                                                                     scale=scale)
                loss = loss + (o.transpose(0, 1) * torch.tensor(pb["do"][b, :, g * G:(g + 1) * G])).sum()
                assert np.allclose(out[b, :, g * G:(g + 1) * G], o.transpose(0, 1).detach().numpy(), atol=1e-12)
        loss.backward()
        for got, name in ((dq, "q"), (dqr, "qr"), (dk, "kc"), (dkr, "krc"), (dv, "vc")):
            assert np.allclose(got, t[name].grad.numpy(), atol=1e-12), name


def test_sfa_backward_finite_differences():
    rng = np.random.default_rng(12)
    pb = _sfa_small(rng)
    scale = 0.35
    args = lambda: (pb["table"], pb["idx"], pb["seqused"], pb["page"], pb["sbs"], scale)  # noqa: E731
    dq, dqr, dk, dkr, dv, _, _ = A.sfa_backward(pb["q"], pb["qr"], pb["kc"], pb["krc"], pb["vc"], pb["do"], *args())

    def loss():
        return float(np.sum(pb["do"] * A.sfa_decode(pb["q"], pb["qr"], pb["kc"], pb["krc"], pb["vc"], *args())[0]))

    _fd_check(loss, [pb["q"], pb["qr"]], [dq, dqr])
    # the cache rows of one read page of each kind (a page read twice through the duplicated block)
    page = int(pb["table"][0, 3 * 2])  # block 3 of batch 0 = logical pages 6, 7
    for name, g in (("kc", dk), ("krc", dkr), ("vc", dv)):
        _fd_check(loss, [pb[name][page]], [g[page]])


# ---------------------------------------------------------------------------------------------
# finite differences
# ---------------------------------------------------------------------------------------------
def _fd_check(loss, params, grads, h=1e-6, tol=1e-7):
    for x, g in zip(params, grads):
        flat = x.reshape(-1)
        gf = g.reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + h
            lp = loss()
            flat[i] = old - h
            lm = loss()
            flat[i] = old
            num = (lp - lm) / (2 * h)
            assert abs(num - gf[i]) <= tol * max(1.0, abs(num)) + 1e-8, (i, num, gf[i])


def test_bsa_finite_differences():
    rng = np.random.default_rng(6)
    B, N1, N2, S, D, bs = 1, 2, 1, 16, 4, 4
    q, k, v, do = _rand(rng, B, N1, S, D), _rand(rng, B, N2, S, D), _rand(rng, B, N2, S, D), \
        _rand(rng, B, N1, S, D)
    mask = (rng.random((B, N1, 4, 4)) < 0.6).astype(np.uint8)
    for i in range(4):
        mask[:, :, i, i] = 1
    sc = 0.6
    dq, dk, dv, _, _ = A.bsa_backward(q, k, v, do, mask, bs, bs, 2, sc)
    loss = lambda: float(np.sum(do * A.bsa_forward(q, k, v, mask, bs, bs, 2, sc)[0]))  # noqa: E731
    _fd_check(loss, [q, k, v], [dq, dk, dv])


def test_nsa_finite_differences():
    rng = np.random.default_rng(7)
    S, N1, N2, D, bs = 16, 2, 1, 4, 4
    q, k, v, do = _rand(rng, S, N1, D), _rand(rng, S, N2, D), _rand(rng, S, N2, D), _rand(rng, S, N1, D)
    topk = np.full((S, N2, 3), -1, np.int32)
    for t in range(S):
        own = t // bs
        topk[t, 0, 0] = own
        if own:
            topk[t, 0, 1] = rng.integers(0, own)
    cu = np.array([0, S])
    dq, dk, dv, _, _ = A.nsa_backward(q, k, v, do, topk, cu, bs, 2, 0.7)
    loss = lambda: float(np.sum(do * A.nsa_forward(q, k, v, topk, cu, bs, 2, 0.7)[0]))  # noqa: E731
    _fd_check(loss, [q, k, v], [dq, dk, dv])


# ---------------------------------------------------------------------------------------------
# invariants and closed forms
# ---------------------------------------------------------------------------------------------
def test_invariants_on_tiny_workload():
    """The tiny BSA workload (64x64 blocks, S=512): P rows sum to 1, rowsum(dS) = 0,
    sum_k dV[k] = sum_i dOut_i, sum_k dK[k] = 0, LSE = logsumexp(visible scores) >= max."""
    w = synth.workload(1)
    mask = w.block_mask()
    q, k, v, do = (A.bf16_to_f64(w.tensor(t)) for t in ("q", "k", "v", "dout"))
    dq, dk, dv, out, lse = A.bsa_backward(q, k, v, do, mask, w.block, w.block, 2, w.scale)
    assert np.allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-9)
    assert np.allclose(dk.sum(axis=2), 0, atol=1e-9)
    # per-row checks on a few units through the building blocks
    for (h, qb) in [(0, 0), (1, 5), (0, 7)]:
        rows = np.arange(qb * 64, (qb + 1) * 64)
        keys = A.bsa_unit_keys(mask[0, h, qb], 64, 512)
        vis = A.visible(rows, keys, 2, 512, 512, 512)
        o, l, p = A.attend(q[0, h, rows], k[0, h, keys], v[0, h, keys], vis, w.scale)
        assert np.allclose(p.sum(axis=1), 1, atol=1e-14)
        s = w.scale * q[0, h, rows] @ k[0, h, keys].T
        assert np.allclose(l, logsumexp(np.where(vis, s, -np.inf), axis=1), atol=1e-12)
        assert np.all(l >= np.where(vis, s, -np.inf).max(axis=1))
        dp = do[0, h, rows] @ v[0, h, keys].T
        ds = p * (dp - np.sum(do[0, h, rows] * o, axis=1)[:, None])
        assert np.allclose(ds.sum(axis=1), 0, atol=1e-12)
        assert np.allclose(o, out[0, h, rows], atol=0) and np.allclose(l, lse[0, h, rows], atol=0)


def test_closed_forms():
    rng = np.random.default_rng(8)
    B, N, S, D, bs = 1, 1, 32, 8, 8
    q, k, v, do = (_rand(rng, B, N, S, D) for _ in range(4))
    mask = np.tril(np.ones((4, 4), np.uint8))[None, None]
    sc = 0.3
    dq, dk, dv, out, lse = A.bsa_backward(q, k, v, do, mask, bs, bs, 2, sc)
    # row 0 sees only key 0: Out = v0, LSE = scale q0.k0, zero dQ
    assert np.allclose(out[0, 0, 0], v[0, 0, 0], atol=1e-15)
    assert np.isclose(lse[0, 0, 0], sc * q[0, 0, 0] @ k[0, 0, 0])
    assert np.allclose(dq[0, 0, 0], 0, atol=1e-15)
    # constant V: Out = c, dQ = dK = 0
    vc = np.full_like(v, 1.75)
    dq2, dk2, _, out2, _ = A.bsa_backward(q, k, vc, do, mask, bs, bs, 2, sc)
    assert np.allclose(out2, 1.75, atol=1e-14)
    assert np.allclose(dq2, 0, atol=1e-13) and np.allclose(dk2, 0, atol=1e-13)
    # shifting every key by c: Out unchanged, LSE shifts by scale q.c
    c = _rand(rng, D)
    out3, lse3 = A.bsa_forward(q, k + c, v, mask, bs, bs, 2, sc)
    assert np.allclose(out3, out, atol=1e-12)
    assert np.allclose(lse3, lse + sc * q @ c, atol=1e-12)


def test_golden_two_key_example():
    """Hand-worked fixture: forward and backward formulas on two keys (values derived by hand)."""
    with open(os.path.join(GOLDEN, "two_key_example.json")) as f:
        g = json.load(f)
    q = np.array(g["q"], float)[None]
    k = np.array(g["k"], float)
    v = np.array(g["v"], float)
    do = np.array(g["dout"], float)[None]
    vis = np.ones((1, 2), bool)
    out, lse, p = A.attend(q, k, v, vis, g["scale"])
    dq, dk, dv = A.attend_grad(q, k, v, do, out, p, g["scale"])
    ex = g["expected"]
    assert np.allclose(p[0], ex["P"], atol=1e-15)
    assert np.allclose(out[0], ex["out"], atol=1e-14)
    assert np.isclose(lse[0], ex["lse"], atol=1e-15)
    assert np.allclose(dq[0], ex["dq"], atol=1e-14)
    assert np.allclose(dk, ex["dk"], atol=1e-14)
    assert np.allclose(dv, ex["dv"], atol=1e-14)


def test_planted_mistakes_are_caught(monkeypatch):
    """Plant plausible mistakes in the oracle's backward and check the dense pin rejects them."""
    rng = np.random.default_rng(9)
    B, N, S, D, bs = 1, 2, 32, 8, 8
    q, k, v, do = (_rand(rng, B, N, S, D) for _ in range(4))
    mask = np.tril(np.ones((4, 4), np.uint8))[None, None].repeat(N, 1)
    dense = _dense_mask_bsa(mask, bs, bs, S, S, 2)
    _, _, r_dq, r_dk, r_dv = _torch_sdpa(q, k, v, dense, 0.5, do)
    good = A.attend_grad

    def dropped_term(q_, k_, v_, dout, out, p, scale, *a):
        dq, dk, dv = good(q_, k_, v_, dout, out * 0, p, scale)   # softmax_grad term dropped
        return dq, dk, dv

    def wrong_operand(q_, k_, v_, dout, out, p, scale, *a):
        dq, dk, dv = good(q_, k_, v_, dout, out, p, scale)
        return dq, (p.T @ dout) * scale if dk.shape == (p.T @ dout).shape else dk, dv

    for bad in (dropped_term, wrong_operand):
        monkeypatch.setattr(A, "attend_grad", bad)
        dq, dk, dv, _, _ = A.bsa_backward(q, k, v, do, mask, bs, bs, 2, 0.5)
        assert not (np.allclose(dq, r_dq, atol=1e-9) and np.allclose(dk, r_dk, atol=1e-9)
                    and np.allclose(dv, r_dv, atol=1e-9))
    monkeypatch.setattr(A, "attend_grad", good)


def test_stored_out_softmax_grad_correction():
    """softmax_grad taken from the bf16-stored attentionOut: since dS = P o (dP - D) is linear in D,
    dQ_i moves by exactly -scale * dD_i * (P K)_i and dK_k by -scale * sum_i dD_i P_ik q_i, with
    dD_i = dOut_i . (bf16(O_i) - O_i); dV does not move.  P, O and the base gradients come from
    torch (float64) here, not from the oracle."""
    rng = np.random.default_rng(10)
    B, N, S, D, bs = 1, 1, 32, 16, 8
    bits = [synth.f32_to_bf16_bits(rng.standard_normal((B, N, S, D), dtype=np.float32)) for _ in range(4)]
    q, k, v, do = (A.bf16_to_f64(x) for x in bits)
    mask = np.tril(np.ones((4, 4), np.uint8))[None, None]
    sc = 0.25
    dq_b, dk_b, dv_b, _, _ = A.bsa_backward(*bits, mask, bs, bs, 2, sc)   # bf16 inputs: stored Out
    dense = _dense_mask_bsa(mask, bs, bs, S, S, 2)
    _, _, r_dq, r_dk, r_dv = _torch_sdpa(q, k, v, dense, sc, do)          # exact D
    s = sc * np.einsum("bhid,bhjd->bhij", q, k)
    s = np.where(dense, s, -np.inf)
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    o = p @ v
    dD = np.sum(do * (_nearest_bf16_bruteforce(o) - o), axis=-1)         # [B, N, S]
    exp_dq = r_dq - sc * dD[..., None] * (p @ k)
    exp_dk = r_dk - sc * np.einsum("bhi,bhij,bhid->bhjd", dD, p, q)
    assert np.abs(dD).max() > 0                                          # the reading matters here
    assert np.allclose(dq_b, exp_dq, atol=1e-11)
    assert np.allclose(dk_b, exp_dk, atol=1e-11)
    assert np.allclose(dv_b, r_dv, atol=1e-11)


# ---------------------------------------------------------------------------------------------
# round_to_bf16 (the stored-attentionOut reading rests on it): pinned against torch's float32 ->
# bfloat16 cast, a brute-force nearest search over every finite bf16 value, and a hand-worked table
# ---------------------------------------------------------------------------------------------
def _all_finite_bf16():
    """Every finite bf16 value (as float64) with its bit pattern, sorted by value."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    vals = (bits << 16).view(np.float32).astype(np.float64)
    fin = np.isfinite(vals)
    vals, bits = vals[fin], bits[fin]
    order = np.lexsort((bits, vals))
    vals, bits = vals[order], bits[order]
    keep = np.concatenate([[True], vals[1:] != vals[:-1]])   # +0 and -0 collapse to one grid point
    return vals[keep], bits[keep]


def _nearest_bf16_bruteforce(x):
    """Nearest grid point of the finite bf16 values extended by +-2^128 (standing for +-inf), ties
    to the point whose bit pattern is even."""
    vals, bits = _all_finite_bf16()
    vals = np.concatenate([[-2.0 ** 128], vals, [2.0 ** 128]])
    bits = np.concatenate([[0xFF80], bits, [0x7F80]]).astype(np.uint32)
    i = np.clip(np.searchsorted(vals, x), 1, len(vals) - 1)
    lo, hi = vals[i - 1], vals[i]
    dlo, dhi = x - lo, hi - x
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (bits[i] % 2 == 0))
    y = np.where(pick_hi, hi, lo)
    y = np.where(np.abs(y) >= 2.0 ** 128, np.copysign(np.inf, y), y)
    return np.where(y == 0, np.copysign(0.0, x), y)


def test_round_to_bf16_matches_torch_on_float32_values():
    """On float32 inputs (no rounding before the bf16 step) torch's cast is round-to-nearest-even:
    every finite float32 exponent, ties (low 16 bits exactly 0x8000), overflow, subnormals."""
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 1 << 32, size=300_000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 1 << 16, size=50_000, dtype=np.uint64).astype(np.uint32) << 16) | np.uint32(0x8000)
    edges = np.array([0x7F7F7FFF, 0x7F7F8000, 0x7F7F8001, 0xFF7F8000, 0x00008000, 0x00018000, 0x007FFFFF,
                      0x00800000, 0x3F808000, 0x3F818000, 0x80000000, 0x00000000], dtype=np.uint32)
    x = np.concatenate([bits, ties, edges]).view(np.float32)
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    got = A.round_to_bf16(x.astype(np.float64))
    assert np.array_equal(np.signbit(got), np.signbit(ref))
    assert np.array_equal(got, ref)


def test_round_to_bf16_is_the_nearest_bf16_of_float64_values():
    """For float64 inputs (between float32 values too) the result is the nearest bf16 value found
    by brute force over the whole bf16 grid, ties to even; rounding through float32 first would
    differ on values just above a tie, which this set contains."""
    rng = np.random.default_rng(13)
    x = rng.standard_normal(200_000) * np.exp2(rng.integers(-140, 129, size=200_000))
    vals, _ = _all_finite_bf16()
    mids = (vals[1:] + vals[:-1]) / 2
    near_ties = rng.choice(mids, 20_000) * (1 + rng.choice([-1, 1], 20_000) * 2.0 ** -40)
    x = np.concatenate([x, rng.choice(mids, 20_000), near_ties])
    x = x[np.isfinite(x)]
    assert np.array_equal(A.round_to_bf16(x), _nearest_bf16_bruteforce(x))


def test_round_to_bf16_golden_table():
    with open(os.path.join(GOLDEN, "bf16_rounding.json")) as f:
        doc = json.load(f)
    for c in doc["cases"]:
        x, want = float.fromhex(c["x"]), float.fromhex(c["bf16"])
        got = float(A.round_to_bf16(np.array([x]))[0])
        assert got == want and np.signbit(got) == np.signbit(want), (c["why"], got, want)


def test_backward_with_given_attention_out():
    """The backward operator's attentionOut input enters only softmax_grad = rowsum(dOut o Out):
    with Out_in = Out + E, dQ moves by -scale (dOut.E)_i (P K)_i, dK by -scale sum_i (dOut.E)_i
    P_ik q_i and dV not at all; P, Out and the base gradients from torch (float64).  Checked for
    the BSA and the NSA entry points (NSA: one token per block, so its keys are a BSA block)."""
    rng = np.random.default_rng(14)
    B, N, S, D, bs = 1, 2, 32, 16, 8
    q, k, v, do = (_rand(rng, B, N, S, D) for _ in range(4))
    mask = np.tril(np.ones((4, 4), np.uint8))[None, None].repeat(N, 1)
    sc = 0.3
    dense = _dense_mask_bsa(mask, bs, bs, S, S, 2)
    r_out, _, r_dq, r_dk, r_dv = _torch_sdpa(q, k, v, dense, sc, do)
    E = _rand(rng, B, N, S, D) * 0.01
    dq, dk, dv, _, _ = A.bsa_backward(q, k, v, do, mask, bs, bs, 2, sc, out_in=r_out + E)
    s = sc * np.einsum("bhid,bhjd->bhij", q, k)
    s = np.where(dense, s, -np.inf)
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    dD = np.sum(do * E, axis=-1)
    assert np.allclose(dq, r_dq - sc * dD[..., None] * (p @ k), atol=1e-11)
    assert np.allclose(dk, r_dk - sc * np.einsum("bhi,bhij,bhid->bhjd", dD, p, q), atol=1e-11)
    assert np.allclose(dv, r_dv, atol=1e-11)
    # NSA: TND with N2 = N (G = 1), every token lists all causal blocks
    qt, kt, vt, dot = (x[0].transpose(1, 0, 2) for x in (q, k, v, do))      # [S, N, D]
    topk = np.array([[list(range(t // bs + 1)) + [-1] * (3 - t // bs) for _ in range(N)] for t in range(S)],
                    dtype=np.int32)
    Et = E[0].transpose(1, 0, 2)
    ndq, ndk, ndv, _, _ = A.nsa_backward(qt, kt, vt, dot, topk, np.array([0, S]), bs, 2, sc,
                                         out_in=r_out[0].transpose(1, 0, 2) + Et)
    assert np.allclose(ndq, (r_dq - sc * dD[..., None] * (p @ k))[0].transpose(1, 0, 2), atol=1e-11)
    assert np.allclose(ndv, r_dv[0].transpose(1, 0, 2), atol=1e-11)


@pytest.mark.parametrize("mode,s_q,s_kv", [(2, 48, 48), (0, 40, 56), (3, 32, 48)])
def test_bsa_dense_atten_mask_matches_sdpa(mode, s_q, s_kv):
    """The dense atten_mask ([S_q, S_kv], nonzero = masked out) on top of the block selection and
    the mode: forward and gradients equal torch SDPA (float64) under the combined boolean mask;
    rows the mask leaves without a key give Out = 0, LSE = -inf and zero dQ."""
    rng = np.random.default_rng(15)
    B, N1, N2, D, bx, by = 1, 2, 1, 8, 8, 8
    q, do = _rand(rng, B, N1, s_q, D), _rand(rng, B, N1, s_q, D)
    k, v = _rand(rng, B, N2, s_kv, D), _rand(rng, B, N2, s_kv, D)
    nqb, nkb = -(-s_q // bx), -(-s_kv // by)
    mask = (rng.random((B, N1, nqb, nkb)) < 0.7).astype(np.uint8)
    am = (rng.random((s_q, s_kv)) < 0.3).astype(np.uint8)
    am[5] = 1  # a row with no key left
    dense = _dense_mask_bsa(mask, bx, by, s_q, s_kv, mode) & (am == 0)[None, None]
    dq, dk, dv, out, lse = A.bsa_backward(q, k, v, do, mask, bx, by, mode, 0.4, atten_mask=am)
    live = dense.any(-1)                                     # [B, N1, S_q]
    assert not live[..., 5].any()
    r_out, r_lse, r_dq, r_dk, r_dv = _torch_sdpa(q, k, v, np.where(live[..., None], dense, True), 0.4,
                                                 np.where(live[..., None], do, 0.0))
    assert np.allclose(out[live], r_out[live], atol=1e-12)
    assert np.allclose(lse[live], r_lse[live], atol=1e-12)
    assert np.all(out[~live] == 0) and np.all(np.isneginf(lse[~live])) and np.all(dq[~live] == 0)
    assert np.allclose(dq, np.where(live[..., None], r_dq, 0.0), atol=1e-11)
    assert np.allclose(dk, r_dk, atol=1e-11) and np.allclose(dv, r_dv, atol=1e-11)
