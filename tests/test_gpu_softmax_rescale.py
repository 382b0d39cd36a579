"""GPU parity of the online softmax's rescale path: inputs whose every later KV tile raises the
running row maximum by more than the 2^8 a tile may exceed it without a rescale (each test checks
that on its inputs before the launch), so the output accumulated so far is rescaled at every
tile, in the BSA forward, the NSA forward and the paged decode.  Random N(0, 1) inputs never reach
that path.  The softmax stays spread over many keys, so bf16 P rounding stays well inside the
tolerance."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import attention as A
from parity import LSE_ATOL, check_close, check_lse, dev_bf16
from test_gpu_nsa import D, _fwd as _nsa_fwd, _problem as _nsa_problem
from test_gpu_sfa import _run as _sfa_run
from workloads import synth

pytestmark = pytest.mark.gpu


def _bsa_rescale_problem(seed=13):
    """B=1, two query heads on one kv head, S=512 in four 128-key blocks, every block selected, no
    mask.  Every query has +16 in dim 0 and every key of block j has 14 j there, so block j's
    scores sit ~10 j (natural units, at half the usual scale) above block 0's."""
    rng = np.random.default_rng(seed)
    B, N1, N2, S, D, blk = 1, 2, 1, 512, 128, 128
    f = lambda *s: rng.standard_normal(s, dtype=np.float32)  # noqa: E731
    q, k, v = f(B, N1, S, D), f(B, N2, S, D), f(B, N2, S, D)
    q[..., 0] += 16.0
    k[..., 0] = 14.0 * (np.arange(S) // blk)
    bits = synth.f32_to_bf16_bits
    mask = np.ones((B, N1, S // blk, S // blk), np.uint8)
    return bits(q), bits(k), bits(v), mask, blk, 0.5 / np.sqrt(D)  # half scale: flatter within a block


def _bsa_block_jumps(q, k, blk, scale):
    """Smallest, over rows and KV blocks after the first, of (the block's max score) - (max over
    the earlier blocks), in log2 units: the forward visits a unit's blocks in ascending order."""
    qq = synth.bf16_bits_to_f32(q).astype(np.float64)[0]
    kk = synth.bf16_bits_to_f32(k).astype(np.float64)[0, 0]
    s = np.einsum("hsd,td->hst", qq, kk) * scale / np.log(2.0)
    bm = s.reshape(s.shape[0], s.shape[1], -1, blk).max(-1)
    run = np.maximum.accumulate(bm, axis=-1)
    return float((bm[..., 1:] - run[..., :-1]).min())


def test_bsa_fwd_lazy_rescale(cuda_ok):
    """Each KV tile raises every row's running maximum by far more than the 2^8 a tile may exceed
    it without a rescale (checked on the inputs), so the output accumulated in TMEM is rescaled at
    every tile; the softmax stays spread over the last block's keys."""
    q, k, v, mask, blk, scale = _bsa_rescale_problem()
    assert _bsa_block_jumps(q, k, blk, scale) > 8.0
    out, lse = sa.bsa_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), torch.from_numpy(mask).cuda(), blk, blk, 0, scale)
    torch.cuda.synchronize()
    r_out, r_lse = A.bsa_forward(q, k, v, mask, blk, blk, 0, scale)
    check_close(out.float().cpu().numpy(), r_out, "out")
    assert np.abs(lse.cpu().numpy() - r_lse).max() <= LSE_ATOL


def _nsa_rescale_problem(seed=29):
    """One 320-token batch (five 64-token blocks), G = 16 heads on one kv head, every block
    selected, no mask.  Every query has +16 in dim 0 and every key of block j has 14 j there, so
    block j's scores sit ~10 j (natural units, at half the usual scale) above block 0's."""
    pb = _nsa_problem([320], N1=16, N2=1, bs=64, K=5, mode=0, seed=seed)
    q = synth.bf16_bits_to_f32(pb["q"])
    k = synth.bf16_bits_to_f32(pb["k"])
    q[..., 0] += 16.0
    k[:, :, 0] = 14.0 * (np.arange(320) // 64)[:, None]
    pb["q"], pb["k"] = synth.f32_to_bf16_bits(q), synth.f32_to_bf16_bits(k)
    pb["scale"] = 0.5 / np.sqrt(D)  # flatter within a block: no single bf16 P carries a row
    return pb


def _nsa_block_jumps(pb):
    """Smallest, over (token, head) and selected blocks after the first, of (the block's max
    score) - (max over the earlier selected blocks), in log2 units: the token kernels visit a
    token's blocks in ascending id order."""
    q = synth.bf16_bits_to_f32(pb["q"]).astype(np.float64)
    k = synth.bf16_bits_to_f32(pb["k"]).astype(np.float64)[:, 0]
    worst = np.inf
    for t in range(q.shape[0]):
        ids = sorted(int(x) for x in pb["topk"][t, 0] if x >= 0)
        s = q[t] @ k.T * pb["scale"] / np.log(2.0)  # [heads, keys]
        bm = np.stack([s[:, i * 64:(i + 1) * 64].max(-1) for i in ids], -1)
        run = np.maximum.accumulate(bm, axis=-1)
        worst = min(worst, float((bm[:, 1:] - run[:, :-1]).min()))
    return worst


def test_nsa_fwd_lazy_rescale(cuda_ok):
    """Each selected block raises every (token, head) row's running maximum by far more than the
    2^8 a chunk may exceed it without a rescale (checked on the inputs), so the output accumulated
    in registers is rescaled at every block; the softmax stays spread over the top block's keys."""
    pb = _nsa_rescale_problem()
    assert (pb["topk"] >= 0).all() and _nsa_block_jumps(pb) > 8.0
    out, lse = _nsa_fwd(pb)
    r_out, r_lse = A.nsa_forward(pb["q"], pb["k"], pb["v"], pb["topk"], pb["cu"], pb["bs"], pb["mode"], pb["scale"])
    check_close(out.float().cpu().numpy(), r_out, "out")
    check_lse(lse.cpu().numpy(), r_lse)


def _sfa_rescale_problem(seed=5):
    """One batch, 128 query heads, 150 selected one-page blocks of a 10000-token sequence.  All
    query heads share a component of 16 along dim 0, and the keys of every page at a list position
    = 2 (mod 3) carry +40 there: their scores sit ~27 (natural units) above the others, uniformly
    over the page's tokens."""
    rng = np.random.default_rng(seed)
    n1, page, n_logical, k_sel, used = 128, 64, 160, 150, 10000
    n_pages = n_logical + 5
    table = rng.permutation(n_pages)[:n_logical].reshape(1, n_logical).astype(np.int32)
    nsb = -(-used // page)
    idx = rng.choice(nsb, size=k_sel, replace=False).astype(np.int32).reshape(1, 1, 1, k_sel)
    f = lambda *s: rng.standard_normal(s, dtype=np.float32)  # noqa: E731
    q, qr = f(1, 1, n1, 512), f(1, 1, n1, 64)
    kc, krc, vc = f(n_pages, page, 1, 512), f(n_pages, page, 1, 64), f(n_pages, page, 1, 512)
    q[..., 0] += 16.0
    kc[table[0, idx[0, 0, 0, 2::3]], :, 0, 0] += 40.0
    bits = synth.f32_to_bf16_bits
    return dict(q=bits(q), qr=bits(qr), kc=bits(kc), krc=bits(krc), vc=bits(vc), table=table, idx=idx,
                seqused=np.array([used], np.int32), page=page, sbs=page)


def _sfa_tile_maxima_jump(pb, scale, wave=148):
    """Smallest, over pieces and heads, of (max score of a piece's second tile) - (max of its
    first), in log2 units, for the decode's work split: units (batch, kv head, head half of 64),
    pieces of `chunk` consecutive pages (the smallest chunk whose pieces fit one wave), tiles of
    128 tokens (two pages of 64)."""
    f64 = lambda b: synth.bf16_bits_to_f32(b).astype(np.float64)  # noqa: E731
    page, used = pb["page"], int(pb["seqused"][0])
    pages = [int(pb["table"][0, j]) for j in pb["idx"][0, 0, 0]]
    n = len(pages)
    units = 2  # G = 128: two head halves
    chunk = next(c for c in range(1, n + 1) if units * -(-n // c) <= wave)
    q = f64(pb["q"])[0, 0]
    qr = f64(pb["qr"])[0, 0]
    kc, krc = f64(pb["kc"])[:, :, 0], f64(pb["krc"])[:, :, 0]
    sc = scale / np.log(2.0)
    worst = np.inf
    for p0 in range(0, n, chunk):
        tiles = [pages[p0:p0 + chunk][t:t + 2] for t in range(0, min(chunk, n - p0), 2)]
        if len(tiles) < 2:
            continue
        mx = []
        for tl in tiles[:2]:
            rows = []
            for pos, pg in zip(range(p0, p0 + chunk), tl):
                blk = int(pb["idx"][0, 0, 0, pages.index(pg)])
                valid = min(page, used - blk * page)
                rows.append((kc[pg, :valid] @ q.T + krc[pg, :valid] @ qr.T) * sc)
            mx.append(np.concatenate(rows).max(axis=0))
        worst = min(worst, float((mx[1] - mx[0]).min()))
    return chunk, worst


def test_sfa_decode_lazy_rescale(cuda_ok):
    """Every piece's second tile raises the running maximum by far more than the 2^8 a tile may
    exceed it without a rescale (checked on the inputs first), so the output columns the first
    tile accumulated are rescaled in every piece; the softmax stays spread over the hot pages'
    tokens, so bf16 P rounding stays well inside the tolerance."""
    pb = _sfa_rescale_problem()
    scale = 1 / np.sqrt(576)
    chunk, jump = _sfa_tile_maxima_jump(pb, scale)
    assert chunk == 3 and jump > 8.0
    used_pages = sorted({int(p) for p in pb["table"][0, pb["idx"][0, 0, 0]]})
    pb["dev"] = {}
    for name, arr in (("k", pb["kc"]), ("kr", pb["krc"]), ("v", pb["vc"])):
        t = torch.full(arr.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        t[used_pages] = dev_bf16(arr[used_pages])
        pb["dev"][name] = t
    out, lse, r_out, r_lse = _sfa_run(pb, scale)
    check_close(out.float().cpu().numpy(), r_out, "out")
    assert np.abs(lse.cpu().numpy() - r_lse).max() <= LSE_ATOL
