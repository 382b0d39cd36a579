"""GPU parity of block-sparse attention in the BSND layout (q [B, S_q, N1, D], k/v [B, S_kv, N2, D],
LSE [B, S_q, N1]) and of the right-down causal mask (mode 3) with S_q != S_kv, forward and
backward, against the fp64 oracle (which is written for BNSD: the test transposes).  The
backward receives the oracle's forward outputs (Out stored as bf16) as its attentionOut, as in
the BNSD backward tests."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import attention as A
from parity import check_close, check_lse, dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu
D = 128


def _problem(B, N1, N2, Sq, Skv, bx, by, seed, p_sel=0.6):
    rng = np.random.default_rng(seed)
    bits = lambda *s: synth.f32_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))  # noqa: E731
    q, k, v, do = bits(B, N1, Sq, D), bits(B, N2, Skv, D), bits(B, N2, Skv, D), bits(B, N1, Sq, D)
    nqb, nkb = -(-Sq // bx), -(-Skv // by)
    mask = (rng.random((B, N1, nqb, nkb)) < p_sel).astype(np.uint8)
    mask[..., :, 0] = 1  # every q block sees the first kv block (most rows keep a key)
    return q, k, v, do, mask


def _bsnd(bits):  # BNSD bit array -> BSND device tensor
    return dev_bf16(np.ascontiguousarray(bits.transpose(0, 2, 1, 3)))


def _bnsd(t):  # BSND device tensor -> BNSD float64 array
    return t.float().cpu().numpy().transpose(0, 2, 1, 3)


CASES = [
    dict(B=2, N1=4, N2=2, Sq=300, Skv=300, bx=128, by=128, mode=2),                # ragged, GQA, causal
    dict(B=1, N1=2, N2=1, Sq=200, Skv=328, bx=64, by=64, mode=3),                  # right-down, Sq < Skv
    dict(B=1, N1=2, N2=2, Sq=256, Skv=192, bx=128, by=64, mode=3),                 # right-down, Sq > Skv
    dict(B=1, N1=2, N2=2, Sq=384, Skv=384, bx=128, by=128, mode=4, wl=127, wr=0),  # band
]


@pytest.mark.parametrize("case", CASES)
def test_bsa_bsnd_fwd_bwd(cuda_ok, case):
    case = dict(case)
    wl, wr = case.pop("wl", 0), case.pop("wr", 0)
    B, N1, N2, Sq, Skv, bx, by, mode = (case[x] for x in ("B", "N1", "N2", "Sq", "Skv", "bx", "by", "mode"))
    q, k, v, do, mask = _problem(B, N1, N2, Sq, Skv, bx, by, seed=41)
    scale = 1 / np.sqrt(D)
    r_dq, r_dk, r_dv, r_out, r_lse = A.bsa_backward(q, k, v, do, mask, bx, by, mode, scale, wl, wr)
    dmask = torch.from_numpy(mask).cuda()
    tq, tk, tv, tdo = _bsnd(q), _bsnd(k), _bsnd(v), _bsnd(do)
    out, lse = sa.bsa_fwd(tq, tk, tv, dmask, bx, by, mode, scale, wl, wr, layout=sa.LAYOUT_BSND)
    torch.cuda.synchronize()
    assert tuple(out.shape) == (B, Sq, N1, D) and tuple(lse.shape) == (B, Sq, N1)
    check_close(_bnsd(out), r_out, "out (BSND)")
    check_lse(lse.cpu().numpy().transpose(0, 2, 1), r_lse, "lse (BSND)")
    # backward on the oracle's forward outputs, in BSND
    o_in = dev_bf16(np.ascontiguousarray(synth.f32_to_bf16_bits(np.asarray(r_out, np.float32)).transpose(0, 2, 1, 3)))
    l_in = torch.from_numpy(np.ascontiguousarray(np.asarray(r_lse, np.float32).transpose(0, 2, 1))).cuda()
    gq, gk, gv = sa.bsa_bwd(tq, tk, tv, o_in, tdo, l_in, dmask, bx, by, mode, scale, wl, wr, layout=sa.LAYOUT_BSND)
    torch.cuda.synchronize()
    check_close(_bnsd(gq), r_dq, "dq (BSND)")
    check_close(_bnsd(gk), r_dk, "dk (BSND)")
    check_close(_bnsd(gv), r_dv, "dv (BSND)")


@pytest.mark.parametrize("case", CASES[1:3])
def test_bsa_right_down_causal_bwd_bnsd(cuda_ok, case):
    """Mode 3 (right-down causal) backward in BNSD with S_q != S_kv, including rows that see no
    key (S_q > S_kv: the first S_q - S_kv rows), whose gradients are zero."""
    case = dict(case)
    B, N1, N2, Sq, Skv, bx, by, mode = (case[x] for x in ("B", "N1", "N2", "Sq", "Skv", "bx", "by", "mode"))
    q, k, v, do, mask = _problem(B, N1, N2, Sq, Skv, bx, by, seed=43)
    scale = 1 / np.sqrt(D)
    r_dq, r_dk, r_dv, r_out, r_lse = A.bsa_backward(q, k, v, do, mask, bx, by, mode, scale)
    dmask = torch.from_numpy(mask).cuda()
    o_in = dev_bf16(synth.f32_to_bf16_bits(np.asarray(r_out, np.float32)))
    l_in = torch.from_numpy(np.asarray(r_lse, np.float32)).cuda()
    gq, gk, gv = sa.bsa_bwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), o_in, dev_bf16(do), l_in, dmask, bx, by, mode,
                            scale)
    torch.cuda.synchronize()
    check_close(gq.float().cpu().numpy(), r_dq, "dq")
    check_close(gk.float().cpu().numpy(), r_dk, "dk")
    check_close(gv.float().cpu().numpy(), r_dv, "dv")


@pytest.mark.parametrize("case", [
    dict(B=1, N1=2, N2=1, Sq=256, Skv=256, bx=128, by=128, mode=2, layout="bnsd"),   # aligned rows
    dict(B=2, N1=2, N2=2, Sq=200, Skv=236, bx=64, by=64, mode=3, layout="bnsd"),     # rows of 236 bytes
    dict(B=1, N1=4, N2=2, Sq=300, Skv=300, bx=128, by=128, mode=0, layout="bsnd"),
])
def test_bsa_dense_atten_mask(cuda_ok, case):
    """The dense atten_mask (uint8 [S_q, S_kv], nonzero = masked out, shared by batches and heads)
    inside the selected blocks, forward and backward, with a row the mask empties completely."""
    case = dict(case)
    lay = case.pop("layout")
    B, N1, N2, Sq, Skv, bx, by, mode = (case[x] for x in ("B", "N1", "N2", "Sq", "Skv", "bx", "by", "mode"))
    q, k, v, do, mask = _problem(B, N1, N2, Sq, Skv, bx, by, seed=47, p_sel=0.8)
    rng = np.random.default_rng(48)
    am = (rng.random((Sq, Skv)) < 0.3).astype(np.uint8)
    am[7] = 1
    scale = 1 / np.sqrt(D)
    r_dq, r_dk, r_dv, r_out, r_lse = A.bsa_backward(q, k, v, do, mask, bx, by, mode, scale, atten_mask=am)
    dmask, dam = torch.from_numpy(mask).cuda(), torch.from_numpy(am).cuda()
    layout = sa.LAYOUT_BSND if lay == "bsnd" else sa.LAYOUT_BNSD
    dev = _bsnd if lay == "bsnd" else dev_bf16
    back = _bnsd if lay == "bsnd" else (lambda t: t.float().cpu().numpy())
    tq, tk, tv, tdo = dev(q), dev(k), dev(v), dev(do)
    out, lse = sa.bsa_fwd(tq, tk, tv, dmask, bx, by, mode, scale, layout=layout, atten_mask=dam)
    torch.cuda.synchronize()
    lse_np = lse.cpu().numpy()
    if lay == "bsnd":
        lse_np = lse_np.transpose(0, 2, 1)
    check_close(back(out), r_out, "out (atten_mask)")
    check_lse(lse_np, r_lse, "lse (atten_mask)")
    assert np.all(np.isneginf(lse_np[:, :, 7]))
    o_bits = synth.f32_to_bf16_bits(np.asarray(r_out, np.float32))
    l_f = np.asarray(r_lse, np.float32)
    if lay == "bsnd":
        o_in, l_in = _bsnd(o_bits), torch.from_numpy(np.ascontiguousarray(l_f.transpose(0, 2, 1))).cuda()
    else:
        o_in, l_in = dev_bf16(o_bits), torch.from_numpy(l_f).cuda()
    gq, gk, gv = sa.bsa_bwd(tq, tk, tv, o_in, tdo, l_in, dmask, bx, by, mode, scale, layout=layout, atten_mask=dam)
    torch.cuda.synchronize()
    check_close(back(gq), r_dq, "dq (atten_mask)")
    check_close(back(gk), r_dk, "dk (atten_mask)")
    check_close(back(gv), r_dv, "dv (atten_mask)")
