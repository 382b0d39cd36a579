"""GPU parity of the BSA backward (dQ, dK, dV) against the fp64 oracle, plus determinism.

The backward operator takes the forward's Out and LSE as inputs (BlockSparseAttentionGrad page:
softmax_grad = softmaxGrad(dOut, attentionOut)).  Parity tests hand the GPU backward the
oracle's own forward outputs, Out stored as bf16 and LSE as fp32, so both sides differentiate
the same attentionOut; the forward is checked on its own elsewhere.  The chained GPU forward ->
GPU backward run is checked element by element against the oracle's backward given the GPU's Out
as attentionOut, and for determinism."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import attention as A
from parity import check_close, dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def _fwd_bwd(q, k, v, do, mask, bx, by, mode, scale, wl=0, wr=0):
    """GPU forward, then GPU backward on its outputs."""
    dq_, dk_, dv_, do_ = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(do)
    dmask = torch.from_numpy(mask).cuda()
    out, lse = sa.bsa_fwd(dq_, dk_, dv_, dmask, bx, by, mode, scale, wl, wr)
    gq, gk, gv = sa.bsa_bwd(dq_, dk_, dv_, out, do_, lse, dmask, bx, by, mode, scale, wl, wr)
    torch.cuda.synchronize()
    return out, lse, gq, gk, gv


def _bwd_from(q, k, v, do, r_out, r_lse, mask, bx, by, mode, scale, wl=0, wr=0):
    """GPU backward on the oracle's forward outputs (Out rounded to bf16, LSE to fp32)."""
    out = dev_bf16(synth.f32_to_bf16_bits(np.asarray(r_out, np.float32)))
    lse = torch.from_numpy(np.asarray(r_lse, np.float32)).cuda()
    gq, gk, gv = sa.bsa_bwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), out, dev_bf16(do), lse,
                            torch.from_numpy(mask).cuda(), bx, by, mode, scale, wl, wr)
    torch.cuda.synchronize()
    return gq, gk, gv


def test_bsa_bwd_tiny_workload(cuda_ok):
    w = synth.workload(1)
    mask = w.block_mask()
    q, k, v, do = (w.tensor(t) for t in ("q", "k", "v", "dout"))
    r_dq, r_dk, r_dv, r_out, r_lse = A.bsa_backward(q, k, v, do, mask, 64, 64, 2, w.scale)
    gq, gk, gv = _bwd_from(q, k, v, do, r_out, r_lse, mask, 64, 64, 2, w.scale)
    check_close(gq.float().cpu().numpy(), r_dq, "dq")
    check_close(gk.float().cpu().numpy(), r_dk, "dk")
    check_close(gv.float().cpu().numpy(), r_dv, "dv")
    # chained GPU forward -> GPU backward, element by element against the oracle's backward given
    # the GPU's Out as its attentionOut input (the backward operator's signature); and bit-identical
    # results across runs
    cout, _, cq, ck, cv = _fwd_bwd(q, k, v, do, mask, 64, 64, 2, w.scale)
    gpu_out = cout.view(torch.int16).cpu().numpy().view(np.uint16)
    c_dq, c_dk, c_dv, _, _ = A.bsa_backward(q, k, v, do, mask, 64, 64, 2, w.scale, out_in=gpu_out)
    check_close(cq.float().cpu().numpy(), c_dq, "chained dq")
    check_close(ck.float().cpu().numpy(), c_dk, "chained dk")
    check_close(cv.float().cpu().numpy(), c_dv, "chained dv")
    _, _, cq2, ck2, cv2 = _fwd_bwd(q, k, v, do, mask, 64, 64, 2, w.scale)
    assert torch.equal(cq, cq2) and torch.equal(ck, ck2) and torch.equal(cv, cv2)


@pytest.mark.parametrize("case", [
    dict(B=1, N1=2, N2=2, S=384, bx=128, by=128, mode=2),
    dict(B=2, N1=4, N2=2, S=300, bx=128, by=128, mode=2),           # ragged tail, GQA
    dict(B=1, N1=4, N2=1, S=328, bx=64, by=64, mode=0),             # GQA G=4, no mask
    dict(B=1, N1=2, N2=2, S=512, bx=64, by=128, mode=4, wl=127, wr=0),  # band
    dict(B=1, N1=2, N2=2, S=256, bx=128, by=64, mode=2),
])
def test_bsa_bwd_cases(cuda_ok, case):
    case = dict(case)
    wl, wr = case.pop("wl", 0), case.pop("wr", 0)
    B, N1, N2, S, bx, by, mode = (case[x] for x in ("B", "N1", "N2", "S", "bx", "by", "mode"))
    rng = np.random.default_rng(11)
    D = 128
    q = synth.f32_to_bf16_bits(rng.standard_normal((B, N1, S, D), dtype=np.float32))
    k = synth.f32_to_bf16_bits(rng.standard_normal((B, N2, S, D), dtype=np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal((B, N2, S, D), dtype=np.float32))
    do = synth.f32_to_bf16_bits(rng.standard_normal((B, N1, S, D), dtype=np.float32))
    nqb, nkb = -(-S // bx), -(-S // by)
    mask = (rng.random((B, N1, nqb, nkb)) < 0.6).astype(np.uint8)
    mask[..., 1, :] = 0    # an empty unit: zero dQ rows
    mask[..., :, -1] = 0   # a KV block nobody selects: zero dK/dV rows
    scale = 1 / np.sqrt(D)
    r_dq, r_dk, r_dv, r_out, r_lse = A.bsa_backward(q, k, v, do, mask, bx, by, mode, scale, wl, wr)
    gq, gk, gv = _bwd_from(q, k, v, do, r_out, r_lse, mask, bx, by, mode, scale, wl, wr)
    check_close(gq.float().cpu().numpy(), r_dq, "dq")
    check_close(gk.float().cpu().numpy(), r_dk, "dk")
    check_close(gv.float().cpu().numpy(), r_dv, "dv")


def test_bsa_bwd_full_size_sampled(cuda_ok):
    """BSA S=8192 workload, full-size launch; sampled Q blocks (dQ) and KV blocks (dK, dV)."""
    w = synth.workload(2)
    mask = w.block_mask()
    q, k, v, do = (w.tensor(t) for t in ("q", "k", "v", "dout"))
    r_out, r_lse = A.bsa_forward(q, k, v, mask, w.block, w.block, 2, w.scale)
    gq, gk, gv = _bwd_from(q, k, v, do, r_out, r_lse, mask, w.block, w.block, 2, w.scale)
    for (b, h) in [(0, 3), (1, 14)]:
        qb_s, kb_s = [0, 31, 63], [0, 1, 40, 63]
        r = A.bsa_slice_backward(A.bf16_to_f64(q[b, h])[None], A.bf16_to_f64(k[b, h]), A.bf16_to_f64(v[b, h]),
                                 A.bf16_to_f64(do[b, h])[None], mask[b, h][None], w.block, w.block, 2, w.scale,
                                 q_blocks=qb_s, kv_blocks=kb_s, out_storage="bf16")
        r_dq, r_dk, r_dv = r[0][0], r[1], r[2]
        for qb in qb_s:
            sl = slice(qb * 128, (qb + 1) * 128)
            check_close(gq[b, h, sl].float().cpu().numpy(), r_dq[sl], f"dq[{b},{h},{qb}]")
        for kb in kb_s:
            sl = slice(kb * 128, (kb + 1) * 128)
            check_close(gk[b, h, sl].float().cpu().numpy(), r_dk[sl], f"dk[{b},{h},{kb}]")
            check_close(gv[b, h, sl].float().cpu().numpy(), r_dv[sl], f"dv[{b},{h},{kb}]")
