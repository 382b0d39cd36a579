"""GPU parity of block-sparse attention on the long workload (B=1, N=32, S=131072, D=128, 1024
KV blocks per head, 64 selected per q block: the diagonal, 4 previous, the first block and 58
uniform earlier ones), forward and backward at full size in one launch each.

The forward is checked on sampled q blocks of two heads.  For the backward, the oracle's forward
outputs (Out rounded to bf16, LSE) are written into every row that the sampled dQ, dK and dV
blocks depend on (the q blocks that selected a sampled KV block, and the sampled q blocks), then
the GPU backward runs at full size and the samples are compared with the oracle."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import attention as A
from parity import LSE_ATOL, check_close, dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def test_bsa_long_workload_sampled(cuda_ok):
    w = synth.workload(5)
    mask = w.block_mask()
    host = {t: w.tensor(t) for t in ("q", "k", "v", "dout")}
    q, k, v, do = (dev_bf16(host[t]) for t in ("q", "k", "v", "dout"))
    dmask = torch.from_numpy(mask).cuda()
    out, lse = sa.bsa_fwd(q, k, v, dmask, w.block, w.block, w.mask_mode, w.scale)
    torch.cuda.synchronize()
    f = A.bf16_to_f64
    samples = [(0, 3, [1023, 511, 7], [1000, 900]), (0, 29, [640], [1020])]
    refs = {}
    for b, h, qbs, kvbs in samples:
        qg, kg, vg = f(host["q"][b, h])[None], f(host["k"][b, h]), f(host["v"][b, h])
        r_out, r_lse = A.bsa_slice_forward(qg, kg, vg, mask[b, h][None], w.block, w.block, w.mask_mode, w.scale,
                                           q_blocks=qbs)
        for qb in qbs:
            sl = slice(qb * w.block, (qb + 1) * w.block)
            check_close(out[b, h, sl].float().cpu().numpy(), r_out[0, sl], f"out[{b},{h},{qb}]")
            assert np.abs(lse[b, h, sl].cpu().numpy() - r_lse[0, sl]).max() <= LSE_ATOL
        r = A.bsa_slice_backward(qg, kg, vg, f(host["dout"][b, h])[None], mask[b, h][None], w.block, w.block,
                                 w.mask_mode, w.scale, q_blocks=qbs, kv_blocks=kvbs, out_storage="bf16")
        refs[(b, h)] = r
        # the oracle's forward outputs for every row the samples depend on
        r_o, r_l = r[3][0], r[4][0]
        rows = np.nonzero(np.isfinite(r_l))[0]
        tr = torch.from_numpy(rows).long().cuda()
        out[b, h, tr] = dev_bf16(synth.f32_to_bf16_bits(np.asarray(r_o[rows], np.float32)))
        lse[b, h, tr] = torch.from_numpy(np.asarray(r_l[rows], np.float32)).cuda()
    gq, gk, gv = sa.bsa_bwd(q, k, v, out, do, lse, dmask, w.block, w.block, w.mask_mode, w.scale)
    torch.cuda.synchronize()
    for b, h, qbs, kvbs in samples:
        r_dq, r_dk, r_dv = refs[(b, h)][0][0], refs[(b, h)][1], refs[(b, h)][2]
        for qb in qbs:
            sl = slice(qb * w.block, (qb + 1) * w.block)
            check_close(gq[b, h, sl].float().cpu().numpy(), r_dq[sl], f"dq[{b},{h},{qb}]")
        for kb in kvbs:
            sl = slice(kb * w.block, (kb + 1) * w.block)
            check_close(gk[b, h, sl].float().cpu().numpy(), r_dk[sl], f"dk[{b},{h},{kb}]")
            check_close(gv[b, h, sl].float().cpu().numpy(), r_dv[sl], f"dv[{b},{h},{kb}]")
