"""Run-to-run bitwise determinism of every output at full size, on the four large workloads:
block-sparse S=8192 and S=131072 (forward + backward), NSA selected attention (forward +
backward) and the paged sparse decode.  Each op runs twice on the same inputs into fresh
outputs; Out, LSE, dQ, dK and dV must be bit-identical (dK/dV are accumulated in a fixed order,
with no atomics)."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from parity import dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def _same(a, b, what):
    assert torch.equal(a, b), f"{what}: runs differ in {int((a != b).sum())} elements"


@pytest.mark.parametrize("config", [2, 5])
def test_bsa_fwd_bwd_bitwise_deterministic(cuda_ok, config):
    w = synth.workload(config)
    mask = torch.from_numpy(w.block_mask()).cuda()
    q, k, v, do = (dev_bf16(w.tensor(t)) for t in ("q", "k", "v", "dout"))
    runs = []
    for _ in range(2):
        out, lse = sa.bsa_fwd(q, k, v, mask, w.block, w.block, w.mask_mode, w.scale)
        gq, gk, gv = sa.bsa_bwd(q, k, v, out, do, lse, mask, w.block, w.block, w.mask_mode, w.scale)
        torch.cuda.synchronize()
        runs.append((out, lse, gq, gk, gv))
    for name, a, b in zip(("out", "lse", "dq", "dk", "dv"), *runs):
        _same(a, b, f"workload {config} {name}")
    assert torch.isfinite(runs[0][2]).all() and torch.isfinite(runs[0][3]).all()


def test_nsa_fwd_bwd_bitwise_deterministic(cuda_ok):
    w = synth.workload(3)
    q, k, v, do = (dev_bf16(w.tensor(t)) for t in ("q", "k", "v", "dout"))
    tk, cu = torch.from_numpy(w.topk()).cuda(), torch.from_numpy(w.cu_seqlens()).cuda()
    S = max(w.seqlens)
    runs = []
    for _ in range(2):
        out, lse = sa.nsa_selected_fwd(q, k, v, tk, cu, S, w.sel_block, w.mask_mode, w.scale)
        gq, gk, gv = sa.nsa_selected_bwd(q, k, v, out, do, lse, tk, cu, S, w.sel_block, w.mask_mode, w.scale)
        torch.cuda.synchronize()
        runs.append((out, lse, gq, gk, gv))
    for name, a, b in zip(("out", "lse", "dq", "dk", "dv"), *runs):
        _same(a, b, f"NSA workload {name}")


def test_sfa_decode_bitwise_deterministic(cuda_ok):
    w = synth.workload(4)
    table, idx = w.selection()
    seqused = np.full(w.B, w.context, np.int32)
    used = np.unique(table[np.arange(w.B)[:, None], idx[:, 0, 0, :]].ravel())
    caches = {}
    for tag, d in (("k", 512), ("k_rope", 64), ("v", 512)):
        t = torch.zeros((w.n_pages, w.page, 1, d), dtype=torch.bfloat16, device="cuda")
        t[torch.from_numpy(used).long().cuda()] = dev_bf16(w.pages(tag, used))
        caches[tag] = t
    q, qr = dev_bf16(w.query("q")), dev_bf16(w.query("q_rope"))
    tb, ti, tu = (torch.from_numpy(x).cuda() for x in (table, idx, seqused))
    runs = []
    for _ in range(2):
        out, lse = sa.sfa_sparse_decode(q, qr, caches["k"], caches["k_rope"], caches["v"], tb, ti, tu,
                                        w.sparse_block, w.scale)
        torch.cuda.synchronize()
        runs.append((out, lse))
    _same(runs[0][0], runs[1][0], "decode out")
    _same(runs[0][1], runs[1][1], "decode lse")
