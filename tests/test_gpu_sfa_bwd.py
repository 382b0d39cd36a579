"""GPU parity of the sparse-decode backward (the BlockSparseAttentionGrad formulas on the gathered
keys of a SparseFlashAttention step) against the fp64 oracle, through the C ABI.

As for the other backward tests, the GPU backward receives the oracle's forward outputs (Out stored
as bf16, LSE as fp32), so both sides differentiate the same attentionOut.  The cache gradients are
compared whole: rows the step read must hold their summed gradient, every other row must be left
as it was (zero here)."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import attention as A
from parity import check_close, dev_bf16
from test_gpu_sfa import _problem
from workloads import synth

pytestmark = pytest.mark.gpu


def _bwd(pb, scale=None, nan_tails=False):
    scale = 1 / np.sqrt(576) if scale is None else scale
    rng = np.random.default_rng(99)
    B, N1 = pb["q"].shape[0], pb["q"].shape[2]
    do = synth.f32_to_bf16_bits(rng.standard_normal((B, 1, N1, 512), dtype=np.float32))
    r = A.sfa_backward(pb["q"], pb["qr"], pb["kc"], pb["krc"], pb["vc"], do, pb["table"], pb["idx"], pb["seqused"],
                       pb["page"], pb["sbs"], scale)
    r_dq, r_dqr, r_dk, r_dkr, r_dv, r_out, r_lse = r
    dev = pb["dev"]
    if nan_tails:  # rows past seqused inside the last page of each sequence hold NaN
        for b in range(B):
            used = int(pb["seqused"][b])
            if used % pb["page"]:
                lp = used // pb["page"]
                if lp < pb["table"].shape[1]:
                    phys = int(pb["table"][b, lp])
                    for t in (dev["k"], dev["kr"], dev["v"]):
                        t[phys, used % pb["page"]:] = float("nan")
    o_in = dev_bf16(synth.f32_to_bf16_bits(np.nan_to_num(np.asarray(r_out, np.float32))))
    l_in = torch.from_numpy(np.asarray(r_lse, np.float32)).cuda()
    g = sa.sfa_sparse_decode_bwd(dev_bf16(pb["q"]), dev_bf16(pb["qr"]), dev["k"], dev["kr"], dev["v"], o_in,
                                 dev_bf16(do), l_in, torch.from_numpy(pb["table"]).cuda(),
                                 torch.from_numpy(pb["idx"]).cuda(), torch.from_numpy(pb["seqused"]).cuda(),
                                 pb["sbs"], scale)
    torch.cuda.synchronize()
    return [x.float().cpu().numpy() for x in g], (r_dq, r_dqr, r_dk, r_dkr, r_dv)


CASES = [
    dict(B=3, N1=128, N2=1, page=64, n_logical=16, K=6, sbs=64, seqused=[1024, 1000, 700]),  # partial pages
    dict(B=2, N1=64, N2=1, page=64, n_logical=20, K=9, sbs=128, seqused=[1280, 1250]),       # G = 64, 2 pages/block
    dict(B=2, N1=128, N2=2, page=32, n_logical=24, K=5, sbs=64, seqused=[768, 600]),         # two kv heads, 32-token pages
    dict(B=3, N1=128, N2=1, page=64, n_logical=8, K=4, sbs=64, seqused=[512, 0, 130]),       # an empty batch
    dict(B=2, N1=128, N2=1, page=64, n_logical=16, K=7, sbs=64, seqused=[1024, 900], dup=True),  # a block read twice
]


@pytest.mark.parametrize("case", CASES)
def test_sfa_bwd_cases(cuda_ok, case):
    pb = _problem(**case, seed=23)
    got, ref = _bwd(pb)
    for x, y, name in zip(got, ref, ("dq", "dq_rope", "dk_cache", "dk_rope_cache", "dv_cache")):
        check_close(x, y, name)


def test_sfa_bwd_shared_pages_and_nan_tails(cuda_ok):
    """Two batches whose block tables share pages (the same cache rows read by both: their
    gradients add), and NaN in the cache rows past each sequence's end."""
    pb = _problem(B=2, N1=128, N2=1, page=64, n_logical=12, K=8, sbs=64, seqused=[768, 700], seed=29)
    pb["table"][1, :6] = pb["table"][0, :6]  # batch 1's first six logical pages are batch 0's
    pb["idx"][1, 0, 0, :4] = [0, 1, 2, 3]
    pb["idx"][0, 0, 0, :4] = [3, 2, 1, 0]
    used = sorted({int(pb["table"][b, j]) for b in range(2) for j in pb["idx"][b, 0, 0] if j >= 0})
    for name, arr in (("k", pb["kc"]), ("kr", pb["krc"]), ("v", pb["vc"])):
        pb["dev"][name][used] = dev_bf16(arr[used])
    got, ref = _bwd(pb, nan_tails=True)
    for x, y, name in zip(got, ref, ("dq", "dq_rope", "dk_cache", "dk_rope_cache", "dv_cache")):
        assert np.all(np.isfinite(x)), name
        check_close(x, y, name)


def test_sfa_bwd_deterministic(cuda_ok):
    pb = _problem(B=2, N1=128, N2=1, page=64, n_logical=16, K=7, sbs=64, seqused=[1024, 900], seed=31, dup=True)
    a, _ = _bwd(pb)
    b, _ = _bwd(pb)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
