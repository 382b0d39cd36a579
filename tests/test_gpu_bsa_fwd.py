"""GPU parity of the tcgen05 tile machinery, the BSA metadata and the BSA forward pass against
the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import attention as A
from oracle import metadata as M
from parity import LSE_ATOL, check_close, dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu
_dev = dev_bf16
_close = check_close


def test_diag_mma_tile(cuda_ok):
    rng = np.random.default_rng(0)
    a = synth.f32_to_bf16_bits(rng.standard_normal((128, 128), dtype=np.float32))
    b = synth.f32_to_bf16_bits(rng.standard_normal((128, 128), dtype=np.float32))
    fa, fb = A.bf16_to_f64(a), A.bf16_to_f64(b)
    c, ws = sa.bsa_diag_mma_tile(_dev(a), _dev(b), False)
    torch.cuda.synchronize()
    assert sa.bsa_get_status(ws) == 0
    assert np.abs(c.cpu().numpy() - fa @ fb.T).max() < 1e-3
    c, ws = sa.bsa_diag_mma_tile(_dev(a), _dev(b), True)
    torch.cuda.synchronize()
    assert np.abs(c.cpu().numpy() - fa @ fb).max() < 1e-3
    # A staged in tensor memory, B K-major then MN-major
    c, ws = sa.bsa_diag_mma_tile(_dev(a), _dev(b), 2)
    torch.cuda.synchronize()
    assert np.abs(c.cpu().numpy() - fa @ fb.T).max() < 1e-3
    c, ws = sa.bsa_diag_mma_tile(_dev(a), _dev(b), 3)
    torch.cuda.synchronize()
    assert np.abs(c.cpu().numpy() - fa @ fb).max() < 1e-3
    # A MN-major (the buffer holds A^T), B K-major then MN-major
    c, ws = sa.bsa_diag_mma_tile(_dev(a), _dev(b), 4)
    torch.cuda.synchronize()
    assert np.abs(c.cpu().numpy() - fa.T @ fb.T).max() < 1e-3
    c, ws = sa.bsa_diag_mma_tile(_dev(a), _dev(b), 5)
    torch.cuda.synchronize()
    assert sa.bsa_get_status(ws) == 0
    assert np.abs(c.cpu().numpy() - fa.T @ fb).max() < 1e-3


def test_diag_exp2_polynomial(cuda_ok):
    """The FMA-pipe exponential the softmax loops use for part of their elements: relative error
    against the exact 2^x within the fit's bound (degree 3: 7.5e-5, degree 4: 2.7e-6, plus fp32
    rounding), on a dense sweep of [-126, 9] and on integers (n + f with f = 0)."""
    x = np.concatenate([np.linspace(-126.0, 9.0, 1 << 20), np.arange(-126, 9)]).astype(np.float32)
    ref = np.exp2(x.astype(np.float64))
    for degree, bound in ((3, 7.6e-5), (4, 2.8e-6)):
        y = sa.bsa_diag_exp2(torch.from_numpy(x).cuda(), degree).cpu().numpy().astype(np.float64)
        normal = x >= -125.5  # below that the result sits at the edge of the normal range
        rel = np.abs(y[normal] - ref[normal]) / ref[normal]
        assert rel.max() <= bound, (degree, rel.max())


@pytest.mark.parametrize("config", [1, 2, 5])
def test_bsa_metadata_bit_exact(cuda_ok, config):
    w = synth.workload(config)
    mask = w.block_mask()
    p = sa.bsa_params(torch.empty(w.B, w.N1, w.S, w.D, device="meta"),
                      torch.empty(w.B, w.N2, w.S, w.D, device="meta"),
                      torch.from_numpy(mask).cuda(), w.block, w.block)
    dmask = torch.from_numpy(mask).cuda()
    p.block_mask = dmask.data_ptr()
    for op, ref in ((sa.META_BSA_KV, M.bsa_kv_csr(mask)), (sa.META_BSA_Q, M.bsa_q_csr(mask, w.N2))):
        plan, lay = sa.sparse_attn_metadata(p, op, "cuda")
        torch.cuda.synchronize()
        rp = sa.plan_array(plan, lay, 1, len(ref[0])).cpu().numpy()
        col = sa.plan_array(plan, lay, 2, len(ref[1])).cpu().numpy()
        assert np.array_equal(rp, ref[0]) and np.array_equal(col, ref[1])
        assert sa.bsa_get_status(plan) == 0


def _run_case(B, N1, N2, S_q, S_kv, bx, by, mode, mask, seed, wl=0, wr=0):
    rng = np.random.default_rng(seed)
    D = 128
    q = synth.f32_to_bf16_bits(rng.standard_normal((B, N1, S_q, D), dtype=np.float32))
    k = synth.f32_to_bf16_bits(rng.standard_normal((B, N2, S_kv, D), dtype=np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal((B, N2, S_kv, D), dtype=np.float32))
    scale = 1 / np.sqrt(D)
    out, lse = sa.bsa_fwd(_dev(q), _dev(k), _dev(v), torch.from_numpy(mask).cuda(), bx, by, mode, scale, wl, wr)
    torch.cuda.synchronize()
    r_out, r_lse = A.bsa_forward(q, k, v, mask, bx, by, mode, scale, wl, wr)
    got_out = out.float().cpu().numpy()
    got_lse = lse.cpu().numpy()
    fin = np.isfinite(r_lse)
    _close(got_out, r_out, "out")
    assert np.all(np.isneginf(got_lse[~fin])) and np.all(got_out[~fin] == 0)
    assert np.abs(got_lse[fin] - r_lse[fin]).max() <= LSE_ATOL
    return out, lse


def test_bsa_fwd_tiny_workload(cuda_ok):
    """The tiny BSA workload (B=1, N=2, S=512, 64x64 blocks), full parity."""
    w = synth.workload(1)
    mask = w.block_mask()
    q, k, v = (_dev(w.tensor(t)) for t in ("q", "k", "v"))
    out, lse = sa.bsa_fwd(q, k, v, torch.from_numpy(mask).cuda(), 64, 64, 2, w.scale)
    torch.cuda.synchronize()
    r_out, r_lse = A.bsa_forward(w.tensor("q"), w.tensor("k"), w.tensor("v"), mask, 64, 64, 2, w.scale)
    _close(out.float().cpu().numpy(), r_out, "out")
    assert np.abs(lse.cpu().numpy() - r_lse).max() <= LSE_ATOL
    # run-to-run bit identical
    out2, lse2 = sa.bsa_fwd(q, k, v, torch.from_numpy(mask).cuda(), 64, 64, 2, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("case", [
    dict(B=1, N1=2, N2=2, S_q=384, S_kv=384, bx=128, by=128, mode=2),   # 3 blocks, causal
    dict(B=2, N1=4, N2=2, S_q=300, S_kv=300, bx=128, by=128, mode=2),   # ragged tail, GQA
    dict(B=1, N1=2, N2=1, S_q=200, S_kv=328, bx=64, by=64, mode=0),     # no mask, Sq != Skv
    dict(B=1, N1=2, N2=2, S_q=256, S_kv=384, bx=128, by=64, mode=3),    # right-down causal
    dict(B=1, N1=2, N2=2, S_q=512, S_kv=512, bx=64, by=128, mode=4, wl=127, wr=0),  # band
])
def test_bsa_fwd_cases(cuda_ok, case):
    case = dict(case)
    wl, wr = case.pop("wl", 0), case.pop("wr", 0)
    rng = np.random.default_rng(7)
    nqb = -(-case["S_q"] // case["bx"])
    nkb = -(-case["S_kv"] // case["by"])
    mask = (rng.random((case["B"], case["N1"], nqb, nkb)) < 0.6).astype(np.uint8)
    mask[..., 0, :] = 0  # first Q block selects nothing: empty rows -> Out = 0, LSE = -inf
    _run_case(**case, mask=mask, seed=3, wl=wl, wr=wr)


@pytest.mark.parametrize("case", [
    dict(B=2, N1=4, N2=4, S_q=300, S_kv=300, bx=128, by=128, mode=2),
    dict(B=1, N1=4, N2=1, S_q=328, S_kv=328, bx=64, by=64, mode=2),
])
def test_bsa_fwd_short_lists(cuda_ok, case):
    """Units with one or two KV tiles and no diagonal block: the epilogue must wait for the last
    O += P V even when softmax finishes long before it."""
    rng = np.random.default_rng(11)
    nqb = -(-case["S_q"] // case["bx"])
    nkb = -(-case["S_kv"] // case["by"])
    mask = (rng.random((case["B"], case["N1"], nqb, nkb)) < 0.6).astype(np.uint8)
    mask[..., 1, :] = 0
    mask[..., :, -1] = 0
    _run_case(**case, mask=mask, seed=4)


def test_bsa_fwd_full_size_sampled(cuda_ok):
    """BSA S=8192 workload at full size in one launch; two heads checked against the oracle."""
    w = synth.workload(2)
    mask = w.block_mask()
    q, k, v = (_dev(w.tensor(t)) for t in ("q", "k", "v"))
    out, lse = sa.bsa_fwd(q, k, v, torch.from_numpy(mask).cuda(), w.block, w.block, 2, w.scale)
    torch.cuda.synchronize()
    for (b, h) in [(0, 0), (1, 15)]:
        r_out, r_lse = A.bsa_slice_forward(
            A.bf16_to_f64(w.tensor("q", b, h))[None], A.bf16_to_f64(w.tensor("k", b, h)),
            A.bf16_to_f64(w.tensor("v", b, h)), mask[b, h][None], w.block, w.block, 2, w.scale)
        _close(out[b, h].float().cpu().numpy(), r_out[0], f"out[{b},{h}]")
        assert np.abs(lse[b, h].cpu().numpy() - r_lse[0]).max() <= LSE_ATOL

