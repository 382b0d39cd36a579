"""Metadata plans as op inputs (SparseAttnSharedkvMetadata page: the metadata operator's output
drives the attention operators).  A plan made once by sparse_attn_metadata and handed to the ops
must give the same lists (bit for bit against the CPU metadata reference) and outputs bit-identical
to the ops building their own lists, for the forward and backward of both block-sparse and NSA
attention; with a plan the no-allocation forward also runs problems whose lists exceed its array."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import metadata as M
from parity import dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu
D = 128


def _bsa_problem(B, N1, N2, S, blk, p_sel, seed):
    rng = np.random.default_rng(seed)
    bits = lambda *s: synth.f32_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))  # noqa: E731
    nb = -(-S // blk)
    mask = (rng.random((B, N1, nb, nb)) < p_sel).astype(np.uint8)
    mask[..., np.arange(nb), np.arange(nb)] = 1
    return (dev_bf16(bits(B, N1, S, D)), dev_bf16(bits(B, N2, S, D)), dev_bf16(bits(B, N2, S, D)),
            dev_bf16(bits(B, N1, S, D)), mask)


def _equal(a, b):
    return torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b)


def test_bsa_plan_lists_and_outputs(cuda_ok):
    B, N1, N2, S, blk = 2, 4, 2, 1000, 128
    q, k, v, do, mask = _bsa_problem(B, N1, N2, S, blk, 0.4, seed=71)
    dmask = torch.from_numpy(mask).cuda()
    p = sa.bsa_params(q, k, dmask, blk, blk)
    plan_b, lay_b = sa.sparse_attn_metadata(p, sa.META_BSA_BWD, "cuda")
    plan_k, _ = sa.sparse_attn_metadata(p, sa.META_BSA_KV, "cuda")
    torch.cuda.synchronize()
    kv_ref, q_ref = M.bsa_kv_csr(mask), M.bsa_q_csr(mask, N2)
    for i, ref in ((1, kv_ref[0]), (2, kv_ref[1]), (3, q_ref[0]), (4, q_ref[1])):
        got = sa.plan_array(plan_b, lay_b, i, len(ref)).cpu().numpy()
        assert np.array_equal(got, ref), f"array {i}"
    assert sa.bsa_get_status(plan_b) == 0
    out0, lse0 = sa.bsa_fwd(q, k, v, dmask, blk, blk)
    for plan in ((plan_k, sa.META_BSA_KV), (plan_b, sa.META_BSA_BWD)):
        out1, lse1 = sa.bsa_fwd(q, k, v, dmask, blk, blk, plan=plan)
        torch.cuda.synchronize()
        assert _equal(out0, out1) and _equal(lse0, lse1)
    g0 = sa.bsa_bwd(q, k, v, out0, do, lse0, dmask, blk, blk)
    g1 = sa.bsa_bwd(q, k, v, out0, do, lse0, dmask, blk, blk, plan=(plan_b, sa.META_BSA_BWD))
    torch.cuda.synchronize()
    assert all(_equal(a, b) for a, b in zip(g0, g1))
    with pytest.raises(sa.BsaError):  # the backward needs the transposed lists too
        sa.bsa_bwd(q, k, v, out0, do, lse0, dmask, blk, blk, plan=(plan_k, sa.META_BSA_KV))


def test_nsa_plan_outputs(cuda_ok):
    rng = np.random.default_rng(72)
    seqlens, N1, N2, bs, K = [700, 1300], 32, 2, 64, 8
    T = sum(seqlens)
    bits = lambda *s: synth.f32_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))  # noqa: E731
    q, k, v, do = (dev_bf16(bits(T, n, D)) for n in (N1, N2, N2, N1))
    rows = []
    for S in seqlens:
        for t in range(S):
            own = t // bs
            for _ in range(N2):
                pool = np.arange(own)
                ids = [own] + list(rng.choice(pool, size=min(K - 1, own), replace=False))
                rows.append(list(rng.permutation(ids)) + [-1] * (K - len(ids)))
    tk = torch.from_numpy(np.asarray(rows, np.int32).reshape(T, N2, K)).cuda()
    cu = torch.from_numpy(np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)).cuda()
    S = max(seqlens)
    p = sa.nsa_params(q, k, tk, cu, S, bs)
    plan, _ = sa.sparse_attn_metadata(p, sa.META_NSA_TOKENS, "cuda")
    out0, lse0 = sa.nsa_selected_fwd(q, k, v, tk, cu, S, bs)
    out1, lse1 = sa.nsa_selected_fwd(q, k, v, tk, cu, S, bs, plan=(plan, sa.META_NSA_TOKENS))
    torch.cuda.synchronize()
    assert _equal(out0, out1) and _equal(lse0, lse1)
    g0 = sa.nsa_selected_bwd(q, k, v, out0, do, lse0, tk, cu, S, bs)
    g1 = sa.nsa_selected_bwd(q, k, v, out0, do, lse0, tk, cu, S, bs, plan=(plan, sa.META_NSA_TOKENS))
    torch.cuda.synchronize()
    assert all(_equal(a, b) for a, b in zip(g0, g1))
    assert sa.bsa_get_status(plan) == 0


def test_noalloc_forward_with_plan_beyond_its_array(cuda_ok):
    """32 heads x 256 q blocks x 256 kv blocks: the forward's own lists need more than the
    no-allocation array's 8 MiB, so without a plan the call is refused before any launch; with a
    plan the array holds only the status header and the result equals bsa_fwd's bit for bit."""
    B, N1, N2, S, blk = 1, 32, 4, 32768, 128
    q, k, v, _, mask = _bsa_problem(B, N1, N2, S, blk, 0.05, seed=73)
    dmask = torch.from_numpy(mask).cuda()
    with pytest.raises(sa.BsaError) as e:
        sa.bsa_fwd_noalloc(q, k, v, dmask, blk, blk)
    assert e.value.code == sa.BSA_ERR_WORKSPACE_TOO_SMALL
    p = sa.bsa_params(q, k, dmask, blk, blk)
    plan, _ = sa.sparse_attn_metadata(p, sa.META_BSA_KV, "cuda")
    out1, lse1 = sa.bsa_fwd_noalloc(q, k, v, dmask, blk, blk, plan=(plan, sa.META_BSA_KV))
    out0, lse0 = sa.bsa_fwd(q, k, v, dmask, blk, blk)
    torch.cuda.synchronize()
    assert sa.bsa_fwd_noalloc_get_status() == 0
    assert _equal(out0, out1) and _equal(lse0, lse1)
