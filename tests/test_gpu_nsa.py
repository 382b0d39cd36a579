"""GPU parity of NSA selected attention (NsaSelectedAttention page: per-token topk_indices,
TND varlen, GQA) and of its metadata, against the fp64 oracle, through the C ABI.

As for BSA, the backward parity tests hand the GPU backward the oracle's own forward outputs
(Out stored as bf16, LSE as fp32), so both sides differentiate the same attentionOut."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import attention as A
from oracle import metadata as M
from parity import check_close, check_lse, dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu

D = 128


def _topk(rng, seqlens, N2, bs, K, causal, dup=False, past=False):
    """Own block plus distinct random others (earlier ones under the causal mask), random order,
    -1 padding; optionally a duplicated id and an id past the batch's blocks."""
    rows = []
    for S in seqlens:
        nb = -(-S // bs)
        for t in range(S):
            own = t // bs
            for _ in range(N2):
                pool = np.arange(own) if causal else np.setdiff1d(np.arange(nb), [own])
                n = min(K - 1, len(pool))
                ids = [own] + list(rng.choice(pool, size=n, replace=False)) if n else [own]
                if dup and len(ids) < K and rng.random() < 0.5:
                    ids.append(ids[int(rng.integers(len(ids)))])
                if past and len(ids) < K and rng.random() < 0.02:
                    ids.append(nb + int(rng.integers(3)))
                ids = list(rng.permutation(ids)) + [-1] * (K - len(ids))
                rows.append(ids)
    T = sum(seqlens)
    return np.asarray(rows, np.int32).reshape(T, N2, K)


def _problem(seqlens, N1, N2, bs, K, mode, seed, dup=False, past=False, dqk=D):
    """dqk: head dim of q and k (v, Out and dOut keep D = 128)."""
    rng = np.random.default_rng(seed)
    T = sum(seqlens)
    bits = lambda *s: synth.f32_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))  # noqa: E731
    q, k, v, do = bits(T, N1, dqk), bits(T, N2, dqk), bits(T, N2, D), bits(T, N1, D)
    topk = _topk(rng, seqlens, N2, bs, K, causal=(mode == 2), dup=dup, past=past)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    return dict(q=q, k=k, v=v, do=do, topk=topk, cu=cu, S=max(seqlens), bs=bs, mode=mode,
                scale=1 / np.sqrt(dqk))


def _dev(pb):
    return (dev_bf16(pb["q"]), dev_bf16(pb["k"]), dev_bf16(pb["v"]), torch.from_numpy(pb["topk"]).cuda(),
            torch.from_numpy(pb["cu"]).cuda())


def _fwd(pb):
    q, k, v, tk, cu = _dev(pb)
    out, lse = sa.nsa_selected_fwd(q, k, v, tk, cu, pb["S"], pb["bs"], pb["mode"], pb["scale"])
    torch.cuda.synchronize()
    return out, lse


def _bwd(pb, out, lse):
    q, k, v, tk, cu = _dev(pb)
    gq, gk, gv = sa.nsa_selected_bwd(q, k, v, out, dev_bf16(pb["do"]), lse, tk, cu, pb["S"], pb["bs"], pb["mode"],
                                     pb["scale"])
    torch.cuda.synchronize()
    return gq, gk, gv


def _as_dev_out(r_out, r_lse):
    return (dev_bf16(synth.f32_to_bf16_bits(np.asarray(r_out, np.float32))),
            torch.from_numpy(np.asarray(r_lse, np.float32)).cuda())


CASES = [
    dict(seqlens=[200, 77], N1=16, N2=1, bs=64, K=4, mode=2),            # G = 16, ragged tails
    dict(seqlens=[130, 256, 33], N1=16, N2=2, bs=32, K=6, mode=0),       # G = 8, no mask
    dict(seqlens=[96, 160], N1=64, N2=2, bs=16, K=8, mode=2),            # G = 32: two head tiles
    dict(seqlens=[150], N1=12, N2=3, bs=48, K=3, mode=0, dup=True),      # G = 4, duplicated ids
    dict(seqlens=[64, 300, 1], N1=8, N2=1, bs=128, K=2, mode=2, dup=True),  # 128-token blocks, 1-token batch
    # 64-token blocks with G in {8, 16, 32, 64, 128}: the tensor-core dK/dV pass
    dict(seqlens=[300, 129], N1=32, N2=4, bs=64, K=5, mode=0, dup=True),     # G = 8, duplicated ids
    dict(seqlens=[200, 64], N1=16, N2=1, bs=64, K=4, mode=2, dup=True),      # G = 16, duplicated ids
    dict(seqlens=[200], N1=64, N2=2, bs=64, K=3, mode=2),                    # G = 32
    dict(seqlens=[130, 70], N1=64, N2=1, bs=64, K=3, mode=0),                # G = 64
    dict(seqlens=[130, 70], N1=128, N2=1, bs=64, K=3, mode=2),               # G = 128
    # 192-dim q / k with 128-dim v (NsaSelectedAttention constraints: a head-dim pair)
    dict(seqlens=[200, 77], N1=16, N2=1, bs=64, K=4, mode=2, dqk=192),       # G = 16
    dict(seqlens=[130, 256, 33], N1=16, N2=2, bs=32, K=6, mode=0, dup=True, dqk=192),  # G = 8, 32-token blocks
]


def test_nsa_metadata_bit_exact(cuda_ok):
    seqlens = [100, 257, 0, 64, 31]
    pb = _problem(seqlens, N1=4, N2=2, bs=32, K=6, mode=0, seed=5, dup=True, past=True)
    q, k, _, tk, cu = _dev(pb)
    p = sa.nsa_params(q, k, tk, cu, pb["S"], pb["bs"], 0)
    plan, lay = sa.sparse_attn_metadata(p, sa.META_NSA_TOKENS, "cuda")
    torch.cuda.synchronize()
    T, N2, K = pb["topk"].shape
    nblk_max = -(-pb["S"] // pb["bs"])
    ids = sa.plan_array(plan, lay, 1, T * N2 * K).cpu().numpy().reshape(T, N2, K)
    cnt = sa.plan_array(plan, lay, 2, T * N2).cpu().numpy().reshape(T, N2)
    rows = len(seqlens) * N2 * nblk_max
    rp = sa.plan_array(plan, lay, 3, rows + 1).cpu().numpy()
    r_ids, r_cnt, r_status = M.nsa_kv_lists(pb["topk"], pb["cu"], pb["bs"])
    r_rp, r_col = M.nsa_token_csr(r_ids, r_cnt, pb["cu"], pb["bs"], nblk_max)
    col = sa.plan_array(plan, lay, 4, int(r_rp[-1])).cpu().numpy()
    assert np.array_equal(ids, r_ids) and np.array_equal(cnt, r_cnt)
    assert np.array_equal(rp, r_rp) and np.array_equal(col, r_col)
    assert r_status == M.BAD_INDEX and sa.bsa_get_status(plan) & sa.DEV_BAD_INDEX


@pytest.mark.parametrize("case", CASES)
def test_nsa_fwd_cases(cuda_ok, case):
    case = dict(case)
    pb = _problem(**case, seed=17)
    out, lse = _fwd(pb)
    r_out, r_lse = A.nsa_forward(pb["q"], pb["k"], pb["v"], pb["topk"], pb["cu"], pb["bs"], pb["mode"], pb["scale"])
    check_close(out.float().cpu().numpy(), r_out, "out")
    check_lse(lse.cpu().numpy(), r_lse)


@pytest.mark.parametrize("case", CASES)
def test_nsa_bwd_cases(cuda_ok, case):
    case = dict(case)
    pb = _problem(**case, seed=23)
    r_dq, r_dk, r_dv, r_out, r_lse = A.nsa_backward(pb["q"], pb["k"], pb["v"], pb["do"], pb["topk"], pb["cu"],
                                                    pb["bs"], pb["mode"], pb["scale"])
    gq, gk, gv = _bwd(pb, *_as_dev_out(r_out, r_lse))
    check_close(gq.float().cpu().numpy(), r_dq, "dq")
    check_close(gk.float().cpu().numpy(), r_dk, "dk")
    check_close(gv.float().cpu().numpy(), r_dv, "dv")


def test_nsa_chained_determinism_and_invariants(cuda_ok):
    """GPU forward -> GPU backward, twice: bit-identical, and element by element against the
    oracle's backward on the GPU's Out; per (token, head) the softmax Jacobian
    gives sum over keys of dS = 0, so sum_t dK[t, g] = 0 per kv head, and sum_t dV[t, g] equals
    the sum of dOut over the group's heads and the tokens that see at least one key.  The sums run
    over bf16-stored rows, each within 2^-8 relative of its fp32 value, which sets the bound."""
    pb = _problem(seqlens=[200, 333], N1=16, N2=2, bs=64, K=5, mode=2, seed=29)
    runs = []
    for _ in range(2):
        out, lse = _fwd(pb)
        runs.append((out, lse) + _bwd(pb, out, lse))
    for a, b in zip(runs[0], runs[1]):
        assert torch.equal(a, b)
    # element by element against the oracle's backward given the GPU's Out as attentionOut
    gpu_out = runs[0][0].view(torch.int16).cpu().numpy().view(np.uint16)
    c_dq, c_dk, c_dv, _, _ = A.nsa_backward(pb["q"], pb["k"], pb["v"], pb["do"], pb["topk"], pb["cu"], pb["bs"],
                                            pb["mode"], pb["scale"], out_in=gpu_out)
    check_close(runs[0][2].float().cpu().numpy(), c_dq, "chained dq")
    check_close(runs[0][3].float().cpu().numpy(), c_dk, "chained dk")
    check_close(runs[0][4].float().cpu().numpy(), c_dv, "chained dv")
    _, _, _, gk, gv = runs[0]
    G = 8
    do = A.bf16_to_f64(pb["do"]).reshape(-1, 2, G, D).sum(axis=2)        # [T, N2, D]
    gkf, gvf = gk.float().cpu().numpy().astype(np.float64), gv.float().cpu().numpy().astype(np.float64)
    tol_v = 2.0 ** -8 * np.abs(gvf).sum(axis=0) + 1e-2
    tol_k = 2.0 ** -8 * np.abs(gkf).sum(axis=0) + 1e-2
    assert np.all(np.abs(gvf.sum(axis=0) - do.sum(axis=0)) <= tol_v)
    assert np.all(np.abs(gkf.sum(axis=0)) <= tol_k)


def test_nsa_host_errors(cuda_ok):
    pb = _problem(seqlens=[64], N1=4, N2=2, bs=32, K=2, mode=2, seed=1)
    q, k, v, tk, cu = _dev(pb)
    with pytest.raises(sa.BsaError):
        sa.nsa_selected_fwd(q, k, v, tk, cu, 64, 24, 2)       # block size not a multiple of 16
    with pytest.raises(sa.BsaError):
        sa.nsa_selected_fwd(q, k, v, tk, cu, 64, 32, 3)       # mask mode outside {0, 2}
    bad_cu = torch.tensor([0, 65], dtype=torch.int32, device="cuda")  # does not end at T
    p = sa.nsa_params(q, k, tk, bad_cu, 64, 32, 2)
    plan, _ = sa.sparse_attn_metadata(p, sa.META_NSA_KV, "cuda")
    assert sa.bsa_get_status(plan) & sa.DEV_BAD_SEQLEN
    long_cu = torch.tensor([0, 64], dtype=torch.int32, device="cuda")  # batch longer than max_seqlen
    p = sa.nsa_params(q, k, tk, long_cu, 48, 32, 2)
    plan, _ = sa.sparse_attn_metadata(p, sa.META_NSA_KV, "cuda")
    assert sa.bsa_get_status(plan) & sa.DEV_BAD_SEQLEN


def test_nsa_workload_full_size_sampled(cuda_ok):
    """TND GQA workload (4 batches of 4096..32768 tokens, 64 query heads over 4 kv heads, 16
    blocks of 64 selected): full-size launches, checked on sampled tokens and key blocks.

    The forward is checked on sampled tokens.  For the backward, the oracle's forward outputs
    are written into Out/LSE for every token that the sampled checks depend on (the tokens
    listing a sampled block, and the sampled dQ tokens), then the GPU backward runs at full
    size and dQ / dK / dV of the samples are compared with the oracle."""
    w = synth.workload(3)
    topk = w.topk()
    cu = w.cu_seqlens()
    q, k, v, do = (w.tensor(t) for t in ("q", "k", "v", "dout"))
    dq_, dk_, dv_ = dev_bf16(q), dev_bf16(k), dev_bf16(v)
    dtk, dcu = torch.from_numpy(topk).cuda(), torch.from_numpy(cu).cuda()
    S = max(w.seqlens)
    out, lse = sa.nsa_selected_fwd(dq_, dk_, dv_, dtk, dcu, S, w.sel_block, w.mask_mode, w.scale)
    torch.cuda.synchronize()
    assert np.isfinite(out[::97].float().cpu().numpy()).all()
    G = w.N1 // w.N2
    ids, cnt, _ = M.nsa_kv_lists(topk, cu, w.sel_block)
    samples = [(1, 2, [0, 37, 127], [5, 4100]), (3, 1, [511, 200], [0, 32767, 20000])]
    refs = {}
    for b, g, blocks, dq_pos in samples:
        t0, t1 = int(cu[b]), int(cu[b + 1])
        lists = [t - t0 for t in range(t0, t1) if any(x in blocks for x in ids[t, g, :cnt[t, g]])]
        toks = sorted(set(lists) | set(dq_pos))
        hs = slice(g * G, (g + 1) * G)
        f = A.bf16_to_f64
        r = A.nsa_slice(f(q[t0:t1, hs]), f(k[t0:t1, g]), f(v[t0:t1, g]), topk[t0:t1, g], w.sel_block, w.mask_mode,
                        w.scale, dout_g=f(do[t0:t1, hs]), tokens=toks, out_storage="bf16")
        refs[(b, g)] = r
        r_out, r_lse = r[0], r[1]
        for tp in dq_pos:                      # forward on the sampled tokens
            check_close(out[t0 + tp, hs].float().cpu().numpy(), r_out[tp], f"out[{b},{g},{tp}]")
            check_lse(lse[t0 + tp, hs].cpu().numpy(), r_lse[tp], f"lse[{b},{g},{tp}]")
        # the oracle's outputs for every token the samples depend on
        tt = torch.tensor([t0 + x for x in toks], dtype=torch.long, device="cuda")
        o_dev, l_dev = _as_dev_out(r_out[toks], r_lse[toks])
        out[tt, hs] = o_dev
        lse[tt, hs] = l_dev
    gq, gk, gv = sa.nsa_selected_bwd(dq_, dk_, dv_, out, dev_bf16(do), lse, dtk, dcu, S, w.sel_block, w.mask_mode,
                                     w.scale)
    torch.cuda.synchronize()
    for b, g, blocks, dq_pos in samples:
        t0 = int(cu[b])
        hs = slice(g * G, (g + 1) * G)
        _, _, r_dq, r_dk, r_dv = refs[(b, g)]
        for tp in dq_pos:
            check_close(gq[t0 + tp, hs].float().cpu().numpy(), r_dq[tp], f"dq[{b},{g},{tp}]")
        for kb in blocks:
            sl = slice(kb * w.sel_block, (kb + 1) * w.sel_block)
            check_close(gk[t0 + sl.start:t0 + sl.stop, g].float().cpu().numpy(), r_dk[sl], f"dk[{b},{g},{kb}]")
            check_close(gv[t0 + sl.start:t0 + sl.stop, g].float().cpu().numpy(), r_dv[sl], f"dv[{b},{g},{kb}]")

