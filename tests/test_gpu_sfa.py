"""GPU parity of sparse decode over a paged KV cache (SparseFlashAttention) and of its page-list
metadata, against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import attention as A
from oracle import metadata as M
from parity import LSE_ATOL, check_close, dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def _problem(B, N1, N2, page, n_logical, K, sbs, seqused, seed, fill_nan=True, dup=False):
    """Random paged problem; unselected pages are NaN so a wrong gather shows up.  dup: the last
    slot of every row repeats the first (a duplicated id is gathered twice)."""
    rng = np.random.default_rng(seed)
    n_pages = B * n_logical + 5
    table = rng.permutation(n_pages)[:B * n_logical].reshape(B, n_logical).astype(np.int32)
    ppb = sbs // page
    idx = np.full((B, 1, N2, K), -1, np.int32)
    for b in range(B):
        nsb = -(-int(seqused[b]) // sbs)
        for g in range(N2):
            idx[b, 0, g] = rng.choice(max(nsb, K), size=K, replace=False)
            idx[b, 0, g][idx[b, 0, g] >= nsb] = -1
    if dup:
        idx[:, 0, :, -1] = idx[:, 0, :, 0]
    bits = lambda *s: synth.f32_to_bf16_bits(rng.standard_normal(s, dtype=np.float32))  # noqa: E731
    q, qr = bits(B, 1, N1, 512), bits(B, 1, N1, 64)
    kc, krc, vc = bits(n_pages, page, N2, 512), bits(n_pages, page, N2, 64), bits(n_pages, page, N2, 512)
    used_pages = sorted({int(table[b, j * ppb + p]) for b in range(B) for g in range(N2) for j in idx[b, 0, g]
                         if j >= 0 for p in range(ppb) if (j * ppb + p) < n_logical})
    dev = {}
    for name, arr in (("k", kc), ("kr", krc), ("v", vc)):
        t = torch.full(arr.shape, float("nan"), dtype=torch.bfloat16, device="cuda") if fill_nan \
            else dev_bf16(arr)
        if fill_nan:
            t[used_pages] = dev_bf16(arr[used_pages])
        dev[name] = t
    return dict(q=q, qr=qr, kc=kc, krc=krc, vc=vc, table=table, idx=idx, seqused=np.asarray(seqused, np.int32),
                page=page, sbs=sbs, dev=dev)


def _run(pb, scale=None):
    scale = 1 / np.sqrt(576) if scale is None else scale
    out, lse = sa.sfa_sparse_decode(dev_bf16(pb["q"]), dev_bf16(pb["qr"]), pb["dev"]["k"], pb["dev"]["kr"],
                                    pb["dev"]["v"], torch.from_numpy(pb["table"]).cuda(),
                                    torch.from_numpy(pb["idx"]).cuda(), torch.from_numpy(pb["seqused"]).cuda(),
                                    pb["sbs"], scale)
    torch.cuda.synchronize()
    r_out, r_lse = A.sfa_decode(pb["q"], pb["qr"], pb["kc"], pb["krc"], pb["vc"], pb["table"], pb["idx"],
                                pb["seqused"], pb["page"], pb["sbs"], scale)
    return out, lse, r_out, r_lse


@pytest.mark.parametrize("case", [
    dict(B=3, N1=128, N2=1, page=64, n_logical=16, K=6, sbs=64, seqused=[1024, 1000, 700]),
    dict(B=2, N1=64, N2=1, page=64, n_logical=20, K=9, sbs=128, seqused=[1280, 1250]),   # G = 64, 2 pages/block
    dict(B=2, N1=128, N2=2, page=32, n_logical=24, K=5, sbs=64, seqused=[768, 600]),     # two kv heads, 32-token pages
    dict(B=1, N1=128, N2=1, page=64, n_logical=8, K=8, sbs=64, seqused=[512]),           # every block selected
    dict(B=3, N1=128, N2=1, page=64, n_logical=8, K=4, sbs=64, seqused=[512, 0, 130]),   # an empty batch
])
def test_sfa_decode_cases(cuda_ok, case):
    pb = _problem(**case, seed=21)
    out, lse, r_out, r_lse = _run(pb)
    check_close(out.float().cpu().numpy(), r_out, "out")
    fin = np.isfinite(r_lse)
    got = lse.cpu().numpy()
    assert np.all(np.isneginf(got[~fin]))
    assert np.abs(got[fin] - r_lse[fin]).max() <= LSE_ATOL


def test_sfa_page_lists_bit_exact(cuda_ok):
    pb = _problem(B=3, N1=128, N2=2, page=32, n_logical=24, K=5, sbs=64, seqused=[768, 600, 97], seed=3,
                  fill_nan=False)
    idx = pb["idx"].copy()
    idx[2, 0, 1, 0] = 40  # past the sequence: dropped, flagged
    p = sa.sfa_params(torch.empty(3, 1, 128, 512, device="meta"), pb["dev"]["k"],
                      torch.from_numpy(pb["table"]).cuda(), torch.from_numpy(idx).cuda(),
                      torch.from_numpy(pb["seqused"]).cuda(), pb["sbs"])
    tb, ti, tu = torch.from_numpy(pb["table"]).cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(pb["seqused"]).cuda()
    p.block_table, p.sparse_indices, p.seqused_kv = tb.data_ptr(), ti.data_ptr(), tu.data_ptr()
    plan, lay = sa.sparse_attn_metadata(p, sa.META_SFA_PAGES, "cuda")
    torch.cuda.synchronize()
    cap = 5 * 2
    pages = sa.plan_array(plan, lay, 1, 3 * 2 * cap).cpu().numpy().reshape(3, 2, cap)
    count = sa.plan_array(plan, lay, 3, 3 * 2).cpu().numpy().reshape(3, 2)
    ref, status = M.sfa_page_lists(idx, pb["table"], pb["seqused"], pb["sbs"], pb["page"])
    for b in range(3):
        for g in range(2):
            want = [int(x) for x in ref[b, g] if x >= 0]
            assert count[b, g] == len(want)
            assert pages[b, g, :len(want)].tolist() == want
    assert status == M.BAD_INDEX and sa.bsa_get_status(plan) & sa.DEV_BAD_INDEX


def test_sfa_decode_workload_sampled(cuda_ok):
    """Paged sparse decode workload (B=32, 128 heads, 65536-token cache, 32 pages of 64 selected)
    at full size in one launch; unselected pages hold NaN; four batches checked against the oracle."""
    w = synth.workload(4)
    table, idx = w.selection()
    seqused = np.full(w.B, w.context, np.int32)
    used = np.unique(table[np.arange(w.B)[:, None], idx[:, 0, 0, :]].ravel())
    caches = {}
    for tag, d in (("k", 512), ("k_rope", 64), ("v", 512)):
        t = torch.full((w.n_pages, w.page, 1, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        t[torch.from_numpy(used).long().cuda()] = dev_bf16(w.pages(tag, used))
        caches[tag] = t
    q, qr = w.query("q"), w.query("q_rope")
    out, lse = sa.sfa_sparse_decode(dev_bf16(q), dev_bf16(qr), caches["k"], caches["k_rope"], caches["v"],
                                    torch.from_numpy(table).cuda(), torch.from_numpy(idx).cuda(),
                                    torch.from_numpy(seqused).cuda(), w.sparse_block, w.scale)
    torch.cuda.synchronize()
    batches = [0, 7, 19, 31]
    kc = {int(pg): w.pages("k", [pg])[0] for b in batches for pg in table[b, idx[b, 0, 0]]}
    krc = {pg: w.pages("k_rope", [pg])[0] for pg in kc}
    vc = {pg: w.pages("v", [pg])[0] for pg in kc}
    r_out, r_lse = A.sfa_decode(q, qr, kc, krc, vc, table, idx, seqused, w.page, w.sparse_block, w.scale,
                                batches=batches)
    for b in batches:
        check_close(out[b].float().cpu().numpy(), r_out[b], f"out[{b}]")
        assert np.abs(lse[b].cpu().numpy() - r_lse[b]).max() <= LSE_ATOL
    assert np.isfinite(out.float().cpu().numpy()).all()



def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("case", [
    dict(B=3, N1=128, N2=2, page=32, n_logical=24, K=5, sbs=64, seqused=[768, 600, 97]),   # 12 units
    dict(B=40, N1=64, N2=1, page=64, n_logical=6, K=4, sbs=64, seqused=[384 - 7 * (i % 5) for i in range(40)]),
    dict(B=80, N1=128, N2=1, page=64, n_logical=6, K=3, sbs=128, seqused=[384 - 50 * (i % 7) for i in range(80)]),
    dict(B=1, N1=64, N2=1, page=64, n_logical=40, K=19, sbs=64, seqused=[2500]),            # one unit
])
def test_sfa_work_split_bit_exact(cuda_ok, case):
    """The decode's own split of its work (the prologue code, run by the metadata op): per piece
    the unit's compacted page list and (n, begin, len), against the CPU reference, bit for bit;
    pieces per unit as one wave of SMs allows (1 to 4 here)."""
    pb = _problem(**case, seed=31, fill_nan=False)
    idx = pb["idx"].copy()
    idx[0, 0, 0, -1] = 10 ** 6  # past the sequence: dropped, flagged
    tb, ti, tu = (torch.from_numpy(x).cuda() for x in (pb["table"], idx, pb["seqused"]))
    q = torch.empty(case["B"], 1, case["N1"], 512, device="meta")
    p = sa.sfa_params(q, pb["dev"]["k"], tb, ti, tu, pb["sbs"])
    plan, lay = sa.sparse_attn_metadata(p, sa.META_SFA_WORK, "cuda")
    torch.cuda.synchronize()
    N2, G = case["N2"], case["N1"] // case["N2"]
    HH = 2 if G > 64 else 1
    units = case["B"] * N2 * HH
    P = M.sfa_pieces_per_unit(units, _sms())
    assert lay.info[0] == units * P and lay.info[1] == P
    cap = case["K"] * (pb["sbs"] // pb["page"])
    pieces = units * P
    rec = sa.plan_array(plan, lay, 3, pieces * 3).cpu().numpy().reshape(pieces, 3)
    pages = sa.plan_array(plan, lay, 1, pieces * cap).cpu().numpy().reshape(pieces, cap)
    tokens = sa.plan_array(plan, lay, 2, pieces * cap).cpu().numpy().reshape(pieces, cap)
    ref_pages, status = M.sfa_page_lists(idx, pb["table"], pb["seqused"], pb["sbs"], pb["page"])
    count = (ref_pages >= 0).sum(axis=2).reshape(-1)
    assert np.array_equal(rec, M.sfa_pieces(count, HH, P))
    for piece in range(pieces):
        bg = piece // P // HH
        b, g = bg // N2, bg % N2
        want = [int(x) for x in ref_pages[b, g] if x >= 0]
        n = len(want)
        assert pages[piece, :n].tolist() == want
        # tokens in use of each listed page: a full page except where the sequence ends inside it
        lp = [j * (pb["sbs"] // pb["page"]) + k for j in idx[b, 0, g] if 0 <= j < 10 ** 6
              for k in range(pb["sbs"] // pb["page"]) if (j * (pb["sbs"] // pb["page"]) + k) * pb["page"] < pb["seqused"][b]]
        want_tok = [min(pb["page"], int(pb["seqused"][b]) - x * pb["page"]) for x in lp]
        assert tokens[piece, :n].tolist() == want_tok
    assert status == M.BAD_INDEX and sa.bsa_get_status(plan) & sa.DEV_BAD_INDEX


@pytest.mark.parametrize("case", [
    dict(B=3, N1=128, N2=1, page=64, n_logical=16, K=6, sbs=64, seqused=[1000, 700, 1023]),   # 4 pieces a unit
    dict(B=40, N1=64, N2=1, page=64, n_logical=6, K=4, sbs=64, seqused=[377 - 3 * (i % 9) for i in range(40)]),
    dict(B=80, N1=128, N2=1, page=32, n_logical=8, K=3, sbs=64, seqused=[250 - 9 * (i % 6) for i in range(80)]),
])
def test_sfa_decode_nan_past_seqused(cuda_ok, case):
    """Cache rows past seqused_kv inside the last, partly used page hold NaN (an uninitialised tail,
    as paged caches leave it): they get weight 0 and must not reach Out.  Pieces per unit from 1
    to 4 (the cluster merge at 3 and 4 pieces, a single CTA per unit when units exceed the SMs)."""
    pb = _problem(**case, seed=37)
    page = pb["page"]
    for b, used in enumerate(pb["seqused"]):
        if used % page:
            phys = int(pb["table"][b, used // page])
            for name in ("k", "kr", "v"):
                pb["dev"][name][phys, used % page:] = float("nan")
    out, lse, r_out, r_lse = _run(pb)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    check_close(got, r_out, "out")
    fin = np.isfinite(r_lse)
    assert np.abs(lse.cpu().numpy()[fin] - r_lse[fin]).max() <= LSE_ATOL
