"""The C-ABI library loads, exports every symbol include/*.h declares, and its host-side
validation rejects problems the pages rule out, all without a GPU (no compute calls)."""
import ctypes
import os
import re

import pytest

import selected_attention_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            txt = open(os.path.join(inc, f)).read()
            names |= set(re.findall(r"^BSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt, flags=re.M))
    return names


@pytest.fixture(scope="module", autouse=True)
def built():
    from selected_attention_b200 import build
    build.build()


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 15
    L = sa.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(sa.EXPORTED) <= names
    assert "sm_100a" in sa.version()


def _bsa(**kw):
    p = sa.Params()
    p.q_layout = p.kv_layout = sa.LAYOUT_BNSD
    p.B, p.N1, p.N2, p.S_q, p.S_kv, p.D, p.Dv = 2, 4, 2, 1000, 1000, 128, 128
    p.block_x, p.block_y, p.mask_mode, p.scale = 128, 128, 2, 0.088
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def _ws(fn, p):
    n = ctypes.c_size_t()
    return getattr(sa.lib(), fn)(ctypes.byref(p), ctypes.byref(n)), n.value


def test_bsa_host_validation():
    code, n = _ws("bsa_fwd_workspace_size", _bsa())
    assert code == sa.BSA_OK and n > 0 and n % 256 == 0
    assert _ws("bsa_fwd_workspace_size", _bsa(N2=3))[0] == sa.BSA_ERR_INVALID_ARG      # N1 % N2
    assert _ws("bsa_fwd_workspace_size", _bsa(N1=1, N2=2))[0] == sa.BSA_ERR_INVALID_ARG  # N1 < N2
    assert _ws("bsa_fwd_workspace_size", _bsa(D=64, Dv=64))[0] == sa.BSA_ERR_UNSUPPORTED  # headdim=128
    assert _ws("bsa_fwd_workspace_size", _bsa(q_layout=sa.LAYOUT_TND))[0] == sa.BSA_ERR_UNSUPPORTED
    assert _ws("bsa_fwd_workspace_size", _bsa(block_y=96))[0] == sa.BSA_ERR_UNSUPPORTED
    assert _ws("bsa_fwd_workspace_size", _bsa(mask_mode=1))[0] == sa.BSA_ERR_INVALID_ARG
    assert _ws("bsa_fwd_workspace_size", _bsa(S_q=0))[0] == sa.BSA_ERR_INVALID_ARG
    assert _ws("bsa_fwd_workspace_size", _bsa(scale=float("nan")))[0] == sa.BSA_ERR_INVALID_ARG
    assert _ws("bsa_fwd_workspace_size", _bsa(scale=-0.1))[0] == sa.BSA_ERR_INVALID_ARG
    L = sa.lib()
    assert L.bsa_fwd_workspace_size(None, None) == sa.BSA_ERR_NULLPTR
    # op call with NULL tensors fails validation before any launch
    p = _bsa()
    assert L.bsa_fwd(ctypes.byref(p), None, None, None, None, None, None, 0, None) == sa.BSA_ERR_NULLPTR


def test_workspace_size_matches_layout():
    p = _bsa(B=1, N1=2, N2=2, S_q=512, S_kv=512, block_x=64, block_y=64)
    code, n = _ws("bsa_fwd_workspace_size", p)
    units, nkb = 1 * 2 * 8, 8
    assert code == sa.BSA_OK and n >= 4 * (units + units + 1 + units * nkb)
    lay = sa.sparse_attn_metadata_layout(p, sa.META_BSA_KV)
    assert lay.count == 4 and lay.total_bytes >= lay.offsets[3] + 4 * units


def _sfa(**kw):
    p = sa.Params()
    p.q_layout, p.kv_layout = sa.LAYOUT_BSND, sa.LAYOUT_PA_ND
    p.B, p.N1, p.N2, p.S_q, p.D, p.Dv, p.D_rope = 2, 128, 1, 1, 512, 512, 64
    p.page_size, p.sparse_block_size, p.sparse_count = 64, 64, 32
    p.max_pages_per_seq, p.num_pages, p.scale = 1024, 2048, 576 ** -0.5
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_sfa_host_validation():
    """SparseFlashAttention constraints: D = Dv = 512 with a 64-dim rope part, one query row,
    a page size that is a multiple of 16 (here of 32), sparse blocks of whole pages."""
    fn = "sfa_sparse_decode_workspace_size"
    code, n = _ws(fn, _sfa())
    assert code == sa.BSA_OK and n > 0
    assert _ws(fn, _sfa(S_q=2))[0] == sa.BSA_ERR_UNSUPPORTED
    assert _ws(fn, _sfa(D=256, Dv=256))[0] == sa.BSA_ERR_UNSUPPORTED
    assert _ws(fn, _sfa(D_rope=0))[0] == sa.BSA_ERR_UNSUPPORTED
    assert _ws(fn, _sfa(page_size=48, sparse_block_size=96))[0] == sa.BSA_ERR_UNSUPPORTED  # not a multiple of 32
    assert _ws(fn, _sfa(page_size=40))[0] == sa.BSA_ERR_INVALID_ARG
    assert _ws(fn, _sfa(page_size=2048, sparse_block_size=2048))[0] == sa.BSA_ERR_INVALID_ARG
    assert _ws(fn, _sfa(sparse_block_size=96))[0] == sa.BSA_ERR_INVALID_ARG  # not whole pages
    assert _ws(fn, _sfa(N2=3))[0] == sa.BSA_ERR_INVALID_ARG
    assert _ws(fn, _sfa(N1=256))[0] == sa.BSA_ERR_UNSUPPORTED  # G > 128
    assert _ws(fn, _sfa(num_pages=1 << 25))[0] == sa.BSA_ERR_UNSUPPORTED  # token index past int32
    assert _ws(fn, _sfa(scale=float("inf")))[0] == sa.BSA_ERR_INVALID_ARG
    assert _ws(fn, _sfa(kv_layout=sa.LAYOUT_BNSD))[0] == sa.BSA_ERR_UNSUPPORTED
    assert _ws(fn, _sfa(page_size=32, sparse_block_size=64))[0] == sa.BSA_OK  # 32-token pages
    # a group of more than 64 query heads is split into two head halves, each with its own pieces
    n64 = _ws(fn, _sfa(N1=64))[1]
    assert _ws(fn, _sfa(N1=96))[1] > n64
    L = sa.lib()
    p = _sfa()
    assert L.sfa_sparse_decode(ctypes.byref(p), None, None, None, None, None, None, None, None, 0,
                               None) == sa.BSA_ERR_NULLPTR


def _nsa(**kw):
    p = sa.Params()
    p.q_layout = p.kv_layout = sa.LAYOUT_TND
    p.B, p.N1, p.N2, p.T_q, p.T_kv, p.S_q, p.D, p.Dv = 2, 64, 4, 4096, 4096, 2048, 128, 128
    p.sel_block_size, p.sel_block_count, p.mask_mode, p.scale = 64, 16, 2, 0.088
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_nsa_host_validation():
    """NsaSelectedAttention constraints: TND, headdim 128, block size a multiple of 16 up to 128,
    at most 128 blocks and 8K selected tokens, sparseMode 0 or 2, equal query and key lengths."""
    for fn in ("nsa_selected_fwd_workspace_size", "nsa_selected_bwd_workspace_size"):
        code, n = _ws(fn, _nsa())
        assert code == sa.BSA_OK and n > 0
        assert _ws(fn, _nsa(q_layout=sa.LAYOUT_BNSD))[0] == sa.BSA_ERR_UNSUPPORTED
        assert _ws(fn, _nsa(D=64, Dv=64))[0] == sa.BSA_ERR_UNSUPPORTED
        assert _ws(fn, _nsa(sel_block_size=40))[0] == sa.BSA_ERR_INVALID_ARG
        assert _ws(fn, _nsa(sel_block_size=256))[0] == sa.BSA_ERR_INVALID_ARG
        assert _ws(fn, _nsa(sel_block_count=129))[0] == sa.BSA_ERR_INVALID_ARG
        assert _ws(fn, _nsa(sel_block_count=128, sel_block_size=128))[0] == sa.BSA_ERR_INVALID_ARG  # > 8K tokens
        assert _ws(fn, _nsa(mask_mode=3))[0] == sa.BSA_ERR_INVALID_ARG
        assert _ws(fn, _nsa(T_kv=4000))[0] == sa.BSA_ERR_INVALID_ARG
        assert _ws(fn, _nsa(N2=3))[0] == sa.BSA_ERR_INVALID_ARG
        assert _ws(fn, _nsa(N1=256, N2=4))[0] == sa.BSA_ERR_INVALID_ARG
        assert _ws(fn, _nsa(S_q=5000))[0] == sa.BSA_ERR_INVALID_ARG  # longer than T
        assert _ws(fn, _nsa(scale=0.0))[0] == sa.BSA_ERR_INVALID_ARG


def test_metadata_layouts_without_gpu():
    """Plan layouts of the NSA and decode metadata ops: array offsets in order, 256-byte aligned,
    inside the plan, sized for the problem."""
    p = _sfa()
    lay = sa.sparse_attn_metadata_layout(p, sa.META_SFA_PAGES)
    lists = p.B * p.N2 * p.sparse_count * (p.sparse_block_size // p.page_size)
    assert lay.count == 4
    offs = [lay.offsets[i] for i in range(1, 4)]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert offs[1] - offs[0] >= 4 * lists and lay.total_bytes >= offs[2] + 4 * p.B * p.N2
    q = _nsa()
    kv = sa.sparse_attn_metadata_layout(q, sa.META_NSA_KV)
    tok = sa.sparse_attn_metadata_layout(q, sa.META_NSA_TOKENS)
    assert kv.count == 3 and tok.count == 5
    ids_bytes = 4 * q.T_q * q.N2 * q.sel_block_count
    assert kv.offsets[2] - kv.offsets[1] >= ids_bytes and tok.total_bytes > kv.total_bytes
    assert sa.lib().sparse_attn_metadata_layout(ctypes.byref(q), 99, ctypes.byref(sa.MetaLayout())) \
        == sa.BSA_ERR_UNSUPPORTED


def test_plan_input_validation():
    """A metadata plan passed to an op must come from an op that holds the lists it reads, be
    256-byte aligned, and shrinks the op's workspace to its scratch; the decode takes none."""
    fake = 1 << 20  # an aligned address: sizing calls never dereference the plan
    n_plain = _ws("bsa_fwd_workspace_size", _bsa())[1]
    code, n = _ws("bsa_fwd_workspace_size", _bsa(plan=fake, plan_op=sa.META_BSA_KV))
    assert code == sa.BSA_OK and n == 256 < n_plain
    assert _ws("bsa_fwd_workspace_size", _bsa(plan=fake, plan_op=sa.META_BSA_BWD))[0] == sa.BSA_OK
    assert _ws("bsa_fwd_workspace_size", _bsa(plan=fake, plan_op=sa.META_BSA_Q))[0] == sa.BSA_ERR_INVALID_ARG
    assert _ws("bsa_fwd_workspace_size", _bsa(plan=fake + 4, plan_op=sa.META_BSA_KV))[0] == sa.BSA_ERR_INVALID_ARG
    b_plain = _ws("bsa_bwd_workspace_size", _bsa())[1]
    code, b = _ws("bsa_bwd_workspace_size", _bsa(plan=fake, plan_op=sa.META_BSA_BWD))
    assert code == sa.BSA_OK and b < b_plain
    assert _ws("bsa_bwd_workspace_size", _bsa(plan=fake, plan_op=sa.META_BSA_KV))[0] == sa.BSA_ERR_INVALID_ARG
    q = _nsa()
    q.plan, q.plan_op = fake, sa.META_NSA_KV
    assert _ws("nsa_selected_fwd_workspace_size", q)[0] == sa.BSA_OK
    assert _ws("nsa_selected_bwd_workspace_size", q)[0] == sa.BSA_ERR_INVALID_ARG
    q.plan_op = sa.META_NSA_TOKENS
    code, nb = _ws("nsa_selected_bwd_workspace_size", q)
    q.plan = None
    assert code == sa.BSA_OK and nb < _ws("nsa_selected_bwd_workspace_size", q)[1]
    assert _ws("sfa_sparse_decode_workspace_size", _sfa(plan=fake, plan_op=sa.META_SFA_WORK))[0] \
        == sa.BSA_ERR_UNSUPPORTED


def test_bsa_bwd_plan_layout():
    """The backward plan holds both list sets: forward CSR then transposed CSR, each array
    256-byte aligned and sized like the single-op plans."""
    p = _bsa(B=1, N1=4, N2=2, S_q=1000, S_kv=1000)
    units, nkb, trows = 1 * 4 * 8, 8, 1 * 2 * 8
    lay = sa.sparse_attn_metadata_layout(p, sa.META_BSA_BWD)
    assert lay.count == 6
    offs = [lay.offsets[i] for i in range(1, 6)]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert offs[1] - offs[0] >= 4 * (units + 1) and offs[2] - offs[1] >= 4 * units * nkb
    assert offs[3] - offs[2] >= 4 * (trows + 1) and offs[4] - offs[3] >= 4 * units * nkb
    assert lay.total_bytes >= offs[4] + 4 * (units + trows) + units * nkb


def test_partition_matches_cpu_reference():
    """bsa_partition (host code in the library, no device access) against the CPU reference's
    slice_cuts, bit for bit, and its argument checks."""
    from oracle import metadata as M
    import numpy as np
    rng = np.random.default_rng(11)
    for _ in range(200):
        n, parts = int(rng.integers(0, 40)), int(rng.integers(1, 10))
        w = rng.integers(0, 1000, n) * (rng.random(n) < 0.8)
        assert sa.partition(w, parts).tolist() == M.slice_cuts(w, parts).tolist()
    big = np.full(1024, 2 ** 40, np.int64)  # totals past 2^32
    assert sa.partition(big, 7).tolist() == M.slice_cuts(big, 7).tolist()
    starts = (ctypes.c_int32 * 3)()
    neg = (ctypes.c_int64 * 2)(1, -1)
    assert sa.lib().bsa_partition(neg, 2, 2, starts) == sa.BSA_ERR_INVALID_ARG
    assert sa.lib().bsa_partition(neg, 2, 0, starts) == sa.BSA_ERR_INVALID_ARG
    assert sa.lib().bsa_partition(None, 2, 2, starts) == sa.BSA_ERR_NULLPTR


def test_sfa_bwd_host_validation():
    """The decode backward takes the decode's constraints; its workspace holds the gathered-order
    row gradients (~2.2 KB per selected token) and takes no metadata plan."""
    p = _sfa()
    code, n = _ws("sfa_sparse_decode_bwd_workspace_size", p)
    tokens = p.B * p.N2 * p.sparse_count * p.sparse_block_size
    assert code == sa.BSA_OK and n >= tokens * (576 + 512) * 2
    assert _ws("sfa_sparse_decode_bwd_workspace_size", _sfa(S_q=2))[0] == sa.BSA_ERR_UNSUPPORTED
    assert _ws("sfa_sparse_decode_bwd_workspace_size", _sfa(plan=1 << 20, plan_op=sa.META_SFA_WORK))[0] \
        == sa.BSA_ERR_UNSUPPORTED
    assert sa.lib().sfa_sparse_decode_bwd(ctypes.byref(p), *([None] * 14), 0, None) == sa.BSA_ERR_NULLPTR


def test_nsa_head_dim_pairs():
    """q / k / v head dims 128 / 128, or 192 / 128 with query groups of at most 16 heads."""
    fn = "nsa_selected_fwd_workspace_size"
    assert _ws(fn, _nsa(D=192, Dv=128, N1=64, N2=4))[0] == sa.BSA_OK          # G = 16
    assert _ws(fn, _nsa(D=192, Dv=128, N1=64, N2=2))[0] == sa.BSA_ERR_UNSUPPORTED  # G = 32
    assert _ws(fn, _nsa(D=192, Dv=192))[0] == sa.BSA_ERR_UNSUPPORTED
    assert _ws(fn, _nsa(D=64, Dv=128))[0] == sa.BSA_ERR_UNSUPPORTED
