"""Python binding of the sm_100a block-sparse attention library (libselected_attention.so).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
Torch supplies device memory (outputs, workspaces) and the current stream.  The functions carry
the C ABI's names (include/selected_attention.h).  If the library is missing or fails to load,
every call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libselected_attention.so")

BSA_OK, BSA_ERR_NULLPTR, BSA_ERR_INVALID_ARG, BSA_ERR_UNSUPPORTED, BSA_ERR_WORKSPACE_TOO_SMALL, BSA_ERR_CUDA = range(6)
STATUS_NAMES = {0: "BSA_OK", 1: "BSA_ERR_NULLPTR", 2: "BSA_ERR_INVALID_ARG", 3: "BSA_ERR_UNSUPPORTED",
                4: "BSA_ERR_WORKSPACE_TOO_SMALL", 5: "BSA_ERR_CUDA"}
LAYOUT_BNSD, LAYOUT_TND, LAYOUT_BSND, LAYOUT_PA_ND = 0, 1, 2, 3
MASK_NONE, MASK_CAUSAL, MASK_RIGHT_DOWN_CAUSAL, MASK_BAND = 0, 2, 3, 4
META_BSA_KV, META_BSA_Q, META_NSA_KV, META_NSA_TOKENS, META_SFA_PAGES, META_SFA_WORK, META_BSA_BWD = range(7)
DEV_BAD_INDEX, DEV_BAD_SEQLEN, DEV_TIMEOUT = 1, 2, 4

EXPORTED = [
    "bsa_fwd_workspace_size", "bsa_bwd_workspace_size", "nsa_selected_fwd_workspace_size",
    "nsa_selected_bwd_workspace_size", "sfa_sparse_decode_workspace_size", "bsa_fwd", "bsa_bwd",
    "nsa_selected_fwd", "nsa_selected_bwd", "sfa_sparse_decode", "sparse_attn_metadata_layout",
    "sparse_attn_metadata", "bsa_get_status", "bsa_version", "bsa_diag_mma_tile",
    "bsa_profile_enable", "bsa_profile_collect", "bsa_fwd_noalloc", "bsa_fwd_noalloc_get_status", "bsa_diag_exp2",
    "bsa_diag_wait", "bsa_profile_cta_clock", "bsa_partition", "sfa_sparse_decode_bwd_workspace_size",
    "sfa_sparse_decode_bwd",
]


class BsaError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(code, code)}")
        self.code = code


class Params(ctypes.Structure):
    _fields_ = [
        ("q_layout", ctypes.c_int32), ("kv_layout", ctypes.c_int32),
        ("B", ctypes.c_int32), ("N1", ctypes.c_int32), ("N2", ctypes.c_int32),
        ("S_q", ctypes.c_int32), ("S_kv", ctypes.c_int32),
        ("T_q", ctypes.c_int32), ("T_kv", ctypes.c_int32),
        ("D", ctypes.c_int32), ("Dv", ctypes.c_int32), ("D_rope", ctypes.c_int32),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_kv", ctypes.c_void_p),
        ("seqused_kv", ctypes.c_void_p),
        ("block_x", ctypes.c_int32), ("block_y", ctypes.c_int32),
        ("block_mask", ctypes.c_void_p),
        ("sel_block_size", ctypes.c_int32), ("sel_block_count", ctypes.c_int32),
        ("topk_indices", ctypes.c_void_p),
        ("page_size", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("block_table", ctypes.c_void_p),
        ("sparse_block_size", ctypes.c_int32), ("sparse_count", ctypes.c_int32),
        ("sparse_indices", ctypes.c_void_p),
        ("mask_mode", ctypes.c_int32), ("win_left", ctypes.c_int32), ("win_right", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("atten_mask", ctypes.c_void_p),
        ("plan", ctypes.c_void_p), ("plan_op", ctypes.c_int32),
    ]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_double)]


class MetaLayout(ctypes.Structure):
    _fields_ = [("total_bytes", ctypes.c_size_t), ("offsets", ctypes.c_size_t * 6), ("count", ctypes.c_int32),
                ("info", ctypes.c_size_t * 2)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it is missing: there is no CPU path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with python -m selected_attention_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(Params)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        for name in ("bsa_fwd_workspace_size", "bsa_bwd_workspace_size", "nsa_selected_fwd_workspace_size",
                     "nsa_selected_bwd_workspace_size", "sfa_sparse_decode_workspace_size",
                     "sfa_sparse_decode_bwd_workspace_size"):
            getattr(L, name).argtypes = [P, ctypes.POINTER(sz)]
        L.bsa_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        L.nsa_selected_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        L.bsa_fwd_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp]
        L.bsa_fwd_noalloc_get_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.bsa_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.nsa_selected_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sfa_sparse_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.sfa_sparse_decode_bwd.argtypes = [P] + [vp] * 14 + [sz, vp]
        L.sparse_attn_metadata_layout.argtypes = [P, ctypes.c_int32, ctypes.POINTER(MetaLayout)]
        L.sparse_attn_metadata.argtypes = [P, ctypes.c_int32, vp, sz, vp]
        L.bsa_get_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
        L.bsa_diag_mma_tile.argtypes = [vp, vp, vp, ctypes.c_int32, vp, vp]
        L.bsa_diag_exp2.argtypes = [vp, vp, ctypes.c_int32, ctypes.c_int32, vp]
        L.bsa_diag_wait.argtypes = [vp, ctypes.c_int32, vp]
        L.bsa_profile_enable.argtypes = [ctypes.c_int32]
        L.bsa_profile_cta_clock.argtypes = [vp, ctypes.c_int32]
        L.bsa_partition.argtypes = [vp, ctypes.c_int32, ctypes.c_int32, vp]
        L.bsa_profile_collect.argtypes = [ctypes.POINTER(KernelTime), ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]
        L.bsa_version.restype = ctypes.c_char_p
        for name in EXPORTED:
            if name != "bsa_version":
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(fn, code):
    if code != BSA_OK:
        raise BsaError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors (the library has no CPU path)")


def _workspace(nbytes, device):
    return torch.empty(max(256, int(nbytes)), dtype=torch.uint8, device=device)


def version() -> str:
    return lib().bsa_version().decode()


# ---------------------------------------------------------------------------------------------
# BSA (BNSD)
# ---------------------------------------------------------------------------------------------
def bsa_params(q, k, block_mask, block_x, block_y, mask_mode=MASK_CAUSAL, scale=None, win_left=0,
               win_right=0, layout=LAYOUT_BNSD, atten_mask=None) -> Params:
    """layout LAYOUT_BNSD: q [B, N1, S_q, D], k [B, N2, S_kv, D]; LAYOUT_BSND: q [B, S_q, N1, D],
    k [B, S_kv, N2, D].  atten_mask: optional uint8 CUDA tensor [S_q, S_kv], nonzero = masked out."""
    if layout == LAYOUT_BSND:
        B, S_q, N1, D = q.shape
        _, S_kv, N2, _ = k.shape
    else:
        B, N1, S_q, D = q.shape
        _, N2, S_kv, _ = k.shape
    p = Params()
    p.q_layout = p.kv_layout = layout
    p.B, p.N1, p.N2, p.S_q, p.S_kv = B, N1, N2, S_q, S_kv
    p.D = D
    p.Dv = D
    p.block_x, p.block_y = block_x, block_y
    p.block_mask = block_mask.data_ptr()
    p.mask_mode, p.win_left, p.win_right = mask_mode, win_left, win_right
    p.scale = 1.0 / math.sqrt(D) if scale is None else scale
    if atten_mask is not None:
        _need_cuda(atten_mask)
        assert atten_mask.dtype == torch.uint8 and tuple(atten_mask.shape) == (S_q, S_kv) and atten_mask.is_contiguous()
        p.atten_mask = atten_mask.data_ptr()
    return p


def _set_plan(p: Params, plan):
    """plan: None, or (plan tensor, op) as sparse_attn_metadata made it for this same problem."""
    if plan is not None:
        t, op = plan
        _need_cuda(t)
        p.plan, p.plan_op = t.data_ptr(), op
    return p


def _lse_shape(p: Params):
    return (p.B, p.S_q, p.N1) if p.q_layout == LAYOUT_BSND else (p.B, p.N1, p.S_q)


def bsa_fwd_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check("bsa_fwd_workspace_size", lib().bsa_fwd_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def bsa_fwd(q, k, v, block_mask, block_x, block_y, mask_mode=MASK_CAUSAL, scale=None, win_left=0,
            win_right=0, out=None, lse=None, workspace=None, stream=None, layout=LAYOUT_BNSD, atten_mask=None,
            plan=None):
    """Out, LSE = softmax(Mask(scale Q K_sel^T)) V_sel for BNSD (or BSND) bf16 tensors and a uint8
    BlockSparseMask [B, N1, ceil(S_q/block_x), ceil(S_kv/block_y)].  Out has q's layout; LSE is
    [B, N1, S_q] (BNSD) or [B, S_q, N1] (BSND).  plan: optional (tensor, META_BSA_KV or
    META_BSA_BWD) from sparse_attn_metadata for this problem; the lists are then not rebuilt."""
    _need_cuda(q, k, v, block_mask)
    p = bsa_params(q, k, block_mask, block_x, block_y, mask_mode, scale, win_left, win_right, layout, atten_mask)
    _set_plan(p, plan)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(_lse_shape(p), dtype=torch.float32, device=q.device)
    need = bsa_fwd_workspace_size(p)
    if workspace is None:
        workspace = _workspace(need, q.device)
    _check("bsa_fwd", lib().bsa_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                    _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, lse


def bsa_fwd_noalloc(q, k, v, block_mask, block_x, block_y, mask_mode=MASK_CAUSAL, scale=None, win_left=0,
                    win_right=0, out=None, lse=None, stream=None, layout=LAYOUT_BNSD, plan=None):
    """bsa_fwd without a workspace, for callers that cannot allocate device memory: the library
    keeps the scratch in a fixed 8 MiB device array (shared by all calls on a device; calls that
    overlap on the GPU race).  Out and LSE are still the caller's tensors.  With a plan (as for
    bsa_fwd) the lists are the plan's and the array holds only the status header, so problems
    whose lists exceed 8 MiB run too."""
    _need_cuda(q, k, v, block_mask)
    p = bsa_params(q, k, block_mask, block_x, block_y, mask_mode, scale, win_left, win_right, layout)
    _set_plan(p, plan)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(_lse_shape(p), dtype=torch.float32, device=q.device)
    _check("bsa_fwd_noalloc", lib().bsa_fwd_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                                    _ptr(lse), _stream(stream)))
    return out, lse


def bsa_fwd_noalloc_get_status(stream=None) -> int:
    """Device status bits of the last bsa_fwd_noalloc call on the current device (synchronises)."""
    v = ctypes.c_uint32()
    _check("bsa_fwd_noalloc_get_status", lib().bsa_fwd_noalloc_get_status(_stream(stream), ctypes.byref(v)))
    return v.value


def bsa_bwd_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check("bsa_bwd_workspace_size", lib().bsa_bwd_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def bsa_bwd(q, k, v, out, dout, lse, block_mask, block_x, block_y, mask_mode=MASK_CAUSAL, scale=None,
            win_left=0, win_right=0, dq=None, dk=None, dv=None, workspace=None, stream=None, layout=LAYOUT_BNSD,
            atten_mask=None, plan=None):
    """dQ, dK, dV of block-sparse attention (BNSD or BSND, the gradients in the inputs' layout).
    plan: optional (tensor, META_BSA_BWD) from sparse_attn_metadata for this problem."""
    _need_cuda(q, k, v, out, dout, lse, block_mask)
    p = bsa_params(q, k, block_mask, block_x, block_y, mask_mode, scale, win_left, win_right, layout, atten_mask)
    _set_plan(p, plan)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bsa_bwd_workspace_size(p)
    if workspace is None:
        workspace = _workspace(need, q.device)
    _check("bsa_bwd", lib().bsa_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                                    _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel(),
                                    _stream(stream)))
    return dq, dk, dv


# ---------------------------------------------------------------------------------------------
# metadata
# ---------------------------------------------------------------------------------------------
def sparse_attn_metadata_layout(p: Params, op: int) -> MetaLayout:
    L = MetaLayout()
    _check("sparse_attn_metadata_layout", lib().sparse_attn_metadata_layout(ctypes.byref(p), op, ctypes.byref(L)))
    return L


def sparse_attn_metadata(p: Params, op: int, device, stream=None):
    """Runs the metadata kernels for `op`; returns (plan tensor, layout)."""
    L = sparse_attn_metadata_layout(p, op)
    plan = _workspace(L.total_bytes, device)
    _check("sparse_attn_metadata", lib().sparse_attn_metadata(ctypes.byref(p), op, _ptr(plan), plan.numel(),
                                                              _stream(stream)))
    return plan, L


def plan_array(plan, layout: MetaLayout, index: int, count: int, dtype=torch.int32):
    """View `count` elements of array `index` of a metadata plan."""
    off = layout.offsets[index]
    itemsize = torch.empty(0, dtype=dtype).element_size()
    return plan[off:off + count * itemsize].view(dtype)


# ---------------------------------------------------------------------------------------------
# NSA selected attention (TND)
# ---------------------------------------------------------------------------------------------
def nsa_params(q, k, topk_indices, cu_seqlens, max_seqlen, sel_block_size, mask_mode=MASK_CAUSAL,
               scale=None, dv=None) -> Params:
    """q [T, N1, D], k [T, N2, D] (D = 128, or 192 with v's 128: dv), topk_indices [T, N2, K] int32,
    cu_seqlens [B+1] int32 (device)."""
    T, N1, D = q.shape
    _, N2, _ = k.shape
    p = Params()
    p.q_layout = p.kv_layout = LAYOUT_TND
    p.B, p.N1, p.N2 = cu_seqlens.shape[0] - 1, N1, N2
    p.S_q = p.S_kv = int(max_seqlen)
    p.T_q = p.T_kv = T
    p.D = D
    p.Dv = D if dv is None else dv
    p.cu_seqlens_q = p.cu_seqlens_kv = cu_seqlens.data_ptr()
    p.sel_block_size, p.sel_block_count = sel_block_size, topk_indices.shape[-1]
    p.topk_indices = topk_indices.data_ptr()
    p.mask_mode = mask_mode
    p.scale = 1.0 / math.sqrt(D) if scale is None else scale
    return p


def nsa_selected_fwd_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check("nsa_selected_fwd_workspace_size", lib().nsa_selected_fwd_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def nsa_selected_bwd_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check("nsa_selected_bwd_workspace_size", lib().nsa_selected_bwd_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def nsa_selected_fwd(q, k, v, topk_indices, cu_seqlens, max_seqlen, sel_block_size, mask_mode=MASK_CAUSAL,
                     scale=None, out=None, lse=None, workspace=None, stream=None, plan=None):
    """Out [T, N1, Dv] bf16, LSE [T, N1] fp32 of NSA selected attention (q, k [.., D], v [.., Dv]).
    plan: optional (tensor, META_NSA_KV or META_NSA_TOKENS) from sparse_attn_metadata for this
    problem."""
    _need_cuda(q, k, v, topk_indices, cu_seqlens)
    p = nsa_params(q, k, topk_indices, cu_seqlens, max_seqlen, sel_block_size, mask_mode, scale, v.shape[-1])
    _set_plan(p, plan)
    out = torch.empty(q.shape[0], q.shape[1], v.shape[-1], dtype=torch.bfloat16, device=q.device) if out is None else out
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device) if lse is None else lse
    if workspace is None:
        workspace = _workspace(nsa_selected_fwd_workspace_size(p), q.device)
    _check("nsa_selected_fwd", lib().nsa_selected_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                                      _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, lse


def nsa_selected_bwd(q, k, v, out, dout, lse, topk_indices, cu_seqlens, max_seqlen, sel_block_size,
                     mask_mode=MASK_CAUSAL, scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None,
                     plan=None):
    """dQ, dK, dV of NSA selected attention.  plan: optional (tensor, META_NSA_TOKENS) from
    sparse_attn_metadata for this problem."""
    _need_cuda(q, k, v, out, dout, lse, topk_indices, cu_seqlens)
    p = nsa_params(q, k, topk_indices, cu_seqlens, max_seqlen, sel_block_size, mask_mode, scale, v.shape[-1])
    _set_plan(p, plan)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = _workspace(nsa_selected_bwd_workspace_size(p), q.device)
    _check("nsa_selected_bwd", lib().nsa_selected_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout),
                                                      _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                                      workspace.numel(), _stream(stream)))
    return dq, dk, dv


# ---------------------------------------------------------------------------------------------
# SFA: sparse decode over a paged KV cache
# ---------------------------------------------------------------------------------------------
def sfa_params(q, k_cache, block_table, sparse_indices, seqused_kv, sparse_block_size, scale=None) -> Params:
    """q [B, 1, N1, 512]; caches [num_pages, page_size, N2, D]; block_table [B, max_pages];
    sparse_indices [B, 1, N2, K] int32; seqused_kv [B] int32 (all device tensors)."""
    B, Sq, N1, D = q.shape
    num_pages, page_size, N2, _ = k_cache.shape
    p = Params()
    p.q_layout = LAYOUT_BSND
    p.kv_layout = LAYOUT_PA_ND
    p.B, p.N1, p.N2, p.S_q = B, N1, N2, Sq
    p.D, p.Dv, p.D_rope = D, D, 64
    p.seqused_kv = seqused_kv.data_ptr()
    p.page_size, p.max_pages_per_seq, p.num_pages = page_size, block_table.shape[1], num_pages
    p.block_table = block_table.data_ptr()
    p.sparse_block_size, p.sparse_count = sparse_block_size, sparse_indices.shape[-1]
    p.sparse_indices = sparse_indices.data_ptr()
    p.mask_mode = MASK_NONE
    p.scale = 1.0 / math.sqrt(D + 64) if scale is None else scale
    return p


def sfa_sparse_decode_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check("sfa_sparse_decode_workspace_size", lib().sfa_sparse_decode_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def sfa_sparse_decode(q, q_rope, k_cache, k_rope_cache, v_cache, block_table, sparse_indices, seqused_kv,
                      sparse_block_size, scale=None, out=None, lse=None, workspace=None, stream=None):
    """Out [B, 1, N1, 512] bf16, LSE [B, 1, N1] fp32 of sparse decode attention."""
    _need_cuda(q, q_rope, k_cache, k_rope_cache, v_cache, block_table, sparse_indices, seqused_kv)
    p = sfa_params(q, k_cache, block_table, sparse_indices, seqused_kv, sparse_block_size, scale)
    B, Sq, N1, D = q.shape
    if out is None:
        out = torch.empty(B, Sq, N1, v_cache.shape[-1], dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty(B, Sq, N1, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _workspace(sfa_sparse_decode_workspace_size(p), q.device)
    _check("sfa_sparse_decode", lib().sfa_sparse_decode(ctypes.byref(p), _ptr(q), _ptr(q_rope), _ptr(k_cache),
                                                        _ptr(k_rope_cache), _ptr(v_cache), _ptr(out), _ptr(lse),
                                                        _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, lse


def sfa_sparse_decode_bwd_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t()
    _check("sfa_sparse_decode_bwd_workspace_size",
           lib().sfa_sparse_decode_bwd_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def sfa_sparse_decode_bwd(q, q_rope, k_cache, k_rope_cache, v_cache, out, dout, lse, block_table, sparse_indices,
                          seqused_kv, sparse_block_size, scale=None, dq=None, dq_rope=None, dk_cache=None,
                          dk_rope_cache=None, dv_cache=None, workspace=None, stream=None):
    """dQ, dQ_rope and the cache gradients of sparse decode attention.  The cache rows the step
    read are set to their gradient; rows it did not read are left as they are (the caches this
    function allocates when none are given start at zero)."""
    _need_cuda(q, q_rope, k_cache, k_rope_cache, v_cache, out, dout, lse, block_table, sparse_indices, seqused_kv)
    p = sfa_params(q, k_cache, block_table, sparse_indices, seqused_kv, sparse_block_size, scale)
    dq = torch.empty_like(q) if dq is None else dq
    dq_rope = torch.empty_like(q_rope) if dq_rope is None else dq_rope
    dk_cache = torch.zeros_like(k_cache) if dk_cache is None else dk_cache
    dk_rope_cache = torch.zeros_like(k_rope_cache) if dk_rope_cache is None else dk_rope_cache
    dv_cache = torch.zeros_like(v_cache) if dv_cache is None else dv_cache
    if workspace is None:
        workspace = _workspace(sfa_sparse_decode_bwd_workspace_size(p), q.device)
    _check("sfa_sparse_decode_bwd", lib().sfa_sparse_decode_bwd(
        ctypes.byref(p), _ptr(q), _ptr(q_rope), _ptr(k_cache), _ptr(k_rope_cache), _ptr(v_cache), _ptr(out),
        _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dq_rope), _ptr(dk_cache), _ptr(dk_rope_cache), _ptr(dv_cache),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return dq, dq_rope, dk_cache, dk_rope_cache, dv_cache


def partition(weights, parts: int):
    """Contiguous balanced split (the C bsa_partition): int32 starts [parts + 1], part s taking
    items [starts[s], starts[s + 1]) of the int64 weights."""
    import numpy as np
    w = np.ascontiguousarray(weights, dtype=np.int64)
    starts = np.zeros(parts + 1, dtype=np.int32)
    _check("bsa_partition", lib().bsa_partition(w.ctypes.data_as(ctypes.c_void_p), len(w), parts,
                                                starts.ctypes.data_as(ctypes.c_void_p)))
    return starts


def bsa_get_status(workspace, stream=None) -> int:
    v = ctypes.c_uint32()
    _check("bsa_get_status", lib().bsa_get_status(_ptr(workspace), _stream(stream), ctypes.byref(v)))
    return v.value


def bsa_profile_enable(on: bool = True) -> None:
    """Start (or stop) timing every kernel launch the library makes."""
    _check("bsa_profile_enable", lib().bsa_profile_enable(1 if on else 0))


def bsa_profile_cta_clock(buf=None) -> None:
    """Record per-CTA start / finish times of the persistent block-sparse kernels into `buf`, a
    CUDA int64 tensor [3, capacity, 2] (slot 0 forward, 1 KV-major pass, 2 Q-major pass); None
    stops recording."""
    if buf is None:
        _check("bsa_profile_cta_clock", lib().bsa_profile_cta_clock(None, 0))
        return
    _need_cuda(buf)
    assert buf.dtype == torch.int64 and buf.dim() == 3 and buf.shape[0] == 3 and buf.shape[2] == 2
    _check("bsa_profile_cta_clock", lib().bsa_profile_cta_clock(_ptr(buf), buf.shape[1]))


def bsa_profile_collect() -> dict:
    """{kernel name: (launches, total ms)} for the launches recorded since enabling (synchronises)."""
    buf = (KernelTime * 64)()
    n = ctypes.c_int32()
    _check("bsa_profile_collect", lib().bsa_profile_collect(buf, 64, ctypes.byref(n)))
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(min(n.value, 64))}


# ---------------------------------------------------------------------------------------------
# diagnostics
# ---------------------------------------------------------------------------------------------
def bsa_diag_mma_tile(a, b, mode, stream=None):
    """One tcgen05 tile.  mode 0/2: c = a @ b.T; 1/3: c = a @ b (2, 3 stage a in tensor memory);
    4: c = a.T @ b.T; 5: c = a.T @ b (a read as the MN-major A operand)."""
    _need_cuda(a, b)
    c = torch.empty(128, 128, dtype=torch.float32, device=a.device)
    ws = _workspace(256, a.device)
    _check("bsa_diag_mma_tile", lib().bsa_diag_mma_tile(_ptr(a), _ptr(b), _ptr(c), int(mode), _ptr(ws),
                                                        _stream(stream)))
    return c, ws


def bsa_diag_wait(arrive: bool, device="cuda", stream=None) -> int:
    """Run the bounded-wait diagnostic and return the device status bits (SA_DEV_TIMEOUT = 4 when
    nothing arrived)."""
    ws = _workspace(256, torch.device(device))
    _check("bsa_diag_wait", lib().bsa_diag_wait(_ptr(ws), 1 if arrive else 0, _stream(stream)))
    return bsa_get_status(ws, stream)


def bsa_diag_exp2(x, degree, stream=None):
    """2^x by the device polynomial of the given degree (3 or 4); x a CUDA float32 tensor."""
    _need_cuda(x)
    y = torch.empty_like(x)
    _check("bsa_diag_exp2", lib().bsa_diag_exp2(_ptr(x), _ptr(y), x.numel(), degree, _stream(stream)))
    return y
