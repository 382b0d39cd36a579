"""bsa_fwd_noalloc: the forward for callers that cannot allocate device memory (a host that owns
all device memory and gives plugins no scratch, or a path where cudaMalloc is not acceptable).
It keeps its scratch in a fixed 8 MiB device array inside the library instead of a caller
workspace.  Checked through the C ABI against bsa_fwd (which the oracle pins elsewhere): both run
the same kernels on the same lists, so Out and LSE must be bit-identical, on two calls in a row
(the second reuses the array the first left behind), on a larger problem followed by a smaller
one (stale lists of the larger one must not leak into the smaller), and for its size limit.  The
device status word of the last call is read back through bsa_fwd_noalloc_get_status.

This file is collected last on purpose, so a failure here comes after every other test ran."""
import ctypes

import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from parity import dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def _inputs(case):
    if case == "tiny":
        w = synth.workload(1)
        mask = w.block_mask()
        return (dev_bf16(w.tensor("q")), dev_bf16(w.tensor("k")), dev_bf16(w.tensor("v")),
                torch.from_numpy(mask).cuda(), 64, 64, w.scale)
    rng = np.random.default_rng(5 if case == "ragged_gqa" else 6)
    B, N1, N2, S, D = (2, 4, 2, 300, 128) if case == "ragged_gqa" else (2, 8, 4, 2048, 128)
    nb = -(-S // 128)
    q = synth.f32_to_bf16_bits(rng.standard_normal((B, N1, S, D), dtype=np.float32))
    k = synth.f32_to_bf16_bits(rng.standard_normal((B, N2, S, D), dtype=np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal((B, N2, S, D), dtype=np.float32))
    mask = (rng.random((B, N1, nb, nb)) < 0.6).astype(np.uint8)
    return dev_bf16(q), dev_bf16(k), dev_bf16(v), torch.from_numpy(mask).cuda(), 128, 128, 1 / np.sqrt(D)


def _noalloc(q, k, v, mask, bx, by, scale):
    p = sa.bsa_params(q, k, mask, bx, by, sa.MASK_CAUSAL, scale)
    out = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=q.device)
    rc = sa.lib().bsa_fwd_noalloc(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                  ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                  ctypes.c_void_p(lse.data_ptr()),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == sa.BSA_OK
    bits = ctypes.c_uint32(0xFFFFFFFF)
    rc = sa.lib().bsa_fwd_noalloc_get_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                             ctypes.byref(bits))
    assert rc == sa.BSA_OK and bits.value == 0
    return out, lse


def _check_against_fwd(inp, label):
    q, k, v, mask, bx, by, scale = inp
    ref_out, ref_lse = sa.bsa_fwd(q, k, v, mask, bx, by, sa.MASK_CAUSAL, scale)
    torch.cuda.synchronize()
    out, lse = _noalloc(q, k, v, mask, bx, by, scale)
    assert torch.equal(out, ref_out), f"{label}: Out differs from bsa_fwd"
    assert torch.equal(lse, ref_lse), f"{label}: LSE differs from bsa_fwd"


@pytest.mark.parametrize("case", ["tiny", "ragged_gqa"])
def test_fwd_noalloc_matches_fwd(cuda_ok, case):
    inp = _inputs(case)
    for i in range(2):  # two calls in a row share the library's scratch array
        _check_against_fwd(inp, f"{case} call {i}")


def test_fwd_noalloc_larger_then_smaller(cuda_ok):
    """A larger problem leaves longer lists in the array; the smaller one after it must not see them."""
    big, small = _inputs("larger"), _inputs("ragged_gqa")
    _check_against_fwd(big, "larger problem")
    _check_against_fwd(small, "smaller problem after a larger one")
    _check_against_fwd(big, "larger problem again")


def test_fwd_noalloc_rejects_problems_over_its_scratch(cuda_ok):
    """The long-context workload (32 heads x 1024 blocks) needs ~128 MiB of lists: rejected
    before any launch, with the workspace error code."""
    p = sa.Params()
    p.q_layout = p.kv_layout = sa.LAYOUT_BNSD
    p.B, p.N1, p.N2, p.S_q, p.S_kv, p.D, p.Dv = 1, 32, 32, 131072, 131072, 128, 128
    p.block_x = p.block_y = 128
    p.mask_mode, p.scale = sa.MASK_CAUSAL, 0.088
    rc = sa.lib().bsa_fwd_noalloc(ctypes.byref(p), None, None, None, None, None, None)
    assert rc == sa.BSA_ERR_WORKSPACE_TOO_SMALL
