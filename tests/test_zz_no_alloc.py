"""bsa_fwd_noalloc: the forward for callers that cannot allocate device memory (a host that owns
all device memory and gives plugins no scratch, or a path where cudaMalloc is not acceptable).
It keeps its scratch in a fixed 8 MiB device array inside the library instead of a caller
workspace.  Checked through the C ABI against bsa_fwd on two calls in a row (the second call
reuses the array the first one left behind), and for its size limit.

This file is collected last on purpose, so a failure here comes after every other test ran."""
import ctypes

import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from parity import LSE_ATOL, check_close, dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def _inputs(case):
    if case == "tiny":
        w = synth.workload(1)
        mask = w.block_mask()
        return (dev_bf16(w.tensor("q")), dev_bf16(w.tensor("k")), dev_bf16(w.tensor("v")),
                torch.from_numpy(mask).cuda(), 64, 64, w.scale)
    rng = np.random.default_rng(5)
    B, N1, N2, S, D = 2, 4, 2, 300, 128
    q = synth.f32_to_bf16_bits(rng.standard_normal((B, N1, S, D), dtype=np.float32))
    k = synth.f32_to_bf16_bits(rng.standard_normal((B, N2, S, D), dtype=np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal((B, N2, S, D), dtype=np.float32))
    mask = (rng.random((B, N1, 3, 3)) < 0.6).astype(np.uint8)
    return dev_bf16(q), dev_bf16(k), dev_bf16(v), torch.from_numpy(mask).cuda(), 128, 128, 1 / np.sqrt(D)


@pytest.mark.parametrize("case", ["tiny", "ragged_gqa"])
def test_fwd_noalloc_matches_fwd(cuda_ok, case):
    q, k, v, mask, bx, by, scale = _inputs(case)
    ref_out, ref_lse = sa.bsa_fwd(q, k, v, mask, bx, by, sa.MASK_CAUSAL, scale)
    torch.cuda.synchronize()
    ref_out = ref_out.float().cpu().numpy()
    ref_lse = ref_lse.cpu().numpy()
    fin = np.isfinite(ref_lse)
    p = sa.bsa_params(q, k, mask, bx, by, sa.MASK_CAUSAL, scale)
    for _ in range(2):  # two calls in a row share the library's scratch array
        out = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device=q.device)
        rc = sa.lib().bsa_fwd_noalloc(ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                      ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                      ctypes.c_void_p(lse.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == sa.BSA_OK
        torch.cuda.synchronize()
        got_lse = lse.cpu().numpy()
        check_close(out.float().cpu().numpy(), ref_out, f"noalloc out ({case})")
        assert np.all(np.isneginf(got_lse[~fin]))
        assert np.abs(got_lse[fin] - ref_lse[fin]).max() <= LSE_ATOL


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
