"""Failure detection without a GPU fault: every kernel wait is bounded, and a wait that runs out
sets SA_DEV_TIMEOUT in the caller's status word and returns (no trap, no assert), so the context
stays usable.  The diagnostic waits on a barrier that nothing arrives on."""
import time

import numpy as np
import pytest
import torch

import selected_attention_b200 as sa
from oracle import attention as A
from parity import check_close, check_lse, dev_bf16
from workloads import synth

pytestmark = pytest.mark.gpu

SA_DEV_TIMEOUT = 4


def test_bounded_wait_times_out_and_context_survives(cuda_ok):
    assert sa.bsa_diag_wait(True) == 0  # satisfied barrier: no status bits
    t0 = time.perf_counter()
    bits = sa.bsa_diag_wait(False)      # nothing arrives: the wait gives up after its limit
    dt = time.perf_counter() - t0
    assert bits & SA_DEV_TIMEOUT, bits
    assert dt < 30.0, dt
    # the context still works: the tiny forward runs and matches the oracle
    w = synth.workload(1)
    mask = w.block_mask()
    q, k, v = (w.tensor(t) for t in ("q", "k", "v"))
    out, lse = sa.bsa_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), torch.from_numpy(mask).cuda(), w.block, w.block,
                          2, w.scale)
    torch.cuda.synchronize()
    r_out, r_lse = A.bsa_forward(q, k, v, mask, w.block, w.block, 2, w.scale)
    check_close(out.float().cpu().numpy(), r_out, "out after a timed-out wait")
    check_lse(lse.cpu().numpy(), np.asarray(r_lse))


def test_diag_wait_rejects_bad_arguments(cuda_ok):
    L = sa.lib()
    assert L.bsa_diag_wait(None, 0, None) == sa.BSA_ERR_NULLPTR
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert L.bsa_diag_wait(ws.data_ptr(), 2, None) == sa.BSA_ERR_INVALID_ARG
