"""GPU parity of the paged decode on group sizes and lists the other decode cases do not cover: a
group of 96 query heads (the second head half holds 32 heads and 32 padding rows), a group of 8,
and a sparse id listed twice (its pages gathered twice)."""
import numpy as np
import pytest

from parity import LSE_ATOL, check_close
from test_gpu_sfa import _problem, _run

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", [
    dict(B=2, N1=96, N2=1, page=64, n_logical=12, K=7, sbs=64, seqused=[700, 768]),      # second head half of 32
    dict(B=2, N1=16, N2=2, page=64, n_logical=10, K=6, sbs=64, seqused=[640, 500]),      # G = 8
    dict(B=2, N1=128, N2=1, page=64, n_logical=12, K=5, sbs=64, seqused=[700, 768], dup=True),  # an id twice
])
def test_sfa_decode_group_cases(cuda_ok, case):
    pb = _problem(**case, seed=21)
    out, lse, r_out, r_lse = _run(pb)
    check_close(out.float().cpu().numpy(), r_out, "out")
    fin = np.isfinite(r_lse)
    got = lse.cpu().numpy()
    assert np.all(np.isneginf(got[~fin]))
    assert np.abs(got[fin] - r_lse[fin]).max() <= LSE_ATOL
