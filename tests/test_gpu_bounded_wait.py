"""The bounded mbarrier wait of the TMA / tensor-core kernels, made to run
out on the GPU without a fault: a wait on a barrier that nothing arrives at
ends after its limit with QSA_DEV_TIMEOUT in the caller's status word, a
second waiter is released by the CTA's abort flag, a bulk copy in flight is
drained, the host reads QSA_ERR_TIMEOUT, and the context keeps working."""
import numpy as np
import pytest
import torch

from indexer_top_sparse_c4_b200 import workloads as wl
from parity_utils import SCORE_REL, host, values_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from indexer_top_sparse_c4_b200 import build, qsa
    build.build()
    return qsa


@pytest.mark.parametrize("limit_us", [2000, 20000])
def test_wait_runs_out_and_reports(q, oracle, limit_us):
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    report = torch.full((6,), -1, dtype=torch.int32, device="cuda")
    q.qsa_selftest_bounded_wait(limit_us, status, report)
    r = report.cpu().numpy().astype(np.int64)
    assert r[0] == 0, "warp 0's wait on a barrier nothing arrives at must run out"
    assert r[1] == 0, "warp 1 must be released without its barrier completing"
    assert limit_us <= r[2] <= limit_us + 50_000, r[2]
    # warp 1's own limit is 1 s past warp 0's: released well before, by the abort flag
    assert r[3] <= limit_us + 200_000, r[3]
    assert r[4] == 1 and r[5] == 1, "the bulk copy in flight is drained and landed intact"
    code, bits = q.qsa_get_device_status(status)
    assert code == q.QSA_ERR_TIMEOUT and bits & q.QSA_DEV_TIMEOUT
    code, bits = q.qsa_get_device_status(status, clear=True)
    assert code == q.QSA_ERR_TIMEOUT
    assert q.qsa_get_device_status(status) == (q.QSA_OK, 0)
    # the context is intact: a projection on the tensor cores and its status
    T, H, N = 256, 1024, 644
    x = wl.hidden_states(T, H, seed=3, device="cuda")
    w, _, _ = wl.indexer_weights(H, 4, 128, seed=4, device="cuda")
    y = torch.empty((T, N), dtype=torch.float32, device="cuda")
    q.qsa_indexer_project(x, w, y, dev_status=status)
    assert q.qsa_get_device_status(status) == (q.QSA_OK, 0)
    hx, hw = host(x), host(w)
    ref = oracle.indexer_project(hx, hw)
    bound = SCORE_REL * (np.abs(values_f64(hx)) @ np.abs(values_f64(hw)).T)
    assert np.all(np.abs(host(y).astype(np.float64) - ref) <= bound + 1e-30)
