"""The failure path on the GPU, made on purpose without a fault: a bounded wait
that nothing completes gives up, the kernel records BILOCO_ERR_TIMEOUT in the
stream's status word, the host reads it, and the stream stays usable."""

import pytest
import torch

import workloads
from gpu_common import assert_y_close, device_problem, oracle_for, y_to_numpy

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_cleared():
    import nvfp4_binary_rank_b200 as nb
    nb.load()
    s = torch.cuda.Stream()
    assert nb.last_error(s) == 0
    nb.selftest_wait_timeout(s)
    assert nb.last_error(s) == nb._lib.ERR_TIMEOUT
    assert nb.last_error(s) == 0                          # read once, then cleared
    # the context and the stream still work
    w = workloads.CONFIGS["tiny"]
    d, ref = oracle_for(w)
    prob = device_problem(w, d)
    with torch.cuda.stream(s):
        y = nb.gemm(prob["x"], prob["W"], prob["sf"], prob["g"], prob["Ub"], prob["Vb"], prob["alpha"])
    s.synchronize()
    assert nb.last_error(s) == 0
    assert_y_close(y_to_numpy(y), ref["y"], "tiny after a timeout")
