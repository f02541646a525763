"""The failure path on the GPU, made on purpose without a fault: a bounded wait
that nothing completes gives up, the kernel records BILOCO_ERR_TIMEOUT in the
stream's status word, the host reads it, and the stream stays usable.

Two forms: a one-warp self-test kernel, and the GEMM itself with some of its
grid-wide arrivals left out (biloco_selftest_drop_arrivals), so that the fused
kernel's own abort protocol runs: the waiting CTAs give up, leave together,
drain their copies and MMAs, free their tensor memory and return; the host then
resets the counters and the next call on the stream is correct."""

import numpy as np
import pytest
import torch

import workloads
from gpu_common import assert_y_close, device_problem, oracle_for, y_to_numpy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nb():
    import nvfp4_binary_rank_b200 as nb
    nb.load()
    return nb


def test_expired_wait_is_reported_and_cleared(nb):
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


# (mask, M, N, K): 1 drops the z arrivals (1 row: the completing CTA's U side
# waits; 16 rows: the per-contributor tensor-core U side waits), 2 the
# activation-image arrivals (8 rows; from 17 rows the producers' wait on the
# streamed image), 3 both.  The 64- and 128-row cases run the column-chunked
# epilogue's abort path; at N = K = 5120 their CTAs hold two tiles, so the
# 128-row class's single U-side product buffer is waited on for a second segment.
@pytest.mark.timeout(120, method="thread")
@pytest.mark.parametrize("entry", ["gemm", "gemm_noalloc"])
@pytest.mark.parametrize("mask,M,N,K", [(1, 1, 1280, 2048), (1, 16, 1280, 2048), (2, 8, 1280, 2048),
                                        (3, 16, 1280, 2048), (2, 24, 1280, 2048), (1, 32, 1280, 2048),
                                        (1, 64, 1280, 2048), (3, 64, 5120, 5120), (2, 100, 1280, 2048),
                                        (1, 128, 5120, 5120)])
def test_dropped_arrivals_expire_inside_the_gemm(nb, entry, mask, M, N, K):
    if entry == "gemm_noalloc" and M > 64 and N * K > 1280 * 2048:
        pytest.skip("the 128-row class's scratch at this size exceeds the no-allocation array")
    w = workloads.Workload(f"drop_{M}", M, N, K, 256, 60 + M)
    d, ref = oracle_for(w)
    prob = device_problem(w, d)
    args = (prob["x"], prob["W"], prob["sf"], prob["g"], prob["Ub"], prob["Vb"], prob["alpha"])
    fn = getattr(nb, entry)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y0 = fn(*args)                                    # a correct call first
    assert nb.last_error(s) == 0
    nb.selftest_drop_arrivals(mask)
    with torch.cuda.stream(s):
        fn(*args)                                         # its waits expire after ~1 s
    assert nb.last_error(s) == nb._lib.ERR_TIMEOUT
    assert nb.last_error(s) == 0
    with torch.cuda.stream(s):
        y1 = fn(*args)
        y2 = fn(*args)
    assert nb.last_error(s) == 0
    assert_y_close(y_to_numpy(y1), ref["y"], "first call after the timeout")
    np.testing.assert_array_equal(y_to_numpy(y1), y_to_numpy(y0))
    np.testing.assert_array_equal(y_to_numpy(y2), y_to_numpy(y0))


def test_drop_request_is_consumed_by_one_call(nb):
    # a request made before a call that does not take the decode kernel (here the
    # local-z schedule, which runs the general kernel) is consumed by that call and
    # affects nothing
    w = workloads.Workload("drop_general", 40, 256, 512, 32, 77)
    d, ref = oracle_for(w)
    prob = device_problem(w, d)
    nb.set_mode(nb.MODE_LOCAL_Z)
    try:
        assert nb.gemm_kernel_count(w.M, w.N, w.K, w.r) == 2
        nb.selftest_drop_arrivals(1)
        y = nb.gemm(prob["x"], prob["W"], prob["sf"], prob["g"], prob["Ub"], prob["Vb"], prob["alpha"])
    finally:
        nb.set_mode(nb.MODE_AUTO)
    assert nb.last_error() == 0
    assert_y_close(y_to_numpy(y), ref["y"], w.name)
