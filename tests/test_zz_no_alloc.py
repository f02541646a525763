"""biloco_gemm_noalloc against biloco_gemm (through the C-ABI).

The no-allocation variant runs the same kernels with its scratch in a static
device array; two calls in a row must each agree with biloco_gemm within the
y tolerance, also after a different shape has left its data in that array, and
the calls must not change the device's free memory.  This file is collected
last so that it also runs after every other GPU test in one process."""

import numpy as np
import pytest
import torch

import workloads
from gpu_common import assert_y_close, device_problem, oracle_for, y_to_numpy

pytestmark = pytest.mark.gpu

MAX_N = 1 << 18
SCRATCH_BYTES = 16 << 20


@pytest.fixture(scope="module")
def nb():
    import nvfp4_binary_rank_b200 as nb
    nb.load()
    return nb


def _args(prob):
    return (prob["x"], prob["W"], prob["sf"], prob["g"], prob["Ub"], prob["Vb"], prob["alpha"])


def _check_pair(nb, prob, mode):
    nb.set_mode(mode)
    try:
        y_ref = nb.gemm(*_args(prob))
        assert nb.last_error() == 0
        y1 = nb.gemm_noalloc(*_args(prob))
        y2 = nb.gemm_noalloc(*_args(prob))
        st = nb.last_error()
        assert st == 0, nb.status_string(st)
    finally:
        nb.set_mode(nb.MODE_AUTO)
    ref = y_to_numpy(y_ref).astype(np.float64)
    assert_y_close(y_to_numpy(y1), ref, "first no-alloc call")
    assert_y_close(y_to_numpy(y2), ref, "second no-alloc call")
    return y_to_numpy(y2)


# Order matters: each shape reuses the static array after the one before it.
SHAPES = [
    ("decode", workloads.CONFIGS["decode"], 1),
    ("decode", workloads.CONFIGS["decode"], 2),
    ("ragged_m16", workloads.Workload("na_16_256_320_17", 16, 256, 320, 17, 11), 1),
    ("ragged_m16", workloads.Workload("na_16_256_320_17", 16, 256, 320, 17, 11), 2),
    ("m40", workloads.Workload("na_40_384_576_40", 40, 384, 576, 40, 12), 1),
    ("m24", workloads.Workload("na_24_640_1344_100", 24, 640, 1344, 100, 14), 1),
    ("m3_r0", workloads.Workload("na_3_256_512_0", 3, 256, 512, 0, 13), 1),
    ("mlp_up", workloads.CONFIGS["mlp_up"], 1),
    ("m64_full", workloads.sweep_config(64, 512), 1),
    ("m128_small", workloads.Workload("na_128_640_1280_64", 128, 640, 1280, 64, 15), 1),
]


@pytest.mark.parametrize("name,w,mode", SHAPES, ids=[f"{s[0]}-mode{s[2]}" for s in SHAPES])
def test_noalloc_matches_gemm(nb, name, w, mode):
    prob = device_problem(w)
    y = _check_pair(nb, prob, mode)
    if w.M * w.N * w.K <= 16 * 384 * 576:
        # the small cases also against the oracle
        _, ref = oracle_for(w)
        assert_y_close(y, ref["y"], f"{name} vs oracle")


def test_noalloc_allocates_nothing(nb):
    prob = device_problem(workloads.CONFIGS["decode"])
    nb.gemm_noalloc(*_args(prob))                      # set-up call (address look-up)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()                            # a stream biloco_gemm never saw
    out1 = torch.empty((1, 5120), dtype=torch.bfloat16, device="cuda")
    out2 = torch.empty_like(out1)
    with torch.cuda.stream(s):
        out1.zero_()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    with torch.cuda.stream(s):
        nb.gemm_noalloc(*_args(prob), out=out1)
        nb.gemm_noalloc(*_args(prob), out=out2)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert nb.last_error(s) == 0
    assert torch.equal(out1, out2)


def _dev_args(M, N, K):
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((nb_sf_bytes(N, K),), dtype=torch.uint8, device="cuda")
    g = torch.ones((1,), dtype=torch.float32, device="cuda")
    return x, W, sf, g


def nb_sf_bytes(N, K):
    return N * ((K + 255) // 256) * 16


def test_noalloc_refuses_what_does_not_fit(nb):
    # refused on the host, before anything is launched
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    M, N, K = 128, 5120, 5120
    assert 2 * min(n_sms, 40 * 20) * 128 * 512 > SCRATCH_BYTES
    x, W, sf, g = _dev_args(M, N, K)
    with pytest.raises(nb.BilocoError) as e:
        nb.gemm_noalloc(x, W, sf, g, None, None, None)
    assert e.value.status == -2
    x, W, sf, g = _dev_args(1, MAX_N + 128, 64)
    with pytest.raises(nb.BilocoError) as e:
        nb.gemm_noalloc(x, W, sf, g, None, None, None)
    assert e.value.status == -2
    torch.cuda.synchronize()
    assert nb.last_error() == 0
