"""biloco_decompose against the FP64 oracle (through the C-ABI), and its output
fed to biloco_pack_weight and biloco_gemm end to end.

Both sides take every sign decision on an FP64 sum of the same residual (sign(0)
= +1), so the sign factors must agree bit for bit: the smallest |sum| among the
decisions here is many orders of magnitude above FP64 rounding.  The
coefficients and the residual agree to FP64 rounding (different summation
orders, a different linear solver)."""

import numpy as np
import pytest
import torch

import workloads
from oracle import biloco as ob
from oracle import decompose as od
from gpu_common import assert_y_close, to_dev_bf16, y_to_numpy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nb():
    import nvfp4_binary_rank_b200 as nb
    nb.load()
    return nb


def _run(nb, d, r, T):
    W = torch.from_numpy(d["W"]).cuda()
    v0 = torch.from_numpy(ob.pack_signs(d["v0"]).view(np.int32)).cuda() if r else None
    Ub, Vb, alpha, R = nb.decompose(W, r, T, v0)
    assert nb.last_error() == 0
    return (Ub.cpu().numpy().view(np.uint32), Vb.cpu().numpy().view(np.uint32), alpha.cpu().numpy(),
            R.cpu().numpy())


@pytest.mark.parametrize("N,K,r,T,planted", [(1024, 768, 32, 5, 8), (300, 200, 20, 3, 4), (128, 96, 1, 1, 1),
                                             (256, 512, 64, 2, 0)])
def test_decompose_matches_oracle(nb, N, K, r, T, planted):
    d = workloads.decompose_inputs(N, K, r, seed=N + K + r, planted=planted)
    Ub, Vb, alpha, R = _run(nb, d, r, T)
    ref = od.decompose(d["W"], r, T, d["v0"])
    np.testing.assert_array_equal(Ub, ob.pack_signs(ref["U"]))
    np.testing.assert_array_equal(Vb, ob.pack_signs(ref["V"].T))
    np.testing.assert_allclose(alpha, ref["alpha"], rtol=1e-6, atol=1e-9)
    wmax = float(np.abs(d["W"]).max())
    assert np.max(np.abs(R.astype(np.float64) - ref["R"])) <= 1e-6 * wmax
    assert np.linalg.norm(R) < np.linalg.norm(d["W"])


def test_decompose_zero_rank_copies_w(nb):
    d = workloads.decompose_inputs(128, 64, 0, seed=3)
    _, _, _, R = _run(nb, d, 0, 1)
    np.testing.assert_array_equal(R, d["W"])


def test_decompose_feeds_the_gemm(nb):
    # decompose -> NVFP4-pack the residual -> fused GEMM, against the oracle's own
    # decomposition and reference y
    N, K, r, T, M = 1024, 1024, 64, 3, 4
    d = workloads.decompose_inputs(N, K, r, seed=11, planted=16)
    ref = od.decompose(d["W"], r, T, d["v0"])
    W = torch.from_numpy(d["W"]).cuda()
    v0 = torch.from_numpy(ob.pack_signs(d["v0"]).view(np.int32)).cuda()
    Ub, Vb, alpha, R = nb.decompose(W, r, T, v0)
    Wq, Wsf, g = nb.pack_weight(R)
    wx = workloads.Workload("dec_x", M, N, K, 0, 12)
    x = workloads.make_inputs(wx, with_R=False)
    y = nb.gemm(to_dev_bf16(x["x_bf16"]), Wq, Wsf, g, Ub.contiguous(), Vb.contiguous(), alpha)
    assert nb.last_error() == 0
    want = ob.biloco_reference(x["x"], ref["R"].astype(np.float32), ref["U"], ref["V"],
                               ref["alpha"].astype(np.float32))
    assert_y_close(y_to_numpy(y), want["y"], "decompose -> gemm")
