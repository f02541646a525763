"""Parity of biloco_gemm against the FP64 oracle (through the C-ABI).

The GEMM part and the sign correction are pinned separately (r = 0, R = 0)
because at the workload sizes the correction is about 25x larger than the FP4
product and would hide an error in it."""

import numpy as np
import pytest
import torch

import workloads
from oracle import biloco as ob
from gpu_common import (assert_y_close, device_problem, oracle_for, y_errors, y_to_numpy)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nb():
    import nvfp4_binary_rank_b200 as nb
    nb.load()
    return nb


def _run(nb, prob, mode=None):
    if mode is not None:
        nb.set_mode(mode)
    try:
        y = nb.gemm(prob["x"], prob["W"], prob["sf"], prob["g"], prob["Ub"], prob["Vb"], prob["alpha"])
        st = nb.last_error()
        assert st == 0, nb.status_string(st)
    finally:
        nb.set_mode(nb.MODE_AUTO)
    return y_to_numpy(y)


def _small(M, N, K, r, seed, outliers=True):
    return workloads.Workload(f"s{M}_{N}_{K}_{r}", M, N, K, r, seed, outliers=outliers)


# --- the FP4 product alone (r = 0) -------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (1, 256, 256), (5, 384, 320), (16, 128, 1024),
                                   (32, 512, 768), (33, 256, 512), (64, 128, 256), (128, 256, 576)])
def test_fp4_gemm_part(nb, M, N, K):
    w = _small(M, N, K, 0, seed=M + N + K)
    d, ref = oracle_for(w)
    y = _run(nb, device_problem(w, d))
    assert_y_close(y, ref["gemm"], "r=0 y")
    # each element within BF16 rounding of the FP64 value (FP32 accumulation error is far below)
    tol = np.abs(ref["gemm"]) * 2.0 ** -8 + 1e-6 * np.abs(ref["gemm"]).max()
    assert np.all(np.abs(y - ref["gemm"]) <= tol)


# --- the correction alone (R = 0) ---------------------------------------------

@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("M,N,K,r", [(1, 128, 64, 16), (3, 256, 320, 17), (16, 128, 512, 64),
                                     (32, 256, 256, 33), (40, 128, 256, 16)])
def test_correction_part(nb, mode, M, N, K, r):
    w = _small(M, N, K, r, seed=100 + M + r)
    d = workloads.make_inputs(w)
    d["R"] = np.zeros_like(d["R"])
    ref = ob.biloco_reference(d["x"], d["R"], d["U"], d["V"], d["alpha"])
    y = _run(nb, device_problem(w, d), mode)
    assert_y_close(y, ref["corr"], "R=0 y")


def test_all_ones_signs_closed_form(nb):
    w = _small(4, 256, 512, 32, seed=7)
    d = workloads.make_inputs(w)
    d["R"] = np.zeros_like(d["R"])
    d["U"] = np.ones_like(d["U"])
    d["V"] = np.ones_like(d["V"])
    y = _run(nb, device_problem(w, d))
    want = float(d["alpha"].astype(np.float64).sum()) * d["x"].astype(np.float64).sum(axis=1)
    assert_y_close(y, np.repeat(want[:, None], w.N, axis=1), "U=V=1")


# --- full y on the workloads ---------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "decode", "mlp_up", "mlp_down"])
def test_workload_y(nb, name):
    w = workloads.CONFIGS[name]
    d, ref = oracle_for(w)
    y = _run(nb, device_problem(w, d))
    assert_y_close(y, ref["y"], name)


@pytest.mark.parametrize("M", workloads.SWEEP_MS)
@pytest.mark.parametrize("r", workloads.SWEEP_RS)
def test_sweep_y(nb, M, r):
    w = workloads.sweep_config(M, r)
    d, ref = oracle_for(w)
    y = _run(nb, device_problem(w, d))
    assert_y_close(y, ref["y"], w.name)


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("M,N,K,r", [(1, 128, 64, 1), (2, 640, 1344, 100), (17, 384, 832, 255),
                                     (31, 1280, 2560, 1024), (100, 256, 448, 48)])
def test_ragged_shapes_both_modes(nb, mode, M, N, K, r):
    w = _small(M, N, K, r, seed=M * 3 + r)
    d, ref = oracle_for(w)
    y = _run(nb, device_problem(w, d), mode)
    assert_y_close(y, ref["y"], w.name)


@pytest.mark.parametrize("M,N,K,r", [(9, 128, 256, 300), (12, 256, 640, 1024), (13, 384, 5120, 512),
                                     (16, 1280, 1024, 129)])
def test_decode_rank_pieces(nb, M, N, K, r):
    # decode batches of 9-16 rows split V^T x into pieces of 128 ranks x a K slice:
    # more rank blocks than CTAs, pieces of several MMA batches, a partial rank block
    w = _small(M, N, K, r, seed=M * 7 + r)
    d, ref = oracle_for(w)
    y = _run(nb, device_problem(w, d))
    assert_y_close(y, ref["y"], w.name)


def test_deterministic_and_reusable(nb):
    w = workloads.CONFIGS["decode"]
    d, ref = oracle_for(w)
    prob = device_problem(w, d)
    y1 = _run(nb, prob)
    y2 = _run(nb, prob)
    np.testing.assert_array_equal(y1, y2)


def test_shape_and_alignment_errors(nb):
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((128, 32), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((nb.weight_sf_bytes(128, 64),), dtype=torch.uint8, device="cuda")
    g = torch.ones((1,), device="cuda")
    with pytest.raises(nb.BilocoError) as e:
        nb.gemm(torch.zeros((129, 64), dtype=torch.bfloat16, device="cuda"),
                W, sf, g, None, None, None)
    assert e.value.status == -2
    buf = torch.zeros((2 * 64 + 8,), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nb.BilocoError) as e:
        nb.gemm(buf[1:65].view(1, 64), W, sf, g, None, None, None)
    assert e.value.status == -3


# --- full-size grids for the small decode classes and the general kernel ---------

@pytest.mark.parametrize("M", [2, 3, 4])
def test_decode_small_classes_full_grid(nb, M):
    # classes 2 and 4 on a full 148-CTA grid at N = K = 5120, r = 512: the late CTAs
    # that take no share of z, and (4 rows) the per-contributor tensor-core U side
    w = workloads.Workload(f"full_M{M}", M, 5120, 5120, 512, 40 + M)
    d, ref = oracle_for(w)
    y = _run(nb, device_problem(w, d))
    assert_y_close(y, ref["y"], w.name)


@pytest.mark.parametrize("M", [4, 12])
def test_general_kernel_full_size_sampled_rows(nb, M):
    # M <= 16 with more than 16 units per CTA runs the general kernel: quantising per
    # unit at 4 rows, after the activation pre-pass at 12.  The oracle checks a sample
    # of output rows: quantising a weight row depends only on that row and the tensor
    # scale g, so the sampled rows plus the row holding amax|R| give the same codes
    # and the same g as the whole matrix.
    w = workloads.Workload(f"big_M{M}", M, 13824, 13824, 512, 50 + M)
    d = workloads.make_inputs(w)
    y = _run(nb, device_problem(w, d))
    R = d["R"]
    n_max = int(np.unravel_index(np.argmax(np.abs(R)), R.shape)[0])
    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([rng.choice(w.N, 384, replace=False),
                                     [0, 1, 127, 128, 5119, 5120, w.N - 1, n_max]]))
    ref = ob.biloco_reference(d["x"], R[rows], d["U"][rows], d["V"], d["alpha"])
    from oracle import nvfp4 as on
    assert ref["g"] == on.weight_global_scale(R)
    assert_y_close(y[:, rows], ref["y"], w.name)


@pytest.mark.parametrize("flags", [2, 3])
@pytest.mark.parametrize("name", ["decode", "mlp_down"])
def test_cooperative_launch(nb, flags, name):
    # the opt-in launch form that guarantees co-residency of the grid gives the same y
    w = workloads.CONFIGS[name]
    d, ref = oracle_for(w)
    prob = device_problem(w, d)
    y_pdl = _run(nb, prob)
    nb.set_launch(flags)
    try:
        y = _run(nb, prob)
        y2 = _run(nb, prob)
    finally:
        nb.set_launch(nb.LAUNCH_PDL)
    assert_y_close(y, ref["y"], name)
    np.testing.assert_array_equal(y, y2)
    np.testing.assert_array_equal(y, y_pdl)


@pytest.mark.parametrize("M,N,K,r", [(48, 1280, 2048, 256), (128, 5120, 5120, 512)])
def test_cooperative_launch_large_classes(nb, M, N, K, r):
    # the cooperative form on the 64- and 128-row classes (the latter on its capped
    # grid of 2.5 CTAs per tile): same y as the default launch, within tolerance
    w = _small(M, N, K, r, seed=M * 17 + r)
    d, ref = oracle_for(w)
    prob = device_problem(w, d)
    y_pdl = _run(nb, prob)
    nb.set_launch(nb.LAUNCH_COOPERATIVE)
    try:
        y = _run(nb, prob)
    finally:
        nb.set_launch(nb.LAUNCH_PDL)
    assert_y_close(y, ref["y"], w.name)
    np.testing.assert_array_equal(y, y_pdl)


@pytest.mark.parametrize("M,N,K,r", [(5, 384, 832, 255), (7, 2560, 1344, 129), (8, 1280, 5184, 1000),
                                     (6, 13824, 5120, 512), (100, 640, 2624, 300)])
def test_tensor_v_side_from_8_rows_and_capped_grid(nb, M, N, K, r):
    # the 8-row class's V side in tensor-core pieces (ragged K, partial rank blocks,
    # more rank blocks than pieces per CTA), and a 128-row call on a ragged shape
    # whose grid is capped at 2.5 CTAs per tile (5 tiles -> 12 CTAs)
    w = _small(M, N, K, r, seed=M * 19 + r)
    d, ref = oracle_for(w)
    y = _run(nb, device_problem(w, d))
    assert_y_close(y, ref["y"], w.name)


# --- the 32-row class of the decode kernel (17 to 32 rows) ------------------------

@pytest.mark.parametrize("M,N,K,r", [(17, 384, 832, 255), (20, 640, 1344, 0), (24, 1280, 4096, 1024),
                                     (29, 2560, 5184, 600), (32, 128, 64, 3), (32, 5120, 13824, 1024),
                                     (18, 13824, 5120, 512)])
def test_batch32_class(nb, M, N, K, r):
    # activation chunks streamed with the weight stages from the grid's image; ranks
    # above 512 cycle the z tiles through the slot ring (r = 1024: two groups)
    w = _small(M, N, K, r, seed=M * 5 + r)
    d, ref = oracle_for(w)
    y = _run(nb, device_problem(w, d))
    assert_y_close(y, ref["y"], w.name)
    if r == 0:
        tol = np.abs(ref["gemm"]) * 2.0 ** -8 + 1e-6 * np.abs(ref["gemm"]).max()
        assert np.all(np.abs(y - ref["gemm"]) <= tol)


# --- the 64- and 128-row classes of the decode kernel (33 to 128 rows) ------------

@pytest.mark.parametrize("M,N,K,r", [(33, 384, 832, 255), (48, 640, 1344, 0), (64, 1280, 4096, 1024),
                                     (64, 5120, 13824, 512), (65, 2560, 5184, 600), (96, 128, 64, 3),
                                     (100, 13824, 5120, 512), (128, 1280, 2560, 1024), (128, 5120, 5120, 0)])
def test_batch64_128_classes(nb, M, N, K, r):
    # MMA N = 64 or 128 from the streamed image; the two BF16 parts of z summed in
    # one TMEM product (the 128-row class with a single product buffer); z tiles
    # cycled through 3 (64 rows) or 2 (128 rows) slots; the epilogue 16 columns at a
    # time
    w = _small(M, N, K, r, seed=M * 13 + r)
    d, ref = oracle_for(w)
    y = _run(nb, device_problem(w, d))
    assert_y_close(y, ref["y"], w.name)
    if r == 0:
        tol = np.abs(ref["gemm"]) * 2.0 ** -8 + 1e-6 * np.abs(ref["gemm"]).max()
        assert np.all(np.abs(y - ref["gemm"]) <= tol)


# --- the correction arithmetic of the 1-2-row U side: sign-adds and table lookups ---

@pytest.mark.parametrize("arith", [1, 2])
@pytest.mark.parametrize("M,N,K,r", [(1, 5120, 5120, 512), (2, 640, 1344, 100), (1, 128, 64, 1),
                                     (2, 1280, 2560, 1024), (1, 13824, 5120, 33)])
def test_correction_arithmetic(nb, arith, M, N, K, r):
    w = _small(M, N, K, r, seed=M * 11 + r)
    d, ref = oracle_for(w)
    prob = device_problem(w, d)
    nb.set_correction(arith)
    try:
        assert nb.resolve_correction(M, N, K, r) == arith
        y = _run(nb, prob)
        y2 = _run(nb, prob)
    finally:
        nb.set_correction(nb.CORR_AUTO)
    assert_y_close(y, ref["y"], f"{w.name} arith {arith}")
    np.testing.assert_array_equal(y, y2)
