"""Pins for the oracle's GEMM part, correction and sign packer (CPU only).

The dequantisation used as the independent side here decodes codes and scales
with ml_dtypes, not with the oracle's tables; the correction is checked by
pure-Python loops on tiny shapes, by closed forms (R = 0, U = V = 1, one-hot x)
and by invariants that a dropped term, a wrong sign or a transposed operand
would break.
"""

import os

import ml_dtypes
import numpy as np
import pytest

import workloads
from oracle import biloco, nvfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lib_dequant(codes_packed, scales):
    c = np.empty(codes_packed.shape[:-1] + (codes_packed.shape[-1] * 2,), np.uint8)
    c[..., 0::2] = codes_packed & 0xF
    c[..., 1::2] = codes_packed >> 4
    vals = c.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = scales.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return vals * np.repeat(sc, 16, axis=-1)


def _tiny(M=2, N=8, K=64, r=5, seed=11, outliers=False):
    w = workloads.Workload("t", M, N, K, r, seed, outliers=outliers, alpha_decay=0.9)
    return workloads.make_inputs(w)


def test_gemm_part_vs_library_dequant_matmul():
    d = _tiny(M=3, N=16, K=128)
    ref = biloco.biloco_reference(d["x"], d["R"], d["U"], d["V"], d["alpha"])
    Xd = _lib_dequant(ref["xq"], ref["xs"])
    Wd = _lib_dequant(ref["wq"], ref["ws"])
    want = float(ref["g"]) * (Xd @ Wd.T)
    np.testing.assert_allclose(ref["gemm"], want, rtol=1e-12, atol=1e-12)


def test_gemm_part_bruteforce_loops():
    d = _tiny(M=2, N=3, K=32)
    ref = biloco.biloco_reference(d["x"], d["R"], d["U"], d["V"], d["alpha"])
    Xd = _lib_dequant(ref["xq"], ref["xs"])
    Wd = _lib_dequant(ref["wq"], ref["ws"])
    for m in range(2):
        for n in range(3):
            acc = 0.0
            for k in range(32):
                acc += Xd[m, k] * Wd[n, k]
            assert abs(ref["gemm"][m, n] - float(ref["g"]) * acc) < 1e-12


def test_gemm_one_hot_closed_form():
    # x = 6 at column k0, 0 elsewhere: its block has amax 6 -> scale 1 -> code 7
    # (value 6) exactly, other blocks are all-zero.  Then y[n] = g * 6 * deq(R)[n, k0].
    rng = np.random.default_rng(3)
    R = (rng.standard_normal((4, 64)) * 0.02).astype(np.float32)
    for k0 in (0, 17, 63):
        x = np.zeros((1, 64), np.float32)
        x[0, k0] = 6.0
        ref = biloco.biloco_reference(x, R, np.ones((4, 0)), np.ones((64, 0)), np.zeros(0, np.float32))
        Wd = _lib_dequant(ref["wq"], ref["ws"])
        np.testing.assert_allclose(ref["y"][0], float(ref["g"]) * 6.0 * Wd[:, k0], rtol=1e-14)


def test_correction_bruteforce_loops():
    d = _tiny(M=2, N=6, K=64, r=7)
    corr = biloco.correction_part(d["x"], d["U"], d["V"], d["alpha"])
    x, U, V, a = d["x"], d["U"], d["V"], d["alpha"]
    for m in range(2):
        for n in range(6):
            acc = 0.0
            for i in range(7):
                xv = 0.0
                for k in range(64):
                    xv += float(V[k, i]) * float(x[m, k])
                acc += float(a[i]) * xv * float(U[n, i])
            assert abs(corr[m, n] - acc) <= 1e-9 * max(1.0, abs(acc))


def test_r0_and_R0_split_the_two_parts():
    d = _tiny(M=2, N=8, K=64, r=6)
    full = biloco.biloco_reference(d["x"], d["R"], d["U"], d["V"], d["alpha"])
    r0 = biloco.biloco_reference(d["x"], d["R"], d["U"][:, :0], d["V"][:, :0], d["alpha"][:0])
    R0 = biloco.biloco_reference(d["x"], np.zeros_like(d["R"]), d["U"], d["V"], d["alpha"])
    assert not r0["corr"].any() and not R0["gemm"].any() and R0["g"] == 1.0
    np.testing.assert_allclose(full["y"], r0["y"] + R0["y"], rtol=1e-13, atol=1e-13)


def test_all_ones_signs_closed_form():
    # U = V = 1: correction = (sum_i alpha_i) * (sum_k x[m, k]) for every n.
    d = _tiny(M=3, N=5, K=64, r=9)
    U = np.ones((5, 9), np.int8)
    V = np.ones((64, 9), np.int8)
    corr = biloco.correction_part(d["x"], U, V, d["alpha"])
    want = float(np.sum(d["alpha"].astype(np.float64))) * d["x"].astype(np.float64).sum(axis=1)
    np.testing.assert_allclose(corr, np.repeat(want[:, None], 5, axis=1), rtol=1e-12)


def test_correction_invariants():
    d = _tiny(M=2, N=6, K=64, r=5)
    x, U, V, a = d["x"], d["U"], d["V"], d["alpha"]
    base = biloco.correction_part(x, U, V, a)
    # linear in x
    np.testing.assert_allclose(biloco.correction_part(2 * x, U, V, a), 2 * base, rtol=1e-12)
    # flipping weight row n of U negates output column n only
    U2 = U.copy(); U2[3] *= -1
    c2 = biloco.correction_part(x, U2, V, a)
    np.testing.assert_allclose(c2[:, 3], -base[:, 3], rtol=1e-12)
    np.testing.assert_allclose(np.delete(c2, 3, 1), np.delete(base, 3, 1), rtol=1e-12)
    # alpha_i = 0 removes rank i; U and V enter through the same rank index
    a2 = a.copy(); a2[2] = 0
    term2 = np.outer(a[2] * (x.astype(np.float64) @ V[:, 2].astype(np.float64)), U[:, 2].astype(np.float64))
    np.testing.assert_allclose(biloco.correction_part(x, U, V, a2), base - term2, rtol=1e-10, atol=1e-10)


def test_pack_signs_golden():
    with open(os.path.join(GOLDEN, "signs.txt")) as f:
        kv = {}
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.split()
    cols = int(kv["cols"][0])
    S = np.ones((2, cols), np.int8)
    S[0, [int(c) for c in kv["neg_row0"]]] = -1
    S[1, [int(c) for c in kv["neg_row1"]]] = -1
    bits = biloco.pack_signs(S)
    assert bits[0].tolist() == [int(w, 16) for w in kv["words_row0"]]
    assert bits[1].tolist() == [int(w, 16) for w in kv["words_row1"]]


def test_pack_signs_roundtrip_and_independent_unpack():
    rng = np.random.default_rng(0)
    for rows, cols in ((32, 256), (7, 40), (1, 1), (3, 1024)):
        S = (2 * rng.integers(0, 2, (rows, cols)) - 1).astype(np.int8)
        bits = biloco.pack_signs(S)
        np.testing.assert_array_equal(biloco.unpack_signs(bits, cols), S)
        # independent unpack: little-endian bytes, numpy's bit order 'little'
        raw = np.unpackbits(bits.astype("<u4").view(np.uint8), axis=1, bitorder="little")[:, :cols]
        np.testing.assert_array_equal(np.where(raw == 1, -1, 1), S)
        if cols % 32:
            assert not (bits[:, -1] >> np.uint32(cols % 32)).any()      # tail bits zero


def test_sign_storage_is_n_plus_k_times_r_over_8_bytes():
    # A binary rank-one term costs one bit per entry of u and v (BiLoCo README intro:
    # 16x less than BF16), so the factors of a rank-r correction take (N+K) r / 8 bytes.
    N, K, r = 256, 512, 64
    rng = np.random.default_rng(1)
    U = (2 * rng.integers(0, 2, (N, r)) - 1)
    V = (2 * rng.integers(0, 2, (K, r)) - 1)
    nbytes = biloco.pack_signs(U).nbytes + biloco.pack_signs(V.T).nbytes
    assert nbytes == (N + K) * r // 8
    assert nbytes * 16 == (N + K) * r * 2     # BF16 factors would take 16x more


def test_tiny_config_end_to_end_bruteforce():
    w = workloads.CONFIGS["tiny"]
    d = workloads.make_inputs(w)
    ref = biloco.biloco_reference(d["x"], d["R"], d["U"], d["V"], d["alpha"])
    Xd = _lib_dequant(ref["xq"], ref["xs"])
    Wd = _lib_dequant(ref["wq"], ref["ws"])
    Ud = biloco.unpack_signs(ref["Ubits"], w.r).astype(np.float64)
    Vd = biloco.unpack_signs(ref["Vbits"], w.K).astype(np.float64).T
    np.testing.assert_array_equal(Ud, d["U"])
    np.testing.assert_array_equal(Vd, d["V"])
    z = (d["x"].astype(np.float64) @ Vd) * d["alpha"].astype(np.float64)
    want = float(ref["g"]) * (Xd @ Wd.T) + z @ Ud.T
    np.testing.assert_allclose(ref["y"], want, rtol=1e-12, atol=1e-12)


def test_workload_inputs_have_the_stated_distributions():
    w = workloads.Workload("d", 4, 512, 5120, 32, 1)
    d = workloads.make_inputs(w)
    assert d["x_bf16"].dtype == np.uint16
    np.testing.assert_array_equal(workloads.bf16_bits_to_f32(d["x_bf16"]), d["x"])
    big = np.abs(d["x"]).max(axis=0) > 8
    assert 30 <= big.sum() <= 51          # ~1% of 5120 channels x20
    assert abs(float(d["R"].std()) - 0.02) < 1e-3
    assert set(np.unique(d["U"]).tolist()) == {-1, 1}
    assert d["alpha"][0] == np.float32(0.05)
