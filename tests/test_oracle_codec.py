"""Pins for the oracle's NVFP4 codec (CPU only).

Each check ties the oracle to something other than itself: a library codec
(ml_dtypes' float4_e2m1fn / float8_e4m3fn, round-to-nearest-even), a closed
form, or a hand-derived fixture under tests/golden/.
"""

import os

import ml_dtypes
import numpy as np
import pytest

from oracle import nvfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            out[key.strip()] = val.split()
    return out


# --- E2M1 -------------------------------------------------------------------

def test_e2m1_grid_is_the_published_one():
    # The grid {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6} of the NVFP4 element format.
    assert list(nvfp4.E2M1_TABLE[:8]) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert list(nvfp4.E2M1_TABLE[8:]) == [-0.0, -0.5, -1, -1.5, -2, -3, -4, -6]


def test_e2m1_table_matches_library_decode():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(lib, nvfp4.E2M1_TABLE)


def _library_e2m1(q):
    c = np.asarray(q, dtype=np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    # the library keeps -0 as 0x8; the oracle stores every zero as 0x0
    return np.where((c & 7) == 0, 0, c).astype(np.uint8)


def test_e2m1_rounding_matches_library_at_midpoints_and_neighbours():
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5, 1, 1.5, 2, 3, 4], np.float32)
    pts = [mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(100))]
    q = np.concatenate(pts + [-p for p in pts])
    np.testing.assert_array_equal(nvfp4.e2m1_encode(q), _library_e2m1(q))


def test_e2m1_rounding_matches_library_random_and_saturation():
    rng = np.random.default_rng(123)
    q = np.concatenate([rng.uniform(-8, 8, 200000).astype(np.float32),
                        rng.uniform(-1e6, 1e6, 2000).astype(np.float32),
                        np.array([0.0, -0.0, 6.0, 7.9, 1e30, -1e30], np.float32)])
    np.testing.assert_array_equal(nvfp4.e2m1_encode(q), _library_e2m1(q))


def test_e2m1_saturates_and_never_emits_negative_zero():
    assert nvfp4.e2m1_encode(np.float32(1e9)) == 7
    assert nvfp4.e2m1_encode(np.float32(-1e9)) == 15
    assert nvfp4.e2m1_encode(np.float32(-0.2)) == 0
    assert nvfp4.e2m1_encode(np.float32(-0.0)) == 0


# --- E4M3 -------------------------------------------------------------------

def test_e4m3_decode_all_256_codes_against_library():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ours = nvfp4.E4M3_TABLE
    nan = np.isnan(lib)
    np.testing.assert_array_equal(nan, np.isnan(ours))
    np.testing.assert_array_equal(lib[~nan], ours[~nan])
    assert nvfp4.e4m3_value(0x7E) == 448.0 and nvfp4.e4m3_value(0x01) == 2.0 ** -9


def _library_e4m3(t):
    t = np.minimum(np.asarray(t, np.float32), np.float32(448.0))
    return t.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)


def test_e4m3_encode_matches_library_on_sweep():
    pos = nvfp4.E4M3_TABLE[:127]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)        # exact in fp32
    rng = np.random.default_rng(7)
    t = np.concatenate([pos.astype(np.float32), mids,
                        np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e4)),
                        rng.uniform(0, 500, 100000).astype(np.float32),
                        np.exp(rng.uniform(-25, 7, 100000)).astype(np.float32),
                        np.array([0, 1e-30, 448, 460, 464, 1e6], np.float32)])
    np.testing.assert_array_equal(nvfp4.e4m3_encode_nonneg(t), _library_e4m3(t))


def test_e4m3_clamps_to_448():
    assert nvfp4.e4m3_encode_nonneg(np.float32(1e5)) == 0x7E
    assert nvfp4.e4m3_encode_nonneg(np.float32(0.0)) == 0


# --- quantisers ----------------------------------------------------------------

def test_act_block_golden():
    g = _read_golden("act_block.txt")
    x = np.array([float(v) for v in g["x"]], np.float32).reshape(1, 16)
    q, s = nvfp4.quant_act(x)
    assert s.tolist() == [[int(g["scale"][0], 16)]]
    assert q.reshape(-1).tolist() == [int(c, 16) for c in g["codes"]]


def test_weight_blocks_golden():
    g = _read_golden("weight_blocks.txt")
    R = np.array([float(v) for v in g["R0"] + g["R1"]], np.float32).reshape(1, 32)
    q, s, gs = nvfp4.quant_weight(R)
    assert gs == np.float32(float(g["g"][0]))
    assert s.reshape(-1).tolist() == [int(c, 16) for c in g["scales"]]
    assert q.reshape(-1).tolist() == [int(c, 16) for c in g["codes"]]


def test_nibble_order_low_first():
    codes = np.array([[1, 2, 3, 4]], np.uint8)
    assert nvfp4.pack_nibbles(codes).tolist() == [[0x21, 0x43]]
    np.testing.assert_array_equal(nvfp4.unpack_nibbles(nvfp4.pack_nibbles(codes)), codes)


@pytest.mark.parametrize("v", [3.0, -3.0, 0.75, 96.0, -0.0234375])
def test_constant_block_closed_form(v):
    # All 16 values equal v: amax = |v|, s = E4M3(|v|/6).  When |v|/6 is exactly
    # representable the quotient |v|/s is 6, i.e. magnitude code 7.
    x = np.full((1, 16), v, np.float32)
    q, s = nvfp4.quant_act(x)
    assert nvfp4.e4m3_value(int(s[0, 0])) == abs(v) / 6
    want = 7 | (8 if v < 0 else 0)
    assert set(nvfp4.unpack_nibbles(q).reshape(-1).tolist()) == {want}


def test_zero_block_gives_zero_scale_and_codes():
    x = np.zeros((2, 32), np.float32)
    x[1, 16:] = 1.0
    q, s = nvfp4.quant_act(x)
    assert s[0].tolist() == [0, 0] and s[1, 0] == 0 and s[1, 1] != 0
    assert not q[0].any() and not q[1, :8].any()


def test_power_of_two_scaling_shifts_scale_not_codes():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    q0, s0 = nvfp4.quant_act(x)
    for k in (-3, 2, 5):
        q1, s1 = nvfp4.quant_act(x * np.float32(2.0 ** k))
        np.testing.assert_array_equal(q0, q1)
        np.testing.assert_array_equal(nvfp4.e4m3_decode(s1), nvfp4.e4m3_decode(s0) * 2.0 ** k)


def test_weight_zero_matrix_has_unit_tensor_scale():
    q, s, g = nvfp4.quant_weight(np.zeros((2, 32), np.float32))
    assert g == np.float32(1.0) and not q.any() and not s.any()


def test_weight_scale_reconstruction_error_bound():
    # Dequantised weight within half an E2M1 step of R: |R - deq| <= S (the
    # widest gap, between 4 and 6, is 2 S).  Catches a dropped tensor scale.
    rng = np.random.default_rng(9)
    R = (rng.standard_normal((8, 256)) * 0.02).astype(np.float32)
    q, s, g = nvfp4.quant_weight(R)
    deq = nvfp4.dequant(q, s) * float(g)
    S = np.repeat(nvfp4.e4m3_decode(s) * float(g), 16, axis=1)
    assert np.all(np.abs(R - deq) <= S * 1.0000001)
    assert np.linalg.norm(R - deq) / np.linalg.norm(R) < 0.15
